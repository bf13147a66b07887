// Stepping a shared-memory matrix descriptor (the layout smem_desc builds in
// sm100_ptx.cuh) from one tile to the next.
#pragma once
#include <cstdint>

namespace bsattn {

// The descriptor of the tile `byte_off` bytes (a multiple of 16) further on:
// only the start-address field changes, and shared-memory addresses stay
// below 256 KB, so the 14-bit field cannot carry into the next one.  The
// one-tile prefill and the backward issue loops build one descriptor per
// operand and step it with compile-time offsets (about 1 % faster there than
// building both descriptors for every MMA; the two-tile prefill kernel
// measured 3 % slower with it and keeps the per-MMA form).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t byte_off) {
  return desc + (uint64_t)(byte_off >> 4);
}

}  // namespace bsattn
