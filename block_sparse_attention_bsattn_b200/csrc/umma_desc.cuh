// Stepping a shared-memory matrix descriptor (the layout smem_desc builds in
// sm100_ptx.cuh) from one tile to the next, in two forms.
#pragma once
#include <cstdint>

namespace bsattn {

// The descriptor of the tile `byte_off` bytes (a multiple of 16) further on:
// only the start-address field changes, and shared-memory addresses stay
// below 256 KB, so the 14-bit field cannot carry into the next one.  The
// one-tile prefill steps one 64-bit descriptor per operand by compile-time
// offsets (about 1 % faster there than building both descriptors for every
// MMA; the 32-bit form below measured equal on its static masks and 0.6 %
// slower with an all-ones mask).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t byte_off) {
  return desc + (uint64_t)(byte_off >> 4);
}

// The 32-bit form.  A descriptor's high word holds only constants (stride
// offset, version, swizzle); the low word holds the start address and the
// leading offset, so the descriptor of a tile `off` bytes further on is the
// low word plus off / 16.  The backward's issue loops build one low word per
// operand and add the stage and K-step offsets with one 32-bit add per
// operand and MMA (4.9 % faster there than the 64-bit form; the issuing
// thread advances at about the tensor pipe's pace, so every instruction
// between its MMAs shows).  The two-tile prefill builds its descriptors the
// same way with helpers of its own.
__host__ __device__ constexpr uint32_t udesc_hi(uint32_t sbo_bytes, uint32_t swizzle) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | ((swizzle & 0x7u) << 29);
}
__device__ __forceinline__ uint32_t udesc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
// the low word of the tile `byte_off` bytes (a multiple of 16) further on
__device__ __forceinline__ uint32_t udesc_step(uint32_t lo, uint32_t byte_off) {
  return lo + (byte_off >> 4);
}
// the full descriptor of that tile; every operand tile here has its 8-row
// groups 1024 bytes apart and the 128-byte swizzle
__device__ __forceinline__ uint64_t udesc128(uint32_t lo, uint32_t byte_off) {
  constexpr uint32_t hi = udesc_hi(1024, 2);
  return ((uint64_t)hi << 32) | udesc_step(lo, byte_off);
}

}  // namespace bsattn
