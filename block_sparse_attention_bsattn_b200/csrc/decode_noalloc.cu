// bsattn_fwd_decode_noalloc: the split-KV decode of bsattn_fwd_decode for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host framework which owns every byte
// of device memory and does not let extensions call cudaMalloc (for example
// an inference engine that plans one memory arena up front and hands plugins
// only their input and output tensors), and latency-critical paths where an
// allocation -- its cost and its chance to fail -- is not acceptable once the
// service is running.  Such callers cannot provide the decode workspace, so
// this entry point uses a fixed scratch array that lives in the library
// instead.
//
// The scratch is a file-scope __device__ array of BSATTN_NOALLOC_SCRATCH_BYTES
// (32 MiB).  Every GPU on which the library's code is loaded holds one copy
// until the process exits.  Host code cannot use the array's name as a device
// address (in host code it is only a host-side stand-in), so the first call on
// each device, with that device current, asks the runtime for the real address
// with cudaGetSymbolAddress and caches it; that first call therefore does a
// little set-up work and should be made before any stream capture begins.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  Nothing in it has to start at zero: every call writes each partial
// result slot before the combine step reads it.  Calls whose kernels overlap
// on the GPU (different streams, no ordering between them) race on the array;
// order them on one stream or with events.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "bsattn.h"

#define BSATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
#define BSATTN_NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char g_noalloc_scratch[BSATTN_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[BSATTN_NOALLOC_MAX_DEVICES] = {};

// Device address of this device's copy of the scratch array (set up once per
// device, with that device current).  Returns BSATTN_OK or BSATTN_ERR_CUDA.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSATTN_ERR_CUDA;
  if (dev < 0 || dev >= BSATTN_NOALLOC_MAX_DEVICES) return BSATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return BSATTN_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BSATTN_OK;
}

}  // namespace

extern "C" {

int bsattn_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int L, int d, int block, float scale,
                              int causal, float lambda, int num_splits, uint8_t* tile_status,
                              int32_t* d_status, cudaStream_t stream) {
  const size_t need = bsattn_decode_workspace_size(B, Hq, d, num_splits);
  if (need == 0) return BSATTN_ERR_INVALID_ARG;
  // the split outputs of this problem do not fit in the library's scratch
  if (need > BSATTN_NOALLOC_SCRATCH_BYTES) return BSATTN_ERR_CAPACITY;
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  return bsattn_fwd_decode(q, k, v, o, lse, B, Hq, Hkv, L, d, block, scale, causal, lambda,
                           num_splits, scratch, BSATTN_NOALLOC_SCRATCH_BYTES, tile_status,
                           d_status, stream);
}

}  // extern "C"
