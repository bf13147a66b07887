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
// address (in host code it is only a host-side stand-in), so the first call in
// each CUDA context -- in practice once per device, with that device current --
// asks the runtime for the real address with cudaGetSymbolAddress and caches
// it under the context's unique id.  A call from another context (the same
// device after cudaDeviceReset, or a driver context of the caller's own) looks
// the address up again instead of reusing one that may no longer be valid.
// That first call does a little set-up work and should be made before any
// stream capture begins.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  Nothing in it has to start at zero: every call writes each partial
// result slot before the combine step reads it.  Calls whose kernels overlap
// on the GPU (different streams, no ordering between them) race on the array;
// order them on one stream or with events.
#include <cstdint>
#include <mutex>
#include <unordered_map>

#include <cuda.h>
#include <cuda_runtime.h>

#include "bsattn.h"

#define BSATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

static __device__ __align__(256) unsigned char g_noalloc_scratch[BSATTN_NOALLOC_SCRATCH_BYTES];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

std::mutex g_noalloc_mutex;
// context id -> device address of the scratch array in that context
std::unordered_map<unsigned long long, void*> g_noalloc_ptr;

// The unique id of the calling thread's current CUDA context (false when no
// context is current yet or the driver does not provide ids).  The driver
// functions come through the runtime's entry-point query, so the library
// needs no link-time libcuda.
bool current_context_id(unsigned long long* id) {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context, looked up with
// cudaGetSymbolAddress (with the device current) the first time a context
// asks.  Returns BSATTN_OK or BSATTN_ERR_CUDA.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSATTN_ERR_CUDA;
  unsigned long long id = 0;
  bool known = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (known) {
    auto it = g_noalloc_ptr.find(id);
    if (it != g_noalloc_ptr.end()) {
      *out = it->second;
      return BSATTN_OK;
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return BSATTN_ERR_CUDA;
  // the lookup makes the device's primary context current if none was
  if (!known) known = current_context_id(&id);
  if (known) g_noalloc_ptr[id] = p;
  *out = p;
  return BSATTN_OK;
}

}  // namespace

extern "C" {

int bsattn_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int L, int d, int block, float scale,
                              int causal, float lambda, int num_splits, uint8_t* tile_status,
                              int32_t* d_status, cudaStream_t stream) {
  // the argument errors bsattn_fwd_decode would report come first, then the
  // scratch capacity
  if (!q || !k || !v || !o) return BSATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || Hq % Hkv != 0 || num_splits < 1)
    return BSATTN_ERR_INVALID_ARG;
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
