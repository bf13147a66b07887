// bsattn_fwd_prefill_host: block-sparse prefill for inputs that live in host
// memory, with the host-to-device copies, the kernels and the device-to-host
// copy of O overlapped.
//
// A serving process that keeps Q, K and V on the host pays the PCIe transfers
// on every call; done one after another they take longer than the attention
// itself (about 670 MB per call for the 32-head, 32K-token workload, some
// 12 ms at PCIe rates against 6 ms of kernel time).  The batch is cut into
// chunks of (sequence, kv_heads_per_chunk KV heads) with their query heads --
// independent problems, since every query head reads only its own KV head --
// and for each chunk
//   copy stream   Q, K and V of the chunk, host -> device
//   caller stream the prefill of the chunk (after its copies)
//   out stream    O of the chunk, device -> host (after its prefill)
// so chunk c's kernel runs while chunk c + 1 is copied in and chunk c - 1 is
// copied out.  Both internal streams and a ring of events are created once
// per device and reused.  One cudaMemcpyAsync per tensor slice; host buffers
// must be page-locked for the copies to overlap.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "bsattn.h"

namespace {

constexpr int kEvents = 64;   // per kind; chunks reuse them round robin

struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t copied[kEvents], computed[kEvents];
};

constexpr int kMaxDevices = 64;
HostPipe g_pipes[kMaxDevices];
std::mutex g_pipe_mutex;

// The current device's streams and events, created on first use.
HostPipe* pipe_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe& p = g_pipes[dev];
  if (p.ready) return &p;
  bool ok = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; ok && i < kEvents; ++i)
    ok = cudaEventCreateWithFlags(&p.copied[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.computed[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) return nullptr;   // partially created objects stay until process exit
  p.ready = true;
  return &p;
}

}  // namespace

extern "C" {

int bsattn_fwd_prefill_host(const void* h_q, const void* h_k, const void* h_v, void* h_o,
                            void* d_q, void* d_k, void* d_v, void* d_o, int B, int Hq, int Hkv,
                            int N, int d, int block, float scale, int causal, float lambda,
                            const int32_t* row_ptr, const int32_t* col_idx,
                            const int32_t* row_order, int mask_heads, int kv_heads_per_chunk,
                            int32_t* d_status, cudaStream_t stream) {
  // every check a chunk's bsattn_fwd_prefill would make, before any copy is
  // enqueued, so that a rejected call leaves nothing running
  if (!h_q || !h_k || !h_v || !h_o || !d_q || !d_k || !d_v || !d_o)
    return BSATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return BSATTN_ERR_INVALID_ARG;
  if (kv_heads_per_chunk < 1 || Hkv % kv_heads_per_chunk != 0) return BSATTN_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda <= 1.f) || !std::isfinite(scale) || !(scale > 0.f))
    return BSATTN_ERR_INVALID_ARG;
  if (row_order && !row_ptr) return BSATTN_ERR_INVALID_ARG;
  if (row_ptr && (!col_idx || (mask_heads != 1 && mask_heads != Hq)))
    return BSATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSATTN_ERR_UNSUPPORTED;
  if (block != 64 && block != 128) return BSATTN_ERR_UNSUPPORTED;
  // chunk offsets are multiples of N * d * 2 bytes, so aligned bases suffice
  for (const void* ptr : {static_cast<const void*>(d_q), static_cast<const void*>(d_k),
                          static_cast<const void*>(d_v), static_cast<const void*>(d_o)})
    if (reinterpret_cast<uintptr_t>(ptr) & 15u) return BSATTN_ERR_ALIGNMENT;
  {
    // the chunks' kernels need compute capability 10.x: refuse before any copy
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return BSATTN_ERR_CUDA;
    if (major != 10) return BSATTN_ERR_UNSUPPORTED;
  }
  const int64_t nq_all = (N + block - 1) / block;
  if ((int64_t)(Hq / Hkv) * kv_heads_per_chunk * nq_all > INT32_MAX) return BSATTN_ERR_UNSUPPORTED;
  HostPipe* pipe = pipe_for_current_device();
  if (!pipe) return BSATTN_ERR_CUDA;
  // On a failure part-way, the caller's stream is still made to wait for
  // everything already queued on the internal streams (copies and kernels that
  // read or write the caller's buffers) before the error is returned.
  auto fail = [&](int rc) {
    if (cudaEventRecord(pipe->done, pipe->in) == cudaSuccess)
      cudaStreamWaitEvent(stream, pipe->done, 0);
    if (cudaEventRecord(pipe->done, pipe->out) == cudaSuccess)
      cudaStreamWaitEvent(stream, pipe->done, 0);
    return rc;
  };

  const int G = Hq / Hkv;
  const int hkc = kv_heads_per_chunk, hqc = hkc * G;     // heads per chunk
  const int nq = (N + block - 1) / block;
  const size_t row = (size_t)N * d * 2;                  // bytes of one head's [N, d] bf16
  auto at = [](const void* base, size_t off) {
    return static_cast<const char*>(base) + off;
  };
  auto atw = [](void* base, size_t off) { return static_cast<char*>(base) + off; };

  // the staging buffers may still be in use by earlier work on `stream`
  if (cudaEventRecord(pipe->start, stream) != cudaSuccess ||
      cudaStreamWaitEvent(pipe->in, pipe->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(pipe->out, pipe->start, 0) != cudaSuccess)
    return fail(BSATTN_ERR_CUDA);

  // One KV head per chunk (the finest setting) with an even group of at least
  // 4 query heads: the first and the last chunk go in pieces of 2 query
  // heads (the first piece brings the KV head's K and V), so that the first
  // kernel starts after a smaller copy and the last copy out follows a
  // smaller kernel -- the copies in set the pace, and these two ends are the
  // part of the call they cannot hide.
  const bool split_ends = hkc == 1 && G % 2 == 0 && G >= 4;
  int c = 0;
  for (int b = 0; b < B; ++b) {
    for (int kv0 = 0; kv0 < Hkv; kv0 += hkc) {
      const bool end = (b == 0 && kv0 == 0) || (b == B - 1 && kv0 + hkc == Hkv);
      const int piece = split_ends && end ? 2 : hqc;   // query heads per piece
      for (int h0 = 0; h0 < hqc; h0 += piece, ++c) {
        const int hq0 = kv0 * G + h0;
        const size_t qoff = ((size_t)b * Hq + hq0) * row, qlen = (size_t)piece * row;
        const size_t koff = ((size_t)b * Hkv + kv0) * row, klen = (size_t)hkc * row;
        cudaEvent_t copied = pipe->copied[c % kEvents], computed = pipe->computed[c % kEvents];
        if (cudaMemcpyAsync(atw(d_q, qoff), at(h_q, qoff), qlen, cudaMemcpyHostToDevice,
                            pipe->in) != cudaSuccess ||
            (h0 == 0 && (cudaMemcpyAsync(atw(d_k, koff), at(h_k, koff), klen,
                                         cudaMemcpyHostToDevice, pipe->in) != cudaSuccess ||
                         cudaMemcpyAsync(atw(d_v, koff), at(h_v, koff), klen,
                                         cudaMemcpyHostToDevice, pipe->in) != cudaSuccess)) ||
            cudaEventRecord(copied, pipe->in) != cudaSuccess ||
            cudaStreamWaitEvent(stream, copied, 0) != cudaSuccess)
          return fail(BSATTN_ERR_CUDA);
        // the piece as a problem of its own: one sequence, `piece` query
        // heads of hkc KV heads; per-head CSR rows and orders start at its
        // first head
        const bool per_head = row_ptr && mask_heads == Hq;
        const int rc = bsattn_fwd_prefill(
            at(d_q, qoff), at(d_k, koff), at(d_v, koff), atw(d_o, qoff), nullptr, 1, piece, hkc, N,
            d, block, scale, causal, lambda,
            row_ptr ? row_ptr + (per_head ? (size_t)hq0 * (nq + 1) : 0) : nullptr, col_idx,
            row_order ? row_order + (per_head ? (size_t)hq0 * nq : 0) : nullptr,
            per_head ? piece : 1, nullptr, d_status, stream);
        if (rc != BSATTN_OK) return fail(rc);
        if (cudaEventRecord(computed, stream) != cudaSuccess ||
            cudaStreamWaitEvent(pipe->out, computed, 0) != cudaSuccess ||
            cudaMemcpyAsync(atw(h_o, qoff), at(d_o, qoff), qlen, cudaMemcpyDeviceToHost,
                            pipe->out) != cudaSuccess)
          return fail(BSATTN_ERR_CUDA);
      }
    }
  }
  // the caller's stream completes after the last copy out
  if (cudaEventRecord(pipe->done, pipe->out) != cudaSuccess ||
      cudaStreamWaitEvent(stream, pipe->done, 0) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  return BSATTN_OK;
}

}  // extern "C"
