// Split-KV decode with the BLASST skip, and the exact combine of the splits.
//
// "BLASST: Dynamic Blocked Attention Sparsity via Softmax Thresholding",
// section 4.2: decode is bound by HBM reads of the KV cache, so the kernel
// streams every K tile, decides after the scores whether the tile is skipped,
// and issues the V load only for kept tiles; K loads run ahead so that the
// decision and the remaining V loads overlap.
//
// decode_split_kernel: one CTA per (batch, KV head, split), 256 threads.
//   Query tile = the G query heads sharing the KV head (one token each).
//   K and V tiles are TMA-loaded (128-byte swizzle, so that per-key rows can
//   be read without bank conflicts) into rings of KST and VST stages.
//   Per visited tile t:
//     QK     each key is owned by 32/KPW lanes of a warp (KPW keys per warp),
//            each lane dots a slice of d for all G rows; lanes combine with
//            xor-shuffles; masks keys past the cache length.
//     max    warp max -> shared memory -> every thread forms the tile max
//            per row, the skip decision (all G rows below running max +
//            log2(lambda)) and the new running max, identically.
//     keep   scores are parked in a ring slot and V_t's load is issued; the
//            P*V of tile t runs LA tiles later, so V_t's latency hides behind
//            the next tiles' K streaming and scores.  The exponent shift is
//            lazy: it only moves when the running max exceeds it by more than
//            TAU, and then the partial O and row sums are rescaled first.
//   The split writes its unnormalised O (fp32), shift and row sum.  Options
//   as in the tensor-core kernel: sink-seeded splits, per-sequence lengths.
// decode_combine_kernel: one CTA per (batch, query head): log-sum-exp merge of
//   the splits into bf16 O and fp32 LSE.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsattn_internal.h"
#include "sm100_ptx.cuh"

namespace bsattn {

template <int D, int BLK, int G>
struct DecodeCfg {
  static constexpr int THREADS = 256;
  static constexpr int WARPS = 8;
  static constexpr int KST = G >= 8 ? 2 : 3;    // K ring stages
  static constexpr int LA = 2;                  // P*V lags the scores by LA tiles
  static constexpr int VST = LA + 1;            // V ring stages (and parked score slots)
  static constexpr int HALVES = D / 64;
  static constexpr int T_HALF = BLK * 128;
  static constexpr int T_BYTES = HALVES * T_HALF;
  static constexpr int KPW = BLK / WARPS;       // keys per warp in the score phase
  static constexpr int PARTS = 32 / KPW;        // lanes per key
  static constexpr int DPART = D / PARTS;       // dims per lane
  static constexpr int DP = D / 2;              // dim pairs in the P*V phase
  static constexpr int KGROUPS = THREADS / DP;  // key groups in the P*V phase
  static constexpr int KPG = BLK / KGROUPS;     // keys per group
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KST * T_BYTES;
  static constexpr int S_OFF = V_OFF + VST * T_BYTES;           // float [VST][BLK][G]
  static constexpr int P_OFF = S_OFF + VST * BLK * G * 4;       // float [BLK][G]
  static constexpr int Q_OFF = P_OFF + BLK * G * 4;             // float [G][D]
  static constexpr int RED_OFF = Q_OFF + G * D * 4;             // float [2][WARPS][G]
  static constexpr int ORED_OFF = RED_OFF + 2 * WARPS * G * 4;  // float [KGROUPS][G][D]
  static constexpr int BAR_OFF = ORED_OFF + KGROUPS * G * D * 4;
  static constexpr int SMEM = BAR_OFF + 128 + 1024;
  static constexpr float TAU = 8.0f;
  static_assert(KPW >= 8 && 32 % KPW == 0, "score mapping");
  static_assert(DPART % 8 == 0, "8-element chunks");
  static_assert(THREADS % DP == 0, "P*V mapping");
};

struct DecodeBarriers {
  uint64_t k_full[3];
  uint64_t v_full[3];
  int abort;
};

// Address of element chunk `c` (8 bf16 = 16 bytes) of row `r` in a tile laid
// out as HALVES boxes of [rows][64] with the 128-byte swizzle.
template <int T_HALF>
__device__ __forceinline__ const uint8_t* swz_chunk(const uint8_t* tile, int r, int c) {
  const int half = c / 8, cc = c % 8;
  return tile + half * T_HALF + r * 128 + ((cc ^ (r & 7)) << 4);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

template <int D, int BLK, int G>
__global__ void __launch_bounds__(256, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using C = DecodeCfg<D, BLK, G>;
  static_assert(sizeof(DecodeBarriers) <= 128, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* k_smem = smem + C::K_OFF;
  uint8_t* v_smem = smem + C::V_OFF;
  float* s_park = reinterpret_cast<float*>(smem + C::S_OFF);
  float* p_s = reinterpret_cast<float*>(smem + C::P_OFF);
  float* q_s = reinterpret_cast<float*>(smem + C::Q_OFF);
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  float* ored = reinterpret_cast<float*>(smem + C::ORED_OFF);
  DecodeBarriers* bars = reinterpret_cast<DecodeBarriers*>(smem + C::BAR_OFF);
  volatile int* abort = &bars->abort;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int split = blockIdx.x % p.splits;
  const int bk = blockIdx.x / p.splits;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  // cache length (the splits cut the sequence's own tiles) and tile range
  const int lenb = p.seq_lens ? min(max(p.seq_lens[b], 0), p.L) : p.L;
  const int Tb = p.seq_lens ? (lenb + BLK - 1) / BLK : p.T;
  const int chunk = p.seq_lens ? (Tb > 0 ? (Tb + p.splits - 1) / p.splits : 1) : p.chunk;
  const int t_begin = split * chunk;
  const int t_end = min(Tb, t_begin + chunk);
  // tile stream of the split: with sink seeding, step 0 scores key tile 0
  // only to start the running max; step t >= sd is key tile t_begin + t - sd
  const int sd = (p.sink_seed && split > 0 && t_end > t_begin) ? 1 : 0;
  const int nt = max(0, t_end - t_begin) + sd;
  auto tile_of = [&](int t) { return (sd && t == 0) ? 0 : t_begin + t - sd; };
  const int zc = b * p.Hkv + kvh;

  if (tid == 0) trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, 1);
  if (tid == 0) {
    for (int s = 0; s < C::KST; ++s) mbar_init(&bars->k_full[s], 1);
    for (int s = 0; s < C::VST; ++s) mbar_init(&bars->v_full[s], 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  // queries of the group -> fp32 in shared memory
  const __nv_bfloat16* qg = p.q + ((int64_t)b * p.Hq + (int64_t)kvh * G) * D;
  for (int x = tid; x < G * D; x += C::THREADS) q_s[x] = __bfloat162float(qg[x]);
  __syncthreads();

  if (tid == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    for (int s = 0; s < C::KST && s < nt; ++s) {
      mbar_arrive_expect_tx(&bars->k_full[s], C::T_BYTES);
      for (int hf = 0; hf < C::HALVES; ++hf)
        tma_load_3d(k_smem + s * C::T_BYTES + hf * C::T_HALF, &tmK, &bars->k_full[s], hf * 64,
                    tile_of(s) * BLK, zc);
    }
  }

  // score-phase mapping
  const int key_w = lane % C::KPW;              // key inside the warp's group
  const int part = lane / C::KPW;               // which slice of d
  const int key = warp * C::KPW + key_w;        // key inside the tile
  // P*V-phase mapping
  const int dp = tid % C::DP;                   // dim pair
  const int kg = tid / C::DP;                   // key group

  float m_run[G], m_ref[G];
  float lpart[G];        // row-sum partials of key `tid` (tid < BLK)
  float oacc[G][2];      // O partials: rows x (2 dims of pair dp) over key group kg
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    m_ref[g] = -INFINITY;
    lpart[g] = 0.f;
    oacc[g][0] = oacc[g][1] = 0.f;
  }
  int kept_total = 0;     // kept tiles so far
  uint32_t hist = 0;      // bit k: tile (it - k) was kept
  int issued_k = min(C::KST, nt), issued_v = 0;
  const uint64_t lim = p.wait_limit_ns;
  bool aborted = false;

  for (int it = 0; it < nt + C::LA; ++it) {
    hist <<= 1;
    // ------------------------------------------------ scores of tile `it`
    if (it < nt) {
      const int t = it;
      const int ks = t % C::KST;
      // warp-uniform outcome: the shuffles below need every lane
      const bool failed =
          __any_sync(0xffffffffu, !mbar_wait(&bars->k_full[ks], (t / C::KST) & 1, abort, lim));
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0.f;
      if (!failed) {
        const uint8_t* kt = k_smem + ks * C::T_BYTES;
#pragma unroll
        for (int c = 0; c < C::DPART / 8; ++c) {
          const int chunk = part * (C::DPART / 8) + c;
          const uint4 u = *reinterpret_cast<const uint4*>(swz_chunk<C::T_HALF>(kt, key, chunk));
          float kf[8];
          bf16x8_to_f32(u, kf);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4 q0 = *reinterpret_cast<const float4*>(q_s + g * D + chunk * 8);
            const float4 q1 = *reinterpret_cast<const float4*>(q_s + g * D + chunk * 8 + 4);
            acc[g] = fmaf(q0.x, kf[0], acc[g]);
            acc[g] = fmaf(q0.y, kf[1], acc[g]);
            acc[g] = fmaf(q0.z, kf[2], acc[g]);
            acc[g] = fmaf(q0.w, kf[3], acc[g]);
            acc[g] = fmaf(q1.x, kf[4], acc[g]);
            acc[g] = fmaf(q1.y, kf[5], acc[g]);
            acc[g] = fmaf(q1.z, kf[6], acc[g]);
            acc[g] = fmaf(q1.w, kf[7], acc[g]);
          }
        }
#pragma unroll
        for (int off = C::KPW; off < 32; off <<= 1)
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], off);
        const int kpos = tile_of(t) * BLK + key;
        if (kpos >= lenb)
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g] = -INFINITY;
        // warp max over its KPW keys
        float mx[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          mx[g] = acc[g];
#pragma unroll
          for (int off = 1; off < C::KPW; off <<= 1)
            mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], off));
        }
        if (lane == 0)
#pragma unroll
          for (int g = 0; g < G; ++g) red[((it & 1) * C::WARPS + warp) * G + g] = mx[g];
      }
      if (__syncthreads_or(failed)) { aborted = true; break; }
      // K slot `ks` is free again: stream the tile KST ahead into it
      if (tid == 0 && issued_k < nt) {
        const int tn = issued_k;
        mbar_arrive_expect_tx(&bars->k_full[ks], C::T_BYTES);
        for (int hf = 0; hf < C::HALVES; ++hf)
          tma_load_3d(k_smem + ks * C::T_BYTES + hf * C::T_HALF, &tmK, &bars->k_full[ks],
                      hf * 64, tile_of(tn) * BLK, zc);
      }
      issued_k = min(issued_k + 1, nt);
      // tile max per row (base-2 units), the vote, the running max
      float mt[G];
      bool all_pass = true;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float m = -INFINITY;
#pragma unroll
        for (int w = 0; w < C::WARPS; ++w) m = fmaxf(m, red[((it & 1) * C::WARPS + w) * G + g]);
        mt[g] = m * p.scale_log2;
        all_pass = all_pass && (mt[g] - m_run[g] < p.thr_log2);
      }
      // the seed step only starts the running max: never kept, not a visit
      const bool seed = sd && t == 0;
      const bool skip = seed || (p.use_skip && all_pass);
#pragma unroll
      for (int g = 0; g < G; ++g) m_run[g] = fmaxf(m_run[g], mt[g]);
      if (tid == 0 && p.tile_status && !seed)
        p.tile_status[(int64_t)zc * p.T + tile_of(t)] = skip ? 1 : 2;
      if (!skip) {
        const int slot = kept_total % C::VST;
        // park the raw scores for the delayed P*V
        if (part == 0)
#pragma unroll
          for (int g = 0; g < G; ++g) s_park[(slot * BLK + key) * G + g] = acc[g];
        if (tid == 0) {
          mbar_arrive_expect_tx(&bars->v_full[slot], C::T_BYTES);
          for (int hf = 0; hf < C::HALVES; ++hf)
            tma_load_3d(v_smem + slot * C::T_BYTES + hf * C::T_HALF, &tmV, &bars->v_full[slot],
                        hf * 64, tile_of(t) * BLK, zc);
        }
        ++issued_v;
        // lazy exponent shift
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (kept_total == 0) {
            m_ref[g] = m_run[g];
          } else if (m_run[g] > m_ref[g] + C::TAU) {
            const float alpha = fast_exp2(m_ref[g] - m_run[g]);
            lpart[g] *= alpha;
            oacc[g][0] *= alpha;
            oacc[g][1] *= alpha;
            m_ref[g] = m_run[g];
          }
        }
        ++kept_total;
        hist |= 1u;
      }
    }
    // ------------------------------------------------ P*V of tile `it - LA`
    if (it >= C::LA && (hist >> C::LA) & 1u) {
      const int kidx = kept_total - 1 - __popc(hist & ((1u << C::LA) - 1u));
      const int slot = kidx % C::VST;
      const int vphase = (kidx / C::VST) & 1;
      const bool failed =
          __any_sync(0xffffffffu, !mbar_wait(&bars->v_full[slot], vphase, abort, lim));
      if (!failed && tid < BLK) {
        float pr[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float sh = m_ref[g] == -INFINITY ? 0.f : m_ref[g];
          pr[g] = fast_exp2(fmaf(s_park[(slot * BLK + tid) * G + g], p.scale_log2, -sh));
          lpart[g] += pr[g];
        }
#pragma unroll
        for (int g = 0; g < G; ++g) p_s[tid * G + g] = pr[g];
      }
      if (__syncthreads_or(failed)) { aborted = true; break; }
      const uint8_t* vt = v_smem + slot * C::T_BYTES;
      const int dim0 = dp * 2;
      const int chunk = dim0 / 8;
#pragma unroll 4
      for (int kk = 0; kk < C::KPG; ++kk) {
        const int kr = kg * C::KPG + kk;
        const uint32_t w2 = *reinterpret_cast<const uint32_t*>(
            swz_chunk<C::T_HALF>(vt, kr, chunk) + (dim0 % 8) * 2);
        const float v0 = __uint_as_float(w2 << 16);
        const float v1 = __uint_as_float(w2 & 0xffff0000u);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = p_s[kr * G + g];
          oacc[g][0] = fmaf(pg, v0, oacc[g][0]);
          oacc[g][1] = fmaf(pg, v1, oacc[g][1]);
        }
      }
    }
  }

  if (aborted) {
    if (tid == 0) {
      for (int t = max(0, issued_k - C::KST); t < issued_k; ++t)
        mbar_wait_drain(&bars->k_full[t % C::KST], (t / C::KST) & 1, lim);
      for (int k = max(0, issued_v - C::VST); k < issued_v; ++k)
        mbar_wait_drain(&bars->v_full[k % C::VST], (k / C::VST) & 1, lim);
      report_status(p.status, kDevTimeout);
      trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, 13);
    }
    return;
  }

  // ------------------------------------------------ reduce and write the split
  __syncthreads();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    ored[(kg * G + g) * D + dp * 2] = oacc[g][0];
    ored[(kg * G + g) * D + dp * 2 + 1] = oacc[g][1];
  }
  // row sums: reduce the per-key partials (threads < BLK) through `red`
  float lsum[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float x = tid < BLK ? lpart[g] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    lsum[g] = x;
  }
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) red[warp * G + g] = lsum[g];
  __syncthreads();
  const int64_t base = ((int64_t)b * p.Hq + (int64_t)kvh * G) * p.splits + split;
  for (int x = tid; x < G * D; x += C::THREADS) {
    const int g = x / D, dd = x % D;
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < C::KGROUPS; ++q) s += ored[(q * G + g) * D + dd];
    p.ws_o[(base + (int64_t)g * p.splits) * D + dd] = s;
  }
  if (tid < G) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) s += red[w * G + tid];
    p.ws_l[base + (int64_t)tid * p.splits] = kept_total > 0 ? s : 0.f;
    p.ws_m[base + (int64_t)tid * p.splits] = kept_total > 0 ? m_ref[tid] : -INFINITY;
  }
  if (tid == 0) trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, 3);
}

// One CTA per (batch, query head), one thread per output dimension.
__global__ void decode_combine_kernel(const CombineParams p) {
  const int64_t bh = blockIdx.x;
  const int dd = threadIdx.x;
  const float* m = p.ws_m + bh * p.splits;
  const float* l = p.ws_l + bh * p.splits;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, m[s]);
  float num = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      if (m[s] == -INFINITY) continue;
      const float w = fast_exp2(m[s] - M);
      den += w * l[s];
      num += w * p.ws_o[(bh * p.splits + s) * p.D + dd];
    }
  }
  const bool have = den > 0.f;
  p.o[bh * p.D + dd] = __float2bfloat16_rn(have ? num / den : 0.f);
  if (dd == 0 && p.lse) p.lse[bh] = have ? (M + __log2f(den)) * 0.69314718055994531f : -INFINITY;
}

template <int D, int BLK, int G>
cudaError_t launch_decode_split(const CUtensorMap& tk, const CUtensorMap& tv,
                                const DecodeParams& p, int grid, cudaStream_t stream) {
  using C = DecodeCfg<D, BLK, G>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, BLK, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D, BLK, G><<<grid, C::THREADS, C::SMEM, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

#define BSATTN_INST(DD, BB, GG)                                                            \
  template cudaError_t launch_decode_split<DD, BB, GG>(const CUtensorMap&, const CUtensorMap&, \
                                                       const DecodeParams&, int, cudaStream_t);
BSATTN_INST(128, 128, 1) BSATTN_INST(128, 128, 2) BSATTN_INST(128, 128, 4) BSATTN_INST(128, 128, 8)
BSATTN_INST(64, 128, 1) BSATTN_INST(64, 128, 2) BSATTN_INST(64, 128, 4) BSATTN_INST(64, 128, 8)
BSATTN_INST(128, 64, 1) BSATTN_INST(128, 64, 2) BSATTN_INST(128, 64, 4) BSATTN_INST(128, 64, 8)
BSATTN_INST(64, 64, 1) BSATTN_INST(64, 64, 2) BSATTN_INST(64, 64, 4) BSATTN_INST(64, 64, 8)
#undef BSATTN_INST

cudaError_t launch_decode_combine(const CombineParams& p, int grid, int threads,
                                  cudaStream_t stream) {
  decode_combine_kernel<<<grid, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsattn
