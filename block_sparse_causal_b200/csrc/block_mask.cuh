// block_mask.cuh -- dynamic block mask: pool, score, top-k with the diagonal kept.
//
// Ultra Flash (papernotes notes), Method, key design 3: the token grid is cut
// into non-overlapping blocks; queries and keys are mean-pooled per block;
// block relevance is the dot product of the pooled query and key; each head
// keeps its top-k highest-scoring blocks.
//
// One thread block per (TQ = 8 consecutive q-blocks, query head h, batch b),
// 256 threads:
//   1. pool: the block's Q tokens are streamed once from HBM with 16-byte
//      loads (16 token lanes x 16 column chunks) and summed in fp32;
//   2. score: pooled K (written by the append call, one fp32 row per window
//      block) is staged 64 rows at a time in shared memory; each warp takes 8
//      kv rows, each lane a quarter of the head dim for all 8 q-blocks, and
//      two xor-shuffles finish the dot products;
//   3. select: one warp per q-block row finds the (k-1)-th largest
//      non-diagonal score by a 32-step bitwise search over order-preserving
//      integer keys, takes every key above it plus the lowest-index keys equal
//      to it, and writes the kept ids in ascending order with the diagonal.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int MASK_TQ = 8;        // q-blocks per thread block (= warps)
constexpr int MASK_KT = 64;       // pooled-K rows per shared-memory tile
constexpr int MASK_KSTRIDE = 144; // padded row stride (floats): conflict-free float4 reads

struct MaskParams {
  const __nv_bfloat16 *q;   // [B, Lc, H, D]
  const float *kpool;       // [B, G, W*nb, D] physical slot order
  const int32_t *meta;
  int32_t *idx;             // [B, H, nb, k]
  int32_t *cnt;             // [B, H, nb]
  float *scores;            // optional [B, H, nb, W*nb]
  int32_t H, G, W, Lc, nb, k;
  float scale;
};

// Order-preserving map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_excl_scan(int v, int lane) {
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

template <int BLK>
__global__ void __launch_bounds__(256) block_mask_kernel(const MaskParams p) {
  constexpr int D = 128;
  constexpr int PASSES = BLK / 16;
  extern __shared__ __align__(16) float msm[];
  float *s_qpool = msm;                                  // [TQ][D]
  float *s_red = s_qpool + MASK_TQ * D;                  // [16][D]
  float *s_kt = s_red + 16 * D;                          // [KT][KSTRIDE]
  float *s_sc = s_kt + MASK_KT * MASK_KSTRIDE;           // [TQ][W*nb]
  __shared__ int32_t s_meta[2];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.H / p.G);
  const int i0 = blockIdx.x * MASK_TQ;
  const int nkv_max = p.W * p.nb;

  if (tid == 0) {
    int32_t start = __ldcg(p.meta + 0), n = __ldcg(p.meta + 1);
    if (start < 0 || start >= p.W || n < 1 || n > p.W) {
      record_error(UF_EBOUNDS);
      n = 0;
      start = 0;
    }
    s_meta[0] = start;
    s_meta[1] = n;
  }
  __syncthreads();
  const int start = s_meta[0], n_valid = s_meta[1];
  const int NKV = n_valid * p.nb;
  const int tq_count = min(MASK_TQ, p.nb - i0);
  if (n_valid == 0) {     // empty window: nothing to select
    for (int e = tid; e < tq_count * p.k; e += blockDim.x) {
      const int tq = e / p.k, c = e % p.k;
      p.idx[((static_cast<size_t>(b) * p.H + h) * p.nb + i0 + tq) * p.k + c] = -1;
    }
    if (tid < tq_count) p.cnt[(static_cast<size_t>(b) * p.H + h) * p.nb + i0 + tid] = 0;
    return;
  }

  // ---- 1. pool the query blocks -------------------------------------------
  const int tl = tid >> 4, dc = tid & 15;
  const size_t qstride = static_cast<size_t>(p.H) * D;
  for (int tq = 0; tq < tq_count; ++tq) {
    const int t0 = (i0 + tq) * BLK;
    const int ntok = min(BLK, p.Lc - t0);
    const __nv_bfloat16 *src = p.q + (static_cast<size_t>(b) * p.Lc + t0) * qstride + h * D + dc * 8;
    uint4 r[PASSES];
#pragma unroll
    for (int m = 0; m < PASSES; ++m) {
      const int t = tl + 16 * m;
      r[m] = (t < ntok) ? __ldg(reinterpret_cast<const uint4 *>(src + t * qstride)) : make_uint4(0, 0, 0, 0);
    }
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int m = 0; m < PASSES; ++m) {
      const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&r[m]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
    *reinterpret_cast<float4 *>(&s_red[tl * D + dc * 8]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4 *>(&s_red[tl * D + dc * 8 + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) s += s_red[q * D + tid];
      s_qpool[tq * D + tid] = s / static_cast<float>(ntok);
    }
    __syncthreads();
  }
  for (int e = tid; e < (MASK_TQ - tq_count) * D; e += blockDim.x) s_qpool[tq_count * D + e] = 0.f;

  // ---- 2. pooled scores against every block of the window -----------------
  const float *kp_head = p.kpool + (static_cast<size_t>(b) * p.G + g) * nkv_max * D;
  const int jr = lane >> 2, dq = lane & 3;
  for (int j0 = 0; j0 < NKV; j0 += MASK_KT) {
    __syncthreads();   // previous tile fully consumed
#pragma unroll
    for (int it = 0; it < (MASK_KT * D / 4) / 256; ++it) {
      const int e = it * 256 + tid;
      const int row = e >> 5, c4 = e & 31;
      const int j = j0 + row;
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < NKV) {
        const int c = j / p.nb, rr = j - c * p.nb;
        const int slot = (start + c) % p.W;
        val = __ldg(reinterpret_cast<const float4 *>(kp_head + (static_cast<size_t>(slot) * p.nb + rr) * D) + c4);
      }
      *reinterpret_cast<float4 *>(&s_kt[row * MASK_KSTRIDE + c4 * 4]) = val;
    }
    __syncthreads();
    const int jl = warp * 8 + jr;
    float acc[MASK_TQ];
#pragma unroll
    for (int t = 0; t < MASK_TQ; ++t) acc[t] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int d = c * 16 + dq * 4;
      const float4 kv = *reinterpret_cast<const float4 *>(&s_kt[jl * MASK_KSTRIDE + d]);
#pragma unroll
      for (int t = 0; t < MASK_TQ; ++t) {
        const float4 qv = *reinterpret_cast<const float4 *>(&s_qpool[t * D + d]);
        acc[t] = fmaf(qv.x, kv.x, acc[t]);
        acc[t] = fmaf(qv.y, kv.y, acc[t]);
        acc[t] = fmaf(qv.z, kv.z, acc[t]);
        acc[t] = fmaf(qv.w, kv.w, acc[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < MASK_TQ; ++t) {
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
    }
    const int j = j0 + jl;
    if (j < NKV) {
      s_sc[(2 * dq) * nkv_max + j] = acc[2 * dq] * p.scale;
      s_sc[(2 * dq + 1) * nkv_max + j] = acc[2 * dq + 1] * p.scale;
    }
  }
  __syncthreads();

  // ---- 3. per-row selection (one warp per q-block) --------------------------
  if (warp < tq_count) {
    const int i = i0 + warp;
    const float *sc = s_sc + warp * nkv_max;
    const size_t row = (static_cast<size_t>(b) * p.H + h) * p.nb + i;
    if (p.scores) {
      for (int j = lane; j < NKV; j += 32) p.scores[row * nkv_max + j] = sc[j];
    }
    const int diag = (n_valid - 1) * p.nb + i;
    const int k_eff = min(p.k, NKV);
    const int need = k_eff - 1;            // non-diagonal blocks to keep
    const int per = (NKV + 31) / 32;
    const int jb = lane * per, je = min(NKV, jb + per);

    uint32_t T = 0xFFFFFFFFu;              // threshold key (need == 0: nothing passes)
    int take_eq = 0;
    if (need > 0) {
      T = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        int c = 0;
        for (int j = jb; j < je; ++j) c += (j != diag && order_key(sc[j]) >= cand);
        c = __reduce_add_sync(0xffffffffu, c);
        if (c >= need) T = cand;
      }
      int gt = 0;
      for (int j = jb; j < je; ++j) gt += (j != diag && order_key(sc[j]) > T);
      gt = __reduce_add_sync(0xffffffffu, gt);
      take_eq = need - gt;
    }
    // lowest-index ties first: rank of this lane's equal keys among all lanes
    int eq_l = 0;
    if (need > 0)
      for (int j = jb; j < je; ++j) eq_l += (j != diag && order_key(sc[j]) == T);
    int eq_before = warp_excl_scan(eq_l, lane);
    // selected ids of this lane's range, ascending
    int sel_l = 0;
    {
      int eq_run = eq_before;
      for (int j = jb; j < je; ++j) {
        bool keep = (j == diag);
        if (!keep && need > 0) {
          const uint32_t key = order_key(sc[j]);
          if (key > T) keep = true;
          else if (key == T && eq_run < take_eq) keep = true;
          if (key == T) ++eq_run;
        }
        sel_l += keep;
      }
    }
    int pos = warp_excl_scan(sel_l, lane);
    int32_t *out = p.idx + row * p.k;
    {
      int eq_run = eq_before;
      for (int j = jb; j < je; ++j) {
        bool keep = (j == diag);
        if (!keep && need > 0) {
          const uint32_t key = order_key(sc[j]);
          if (key > T) keep = true;
          else if (key == T && eq_run < take_eq) keep = true;
          if (key == T) ++eq_run;
        }
        if (keep && pos < k_eff) out[pos++] = j;
      }
    }
    for (int c = k_eff + lane; c < p.k; c += 32) out[c] = -1;
    if (lane == 0) p.cnt[row] = k_eff;
  }
}

}  // namespace uf
