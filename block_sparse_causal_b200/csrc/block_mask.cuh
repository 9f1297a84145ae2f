// block_mask.cuh -- dynamic block mask: pool, score, top-k with the diagonal kept.
//
// Ultra Flash (papernotes notes), Method, key design 3: the token grid is cut
// into non-overlapping blocks; queries and keys are mean-pooled per block;
// block relevance is the dot product of the pooled query and key; each head
// keeps its top-k highest-scoring blocks.
//
// One thread block per (TQ = 8 consecutive q-blocks, query head h, batch b),
// 256 threads, two thread blocks per SM:
//   1. pool: TMA copies each q-block's slice of Q (BLK tokens x 128 channels,
//      two 64-channel panels) into a double-buffered shared-memory ring, so a
//      whole slice is in flight while the previous one is reduced; each
//      thread sums a channel pair over a quarter of the tokens in fp32;
//   2. score: pooled K (written by the append call, one fp32 row per window
//      block) is staged 32 rows at a time in shared memory; each warp takes 4
//      kv rows, each lane an eighth of the head dim for all 8 q-blocks, and
//      three xor-shuffles finish the dot products;
//   3. select: one warp per q-block row finds the (k-1)-th largest
//      non-diagonal score by a 32-step bitwise search over order-preserving
//      integer keys, takes every key above it plus the lowest-index keys equal
//      to it, and writes the kept ids in ascending order with the diagonal.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int MASK_TQ = 8;        // q-blocks per thread block (= warps)
constexpr int MASK_KT = 32;       // pooled-K rows per shared-memory tile
constexpr int MASK_KSTRIDE = 144; // padded row stride (floats): conflict-free float4 reads
constexpr int MASK_QBUF = 2;      // q-block slices in flight per thread block

// Dynamic shared memory of the mask kernel for a window of nkv_max blocks.
__host__ __device__ constexpr int mask_smem_bytes(int blk, int nkv_max) {
  return 1024 + MASK_QBUF * blk * 256 + (MASK_TQ * 128 + 2 * 4 * 128 + MASK_KT * MASK_KSTRIDE + MASK_TQ * nkv_max) * 4;
}

struct MaskParams {
  const __nv_bfloat16 *q;   // [B, Lc, H, D]
  const float *kpool;       // [B, G, W*nb, D] physical slot order
  const int32_t *meta;
  int32_t *idx;             // [B, H, nb, k]
  int32_t *cnt;             // [B, H, nb]
  float *scores;            // optional [B, H, nb, W*nb]
  int32_t H, G, W, Lc, nb, k;
  int32_t local;            // radius of the forced band of blocks around the diagonal
  int32_t local_only;       // keep the band only (no scored blocks)
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

template <int BLK, int MAXPER>
__global__ void __launch_bounds__(256, 2) block_mask_kernel(const __grid_constant__ CUtensorMap tmQ, const MaskParams p) {
  constexpr int D = 128;
  constexpr int QSLICE = BLK * 256;                     // bytes of one q-block slice (two panels)
  extern __shared__ uint8_t mraw[];
  uint8_t *mbase = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(mraw) + 1023) & ~uintptr_t(1023));
  uint8_t *s_qbuf = mbase;                              // [QBUF][2 panels][BLK][128 B]
  float *s_qpool = reinterpret_cast<float *>(mbase + MASK_QBUF * QSLICE);   // [TQ][D]
  float *s_red = s_qpool + MASK_TQ * D;                 // [2][4][D]
  float *s_kt = s_red + 2 * 4 * D;                      // [KT][KSTRIDE]
  float *s_sc = s_kt + MASK_KT * MASK_KSTRIDE;          // [TQ][W*nb]
  __shared__ int32_t s_meta[3];
  __shared__ uint64_t bar_q[MASK_QBUF];
  __shared__ int32_t s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.H / p.G);
  const int i0 = blockIdx.x * MASK_TQ;
  const int nkv_max = p.W * p.nb;

  if (tid == 0) {
    int32_t start = __ldcg(p.meta + 0), n = __ldcg(p.meta + 1), anc = __ldcg(p.meta + 3);
    if (!window_state_ok(start, n, anc, p.W)) {
      record_error(UF_EBOUNDS);
      n = 0;
      start = 0;
      anc = 0;
    }
    s_meta[0] = start;
    s_meta[1] = n;
    s_meta[2] = anc;
    for (int q = 0; q < MASK_QBUF; ++q) mbar_init(&bar_q[q], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int start = s_meta[0], n_valid = s_meta[1], anchor = s_meta[2];
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
  auto load_slice = [&](int tq) {
    uint64_t *bar = &bar_q[tq % MASK_QBUF];
    uint8_t *dst = s_qbuf + (tq % MASK_QBUF) * QSLICE;
    mbar_arrive_expect_tx(bar, QSLICE);
    tma_load_4d(dst, &tmQ, bar, 0, h, (i0 + tq) * BLK, b);
    tma_load_4d(dst + QSLICE / 2, &tmQ, bar, 64, h, (i0 + tq) * BLK, b);
  };
  if (tid == 0)
    for (int tq = 0; tq < min(MASK_QBUF, tq_count); ++tq) load_slice(tq);
  const int cp = tid & 63, rg = tid >> 6;                // channel pair, quarter of the tokens
  const int pnl = cp >> 5, cpo = (cp & 31) * 4;          // panel and byte offset of the pair in a row
  for (int tq = 0; tq < tq_count; ++tq) {
    const int t0 = (i0 + tq) * BLK;
    const int ntok = min(BLK, p.Lc - t0);                // tokens past Lc were zero-filled by TMA
    if (!wait_bounded(&bar_q[tq % MASK_QBUF], (tq / MASK_QBUF) & 1, &s_abort, 1LL << 31)) break;
    const uint8_t *slice = s_qbuf + (tq % MASK_QBUF) * QSLICE + pnl * (QSLICE / 2) + cpo;
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll 8
    for (int r = rg * (BLK / 4); r < (rg + 1) * (BLK / 4); r += 2) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(slice + r * 128));
      const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(slice + (r + 1) * 128));
      a0 += f.x;
      a1 += f.y;
      b0 += g2.x;
      b1 += g2.y;
    }
    float *red = s_red + (tq & 1) * 4 * D + rg * D;
    red[2 * cp] = a0 + b0;
    red[2 * cp + 1] = a1 + b1;
    __syncthreads();                                     // slice consumed, partial sums visible
    if (tid == 0 && tq + MASK_QBUF < tq_count) load_slice(tq + MASK_QBUF);
    if (tid < D) {
      const float *rr = s_red + (tq & 1) * 4 * D;
      s_qpool[tq * D + tid] = ((rr[tid] + rr[D + tid]) + (rr[2 * D + tid] + rr[3 * D + tid])) / static_cast<float>(ntok);
    }
  }
  for (int e = tid; e < (MASK_TQ - tq_count) * D; e += blockDim.x) s_qpool[tq_count * D + e] = 0.f;

  // ---- 2. pooled scores against every block of the window -----------------
  const float *kp_head = p.kpool + (static_cast<size_t>(b) * p.G + g) * nkv_max * D;
  const int jr = lane >> 3, dq = lane & 7;
  // this thread's share of a pooled-K tile: 4 float4 of rows (e >> 5), e = it*256 + tid
  auto fetch = [&](int j0, float4 (&v)[4]) {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = it * 256 + tid;
      const int j = j0 + (e >> 5);
      v[it] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < NKV) {
        const int c = j / p.nb, rr = j - c * p.nb;
        const int slot = window_slot(c, start, p.W, anchor);
        v[it] = __ldg(reinterpret_cast<const float4 *>(kp_head + (static_cast<size_t>(slot) * p.nb + rr) * D) + (e & 31));
      }
    }
  };
  float4 nxt[4];
  fetch(0, nxt);
  for (int j0 = 0; j0 < NKV; j0 += MASK_KT) {
    __syncthreads();   // previous tile fully consumed (and qpool complete on the first pass)
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = it * 256 + tid;
      *reinterpret_cast<float4 *>(&s_kt[(e >> 5) * MASK_KSTRIDE + (e & 31) * 4]) = nxt[it];
    }
    __syncthreads();
    if (j0 + MASK_KT < NKV) fetch(j0 + MASK_KT, nxt);   // in flight while this tile is scored
    const int jl = warp * 4 + jr;
    float acc[MASK_TQ];
#pragma unroll
    for (int t = 0; t < MASK_TQ; ++t) acc[t] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int d = c * 32 + dq * 4;
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
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 4);
    }
    float mine = acc[0];
#pragma unroll
    for (int t = 1; t < MASK_TQ; ++t)
      if (dq == t) mine = acc[t];
    const int j = j0 + jl;
    if (j < NKV) s_sc[dq * nkv_max + j] = mine * p.scale;
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
    // forced blocks: the band [diag - local, diag + local] of the window
    // (local = 0: the diagonal alone); the host guarantees 2 local + 1 <= k
    const int lo = max(0, diag - p.local), hi = min(NKV - 1, diag + p.local);
    const int n_forced = hi - lo + 1;
    const int k_eff = p.local_only ? n_forced : min(p.k, NKV);
    const int need = k_eff - n_forced;     // scored blocks to keep
    const int per = (NKV + 31) / 32;       // keys of this lane: j in [lane*per, lane*per + per)
    const int jb = lane * per;
    // order-preserving integer keys in registers; forced blocks and padding get
    // 0 (below every real key: a float's key is never 0) and are never counted
    uint32_t key[MAXPER];
#pragma unroll
    for (int m = 0; m < MAXPER; ++m) {
      const int j = jb + m;
      key[m] = (m < per && j < NKV && (j < lo || j > hi)) ? order_key(sc[j]) : 0u;
    }
    uint32_t T = 0xFFFFFFFFu;              // threshold key (need == 0: nothing passes)
    int take_eq = 0;
    if (need > 0) {
      // the need-th largest key: largest T with #(key >= T) >= need, bit by bit
      T = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        int c = 0;
#pragma unroll
        for (int m = 0; m < MAXPER; ++m) c += key[m] >= cand;
        if (__reduce_add_sync(0xffffffffu, c) >= need) T = cand;
      }
      int gt = 0;
#pragma unroll
      for (int m = 0; m < MAXPER; ++m) gt += key[m] > T;
      take_eq = need - __reduce_add_sync(0xffffffffu, gt);
    }
    // lowest-index ties first: rank of this lane's equal keys among all lanes
    int eq_l = 0;
    if (need > 0) {
#pragma unroll
      for (int m = 0; m < MAXPER; ++m) eq_l += key[m] == T;
    }
    const int eq_before = warp_excl_scan(eq_l, lane);
    uint32_t sel_mask = 0;                 // bit m: j = jb + m kept
    {
      int eq_run = eq_before;
#pragma unroll
      for (int m = 0; m < MAXPER; ++m) {
        const int j = jb + m;
        bool keep = (m < per && j >= lo && j <= hi);
        if (need > 0 && key[m] != 0u) {
          if (key[m] > T) keep = true;
          else if (key[m] == T && eq_run < take_eq) keep = true;
          if (key[m] == T) ++eq_run;
        }
        if (keep) sel_mask |= 1u << m;
      }
    }
    int pos = warp_excl_scan(__popc(sel_mask), lane);
    int32_t *out = p.idx + row * p.k;
#pragma unroll
    for (int m = 0; m < MAXPER; ++m)
      if ((sel_mask >> m) & 1u) {
        if (pos < k_eff) out[pos] = jb + m;
        ++pos;
      }
    for (int c = k_eff + lane; c < p.k; c += 32) out[c] = -1;
    if (lane == 0) p.cnt[row] = k_eff;
  }
}

}  // namespace uf
