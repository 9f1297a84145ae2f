// block_mask.cuh -- dynamic block mask: pool, score, top-k with the diagonal kept.
//
// Ultra Flash (papernotes notes), Method, key design 3: the token grid is cut
// into non-overlapping blocks; queries and keys are mean-pooled per block;
// block relevance is the dot product of the pooled query and key; each head
// keeps its top-k highest-scoring blocks.
//
// One thread block per (TQ = 8 consecutive q-blocks, query head h, batch b),
// 256 threads (one warp per q-block), two thread blocks per SM:
//   1. pool: warp w sums q-block i0 + w over its tokens in fp32, each lane 8
//      channels of every other token with 16-byte loads, 16 in flight;
//   2. score: on the tensor core, m16n8k8 tf32 MMAs with fp32 accuracy by a
//      hi / lo split of both operands (hi = the top 19 bits of the fp32
//      value, lo = the exact remainder, which the MMA reads to 11 bits:
//      products within 2^-21 relative), as hi.hi + hi.lo + lo.hi in three
//      accumulators so the MMA chains overlap.  The pooled K (written by the
//      append call, one fp32 row per window block) is read from L2 straight
//      into A fragments: each warp takes 16-row slices of the window in turn,
//      each lane loading 4 consecutive channels of its two rows per 16-byte
//      load.  The MMA's k index runs over the channels in that load order
//      (the dot product does not depend on the order of its channels, up to
//      rounding), and the 8 pooled queries' B fragments, split once, follow
//      the same order from shared memory;
//   3. select: one warp per q-block row forces the diagonal (or the local
//      band around it), finds the need-th largest of the other scores (need =
//      k minus the forced blocks) by a bitwise search over order-preserving
//      integer keys (at most 32 steps; it stops as soon as exactly need keys
//      lie at or above the candidate), takes every key above it plus the
//      lowest-index keys equal to it, and writes the kept ids in ascending
//      order.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int MASK_TQ = 8;        // q-blocks per thread block (= warps)
constexpr int MASK_THREADS = 32 * MASK_TQ;
constexpr int MASK_QLOADS = 16;   // 16-byte Q loads in flight per lane

// Dynamic shared memory of the mask kernel for a window of nkv_max blocks:
// pooled queries, their split B fragments (16 k-steps x 32 lanes x 16 bytes)
// and the scores.
__host__ __device__ constexpr int mask_smem_bytes(int nkv_max) {
  return (MASK_TQ * 128 + 16 * 32 * 4 + MASK_TQ * nkv_max) * 4;
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
  int32_t *err;             // the window's error word, or NULL (the module's)
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
__global__ void __launch_bounds__(MASK_THREADS, 2) block_mask_kernel(const MaskParams p) {
  constexpr int D = 128;
  extern __shared__ __align__(128) float mraw[];
  float *s_qpool = mraw;                                          // [TQ][D]
  uint4 *s_bfrag = reinterpret_cast<uint4 *>(s_qpool + MASK_TQ * D);   // [D / 8][32 lanes]
  float *s_sc = reinterpret_cast<float *>(s_bfrag + (D / 8) * 32);   // [TQ][W*nb]
  __shared__ int32_t s_meta[3];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.H / p.G);
  const int i0 = blockIdx.x * MASK_TQ;
  const int nkv_max = p.W * p.nb;

  if (tid == 0) {
    int32_t start = __ldcg(p.meta + 0), n = __ldcg(p.meta + 1), anc = __ldcg(p.meta + 3);
    if (!window_state_ok(start, n, anc, p.W)) {
      record_error(p.err, UF_EBOUNDS);
      n = 0;
      start = 0;
      anc = 0;
    }
    s_meta[0] = start;
    s_meta[1] = n;
    s_meta[2] = anc;
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

  // ---- 1. pool the query blocks: warp w takes q-block i0 + w ----------------
  {
    const int cg = lane & 15, rpar = lane >> 4;         // channels 8 cg .. 8 cg + 7, token parity
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const int t0 = (i0 + warp) * BLK;
    const int ntok = warp < tq_count ? min(BLK, p.Lc - t0) : 0;
    const size_t tok_stride = static_cast<size_t>(p.H) * D;
    const __nv_bfloat16 *qb = p.q + ((static_cast<size_t>(b) * p.Lc + t0) * p.H + h) * D + cg * 8;
#pragma unroll 1
    for (int r0 = 0; r0 < ntok; r0 += 2 * MASK_QLOADS) {
      uint4 v[MASK_QLOADS];
#pragma unroll
      for (int m = 0; m < MASK_QLOADS; ++m) {
        const int r = r0 + 2 * m + rpar;
        v[m] = r < ntok ? __ldg(reinterpret_cast<const uint4 *>(qb + r * tok_stride)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int m = 0; m < MASK_QLOADS; ++m) {
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v[m]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    if (lane < 16) {
      const float inv = ntok > 0 ? 1.0f / static_cast<float>(ntok) : 0.f;
      float4 *dst = reinterpret_cast<float4 *>(s_qpool + warp * D + cg * 8);
      dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    }
  }
  __syncthreads();                                      // s_qpool complete

  // ---- 2. pooled scores against every block of the window -----------------
  // D[16 kv rows x 8 queries] += A[rows x 8 k] B[8 k x queries] over 16 k-steps,
  // each operand split as x = hi + lo (tf32 parts).  Fragments (m16n8k8, gid =
  // lane / 4, tig = lane % 4): A rows gid, gid + 8 at k = tig, tig + 4; B
  // query gid at k = tig, tig + 4; D rows gid, gid + 8 and queries 2 tig,
  // 2 tig + 1.  Channel of (k-step kk, k = tig + 4 s):
  //   16 (kk / 2) + 4 tig + 2 (kk mod 2) + s,
  // so that one 16-byte load of channels 16 m + 4 tig .. + 3 holds the A
  // values of k-steps 2 m and 2 m + 1.
  const int gid = lane >> 2, tig = lane & 3;
  for (int e = tid; e < (D / 8) * 32; e += MASK_THREADS) {
    const int kk = e >> 5, ln = e & 31, qg = ln >> 2, qt = ln & 3;
    const int c0 = 16 * (kk >> 1) + 4 * qt + 2 * (kk & 1);
    const float v0 = s_qpool[qg * D + c0], v1 = s_qpool[qg * D + c0 + 1];
    const uint32_t h0 = __float_as_uint(v0) & 0xFFFFE000u, h1 = __float_as_uint(v1) & 0xFFFFE000u;
    s_bfrag[e] = make_uint4(h0, h1, __float_as_uint(v0 - __uint_as_float(h0)),
                            __float_as_uint(v1 - __uint_as_float(h1)));
  }
  __syncthreads();                                      // B fragments complete

  const float *kp_head = p.kpool + (static_cast<size_t>(b) * p.G + g) * nkv_max * D;
  // logical window block j -> its pooled-K row (channels 4 tig .. of each 16)
  auto krow = [&](int j) -> const float4 * {
    const int c = j / p.nb, rr = j - c * p.nb;
    const int slot = window_slot(c, start, p.W, anchor);
    return reinterpret_cast<const float4 *>(kp_head + (static_cast<size_t>(slot) * p.nb + rr) * D) + tig;
  };
  const int nslices = (NKV + 15) / 16;
#pragma unroll 1
  for (int sl = warp; sl < nslices; sl += MASK_TQ) {
    const int j = sl * 16 + gid;
    float4 r0[8], r1[8];
    {
      const bool ok0 = j < NKV, ok1 = j + 8 < NKV;
      const float4 *k0 = ok0 ? krow(j) : nullptr;
      const float4 *k1 = ok1 ? krow(j + 8) : nullptr;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        r0[m] = ok0 ? __ldg(k0 + 4 * m) : make_float4(0.f, 0.f, 0.f, 0.f);
        r1[m] = ok1 ? __ldg(k1 + 4 * m) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float dhh[4] = {0.f, 0.f, 0.f, 0.f}, dhl[4] = {0.f, 0.f, 0.f, 0.f}, dlh[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < D / 8; ++kk) {
      const float4 &x0 = r0[kk >> 1], &x1 = r1[kk >> 1];
      const float av[4] = {(kk & 1) ? x0.z : x0.x, (kk & 1) ? x1.z : x1.x, (kk & 1) ? x0.w : x0.y,
                           (kk & 1) ? x1.w : x1.y};
      uint32_t ah[4], al[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ah[e] = __float_as_uint(av[e]) & 0xFFFFE000u;
        al[e] = __float_as_uint(av[e] - __uint_as_float(ah[e]));
      }
      const uint4 bf = s_bfrag[kk * 32 + lane];
      const uint32_t bh[2] = {bf.x, bf.y}, bl[2] = {bf.z, bf.w};
      mma_tf32_16x8x8(dhh, ah, bh);
      mma_tf32_16x8x8(dhl, ah, bl);
      mma_tf32_16x8x8(dlh, al, bh);
    }
    float d[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) d[e] = dhh[e] + (dhl[e] + dlh[e]);
    if (j < NKV) {
      s_sc[(2 * tig) * nkv_max + j] = d[0] * p.scale;
      s_sc[(2 * tig + 1) * nkv_max + j] = d[1] * p.scale;
    }
    if (j + 8 < NKV) {
      s_sc[(2 * tig) * nkv_max + j + 8] = d[2] * p.scale;
      s_sc[(2 * tig + 1) * nkv_max + j + 8] = d[3] * p.scale;
    }
  }
  __syncthreads();                                      // every score written

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
      // the need-th largest key: largest T with #(key >= T) >= need, bit by
      // bit; once exactly need keys are >= T the kept set is fixed (the
      // search could only raise T among keys that are all kept), so it stops
      T = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        int c = 0;
#pragma unroll
        for (int m = 0; m < MAXPER; ++m) c += key[m] >= cand;
        const int tot = __reduce_add_sync(0xffffffffu, c);
        if (tot >= need) {
          T = cand;
          if (tot == need) break;
        }
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
