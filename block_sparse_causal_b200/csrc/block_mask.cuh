// block_mask.cuh -- dynamic block mask: pool, score, top-k with the diagonal kept.
//
// Ultra Flash (papernotes notes), Method, key design 3: the token grid is cut
// into non-overlapping blocks; queries and keys are mean-pooled per block;
// block relevance is the dot product of the pooled query and key; each head
// keeps its top-k highest-scoring blocks.
//
// One thread block per (TQ = 8 consecutive q-blocks, query head h, batch b),
// 256 threads (one warp per q-block), two thread blocks per SM:
//   0. the pooled K (written by the append call, one fp32 row per window
//      block) streams through a ring of 4 tiles of 32 rows: stage s holds
//      tiles s, s + 4, ... and belongs to warps 2s and 2s + 1, which fill it
//      (one bulk copy per row, into rows padded to 132 floats) and consume it;
//      the first four tiles are requested at entry, so they arrive while Q is
//      pooled;
//   1. pool: warp w sums q-block i0 + w over its tokens in fp32, each lane 8
//      channels of every other token with 16-byte loads, 16 in flight;
//   2. score: on the tensor core, m16n8k8 tf32 MMAs with fp32 accuracy by a
//      hi / lo split of both operands (hi = the top 19 bits of the fp32
//      value, lo = the exact remainder, which the MMA reads to 11 bits:
//      products within 2^-21 relative), as hi.hi + hi.lo + lo.hi in three
//      accumulators so the MMA chains overlap; each warp takes one 16-row
//      half of its stage's tiles against the 8 pooled queries (held in
//      registers as B fragments);
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
constexpr int MASK_KT = 32;       // pooled-K rows per tile
constexpr int MASK_KSTAGE = 4;    // pooled-K tiles in flight (stage s: warps 2s, 2s + 1)
constexpr int MASK_KSTRIDE = 132; // floats per pooled-K row in shared memory (conflict-free A fragments)
static_assert(2 * MASK_KSTAGE == MASK_TQ, "each warp pair owns one stage");
constexpr int MASK_QLOADS = 16;   // 16-byte Q loads in flight per lane

// Dynamic shared memory of the mask kernel for a window of nkv_max blocks.
__host__ __device__ constexpr int mask_smem_bytes(int nkv_max) {
  return (MASK_KSTAGE * MASK_KT * MASK_KSTRIDE + MASK_TQ * 128 + MASK_TQ * nkv_max) * 4;
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
  constexpr long long kWait = 1LL << 31;
  extern __shared__ __align__(128) float mraw[];
  float *s_kt = mraw;                                   // [KSTAGE][KT][KSTRIDE]
  float *s_qpool = s_kt + MASK_KSTAGE * MASK_KT * MASK_KSTRIDE;   // [TQ][D]
  float *s_sc = s_qpool + MASK_TQ * D;                  // [TQ][W*nb]
  __shared__ int32_t s_meta[3];
  __shared__ uint64_t bar_k[MASK_KSTAGE];
  __shared__ int32_t s_abort;

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
    for (int q = 0; q < MASK_KSTAGE; ++q) mbar_init(&bar_k[q], 1);
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

  // ---- 0. pooled-K tiles: one 512-byte bulk copy per window block ----------
  const float *kp_head = p.kpool + (static_cast<size_t>(b) * p.G + g) * nkv_max * D;
  const int ntiles = (NKV + MASK_KT - 1) / MASK_KT;
  const int pair = warp >> 1;            // this warp's stage; tiles pair, pair + KSTAGE, ...
  auto issue_tile = [&](int t) {          // all lanes of warp 2 * (t mod KSTAGE)
    const int st = t % MASK_KSTAGE, j0 = t * MASK_KT;
    const int rows = min(MASK_KT, NKV - j0);
    if (lane == 0) mbar_arrive_expect_tx(&bar_k[st], static_cast<uint32_t>(rows) * D * 4);
    __syncwarp();
    if (lane < rows) {
      const int j = j0 + lane;
      const int c = j / p.nb, rr = j - c * p.nb;
      const int slot = window_slot(c, start, p.W, anchor);
      bulk_load(s_kt + (st * MASK_KT + lane) * MASK_KSTRIDE, kp_head + (static_cast<size_t>(slot) * p.nb + rr) * D,
                D * 4, &bar_k[st]);
    }
  };
  int last_issued = -1;                   // (even warps) last tile issued into this warp pair's stage
  if ((warp & 1) == 0 && pair < ntiles) {
    issue_tile(pair);
    last_issued = pair;
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
  // D[16 kv rows x 8 queries] += A[rows x 8 channels] B[8 channels x queries]
  // over 16 channel steps, each operand split as x = hi + lo (tf32 parts).
  // Fragments (m16n8k8, gid = lane / 4, tig = lane % 4): A rows gid, gid + 8
  // and channels tig, tig + 4; B query gid, channels tig, tig + 4; D rows
  // gid, gid + 8 and queries 2 tig, 2 tig + 1.
  const int gid = lane >> 2, tig = lane & 3;
  uint32_t bh[D / 8][2], bl[D / 8][2];
#pragma unroll
  for (int kk = 0; kk < D / 8; ++kk)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float v = s_qpool[gid * D + kk * 8 + tig + 4 * e];
      bh[kk][e] = __float_as_uint(v) & 0xFFFFE000u;
      bl[kk][e] = __float_as_uint(v - __uint_as_float(bh[kk][e]));
    }
  const int mh = warp & 1;                // this warp's 16-row half of each tile
  for (int t = pair; t < ntiles; t += MASK_KSTAGE) {
    // both warps of the pair run the same iterations (the named barrier below
    // needs both); after an abort the waits return at once and nothing is issued
    if (wait_bounded(&bar_k[pair], (t / MASK_KSTAGE) & 1, &s_abort, kWait, p.err)) {
      const float *kt = s_kt + (pair * MASK_KT + mh * 16) * MASK_KSTRIDE;
      float dhh[4] = {0.f, 0.f, 0.f, 0.f}, dhl[4] = {0.f, 0.f, 0.f, 0.f}, dlh[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk) {
        const float av[4] = {kt[gid * MASK_KSTRIDE + kk * 8 + tig], kt[(gid + 8) * MASK_KSTRIDE + kk * 8 + tig],
                             kt[gid * MASK_KSTRIDE + kk * 8 + tig + 4],
                             kt[(gid + 8) * MASK_KSTRIDE + kk * 8 + tig + 4]};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          ah[e] = __float_as_uint(av[e]) & 0xFFFFE000u;
          al[e] = __float_as_uint(av[e] - __uint_as_float(ah[e]));
        }
        mma_tf32_16x8x8(dhh, ah, bh[kk]);
        mma_tf32_16x8x8(dhl, ah, bl[kk]);
        mma_tf32_16x8x8(dlh, al, bh[kk]);
      }
      float d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) d[e] = dhh[e] + (dhl[e] + dlh[e]);
      const int j = t * MASK_KT + mh * 16 + gid;
      if (j < NKV) {
        s_sc[(2 * tig) * nkv_max + j] = d[0] * p.scale;
        s_sc[(2 * tig + 1) * nkv_max + j] = d[1] * p.scale;
      }
      if (j + 8 < NKV) {
        s_sc[(2 * tig) * nkv_max + j + 8] = d[2] * p.scale;
        s_sc[(2 * tig + 1) * nkv_max + j + 8] = d[3] * p.scale;
      }
    }
    // the pair is done with the stage: its even warp refills it
    named_barrier(1 + pair, 64);
    if (mh == 0 && t + MASK_KSTAGE < ntiles && !*reinterpret_cast<volatile int32_t *>(&s_abort)) {
      issue_tile(t + MASK_KSTAGE);
      last_issued = t + MASK_KSTAGE;
    }
  }
  __syncthreads();                                      // every score written
  if (*reinterpret_cast<volatile int32_t *>(&s_abort)) {
    // a wait gave up: each stage's filler lets its last copy land (bounded)
    // before the block exits
    if (mh == 0 && lane == 0 && last_issued >= 0) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&bar_k[pair], (last_issued / MASK_KSTAGE) & 1) && clock64() - t0 < kWait) {
      }
    }
    return;
  }

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
