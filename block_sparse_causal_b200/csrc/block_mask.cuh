// block_mask.cuh -- dynamic block mask: pool, score, top-k with the diagonal kept.
//
// Ultra Flash (papernotes notes), Method, key design 3: the token grid is cut
// into non-overlapping blocks; queries and keys are mean-pooled per block;
// block relevance is the dot product of the pooled query and key; each head
// keeps its top-k highest-scoring blocks.
//
// One thread block per (TQ = 8 consecutive q-blocks, query head h, batch b),
// 256 threads (one warp per q-block), two thread blocks per SM:
//   0. warp 0 starts bulk copies of the pooled K (written by the append call,
//      one fp32 row per window block, 512 bytes; a window chunk's rows are
//      contiguous, so one copy per run of a chunk's rows) into a ring of 3
//      tiles of 32 rows, so the first tiles arrive while Q is pooled;
//   1. pool: warp w sums q-block i0 + w over its tokens in fp32, each lane 8
//      channels of every other token with 16-byte loads, 16 in flight;
//   2. score: each lane keeps 4 channels of the 8 pooled queries in
//      registers (as fp32 pairs for the packed f32x2 FMA); each warp takes 4
//      kv rows of a tile, one 16-byte read per row and lane, and a 5-step
//      reduce-scatter of the 8 partial dot products; the consumed tile's slot
//      is refilled;
//   3. select: one warp per q-block row finds the (k-1)-th largest
//      non-diagonal score by a 32-step bitwise search over order-preserving
//      integer keys, takes every key above it plus the lowest-index keys equal
//      to it, and writes the kept ids in ascending order with the diagonal.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int MASK_TQ = 8;        // q-blocks per thread block (= warps)
constexpr int MASK_LOG_TQ = 3;
constexpr int MASK_THREADS = 32 * MASK_TQ;
constexpr int MASK_KT = 32;       // pooled-K rows per tile
constexpr int MASK_KSTAGE = 3;    // pooled-K tiles in flight
constexpr int MASK_QLOADS = 16;   // 16-byte Q loads in flight per lane

// Dynamic shared memory of the mask kernel for a window of nkv_max blocks.
__host__ __device__ constexpr int mask_smem_bytes(int nkv_max) {
  return (MASK_KSTAGE * MASK_KT * 128 + MASK_TQ * 128 + MASK_TQ * nkv_max) * 4;
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
__global__ void __launch_bounds__(MASK_THREADS, 2) block_mask_kernel(const MaskParams p) {
  constexpr int D = 128;
  constexpr long long kWait = 1LL << 31;
  extern __shared__ __align__(128) float mraw[];
  float *s_kt = mraw;                                   // [KSTAGE][KT][D]
  float *s_qpool = s_kt + MASK_KSTAGE * MASK_KT * D;    // [TQ][D]
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
      record_error(UF_EBOUNDS);
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
  auto issue_tile = [&](int t) {          // all lanes of warp 0
    const int st = t % MASK_KSTAGE, j0 = t * MASK_KT;
    const int rows = min(MASK_KT, NKV - j0);
    if (lane == 0) mbar_arrive_expect_tx(&bar_k[st], static_cast<uint32_t>(rows) * D * 4);
    __syncwarp();
    if (lane < rows) {
      const int j = j0 + lane;
      const int c = j / p.nb, rr = j - c * p.nb;
      if (lane == 0 || rr == 0) {         // first row of a run of one chunk's rows
        const int len = min(rows - lane, p.nb - rr);
        const int slot = window_slot(c, start, p.W, anchor);
        bulk_load(s_kt + (st * MASK_KT + lane) * D, kp_head + (static_cast<size_t>(slot) * p.nb + rr) * D,
                  static_cast<uint32_t>(len) * D * 4, &bar_k[st]);
      }
    }
  };
  int issued = 0;                         // tiles issued (warp 0's count)
  if (warp == 0)
    for (; issued < min(MASK_KSTAGE, ntiles); ++issued) issue_tile(issued);

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
  // lane l keeps channels 4l .. 4l + 3 of the 8 pooled queries in registers,
  // query (i ^ s) in slot i with s = lane >> 2, as fp32 pairs (slots 2i, 2i+1).
  // Per kv row: one 16-byte read, 16 packed FMAs, then a reduce-scatter over
  // the 32 lanes: at the steps xor 16, 8, 4 every lane keeps the lower half
  // of its slots and sends the upper half (its partner's slot order is the
  // same set of queries, so no selects), then xor 2 and 1 sum; each lane ends
  // with the full dot product of query s.
  static_assert(MASK_TQ == 8, "slot order below assumes 8 queries");
  const int s_ord = lane >> 2;
  uint64_t q2[MASK_TQ / 2][4];
#pragma unroll
  for (int i = 0; i < MASK_TQ / 2; ++i) {
    const float4 lo = *reinterpret_cast<const float4 *>(&s_qpool[((2 * i) ^ s_ord) * D + 4 * lane]);
    const float4 hi = *reinterpret_cast<const float4 *>(&s_qpool[((2 * i + 1) ^ s_ord) * D + 4 * lane]);
    q2[i][0] = f2_pack(lo.x, hi.x);
    q2[i][1] = f2_pack(lo.y, hi.y);
    q2[i][2] = f2_pack(lo.z, hi.z);
    q2[i][3] = f2_pack(lo.w, hi.w);
  }
  const int q_own = s_ord;
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % MASK_KSTAGE;
    if (wait_bounded(&bar_k[st], (t / MASK_KSTAGE) & 1, &s_abort, kWait)) {
      const float *kt = s_kt + st * MASK_KT * D;
#pragma unroll
      for (int r = 0; r < MASK_KT / MASK_TQ; ++r) {
        const int jl = r * MASK_TQ + warp;
        const float4 kv = *reinterpret_cast<const float4 *>(&kt[jl * D + 4 * lane]);
        const uint64_t k0 = f2_pack(kv.x, kv.x), k1 = f2_pack(kv.y, kv.y), k2 = f2_pack(kv.z, kv.z),
                       k3 = f2_pack(kv.w, kv.w);
        float a[MASK_TQ];
#pragma unroll
        for (int i = 0; i < MASK_TQ / 2; ++i) {
          const uint64_t acc = f2_fma(q2[i][3], k3, f2_fma(q2[i][2], k2, f2_fma(q2[i][1], k1, f2_mul(q2[i][0], k0))));
          f2_unpack(acc, a[2 * i], a[2 * i + 1]);
        }
#pragma unroll
        for (int step = 0; step < MASK_LOG_TQ; ++step) {
          const int m = 16 >> step, half = MASK_TQ >> (step + 1);
#pragma unroll
          for (int i = 0; i < half; ++i) a[i] += __shfl_xor_sync(0xffffffffu, a[i + half], m);
        }
        float sum = a[0];
#pragma unroll
        for (int m = 16 >> MASK_LOG_TQ; m >= 1; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
        const int j = t * MASK_KT + jl;
        if ((lane & ((32 >> MASK_LOG_TQ) - 1)) == 0 && j < NKV) s_sc[q_own * nkv_max + j] = sum * p.scale;
      }
    }
    __syncthreads();                                    // tile consumed; every wait of this tile is over
    if (*reinterpret_cast<volatile int32_t *>(&s_abort)) break;
    if (warp == 0 && issued < ntiles) issue_tile(issued++);
  }
  if (*reinterpret_cast<volatile int32_t *>(&s_abort)) {
    // a wait gave up: let the copies still in flight land (bounded) before exiting
    if (tid == 0)
      for (int t = max(0, issued - MASK_KSTAGE); t < issued; ++t) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&bar_k[t % MASK_KSTAGE], (t / MASK_KSTAGE) & 1) && clock64() - t0 < kWait) {
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
