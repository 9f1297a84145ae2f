// attention.cuh -- block-sparse chunk-causal attention on tcgen05 tensor cores.
//
// Ultra Flash (papernotes notes), Method, key design 3: attention is computed
// only over the kept (query block, kv block) pairs.  FlashDecoder (xllm-io
// blog), Sec. 3.3: no token mask inside the window (causality by processing
// order); Eq. 4: grouped-query KV heads.
//
// One thread block = one work item (batch b, query head h, q-block i): a
// 128-row Q tile against the item's list of n kept kv blocks, split inside the
// block into two interleaved halves -- the even-numbered kept blocks (t = 0,
// 2, 4, ...) and the odd-numbered ones -- processed by two independent
// pipelines that share only the Q tile.  Pipeline x has its own TMA producer
// warp, ring of K / V shared-memory stages, MMA-issuing warp, S and O
// accumulators in tensor memory and softmax warpgroup; the two partial
// results are merged once at the end with their running maxima and sums (the
// merge rule of online softmax).  Two issuing warps keep two independent
// instruction streams in front of the tensor core, which overlaps them.
// Twelve warps:
//   warps 0, 1   TMA producers of pipelines 0 and 1: the pipeline's K / V
//                tiles gathered by the block list, in the order its MMA warp
//                consumes them (K_x, then V_t, K_{t+2} for t = x, x+2, ...);
//                warp 0 also loads the Q tile;
//   warps 2, 3   MMA issuers (one thread each): S_x = Q K_t^T (SS, K-major
//                operands, 128-byte swizzle) and O_x += P_x V_t (TS: P from
//                tensor memory, V stored transposed in the window so it is a
//                K-major operand too).  P_x is written over the first columns
//                of S_x, so S_x is reused for block t + 2 only after PV_t has
//                completed (MMAs into different accumulators are not ordered
//                by the hardware); warp 2 owns the tensor-memory allocation;
//   warps 4-7    softmax of pipeline 0, warps 8-11 of pipeline 1: each thread
//                owns one row, reads it from S_x (32x32b loads), applies the
//                block's token mask, keeps a running max / sum in the exp2
//                domain, writes P as packed bf16 and rescales its row of O_x
//                only when the running max grew by more than 2^8 (a stale max
//                is exact: O_x and the sum share the same reference).  When
//                S_x for block t arrives, PV_{t-2} into O_x has completed, so
//                the softmax never waits for anything but its S.  The two
//                softmax warpgroups take turns in global block order (t,
//                t + 1, ...), so one always computes exponentials while the
//                other pipeline's MMAs run (two pipelines left alone fall into
//                lockstep and contend for the same units).
// Tensor memory (512 columns): S0 [0,128) O0 [128,256) S1 [256,384)
// O1 [384,512); P_x occupies the first BLK/2 columns of S_x.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int ATTN_THREADS = 384;
constexpr int ATTN_SOFTMAX_THREADS = 256;
constexpr int ATTN_NSTAGE = 6;                   // shared-memory stages, ATTN_NSTAGE / 2 per pipeline
constexpr int ATTN_PSTAGE = ATTN_NSTAGE / 2;
// tensor-memory column of S_x and of O_x
__host__ __device__ constexpr uint32_t tm_s(int x) { return static_cast<uint32_t>(x) * 256u; }
__host__ __device__ constexpr uint32_t tm_o(int x) { return 128u + static_cast<uint32_t>(x) * 256u; }
constexpr float ATTN_RESCALE_LOG2 = 8.0f;

struct AttnParams {
  const int32_t *meta;
  const int32_t *idx;   // [B, H, nb, k] or NULL (dense)
  const int32_t *cnt;   // [B, H, nb] or NULL
  __nv_bfloat16 *o;     // [B, Lc, H, D]
  float *lse;           // [B, H, Lc] or NULL
  int32_t H, G, W, Lc, nb, lslot, k;
  float scale_log2;     // softmax scale * log2(e)
  long long wait_limit;
};

template <int BLK>
struct AttnSmem {
  static constexpr int Q_BYTES = 128 * 256;          // 128 rows x 128 d x bf16, two 64-column panels
  static constexpr int PANEL = BLK * 128;            // one 64-channel panel of a K tile
  static constexpr int VPANEL = 128 * 128;           // one 64-token panel of a V^T tile (128 channels)
  static constexpr int STAGE = BLK * 256;
  static constexpr int DYN = 1024 + Q_BYTES + ATTN_NSTAGE * STAGE;
};

// Logical kv block j of the window -> first row of its tile in the cache and
// its number of true tokens.
__device__ __forceinline__ void kv_block_coords(int j, int start, int W, int nb, int lslot, int blk, int Lc,
                                                int &row, int &valid) {
  const int c = j / nb, r = j - c * nb;
  const int slot = (start + c) % W;
  row = slot * lslot + r * blk;
  valid = (r == nb - 1) ? (Lc - (nb - 1) * blk) : blk;
}

template <int BLK>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, const AttnParams p) {
  using L = AttnSmem<BLK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + L::Q_BYTES;

  __shared__ uint64_t bar_q, bar_l;
  __shared__ uint64_t bar_fin[2];
  __shared__ uint64_t bar_full[ATTN_NSTAGE], bar_empty[ATTN_NSTAGE];
  __shared__ uint64_t bar_s[2], bar_p[2], bar_o[2], bar_turn[2], bar_st[2];
  __shared__ uint32_t s_tbase;
  __shared__ int32_t s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NQ = p.nb;
  const int item = blockIdx.x;
  const int i = item % NQ;
  const int bh = item / NQ;
  const int h = bh % p.H, b = bh / p.H;
  const int g = h / (p.H / p.G);

  // window state (written by the append call earlier on the stream)
  const int start = __ldcg(p.meta + 0), n_valid = __ldcg(p.meta + 1);
  const bool bad_meta = start < 0 || start >= p.W || n_valid < 1 || n_valid > p.W;
  const int NKV = bad_meta ? 0 : n_valid * p.nb;
  const int diag = (n_valid - 1) * p.nb + i;
  const int32_t *row_idx = p.idx ? p.idx + static_cast<size_t>(item) * p.k : nullptr;
  int n = NKV;
  if (row_idx) {
    n = p.cnt ? __ldg(p.cnt + item) : p.k;
    if (n > p.k) n = -1;   // malformed row
  }
  const bool skip = bad_meta || n < 1;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_fin[0], 1);
    mbar_init(&bar_fin[1], 1);
    mbar_init(&bar_l, ATTN_SOFTMAX_THREADS);
    for (int s = 0; s < ATTN_NSTAGE; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_s[s], 1);
      mbar_init(&bar_p[s], ATTN_SOFTMAX_THREADS / 2);
      mbar_init(&bar_o[s], 1);
      mbar_init(&bar_turn[s], ATTN_SOFTMAX_THREADS / 2);
      mbar_init(&bar_st[s], ATTN_SOFTMAX_THREADS / 2);
    }
    s_abort = 0;
    fence_mbar_init();
    if (skip) record_error(UF_EBOUNDS);
  }
  if (warp == 2) {
    tmem_alloc(&s_tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tbase;
  volatile int32_t *abort_flag = &s_abort;

  if (warp < 2) {
    // ------------------------------------------------------------ producer --
    const int x = warp;                         // pipeline of this producer
    const int n_mine = skip ? 0 : (n - x + 1) / 2;
    if (lane == 0 && !skip) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (x == 0) {
        tma_prefetch_desc(&tmQ);
        mbar_arrive_expect_tx(&bar_q, L::Q_BYTES);
        tma_load_4d(sQ, &tmQ, &bar_q, 0, h, i * BLK, b);
        tma_load_4d(sQ + L::Q_BYTES / 2, &tmQ, &bar_q, 64, h, i * BLK, b);
      }
      const int zc = b * p.G + g;
      const int stage0 = x * ATTN_PSTAGE;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      // same order as this pipeline's MMA warp consumes: K_x, then V_t, K_{t+2} for t = x, x+2, ...
      auto load = [&](int t, bool is_v) -> bool {
        if (!wait_bounded(&bar_empty[stage0 + stage], phase ^ 1u, abort_flag, p.wait_limit)) return false;
        int jb = row_idx ? __ldg(row_idx + t) : t;
        if (jb < 0 || jb >= NKV) {
          record_error(UF_EBOUNDS);
          jb = diag;
        }
        int row, valid;
        kv_block_coords(jb, start, p.W, p.nb, p.lslot, BLK, p.Lc, row, valid);
        uint64_t *full = &bar_full[stage0 + stage];
        mbar_arrive_expect_tx(full, L::STAGE);
        uint8_t *dst = sKV + (stage0 + stage) * L::STAGE;
        if (is_v) {
          // V^T tile: 128 channel rows x BLK tokens, in 64-token panels
#pragma unroll
          for (int pnl = 0; pnl < BLK / 64; ++pnl)
            tma_load_3d(dst + pnl * L::VPANEL, &tmV, full, row + 64 * pnl, 0, zc);
        } else {
          // K tile: BLK token rows x 128 channels, in 64-channel panels
          tma_load_3d(dst, &tmK, full, 0, row, zc);
          tma_load_3d(dst + L::PANEL, &tmK, full, 64, row, zc);
        }
        ++issued;
        if (++stage == ATTN_PSTAGE) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      bool ok = n_mine > 0 ? load(x, false) : true;
      for (int u = 0; u < n_mine && ok; ++u) {
        const int t = x + 2 * u;
        ok = load(t, true);
        if (ok && t + 2 < n) ok = load(t + 2, false);
      }
      if (!ok) {
        // unwind: let every load still in flight land before the block exits
        int s = stage;
        uint32_t ph = phase;
        for (int q = 0; q < ATTN_PSTAGE && q < issued; ++q) {
          if (--s < 0) {
            s = ATTN_PSTAGE - 1;
            ph ^= 1u;
          }
          int32_t never = 0;
          wait_bounded(&bar_full[stage0 + s], ph, &never, p.wait_limit);
        }
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ MMA -------
    const int x = warp - 2;                     // pipeline of this issuer
    const int n_mine = skip ? 0 : (n - x + 1) / 2;
    if (lane == 0 && n_mine > 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, BLK, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t kv_addr = smem_u32(sKV);
      const int stage0 = x * ATTN_PSTAGE;
      const uint32_t s_tmem = tb + tm_s(x), o_tmem = tb + tm_o(x);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = wait_bounded(&bar_q, 0, abort_flag, p.wait_limit);
      if (ok) tc_fence_after();
      auto advance = [&]() {
        if (++stage == ATTN_PSTAGE) {
          stage = 0;
          phase ^= 1u;
        }
      };
      auto issue_qk = [&]() -> bool {
        if (!wait_bounded(&bar_full[stage0 + stage], phase, abort_flag, p.wait_limit)) return false;
        tc_fence_after();
        const uint32_t k_addr = kv_addr + (stage0 + stage) * L::STAGE;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * (L::Q_BYTES / 2) + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_addr + (kk >> 2) * L::PANEL + off, 16, 1024);
          mma_ss(s_tmem, ad, bd, idesc_qk, kk > 0);
        }
        mma_commit(&bar_empty[stage0 + stage]);
        mma_commit(&bar_s[x]);
        advance();
        return true;
      };
      auto issue_pv = [&](int u) -> bool {
        if (!wait_bounded(&bar_p[x], u & 1, abort_flag, p.wait_limit)) return false;
        if (!wait_bounded(&bar_full[stage0 + stage], phase, abort_flag, p.wait_limit)) return false;
        tc_fence_after();
        const uint32_t v_addr = kv_addr + (stage0 + stage) * L::STAGE;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(v_addr + (kk >> 2) * L::VPANEL + (kk & 3) * 32, 16, 1024);
          mma_ts(o_tmem, s_tmem + kk * 8, bd, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_empty[stage0 + stage]);
        mma_commit(&bar_o[x]);
        advance();
        return true;
      };
      if (ok) ok = issue_qk();
      for (int u = 0; u < n_mine && ok; ++u) {
        if (!(ok = issue_pv(u))) break;
        if (u + 1 < n_mine) {
          // S_x / P_x is reused for the next block once this PV has read P_x
          if (!(ok = wait_bounded(&bar_o[x], u & 1, abort_flag, p.wait_limit))) break;
          tc_fence_after();
          if (!(ok = issue_qk())) break;
        }
      }
      // every MMA issued by this thread has completed once bar_fin flips
      mma_commit(&bar_fin[x]);
      int32_t never = 0;
      wait_bounded(&bar_fin[x], 0, &never, p.wait_limit);
    }
  } else {
    // ------------------------------------------------------------ softmax ---
    const int x = (warp - 4) >> 2;              // pipeline: 0 = even kept blocks, 1 = odd kept blocks
    const int wq = warp & 3;                    // tensor-memory lane quarter of this warp
    const int row = wq * 32 + lane;             // row of the Q tile
    const uint32_t lane_base = tb + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_col = tm_s(x), o_col = tm_o(x);
    const int q_tok = i * BLK + row;
    const bool row_out = row < BLK && q_tok < p.Lc;
    const float c_log2 = p.scale_log2;
    const uint64_t c2 = f2_pack(c_log2, c_log2);
    float m_run = -INFINITY, l_run = 0.f;
    // tcgen05.ld / st are warp-collective: every wait result is made warp-uniform
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, p.wait_limit));
    };
    bool ok = !skip;
    const int n_mine = skip ? 0 : (n - x + 1) / 2;   // kept blocks of this warpgroup
    for (int u = 0; u < n_mine && ok; ++u) {
      const int t = x + 2 * u;
      int jb = row_idx ? __ldg(row_idx + t) : t;
      if (jb < 0 || jb >= NKV) jb = diag;
      int krow, valid;
      kv_block_coords(jb, start, p.W, p.nb, p.lslot, BLK, p.Lc, krow, valid);
      if (!(ok = wwait(&bar_s[x], u & 1))) break;
      // turn: block t - 1 (the other warpgroup) has finished its exponentials
      if (x == 0 && u > 0) {
        if (!(ok = wwait(&bar_turn[1], (u - 1) & 1))) break;
      } else if (x == 1) {
        if (!(ok = wwait(&bar_turn[0], u & 1))) break;
      }
      tc_fence_after();
      const bool full = valid == BLK;
      const uint64_t negm_run2 = f2_pack(-m_run, -m_run);
      uint32_t pk[BLK / 2];
      uint64_t acc2[4] = {0, 0, 0, 0};
      float m_use = m_run;
      float mx = -INFINITY;
      bool done = false;
      if (full && u > 0) {
        // common case: exponentials against the running (possibly stale)
        // max, with the block max computed in the same pass -- the max
        // instructions hide under the SFU-bound exponentials.  Kept unless a
        // row's block max exceeds the reference by more than 2^8.
        uint32_t s[BLK];
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c)
          tmem_ld32(lane_base + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
        tmem_wait_ld();
        float a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = -INFINITY;
#pragma unroll
        for (int c = 0; c < BLK / 2; ++c) {
          const float s0 = __uint_as_float(s[2 * c]), s1 = __uint_as_float(s[2 * c + 1]);
          a[c & 7] = max3f(a[c & 7], s0, s1);
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s0, s1), c2, negm_run2), x0, x1);
          const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
          acc2[c & 3] = f2_add(acc2[c & 3], f2_pack(e0, e1));
          pk[c] = pack_bf16x2(e0, e1);
        }
        mx = max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
        done = !__any_sync(0xffffffffu, mx * c_log2 > m_run + ATTN_RESCALE_LOG2);
      }
      if (!done) {
        // S is still intact in tensor memory: P is stored only below
        uint32_t s[BLK];
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c)
          tmem_ld32(lane_base + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
        tmem_wait_ld();
        if (!(full && u > 0)) {
          // first block of the row or a partial block: the max first
          float a[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e] = -INFINITY;
          if (full) {
#pragma unroll
            for (int c = 0; c < BLK; c += 16)
#pragma unroll
              for (int e = 0; e < 8; ++e)
                a[e] = max3f(a[e], __uint_as_float(s[c + 2 * e]), __uint_as_float(s[c + 2 * e + 1]));
          } else {
#pragma unroll
            for (int c = 0; c < BLK; ++c)
              if (c < valid) a[c & 7] = fmaxf(a[c & 7], __uint_as_float(s[c]));
          }
          mx = max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
        }
        const float m_new = fmaxf(m_run, mx * c_log2);
        const bool need = m_new > m_run + ATTN_RESCALE_LOG2;
        if (__any_sync(0xffffffffu, need)) {
          m_use = m_new;
          const float factor = ex2_approx(m_run - m_new);
          l_run *= factor;
          if (u > 0) {
            // PV_{t-2} into O_x completed before S_x for block t was computed
            const uint64_t f2 = f2_pack(factor, factor);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(lane_base + o_col + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                float lo, hi;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), f2), lo, hi);
                o[2 * e] = __float_as_uint(lo);
                o[2 * e + 1] = __float_as_uint(hi);
              }
              tmem_st32(lane_base + o_col + 32 * c, o);
            }
          }
        }
        // P = exp2(s * c - m): full-block and masked (partial last block of a
        // chunk) cases are separate loops: a per-element mask test inside the
        // unrolled loop costs two ALU instructions per element
        const uint64_t negm2 = f2_pack(-m_use, -m_use);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc2[e] = 0;
        if (full) {
#pragma unroll
          for (int c = 0; c < BLK / 2; ++c) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), c2, negm2), x0, x1);
            const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
            acc2[c & 3] = f2_add(acc2[c & 3], f2_pack(e0, e1));
            pk[c] = pack_bf16x2(e0, e1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BLK / 2; ++c) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), c2, negm2), x0, x1);
            const float e0 = 2 * c < valid ? ex2_approx(x0) : 0.f;
            const float e1 = 2 * c + 1 < valid ? ex2_approx(x1) : 0.f;
            acc2[c & 3] = f2_add(acc2[c & 3], f2_pack(e0, e1));
            pk[c] = pack_bf16x2(e0, e1);
          }
        }
      }
      {
        float a0, a1;
        f2_unpack(f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3])), a0, a1);
        l_run += a0 + a1;
      }
      m_run = m_use;
      mbar_arrive(&bar_turn[x]);
#pragma unroll
      for (int c = 0; c < BLK / 64; ++c)
        tmem_st32(lane_base + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * c]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p[x]);
    }
    // ---------------------------------------------------------- epilogue ----
    // merge the two pipelines: (m_x, l_x, O_x) -> O, LSE.  Each warpgroup waits
    // for its own pipeline's last PV only (the other pipeline may lag by any
    // number of blocks), then publishes (m, l) in its pipeline's first ring
    // stage, idle once that last PV has completed; bar_l orders both.
    const int n0 = skip ? 0 : (n + 1) / 2, n1 = skip ? 0 : n / 2;
    const int n_x = x == 0 ? n0 : n1;
    float *s_ml_mine = reinterpret_cast<float *>(sKV + x * ATTN_PSTAGE * L::STAGE);
    float *s_ml_other = reinterpret_cast<float *>(sKV + (x ^ 1) * ATTN_PSTAGE * L::STAGE);
    if (ok && !skip && n_x > 0) ok = wwait(&bar_o[x], (n_x - 1) & 1);
    // this warpgroup writes output columns [64x, 64x + 64): its own pipeline's
    // part of them is final already, the other pipeline's after bar_l
    uint32_t own[64];
    if (ok && !skip && n_x > 0) {
      tc_fence_after();
      tmem_ld32(lane_base + tm_o(x) + x * 64, *reinterpret_cast<uint32_t(*)[32]>(&own[0]));
      tmem_ld32(lane_base + tm_o(x) + x * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&own[32]));
      tmem_wait_ld();
    }
    if (ok && !skip) {
      s_ml_mine[row] = m_run;
      s_ml_mine[128 + row] = l_run;
      tc_fence_before();
      mbar_arrive(&bar_l);
      ok = wwait(&bar_l, 0);
    }
    const float *s_ml0 = x == 0 ? s_ml_mine : s_ml_other;
    const float *s_ml1 = x == 0 ? s_ml_other : s_ml_mine;
    if (ok && !skip) {
      tc_fence_after();
      const float m0 = s_ml0[row], m1 = s_ml1[row];
      const float l0 = s_ml0[128 + row], l1 = s_ml1[128 + row];
      const float m = fmaxf(m0, m1);
      const float a0 = n0 > 0 ? ex2_approx(m0 - m) : 0.f;
      const float a1 = n1 > 0 ? ex2_approx(m1 - m) : 0.f;
      const float l_tot = l0 * a0 + l1 * a1;
      const float inv_l = 1.f / l_tot;
      const float w_own = (x == 0 ? a0 : a1) * inv_l, w_oth = (x == 0 ? a1 : a0) * inv_l;
      const int n_oth = x == 0 ? n1 : n0;
      uint32_t oth[64];
      if (n_oth > 0) {
        tmem_ld32(lane_base + tm_o(x ^ 1) + x * 64, *reinterpret_cast<uint32_t(*)[32]>(&oth[0]));
        tmem_ld32(lane_base + tm_o(x ^ 1) + x * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&oth[32]));
        tmem_wait_ld();
      }
      // stage the bf16 row half in the (now idle) Q tile, 128-byte swizzled
      // like a TMA tile: 16-byte chunk c of row r sits at chunk c ^ (r mod 8)
      uint8_t *panel = sQ + x * (L::Q_BYTES / 2) + row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k0 = 8 * c + 2 * e;
          float v0 = 0.f, v1 = 0.f;
          if (n_x > 0) {
            v0 = __uint_as_float(own[k0]) * w_own;
            v1 = __uint_as_float(own[k0 + 1]) * w_own;
          }
          if (n_oth > 0) {
            v0 = fmaf(__uint_as_float(oth[k0]), w_oth, v0);
            v1 = fmaf(__uint_as_float(oth[k0 + 1]), w_oth, v1);
          }
          w[e] = pack_bf16x2(v0, v1);
        }
        *reinterpret_cast<uint4 *>(panel + ((c ^ (row & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      if (row_out && p.lse && x == 0)
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.Lc + q_tok] = (m + log2f(l_tot)) * 0.69314718055994531f;
      mbar_arrive(&bar_st[x]);
      ok = wwait(&bar_st[x], 0);
      if (ok && threadIdx.x == (4 + 4 * x) * 32) {
        // one TMA store of this warpgroup's 64-column panel; rows past the
        // q-block or past Lc are not written
        tma_store_4d(&tmO, sQ + x * (L::Q_BYTES / 2), x * 64, h, i * BLK, b);
        bulk_commit();
        bulk_wait_read();
      }
    } else if (skip && row_out) {
      const size_t o_off = ((static_cast<size_t>(b) * p.Lc + q_tok) * p.H + h) * 128 + x * 64;
      uint4 *dst = reinterpret_cast<uint4 *>(p.o + o_off);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[e] = make_uint4(0, 0, 0, 0);
      if (p.lse && x == 0) p.lse[(static_cast<size_t>(b) * p.H + h) * p.Lc + q_tok] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tb, 512);
  }
}

// One thread waits on a barrier that nothing completes; returns after `limit`
// cycles with UF_ETIMEOUT recorded.  Exercises the bounded-wait path.
__global__ void wait_timeout_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    wait_bounded(&bar, 0, &abort_flag, limit);
  }
}

}  // namespace uf
