// attention.cuh -- block-sparse chunk-causal attention on tcgen05 tensor cores.
//
// Ultra Flash (papernotes notes), Method, key design 3: attention is computed
// only over the kept (query block, kv block) pairs.  FlashDecoder (xllm-io
// blog), Sec. 3.3: no token mask inside the window (causality by processing
// order); Eq. 4: grouped-query KV heads.
//
// One thread block = one work item (batch b, query head h, q-block i): a
// 128-row Q tile against the item's list of kept kv blocks.  Six warps:
//   warp 0     TMA producer: Q tile once, then K_j / V_j tiles gathered by the
//              block list into a ring of NSTAGE shared-memory stages, in the
//              order the MMA warp consumes them (K0, K1, V0, K2, V1, ...);
//   warp 1     allocates tensor memory; one thread issues every tcgen05.mma:
//              S_j = Q K_j^T (SS, both operands K-major, 128-byte swizzle) into
//              one of two S buffers, and O += P_j V_j (TS: P read from tensor
//              memory, V an MN-major shared-memory operand);
//   warps 2-5  softmax: each thread owns one row of the tile, reads its S row
//              from tensor memory (32x32b loads), applies the block's token
//              mask, keeps a running max / sum in the exp2 domain, writes P as
//              packed bf16 back to tensor memory, and rescales O only when the
//              running max grew by more than 2^8 (stale max otherwise; exact
//              because O and the sum share the same reference).
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O [256,384)
// P0 [384,448) P1 [448,512).  Double-buffered S and P let the tensor core
// compute PV_{j-1} and S_{j+1} while the softmax works on S_j.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int ATTN_THREADS = 192;
constexpr int ATTN_NSTAGE = 6;
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_P0 = 384, TM_P1 = 448;
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
  static constexpr int PANEL = BLK * 128;            // one 64-column panel of a K/V tile
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
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem<BLK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + L::Q_BYTES;

  __shared__ uint64_t bar_q, bar_fin;
  __shared__ uint64_t bar_full[ATTN_NSTAGE], bar_empty[ATTN_NSTAGE];
  __shared__ uint64_t bar_s[2], bar_p[2], bar_o[2];
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
    mbar_init(&bar_fin, 1);
    for (int s = 0; s < ATTN_NSTAGE; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_s[s], 1);
      mbar_init(&bar_p[s], 128);
      mbar_init(&bar_o[s], 1);
    }
    s_abort = 0;
    fence_mbar_init();
    if (skip) record_error(UF_EBOUNDS);
  }
  if (warp == 1) {
    tmem_alloc(&s_tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tbase;
  volatile int32_t *abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0 && !skip) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q, L::Q_BYTES);
      tma_load_4d(sQ, &tmQ, &bar_q, 0, h, i * BLK, b);
      tma_load_4d(sQ + L::Q_BYTES / 2, &tmQ, &bar_q, 64, h, i * BLK, b);
      const int zc = b * p.G + g;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int j = 0; j <= n && ok; ++j) {
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const int t = which == 0 ? j : j - 1;
          if ((which == 0 && j >= n) || (which == 1 && j < 1)) continue;
          if (!wait_bounded(&bar_empty[stage], phase ^ 1u, abort_flag, p.wait_limit)) {
            ok = false;
            break;
          }
          int jb = row_idx ? __ldg(row_idx + t) : t;
          if (jb < 0 || jb >= NKV) {
            record_error(UF_EBOUNDS);
            jb = diag;
          }
          int row, valid;
          kv_block_coords(jb, start, p.W, p.nb, p.lslot, BLK, p.Lc, row, valid);
          mbar_arrive_expect_tx(&bar_full[stage], L::STAGE);
          const CUtensorMap *m = which == 0 ? &tmK : &tmV;
          uint8_t *dst = sKV + stage * L::STAGE;
          tma_load_3d(dst, m, &bar_full[stage], 0, row, zc);
          tma_load_3d(dst + L::PANEL, m, &bar_full[stage], 64, row, zc);
          ++issued;
          if (++stage == ATTN_NSTAGE) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // unwind: let every load still in flight land before the block exits
        int s = stage;
        uint32_t ph = phase;
        for (int q = 0; q < ATTN_NSTAGE && q < issued; ++q) {
          if (--s < 0) {
            s = ATTN_NSTAGE - 1;
            ph ^= 1u;
          }
          int32_t never = 0;
          wait_bounded(&bar_full[s], ph, &never, p.wait_limit);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA -------
    if (lane == 0 && !skip) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, BLK, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 1);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t kv_addr = smem_u32(sKV);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = wait_bounded(&bar_q, 0, abort_flag, p.wait_limit);
      if (ok) tc_fence_after();
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n) {
          if (!(ok = wait_bounded(&bar_full[stage], phase, abort_flag, p.wait_limit))) break;
          tc_fence_after();
          const uint32_t k_addr = kv_addr + stage * L::STAGE;
          const uint32_t d_tmem = tb + ((j & 1) ? TM_S1 : TM_S0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * (L::Q_BYTES / 2) + off, 16, 1024);
            const uint64_t bd = sdesc_sw128(k_addr + (kk >> 2) * L::PANEL + off, 16, 1024);
            mma_ss(d_tmem, ad, bd, idesc_qk, kk > 0);
          }
          mma_commit(&bar_empty[stage]);
          mma_commit(&bar_s[j & 1]);
          if (++stage == ATTN_NSTAGE) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (j >= 1) {
          const int jj = j - 1;
          if (!(ok = wait_bounded(&bar_p[jj & 1], (jj >> 1) & 1, abort_flag, p.wait_limit))) break;
          if (!(ok = wait_bounded(&bar_full[stage], phase, abort_flag, p.wait_limit))) break;
          tc_fence_after();
          const uint32_t v_addr = kv_addr + stage * L::STAGE;
          const uint32_t a_tmem = tb + ((jj & 1) ? TM_P1 : TM_P0);
#pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(v_addr + kk * 2048, L::PANEL, 1024);
            mma_ts(tb + TM_O, a_tmem + kk * 8, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar_empty[stage]);
          mma_commit(&bar_o[jj & 1]);
          if (++stage == ATTN_NSTAGE) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every MMA issued by this thread has completed once bar_fin flips
      mma_commit(&bar_fin);
      int32_t never = 0;
      wait_bounded(&bar_fin, 0, &never, p.wait_limit);
    }
  } else {
    // ------------------------------------------------------------ softmax ---
    const int wq = warp & 3;                    // tensor-memory lane quarter of this warp
    const int row = wq * 32 + lane;             // row of the Q tile
    const uint32_t lane_base = tb + (static_cast<uint32_t>(wq * 32) << 16);
    const int q_tok = i * BLK + row;
    const bool row_out = row < BLK && q_tok < p.Lc;
    float m_run = -INFINITY, l_run = 0.f;
    // tcgen05.ld / st are warp-collective: every wait result is made warp-uniform
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, p.wait_limit));
    };
    bool ok = !skip;
    for (int j = 0; j < n && ok; ++j) {
      int jb = row_idx ? __ldg(row_idx + j) : j;
      if (jb < 0 || jb >= NKV) jb = diag;
      int krow, valid;
      kv_block_coords(jb, start, p.W, p.nb, p.lslot, BLK, p.Lc, krow, valid);
      if (!(ok = wwait(&bar_s[j & 1], (j >> 1) & 1))) break;
      tc_fence_after();
      uint32_t s[BLK];
      const uint32_t s_col = (j & 1) ? TM_S1 : TM_S0;
#pragma unroll
      for (int c = 0; c < BLK / 32; ++c) tmem_ld32(lane_base + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BLK; ++c) {
        const float v = (c < valid) ? __uint_as_float(s[c]) : -INFINITY;
        mx = fmaxf(mx, v);
      }
      const float m_new = fmaxf(m_run, mx * p.scale_log2);
      const bool need = m_new > m_run + ATTN_RESCALE_LOG2;
      float m_use = m_run;
      if (__any_sync(0xffffffffu, need)) {
        m_use = m_new;
        const float factor = ex2_approx(m_run - m_new);
        l_run *= factor;
        if (j > 0) {
          // O holds PV_0..PV_{j-1}: rescale it once PV_{j-1} has landed
          if (!(ok = wwait(&bar_o[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + TM_O + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lane_base + TM_O + 32 * c, o);
          }
        }
      }
      const float neg_m = -m_use;
      float rs = 0.f;
      uint32_t pk[BLK / 2];
#pragma unroll
      for (int c = 0; c < BLK / 2; ++c) {
        const float a = (2 * c < valid) ? ex2_approx(fmaf(__uint_as_float(s[2 * c]), p.scale_log2, neg_m)) : 0.f;
        const float bq = (2 * c + 1 < valid) ? ex2_approx(fmaf(__uint_as_float(s[2 * c + 1]), p.scale_log2, neg_m)) : 0.f;
        rs += a + bq;
        pk[c] = pack_bf16x2(a, bq);
      }
      l_run += rs;
      m_run = m_use;
      if (j >= 2) {
        // P buffer (j & 1) is free once PV_{j-2} has completed
        if (!(ok = wwait(&bar_o[j & 1], ((j - 2) >> 1) & 1))) break;
        tc_fence_after();
      }
      const uint32_t p_col = (j & 1) ? TM_P1 : TM_P0;
#pragma unroll
      for (int c = 0; c < BLK / 64; ++c) tmem_st32(lane_base + p_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * c]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p[j & 1]);
    }
    // ---------------------------------------------------------- epilogue ----
    const size_t o_off = ((static_cast<size_t>(b) * p.Lc + q_tok) * p.H + h) * 128;
    if (ok && !skip) ok = wwait(&bar_o[(n - 1) & 1], ((n - 1) >> 1) & 1);
    if (ok && !skip) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_base + TM_O + 32 * c, o);
        tmem_wait_ld();
        if (row_out) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
          uint4 *dst = reinterpret_cast<uint4 *>(p.o + o_off + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (row_out && p.lse)
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.Lc + q_tok] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    } else if (skip && row_out) {
      uint4 *dst = reinterpret_cast<uint4 *>(p.o + o_off);
#pragma unroll
      for (int e = 0; e < 16; ++e) dst[e] = make_uint4(0, 0, 0, 0);
      if (p.lse) p.lse[(static_cast<size_t>(b) * p.H + h) * p.Lc + q_tok] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
