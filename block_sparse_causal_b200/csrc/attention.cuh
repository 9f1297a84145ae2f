// attention.cuh -- block-sparse chunk-causal attention on tcgen05 tensor cores.
//
// Ultra Flash (papernotes notes), Method, key design 3: attention is computed
// only over the kept (query block, kv block) pairs.  FlashDecoder (xllm-io
// blog), Sec. 3.3: no token mask inside the window (causality by processing
// order); Eq. 4: grouped-query KV heads.
//
// Work item = (batch b, query head h, q-block i): a 128-row Q tile against
// the item's list of n kept kv blocks t = 0 .. n-1, accumulated into one O
// tile with an online softmax.  The grid is persistent: thread block c takes
// items c, c + grid, c + 2 grid, ..., and every pipeline below runs on across
// item boundaries, so the next item's Q and K / V tiles load, and its first
// QK products run, while the current item finishes.
//
// Both products run on the tensor core with the A operand in tensor memory
// and a K-major B operand in shared memory:
//   S_t = Q K_t^T   (Q staged by TMA in shared memory, copied into tensor
//                    memory once per item by the QK issuer with tcgen05.cp;
//                    the FP8 variant's e4m3 Q by the softmax threads)
//   O  += P_t V_t   (P_t written to tensor memory by the softmax; V is stored
//                    transposed in the window, so V_t^T is K-major too)
// Tensor memory (512 columns): S buffers 0 and 1 [0,128) [128,256), O
// [256,384), Q [384,448), P [448,512).  Kept blocks are numbered across the
// items of a thread block (g = blocks of earlier items + t); block g uses S
// buffer g mod 2 and is handled by softmax warpgroup g mod 2.  S_{g+2} is
// issued as soon as the softmax has read S_g into registers (P has its own
// columns).
// Twelve warps:
//   warps 0, 3   TMA producers of the K ring and of the V ring, in block
//                order;
//   warps 1, 2   one issuing thread each (an issuing thread waits for every
//                MMA it issues to be accepted, so two of them keep the tensor
//                core busy): warp 1 issues the QK products, requests each
//                item's Q tile once the staging tile is free, and owns the
//                tensor-memory allocation; warp 2 issues the PV products;
//   warps 4-7    softmax of the even-numbered blocks, warps 8-11 of the odd
//                ones: each thread owns one row (32x32b loads), applies the
//                block's token mask, computes exponentials in the exp2 domain
//                against a reference max and writes P as packed bf16.  The
//                reference max of each row lives in shared memory and is
//                raised only when a block's max exceeds it by more than 2^8 (a
//                stale max is exact: O and the sums share it); raising it
//                rescales O in tensor memory.  Per block: S to registers, the
//                block max, then the turn -- block t waits for block t - 1's
//                decision on the reference, so decisions are taken in block
//                order -- then S's buffer is released and the exponentials
//                run from registers, overlapping those of the other
//                warpgroup's block.  Each warpgroup keeps its own partial row
//                sum relative to the reference it last saw; the two are
//                combined in the item's epilogue, which also hands O back to
//                the PV issuer for the next item and stages the bf16 output
//                in the Q staging tile (free between the copy of the next
//                item's Q and the request for the one after), from which the
//                PV issuer writes it with TMA stores.
#pragma once

#include "uf_device.cuh"

namespace uf {

constexpr int ATTN_THREADS = 384;
constexpr int ATTN_SOFTMAX_THREADS = 256;
constexpr int ATTN_KSTAGE = 3;                   // shared-memory stages of the K ring
constexpr int ATTN_VSTAGE = 3;                   // and of the V ring
// tensor-memory columns
__host__ __device__ constexpr uint32_t tm_s(int x) { return static_cast<uint32_t>(x) * 128u; }
constexpr uint32_t TM_O = 256, TM_Q = 384, TM_P = 448;
constexpr float ATTN_RESCALE_LOG2 = 8.0f;
// Registers per thread: the block is launched with ATTN_LAUNCH_REGS (the
// most 384 threads can have); the producer / issuer warpgroup then releases
// registers to the two softmax warpgroups.  The budgets add up to the launch
// allocation exactly (a raise beyond it would wait forever), and the host
// refuses to launch a build whose kernel was compiled to another count.
constexpr int ATTN_LAUNCH_REGS = 168;
constexpr int ATTN_REGS_IO = 56;
constexpr int ATTN_REGS_SOFTMAX = 224;
static_assert(128 * ATTN_REGS_IO + 256 * ATTN_REGS_SOFTMAX == ATTN_THREADS * ATTN_LAUNCH_REGS,
              "register budgets must add up to the launch allocation");

struct AttnParams {
  const int32_t *meta;
  const int32_t *idx;        // [B, H, nb, k] or NULL (dense)
  const int32_t *cnt;        // [B, H, nb] or NULL
  float *lse;                // [B, H, Lc] or NULL
  __nv_bfloat16 *o;          // [B, Lc, H, D]
  int32_t items;             // B * H * nb
  int32_t H, G, W, Lc, nb, lslot, k;
  uint32_t nb_mul;           // floor(2^32 / nb) (2^32 - 1 for nb = 1): j / nb without a divide
  float scale_log2;          // softmax scale * log2(e) (FP8 variant: times q_scale * k_scale)
  float q_inv_scale;         // FP8 variant: 1 / q_scale
  long long wait_limit;      // bound of every pipeline wait (cycles)
  int32_t *err;              // the window's error word, or NULL (the module's)
  // balanced schedule (NULL: thread block c takes items c, c + grid, ...):
  int32_t *ws_cnt;           // [grid] arrival counters of split items, zero at launch
  float *ws_part;            // [2 * grid][ATTN_PART_FLOATS] partial results
  // optional [2]: every thread block adds its SM clock cycles and its global
  // timer nanoseconds from start to end (the kernel's effective SM clock)
  unsigned long long *clk;
};

// One part of a split item: its unnormalised O (fp32, 128 rows x 128
// channels, stored as [half x][16-byte chunk c][row] so that a warp's stores
// are contiguous), then the reference max m (exp2 domain) and the row sum l
// of each row relative to it.
constexpr int ATTN_PART_O = 128 * 128;
constexpr int ATTN_PART_FLOATS = ATTN_PART_O + 2 * 128;

// Bound of the waits that let copies and MMAs already in flight finish before
// a thread block that gave up exits: never below 2^31 cycles (about a second),
// whatever the pipeline bound, since tensor memory must not be released and
// shared memory must not be abandoned while the hardware still uses them.
__device__ __forceinline__ long long drain_limit(long long wait_limit) {
  return wait_limit > (1LL << 31) ? wait_limit : (1LL << 31);
}

template <int BLK>
struct AttnSmem {
  static constexpr int Q_BYTES = 128 * 256;          // 128 rows x 128 channels, two 64-channel panels
  static constexpr int PANEL = BLK * 128;            // one 64-channel panel of a K tile
  static constexpr int VPANEL = 128 * 128;           // one 64-token panel of a V^T tile (128 channels)
  static constexpr int STAGE = BLK * 256;
  static constexpr int DYN = 1024 + Q_BYTES + (ATTN_KSTAGE + ATTN_VSTAGE) * STAGE;
};

// Logical kv block j (0 <= j < n_valid * nb) of the window -> first row of its
// tile in the cache and its number of true tokens.  Chunk c = j / nb comes
// from a multiply-high by floor(2^32 / nb), which is at most one below the
// quotient, and one correction step; the slot (window_slot) wraps with one
// subtraction.  No divide instruction on the per-block path.
__device__ __forceinline__ void kv_block_coords(int j, int start, int W, int anchor, int nb, uint32_t nb_mul,
                                                int lslot, int blk, int Lc, int &row, int &valid) {
  int c = static_cast<int>(__umulhi(static_cast<uint32_t>(j), nb_mul));
  int r = j - c * nb;
  if (r >= nb) {
    ++c;
    r -= nb;
  }
  const int slot = window_slot(c, start, W, anchor);
  row = slot * lslot + r * blk;
  valid = (r == nb - 1) ? (Lc - (nb - 1) * blk) : blk;
}

// Which items a thread block takes, as a sequence v = 0 .. count - 1.
// Plain: items c, c + grid, c + 2 grid, ...  Balanced: the same for the
// `rounds` full rounds of items (items / grid of them), then the remaining
// items are shared out by position: their positions (item, kept block t),
// item-major, with every item counted at its nominal length n_nom (dense:
// NKV, sparse: the row stride k), are cut into g = min(gridDim.x, positions)
// contiguous ranges of equal length (none empty), one per thread block c < g;
// an item that straddles a range boundary is computed in parts by consecutive
// thread blocks and merged (see the epilogue).  Every role of a thread block
// derives the same sequence from this.
struct AttnSched {
  bool split;
  int n_nom;
  int rounds;                 // items taken in the plain order
  int base;                   // first shared-out item: rounds * gridDim.x (split)
  int g;                      // thread blocks with a range of the shared-out items
  long long T;                // positions of the shared-out items
  long long lo, hi;           // this thread block's positions [lo, hi) among them
  int rbegin, rend;           // shared-out items this thread block visits
  int count;                  // items visited in all
};

__device__ __forceinline__ long long sched_start(long long T, int grid, int c) {
  return static_cast<long long>(c) * T / grid;
}
// The thread block whose range holds position x: the largest c with sched_start(c) <= x.
__device__ __forceinline__ int sched_owner(long long T, int grid, long long x) {
  return static_cast<int>(((x + 1) * grid - 1) / T);
}

__device__ __forceinline__ AttnSched attn_sched(const AttnParams &p, int NKV) {
  AttnSched s;
  const int c = blockIdx.x, grid = gridDim.x;
  s.split = p.ws_part != nullptr && NKV > 0;
  s.n_nom = 0;
  s.g = grid;
  s.T = s.lo = s.hi = 0;
  s.rbegin = s.rend = 0;
  if (!s.split) {
    s.rounds = c < p.items ? (p.items - c + grid - 1) / grid : 0;
    s.base = p.items;
    s.count = s.rounds;
    return s;
  }
  s.n_nom = p.idx ? p.k : NKV;
  s.rounds = p.items / grid;
  s.base = s.rounds * grid;
  s.T = static_cast<long long>(p.items - s.base) * s.n_nom;
  s.g = static_cast<int>(s.T < grid ? s.T : grid);
  if (c < s.g) {
    s.lo = sched_start(s.T, s.g, c);
    s.hi = sched_start(s.T, s.g, c + 1);
    s.rbegin = s.base + static_cast<int>(s.lo / s.n_nom);
    s.rend = s.base + static_cast<int>((s.hi - 1) / s.n_nom) + 1;
  }
  s.count = s.rounds + (s.rend - s.rbegin);
  return s;
}

// The v-th item of this thread block's sequence.
__device__ __forceinline__ int sched_item(const AttnSched &s, int v) {
  return v < s.rounds ? static_cast<int>(blockIdx.x) + v * static_cast<int>(gridDim.x) : s.rbegin + (v - s.rounds);
}

// Workspace slot of the part that thread block c computes of shared-out item
// `item`: a block's first such item in slot 2c, its last (when both are split)
// in 2c + 1.
__device__ __forceinline__ int part_slot(const AttnSched &s, int c, int item) {
  return 2 * c + (item == s.base + static_cast<int>(sched_start(s.T, s.g, c) / s.n_nom) ? 0 : 1);
}

// One work item -- or this thread block's segment of it -- as every role of
// the thread block sees it.
struct AttnItem {
  int i, h, b, g;             // q-block, query head, batch, kv head
  int n;                      // kept kv blocks of the segment (< 1: nothing to compute)
  int t0;                     // the segment's first entry in the item's block list
  int diag;                   // the q-block's own block in the newest chunk
  const int32_t *row_idx;     // its block list, or NULL (dense: block t is t)
  bool empty_out;             // nothing to compute: this thread block writes O = 0, LSE = -inf
  int nparts;                 // thread blocks computing a part of the item (1: not split)
  int part0;                  // the first of them
};

__device__ __forceinline__ AttnItem attn_item(const AttnParams &p, const AttnSched &s, int item, int NKV,
                                              int n_valid) {
  AttnItem it;
  it.i = item % p.nb;
  const int bh = item / p.nb;
  it.h = bh % p.H;
  it.b = bh / p.H;
  it.g = it.h / (p.H / p.G);
  it.diag = (n_valid - 1) * p.nb + it.i;
  it.row_idx = p.idx ? p.idx + static_cast<size_t>(item) * p.k : nullptr;
  it.n = NKV;
  if (it.row_idx) {
    it.n = p.cnt ? __ldg(p.cnt + item) : p.k;
    if (it.n > p.k) it.n = -1;   // malformed row
  }
  if (NKV < 1) it.n = -1;
  it.t0 = 0;
  it.nparts = 1;
  it.part0 = blockIdx.x;
  it.empty_out = it.n < 1;
  if (s.split && item >= s.base) {
    const long long base = static_cast<long long>(item - s.base) * s.n_nom;
    if (it.n < 1) {
      // written once, by the thread block holding the item's first position
      it.empty_out = sched_owner(s.T, s.g, base) == static_cast<int>(blockIdx.x);
      it.n = -1;
    } else {
      // this block's positions of the item, clipped to its true length
      const long long tb = s.lo > base ? s.lo - base : 0;
      const long long te = s.hi - base < it.n ? s.hi - base : it.n;
      it.part0 = sched_owner(s.T, s.g, base);
      it.nparts = sched_owner(s.T, s.g, base + it.n - 1) - it.part0 + 1;
      it.t0 = static_cast<int>(tb);
      it.n = te > tb ? static_cast<int>(te - tb) : 0;
    }
  }
  return it;
}

// Kept block t of a segment -> logical kv block of the window; an
// out-of-range entry reads the diagonal block instead (`bad` tells the
// producer to record the error).
__device__ __forceinline__ int attn_block(const AttnItem &it, int t, int NKV, bool &bad) {
  const int jb = it.row_idx ? __ldg(it.row_idx + it.t0 + t) : it.t0 + t;
  bad = jb < 0 || jb >= NKV;
  return bad ? it.diag : jb;
}

// FP8: the QK product from e4m3 queries and keys (kind::f8f6f4, K = 32 per
// instruction): tmK then maps the window's e4m3 copy of K (one 128-byte panel
// per tile row), and the queries go into tensor memory as e4m3 of q / q_scale.
template <int BLK, bool FP8>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const AttnParams p) {
  using L = AttnSmem<BLK>;
  // start of this thread block, when the launch records its clock
  __shared__ long long s_clk0;
  __shared__ unsigned long long s_ns0;
  if (p.clk && threadIdx.x == 0) {
    s_clk0 = clock64();
    s_ns0 = global_ns();
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sQ = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = sQ + L::Q_BYTES;
  uint8_t *sV = sK + ATTN_KSTAGE * L::STAGE;

  // per-item barriers: Q landed in shared memory / free in tensor memory /
  // copied into tensor memory; O read by the epilogue; (m, l) exchange; O
  // staged by each warpgroup; staging tile read by the output stores
  __shared__ uint64_t bar_qfull, bar_qtfree, bar_q, bar_qcp, bar_ofree, bar_l, bar_st[2], bar_ostore;
  // per-block barriers
  __shared__ uint64_t bar_kfull[ATTN_KSTAGE], bar_kempty[ATTN_KSTAGE];
  __shared__ uint64_t bar_vfull[ATTN_VSTAGE], bar_vempty[ATTN_VSTAGE];
  __shared__ uint64_t bar_s[2], bar_sfree[2], bar_o[2], bar_turn[2], bar_p;
  __shared__ uint64_t bar_fin[2];
  // split items: every softmax thread has written its part / the arrival ticket is known
  __shared__ uint64_t bar_pw, bar_tk;
  __shared__ int32_t s_last;      // this thread block's part of the split item finished last
  __shared__ int32_t s_store[2];  // the output of live item k is written (k mod 2)
  __shared__ float s_mref[128];   // reference max of each row (exp2 domain), published block by block
  __shared__ float s_l[2][128];   // epilogue: each warpgroup's partial row sums
  __shared__ uint32_t s_tbase;
  __shared__ int32_t s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // window state (written by the append call earlier on the stream)
  const int start = __ldcg(p.meta + 0), n_valid = __ldcg(p.meta + 1), anchor = __ldcg(p.meta + 3);
  const bool bad_meta = !window_state_ok(start, n_valid, anchor, p.W);
  const int NKV = bad_meta ? 0 : n_valid * p.nb;
  const AttnSched S = attn_sched(p, NKV);

  if (threadIdx.x == 0) {
    mbar_init(&bar_qfull, 1);
    mbar_init(&bar_qtfree, 1);
    mbar_init(&bar_q, ATTN_SOFTMAX_THREADS);
    mbar_init(&bar_qcp, 1);
    mbar_init(&bar_ofree, ATTN_SOFTMAX_THREADS);
    mbar_init(&bar_l, ATTN_SOFTMAX_THREADS);
    mbar_init(&bar_st[0], ATTN_SOFTMAX_THREADS / 2);
    mbar_init(&bar_st[1], ATTN_SOFTMAX_THREADS / 2);
    mbar_init(&bar_ostore, 1);
    for (int s = 0; s < ATTN_KSTAGE; ++s) {
      mbar_init(&bar_kfull[s], 1);
      mbar_init(&bar_kempty[s], 1);
    }
    for (int s = 0; s < ATTN_VSTAGE; ++s) {
      mbar_init(&bar_vfull[s], 1);
      mbar_init(&bar_vempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_s[s], 1);
      mbar_init(&bar_sfree[s], ATTN_SOFTMAX_THREADS / 2);
      mbar_init(&bar_o[s], 1);
      mbar_init(&bar_turn[s], ATTN_SOFTMAX_THREADS / 2);
      mbar_init(&bar_fin[s], 1);
    }
    mbar_init(&bar_p, ATTN_SOFTMAX_THREADS / 2);
    mbar_init(&bar_pw, ATTN_SOFTMAX_THREADS);
    mbar_init(&bar_tk, 1);
    s_abort = 0;
    fence_mbar_init();
    if (bad_meta && blockIdx.x == 0) record_error(p.err, UF_EBOUNDS);
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

  if (warp < 4) {
    // producers and issuers need few registers: hand them to the softmax
    warpgroup_reg_release<ATTN_REGS_IO>();
    if (warp == 0 || warp == 3) {
      // ------------------------------------------------------------ producers -
      const bool is_v = warp == 3;
      const int nst = is_v ? ATTN_VSTAGE : ATTN_KSTAGE;
      uint64_t *full_bars = is_v ? bar_vfull : bar_kfull;
      uint64_t *empty_bars = is_v ? bar_vempty : bar_kempty;
      uint8_t *ring = is_v ? sV : sK;
      if (lane == 0 && NKV > 0) {
        tma_prefetch_desc(is_v ? &tmV : &tmK);
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int v = 0; v < S.count && ok; ++v) {
          const AttnItem it = attn_item(p, S, sched_item(S, v), NKV, n_valid);
          if (it.n < 1) continue;
          const int zc = it.b * p.G + it.g;
          for (int t = 0; t < it.n; ++t) {
            if (!(ok = wait_bounded(&empty_bars[stage], phase ^ 1u, abort_flag, p.wait_limit, p.err))) break;
            bool bad;
            const int jb = attn_block(it, t, NKV, bad);
            if (bad) record_error(p.err, UF_EBOUNDS);
            int row, valid;
            kv_block_coords(jb, start, p.W, anchor, p.nb, p.nb_mul, p.lslot, BLK, p.Lc, row, valid);
            uint64_t *full = &full_bars[stage];
            mbar_arrive_expect_tx(full, (FP8 && !is_v) ? L::STAGE / 2 : L::STAGE);
            uint8_t *dst = ring + stage * L::STAGE;
            if (FP8 && !is_v) {
              // e4m3 K tile: BLK token rows x 128 channels of one byte, one panel
              tma_load_3d(dst, &tmK, full, 0, row, zc);
            } else if (is_v) {
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
            if (++stage == nst) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) {
          // unwind: let every load still in flight land before the block exits
          int32_t never = 0;
          int s = stage;
          uint32_t ph = phase;
          for (int q = 0; q < nst && q < issued; ++q) {
            if (--s < 0) {
              s = nst - 1;
              ph ^= 1u;
            }
            wait_bounded(&full_bars[s], ph, &never, drain_limit(p.wait_limit), p.err);
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ QK issuer -
      if (lane == 0 && NKV > 0) {
        const uint32_t idesc_qk = idesc_bf16_f32(128, BLK, 0);
        const uint32_t k_base = smem_u32(sK);
        int stage = 0;
        uint32_t phase = 0;
        int uses[2] = {0, 0};   // QK products issued into each S buffer so far
        int kq = 0, g0 = 0, q_loads = 0;
        bool ok = true;
        tma_prefetch_desc(&tmQ);
        // Q tile of a live item -> shared memory (rows past Lc read as zero)
        auto request_q = [&](const AttnItem &a) {
          mbar_arrive_expect_tx(&bar_qfull, L::Q_BYTES);
          tma_load_4d(sQ, &tmQ, &bar_qfull, 0, a.h, a.i * BLK, a.b);
          tma_load_4d(sQ + L::Q_BYTES / 2, &tmQ, &bar_qfull, 64, a.h, a.i * BLK, a.b);
          ++q_loads;
        };
        int v = 0;
        AttnItem it;
        for (; v < S.count; ++v) {
          it = attn_item(p, S, sched_item(S, v), NKV, n_valid);
          if (it.n >= 1) break;
        }
        if (v < S.count) request_q(it);
        while (v < S.count && ok) {
          if (FP8) {
            // the softmax threads have written the item's e4m3 Q into tensor memory
            if (!(ok = wait_bounded(&bar_q, kq & 1, abort_flag, p.wait_limit, p.err))) break;
          } else {
            // once the previous item's QK products have read Q's columns and
            // this item's Q has landed: copy it into tensor memory here, one
            // K = 16 slice per copy, and wait for the copies
            if (kq > 0 && !(ok = wait_bounded(&bar_qtfree, (kq - 1) & 1, abort_flag, p.wait_limit, p.err))) break;
            if (!(ok = wait_bounded(&bar_qfull, kq & 1, abort_flag, p.wait_limit, p.err))) break;
            tc_fence_after();
            const uint32_t q_base = smem_u32(sQ);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tmem_cp_128x256b(tb + TM_Q + kk * 8,
                               sdesc_sw128(q_base + (kk >> 2) * (L::Q_BYTES / 2) + (kk & 3) * 32, 16, 1024));
            mma_commit(&bar_qcp);
            if (!(ok = wait_bounded(&bar_qcp, kq & 1, abort_flag, p.wait_limit, p.err))) break;
          }
          tc_fence_after();
          int v_next = S.count;
          AttnItem nxt;
          const int t_request = it.n > 1 ? 1 : 0;
          for (int t = 0; t < it.n; ++t) {
            const int buf = (g0 + t) & 1;
            // the buffer's previous block has been read by the softmax
            if (uses[buf] > 0 && !(ok = wait_bounded(&bar_sfree[buf], (uses[buf] - 1) & 1, abort_flag, p.wait_limit, p.err)))
              break;
            if (!(ok = wait_bounded(&bar_kfull[stage], phase, abort_flag, p.wait_limit, p.err))) break;
            tc_fence_after();
            const uint32_t k_addr = k_base + stage * L::STAGE;
            if (FP8) {
              // four K = 32 steps over the 128-byte rows of the e4m3 tile
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = sdesc_sw128(k_addr + kk * 32, 16, 1024);
                mma_ts_f8(tb + tm_s(buf), tb + TM_Q + kk * 8, bd, idesc_e4m3_f32(128, BLK), kk > 0);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t bd = sdesc_sw128(k_addr + (kk >> 2) * L::PANEL + (kk & 3) * 32, 16, 1024);
                mma_ts(tb + tm_s(buf), tb + TM_Q + kk * 8, bd, idesc_qk, kk > 0);
              }
            }
            mma_commit(&bar_kempty[stage]);
            mma_commit(&bar_s[buf]);
            ++uses[buf];
            if (++stage == ATTN_KSTAGE) {
              stage = 0;
              phase ^= 1u;
            }
            if (t == t_request) {
              // with the item's first products on their way: the next live
              // item's Q, once the previous item's output stores have read
              // the staging tile
              for (v_next = v + 1; v_next < S.count; ++v_next) {
                nxt = attn_item(p, S, sched_item(S, v_next), NKV, n_valid);
                if (nxt.n >= 1) break;
              }
              if (v_next < S.count) {
                if (kq > 0 && !(ok = wait_bounded(&bar_ostore, (kq - 1) & 1, abort_flag, p.wait_limit, p.err))) break;
                request_q(nxt);
              }
            }
          }
          if (!ok) break;
          // Q's columns are free once every QK product of the item has completed
          mma_commit(&bar_qtfree);
          g0 += it.n;
          ++kq;
          v = v_next;
          it = nxt;
        }
        // every MMA issued by this thread has completed once bar_fin flips, and
        // a Q tile still in flight has landed (the next is requested only after
        // the previous one was copied out, so at most one)
        mma_commit(&bar_fin[0]);
        int32_t never = 0;
        wait_bounded(&bar_fin[0], 0, &never, drain_limit(p.wait_limit), p.err);
        if (!ok && q_loads > 0) wait_bounded(&bar_qfull, (q_loads - 1) & 1, &never, drain_limit(p.wait_limit), p.err);
      }
    } else {
      // ------------------------------------------------------------ PV issuer -
      if (lane == 0 && NKV > 0) {
        const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0);
        const uint32_t v_base = smem_u32(sV);
        int stage = 0;
        uint32_t phase = 0;
        int kq = 0, g0 = 0;
        bool ok = true;
        // output of live item number k: once its epilogue has read O and both
        // warpgroups have staged their halves, one TMA store per 64-column
        // panel (rows past the q-block or past Lc are not written); the
        // staging tile is released once the stores have read it
        auto store_output = [&](const AttnItem &a, int k) -> bool {
          if (!wait_bounded(&bar_ofree, k & 1, abort_flag, p.wait_limit, p.err)) return false;
          if (!wait_bounded(&bar_st[0], k & 1, abort_flag, p.wait_limit, p.err)) return false;
          if (!wait_bounded(&bar_st[1], k & 1, abort_flag, p.wait_limit, p.err)) return false;
          if (s_store[k & 1]) {   // (not for a part of a split item that another block merges)
            tma_store_4d(&tmO, sQ, 0, a.h, a.i * BLK, a.b);
            tma_store_4d(&tmO, sQ + L::Q_BYTES / 2, 64, a.h, a.i * BLK, a.b);
            bulk_commit();
            bulk_wait_read();
          }
          mbar_arrive(&bar_ostore);
          return true;
        };
        AttnItem prev;
        for (int v = 0; v < S.count && ok; ++v) {
          const AttnItem it = attn_item(p, S, sched_item(S, v), NKV, n_valid);
          if (it.n < 1) continue;
          // the previous item's output leaves (and its epilogue has read O)
          if (kq > 0 && !(ok = store_output(prev, kq - 1))) break;
          for (int t = 0; t < it.n; ++t) {
            const int gb = g0 + t;
            if (!(ok = wait_bounded(&bar_p, gb & 1, abort_flag, p.wait_limit, p.err))) break;
            if (!(ok = wait_bounded(&bar_vfull[stage], phase, abort_flag, p.wait_limit, p.err))) break;
            tc_fence_after();
            const uint32_t v_addr = v_base + stage * L::STAGE;
#pragma unroll
            for (int kk = 0; kk < BLK / 16; ++kk) {
              const uint64_t bd = sdesc_sw128(v_addr + (kk >> 2) * L::VPANEL + (kk & 3) * 32, 16, 1024);
              mma_ts(tb + TM_O, tb + TM_P + kk * 8, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bar_vempty[stage]);
            mma_commit(&bar_o[gb & 1]);
            if (++stage == ATTN_VSTAGE) {
              stage = 0;
              phase ^= 1u;
            }
          }
          prev = it;
          g0 += it.n;
          ++kq;
        }
        if (ok && kq > 0) ok = store_output(prev, kq - 1);
        mma_commit(&bar_fin[1]);
        int32_t never = 0;
        wait_bounded(&bar_fin[1], 0, &never, drain_limit(p.wait_limit), p.err);
      }
    }
  } else {
    warpgroup_reg_raise<ATTN_REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax ---
    const int x = (warp - 4) >> 2;              // handles blocks g with g mod 2 == x
    const int wq = warp & 3;                    // tensor-memory lane quarter of this warp
    const int row = wq * 32 + lane;             // row of the Q tile
    const uint32_t lane_base = tb + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_col = tm_s(x);
    const float c_log2 = p.scale_log2;
    const uint64_t c2 = f2_pack(c_log2, c_log2);
    // tcgen05.ld / st are warp-collective: every wait result is made warp-uniform
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, p.wait_limit, p.err));
    };
    // an item with nothing to compute: zero output, -inf log-sum-exp
    auto write_empty = [&](const AttnItem &a) {
      const int q_tok = a.i * BLK + row;
      if (row < BLK && q_tok < p.Lc) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((static_cast<size_t>(a.b) * p.Lc + q_tok) * p.H + a.h) * 128 +
                                               x * 64);
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e] = make_uint4(0, 0, 0, 0);
        if (p.lse && x == 0) p.lse[(static_cast<size_t>(a.b) * p.H + a.h) * p.Lc + q_tok] = -INFINITY;
      }
      if (threadIdx.x == 128) record_error(p.err, UF_EBOUNDS);
    };
    // first item at or after `from` (in this block's sequence) with blocks to
    // compute; the empty ones on the way are written here
    auto next_live = [&](int from, AttnItem &out) -> int {
      for (int j = from; j < S.count; ++j) {
        out = attn_item(p, S, sched_item(S, j), NKV, n_valid);
        if (out.n >= 1) return j;
        if (out.empty_out) write_empty(out);
      }
      return S.count;
    };
    // Q of live item number kq -> tensor memory, once it has landed and the
    // previous item's QK products have completed: this warpgroup copies
    // channels [64x, 64x + 64) of its row out of the 128-byte-swizzled tile
    // (32 columns of packed bf16 pairs, the A-operand layout of the QK MMA)
    auto load_q = [&](int kq) -> bool {
      if (!wwait(&bar_qfull, kq & 1)) return false;
      if (kq > 0 && !wwait(&bar_qtfree, (kq - 1) & 1)) return false;
      tc_fence_after();
      uint32_t qw[32];
      const uint8_t *src = sQ + x * (L::Q_BYTES / 2) + row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4 *>(src + ((c ^ (row & 7)) * 16));
        qw[4 * c] = v.x;
        qw[4 * c + 1] = v.y;
        qw[4 * c + 2] = v.z;
        qw[4 * c + 3] = v.w;
      }
      if (FP8) {
        // channels [64x, 64x + 64) as e4m3 of q / q_scale: 16 columns of four
        uint32_t q8[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qw[2 * e]));
          const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qw[2 * e + 1]));
          const float sc = p.q_inv_scale;
          q8[e] = pack_e4m3x4(a.x * sc, a.y * sc, c.x * sc, c.y * sc);
        }
        tmem_st16(lane_base + TM_Q + 16 * x, q8);
      } else {
        tmem_st32(lane_base + TM_Q + 32 * x, qw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_q);
      return true;
    };

    AttnItem cur;
    int v = next_live(0, cur);
    bool ok = v >= S.count || !FP8 || load_q(0);
    int ks = 0;           // parts of split items written so far (parity of bar_pw / bar_tk)
    int kq = 0, g0 = 0;   // live items and kept blocks of this thread block so far
    while (v < S.count && ok) {
      const int item = sched_item(S, v);
      const int n = cur.n;
      float m_run = -INFINITY;   // reference max this warpgroup last saw
      float l_run = 0.f;         // this warpgroup's partial row sum, relative to m_run
      int n_mine = 0;
      for (int t = x ^ (g0 & 1); t < n; t += 2) {
        const int gb = g0 + t;   // this warpgroup's (gb >> 1)-th block
        ++n_mine;
        bool bad;
        const int jb = attn_block(cur, t, NKV, bad);
        int krow, valid;
        kv_block_coords(jb, start, p.W, anchor, p.nb, p.nb_mul, p.lslot, BLK, p.Lc, krow, valid);
        if (!(ok = wwait(&bar_s[x], (gb >> 1) & 1))) break;
        tc_fence_after();
        const bool full = valid == BLK;
        uint32_t s[BLK];
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c)
          tmem_ld32(lane_base + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
        tmem_wait_ld();
        // block max over the block's true tokens
        float mx;
        {
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
        // block t - 1 (the other warpgroup) has settled the reference max:
        // adopt it, bringing this warpgroup's partial sum to the same reference
        if (t > 0) {
          if (!(ok = wwait(&bar_turn[x ^ 1], ((gb - 1) >> 1) & 1))) break;
          const float m_ref = s_mref[row];
          if (m_ref != m_run) {
            l_run *= ex2_approx(m_run - m_ref);
            m_run = m_ref;
          }
        }
        // raise the reference only when the block max exceeds it by more than 2^8
        bool o_ready = false;    // PV of block gb - 1 known to have completed
        const float m_new = fmaxf(m_run, mx * c_log2);
        if (__any_sync(0xffffffffu, m_new > m_run + ATTN_RESCALE_LOG2)) {
          const float factor = ex2_approx(m_run - m_new);
          l_run *= factor;
          if (t > 0) {
            // O holds the item's PV products up to block gb - 1: wait for the
            // last of them, then rescale
            if (!(ok = wwait(&bar_o[(gb - 1) & 1], ((gb - 1) >> 1) & 1))) break;
            o_ready = true;
            tc_fence_after();
            const uint64_t f2 = f2_pack(factor, factor);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(lane_base + TM_O + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                float lo, hi;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), f2), lo, hi);
                o[2 * e] = __float_as_uint(lo);
                o[2 * e + 1] = __float_as_uint(hi);
              }
              tmem_st32(lane_base + TM_O + 32 * c, o);
            }
            tmem_wait_st();
          }
          m_run = m_new;
        }
        // publish the reference for block t + 1, hand over the turn and release
        // the S buffer (held in registers from here on)
        s_mref[row] = m_run;
        tc_fence_before();
        mbar_arrive(&bar_turn[x]);
        mbar_arrive(&bar_sfree[x]);
        // P = exp2(s * c - m): full-block and masked (partial last block of a
        // chunk) cases are separate loops: a per-element mask test inside the
        // unrolled loop costs two ALU instructions per element
        const uint64_t negm2 = f2_pack(-m_run, -m_run);
        uint32_t pk[BLK / 2];
        uint64_t acc2[4] = {0, 0, 0, 0};
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
        {
          float a0, a1;
          f2_unpack(f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3])), a0, a1);
          l_run += a0 + a1;
        }
        // P's columns are free once the PV of block gb - 1 has read them (for
        // the item's first block, the previous item's epilogue waited for it)
        if (t > 0 && !o_ready) {
          if (!(ok = wwait(&bar_o[(gb - 1) & 1], ((gb - 1) >> 1) & 1))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < BLK / 64; ++c)
          tmem_st32(lane_base + TM_P + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * c]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_p);
      }
      if (!ok) break;
      // the next live item's Q goes into tensor memory now, so that its first
      // QK products run during this item's epilogue
      AttnItem nxt;
      const int v_next = next_live(v + 1, nxt);
      if (FP8 && v_next < S.count && !(ok = load_q(kq + 1))) break;
      // ---------------------------------------------------------- epilogue --
      // every PV of the item has completed once its last one has (one issuing
      // thread, completions in order)
      const int gl = g0 + n - 1;
      if (!(ok = wwait(&bar_o[gl & 1], (gl >> 1) & 1))) break;
      // the reference after the item's last decision; each warpgroup's sum
      // brought to it
      mbar_arrive(&bar_l);
      if (!(ok = wwait(&bar_l, 0))) break;
      float m_fin = s_mref[row];
      s_l[x][row] = n_mine > 0 ? l_run * ex2_approx(m_run - m_fin) : 0.f;
      mbar_arrive(&bar_l);
      if (!(ok = wwait(&bar_l, 1))) break;
      float l_tot = s_l[0][row] + s_l[1][row];
      tc_fence_after();
      // this warpgroup's half of the O row; O then goes back to the PV issuer
      uint32_t o[64];
      tmem_ld32(lane_base + TM_O + x * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
      tmem_ld32(lane_base + TM_O + x * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar_ofree);
      bool store = true;
      if (cur.nparts > 1) {
        // a part of a split item: (O relative to m_fin, m_fin, l_tot) goes to
        // the workspace; the thread block whose part arrives last merges all
        // parts (log-sum-exp: every part brought to the largest reference) and
        // writes the output.  No thread block waits for another.
        float *part = p.ws_part + static_cast<size_t>(part_slot(S, blockIdx.x, item)) * ATTN_PART_FLOATS;
        float4 *po = reinterpret_cast<float4 *>(part) + x * 16 * 128 + row;
#pragma unroll
        for (int c = 0; c < 16; ++c)
          po[c * 128] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]),
                                    __uint_as_float(o[4 * c + 2]), __uint_as_float(o[4 * c + 3]));
        if (x == 0) {
          part[ATTN_PART_O + row] = m_fin;
          part[ATTN_PART_O + 128 + row] = l_tot;
        }
        // every thread's stores precede thread 128's fence (the barrier orders
        // them within the block; the fence is cumulative), which precedes the
        // arrival count; the part that counts last fences again before its
        // threads read the other parts (from L2)
        mbar_arrive(&bar_pw);
        if (threadIdx.x == 128) {
          int32_t last = 0;
          if (wait_bounded(&bar_pw, ks & 1, abort_flag, p.wait_limit, p.err)) {
            __threadfence();
            last = atomicAdd(p.ws_cnt + cur.part0, 1) == cur.nparts - 1;
            if (last) __threadfence();
          }
          s_last = last;
          mbar_arrive(&bar_tk);
        }
        if (!(ok = wwait(&bar_tk, ks & 1))) break;
        ++ks;
        store = s_last != 0;
        if (store) {
          // every part, this block's included, in thread-block order from the
          // workspace: the merged result does not depend on which part
          // finished last
          float m_all = m_fin;
          for (int q = cur.part0; q < cur.part0 + cur.nparts; ++q)
            if (q != static_cast<int>(blockIdx.x))
              m_all = fmaxf(m_all, __ldcg(p.ws_part + static_cast<size_t>(part_slot(S, q, item)) * ATTN_PART_FLOATS +
                                          ATTN_PART_O + row));
          float l_all = 0.f;
#pragma unroll
          for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(0.f);
          for (int q = cur.part0; q < cur.part0 + cur.nparts; ++q) {
            const float *pq = p.ws_part + static_cast<size_t>(part_slot(S, q, item)) * ATTN_PART_FLOATS;
            const float fq = ex2_approx(__ldcg(pq + ATTN_PART_O + row) - m_all);
            l_all = fmaf(__ldcg(pq + ATTN_PART_O + 128 + row), fq, l_all);
            const float4 *pq4 = reinterpret_cast<const float4 *>(pq) + x * 16 * 128 + row;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float4 v = __ldcg(pq4 + c * 128);
              o[4 * c] = __float_as_uint(fmaf(v.x, fq, __uint_as_float(o[4 * c])));
              o[4 * c + 1] = __float_as_uint(fmaf(v.y, fq, __uint_as_float(o[4 * c + 1])));
              o[4 * c + 2] = __float_as_uint(fmaf(v.z, fq, __uint_as_float(o[4 * c + 2])));
              o[4 * c + 3] = __float_as_uint(fmaf(v.w, fq, __uint_as_float(o[4 * c + 3])));
            }
          }
          m_fin = m_all;
          l_tot = l_all;
        }
      }
      if (threadIdx.x == 128) s_store[kq & 1] = store;   // read by the PV issuer after bar_st
      // (bf16 path: the QK issuer's copy of the next item's Q out of the staging
      // tile has completed)
      if (!FP8 && v_next < S.count && !(ok = wwait(&bar_qcp, (kq + 1) & 1))) break;
      // this warpgroup's 64-column half of the bf16 row -> the staging tile
      // (the next item's Q has left it), 128-byte swizzled like a TMA tile:
      // 16-byte chunk c of row r at chunk c ^ (r mod 8)
      if (store) {
        const float inv_l = 1.f / l_tot;
        uint8_t *panel = sQ + x * (L::Q_BYTES / 2) + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = 8 * c + 2 * e;
            w[e] = pack_bf16x2(__uint_as_float(o[k0]) * inv_l, __uint_as_float(o[k0 + 1]) * inv_l);
          }
          *reinterpret_cast<uint4 *>(panel + ((c ^ (row & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // (the PV issuer writes the tile out)
      fence_proxy_async_smem();
      mbar_arrive(&bar_st[x]);
      const int q_tok = cur.i * BLK + row;
      if (store && row < BLK && q_tok < p.Lc && p.lse && x == 0)
        p.lse[(static_cast<size_t>(cur.b) * p.H + cur.h) * p.Lc + q_tok] = (m_fin + log2f(l_tot)) * 0.69314718055994531f;
      g0 += n;
      ++kq;
      v = v_next;
      cur = nxt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tb, 512);
  }
  if (p.clk && threadIdx.x == 0) {
    atomicAdd(p.clk, static_cast<unsigned long long>(clock64() - s_clk0));
    atomicAdd(p.clk + 1, global_ns() - s_ns0);
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
