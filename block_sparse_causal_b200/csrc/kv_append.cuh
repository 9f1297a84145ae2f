// kv_append.cuh -- rolling-window append / evict of one chunk's K and V.
//
// FlashDecoder (xllm-io blog), Algorithm 1: after each frame the cache is the
// tail (W - 1) frames of the old cache followed by the new frame's K/V; Eq. 4
// fixes the cache layout B x G x (W L) x D_h.  Ultra Flash (papernotes notes),
// key design 4: reuse of the last denoising step's KV (here: overwrite the
// newest chunk) and adaptive cropping of the SR KV window (here: keep_chunks).
//
// One thread block per (block r of the chunk, KV head g, batch b), 256
// threads.  K is copied row for row (16 token lanes x 16 sixteen-byte column
// chunks of a 256-byte token row: every warp moves two whole rows per
// instruction on both sides) and reduced into the slot's pooled-K row (fp32
// mean over the block's true tokens), which the block-mask call reads instead
// of re-reading the window.  V is stored transposed (head dim outermost,
// tokens contiguous) so that the attention's PV product reads it as a K-major
// operand: each thread loads an 8-token x 8-channel bf16 tile, transposes it
// in registers with byte permutes and writes 8 sixteen-byte token runs, so
// each warp writes two contiguous 256-byte runs per instruction.  Each block
// counts itself out when done (it read the old window state at its start);
// the last one commits the new state to meta, so no block can observe a
// half-updated window, and no block waits for its own writes to drain.
//
// With RoPE (uf_kv_append_rope) each K row is rotated at its stream position
// before it is stored and pooled.  Rotary scores depend only on position
// differences, so stream positions give the same scores as the positions
// relative to the current window that the method assigns (FlashDecoder, long
// video decoding), and a stored K never needs rotating again when the window
// slides.
#pragma once

#include "uf_device.cuh"

namespace uf {

// ------------------------------------------------------------ tile order ----
// Ultra Flash (papernotes notes), Method, key design 3: the spatio-temporal
// token grid is cut into non-overlapping (2, 8, 8) blocks.  A chunk's tokens
// form a (T, Hg, Wg) grid in row-major order; the tiled order takes tiles of
// (bt, by, bx) in row-major tile order and the tokens inside each tile in
// row-major order, with the tiles at the grid's far edges clipped.
struct TileGrid {
  int32_t T, Hg, Wg, bt, by, bx;
};

// Row-major token index -> position in the tiled order.
__host__ __device__ __forceinline__ int32_t tile_pos(const TileGrid &g, int32_t token) {
  const int32_t HW = g.Hg * g.Wg;
  const int32_t t = token / HW, rem = token - t * HW;
  const int32_t y = rem / g.Wg, x = rem - y * g.Wg;
  const int32_t ti = t / g.bt, yi = y / g.by, xi = x / g.bx;
  const int32_t st = min(g.bt, g.T - ti * g.bt), sy = min(g.by, g.Hg - yi * g.by), sx = min(g.bx, g.Wg - xi * g.bx);
  // tokens before the tile: earlier slabs, earlier bands of this slab, earlier tiles of this band
  const int32_t before = ti * g.bt * HW + st * yi * g.by * g.Wg + st * sy * xi * g.bx;
  return before + ((t - ti * g.bt) * sy + (y - yi * g.by)) * sx + (x - xi * g.bx);
}

// Position in the tiled order -> row-major token index (inverse of tile_pos):
// every slab but the last holds bt * Hg * Wg tokens, every band of a slab but
// the last st * by * Wg, every tile of a band but the last st * sy * bx.
__host__ __device__ __forceinline__ int32_t tile_token(const TileGrid &g, int32_t p) {
  const int32_t HW = g.Hg * g.Wg;
  const int32_t ti = p / (g.bt * HW);
  int32_t r = p - ti * g.bt * HW;
  const int32_t st = min(g.bt, g.T - ti * g.bt);
  const int32_t yi = r / (st * g.by * g.Wg);
  r -= yi * st * g.by * g.Wg;
  const int32_t sy = min(g.by, g.Hg - yi * g.by);
  const int32_t xi = r / (st * sy * g.bx);
  r -= xi * st * sy * g.bx;
  const int32_t sx = min(g.bx, g.Wg - xi * g.bx);
  const int32_t dt = r / (sy * sx);
  r -= dt * sy * sx;
  const int32_t dy = r / sx, dx = r - dy * sx;
  return (ti * g.bt + dt) * HW + (yi * g.by + dy) * g.Wg + xi * g.bx + dx;
}

struct AppendParams {
  const __nv_bfloat16 *k_new;  // [B, Lc, G, D]
  const __nv_bfloat16 *v_new;
  __nv_bfloat16 *k;            // [B, G, W*Lslot, D]
  __nv_bfloat16 *v;            // [B, G, D, W*Lslot] (transposed)
  float *kpool;                // [B, G, W*nb, D]
  int32_t *meta;               // {start, n_valid, counter, reserved}
  int32_t G, W, Lc, nb, lslot, keep, replace;
  int32_t make_anchor;         // pin this chunk as the window's anchor (window empty)
  long long pos0;              // RoPE variant: stream position of the chunk's first token
  TileGrid grid;               // tiled variant: the chunk's grid and tile
  uint8_t *k8;                 // FP8 variant: [B, G, W*Lslot, D] e4m3 copy of K (same slots)
  float k8_inv_scale;          // FP8 variant: 1 / k_scale
  double log2_base;
  int32_t *err;                // the window's error word, or NULL (the module's)
};

// New window state and the slot the chunk goes to (see uf_kv_append).  With
// an anchor (window_slot), the rolling part is a ring of W - 1 slots holding
// n - 1 chunks, keep counts the anchor, and the anchor itself is never
// evicted or cropped.
__host__ __device__ __forceinline__ void append_plan(int32_t start, int32_t n, int32_t W, int32_t keep,
                                                     int32_t replace, int32_t anchor, int32_t make_anchor,
                                                     int32_t &slot, int32_t &start2, int32_t &n2,
                                                     int32_t &anchor2) {
  if (make_anchor) {          // the first chunk of an anchored window
    slot = W - 1;
    start2 = 0;
    n2 = 1;
    anchor2 = 1;
    return;
  }
  anchor2 = anchor;
  const int32_t a = anchor ? 1 : 0;
  const int32_t R = W - a, nr = n - a, keep_r = keep - a;   // ring size, ring chunks, ring keep
  if (replace && n > 0) {
    slot = nr > 0 ? (start + nr - 1) % R : W - 1;             // the newest chunk (the anchor when alone)
    start2 = start;
    n2 = n;
  } else {
    slot = (start + nr) % R;   // free: at most keep_r - 1 <= R - 1 ring chunks survive eviction
    const int32_t evict = max(0, nr + 1 - keep_r);
    start2 = (start + evict) % R;
    n2 = n - evict + 1;
  }
  if (n2 - a > keep_r) {      // crop (replace with a smaller keep_chunks)
    start2 = (start2 + (n2 - a - keep_r)) % R;
    n2 = keep_r + a;
  }
}

// In-register transpose of an 8x8 tile of 16-bit values: in[r] holds row r
// (8 values, lowest address first); out[c] receives column c.
__device__ __forceinline__ void transpose8x8_b16(const uint4 (&in)[8], uint4 (&out)[8]) {
  uint32_t w[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    w[r][0] = in[r].x;
    w[r][1] = in[r].y;
    w[r][2] = in[r].z;
    w[r][3] = in[r].w;
  }
  // stage 1: 2x2 blocks of 16-bit values between row pairs (r, r+1)
#pragma unroll
  for (int r = 0; r < 8; r += 2)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t a = w[r][c], b = w[r + 1][c];
      w[r][c] = __byte_perm(a, b, 0x5410);       // (a.lo, b.lo)
      w[r + 1][c] = __byte_perm(a, b, 0x7632);   // (a.hi, b.hi)
    }
  // stage 2: 2x2 blocks of 32-bit words between rows (r, r+2)
#pragma unroll
  for (int r0 = 0; r0 < 8; r0 += 4)
#pragma unroll
    for (int r = r0; r < r0 + 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        const uint32_t t = w[r][c + 1];
        w[r][c + 1] = w[r + 2][c];
        w[r + 2][c] = t;
      }
  // stage 3: 2x2 blocks of 64-bit pairs between rows (r, r+4)
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    uint32_t t0 = w[r][2], t1 = w[r][3];
    w[r][2] = w[r + 4][0];
    w[r][3] = w[r + 4][1];
    w[r + 4][0] = t0;
    w[r + 4][1] = t1;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) out[c] = make_uint4(w[c][0], w[c][1], w[c][2], w[c][3]);
}

// MODE: APPEND_PLAIN, APPEND_ROPE (K rotated), APPEND_TILED (K / V gathered in
// tile order), APPEND_FP8K (also an e4m3 copy of K).
enum { APPEND_PLAIN = 0, APPEND_ROPE = 1, APPEND_TILED = 2, APPEND_FP8K = 3 };

template <int BLK, int MODE>
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
  constexpr bool ROPE = MODE == APPEND_ROPE, TILED = MODE == APPEND_TILED, FP8K = MODE == APPEND_FP8K;
  constexpr int D = 128;
  constexpr int PASSES = BLK / 16;
  const int g = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, tl = tid >> 4, dc = tid & 15;

  __shared__ int32_t s_plan[4];
  __shared__ int32_t s_src[TILED ? BLK : 1];   // tiled variant: source token of each position of the block
  __shared__ __align__(16) float s_red[16][D];

  if (tid == 0) {
    int32_t start = __ldcg(p.meta + 0), n = __ldcg(p.meta + 1), anc = __ldcg(p.meta + 3);
    const bool empty = n == 0 && anc == 0 && start >= 0 && start < p.W;
    if (!empty && !window_state_ok(start, n, anc, p.W)) {
      record_error(p.err, UF_EBOUNDS);
      start = 0;
      n = 0;
      anc = 0;
    }
    int32_t slot, start2, n2, anc2;
    append_plan(start, n, p.W, p.keep, p.replace, anc, p.make_anchor, slot, start2, n2, anc2);
    s_plan[0] = slot;
    s_plan[1] = start2;
    s_plan[2] = n2;
    s_plan[3] = anc2;
  }
  if (TILED && tid < BLK && r * BLK + tid < p.Lc) s_src[tid] = tile_token(p.grid, r * BLK + tid);
  __syncthreads();
  const int slot = s_plan[0];

  const int t0 = r * BLK;
  const int cnt = min(BLK, p.Lc - t0);
  const size_t src_stride = static_cast<size_t>(p.G) * D;                       // elements per token
  // source token of position t0 + t of the chunk (tiled variant: gathered in tile order)
  auto src_row = [&](int t) -> size_t {
    const int tok = TILED ? s_src[t] : t0 + t;
    return (static_cast<size_t>(b) * p.Lc + tok) * src_stride + g * D;
  };
  const size_t dst_row0 = (static_cast<size_t>(b) * p.G + g) * p.W * p.lslot + static_cast<size_t>(slot) * p.lslot + t0;
  __nv_bfloat16 *kdst = p.k + dst_row0 * D + dc * 8;

  uint4 kr[PASSES];
#pragma unroll
  for (int m = 0; m < PASSES; ++m) {
    const int t = tl + 16 * m;
    kr[m] = (t < cnt) ? __ldg(reinterpret_cast<const uint4 *>(p.k_new + src_row(t) + dc * 8))
                      : make_uint4(0, 0, 0, 0);   // padding rows of the chunk's last block
  }
  // V tile of this thread: tokens 8*tg .. 8*tg+7, channels 8*cg .. 8*cg+7
  constexpr int TG = BLK / 8;                      // token groups (16 or 8)
  constexpr int VTILES = (BLK / 8) * 16 / 256;     // 8x8 tiles per thread (1 for BLK 128)
  uint4 vr[VTILES > 0 ? VTILES : 1][8];
  const int vtiles = (BLK / 8) * 16;               // 8x8 tiles in the block
#pragma unroll
  for (int q = 0; q < (VTILES > 0 ? VTILES : 1); ++q) {
    const int tile = tid + 256 * q;
    const int tg = tile % TG, cg = tile / TG;
    if (tile < vtiles) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        vr[q][e] = (8 * tg + e < cnt)
                       ? __ldg(reinterpret_cast<const uint4 *>(p.v_new + src_row(8 * tg + e) + 8 * cg))
                       : make_uint4(0, 0, 0, 0);
    }
  }
  if (ROPE) {
    // channels 8 dc .. 8 dc + 7 of this thread are the pairs 4 dc .. 4 dc + 3
    double theta[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) theta[e] = rope_theta(4 * dc + e, D, p.log2_base);
#pragma unroll
    for (int m = 0; m < PASSES; ++m) {
      const int t = tl + 16 * m;
      if (t < cnt) {
        float sn[4], cs[4];
        rope_sincos4(p.pos0 + t0 + t, theta, sn, cs);
        kr[m] = rope_rotate8(kr[m], sn, cs);
      }
    }
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int m = 0; m < PASSES; ++m) {
    const int t = tl + 16 * m;
    *reinterpret_cast<uint4 *>(kdst + static_cast<size_t>(t) * D) = kr[m];
    if (FP8K) {
      // the same eight channels as e4m3 of K / k_scale (padding rows: zeros)
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&kr[m]);
      float f[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 v = __bfloat1622float2(h[e]);
        f[2 * e] = v.x * p.k8_inv_scale;
        f[2 * e + 1] = v.y * p.k8_inv_scale;
      }
      *reinterpret_cast<uint2 *>(p.k8 + (dst_row0 + t) * D + dc * 8) =
          make_uint2(pack_e4m3x4(f[0], f[1], f[2], f[3]), pack_e4m3x4(f[4], f[5], f[6], f[7]));
    }
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&kr[m]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
  // V^T: row (b, g, channel) holds the window's tokens contiguously
  const size_t vt_row_len = static_cast<size_t>(p.W) * p.lslot;
  const size_t vt_col0 = static_cast<size_t>(slot) * p.lslot + t0;
#pragma unroll
  for (int q = 0; q < (VTILES > 0 ? VTILES : 1); ++q) {
    const int tile = tid + 256 * q;
    const int tg = tile % TG, cg = tile / TG;
    if (tile < vtiles) {
      uint4 vt[8];
      transpose8x8_b16(vr[q], vt);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const size_t ch = (static_cast<size_t>(b) * p.G + g) * D + 8 * cg + e;
        *reinterpret_cast<uint4 *>(p.v + ch * vt_row_len + vt_col0 + 8 * tg) = vt[e];
      }
    }
  }
  // block mean of K over the block's true tokens (padding rows hold zeros)
  *reinterpret_cast<float4 *>(&s_red[tl][dc * 8]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  *reinterpret_cast<float4 *>(&s_red[tl][dc * 8 + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) s += s_red[q][tid];
    const size_t prow = (static_cast<size_t>(b) * p.G + g) * p.W * p.nb + static_cast<size_t>(slot) * p.nb + r;
    p.kpool[prow * D + tid] = s / static_cast<float>(cnt);
  }

  // count this block out; the last one commits the new window state.  Thread
  // 0 read the old state at the start (its value fed the plan above), so every
  // block has read it before the last count, and no block reads it again; no
  // fence: the next kernel on the stream sees all of this one's writes.
  if (tid == 0) {
    const int32_t total = static_cast<int32_t>(gridDim.x * gridDim.y * gridDim.z);
    const int32_t prev = atomicAdd(p.meta + 2, 1);
    if (prev == total - 1) {
      atomicExch(p.meta + 0, s_plan[1]);
      atomicExch(p.meta + 1, s_plan[2]);
      atomicExch(p.meta + 3, s_plan[3]);
      atomicExch(p.meta + 2, 0);
    }
  }
}

}  // namespace uf

namespace uf {

// RoPE of a [B, L, heads, D] bf16 tensor, token t at stream position
// pos0 + t (y may alias x).  One thread per (batch, token, 16-byte run of four
// pairs): the angles depend on the token and the pairs only, so they are
// formed once and applied to the run of every head.
__global__ void __launch_bounds__(256) rope_kernel(const __nv_bfloat16 *x, __nv_bfloat16 *y, long long units,
                                                   int32_t L, int32_t heads, long long pos0, double log2_base) {
  constexpr int D = 128;
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int run = static_cast<int>(u & 15);              // 16 runs of 8 channels per row
    const long long bt = u >> 4;                           // batch * L + token
    const long long tok = bt % L;
    double theta[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) theta[e] = rope_theta(4 * run + e, D, log2_base);
    float sn[4], cs[4];
    rope_sincos4(pos0 + tok, theta, sn, cs);
    const size_t base_run = static_cast<size_t>(bt) * heads * 16 + run;
    for (int h = 0; h < heads; ++h) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x) + base_run + 16 * h);
      reinterpret_cast<uint4 *>(y)[base_run + 16 * h] = rope_rotate8(v, sn, cs);
    }
  }
}

}  // namespace uf

namespace uf {

// x, y [B, L = T * Hg * Wg, heads, D] bf16 (y must not alias x): y in tiled
// order from row-major x (inverse = 0), or row-major y from tiled x
// (inverse = 1).  One warp per token row (heads * D * 2 bytes, contiguous on
// both sides): the position is mapped once, the lanes copy the row's 16-byte
// pieces.
__global__ void __launch_bounds__(256) tile_tokens_kernel(const uint4 *__restrict__ x, uint4 *__restrict__ y,
                                                          long long rows, int32_t L, int32_t row_pieces,
                                                          TileGrid g, int32_t inverse) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const long long b = row / L;
    const int32_t tok = static_cast<int32_t>(row - b * L);
    const int32_t p = tile_pos(g, tok);
    const long long src_row = inverse ? b * L + p : row;
    const long long dst_row = inverse ? row : b * L + p;
    for (int piece = lane; piece < row_pieces; piece += 32)
      y[dst_row * row_pieces + piece] = __ldg(x + src_row * row_pieces + piece);
  }
}

}  // namespace uf
