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
// each warp writes two contiguous 256-byte runs per instruction.  The last
// thread block to finish commits the new window state to meta; every block
// read the old state before counting in, so no block can observe a
// half-updated window.
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
  double log2_base;
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

template <int BLK, bool ROPE>
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
  constexpr int D = 128;
  constexpr int PASSES = BLK / 16;
  const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, tl = tid >> 4, dc = tid & 15;

  __shared__ int32_t s_plan[4];
  __shared__ __align__(16) float s_red[16][D];

  if (tid == 0) {
    int32_t start = __ldcg(p.meta + 0), n = __ldcg(p.meta + 1), anc = __ldcg(p.meta + 3);
    const bool empty = n == 0 && anc == 0 && start >= 0 && start < p.W;
    if (!empty && !window_state_ok(start, n, anc, p.W)) {
      record_error(UF_EBOUNDS);
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
  __syncthreads();
  const int slot = s_plan[0];

  const int t0 = r * BLK;
  const int cnt = min(BLK, p.Lc - t0);
  const size_t src_stride = static_cast<size_t>(p.G) * D;                       // elements per token
  const __nv_bfloat16 *ksrc = p.k_new + (static_cast<size_t>(b) * p.Lc + t0) * src_stride + g * D + dc * 8;
  const size_t dst_row0 = (static_cast<size_t>(b) * p.G + g) * p.W * p.lslot + static_cast<size_t>(slot) * p.lslot + t0;
  __nv_bfloat16 *kdst = p.k + dst_row0 * D + dc * 8;

  uint4 kr[PASSES];
#pragma unroll
  for (int m = 0; m < PASSES; ++m) {
    const int t = tl + 16 * m;
    kr[m] = (t < cnt) ? __ldg(reinterpret_cast<const uint4 *>(ksrc + t * src_stride))
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
      const __nv_bfloat16 *src =
          p.v_new + (static_cast<size_t>(b) * p.Lc + t0 + 8 * tg) * src_stride + g * D + 8 * cg;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        vr[q][e] = (8 * tg + e < cnt) ? __ldg(reinterpret_cast<const uint4 *>(src + e * src_stride))
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

  // commit the new window state once every block has read the old one
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int32_t total = static_cast<int32_t>(gridDim.x * gridDim.y * gridDim.z);
    const int32_t prev = atomicAdd(p.meta + 2, 1);
    if (prev == total - 1) {
      atomicExch(p.meta + 0, s_plan[1]);
      atomicExch(p.meta + 1, s_plan[2]);
      atomicExch(p.meta + 3, s_plan[3]);
      atomicExch(p.meta + 2, 0);
      __threadfence();
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
