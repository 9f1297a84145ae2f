// uf.cu -- C ABI of libuf.so: argument checks, TMA tensor maps, launches.
//
// Single translation unit: the kernels live in the included headers so that the
// device error word is one symbol per device.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "uf.h"
#include "uf_device.cuh"
#include "kv_append.cuh"
#include "block_mask.cuh"
#include "attention.cuh"

namespace {

constexpr int32_t UF_VERSION = 300;   // 0.3.0
constexpr int32_t kMaxW = 64;
constexpr int32_t kMaxMaskNKV = 1024; // window blocks: 32 selection keys per lane
constexpr int32_t kMaxDevices = 64;
std::atomic<long long> g_wait_limit{1LL << 31};
// attention launches add their cycles / nanoseconds here when set
std::atomic<unsigned long long *> g_clock_counters{nullptr};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t ceil_div(int32_t a, int32_t b) { return (a + b - 1) / b; }

bool dims_ok(int32_t B, int32_t G, int32_t D, int32_t W, int32_t Lc, int32_t blk) {
  if (B < 1 || G < 1 || W < 1 || W > kMaxW || Lc < 1) return false;
  if (D != 128) return false;
  if (blk != 64 && blk != 128) return false;
  // every element offset of the window buffers must fit the 32-bit row math
  const long long lslot = static_cast<long long>(ceil_div(Lc, blk)) * blk;
  if (static_cast<long long>(W) * lslot >= (1LL << 30)) return false;
  const long long bytes = static_cast<long long>(B) * G * W * lslot * D * 2;
  return bytes <= (1LL << 40);
}

bool cache_ok(const uf_kv_cache *c) {
  if (!c) return false;
  if (!dims_ok(c->B, c->G, c->D, c->W, c->Lc, c->blk)) return false;
  if (!c->k || !c->v || !c->kpool || !c->meta) return false;
  if (!aligned16(c->k) || !aligned16(c->v) || !aligned16(c->kpool) || !aligned16(c->meta)) return false;
  return true;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor map, 128-byte swizzle, box {64, box[1..]} (64 bf16 = 128 bytes inner).
bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
              const cuuint32_t *box, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B,
              CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, type, rank, const_cast<void *>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

thread_local const char *t_last_cuda_error = "no error";

int32_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return UF_OK;
  t_last_cuda_error = cudaGetErrorString(e);
  return UF_ECUDA;
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` (per device,
// only when a launch needs more than any earlier one).
template <typename K>
int32_t ensure_smem(K kernel, int bytes, std::atomic<int> (&done)[kMaxDevices]) {
  int dev = 0;
  const int32_t st = cuda_status(cudaGetDevice(&dev));
  if (st != UF_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return UF_EUNSUPPORTED;
  if (done[dev].load() >= bytes) return UF_OK;
  const int32_t st2 = cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (st2 != UF_OK) return st2;
  done[dev].store(bytes);
  return UF_OK;
}

int32_t launch_status() { return cuda_status(cudaGetLastError()); }

// The attention kernel splits its launch register allocation between
// warpgroups (setmaxnreg); the split is only valid for the per-thread count
// it was written for, so a build compiled to another count is refused.
template <typename K>
int32_t check_launch_regs(K kernel, std::atomic<int> (&done)[kMaxDevices]) {
  int dev = 0;
  const int32_t st = cuda_status(cudaGetDevice(&dev));
  if (st != UF_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return UF_EUNSUPPORTED;
  if (done[dev].load() == 1) return UF_OK;
  cudaFuncAttributes attr;
  const int32_t st2 = cuda_status(cudaFuncGetAttributes(&attr, kernel));
  if (st2 != UF_OK) return st2;
  if (attr.numRegs != uf::ATTN_LAUNCH_REGS) return UF_EUNSUPPORTED;
  done[dev].store(1);
  return UF_OK;
}
std::atomic<int> g_attn128_regs[kMaxDevices], g_attn64_regs[kMaxDevices], g_attn128f8_regs[kMaxDevices],
    g_attn64f8_regs[kMaxDevices];

// Streaming multiprocessors of the current device (cached per device): the
// persistent attention grid has one thread block per SM.
std::atomic<int> g_sm_count[kMaxDevices];
int32_t sm_count(int *out) {
  int dev = 0;
  const int32_t st = cuda_status(cudaGetDevice(&dev));
  if (st != UF_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return UF_EUNSUPPORTED;
  int v = g_sm_count[dev].load();
  if (v <= 0) {
    const int32_t st2 = cuda_status(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev));
    if (st2 != UF_OK) return st2;
    if (v <= 0) return UF_EUNSUPPORTED;
    g_sm_count[dev].store(v);
  }
  *out = v;
  return UF_OK;
}

std::atomic<int> g_attn128f8_smem[kMaxDevices], g_attn64f8_smem[kMaxDevices];
std::atomic<int> g_attn128_smem[kMaxDevices], g_attn64_smem[kMaxDevices];

// One mask kernel instance per (block size, selection keys per lane).
template <int BLK, int MAXPER>
int32_t launch_mask(const uf::MaskParams &p, dim3 grid, int smem, cudaStream_t st) {
  static std::atomic<int> smem_set[kMaxDevices];
  const int32_t e = ensure_smem(uf::block_mask_kernel<BLK, MAXPER>, smem, smem_set);
  if (e != UF_OK) return e;
  uf::block_mask_kernel<BLK, MAXPER><<<grid, uf::MASK_THREADS, smem, st>>>(p);
  return UF_OK;
}

// keys per lane of the selection: the smallest of 8, 12, 16, 24, 32 >= ceil(W * nb / 32)
template <int BLK>
int32_t launch_mask_per(const uf::MaskParams &p, int nkv_max, dim3 grid, int smem, cudaStream_t st) {
  const int per = (nkv_max + 31) / 32;
  if (per <= 8) return launch_mask<BLK, 8>(p, grid, smem, st);
  if (per <= 12) return launch_mask<BLK, 12>(p, grid, smem, st);
  if (per <= 16) return launch_mask<BLK, 16>(p, grid, smem, st);
  if (per <= 24) return launch_mask<BLK, 24>(p, grid, smem, st);
  return launch_mask<BLK, 32>(p, grid, smem, st);
}

}  // namespace

namespace {

// RoPE arguments: base > 1 and finite; positions in [0, kMaxRopePos): the
// fp64 product pos * theta of a position below 2^40 is within 1.2e-4 rad.
constexpr long long kMaxRopePos = 1LL << 40;
bool rope_args_ok(long long pos0, float base) {
  return pos0 >= 0 && pos0 < kMaxRopePos && isfinite(base) && base > 1.0f;
}

// uf_kv_append and uf_kv_append_rope (rope = 1: K rotated at pos0 + token).
int32_t append_impl(uf_kv_cache *c, const void *k_new, const void *v_new, int32_t keep_chunks, int32_t flags,
                    int32_t rope, long long pos0, double log2_base, uf_stream_t s,
                    const uf::TileGrid *tile_grid = nullptr, void *k8 = nullptr, float k_scale = 1.0f) {
  if (!cache_ok(c)) return UF_EINVAL;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return UF_EINVAL;
  if (keep_chunks < 1 || keep_chunks > c->W) return UF_EINVAL;
  if (flags & ~(UF_APPEND_REPLACE_NEWEST | UF_APPEND_ANCHOR)) return UF_EINVAL;
  const int32_t replace = (flags & UF_APPEND_REPLACE_NEWEST) ? 1 : 0;
  const int32_t make_anchor = (flags & UF_APPEND_ANCHOR) ? 1 : 0;
  if (replace && c->host_n_valid == 0) return UF_EINVAL;
  // an anchor starts an empty window of at least two slots; while one is
  // pinned, keep_chunks counts it and must leave room for a recent chunk
  if (make_anchor && (replace || c->host_n_valid != 0 || c->W < 2)) return UF_EINVAL;
  if (!make_anchor && c->host_anchor && keep_chunks < 2) return UF_EINVAL;

  uf::AppendParams p;
  p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
  p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
  p.k = static_cast<__nv_bfloat16 *>(c->k);
  p.v = static_cast<__nv_bfloat16 *>(c->v);
  p.kpool = c->kpool;
  p.meta = c->meta;
  p.G = c->G;
  p.W = c->W;
  p.Lc = c->Lc;
  p.nb = ceil_div(c->Lc, c->blk);
  p.lslot = p.nb * c->blk;
  p.keep = keep_chunks;
  p.replace = replace;
  p.make_anchor = make_anchor;
  p.pos0 = pos0;
  p.log2_base = log2_base;
  p.err = c->err;
  const bool tiled = tile_grid != nullptr;
  if (tiled) p.grid = *tile_grid;
  p.k8 = static_cast<uint8_t *>(k8);
  p.k8_inv_scale = 1.0f / k_scale;
  const dim3 grid(c->G, p.nb, c->B);   // KV heads fastest: concurrent blocks read each token's heads together
  cudaGetLastError();
  const cudaStream_t st0 = reinterpret_cast<cudaStream_t>(s);
  const int mode = rope ? uf::APPEND_ROPE : tiled ? uf::APPEND_TILED : k8 ? uf::APPEND_FP8K : uf::APPEND_PLAIN;
  if (c->blk == 128) {
    switch (mode) {
      case uf::APPEND_ROPE: uf::kv_append_kernel<128, uf::APPEND_ROPE><<<grid, 256, 0, st0>>>(p); break;
      case uf::APPEND_TILED: uf::kv_append_kernel<128, uf::APPEND_TILED><<<grid, 256, 0, st0>>>(p); break;
      case uf::APPEND_FP8K: uf::kv_append_kernel<128, uf::APPEND_FP8K><<<grid, 256, 0, st0>>>(p); break;
      default: uf::kv_append_kernel<128, uf::APPEND_PLAIN><<<grid, 256, 0, st0>>>(p); break;
    }
  } else {
    switch (mode) {
      case uf::APPEND_ROPE: uf::kv_append_kernel<64, uf::APPEND_ROPE><<<grid, 256, 0, st0>>>(p); break;
      case uf::APPEND_TILED: uf::kv_append_kernel<64, uf::APPEND_TILED><<<grid, 256, 0, st0>>>(p); break;
      case uf::APPEND_FP8K: uf::kv_append_kernel<64, uf::APPEND_FP8K><<<grid, 256, 0, st0>>>(p); break;
      default: uf::kv_append_kernel<64, uf::APPEND_PLAIN><<<grid, 256, 0, st0>>>(p); break;
    }
  }
  const int32_t st = launch_status();
  if (st != UF_OK) return st;
  // host mirror (the kernel's rule)
  int32_t slot2, start2, n2, anchor2;
  uf::append_plan(c->host_start, c->host_n_valid, c->W, keep_chunks, replace, c->host_anchor, make_anchor, slot2,
                  start2, n2, anchor2);
  c->host_anchor = anchor2;
  c->host_start = start2;
  c->host_n_valid = n2;
  return UF_OK;
}

}  // namespace

namespace {
// Workspace of the balanced schedule for `sms` thread blocks: arrival
// counters (one per thread block, padded to 256 bytes), then two partial
// results per thread block.
size_t attn_ws_cnt_bytes(int sms) { return (static_cast<size_t>(sms) * 4 + 255) / 256 * 256; }
size_t attn_ws_bytes(int sms) {
  return attn_ws_cnt_bytes(sms) + 2 * static_cast<size_t>(sms) * uf::ATTN_PART_FLOATS * sizeof(float);
}
// The balanced schedule pays off when there are few items per SM and the
// plain schedule's last round of items leaves SMs idle: ceil(items / sms)
// rounds against items / sms on average, more than 10% apart.  With many
// items, or a whole number of rounds, the plain schedule is as even and keeps
// the items that run at the same time closer together (L2 reuse of K / V).
constexpr long long kBalancedItemsPerSm = 8;
bool balanced_pays(long long items, int sms) {
  if (items >= kBalancedItemsPerSm * sms) return false;
  const long long rounds = (items + sms - 1) / sms;
  return rounds * sms * 10 > items * 11;
}

// uf_block_sparse_attn, its FP8-score variant (k8 != NULL) and the balanced
// variant (ws != NULL: workspace of attn_ws_bytes(SM count) bytes).
int32_t attn_impl(const void *q, int32_t H, const uf_kv_cache *c, const int32_t *idx, const int32_t *cnt, int32_t k,
                  float scale, void *o, float *lse, uf_stream_t s, const void *k8, float q_scale, float k_scale,
                  void *ws = nullptr, size_t ws_bytes = 0) {
  if (!cache_ok(c)) return UF_EINVAL;
  if (!q || !o || !aligned16(q) || !aligned16(o)) return UF_EINVAL;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return UF_EINVAL;
  if (H < 1 || H % c->G != 0) return UF_EINVAL;
  if (!(scale > 0.f) || !isfinite(scale)) return UF_EINVAL;
  const int32_t nb = ceil_div(c->Lc, c->blk);
  if (idx) {
    if (k < 1 || k > c->W * nb) return UF_EINVAL;
    if (reinterpret_cast<uintptr_t>(idx) & 3u) return UF_EINVAL;
    if (cnt && (reinterpret_cast<uintptr_t>(cnt) & 3u)) return UF_EINVAL;
  } else {
    k = 0;
    cnt = nullptr;
  }
  if (c->host_n_valid < 1) return UF_EINVAL;
  const long long items = static_cast<long long>(c->B) * H * nb;
  if (items >= (1LL << 31)) return UF_EINVAL;

  const int32_t lslot = nb * c->blk;
  CUtensorMap tq, tk, tv, to;
  {
    // Q and O: [B, Lc, H, D] as {channels, heads, tokens, batch}.  Q: a
    // 128-row tile of one head per 64-channel load (rows past Lc read as
    // zero); O: one q-block (blk rows) of one head per 64-channel store
    const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(c->Lc),
                                static_cast<cuuint64_t>(c->B)};
    // byte strides of dims 1..3 (head, token, batch)
    const cuuint64_t strides[3] = {256, static_cast<cuuint64_t>(H) * 256, static_cast<cuuint64_t>(c->Lc) * H * 256};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    if (!make_map(&tq, q, 4, dims, strides, box)) return UF_ECUDA;
    const cuuint32_t obox[4] = {64, 1, static_cast<cuuint32_t>(c->blk), 1};
    if (!make_map(&to, o, 4, dims, strides, obox)) return UF_ECUDA;
  }
  if (!k8) {
    // K: [B*G][W*Lslot][128] -> box {64 channels, blk tokens}
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(c->W) * lslot, static_cast<cuuint64_t>(c->B) * c->G};
    const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(c->W) * lslot * 256};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(c->blk), 1};
    if (!make_map(&tk, c->k, 3, dims, strides, box)) return UF_ECUDA;
  } else {
    // e4m3 K: [B*G][W*Lslot][128 bytes] -> box {128 channels, blk tokens}
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(c->W) * lslot, static_cast<cuuint64_t>(c->B) * c->G};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(c->W) * lslot * 128};
    const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(c->blk), 1};
    if (!make_map(&tk, k8, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_UINT8))
      return UF_ECUDA;
  }
  {
    // V^T: [B*G][128][W*Lslot] -> box {64 tokens, 128 channels}
    const cuuint64_t row = static_cast<cuuint64_t>(c->W) * lslot;
    const cuuint64_t dims[3] = {row, 128, static_cast<cuuint64_t>(c->B) * c->G};
    const cuuint64_t strides[2] = {row * 2, row * 2 * 128};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!make_map(&tv, c->v, 3, dims, strides, box)) return UF_ECUDA;
  }
  uf::AttnParams p;
  p.meta = c->meta;
  p.idx = idx;
  p.cnt = cnt;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.items = static_cast<int32_t>(items);
  p.lse = lse;
  p.H = H;
  p.G = c->G;
  p.W = c->W;
  p.Lc = c->Lc;
  p.nb = nb;
  p.lslot = lslot;
  p.k = k;
  p.nb_mul = nb == 1 ? 0xFFFFFFFFu : static_cast<uint32_t>((1ULL << 32) / static_cast<uint64_t>(nb));
  p.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  p.q_inv_scale = 1.0f / q_scale;
  p.wait_limit = g_wait_limit.load();
  p.err = c->err;
  p.ws_cnt = nullptr;
  p.ws_part = nullptr;
  p.clk = g_clock_counters.load();
  int sms = 0;
  const int32_t se = sm_count(&sms);
  if (se != UF_OK) return se;
  unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  cudaGetLastError();
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
  if (ws) {
    if (!aligned16(ws) || ws_bytes < attn_ws_bytes(sms)) return UF_EINVAL;
    if (balanced_pays(items, sms)) {
      // balanced schedule: one thread block per SM, counters zeroed first
      p.ws_cnt = static_cast<int32_t *>(ws);
      p.ws_part = reinterpret_cast<float *>(static_cast<char *>(ws) + attn_ws_cnt_bytes(sms));
      grid = static_cast<unsigned>(sms);
      const int32_t e = cuda_status(cudaMemsetAsync(p.ws_cnt, 0, static_cast<size_t>(sms) * 4, st));
      if (e != UF_OK) return e;
    }
  }
  const bool fp8 = k8 != nullptr;
  if (c->blk == 128) {
    constexpr int smem = uf::AttnSmem<128>::DYN;
    auto kern = fp8 ? uf::attn_kernel<128, true> : uf::attn_kernel<128, false>;
    int32_t e = check_launch_regs(kern, fp8 ? g_attn128f8_regs : g_attn128_regs);
    if (e == UF_OK) e = ensure_smem(kern, smem, fp8 ? g_attn128f8_smem : g_attn128_smem);
    if (e != UF_OK) return e;
    kern<<<grid, uf::ATTN_THREADS, smem, st>>>(tq, tk, tv, to, p);
  } else {
    constexpr int smem = uf::AttnSmem<64>::DYN;
    auto kern = fp8 ? uf::attn_kernel<64, true> : uf::attn_kernel<64, false>;
    int32_t e = check_launch_regs(kern, fp8 ? g_attn64f8_regs : g_attn64_regs);
    if (e == UF_OK) e = ensure_smem(kern, smem, fp8 ? g_attn64f8_smem : g_attn64_smem);
    if (e != UF_OK) return e;
    kern<<<grid, uf::ATTN_THREADS, smem, st>>>(tq, tk, tv, to, p);
  }
  return launch_status();
}
}  // namespace

extern "C" {

int32_t uf_version(void) { return UF_VERSION; }

#ifndef UF_SOURCE_HASH
#define UF_SOURCE_HASH "unknown"
#endif
const char *uf_source_hash(void) { return UF_SOURCE_HASH; }

const char *uf_strerror(int32_t status) {
  switch (status) {
    case UF_OK: return "UF_OK";
    case UF_EINVAL: return "UF_EINVAL: invalid argument";
    case UF_ECUDA: return "UF_ECUDA: CUDA call or kernel launch failed";
    case UF_ETIMEOUT: return "UF_ETIMEOUT: a kernel pipeline wait exceeded its bound";
    case UF_EBOUNDS: return "UF_EBOUNDS: a kernel found an out-of-range index or window state";
    case UF_EUNSUPPORTED: return "UF_EUNSUPPORTED: valid request this library does not implement";
    default: return "UF_UNKNOWN";
  }
}

int32_t uf_kv_cache_bytes(int32_t B, int32_t G, int32_t D, int32_t W, int32_t Lc, int32_t blk, size_t *kv_bytes,
                          size_t *kpool_bytes, size_t *meta_bytes) {
  if (!dims_ok(B, G, D, W, Lc, blk)) return UF_EINVAL;
  const size_t nb = static_cast<size_t>(ceil_div(Lc, blk));
  const size_t lslot = nb * blk;
  if (kv_bytes) *kv_bytes = static_cast<size_t>(B) * G * W * lslot * D * 2;
  if (kpool_bytes) *kpool_bytes = static_cast<size_t>(B) * G * W * nb * D * 4;
  if (meta_bytes) *meta_bytes = 4 * sizeof(int32_t);
  return UF_OK;
}

int32_t uf_kv_cache_init(uf_kv_cache *c, void *k, void *v, float *kpool, int32_t *meta, int32_t B, int32_t G,
                         int32_t D, int32_t W, int32_t Lc, int32_t blk) {
  if (!c) return UF_EINVAL;
  uf_kv_cache t;
  t.k = k;
  t.v = v;
  t.kpool = kpool;
  t.meta = meta;
  t.B = B;
  t.G = G;
  t.D = D;
  t.W = W;
  t.Lc = Lc;
  t.blk = blk;
  t.host_start = 0;
  t.host_n_valid = 0;
  t.host_anchor = 0;
  t.err = nullptr;
  if (!cache_ok(&t)) return UF_EINVAL;
  *c = t;
  return UF_OK;
}

int32_t uf_kv_cache_set_error_word(uf_kv_cache *c, int32_t *err) {
  if (!cache_ok(c)) return UF_EINVAL;
  if (reinterpret_cast<uintptr_t>(err) & 3u) return UF_EINVAL;
  c->err = err;
  return UF_OK;
}

int32_t uf_kv_reset(uf_kv_cache *c, uf_stream_t s) {
  if (!cache_ok(c)) return UF_EINVAL;
  const int32_t st = cuda_status(cudaMemsetAsync(c->meta, 0, 4 * sizeof(int32_t), reinterpret_cast<cudaStream_t>(s)));
  if (st != UF_OK) return st;
  c->host_start = 0;
  c->host_n_valid = 0;
  c->host_anchor = 0;
  return UF_OK;
}

int32_t uf_kv_append(uf_kv_cache *c, const void *k_new, const void *v_new, int32_t keep_chunks, int32_t flags,
                     uf_stream_t s) {
  return append_impl(c, k_new, v_new, keep_chunks, flags, 0, 0, 0.0, s);
}

int32_t uf_kv_append_rope(uf_kv_cache *c, const void *k_new, const void *v_new, int32_t keep_chunks,
                          int32_t flags, int64_t pos0, float base, uf_stream_t s) {
  if (!rope_args_ok(pos0, base)) return UF_EINVAL;
  if (c && pos0 > kMaxRopePos - c->Lc) return UF_EINVAL;
  return append_impl(c, k_new, v_new, keep_chunks, flags, 1, pos0, log2(static_cast<double>(base)), s);
}

int32_t uf_rope(const void *x, void *y, int32_t B, int32_t L, int32_t heads, int64_t pos0, float base,
                uf_stream_t s) {
  if (!x || !y || !aligned16(x) || !aligned16(y)) return UF_EINVAL;
  if (B < 1 || L < 1 || heads < 1) return UF_EINVAL;
  if (!rope_args_ok(pos0, base) || pos0 > kMaxRopePos - L) return UF_EINVAL;
  const long long units = static_cast<long long>(B) * L * 16;   // (batch, token, run); heads loop inside
  if (static_cast<long long>(B) * L * heads > (1LL << 40)) return UF_EINVAL;
  int sms = 0;
  const int32_t se = sm_count(&sms);
  if (se != UF_OK) return se;
  const long long want = (units + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 8LL * sms ? want : 8LL * sms);
  cudaGetLastError();
  uf::rope_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(s)>>>(
      static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(y), units, L, heads, pos0,
      log2(static_cast<double>(base)));
  return launch_status();
}


int32_t uf_block_mask(const void *q, int32_t H, const uf_kv_cache *c, int32_t k, int32_t *idx, int32_t *cnt,
                      float *scores, uf_stream_t s) {
  return uf_block_mask_local(q, H, c, k, 0, 0, idx, cnt, scores, s);
}

int32_t uf_block_mask_local(const void *q, int32_t H, const uf_kv_cache *c, int32_t k, int32_t local,
                            int32_t flags, int32_t *idx, int32_t *cnt, float *scores, uf_stream_t s) {
  if (!cache_ok(c)) return UF_EINVAL;
  if (local < 0 || local > (1 << 20) || (flags & ~UF_MASK_LOCAL_ONLY) != 0) return UF_EINVAL;
  if (2 * local + 1 > k) return UF_EINVAL;
  if (!q || !idx || !cnt || !aligned16(q)) return UF_EINVAL;
  if (!aligned16(idx) || !aligned16(cnt) || (scores && !aligned16(scores))) return UF_EINVAL;
  if (H < 1 || H % c->G != 0) return UF_EINVAL;
  const int32_t nb = ceil_div(c->Lc, c->blk);
  const int32_t nkv_max = c->W * nb;
  if (k < 1 || k > nkv_max) return UF_EINVAL;
  if (c->host_n_valid < 1) return UF_EINVAL;
  if (nkv_max > kMaxMaskNKV) return UF_EUNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(q) & 15u) return UF_EINVAL;

  uf::MaskParams p;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.kpool = c->kpool;
  p.meta = c->meta;
  p.idx = idx;
  p.cnt = cnt;
  p.scores = scores;
  p.H = H;
  p.G = c->G;
  p.W = c->W;
  p.Lc = c->Lc;
  p.nb = nb;
  p.k = k;
  p.local = local;
  p.local_only = (flags & UF_MASK_LOCAL_ONLY) ? 1 : 0;
  p.scale = 1.0f / sqrtf(static_cast<float>(c->D));
  p.err = c->err;
  const int smem = uf::mask_smem_bytes(nkv_max);
  const dim3 grid(ceil_div(nb, uf::MASK_TQ), H, c->B);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
  cudaGetLastError();
  const int32_t e = c->blk == 128 ? launch_mask_per<128>(p, nkv_max, grid, smem, st)
                                  : launch_mask_per<64>(p, nkv_max, grid, smem, st);
  if (e != UF_OK) return e;
  return launch_status();
}

int32_t uf_block_sparse_attn(const void *q, int32_t H, const uf_kv_cache *c, const int32_t *idx, const int32_t *cnt,
                             int32_t k, float scale, void *o, float *lse, uf_stream_t s) {
  return attn_impl(q, H, c, idx, cnt, k, scale, o, lse, s, nullptr, 1.0f, 1.0f);
}

int32_t uf_attn_workspace_bytes(size_t *bytes) {
  if (!bytes) return UF_EINVAL;
  int sms = 0;
  const int32_t se = sm_count(&sms);
  if (se != UF_OK) return se;
  *bytes = attn_ws_bytes(sms);
  return UF_OK;
}

int32_t uf_block_sparse_attn_balanced(const void *q, int32_t H, const uf_kv_cache *c, const int32_t *idx,
                                      const int32_t *cnt, int32_t k, float scale, void *o, float *lse,
                                      void *workspace, size_t workspace_bytes, uf_stream_t s) {
  if (!workspace) return UF_EINVAL;
  return attn_impl(q, H, c, idx, cnt, k, scale, o, lse, s, nullptr, 1.0f, 1.0f, workspace, workspace_bytes);
}

}  // extern "C"

namespace {
// Scratch memory of uf_block_sparse_attn_balanced_noalloc: one fixed array in
// the library's device image, the balanced schedule's workspace for devices
// of at most kNoAllocMaxSms SMs.  It exists on every device that loads the
// library, from module load until the process exits.  Host code must not use
// the symbol itself as an address (on the host it names a host-side shadow):
// the device address comes from cudaGetSymbolAddress, once per device.
constexpr int kNoAllocMaxSms = 160;
constexpr size_t kNoAllocScratchBytes =
    (static_cast<size_t>(kNoAllocMaxSms) * 4 + 255) / 256 * 256 +
    2 * static_cast<size_t>(kNoAllocMaxSms) * uf::ATTN_PART_FLOATS * sizeof(float);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<void *> g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device (looked up on the
// first call per device, with that device current).
int32_t noalloc_scratch(void **out) {
  int dev = 0;
  const int32_t st = cuda_status(cudaGetDevice(&dev));
  if (st != UF_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return UF_EUNSUPPORTED;
  void *p = g_noalloc_addr[dev].load();
  if (!p) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    p = g_noalloc_addr[dev].load();
    if (!p) {
      const int32_t st2 = cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch));
      if (st2 != UF_OK) return st2;
      if (!p) return UF_ECUDA;
      g_noalloc_addr[dev].store(p);
    }
  }
  *out = p;
  return UF_OK;
}
}  // namespace

extern "C" {

int32_t uf_block_sparse_attn_balanced_noalloc(const void *q, int32_t H, const uf_kv_cache *c, const int32_t *idx,
                                              const int32_t *cnt, int32_t k, float scale, void *o, float *lse,
                                              uf_stream_t s) {
  int sms = 0;
  const int32_t se = sm_count(&sms);
  if (se != UF_OK) return se;
  if (attn_ws_bytes(sms) > kNoAllocScratchBytes) return UF_EUNSUPPORTED;   // more SMs than the array serves
  void *ws = nullptr;
  const int32_t sa = noalloc_scratch(&ws);
  if (sa != UF_OK) return sa;
  return attn_impl(q, H, c, idx, cnt, k, scale, o, lse, s, nullptr, 1.0f, 1.0f, ws, kNoAllocScratchBytes);
}

int32_t uf_block_sparse_attn_fp8k(const void *q, int32_t H, const uf_kv_cache *c, const void *k8, float q_scale,
                                  float k_scale, const int32_t *idx, const int32_t *cnt, int32_t k, float scale,
                                  void *o, float *lse, uf_stream_t s) {
  if (!k8 || !aligned16(k8)) return UF_EINVAL;
  if (!(q_scale > 0.f) || !isfinite(q_scale) || !(k_scale > 0.f) || !isfinite(k_scale)) return UF_EINVAL;
  return attn_impl(q, H, c, idx, cnt, k, scale, o, lse, s, k8, q_scale, k_scale);
}

int32_t uf_kv_append_fp8k(uf_kv_cache *c, void *k8, float k_scale, const void *k_new, const void *v_new,
                          int32_t keep_chunks, int32_t flags, uf_stream_t s) {
  if (!k8 || !aligned16(k8) || !(k_scale > 0.f) || !isfinite(k_scale)) return UF_EINVAL;
  return append_impl(c, k_new, v_new, keep_chunks, flags, 0, 0, 0.0, s, nullptr, k8, k_scale);
}


int32_t uf_check_error(int32_t *dev_err_word, uf_stream_t s) {
  if (!dev_err_word || (reinterpret_cast<uintptr_t>(dev_err_word) & 3u)) return UF_EINVAL;
  cudaGetLastError();
  uf::check_error_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(s)>>>(dev_err_word);
  return launch_status();
}

int32_t uf_get_error(int32_t *status, int32_t clear) {
  if (!status) return UF_EINVAL;
  int32_t st = cuda_status(cudaDeviceSynchronize());
  if (st != UF_OK) return st;
  int32_t v = 0;
  st = cuda_status(cudaMemcpyFromSymbol(&v, uf::g_error_word, sizeof(v)));
  if (st != UF_OK) return st;
  if (clear) {
    const int32_t z = 0;
    st = cuda_status(cudaMemcpyToSymbol(uf::g_error_word, &z, sizeof(z)));
    if (st != UF_OK) return st;
  }
  *status = v;
  return UF_OK;
}

const char *uf_last_cuda_error(void) { return t_last_cuda_error; }

int32_t uf_set_wait_limit(int64_t cycles) {
  if (cycles < 1000) return UF_EINVAL;
  g_wait_limit.store(cycles);
  return UF_OK;
}

int32_t uf_set_clock_counters(uint64_t *dev_counters) {
  if (reinterpret_cast<uintptr_t>(dev_counters) & 7u) return UF_EINVAL;
  g_clock_counters.store(reinterpret_cast<unsigned long long *>(dev_counters));
  return UF_OK;
}

int32_t uf_debug_wait_timeout(int64_t cycles, uf_stream_t s) {
  if (cycles < 1000 || cycles > (1LL << 40)) return UF_EINVAL;
  cudaGetLastError();
  uf::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(s)>>>(cycles);
  return launch_status();
}

// Tile-grid arguments: positive, L = T * Hg * Wg within int32, tile sides >= 1.
static bool tile_grid_ok(int32_t T, int32_t Hg, int32_t Wg, int32_t bt, int32_t by, int32_t bx) {
  if (T < 1 || Hg < 1 || Wg < 1 || bt < 1 || by < 1 || bx < 1) return false;
  return static_cast<long long>(T) * Hg * Wg < (1LL << 30);
}

int32_t uf_tile_tokens(const void *x, void *y, int32_t B, int32_t T, int32_t Hg, int32_t Wg, int32_t heads,
                       int32_t bt, int32_t by, int32_t bx, int32_t inverse, uf_stream_t s) {
  if (!x || !y || x == y || !aligned16(x) || !aligned16(y)) return UF_EINVAL;
  if (B < 1 || heads < 1 || (inverse != 0 && inverse != 1) || !tile_grid_ok(T, Hg, Wg, bt, by, bx))
    return UF_EINVAL;
  const int32_t L = T * Hg * Wg;
  const long long row_bytes = static_cast<long long>(heads) * 128 * 2;
  const long long pieces = static_cast<long long>(B) * L * (row_bytes / 16);
  if (pieces / (row_bytes / 16) / L != B || row_bytes / 16 > (1LL << 30)) return UF_EINVAL;
  const char *xe = static_cast<const char *>(x), *ye = static_cast<const char *>(y);
  const long long bytes = pieces * 16;
  if (xe < ye + bytes && ye < xe + bytes) return UF_EINVAL;      // overlapping buffers
  int sms = 0;
  const int32_t se = sm_count(&sms);
  if (se != UF_OK) return se;
  const long long rows = static_cast<long long>(B) * L;
  const long long want = (rows + 7) / 8;                     // 8 warps (rows in flight) per block
  const unsigned grid = static_cast<unsigned>(want < 16LL * sms ? want : 16LL * sms);
  const uf::TileGrid g{T, Hg, Wg, bt, by, bx};
  cudaGetLastError();
  uf::tile_tokens_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(s)>>>(
      static_cast<const uint4 *>(x), static_cast<uint4 *>(y), rows, L, static_cast<int32_t>(row_bytes / 16), g,
      inverse);
  return launch_status();
}

int32_t uf_kv_append_tiled(uf_kv_cache *c, const void *k_new, const void *v_new, int32_t keep_chunks,
                           int32_t flags, int32_t T, int32_t Hg, int32_t Wg, int32_t bt, int32_t by, int32_t bx,
                           uf_stream_t s) {
  if (!cache_ok(c) || !tile_grid_ok(T, Hg, Wg, bt, by, bx)) return UF_EINVAL;
  if (static_cast<long long>(T) * Hg * Wg != c->Lc) return UF_EINVAL;
  const uf::TileGrid g{T, Hg, Wg, bt, by, bx};
  return append_impl(c, k_new, v_new, keep_chunks, flags, 0, 0, 0.0, s, &g);
}

}  // extern "C"
