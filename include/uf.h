/*
 * uf.h -- C ABI of the chunk-causal block-sparse attention library (libuf.so)
 *
 * Three calls make up one attention layer of a streaming video DiT, per chunk:
 *
 *   uf_kv_append         rolling-window append / evict of the new chunk's K and V
 *                        (uf_kv_append_rope / uf_rope: with rotary position
 *                        embedding of K and of the queries)
 *   uf_block_mask        per-head block mean-pooling of Q and K, pooled block
 *                        scores, top-k block selection with the diagonal kept
 *                        (uf_block_mask_local: with a forced local band of
 *                        blocks around the diagonal, or the band alone)
 *   uf_block_sparse_attn softmax attention of the chunk's queries over the kept
 *                        blocks of the window (bf16 in, fp32 softmax, bf16 O and
 *                        fp32 LSE), grouped-query aware
 *
 * Conventions shared by every call
 *   - Every buffer is owned by the caller.  Pointers named "device" point to
 *     device memory of the current CUDA device; they must be 16-byte aligned.
 *   - No call allocates memory, synchronises the device or reads device data
 *     back to the host.  Work is enqueued on the caller's stream `s` (a
 *     cudaStream_t; NULL = legacy default stream) and runs asynchronously.
 *   - Every call returns a status (uf_status).  Argument errors are detected on
 *     the host before anything is enqueued (UF_EINVAL, nothing launched).  A
 *     launch failure returns UF_ECUDA.  Errors found by a kernel while running
 *     (an out-of-range block index, a bad window state, a pipeline wait that
 *     exceeded its bound) are recorded in a device-side error word: the
 *     window's own word when the caller gave it one (uf_kv_cache.err), else
 *     the library's word of the current device, which uf_check_error() moves
 *     into a caller's word in stream order and uf_get_error() reads after a
 *     device synchronisation.  In either word the first error stays.
 *   - bf16 = IEEE bfloat16 (2 bytes), fp32 = IEEE binary32, int32 = int32_t.
 *   - Shapes are listed outermost first; the last dimension is contiguous.
 *
 * Notation: B batch, H query heads, G KV heads (H % G == 0), D head dim (128),
 * Lc tokens per chunk, W window capacity in chunks, blk tokens per block
 * (64 or 128), nb = ceil(Lc / blk) blocks per chunk, Lslot = nb * blk tokens
 * per ring slot (the chunk padded to a whole number of blocks),
 * n_valid <= W chunks currently in the window, NKV = n_valid * nb.
 */
#ifndef UF_H
#define UF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA header. */
typedef struct CUstream_st *uf_stream_t;

typedef enum uf_status {
  UF_OK = 0,
  UF_EINVAL = 1,      /* bad argument: shape, alignment, NULL pointer, range   */
  UF_ECUDA = 2,       /* a CUDA runtime / driver call or launch failed         */
  UF_ETIMEOUT = 3,    /* a kernel pipeline wait exceeded its bound (device)    */
  UF_EBOUNDS = 4,     /* a kernel found an out-of-range index or state (device)*/
  UF_EUNSUPPORTED = 5 /* valid request this library does not implement         */
} uf_status;

/* Flags of uf_kv_append. */
#define UF_APPEND_REPLACE_NEWEST 1
#define UF_APPEND_ANCHOR 2

/*
 * Rolling KV window ("cache") descriptor: plain data, caller-owned.
 *
 * Ring of W slots, each holding one chunk of Lslot tokens.  Logical chunk
 * c (0 = oldest of the window) lives in physical slot (start + c) % W; logical
 * kv block j of the window is block j % nb of logical chunk j / nb.  The
 * physical order is never visible through the API.  Anchored window (HiStream,
 * aipapers summary, innovation 2: one anchor key frame plus a small cache of
 * neighbouring frames): after uf_kv_append(..., UF_APPEND_ANCHOR) on an empty
 * window, logical chunk 0 is that anchor, pinned in slot W - 1 and never
 * evicted or cropped, and chunks 1 .. n_valid - 1 are the most recent ones,
 * on a ring over slots 0 .. W - 2 (slot (start + c - 1) % (W - 1)).
 *
 *   k      device bf16 [B, G, W * Lslot, D] (token rows).
 *   v      device bf16 [B, G, D, W * Lslot] (transposed: each channel holds
 *          the window's tokens contiguously, the layout the PV product reads
 *          as a K-major tensor-core operand).  In both, the tokens past Lc
 *          inside a slot (the padding of the chunk's last block) are zeroed
 *          by uf_kv_append.
 *   kpool  device fp32 [B, G, W * nb, D]: mean of K over the true tokens of
 *          each block of each slot, written by uf_kv_append, read by
 *          uf_block_mask (pooling K once per chunk instead of once per call).
 *   meta   device int32[4] = {start, n_valid, append_counter, anchor}.  The
 *          window state lives on the device so that a captured sequence of
 *          calls stays correct when replayed.  Zeroed by uf_kv_reset.
 *   host_start, host_n_valid, host_anchor: host mirror of meta[0], meta[1],
 *          meta[3], updated by uf_kv_append / uf_kv_reset and used only for
 *          host-side argument checks.
 *   err    optional device int32: errors that kernels of calls on this window
 *          find (UF_EBOUNDS, UF_ETIMEOUT) are recorded here instead of in the
 *          library's device-wide word, so that concurrent windows do not share
 *          one flag.  The first error stays (a non-zero word is never
 *          overwritten); the caller reads and clears it in stream order.  NULL
 *          (set by uf_kv_cache_init) = the library's word.
 *
 * Sources: FlashDecoder (xllm-io blog), Sec. 3, Eq. 4 (cache shape
 * B x G x (W_frm L_frm) x D_h under grouped-query attention) and Algorithm 1
 * (the cache keeps the tail W_frm - 1 frames and appends the new frame);
 * HiStream (aipapers summary), innovation 2 (a fixed-size attention window
 * keeps the KV cache from growing with video length).
 */
typedef struct uf_kv_cache {
  void *k;
  void *v;
  float *kpool;
  int32_t *meta;
  int32_t B, G, D, W, Lc, blk;
  int32_t host_start, host_n_valid, host_anchor;
  int32_t *err;
} uf_kv_cache;

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t uf_version(void);

/*
 * Build identity, not a step of the method: the first 16 hex digits of the
 * SHA-256 over the library's sources (static string, never NULL; "unknown"
 * when built without it).  The Python binding compares it with the sources it
 * ships beside and refuses a library built from others.
 */
const char *uf_source_hash(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *uf_strerror(int32_t status);

/*
 * Byte sizes of the caller-owned buffers of a window with these dimensions:
 * *kv_bytes for each of k and v, *kpool_bytes for kpool, *meta_bytes for meta.
 * Any output pointer may be NULL.  Host only.  UF_EINVAL on bad dimensions
 * (D != 128, blk not 64 or 128, W < 1 or W > 64, any size < 1, or a buffer
 * larger than 2^40 bytes).
 */
int32_t uf_kv_cache_bytes(int32_t B, int32_t G, int32_t D, int32_t W, int32_t Lc, int32_t blk,
                          size_t *kv_bytes, size_t *kpool_bytes, size_t *meta_bytes);

/*
 * Fill *c with the given buffers and dimensions and mark the host mirror
 * empty.  Host only: does not touch device memory (call uf_kv_reset before the
 * first append).  UF_EINVAL on NULL / misaligned pointers or bad dimensions.
 */
int32_t uf_kv_cache_init(uf_kv_cache *c, void *k, void *v, float *kpool, int32_t *meta,
                         int32_t B, int32_t G, int32_t D, int32_t W, int32_t Lc, int32_t blk);

/*
 * Give the window its own device error word (err: device int32, 4-byte
 * aligned, caller-owned; NULL = back to the library's word).  Host only.
 */
int32_t uf_kv_cache_set_error_word(uf_kv_cache *c, int32_t *err);

/* Empty the window: zero meta on stream s and reset the host mirror. */
int32_t uf_kv_reset(uf_kv_cache *c, uf_stream_t s);

/*
 * Append the new chunk's keys and values to the window (FlashDecoder,
 * Algorithm 1: the cache becomes the tail of the previous window followed by
 * the new frame's K/V; Ultra Flash notes, key design 4: reuse of the last
 * denoising step's KV cache and adaptive cropping of the SR KV window).
 *
 *   k_new, v_new  device bf16 [B, Lc, G, D] (token-major, as a fused QKV
 *                 projection writes them).  Read only.
 *   keep_chunks   1..W: after the call the window holds at most keep_chunks
 *                 chunks; the oldest are evicted first (pass W for a plain
 *                 rolling window, less to crop it).
 *   flags         0, or UF_APPEND_REPLACE_NEWEST: overwrite the newest chunk
 *                 (a recomputation of the same chunk) instead of appending.
 *                 Rejected (UF_EINVAL) when the host mirror says the window is
 *                 empty; on the device an empty window turns it into an append.
 *                 Or UF_APPEND_ANCHOR: the chunk becomes the window's pinned
 *                 anchor (the window must be empty and W >= 2; not combined
 *                 with REPLACE_NEWEST).  While an anchor is pinned, keep_chunks
 *                 counts it (2..W) and eviction / cropping remove the oldest
 *                 of the other chunks; REPLACE_NEWEST on a window holding only
 *                 the anchor overwrites the anchor.
 *
 * Writes the chunk into its ring slot of k (BLGD -> BGLD) and v (BLGD ->
 * BGDL), zeroes the slot's padding rows, writes the slot's block means into
 * kpool and advances meta (the last thread block to finish commits the new
 * state).
 * One kernel launch.  Calls on the same cache must be stream-ordered.
 */
int32_t uf_kv_append(uf_kv_cache *c, const void *k_new, const void *v_new,
                     int32_t keep_chunks, int32_t flags, uf_stream_t s);

/*
 * Rotary position embedding with positions relative to the window
 * (FlashDecoder, long video decoding: RoPE positions are assigned relative to
 * the current window rather than the absolute frame index; Algorithm 1
 * offsets the positions by the frame index times the tokens per frame).  The
 * pages do not give the rotation's form; it is RoFormer's (Su et al. 2021):
 * channel pairs (x_2i, x_2i+1) rotate by pos * theta_i,
 * theta_i = base^(-2i / D).
 *
 * Rotary scores q(m) . k(n) depend only on m - n, and so do the pooled block
 * scores, so rotating every token at its position in the stream gives the
 * scores of window-relative positions exactly (up to rounding), and a stored
 * key never has to be rotated again when the window slides.  The caller gives
 * each chunk's stream position pos0 (e.g. chunk number * Lc) to both calls:
 *
 *   uf_kv_append_rope  uf_kv_append whose K rows are rotated at pos0 + token
 *                      (token = 0 .. Lc-1 within the chunk) before they are
 *                      stored and pooled; V is stored as is.
 *   uf_rope            x, y device bf16 [B, L, heads, D]: y = RoPE(x) with
 *                      token t at pos0 + t (y may be x: in place); for the
 *                      queries of the newest chunk, pos0 = that chunk's pos0.
 *
 * pos0 >= 0 and pos0 + Lc (resp. L) <= 2^40; base > 1 and finite (10000 is
 * RoFormer's).  Angles are formed and reduced in fp64 (within 1.2e-4 rad below
 * 2^40), sine / cosine in fp32, results rounded to bf16 (nearest even).
 * UF_EINVAL on bad arguments, otherwise as uf_kv_append.  One kernel launch
 * each.
 */
int32_t uf_kv_append_rope(uf_kv_cache *c, const void *k_new, const void *v_new,
                          int32_t keep_chunks, int32_t flags, int64_t pos0, float base,
                          uf_stream_t s);
int32_t uf_rope(const void *x, void *y, int32_t B, int32_t L, int32_t heads, int64_t pos0,
                float base, uf_stream_t s);

/*
 * 3-D block token order (Ultra Flash notes, Method, key design 3: the
 * spatio-temporal token grid is cut into non-overlapping (2, 8, 8) blocks).
 * A chunk's Lc = T * Hg * Wg tokens form a (T, Hg, Wg) grid in row-major
 * order; the tiled order takes tiles of (bt, by, bx) -- (2, 8, 8) on the
 * pages -- in row-major tile order and the tokens inside each tile in
 * row-major order, with the tiles at the grid's far edges clipped.  In the
 * tiled order every full tile is one run of bt * by * bx tokens, so with
 * blk = bt * by * bx the library's blocks are the pages' 3-D blocks wherever
 * the grid allows.
 *
 *   uf_tile_tokens      x, y device bf16 [B, T * Hg * Wg, heads, D], not
 *                       overlapping: inverse = 0 writes x in tiled order,
 *                       inverse = 1 writes tiled x back in row-major order
 *                       (for the queries before the mask and attention, and
 *                       for O after).
 *   uf_kv_append_tiled  uf_kv_append whose K and V rows are gathered in tiled
 *                       order (T * Hg * Wg must equal Lc): the window holds
 *                       the chunk in tiled order without a separate pass.
 *
 * UF_EINVAL on bad arguments.  One kernel launch each.
 */
int32_t uf_tile_tokens(const void *x, void *y, int32_t B, int32_t T, int32_t Hg, int32_t Wg,
                       int32_t heads, int32_t bt, int32_t by, int32_t bx, int32_t inverse,
                       uf_stream_t s);
int32_t uf_kv_append_tiled(uf_kv_cache *c, const void *k_new, const void *v_new,
                           int32_t keep_chunks, int32_t flags, int32_t T, int32_t Hg, int32_t Wg,
                           int32_t bt, int32_t by, int32_t bx, uf_stream_t s);

/*
 * Dynamic block mask of the newest chunk's queries (Ultra Flash notes, Method,
 * key design 3: tokens are cut into non-overlapping blocks; queries and keys
 * are mean-pooled per block; blocks are scored by the dot product of the
 * pooled query and key; each head keeps its top-k highest-scoring blocks).
 *
 *   q       device bf16 [B, Lc, H, D]: queries of the newest chunk of the
 *           window (the chunk appended last).  H % c->G == 0.
 *   k       kept blocks per q-block, counting the diagonal; 1 <= k <= W * nb.
 *           On the device it is clamped to NKV (first chunks of a stream).
 *   idx     device int32 [B, H, nb, k] out: logical kv block ids of the kept
 *           blocks of each (b, h, q-block i) row, ascending; entries past
 *           cnt are set to -1.
 *   cnt     device int32 [B, H, nb] out: kept blocks per row = min(k, NKV).
 *   scores  optional device fp32 [B, H, nb, W * nb] out (NULL = not written):
 *           pooled scores mean(q_i) . mean(k_j) / sqrt(D) in logical order;
 *           columns >= NKV are not written.
 *
 * Selection rule per row: the diagonal block d_i = (n_valid - 1) * nb + i is
 * always kept; the other blocks are ranked by (score descending, logical id
 * ascending) and the first k - 1 are kept.  Pooling means divide by the true
 * token count of each block (the chunk's last block may be partial).  Scores
 * are computed in fp32.  UF_EUNSUPPORTED when W * nb > 1024.  One kernel launch.
 */
int32_t uf_block_mask(const void *q, int32_t H, const uf_kv_cache *c, int32_t k,
                      int32_t *idx, int32_t *cnt, float *scores, uf_stream_t s);

/* uf_block_mask_local flag: keep the local band only (no scored blocks). */
#define UF_MASK_LOCAL_ONLY 1

/*
 * Block mask with a local sliding-window band (Ultra Flash notes, Method, key
 * design 3: each attention layer combines a local sliding-window mask with the
 * temporal causal mask, then keeps each head's top-k blocks; the ablation
 * table's row that swaps adaptive top-k for a fixed local window is the band
 * alone).
 * The pages do not define the band's shape; here it is the run of logical
 * kv blocks within `local` of the diagonal, [d_i - local, d_i + local]
 * clipped to [0, NKV).
 *
 *   local   band radius in blocks, >= 0, with 2 * local + 1 <= k;
 *           uf_block_mask(...) is uf_block_mask_local(..., local = 0, flags = 0).
 *   flags   0: keep the band, then the other blocks ranked by (score
 *           descending, logical id ascending) until the row has min(k, NKV)
 *           blocks; UF_MASK_LOCAL_ONLY: keep the band only (cnt = its size).
 *   other arguments, outputs and errors as uf_block_mask.
 */
int32_t uf_block_mask_local(const void *q, int32_t H, const uf_kv_cache *c, int32_t k,
                            int32_t local, int32_t flags, int32_t *idx, int32_t *cnt,
                            float *scores, uf_stream_t s);

/*
 * Block-sparse chunk-causal attention (Ultra Flash notes, key design 3:
 * attention computed only over the kept blocks; FlashDecoder Sec. 3.3:
 * causality by processing order, no token mask inside the window; Eq. 4:
 * grouped-query KV heads).
 *
 *   q      device bf16 [B, Lc, H, D]: queries of the newest chunk.
 *   idx    device int32 [B, H, nb, k] logical kv block ids (any order, no
 *          duplicates; as written by uf_block_mask), or NULL for dense
 *          attention over every block of the window (density 1.0).
 *   cnt    device int32 [B, H, nb]: number of valid entries of each idx row
 *          (1..k); NULL = every row has k entries.  Ignored when idx is NULL.
 *   k      row stride of idx (ignored when idx is NULL).
 *   scale  softmax scale applied to q . k (1 / sqrt(D) for standard attention).
 *   o      device bf16 [B, Lc, H, D] out: sum_j softmax_j(scale q.k_j) v_j over
 *          the valid tokens of the kept blocks; query head h reads KV head
 *          h / (H / G).
 *   lse    optional device fp32 [B, H, Lc] out: natural-log
 *          log-sum-exp of scale * q . k over the same tokens (NULL = skip).
 *
 * Device checks: an idx entry outside [0, NKV) is replaced by the row's
 * diagonal block and UF_EBOUNDS is recorded; a row with cnt < 1 gets O = 0,
 * LSE = -inf and UF_EBOUNDS.  One kernel launch (tcgen05 tensor cores, TMA)
 * with at most one thread block per SM, each looping over (b, h, q-block)
 * items.  q and o must be 16-byte aligned.  UF_EUNSUPPORTED when the library's kernel
 * was compiled to a register count its warp specialisation does not expect.
 */
int32_t uf_block_sparse_attn(const void *q, int32_t H, const uf_kv_cache *c,
                             const int32_t *idx, const int32_t *cnt, int32_t k, float scale,
                             void *o, float *lse, uf_stream_t s);

/*
 * Balanced variant of uf_block_sparse_attn, for workloads with few work items
 * per SM (grouped-query decoder steps, small chunks): the full rounds of
 * (b, h, q-block) items go to the SMs whole, and the positions (item, kept
 * block) of the remaining items, every item counted at its nominal length
 * (dense: every block of the window; sparse: the row stride k), are cut into
 * one contiguous range of equal length per SM, so every SM computes the same
 * number of kept blocks.  An item whose blocks fall into several
 * ranges is computed in parts; each part writes its unnormalised O, row max
 * and row sum to the workspace, and the part that finishes last merges them
 * (log-sum-exp, in fp32) and writes O and LSE.  No thread block waits for
 * another.  Softmax attention is exact on its kept set, so the result is
 * uf_block_sparse_attn's up to fp32 rounding (Ultra Flash notes, key design
 * 3; FlashDecoder Sec. 3, Eq. 4).
 *
 *   workspace        device memory of at least uf_attn_workspace_bytes()
 *                    bytes, 16-byte aligned, caller-owned; its contents need
 *                    no initialisation (the call zeroes the counters it uses
 *                    on stream s before the kernel).  Calls that may run at
 *                    the same time need separate workspaces.
 *   workspace_bytes  its size.
 *   other arguments, outputs and errors as uf_block_sparse_attn.
 *
 * Where the plain schedule is already even -- at least 8 items per SM, or
 * its last round of items within 10% of full -- it is used unchanged (the
 * workspace is not touched).  One memset and one kernel launch.
 */
int32_t uf_block_sparse_attn_balanced(const void *q, int32_t H, const uf_kv_cache *c, const int32_t *idx,
                                      const int32_t *cnt, int32_t k, float scale, void *o, float *lse,
                                      void *workspace, size_t workspace_bytes, uf_stream_t s);

/*
 * uf_block_sparse_attn_balanced for callers that cannot allocate device
 * memory.  The pages have no counterpart to this call: it only changes where
 * the balanced schedule keeps its scratch data.  Some callers cannot call
 * cudaMalloc or hand the library a buffer of their own: a plugin inside a host
 * framework that owns every device byte through its own pool, a real-time
 * streaming loop that must not allocate after start-up (an allocation can
 * synchronise the device and stall the stream), or a process that has
 * reserved all free memory for its KV windows.  This call allocates nothing:
 * it calls no cudaMalloc, cudaFree or allocating library routine, and the
 * scratch is a fixed array of 21,299,968 bytes compiled into the library (two
 * 65 KB partial results per SM for up to 160 SMs, plus counters), which every
 * device that loads the library holds until the process exits.
 *
 *   arguments, outputs and errors as uf_block_sparse_attn_balanced, without
 *   workspace and workspace_bytes.  UF_EUNSUPPORTED when the current device
 *   has more than 160 SMs (its scratch would not fit the array).
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  All calls on a device share the one array, and each call clears
 * the counters it needs on stream s before its kernel: calls that may run on
 * the GPU at the same time (other streams, other host threads) race on it and
 * must be ordered by the caller.
 */
int32_t uf_block_sparse_attn_balanced_noalloc(const void *q, int32_t H, const uf_kv_cache *c,
                                              const int32_t *idx, const int32_t *cnt, int32_t k, float scale,
                                              void *o, float *lse, uf_stream_t s);

/*
 * Workspace size of uf_block_sparse_attn_balanced on the current device
 * (two partial results of 65 KB per SM plus counters; 19.7 MB on a 148-SM
 * B200), into *bytes.  Host only.
 */
int32_t uf_attn_workspace_bytes(size_t *bytes);

/*
 * FP8-score variant, append side (FlashDecoder, inference optimisations:
 * statically calibrated FP8).  uf_kv_append(c, k_new, v_new, keep_chunks,
 * flags, s) that also writes an e4m3 copy of each appended K row:
 *
 *   k8       device uint8 [B, G, W * Lslot, D], caller-owned, same slots and
 *            token rows as c->k: k8 = e4m3(K / k_scale), rounded to nearest
 *            (ties to even) from the fp32 product K * (1 / k_scale) and
 *            saturated at +-448; padding rows get 0.  Must be 16-byte aligned.
 *   k_scale  static per-tensor K scale, finite and > 0 (for instance
 *            amax(K) / 448 of a calibration chunk).
 *
 * Use the same k8 buffer and k_scale for every append of a window; chunks
 * appended without it have no e4m3 copy.  No RoPE or tile-order form.
 * Errors as uf_kv_append, plus UF_EINVAL for a NULL or unaligned k8 or a bad
 * k_scale.
 */
int32_t uf_kv_append_fp8k(uf_kv_cache *c, void *k8, float k_scale, const void *k_new,
                          const void *v_new, int32_t keep_chunks, int32_t flags, uf_stream_t s);

/*
 * FP8-score variant, attention side: uf_block_sparse_attn with the scores
 * q . k taken on the tensor cores in e4m3 x e4m3 with fp32 accumulation:
 *
 *   s = scale * q_scale * k_scale * (e4m3(q / q_scale) . k8)
 *
 * where e4m3(q / q_scale) rounds the fp32 product q * (1 / q_scale) to
 * nearest (ties to even, saturated at +-448) and k8 is the buffer written by
 * uf_kv_append_fp8k with k_scale.  The softmax (fp32), the probabilities
 * (bf16) and the PV product (bf16 V) are those of uf_block_sparse_attn.
 *
 *   k8       device uint8 [B, G, W * Lslot, D] as above, 16-byte aligned.
 *   q_scale  static per-tensor query scale, finite and > 0.
 *   k_scale  the scale the window's k8 rows were written with.
 *   other arguments, outputs and errors as uf_block_sparse_attn.
 */
int32_t uf_block_sparse_attn_fp8k(const void *q, int32_t H, const uf_kv_cache *c, const void *k8,
                                  float q_scale, float k_scale, const int32_t *idx,
                                  const int32_t *cnt, int32_t k, float scale, void *o, float *lse,
                                  uf_stream_t s);

/*
 * Stream-ordered error read (failure detection without a device
 * synchronisation): enqueue on s one single-thread kernel that takes the
 * library's device-wide error word of the current device (the first error a
 * kernel of a window without its own word recorded since the last clear),
 * clears it, and stores it into *dev_err_word unless that already holds a
 * non-zero code (so one word collects the first error over many calls or
 * graph replays; the caller zeroes it).  dev_err_word: device int32, 4-byte
 * aligned, caller-owned.  Never synchronises; can be captured in a CUDA
 * graph.  UF_EINVAL on a NULL or misaligned pointer, UF_ECUDA on a launch
 * failure.
 */
int32_t uf_check_error(int32_t *dev_err_word, uf_stream_t s);

/*
 * Read the device-side error word of the current device (the first error a
 * kernel recorded since the last clear) into *status; clear it if `clear` is
 * non-zero.  Synchronises the device (this is the one call that does).
 */
int32_t uf_get_error(int32_t *status, int32_t clear);

/*
 * Text of the last CUDA error that made a call of this thread return
 * UF_ECUDA (static string, never NULL; "no error" if none).
 */
const char *uf_last_cuda_error(void);

/*
 * Set the bound on every pipeline wait inside the kernels, in SM clock cycles
 * (default 2^31, about one second at B200 clocks).  A wait that reaches the
 * bound records UF_ETIMEOUT and makes its kernel return early.  Host only;
 * applies to launches made after the call.  UF_EINVAL if cycles < 1000.
 */
int32_t uf_set_wait_limit(int64_t cycles);

/*
 * Measurement hook (the pages have no counterpart: it serves the benchmark's
 * clock record).  dev_counters: NULL (off, the default) or a device uint64[2],
 * 8-byte aligned, owned by the caller, who zeroes it.  While set, every thread
 * block of every attention launch made after the call adds, when it ends, the
 * SM clock cycles (clock64) and the global-timer nanoseconds that passed since
 * it started to dev_counters[0] and dev_counters[1] (atomic adds).  The ratio
 * cycles / nanoseconds is the attention kernel's effective SM clock in GHz,
 * averaged over its thread blocks: the clock it really ran at, which a sampled
 * clock reading taken every few hundred milliseconds does not show.  The
 * buffer must stay valid until every such launch has completed; set NULL to
 * stop.  Host only; one setting for all devices and threads.  UF_EINVAL on a
 * misaligned pointer.
 */
int32_t uf_set_clock_counters(uint64_t *dev_counters);

/*
 * Self-test of the bounded-wait path: launch one thread that waits on a
 * pipeline barrier that nothing will ever complete, with a bound of `cycles`.
 * The kernel records UF_ETIMEOUT and returns; it never hangs.  For tests.
 */
int32_t uf_debug_wait_timeout(int64_t cycles, uf_stream_t s);

#ifdef __cplusplus
}
#endif

#endif /* UF_H */
