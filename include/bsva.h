/*
 * bsva.h -- C ABI of the block-sparse INT8 video attention library (sm_100a).
 *
 * The method: every 128-token query block scores each 64-token key block with
 * a cheap proxy on per-block INT8 Q/K, keeps a block exact iff its score is at
 * least mean + tau*std over the query block's row (the Sol rule), runs
 * FlashAttention-style online softmax over the kept blocks only and adds one
 * (1x64) or two (2x32) centroid terms for every skipped block
 * ("Configure Sol Sparse Attention", How it works; The inputs that matter).
 * A second entry point runs an explicit logical 128x128 block mask such as
 * FlashVSR's LCSA streaming mask, with no centroids ("FlashVSR Sparge
 * Attention", intro and How it works; "FlashVSR Kitchen Sparse Attention",
 * intro). A third runs the residual mode of a static virtual K/V context:
 * the physical keys exact, every added virtual slice as centroid terms
 * ("Configure H3 Static Virtual KV", the mode list).
 *
 * Conventions shared by every entry point
 *  - Tensors are contiguous row-major: Q, O [B, H, Lq, d]; K, V [B, H, Lk, d].
 *    bf16 buffers are passed as void pointers (raw IEEE bfloat16 bits).
 *  - nQB = ceil(Lq/128) query blocks, nKB = ceil(Lk/64) key blocks,
 *    nLK = ceil(Lk/128) logical key blocks of the mask entry.
 *  - d is 64 or 128. n_prefix is a multiple of 128 (0 = no dense prefix).
 *  - Device pointers only, 16-byte aligned; the caller owns every buffer,
 *    including the workspace. The library never allocates, frees or
 *    synchronises (bsva_check_status is the one call that synchronises).
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) of the current device.
 *  - Every call returns a status code. On a validation failure nothing is
 *    launched and no output is touched; bsva_last_error() then holds a
 *    message for the calling thread. There is no fallback path.
 */
#ifndef BSVA_H
#define BSVA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSVA_ABI_VERSION 5

enum bsva_status {
  BSVA_OK = 0,
  BSVA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misalignment      */
  BSVA_ERR_UNSUPPORTED = 2,    /* device is not sm_100, d not in {64, 128}  */
  BSVA_ERR_WORKSPACE = 3,      /* workspace missing or too small            */
  BSVA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed      */
  BSVA_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up        */
  BSVA_ERR_DEVICE_BOUNDS = 6   /* a device-side index check failed (only the
                                  BSVA_DEVICE_CHECKS build checks)          */
};

/* Element type of the attention output `out`. */
enum bsva_out_dtype {
  BSVA_OUT_BF16 = 0,   /* bf16 [B,H,Lq,d]                                   */
  BSVA_OUT_F32 = 1     /* fp32 [B,H,Lq,d]; bf16 output equals its rounding  */
};

typedef struct CUstream_st* bsva_stream_t;

typedef struct bsva_shape {
  int B, H;      /* batch, heads                                  */
  int Lq, Lk;    /* query and key lengths (tokens)                */
  int d;         /* head dim: 64 or 128                           */
  int n_prefix;  /* leading tokens kept dense (multiple of 128)   */
} bsva_shape;

/* ABI version of the loaded library; loaders compare it with BSVA_ABI_VERSION
 * ("FlashVSR Kitchen Sparse Attention", When it bites: ABI check on load). */
int bsva_abi_version(void);

/* 1 if this library was built with BSVA_DEVICE_CHECKS (libbsva_checked.so), else 0.
 * In that build the kernels check every index they take from caller data (kept
 * counts and kept lists of a route, table rows) before using it; a value out of
 * range is recorded in the workspace status word (reported by bsva_check_status
 * as BSVA_ERR_DEVICE_BOUNDS) and clamped into range, so that no access leaves its
 * buffer; the outputs of that call are then invalid. The checks cost time; the
 * default build does not make them. */
int bsva_device_checks(void);

/* Message for the last failed call on this thread ("" if none). The pointer
 * stays valid until the next call on the same thread. */
const char* bsva_last_error(void);

/* Bytes of device workspace needed by sparse_attn_fwd (centroid_mode 1 or 2)
 * or masked_block_attn_fwd (centroid_mode 0) for shape s; 0 on a bad shape.
 * The first 256 bytes hold the device status word and must be zero before the
 * first call (bsva_check_status clears them). A workspace of this size also
 * serves sparse_attn_route: its score region comes right after the status
 * word and no other call writes it. */
size_t bsva_workspace_bytes(bsva_shape s, int centroid_mode);

/* Bytes of device workspace sparse_attn_route needs alone (status word plus
 * the fp64 score matrix, BH*nQB*nKB*8 bytes); 0 on a bad shape. */
size_t bsva_route_workspace_bytes(bsva_shape s);

/* Per-block symmetric INT8 quantisation and integer sum-pools, alone.
 * ("Configure Sol Sparse Attention", How it works: the proxy and the exact
 * path read the same prequantized INT8 Q/K.)
 *   q, k      in : bf16 [B,H,Lq,d], [B,H,Lk,d]
 *   q8, k8    out: int8, same shapes. Per block: s = fl32(amax/127),
 *                  x8 = clamp(rint_half_even(fl32(x/s)), -127, 127); 0 if s = 0.
 *   q_scale   out: fp32 [B,H,nQB]  (128-row Q blocks)
 *   k_scale   out: fp32 [B,H,nKB]  (64-row K blocks)
 *   q_pool    out: int32 [B,H,nQB,d]   column sums of each Q block's INT8 rows
 *   k_pool    out: int32 [B,H,nKB,2,d] column sums of each 32-row half of
 *                  each K block (a tail block's halves are rows [0,min(32,n))
 *                  and [32,n); an empty half is 0).                          */
int bsva_quantize_qk(bsva_shape s, const void* q, const void* k,
                     int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                     int32_t* q_pool, int32_t* k_pool, bsva_stream_t stream);

/* Quantise + proxy score + Sol routing ("Configure Sol Sparse Attention",
 * How it works; The inputs that matter: routing_threshold, prefix_policy).
 * Runs bsva_quantize_qk, then for every query-block row i:
 *   s_ij = fl64(fl64(dot_ij * k_scale_j) / n_j),
 *   dot_ij = sum_c q_pool_i[c] * (k_pool_j0[c] + k_pool_j1[c]) (exact int64),
 *   mu, sigma = population mean and std of s_ij over the routed key blocks
 *   (those starting at or after n_prefix), T = mu + tau*sigma, keep iff s >= T.
 * Rows of query blocks starting before n_prefix, rows whose routed scores are
 * all equal, and tau = -inf keep every block; key blocks before n_prefix are
 * always kept.
 *   tau        routing threshold (the pages' default is 1.0; -INFINITY = dense)
 *   kept_mask  out: uint8 [B,H,nQB,nKB], 1 = exact
 *   kept_idx   out: int32 [B,H,nQB,nKB], kept key-block indices ascending;
 *                   entries at and after kept_cnt are unspecified
 *   kept_cnt   out: int32 [B,H,nQB]
 *   row_stats  out, nullable: fp64 [B,H,nQB,3] = (mu, sigma, T); T = -inf for
 *                   rows that keep every block.
 *   workspace  device scratch of >= bsva_route_workspace_bytes(s) bytes,
 *              256-aligned, owned by the caller (the scores s_ij are staged
 *              there); BSVA_ERR_WORKSPACE if missing or too small.         */
int sparse_attn_route(bsva_shape s, const void* q, const void* k, double tau,
                      int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                      int32_t* q_pool, int32_t* k_pool,
                      uint8_t* kept_mask, int32_t* kept_idx, int32_t* kept_cnt,
                      double* row_stats, void* workspace, size_t workspace_bytes,
                      bsva_stream_t stream);

/* Quantise + proxy score + fixed-sparsity top-k routing ("Ref2VA VSA",
 * 2-stage attention patch: top-k pruning applies only to the generated-video
 * key tiles and the conditioning prefix stays dense; Wiring it into a
 * workflow: the recipe runs at sparsity 0.75). The pages rank tiles with a
 * learned gate; this entry ranks them by the same proxy scores s_ij as
 * sparse_attn_route, so its outputs feed sparse_attn_fwd unchanged (skipped
 * blocks keep their centroid terms).
 * Each row of a query block starting at or after n_prefix keeps
 *   k = |R| - floor(sparsity * |R|)   (fp64 product)
 * of its routed key blocks R (those starting at or after n_prefix): the k
 * largest scores, ties to the lower key-block index. Rows before n_prefix and
 * rows with k = |R| keep every block; key blocks before n_prefix are always
 * kept.
 *   sparsity   skipped fraction of the routed blocks, in [0, 1]
 *              (BSVA_ERR_INVALID_ARG otherwise, NaN included)
 *   row_stats  out, nullable: (mu, sigma, T) with T the k-th largest routed
 *              score, -inf when every routed block is kept, +inf when k = 0.
 *   Every other argument, the workspace and the outputs are as for
 *   sparse_attn_route.                                                       */
int sparse_attn_route_topk(bsva_shape s, const void* q, const void* k, double sparsity,
                           int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                           int32_t* q_pool, int32_t* k_pool,
                           uint8_t* kept_mask, int32_t* kept_idx, int32_t* kept_cnt,
                           double* row_stats, void* workspace, size_t workspace_bytes,
                           bsva_stream_t stream);

/* Sparse attention over the routed blocks plus centroid terms
 * ("Configure Sol Sparse Attention", How it works: skipped blocks are
 * replaced by one 64-token centroid, or two 32-token centroids in 2x32 mode,
 * inside the same online softmax).
 *   Inputs are the outputs of sparse_attn_route (k_pool feeds the centroid
 *   keys; v is bf16 [B,H,Lk,d]).
 *   Exact term (row r, key t of kept block j): logit = sq_i*sk_j*scale*(q8_r . k8_t).
 *   Centroid term (group g of skipped block j): kbar = sk_j*pool_g/|g|,
 *     logit = sq_i*scale*(q8_r . kbar) + ln|g|, value = mean of V over g.
 *   centroid_mode  1 = 1x64, 2 = 2x32
 *   softmax_scale  <= 0 selects 1/sqrt(d)
 *   out_dtype      BSVA_OUT_BF16 or BSVA_OUT_F32 (element type of out)
 *   out  out: [B,H,Lq,d]; lse out, nullable: fp32 [B,H,Lq] (natural log)
 *   workspace      >= bsva_workspace_bytes(s, centroid_mode) bytes, 256-aligned */
int sparse_attn_fwd(bsva_shape s, const int8_t* q8, const float* q_scale,
                    const int8_t* k8, const float* k_scale,
                    const int32_t* k_pool, const void* v,
                    const uint8_t* kept_mask, const int32_t* kept_idx,
                    const int32_t* kept_cnt, int centroid_mode,
                    float softmax_scale, int out_dtype, void* out, float* lse,
                    void* workspace, size_t workspace_bytes,
                    bsva_stream_t stream);

/* The two halves of sparse_attn_fwd, for callers that reuse one K/V (and so
 * one centroid table) across several query batches, or that time the phases:
 * sparse_attn_fwd(...) launches exactly bsva_build_centroids(...) followed by
 * bsva_sparse_attn_core(...).
 * bsva_build_centroids writes the centroid table of (k_pool, k_scale, v) into
 * the workspace: per group, the INT8 key rows (hi, lo) with pool = 128*hi + lo,
 * the value rows (bf16(vbar), bf16(vbar - bf16(vbar))), sk_j/|g| and log2|g|.
 * bsva_sparse_attn_core runs the attention kernel and reads that table; its
 * arguments mean what they mean for sparse_attn_fwd.                        */
int bsva_build_centroids(bsva_shape s, const int32_t* k_pool,
                         const float* k_scale, const void* v, int centroid_mode,
                         void* workspace, size_t workspace_bytes,
                         bsva_stream_t stream);

int bsva_sparse_attn_core(bsva_shape s, const int8_t* q8, const float* q_scale,
                          const int8_t* k8, const float* k_scale, const void* v,
                          const uint8_t* kept_mask, const int32_t* kept_idx,
                          const int32_t* kept_cnt, int centroid_mode,
                          float softmax_scale, int out_dtype, void* out,
                          float* lse, void* workspace, size_t workspace_bytes,
                          bsva_stream_t stream);

/* The LCSA logical block mask built on the device from frame geometry
 * ("FlashVSR Sparge Attention", intro: local causal sparse attention, each
 * query block attends only to a small, locally causal set of key blocks; the
 * sampler builds that mask). A logical 128-token block belongs to the frame
 * of its first token, f(x) = floor(128 x / frame_tokens); key block x_k is
 * allowed for query block x_q iff f(x_q) - window_frames <= f(x_k) <= f(x_q).
 *   mask   out: uint8 [batch, 1, ceil(Lq/128), ceil(Lk/128)] (every batch
 *          entry the same), ready for masked_block_attn_fwd with
 *          mask_heads = 1.
 *   BSVA_ERR_INVALID_ARG for Lq, Lk, batch or frame_tokens < 1,
 *   window_frames < 0 or a NULL mask; asynchronous on stream otherwise.     */
int bsva_build_lcsa_mask(int Lq, int Lk, int frame_tokens, int window_frames,
                         int batch, uint8_t* mask, bsva_stream_t stream);

/* Attention over an explicit logical block mask, exact terms only
 * ("FlashVSR Sparge Attention", How it works: routing on logical
 * 128-query x 128-key blocks, converted to the kernel's physical geometry
 * after routing, one sparse call).
 *   block_mask  uint8 [B, mask_heads, nQB, nLK]; mask_heads is 1 (shared by
 *               all heads) or H. Physical 64-key block j of query block i runs
 *               iff block_mask[b, h % mask_heads, i, j/2] != 0.
 *   A query row with no allowed block gets out = 0 and lse = -inf.
 *   workspace   >= bsva_workspace_bytes(s, 0) bytes, 256-aligned.
 *   Other arguments as in sparse_attn_fwd.                                   */
int masked_block_attn_fwd(bsva_shape s, const int8_t* q8, const float* q_scale,
                          const int8_t* k8, const float* k_scale,
                          const void* v, const uint8_t* block_mask,
                          int mask_heads, float softmax_scale, int out_dtype,
                          void* out, float* lse, void* workspace,
                          size_t workspace_bytes,
                          bsva_stream_t stream);

/* Per-block symmetric INT8 quantisation of V with the K quantiser (64-row
 * blocks, s = fl32(amax/127), x8 = rint_half_even(fl32(x/s))), the format of
 * an INT8 K/V cache ("FlashVSR Kitchen Sparse Attention", intro: the
 * streaming cache keeps K and V as INT8).
 *   v        bf16 [B,H,Lk,d]
 *   v8       out: int8 [B,H,Lk,d]
 *   v_scale  out: fp32 [B,H,nKB]                                             */
int bsva_quantize_v(bsva_shape s, const void* v, int8_t* v8, float* v_scale,
                    bsva_stream_t stream);

/* masked_block_attn_fwd on an INT8 V ("FlashVSR Kitchen Sparse Attention",
 * intro: the INT8 cache is fed straight to the kernel, with no
 * full-precision rebuild of K and V). The output is softmax attention over
 * the dequantised values v8 * v_scale[block]; in the kernel the block scale
 * rides in the weights, P' = P * s_j, the INT8 tile is widened to f16 in
 * shared memory (exact), and PV runs as f16 x f16 with fp32 accumulation.
 *   v8, v_scale  as written by bsva_quantize_v
 *   Every other argument as in masked_block_attn_fwd.                        */
int masked_block_attn_fwd_v8(bsva_shape s, const int8_t* q8, const float* q_scale,
                             const int8_t* k8, const float* k_scale,
                             const int8_t* v8, const float* v_scale,
                             const uint8_t* block_mask, int mask_heads,
                             float softmax_scale, int out_dtype, void* out,
                             float* lse, void* workspace, size_t workspace_bytes,
                             bsva_stream_t stream);

/* Workspace bytes for virtual_kv_residual_fwd (0 on a bad shape or
 * geometry); independent of the source map and of n_virtual. */
size_t bsva_virtual_kv_workspace_bytes(bsva_shape s, int slice_tokens,
                                       int n_src_slices, int centroid_mode);

/* Residual mode of a static virtual K/V context ("Configure H3 Static Virtual
 * KV", the mode list and "What virtual means physically"): queries and
 * outputs stay on the physical rows; every physical key block is an exact
 * term (the real slices stay dense); each added virtual slice l re-reads
 * source slice src_map[l] through the logical source map and enters the same
 * online softmax only as skipped-block centroid terms (2x32 on the page: two
 * 32-token centroids per 64-token block, log-count |g| in the logit). Nothing
 * of the virtual context is materialised: the centroid table is built once
 * per source slice and every virtual tile reads it through the map.
 *   q8, q_scale, k8, k_scale  physical Q/K as written by bsva_quantize_qk
 *   v              bf16 [B,H,Lk,d], the physical values
 *   slice_tokens   tokens per latent-time slice, a positive multiple of 64,
 *                  so a slice is a whole number of key blocks
 *   n_src_slices   slices in the source, which holds n_src_slices *
 *                  slice_tokens tokens per head
 *   src_k_scale, src_k_pool  fp32 [B,H,nSB], int32 [B,H,nSB,2,d] of the
 *                  source keys as written by bsva_quantize_qk (nSB =
 *                  n_src_slices * slice_tokens / 64). With Lk = n_src_slices *
 *                  slice_tokens the physical k_scale and k_pool serve.
 *   src_v          bf16 [B,H,n_src_slices*slice_tokens,d] source values (v
 *                  itself in that case). The keys are used as given: a
 *                  temporal phase wanted on a virtual slice must already be
 *                  in the source passed here.
 *   src_map        HOST array of n_virtual entries in [0, n_src_slices);
 *                  read during the call only. n_virtual in [0, 32]; 0 gives
 *                  dense exact attention over the physical keys.
 *   centroid_mode  2 (2x32) or 1 (1x64)
 *   workspace      >= bsva_virtual_kv_workspace_bytes(...) bytes, 256-aligned.
 *   Other arguments as in sparse_attn_fwd. BSVA_ERR_INVALID_ARG for a bad
 *   geometry, map entry or pointer; nothing is launched then.               */
int virtual_kv_residual_fwd(bsva_shape s, const int8_t* q8, const float* q_scale,
                            const int8_t* k8, const float* k_scale,
                            const void* v, int slice_tokens, int n_src_slices,
                            const float* src_k_scale, const int32_t* src_k_pool,
                            const void* src_v, const int* src_map, int n_virtual,
                            int centroid_mode, float softmax_scale, int out_dtype,
                            void* out, float* lse, void* workspace,
                            size_t workspace_bytes, bsva_stream_t stream);

/* Per-block INT8 quantisation of Q alone (128-row blocks, the quantiser of
 * bsva_quantize_qk), for queries that attend to keys quantised elsewhere,
 * such as the INT8 streaming cache below. s.Lk is not used.
 *   q        bf16 [B,H,Lq,d]
 *   q8       out: int8 [B,H,Lq,d];  q_scale out: fp32 [B,H,nQB]
 *   q_pool   out: int32 [B,H,nQB,d] (column sums of each block's codes)         */
int bsva_quantize_q(bsva_shape s, const void* q, int8_t* q8, float* q_scale,
                    int32_t* q_pool, bsva_stream_t stream);

/* INT8 streaming K/V cache in 128-row slabs ("FlashVSR Kitchen Sparse
 * Attention", intro: the streaming modes keep a sliding cache of past K and V
 * as INT8 and hand bounded 128-row slabs straight to the sparse kernel, with
 * no full-precision rebuild; When it bites: the INT8 path needs an INT8 cache
 * to feed). Per (batch, head) the cache is a ring of n_slots slabs: logical
 * slab x (0 = the oldest live slab) sits in slot (first + x) % n_slots. A slab
 * holds up to 128 consecutive tokens of one appended chunk; its K and V are
 * quantised in 64-row blocks with the K quantiser (s = fl32(amax/127), codes
 * rint_half_even(fl32(x/s)) over the block's valid rows).
 * The caller allocates the device buffers (zero-initialised or not: nothing is
 * read before it is written) and owns the struct; bsva_kv_cache_append updates
 * first and count. Start with first = count = 0. */
typedef struct bsva_kv_cache {
  int B, H, d;          /* heads and head dim of every chunk (d = 64 or 128)      */
  int n_slots;          /* capacity in slabs, >= 1                                */
  int8_t* k8;           /* device int8 [B, H, n_slots*128, d]                     */
  float* k_scale;       /* device fp32 [B, H, n_slots*2], one per 64-row block    */
  int8_t* v8;           /* device int8 [B, H, n_slots*128, d]                     */
  float* v_scale;       /* device fp32 [B, H, n_slots*2]                          */
  int32_t* slab_rows;   /* device int32 [n_slots]: valid rows of each slot's slab */
  int first;            /* slot of the oldest live slab                           */
  int count;            /* live slabs                                             */
} bsva_kv_cache;

/* Appends a chunk of Lc >= 1 new tokens, k and v bf16 [B, H, Lc, d]. The chunk
 * becomes ceil(Lc/128) slabs, the last one holding Lc - 128*(ceil(Lc/128)-1)
 * rows. When the ring would overflow, the oldest slabs are evicted first; a
 * chunk longer than the whole ring keeps only its last n_slots slabs.
 * c->first and c->count are updated on the host when the call returns; the
 * quantisation runs on `stream`. Returns BSVA_ERR_INVALID_ARG for a bad
 * geometry or pointer, leaving the cache untouched. */
int bsva_kv_cache_append(bsva_kv_cache* c, const void* k, const void* v, int Lc,
                         bsva_stream_t stream);

/* Workspace bytes of masked_block_attn_fwd_kvcache for Lq query tokens against
 * the cache's current live slabs; 0 on a bad geometry. */
size_t bsva_kv_cache_workspace_bytes(const bsva_kv_cache* c, int Lq);

/* The mask entry over the live slabs of the INT8 cache, reading INT8 K and V
 * straight from their slots (no copy, no bf16 rebuild). The keys are the valid
 * rows of the live slabs, oldest first; one logical mask column per live slab
 * (a slab is a 128-key logical block). The output is softmax attention over
 * the dequantised cache, exact terms only, as in masked_block_attn_fwd_v8.
 *   Lq            query tokens
 *   q8, q_scale   int8 [B,H,Lq,d], fp32 [B,H,nQB] (bsva_quantize_q)
 *   block_mask    uint8 [B, mask_heads, nQB, c->count]: query block i attends
 *                 to logical slab x iff block_mask[b, h % mask_heads, i, x] != 0
 *   workspace     >= bsva_kv_cache_workspace_bytes(c, Lq) bytes, 256-aligned
 *   Other arguments as in masked_block_attn_fwd. A query row with no allowed
 *   key gets out = 0 and lse = -inf. */
int masked_block_attn_fwd_kvcache(const bsva_kv_cache* c, int Lq, const int8_t* q8,
                                  const float* q_scale, const uint8_t* block_mask,
                                  int mask_heads, float softmax_scale, int out_dtype,
                                  void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, bsva_stream_t stream);

/* masked_block_attn_fwd without a workspace. The source pages have no
 * counterpart: this entry point is for callers that cannot allocate device
 * memory, such as a plugin inside a host application whose allocator already
 * owns the device (on a small card every byte is budgeted, and a private
 * cudaMalloc can fail or fragment the host's pool), or code on a streaming
 * path that must not call cudaMalloc because it can synchronise the device.
 * The kept-block lists live in a scratch array compiled into the library:
 * 8,651,008 bytes on every GPU that loads it, held until the process exits.
 * Limits: B*H*nQB <= 65,536 and B*H*nQB*nKB <= 2,097,152; a larger shape
 * returns BSVA_ERR_WORKSPACE and launches nothing.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current, and so does the first call
 * after the device's context has been recreated (cudaDeviceReset); make such
 * a first call before any stream capture. Every call shares the one array, which keeps the
 * last call's contents: calls whose GPU work overlaps (two streams, two host
 * threads) race on it, so the caller must serialise them. A device-side wait
 * that runs out is recorded in the array's status word, which this entry
 * point cannot report; use masked_block_attn_fwd and bsva_check_status where
 * that matters. Other arguments as in masked_block_attn_fwd. */
int masked_block_attn_fwd_noalloc(bsva_shape s, const int8_t* q8,
                                  const float* q_scale, const int8_t* k8,
                                  const float* k_scale, const void* v,
                                  const uint8_t* block_mask, int mask_heads,
                                  float softmax_scale, int out_dtype, void* out,
                                  float* lse, bsva_stream_t stream);

/* Synchronises `stream`, reads and clears the workspace's status word.
 * Returns BSVA_OK, or BSVA_ERR_DEVICE_TIMEOUT if a kernel's bounded wait gave
 * up since the last check (its outputs are then invalid). */
int bsva_check_status(void* workspace, bsva_stream_t stream);

/* Test hook for the failure path: launches one CTA that waits on a barrier
 * nothing arrives at, with a wait bound of limit_ns nanoseconds
 * (1e3 <= limit_ns <= 1e9). The wait runs out, the kernel records
 * BSVA_ERR_DEVICE_TIMEOUT in the workspace status word and returns. */
int bsva_selftest_timeout(void* workspace, size_t workspace_bytes,
                          long long limit_ns, bsva_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSVA_H */
