/*
 * sparse_attn.h -- C ABI of libsparseattn.so: training-free block-sparse
 * attention forward on NVIDIA B200 (sm_100a).
 *
 * The path, in call order:
 *   sa_layout_build  -> token permutation (identity, [t,h,w] windows, Hilbert)
 *   sa_reorder_predict_mask -> Q, K gathered into the permuted order while
 *                       their blocks are pooled; block mask M_g + CSR kept
 *                       lists + work order (sa_reorder + sa_predict_mask
 *                       do the same in two passes)
 *   sa_reorder       -> V gathered into the permuted order
 *   sa_block_sparse_attn -> O and per-row LSE over the kept blocks, stored
 *                       back in the original order (out_perm; sa_unreorder
 *                       does that as a separate pass)
 *   sa_dense_attn    -> the same kernel with every block kept (reference)
 *   sa_l1_error      -> relative L1 error of an output (calibration)
 *
 * Sources of the operations (page title, section):
 *   [P1] "AIGC 基本功｜视频稀疏注意力的误差与布局" (jefxiong.cn)
 *        3.1 restricted softmax, 3.4 permutation equivariance, 4 block ledger.
 *   [P2] MindIE-SD documentation "稀疏": rf_v2 block representatives,
 *        [t,h,w] window reorder, first-frame sink; sparse_attention(q, k, v,
 *        head_num, input_layout="BNSD", sparsity, txt_len, latent_shape...).
 *   [P3] "SpargeAttention：中文精读笔记": 2.1 sparse FlashAttention (online
 *        softmax m/l/O, M_g), 2.2 selective token compression (mean pooling,
 *        CosSim guard theta, TopCdf tau, forced rows/columns), 2.3 PV skip
 *        with lambda, 2.5 Hilbert permutation.
 *   [P4] "44. Local Sliding and Sparse Attention": local causal window,
 *        block pairs with causal filter.
 *   [P5] "78. Attention Access Pattern Benchmark": window + anchor keys.
 *
 * Conventions (every entry point):
 *   - Tensors are BNSD and contiguous: q [B, Hq, N, d], k [B, Hkv, N, d],
 *     v [B, Hkv, N, dv], out [B, Hq, N, dv], lse [B, Hq, N] (fp32, natural
 *     log).  Query head h reads kv head h / (Hq / Hkv).
 *   - Every pointer argument to data is a DEVICE pointer unless stated;
 *     struct arguments are HOST pointers.  The caller owns all memory; the
 *     library never allocates device memory (sa_predict_mask_noalloc uses a
 *     fixed array that is part of the loaded library) and keeps no state
 *     between calls except a thread-local error string.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued asynchronously on it.  Argument errors are detected on the
 *     host and returned synchronously before anything is enqueued; errors
 *     found by a kernel (empty row, list capacity, wait timeout) are written
 *     to a device status word and read back with sa_read_status().
 *   - Nothing falls back to the CPU: without a usable CUDA device every
 *     compute entry point returns SA_ERR_CUDA.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* bad pointer, size, or parameter value        */
  SA_ERR_UNSUPPORTED = 2,   /* valid, but outside the kernels' shapes       */
  SA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than queried    */
  SA_ERR_EMPTY_ROW = 4,     /* a query row would keep no key ([P1] 3.1)     */
  SA_ERR_TIMEOUT = 5,       /* a bounded device wait gave up                */
  SA_ERR_CUDA = 6,          /* a CUDA runtime call failed (see last_error)  */
  SA_ERR_CAPACITY = 7       /* kept blocks exceed mask->col_capacity        */
} sa_status;

typedef enum { SA_BF16 = 0, SA_FP32 = 1 } sa_dtype;

/* Problem shape.  dtype applies to q, k, v and out. */
typedef struct {
  int64_t B, Hq, Hkv, N, d, dv;
  int32_t dtype;
  int32_t reserved;
} sa_shape;

typedef enum {
  SA_ORDER_IDENTITY = 0,
  SA_ORDER_WINDOW = 1,   /* [P2] [t,h,w] windows of size win[0..2]          */
  SA_ORDER_HILBERT = 2   /* [P3] 2.5; Skilling's curve on the 2^b cube      */
} sa_order;

/* Token layout: N = T*H*W + txt_len tokens, raster frame-major video tokens
 * (i = t*H*W + h*W + w) followed by text tokens.  The first sink_frames
 * frames and the text tokens keep their positions; the remaining frames are
 * reordered.  Window mode: windows tile the frames after the sink in raster
 * order of window coordinates, tokens raster-ordered inside a window, edge
 * windows smaller.  Hilbert mode: tokens sorted by the index of (t', h, w)
 * on the 2^b cube, b = ceil(log2(max(T - sink_frames, H, W))), t' most
 * significant; b <= 9. */
typedef struct {
  int64_t T, H, W, txt_len, sink_frames;
  int64_t win[3];
  int32_t mode;          /* sa_order */
  int32_t reserved;
} sa_layout_desc;

/* Mask prediction parameters ([P3] 2.2, [P2], [P5]).
 *   bq, bk        query / key block sizes (1..128).
 *   tau           TopCdf threshold in (0, 1]: a block is kept iff the
 *                 probability mass sorted before it is < tau * row total.
 *   theta         similarity guard; blocks whose mean pairwise cosine is
 *                 < theta get forced full rows (queries) or columns (keys)
 *                 and key blocks below theta leave the compressed softmax.
 *                 theta <= 0 disables the guard.
 *   sink_tokens   tokens at the front whose blocks get full rows+columns.
 *   txt_len       tokens at the back whose blocks get full rows+columns.
 *   local_window  w > 0 keeps every block pair holding some (i, j) with
 *                 0 <= i - j < w ([P4], block level); 0 = off.
 *   anchor_tokens tokens at the front whose key blocks get full columns.
 *   causal        1 = key j visible to query i only if j <= i.
 *   order_group   the work order of the mask's rows (sa_mask.order).  0:
 *                 every row by descending kept count, ties by ascending row
 *                 index.  g > 0: rows in groups of g consecutive (batch,
 *                 query head) pairs, the groups in order, and the rows of a
 *                 group by descending count, ties by ascending row index, so
 *                 that the rows running at the same time share their heads'
 *                 K and V in L2.  sa_order_group_hint() gives the library's
 *                 choice for a shape.  Must be >= 0, and order_group * nqb
 *                 <= 32768. */
typedef struct {
  int32_t bq, bk;
  float tau, theta;
  int64_t sink_tokens, txt_len, local_window, anchor_tokens;
  int32_t causal;
  int32_t order_group;
} sa_mask_params;

/* A block mask and its compacted lists.  All pointers are device buffers
 * owned by the caller and sized by the caller:
 *   block_mask  uint8 [B*Hq, nqb, nkb], 1 = kept
 *   row_ptr     int32 [B*Hq*nqb + 1], CSR offsets into col_idx
 *   col_idx     int32 [col_capacity], kept key blocks, ascending per row
 *   order       int32 [B*Hq*nqb], rows by descending kept count, ties by
 *               ascending row index (work order of the attention kernel)
 *   kept_total  int64 [1]
 *   status      int32 [1], device status word (sa_status code, 0 = OK)
 * The producer (sa_predict_mask / sa_mask_from_blocks) fills nqb, nkb, bq,
 * bk, causal.  A row index is (b*Hq + h)*nqb + qb.  col_capacity of
 * B*Hq*nqb*nkb always suffices. */
typedef struct {
  uint8_t* block_mask;
  int32_t* row_ptr;
  int32_t* col_idx;
  int32_t* order;
  int64_t* kept_total;
  int32_t* status;
  int64_t col_capacity;
  int64_t nqb, nkb;
  int32_t bq, bk, causal;
  int32_t reserved;
} sa_mask;

/* Flags for the attention entry points. */
#define SA_FLAG_FORCE_SIMT 1   /* use the portable CUDA-core kernel even where
                                  the tensor-core kernel applies (testing) */
#define SA_FLAG_OUT_PERM_PER_HEAD 2   /* out_perm is int32 [B*Hq][N], one
                                         permutation per query head */
#define SA_FLAG_TEST_STALL 4          /* testing the timeout path: on the
                                         tensor-core kernel, the first CTA loads
                                         no K tile, so its bounded waits (10 ms
                                         under this flag instead of 2 s) run out
                                         and the status word gets
                                         SA_ERR_TIMEOUT; that CTA's query rows are
                                         not computed.  Never set in normal use. */

/* Library version string and the calling thread's last error message. */
const char* sa_version(void);
const char* sa_last_error(void);

/* Which attention kernel serves a shape: 1 = tcgen05 tensor-core kernel
 * (bf16, d = dv = 128, bq = 128, bk in {64, 128}), 0 = CUDA-core kernel,
 * -1 = unsupported. */
int32_t sa_attn_kernel_path(const sa_shape* shape, int32_t bq, int32_t bk, int32_t flags);

/* ---- a0: layout ([P2] window reorder; [P3] 2.5 Hilbert) ----------------
 * perm[n] = source index of output position n; inv[perm[n]] = n.  Both are
 * int32 [N] device buffers.  Window and identity modes need no workspace;
 * Hilbert mode needs sa_layout_workspace() bytes (256-byte aligned). */
size_t sa_layout_workspace(const sa_layout_desc* desc);
sa_status sa_layout_build(const sa_layout_desc* desc, int32_t* perm, int32_t* inv,
                          void* ws, size_t ws_bytes, void* stream);

/* ---- a1/a7: reorder ([P1] 3.4) -------------------------------------------
 * x, y are [outer, N, row] arrays of `row` elements of `dtype` per token
 * (outer = B*H).  sa_reorder: y[o, n, :] = x[o, perm[n], :].
 * sa_unreorder: x[o, perm[n], :] = y[o, n, :] (pass the same perm).
 * perm must be a permutation of [0, N) (device int32; not checked here:
 * sa_layout_build produces one).  x and y must not overlap.  row = 1 with
 * SA_FP32 reorders LSE. */
sa_status sa_reorder(const int32_t* perm, const void* x, void* y, int64_t outer,
                     int64_t N, int64_t row, int32_t dtype, void* stream);
sa_status sa_unreorder(const int32_t* perm, const void* y, void* x, int64_t outer,
                       int64_t N, int64_t row, int32_t dtype, void* stream);

/* ---- a2-a4: mask prediction ([P3] 2.2) -----------------------------------
 * Pools q and k per block (mean over the block's real tokens), computes the
 * mean pairwise cosine of each block, scores the compressed matrix
 * q_hat k_hat^T / sqrt(d) (ineligible key blocks -inf), softmaxes and
 * TopCdf-selects each row, ORs in the forced rows/columns, sink, text,
 * anchors and local window, ANDs causal validity, checks that every query
 * row keeps a key, and builds the CSR lists and work order into *out.
 * Needs d a power of two with d*elem_size a multiple of 16 and d <= 256,
 * N/bk <= 4095.  ws: sa_predict_mask_workspace() bytes, 256-byte aligned.
 * sa_predict_mask_ws_layout() reports the byte offsets of its regions, for
 * inspection: [0] q_hat fp32 [B*Hq, nqb, d]; [1] k_hat fp32 [B*Hkv, d, nkb4]
 * (feature-major, nkb4 = nkb rounded up to a multiple of 4, columns >= nkb
 * unused); [2] query-block similarity fp32 [B*Hq, nqb]; [3] key-block
 * similarity fp32 [B*Hkv, nkb]; [4] row counts int32 [B*Hq*nqb]; [5] sort
 * scratch. */
size_t sa_predict_mask_workspace(const sa_shape* shape, const sa_mask_params* params);
/* order_group for a shape: 0 (one global order) when the K and V of one KV
 * head take less than 32 MiB (several heads' K/V stay in L2 anyway);
 * otherwise the largest power of two g <= B*Hq whose g consecutive query
 * heads touch at most 96 MiB of K and V (at least 1).  -1 for an invalid
 * shape. */
int32_t sa_order_group_hint(const sa_shape* shape);
sa_status sa_predict_mask_ws_layout(const sa_shape* shape, const sa_mask_params* params,
                                    size_t offsets[6]);
sa_status sa_predict_mask(const void* q, const void* k, const sa_shape* shape,
                          const sa_mask_params* params, void* ws, size_t ws_bytes,
                          sa_mask* out, void* stream);

/* ---- a1 + a2-a4 fused: reorder Q and K while pooling them ([P1] 3.4,
 * [P3] 2.2) ------------------------------------------------------------------
 * sa_predict_mask on the permuted sequence, for q and k given in the
 * original token order: the pooling pass reads token n of the permuted
 * order from row perm[n] of q and k and also writes it to row n of q_r and
 * k_r (q_r[o, n, :] = q[o, perm[n], :], as sa_reorder), so Q and K cross HBM
 * once for both steps.  perm: int32 [N], a permutation of [0, N) (an entry
 * outside that range raises SA_ERR_INVALID_ARG in the status word and the
 * token is skipped).  q_r, k_r: device buffers of the shapes of q and k,
 * 16-byte aligned, overlapping neither q, k nor each other.  Workspace, the
 * other arguments and the results are those of sa_predict_mask (the mask
 * describes the permuted sequence). */
sa_status sa_reorder_predict_mask(const int32_t* perm, const void* q, const void* k, void* q_r, void* k_r,
                                  const sa_shape* shape, const sa_mask_params* params, void* ws,
                                  size_t ws_bytes, sa_mask* out, void* stream);

/* sa_predict_mask without a caller workspace.  The pages describe no such
 * call: it exists for callers that cannot allocate device memory at all (code
 * running inside another runtime's memory pool without access to it, a
 * plug-in handed only pre-sized inputs and outputs, a serving process whose
 * device footprint must not grow).  The scratch comes from a 32 MiB array
 * that the library itself holds on each device for the life of the process;
 * the function allocates nothing.  Shapes whose sa_predict_mask_workspace()
 * exceeds 32 MiB are rejected with SA_ERR_WORKSPACE (the largest shipped
 * workload needs about 25 MiB).  Arguments and results are those of
 * sa_predict_mask.  Every call shares the one array; each call writes every
 * scratch value before reading it, so it needs no clearing, but calls that
 * overlap on the GPU (other streams, other threads) race on it and must be
 * serialised by the caller.  The first call on a device (with that device
 * current) looks up the array's address; make it before any stream capture
 * begins on that device.  The address is kept for the life of the process,
 * so do not use this entry point across a cudaDeviceReset of the device. */
sa_status sa_predict_mask_noalloc(const void* q, const void* k, const sa_shape* shape,
                                  const sa_mask_params* params, sa_mask* out, void* stream);

/* A caller-supplied block mask (uint8 [B*Hq, nqb, nkb], nonzero = kept) is
 * ANDed with causal validity, copied to out->block_mask (may alias), checked
 * for empty rows and compacted into lists exactly as sa_predict_mask does. */
size_t sa_mask_from_blocks_workspace(const sa_shape* shape, int32_t bq, int32_t bk);
sa_status sa_mask_from_blocks(const uint8_t* block_mask, const sa_shape* shape, int32_t bq,
                              int32_t bk, int32_t causal, void* ws, size_t ws_bytes,
                              sa_mask* out, void* stream);

/* Scratch of the attention entry points (a work counter the kernel zeroes
 * with an asynchronous memset before each launch): sa_attn_workspace() bytes,
 * 256-byte aligned.  Calls that share one workspace must not overlap on the
 * GPU. */
size_t sa_attn_workspace(void);

/* ---- a5/a6: block-sparse attention ([P3] 2.1, 2.3) -----------------------
 * For every query block, visits its kept key blocks in ascending order with
 * the online-softmax recurrence; skips P~V of a tile when the largest
 * (tile row max - running row max) over the block's rows is < lambda
 * (lambda = -INFINITY disables the skip; the normaliser l still counts the
 * tile).  scale = 0 means 1/sqrt(d).  out gets O / l in the input dtype,
 * lse (nullable) gets m + ln l.  out_perm (nullable, int32 [N]) fuses the
 * inverse reorder into the store: row n of the problem is written to row
 * out_perm[n] of out and lse (pass the layout's perm to get the original
 * token order back; out must not alias q).  pv_skip_log (nullable) gets one
 * byte per kept tile in CSR order, 1 = PV skipped; size it like col_idx
 * (mask->col_capacity bytes).  The mask's status word also receives kernel
 * errors.  A row whose list reaches past mask->col_capacity (the mask's
 * builder raised SA_ERR_CAPACITY) is not computed: its O and LSE rows are
 * left as they were, and nothing past col_capacity is read or written, so
 * the call may be enqueued right after the builder, before the status is
 * read. */
sa_status sa_block_sparse_attn(const void* q, const void* k, const void* v,
                               const sa_shape* shape, const sa_mask* mask, float lambda,
                               float scale, void* out, float* lse, const int32_t* out_perm,
                               uint8_t* pv_skip_log, void* ws, size_t ws_bytes, int32_t flags,
                               void* stream);

/* ---- 8-bit QK ([P3] 2.4: SageAttention's per-block quantisation) ---------
 * The QK product on 8-bit codes with per-block dequantisation scales; P and
 * V stay bf16.  Two code formats:
 *   SA_Q_INT8: int8, scale = absmax / 127, code = rint(x * (127 / absmax))
 *     in float32, round half to even, in [-127, 127];
 *   SA_Q_E4M3: FP8 E4M3 bytes, scale = absmax / 448, code = the E4M3 value
 *     nearest to x * (448 / absmax) (float32 product; ties to even,
 *     saturated to +-448).
 * An all-zero block gets scale 0 and codes 0.
 *
 * sa_quantize_blocks: x bf16 [heads][N][d] (16-byte aligned) -> x8 codes
 * [heads][N][d] (8-byte aligned) and scales float [heads][ceil(N/rows)]; a
 * block is `rows` consecutive tokens of one head.  Needs d a multiple of 8
 * and rows * d <= 16384.  Quantise Q with rows = the mask's bq and K with
 * rows = its bk.
 *
 * sa_block_sparse_attn_qk8: sa_block_sparse_attn with q8, k8 BNSD codes of
 * `format` and their scales (q_scales [B*Hq][ceil(N/bq)], k_scales
 * [B*Hkv][ceil(N/bk)]): the score of a pair is (q8 . k8) * q_scale *
 * k_scale * scale (an exact int32 product for INT8, an fp32-accumulated
 * one for E4M3, on the tensor cores).  Same
 * mask, lambda, out, lse, out_perm, skip log and flags as
 * sa_block_sparse_attn (SA_FLAG_FORCE_SIMT: SA_ERR_UNSUPPORTED; there is no
 * other kernel).  Needs bf16 V and out, d = dv = 128, bq = 128, bk in
 * {64, 128}, an sm_100 device, 16-byte aligned q8, k8, v, out.  ws:
 * sa_attn_qk8_workspace(mask) bytes, 256-byte aligned (the work counter and
 * one scale per list entry). */
#define SA_Q_INT8 0
#define SA_Q_E4M3 1
sa_status sa_quantize_blocks(const void* x, int64_t heads, int64_t N, int64_t d, int32_t rows, int32_t dtype,
                             int32_t format, void* x8, float* scales, void* stream);
size_t sa_attn_qk8_workspace(const sa_mask* mask);
/* sa_reorder_predict_mask with the quantisation fused into its pooling
 * pass: instead of reordered bf16 copies it writes the reordered 8-bit
 * codes q8 [B*Hq][N][d], k8 [B*Hkv][N][d] (16-byte aligned) and the block
 * scales q_scales [B*Hq][ceil(N/bq)], k_scales [B*Hkv][ceil(N/bk)], equal
 * to sa_quantize_blocks of the reordered tensors (query blocks for Q, key
 * blocks for K).  perm may be NULL (the original order).  bf16 q, k only. */
sa_status sa_reorder_predict_mask_q8(const int32_t* perm, const void* q, const void* k, int32_t format, void* q8,
                                     float* q_scales, void* k8, float* k_scales, const sa_shape* shape,
                                     const sa_mask_params* params, void* ws, size_t ws_bytes, sa_mask* out,
                                     void* stream);
sa_status sa_block_sparse_attn_qk8(const void* q8, const float* q_scales, const void* k8, const float* k_scales,
                                   int32_t format, const void* v, const sa_shape* shape, const sa_mask* mask,
                                   float lambda, float scale, void* out, float* lse, const int32_t* out_perm,
                                   uint8_t* pv_skip_log, void* ws, size_t ws_bytes, int32_t flags, void* stream);

/* ---- a8: dense reference --------------------------------------------------
 * The same recurrence with every (causally valid) key visible and no lists
 * (lambda = -inf); the library picks the tile shape.  status (device int32,
 * nullable) receives kernel errors. */
sa_status sa_dense_attn(const void* q, const void* k, const void* v, const sa_shape* shape,
                        int32_t causal, float scale, void* out, float* lse, int32_t* status,
                        void* ws, size_t ws_bytes, int32_t flags, void* stream);

/* ---- a0-a7 end to end from host buffers ([P1] 6: the permutation and the
 * data movement count in end-to-end time) -----------------------------------
 * The whole path for host buffers (pinned, so that the copies are
 * asynchronous): q_host [B*Hq][N][d], k_host and v_host [B*Hkv][N][d | dv],
 * out_host [B*Hq][N][dv] in the input dtype and lse_host float [B*Hq][N], all
 * in the original token order.  The problem is cut into `chunks` groups of
 * (batch, head) rows (chunks divides B*Hkv, at most 16; query row r reads kv
 * row r / (Hq/Hkv)).  Chunk i's copies in run on streams[1], its path on
 * streams[0] (sa_layout_build once; sa_reorder_predict_mask and sa_reorder of
 * V, or sa_predict_mask for the identity layout; sa_block_sparse_attn with
 * out_perm = the layout's perm) and its copies out on streams[2], so the
 * copies of one chunk overlap the kernels of its neighbours.  The work is
 * ordered after what the caller enqueued on streams[0] before the call, and
 * is complete on streams[0] once the last copy out is; the three streams may
 * be one stream (no overlap).  shape->N must equal the layout's token count.
 * ws: sa_forward_host_workspace() bytes, 256-byte aligned, owned by the
 * caller (device copies of the inputs and outputs, one chunk's reordered
 * copies, mask and scratch); calls sharing it must not overlap.  status
 * (device int32 [1]) is cleared and then receives the largest status code of
 * any chunk.  The host buffers must stay valid until the work completes.
 * Argument and CUDA errors return synchronously; work already enqueued stays
 * enqueued. */
size_t sa_forward_host_workspace(const sa_shape* shape, const sa_layout_desc* layout,
                                 const sa_mask_params* params, int32_t chunks);
sa_status sa_forward_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                          float* lse_host, const sa_shape* shape, const sa_layout_desc* layout,
                          const sa_mask_params* params, float lambda, float scale, int32_t chunks,
                          void* ws, size_t ws_bytes, int32_t* status, void* const streams[3]);

/* Synchronises `stream` and returns the device status word's code (0 =
 * SA_OK).  The word is not cleared. */
sa_status sa_read_status(const int32_t* status, void* stream);

/* ---- per-head spatial / temporal placement ([P1] 3.3, 3.4, 4, 5) ---------
 * The Sparse VideoGen comparison of [P1] section 5.  On a T x H x W video
 * (P = H*W, nv = T*P frame-major tokens t*P + p, then txt_len text tokens;
 * N = nv + txt_len) a spatial head keeps the pairs of one frame and a
 * temporal head the pairs of one position across frames; text tokens pair
 * with every token.  A spatial head runs in the frame-major order, a
 * temporal head in the token-major order (place n < nv holds frame n % T of
 * position n / T; text stays in place), where its pairs fill whole tiles
 * (the tile ledger of [P1] section 4).
 *
 * sa_head_placement, for kinds (device int32 [heads], SA_HEAD_SPATIAL or
 * SA_HEAD_TEMPORAL):
 *   perms (device int32 [heads][N], nullable): perms[h][n] = the original
 *     token at place n of head h's order;
 *   block_mask (device uint8 [heads][ceil(N/bq)][ceil(N/bk)], nullable): 1
 *     where the tile of head h's order holds an allowed pair (the block
 *     cover of the element mask, [P1] section 4); feed it to
 *     sa_mask_from_blocks.
 * Another kind value raises SA_ERR_INVALID_ARG in status (device int32,
 * nullable) and leaves that head's tiles empty.  The usual run: perms and
 * block_mask from here, Q, K, V through sa_reorder_heads, then
 * sa_block_sparse_attn with out_perm = perms and SA_FLAG_OUT_PERM_PER_HEAD,
 * which stores every head back in the original order. */
#define SA_HEAD_SPATIAL 0
#define SA_HEAD_TEMPORAL 1
sa_status sa_head_placement(int64_t T, int64_t H, int64_t W, int64_t txt_len, const int32_t* kinds,
                            int64_t heads, int32_t bq, int32_t bk, int32_t* perms, uint8_t* block_mask,
                            int32_t* status, void* stream);

/* y[o, n, :] = x[o, perms[o*N + n], :]: sa_reorder with one permutation per
 * outer index (x, y [outer, N, row] of dtype; perms device int32
 * [outer][N], each entry in [0, N)).  x and y must not overlap. */
sa_status sa_reorder_heads(const int32_t* perms, const void* x, void* y, int64_t outer, int64_t N, int64_t row,
                           int32_t dtype, void* stream);

/* Attention of a few query rows, the online profile of [P1] section 5 (only
 * the sampled rows are computed).  For each query head bh = b*Hq + h and
 * sampled row r, the query token rows[r] (device int32, in [0, N)) attends
 * to: every key (block_mask NULL), or the keys of the kept tiles of its
 * query block in head bh's order (block_mask uint8 [B*Hq][ceil(N/bq)]
 * [ceil(N/bk)], e.g. from sa_head_placement; perms int32 [B*Hq][N], the
 * token at each place of that order, NULL = the original order).  q, k, v
 * BNSD (bf16 or fp32, 16-byte aligned, d = dv in {64, 128},
 * N / bk <= 4096); scale
 * 0 means 1/sqrt(d).  out: float [B*Hq][nrows][dv], lse (nullable): float
 * [B*Hq][nrows], natural log.  A row outside [0, N) or missing from its
 * head's order raises SA_ERR_INVALID_ARG in status (device int32,
 * nullable) and is not written; a row with no key raises SA_ERR_EMPTY_ROW. */
sa_status sa_rows_attn(const void* q, const void* k, const void* v, const sa_shape* shape, const int32_t* rows,
                       int64_t nrows, const int32_t* perms, const uint8_t* block_mask, int32_t bq, int32_t bk,
                       float scale, float* out, float* lse, int32_t* status, void* stream);

/* Sampled-row error of [P1] section 5: out[h] (device double [BH]) = mean of
 * (ref - x)^2 over the nrows sampled query rows (rows: device int32, each in
 * [0, N)) and the dv outputs of head h; ref and x are [BH, N, dv] of dtype.
 * A row outside [0, N) is skipped and raises SA_ERR_INVALID_ARG in status
 * (device int32, nullable). */
sa_status sa_rows_mse(const void* ref, const void* x, const int32_t* rows, int64_t nrows, int64_t BH, int64_t N,
                      int64_t dv, int32_t dtype, double* out, int32_t* status, void* stream);

/* ---- calibration support ([P3] 2.4) ---------------------------------------
 * The per-layer calibration of the SpargeAttention notes bounds the relative
 * L1 error sum |O - O'| / sum |O| of the sparse output O' against the dense
 * output O.  sums (device double[2], overwritten) receives sum |ref - x| and
 * sum |ref| over n elements of dtype; ref and x are 16-byte aligned device
 * buffers, n a multiple of 8 (bf16) or 4 (fp32).  Asynchronous on stream. */
sa_status sa_l1_error(const void* ref, const void* x, int64_t n, int32_t dtype, double* sums, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
