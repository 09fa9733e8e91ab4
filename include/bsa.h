/*
 * bsa.h -- C ABI of libbsa: training-free block-sparse "sol-attn" attention
 * on NVIDIA B200 (sm_100a).
 *
 * The operation (sources are web pages, cited by title and section):
 *   [DOC]  "BlockSparseAttention - ComfyUI Built-in Node Documentation":
 *          general-inputs table (extra_tokens, sink_conditioning),
 *          "sol-attn inputs" (tau), "sla inputs" (keep_percent).
 *   [STAR] "minimax-h3-chunk-star7" README, sections "SLA" and "Sol".
 *
 *   1. bsa_pool       -- Q and K (and V, for the centroids) are mean-pooled per
 *                        block of consecutive tokens (Q64/K64 for Sol, Q128/K64
 *                        for SLA: [STAR] "SLA", "Sol").
 *   2. bsa_select     -- per (batch, head, query block) row of pooled scores
 *                        S = qbar . kbar / sqrt(d): Sol keeps the blocks above
 *                        mean + tau * std of the row ([DOC] tau: a threshold in
 *                        standard deviations of the score distribution); SLA
 *                        keeps the top keep_percent % ([DOC] keep_percent).  Sink,
 *                        prefix and diagonal blocks are kept in addition.
 *                        Optionally picks extra_tokens top-scoring tokens per
 *                        query block outside its kept blocks ([DOC] extra_tokens).
 *   3. bsa_attention  -- exact attention over the kept key blocks (and extra
 *                        tokens); every unselected block contributes through its
 *                        K/V centroid with logit q.kbar/sqrt(d) + ln(n_b); both
 *                        merge into one FP32 online softmax ([STAR] "Sol").
 *                        Rows in [dense_row_begin, dense_row_end) are computed
 *                        densely and replace the sparse result ([DOC]
 *                        sink_conditioning = exact_kv_and_rows).
 *   4. bsa_dense_ref_rows -- dense softmax attention for a range of query rows.
 *
 * Cube tiling (method BSA_VSA): block b < prefix_len / 64 is the prefix's
 * b-th run of 64 tokens; block prefix_len / 64 + c is cube c of the grid in
 * t-major cube order, its 64 tokens taken t-major inside the cube.  Query and
 * key blocks are the same cubes (q_block = k_block = 64).  Pooled means, rows
 * of the CSR and the diagonal ("key block = query block") are in that block
 * order; Q, K, V, O and LSE stay in token order.  Needs B == 1, prefix_len a
 * multiple of 64, dense rows inside the prefix, centroid 0, extra_tokens 0.
 *
 * Conventions shared by every call:
 *   - Tensors Q, K, V and O are [B, N, H, d] with element strides stride_b,
 *     stride_n, stride_h and a contiguous channel dimension; all four share the
 *     same strides.  Base pointers must be 16-byte aligned and stride_b,
 *     stride_n, stride_h multiples of 8 elements (bf16) or 4 elements (f32).
 *   - Every pointer argument is a device pointer unless stated otherwise; the
 *     caller owns all memory.  The library allocates no device memory.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream).  Argument errors are detected on the host
 *     and returned before anything is launched; launch failures return
 *     BSA_ERR_CUDA.  Errors found by the kernels (e.g. a CSR capacity overflow)
 *     are written to a status word inside the workspace and read back with
 *     bsa_device_status().  No kernel traps.
 *   - Calls are thread-safe; the library keeps no global state apart from a
 *     thread-local message describing the last host-side error.
 *   - Rows are ordered [B, H, nQB]: row r = (b * H + h) * nQB + i, where
 *     nQB = ceil(N / q_block) and nKB = ceil(N / k_block).
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, stride, alignment or parameter */
    BSA_ERR_UNSUPPORTED = 2,   /* valid request outside this build (d not in {64,128}, ...) */
    BSA_ERR_CAPACITY = 3,      /* an output array is too small (host- or device-detected) */
    BSA_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than bsa_workspace_size() */
    BSA_ERR_CUDA = 5,          /* a CUDA runtime call or a kernel launch failed */
    BSA_ERR_DEVICE = 6         /* a kernel reported an internal error (status word) */
} bsa_status;

typedef enum { BSA_DT_BF16 = 0, BSA_DT_F32 = 1 } bsa_dtype;
/* BSA_VSA: the fine stage of [DOC]'s vsa method without its learned coarse
 * branch (the node runs it so when the model lacks that layer): key blocks and
 * query blocks are 3-D cubes of the latent video grid, the top keep_percent %
 * of key cubes per query cube are attended exactly, the rest dropped. */
typedef enum { BSA_SOL = 0, BSA_SLA = 1, BSA_VSA = 2 } bsa_method;

typedef struct {
    int32_t B, H, N, d;            /* batch, heads, tokens, head dim (64 or 128) */
    int64_t stride_b, stride_n, stride_h;   /* element strides of Q, K, V, O */
    int32_t dtype;                 /* bsa_dtype of Q, K, V and O */
    int32_t method;                /* bsa_method */
    int32_t q_block, k_block;      /* Sol 64/64, SLA 128/64 ([STAR] "SLA", "Sol"); k_block must be 64 */
    double  tau;                   /* Sol threshold in standard deviations; -inf keeps all, +inf none */
    double  keep_percent;          /* SLA: percent of key blocks kept per query block, (0, 100] */
    int32_t sink_blocks;           /* leading key blocks always kept (default 1) */
    int32_t keep_diag;             /* 1: key blocks meeting the query block's tokens always kept */
    int32_t prefix_len;            /* P: packed conditioning rows [0, P) every query attends to exactly
                                      (exact_kv); 0 disables */
    int32_t dense_row_begin;       /* query rows [begin, end) run dense and replace the sparse result */
    int32_t dense_row_end;         /*   (exact_kv_and_rows); begin == end disables */
    int32_t extra_tokens;          /* E: extra top-scoring tokens per query block, 0..256; 0 disables */
    int32_t centroid;              /* 1: unselected blocks contribute through centroids (Sol);
                                      0: they are dropped (SLA without its trained linear branch) */
    int32_t grid_t, grid_h, grid_w;  /* BSA_VSA: the latent grid T x Hs x Ws of the tokens after the
                                        prefix, flattened t-major (prefix_len + T*Hs*Ws == N) */
    int32_t cube_t, cube_h, cube_w;  /* BSA_VSA: cube extents (4, 4, 4); product 64, each dividing its
                                        grid extent ([DOC] vsa: 3-D video cube tiling) */
    int32_t qk_fp8;                /* 1: the fine pass takes S = Q K^T in fp8 (e4m3, one scale per 64
                                      tokens of Q and of K and per 64 centroids), P V in bf16 -- the
                                      B200 form of [STAR] "attention modes" qk_int8_pv_fp16; needs
                                      bf16 inputs, d = 128, extra_tokens 0, method Sol or SLA */
    int32_t modcent_per_row;       /* E > 0: the workspace holds rows * modcent_per_row modified
                                      centroids in all (one per block that gave extra tokens and keeps
                                      some; a row may use more than this as long as the total fits);
                                      0 = min(E, nKB) per row, always enough.  If the rows' total
                                      exceeds the capacity, the status word reports BSA_ERR_CAPACITY
                                      and the rows past it lose the modified centroids that did not
                                      fit (their other terms are unchanged). */
    int32_t pv_fp8;                /* 1 (with qk_fp8 = 1): P V in fp8 too -- P rounded to e4m3 as the
                                      softmax writes it, V and the value centroids in e4m3 with one
                                      scale per (batch, head, channel) applied to the output -- the
                                      B200 form of [STAR] "attention modes" all_int8 / Sol "PV INT8" */
} bsa_params;

/* Fill *p with the defaults of the node documentation for `method`
 * (Sol: tau 1.3, Q64/K64, centroid on; SLA: keep_percent 10, Q128/K64,
 * centroid off; both: sink 1, diagonal kept, no prefix, no dense rows, E 0).
 * Shapes and strides are left zero. */
BSA_API void bsa_default_params(bsa_params *p, int32_t method);

/* Bytes of device workspace the select and attention calls need for these
 * parameters (*bytes), and the largest possible number of kept entries,
 * B*H*nQB*nKB (*max_nnz), an always-sufficient CSR capacity.  The scratch of
 * bsa_select and that of the attention calls share the same bytes (nothing of
 * one is read by the other; the status word is kept apart): calls that share a
 * workspace must not overlap on the GPU (issue them on one stream, or order
 * the streams). */
BSA_API bsa_status bsa_workspace_size(const bsa_params *p, size_t *bytes, int64_t *max_nnz);

/* Step 1, pooling ([STAR] "SLA", "Sol": Q/K blocks; K/V centroids).
 *   q, k, v   : [B, N, H, d] inputs (dtype, strides from p).
 *   qbar      : out [B, H, nQB, d] f32, mean of Q over each query block.
 *   kbar, vbar: out [B, H, nKB, d] f32, means of K and V over each key block.
 *   blk_count : out [nKB] int32, tokens in each key block (the last may be partial).
 * Sums run in fp64 in token order; each mean is rounded once to f32. */
BSA_API bsa_status bsa_pool(const bsa_params *p, const void *q, const void *k, const void *v,
                    float *qbar, float *kbar, float *vbar, int32_t *blk_count, void *stream);

/* Steps before 1 and 1 in one kernel: the QKV projection with pooling folded
 * into its epilogue ([STAR] "Sol": a producer with fused preprocessing that
 * reuses the current input statistics).  [Q | K | V] = X W^T in bf16 with
 * fp32 accumulation, and the block means of the rounded outputs exactly as
 * bsa_pool computes them (fp64 sums in token order, rounded once to f32),
 * without reading Q, K and V back.
 *   x         : [B, N, d_model] bf16, contiguous (d_model a multiple of 64).
 *   w_qkv     : [3 * H * d, d_model] bf16, contiguous: the rows of Q's heads,
 *               then K's, then V's, d rows per head (a linear layer's weight).
 *   q, k, v   : out [B, N, H, d] bf16 with p's strides.
 *   qbar, kbar, vbar, blk_count: out, as for bsa_pool.
 *   ws        : NULL, or a workspace whose status word receives kernel errors.
 * Needs bf16, H * d a multiple of 256, and a method other than BSA_VSA (cubes
 * are not runs of tokens); no bias term. */
BSA_API bsa_status bsa_qkv_pool(const bsa_params *p, const void *x, int32_t d_model, const void *w_qkv,
                                void *q, void *k, void *v, float *qbar, float *kbar, float *vbar,
                                int32_t *blk_count, void *ws, void *stream);

/* Step 2, selection ([DOC] "sol-attn inputs" tau, "sla inputs" keep_percent,
 * general inputs extra_tokens).
 *   qbar, kbar  : pooled means from bsa_pool.
 *   k           : [B, N, H, d] keys (read only when p->extra_tokens > 0).
 *   row_ptr     : out [rows + 1] int64 CSR offsets.
 *   col_idx     : out [col_capacity] int32 kept key-block indices, ascending per row.
 *   kept_count  : out [rows] int32 kept blocks per row.
 *   extra_idx   : out [rows, E] int32 extra tokens, ascending, -1 padded (NULL if E == 0).
 *   extra_count : out [rows] int32 (NULL if E == 0).
 *   ws, ws_bytes: workspace of at least bsa_workspace_size() bytes.
 * A query block whose every row lies in [dense_row_begin, dense_row_end) gets
 * no extra tokens (extra_count 0): those rows are computed densely by
 * bsa_attention and never read the list.
 * Scores are computed in fp64 and rounded to f32 (S = fl32(qbar.kbar / sqrt d));
 * row mean and population std are taken in fp64 over all nKB scores;
 * thr = fl32(mean + tau * std); block b is kept iff S_b > thr.  If the total
 * kept count exceeds col_capacity, the status word reports BSA_ERR_CAPACITY and
 * col_idx holds only the entries that fit. */
BSA_API bsa_status bsa_select(const bsa_params *p, const float *qbar, const float *kbar, const void *k,
                      int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                      int32_t *kept_count, int32_t *extra_idx, int32_t *extra_count,
                      void *ws, size_t ws_bytes, void *stream);

/* bsa_select without a workspace, for callers that cannot allocate device
 * memory: a process whose allocator is owned by a host framework, a plugin
 * that may not call cudaMalloc, a server that must not allocate while it
 * serves.  The pages describe no such variant; it is a deployment convenience.
 *   Arguments as for bsa_select (extra tokens are not picked: p->extra_tokens
 *   must be 0).  The scratch lives in a 32 MiB device array inside the library
 *   (every GPU that loads the library holds it until the process exits); a
 *   problem whose selection scratch -- rows*nKB*4 + rows*ceil(nKB/32)*4 +
 *   rows*4 bytes plus alignment -- exceeds it is rejected with
 *   BSA_ERR_CAPACITY before anything is launched.
 *   The first call on a device looks the array's device address up (one
 *   cudaGetSymbolAddress); make that first call before any stream capture.
 *   The address is remembered per device together with the CUDA context it
 *   belongs to, and looked up again when a call finds another context current
 *   (after a device reset the module, and the array, may sit elsewhere); the
 *   contents do not survive such a reset.
 *   Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   All calls share the one array: calls whose work overlaps on the GPU (on
 *   different streams) race; serialise them.  The array keeps the last call's
 *   contents, and each call clears what must start at zero.
 *   A CSR overflow shows as row_ptr[rows] > col_capacity (the status word of
 *   this variant is not reported). */
BSA_API bsa_status bsa_select_static(const bsa_params *p, const float *qbar, const float *kbar,
                                     int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                                     int32_t *kept_count, void *stream);

/* Step 3, fine pass ([STAR] "Sol": exact kept blocks + centroids of the
 * others in one FP32 online softmax; [DOC] sink_conditioning).
 *   q, k, v        : [B, N, H, d] inputs.
 *   kbar, vbar     : [B, H, nKB, d] f32 centroids from bsa_pool.
 *   blk_count      : [nKB] int32 block sizes from bsa_pool.
 *   row_ptr, col_idx: CSR of kept blocks (ascending within each row), e.g. from bsa_select.
 *   extra_idx, extra_count: extra tokens ([rows, E], [rows]); NULL when E == 0.
 *   out            : out [B, N, H, d] attention output, dtype of q.
 *   lse            : out [B, H, N] f32 natural-log softmax normaliser; may be NULL.
 * A block that gave extra tokens keeps a centroid over its remaining tokens
 * (bias ln of their count); a block left empty contributes nothing.  Rows in
 * [dense_row_begin, dense_row_end) are computed densely by this call. */
BSA_API bsa_status bsa_attention(const bsa_params *p, const void *q, const void *k, const void *v,
                         const float *kbar, const float *vbar, const int32_t *blk_count,
                         const int64_t *row_ptr, const int32_t *col_idx,
                         const int32_t *extra_idx, const int32_t *extra_count,
                         void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* bsa_attention in two calls on the same stream, with the same arguments:
 * bsa_attention_prepare launches the preparation kernels (bf16 copies of f32
 * inputs, bf16 centroids, the modified centroids of blocks that gave extra
 * tokens and the per-tile extra-token lists, all written to the workspace);
 * bsa_attention_run then launches the fine pass itself (and the dense-row
 * merge), reading them.  prepare followed by run is exactly bsa_attention;
 * the split lets a caller overlap or time the two parts. */
BSA_API bsa_status bsa_attention_prepare(const bsa_params *p, const void *q, const void *k, const void *v,
                                 const float *kbar, const float *vbar, const int32_t *blk_count,
                                 const int64_t *row_ptr, const int32_t *col_idx,
                                 const int32_t *extra_idx, const int32_t *extra_count,
                                 void *out, float *lse, void *ws, size_t ws_bytes, void *stream);
BSA_API bsa_status bsa_attention_run(const bsa_params *p, const void *q, const void *k, const void *v,
                             const float *kbar, const float *vbar, const int32_t *blk_count,
                             const int64_t *row_ptr, const int32_t *col_idx,
                             const int32_t *extra_idx, const int32_t *extra_count,
                             void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* Step 4, dense rows ([DOC] sink_conditioning = exact_kv_and_rows: designated
 * query rows attend densely): rows [row_begin, row_end) of every (b, h) attend
 * to all N keys; writes those rows of out (and lse, if not NULL). */
BSA_API bsa_status bsa_dense_ref_rows(const bsa_params *p, const void *q, const void *k, const void *v,
                              int32_t row_begin, int32_t row_end, void *out, float *lse,
                              void *ws, size_t ws_bytes, void *stream);

/* Device buffers for bsa_layer_host.  q, k, v, out hold the whole layer ([B, N,
 * H, d] with p's strides); the others serve one chunk of heads at a time, sized
 * for heads_per_chunk heads as bsa_pool / bsa_select / bsa_attention describe
 * them (qbar [B, hc, nQB, d], kbar and vbar [B, hc, nKB, d], blk_count [nKB],
 * row_ptr [B*hc*nQB + 1], col_idx [col_capacity], kept_count [B*hc*nQB], and
 * with E > 0 extra_idx [B*hc*nQB, E] and extra_count [B*hc*nQB]); ws holds at
 * least bsa_workspace_size() bytes for p with H = heads_per_chunk. */
typedef struct {
    void *q, *k, *v, *out;
    float *qbar, *kbar, *vbar;
    int32_t *blk_count;
    int64_t *row_ptr;
    int32_t *col_idx;
    int64_t col_capacity;
    int32_t *kept_count;
    int32_t *extra_idx, *extra_count;
    void *ws;
    size_t ws_bytes;
} bsa_layer_device;

/* One layer (pool, select, attention, dense rows) whose inputs and output live
 * in host memory: heads are independent, so the layer runs chunk by chunk of
 * heads_per_chunk heads (0: about a sixteenth of them), the copy of chunk c + 1's
 * Q, K, V to the device (on copy_in) and of chunk c - 1's output back (on
 * copy_out) overlapping chunk c's kernels (on stream).  A host array has p's
 * strides, and a chunk is copied as rows of its heads (cudaMemcpy2DAsync);
 * pinned host memory lets the copies run asynchronously.  copy_in / copy_out
 * NULL: everything on `stream`, in order.  No LSE is produced.  Returns after
 * enqueueing; `stream` then waits for the last copy back, so synchronising it
 * (or bsa_device_status(dev->ws, stream, ...)) covers the whole layer.
 * Device-side errors of any chunk go to the status word of dev->ws. */
BSA_API bsa_status bsa_layer_host(const bsa_params *p, const void *q_host, const void *k_host, const void *v_host,
                                  void *out_host, const bsa_layer_device *dev, int32_t heads_per_chunk,
                                  void *stream, void *copy_in, void *copy_out);

/* Synchronise `stream`, return the status the kernels wrote into `ws` since the
 * last call (BSA_OK if none) in *device_status, and clear it.  The return value
 * is BSA_ERR_CUDA if the synchronisation itself failed. */
BSA_API bsa_status bsa_device_status(void *ws, void *stream, int32_t *device_status);

/* Kernels this library has launched since it was loaded, from every thread and
 * on every device (a diagnostic: the difference across a stretch of calls is
 * the number of kernel launches those calls made). */
BSA_API int64_t bsa_launch_count(void);

/* Self-test of the kernels' bounded waits (not a step of the method): one warp
 * waits on an mbarrier that nothing ever arrives on, with a limit of `cycles`
 * SM clock cycles (1 .. 2e9; the pipelines use about one second).  The wait
 * gives up, writes BSA_ERR_DEVICE's timeout code 7 into the status word of
 * `ws` (read it with bsa_device_status) and the kernel returns; nothing traps
 * and the context stays usable. */
BSA_API bsa_status bsa_selftest_bounded_wait(void *ws, int64_t cycles, void *stream);

/* Per-step policy ([DOC] general inputs start_percent, end_percent,
 * dense_blocks, min_tokens and "constraints and limitations"; [STAR]
 * "Hybrid"): whether one attention call takes the sparse path or stays dense.
 * Host-only; nothing is launched.  A dense call runs bsa_dense_ref_rows over
 * all N rows in place of pool / select / attention. */
typedef struct {
    double start_percent;        /* sparse from this fraction of the sampling schedule on ...     */
    double end_percent;          /* ... up to and including this one (both in [0, 1]; 0.2 / 1.0)   */
    int32_t min_tokens;          /* sequences shorter than this stay dense (12288)                */
    int32_t hybrid;              /* 1: the first and last hybrid_guard_steps sampling steps dense */
    int32_t hybrid_guard_steps;  /* guard steps at each end of the schedule (1)                   */
    int32_t pad_;
    const char *dense_blocks;    /* transformer blocks always dense, e.g. "0, 1, 47-49"; NULL or
                                    "" for none (host string, read during the call only)          */
} bsa_policy;

typedef enum {
    BSA_RUN_SPARSE = 0,          /* take the sparse path                                          */
    BSA_DENSE_SHORT = 1,         /* n_tokens < min_tokens                                         */
    BSA_DENSE_BLOCK = 2,         /* block_index listed in dense_blocks                            */
    BSA_DENSE_HYBRID = 3,        /* a guard step of the hybrid schedule                           */
    BSA_DENSE_WINDOW = 4         /* progress outside [start_percent, end_percent]                 */
} bsa_decision;

/* Defaults of the node documentation: window [0.2, 1.0], min_tokens 12288,
 * no dense blocks, hybrid off with one guard step at each end. */
BSA_API void bsa_default_policy(bsa_policy *pol);

/* Decide one call.  n_tokens: sequence length N (>= 1); block_index: the
 * transformer block's index, or < 0 when the model reports none (dense_blocks
 * is then ignored); progress: fraction of the sampling schedule done, in
 * [0, 1]; step / n_steps: the sampling step (0-based) and their number, needed
 * only when hybrid is on (BSA_ERR_INVALID_ARG when they cannot place the step,
 * as the hybrid mode stops when it cannot tell the step).  *decision gets a
 * bsa_decision; reasons are checked in the order of the enum.  A malformed
 * dense_blocks list is BSA_ERR_INVALID_ARG. */
BSA_API bsa_status bsa_policy_decide(const bsa_policy *pol, int32_t n_tokens, int32_t block_index,
                                     double progress, int32_t step, int32_t n_steps, int32_t *decision);

/* Static description of a status code. */
BSA_API const char *bsa_status_string(bsa_status s);

/* Thread-local text of the most recent host-side error of this thread ("" if none). */
BSA_API const char *bsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
