/*
 * st_attn.h -- C ABI of the B200 (sm_100a) factorized sparse causal self-attention library.
 *
 * The method: "Sparse Transformers（稀疏 Transformer）深度解读报告" §2.1-§2.2 (factorized heads,
 * strided and fixed patterns), §3.1 (head integration, Eq.6-8), §3.4 (recompute in the
 * backward pass), §3.5 (block-sparse kernels: blocked computation, fused softmax, the upper
 * triangle never computed).  The block layout follows "长序列为何不必让每个 token 看见全部历史？
 * 滑动窗口、块稀疏与全局 token" §05 (only selected block pairs enter the kernel, boundary blocks
 * carry an element mask) and the attention arithmetic its §01-§02.
 *
 * Allowed sets (0-based positions, every set restricted to j <= i):
 *   strided  A1(i) = {max(0, i-l) .. i}          A2(i) = {j : (i-j) mod l == 0}
 *   fixed    A1(i) = {j : j/l == i/l}            A2(i) = {j : j mod l in [l-c-o, l-1-o]}
 * where o is the fixed pattern-2 head's sub-block offset (below).  A merged head attends to
 * A1 union A2 with one softmax.
 *
 * Arithmetic (per batch b, head h, row i):  S_ij = q_i.k_j / sqrt(d) for j in A(h, i);
 * P_ij = softmax_j(S_ij); O_i = sum_j P_ij v_j; lse_i = ln sum_j exp(S_ij) (natural log, fp32).
 * A row whose allowed set is empty (only the first l-c-o rows of a fixed pattern-2 head) gets
 * O_i = 0 and lse_i = -inf and passes no gradient.  No dropout.  bf16 I/O computes with bf16
 * tensor-core products and fp32 accumulation; fp32 I/O keeps the score product in three-term
 * bf16 split precision (error about 2^-16) and the rest in bf16 products, fp32 accumulation.
 *
 * Conventions for every call:
 *   - Tensors are contiguous row-major [batch, heads, n, width] (lse and the like
 *     [batch, heads, n]), in device memory owned by the caller, each 16-byte aligned; the row
 *     widths are the descriptor's d (Q, K) and dv (V, O), both 64 for the kernels.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *     return after enqueueing work; argument errors are reported before anything is enqueued.
 *   - No call allocates device memory except st_layout_upload (the layout's own tables).
 *   - Nothing throws across this boundary.  A device-side bounded wait that gives up sets the
 *     layout's device error word; st_layout_check reports it (ST_ERR_DEVICE_TIMEOUT).
 */
#ifndef ST_ATTN_H
#define ST_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ST_API __attribute__((visibility("default")))
#else
#define ST_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *st_stream_t; /* same type as cudaStream_t */

typedef enum {
    ST_OK = 0,
    ST_ERR_INVALID_ARG = 1,     /* NULL pointer, bad enum, inconsistent or non-positive sizes */
    ST_ERR_UNSUPPORTED = 2,     /* valid for the method, not handled by the kernels (d != 64 ...) */
    ST_ERR_ALIGNMENT = 3,       /* a tensor pointer is not 16-byte aligned */
    ST_ERR_NOT_UPLOADED = 4,    /* st_layout_upload has not been called for this layout */
    ST_ERR_CUDA = 5,            /* a CUDA runtime or driver call failed */
    ST_ERR_OOM = 6,             /* host or device allocation failed */
    ST_ERR_DEVICE_TIMEOUT = 7,  /* a bounded device wait gave up (see st_layout_check) */
    ST_ERR_WORKSPACE = 8,       /* workspace NULL or smaller than the *_workspace_bytes figure */
    ST_ERR_INTERNAL = 9
} st_status_t;

typedef enum { ST_STRIDED = 1, ST_FIXED = 2 } st_family_t;

/* Head integration ("Sparse Transformers 深度解读报告" §3.1):
 *   ST_PER_HEAD_ALTERNATING  heads alternate pattern head 1 (h even) and head 2 (h odd), Eq.8
 *   ST_MERGED                every head attends to A1 union A2, Eq.7
 *   ST_SINGLE_A1/_A2         every head uses head 1 (resp. head 2): one layer of Eq.6 */
typedef enum {
    ST_PER_HEAD_ALTERNATING = 1,
    ST_MERGED = 2,
    ST_SINGLE_A1 = 3,
    ST_SINGLE_A2 = 4
} st_head_mode_t;

/* Pattern-2 heads of the fixed family are numbered k = 0, 1, ... in head order (k = h/2 when
 * alternating, k = h otherwise) and look at the sub-block shifted by o_k = (k * step) mod l,
 * step = a2_offset_step, or c when a2_offset_step <= 0 (the page's advice that several heads
 * should attend different c-wide sub-blocks, §2.2).  Unused by the strided family. */
typedef struct {
    int32_t family;         /* st_family_t */
    int32_t head_mode;      /* st_head_mode_t */
    int32_t num_heads;      /* 1 .. 64 */
    int32_t a2_offset_step; /* <= 0: c */
} st_pattern_t;

typedef enum { ST_BF16 = 1, ST_FP32 = 2 } st_dtype_t;

/* Shapes of one call.  Q, K, dQ, dK are [batch, heads, n, d]; V, O, dO, dV are
 * [batch, heads, n, dv] ("Sparse Transformers 深度解读报告" §4.5: the models' per-head widths
 * are 32, 64 and 128, and the CIFAR-10 model halves its query-key projection, d = dv / 2).
 * Scores are scaled by 1/sqrt(d).  Widths with kernels: the forward (bf16) and the decode step
 * take (d, dv) = (32, 32), (64, 64), (128, 128) and (64, 128); the backward pass and the fp32
 * forward take (64, 64).  Other widths are valid arguments and return ST_ERR_UNSUPPORTED. */
typedef struct {
    int64_t batch, heads, n, d; /* heads must equal the layout's num_heads, n its n */
    int32_t dtype;              /* st_dtype_t: Q, K, V, O, dO, dQ, dK, dV all in this type */
    int32_t dv;                 /* width of the V, O, dO, dV rows; 0 means d; negative: invalid */
} st_desc_t;

/* Allowed-set kind of one head (st_layout_head_kind). */
typedef enum {
    ST_KIND_SA1 = 1, ST_KIND_SA2 = 2, ST_KIND_SU = 3,
    ST_KIND_FA1 = 4, ST_KIND_FA2 = 5, ST_KIND_FU = 6
} st_kind_t;

typedef struct st_layout st_layout_t; /* opaque; owns its host tables and its device copy */

/* Build the block layout of a pattern (host only, no CUDA call).
 *   n      sequence length, >= 1; the kernels further need n % 128 == 0 and n % l == 0
 *   l      stride / block length, >= 1
 *   c      fixed family: summary width, 1 <= c <= l (kernels: c a power of two <= 128 and
 *          every o_k + c <= l); strided family: ignored
 *   block  64 or 128: granularity of the natural-frame CSR that st_layout_export returns
 * The layout holds, per distinct head kind, the natural-frame CSR of active key blocks per
 * query block with deduplicated element masks of boundary blocks (the bit-exact contract), and
 * the execution-frame work lists the kernels run (128 x 128 tiles; the strided pattern-2 head
 * runs on the (n/l) x l grid view of the sequence, one column per tile row group, the fixed
 * pattern-2 head on its compacted summary keys).  Errors: ST_ERR_INVALID_ARG for invalid
 * values, ST_ERR_OOM.  *out is set only on ST_OK; release with st_layout_destroy. */
ST_API st_status_t st_layout_build(const st_pattern_t *pattern, int64_t n, int32_t l, int32_t c,
                            int32_t block, st_layout_t **out);

/* Copy the execution tables to the current CUDA device, asynchronously on `stream`.  Allocates
 * the layout's device buffers on first call (the only allocation in this library).  A layout
 * is bound to the device current at upload.  Errors: ST_ERR_UNSUPPORTED if the kernels cannot
 * run this layout (n % 128, n % l, c, heads > 64), ST_ERR_CUDA, ST_ERR_OOM. */
ST_API st_status_t st_layout_upload(st_layout_t *layout, st_stream_t stream);

/* Kind (st_kind_t) and fixed sub-block offset o of head `head` (host only).
 * Errors: ST_ERR_INVALID_ARG (NULL layout, head outside [0, num_heads)). */
ST_API st_status_t st_layout_head_kind(const st_layout_t *layout, int32_t head, int32_t *kind,
                                int32_t *offset);

/* Natural-frame CSR of head `head` (borrowed pointers, valid until st_layout_destroy):
 *   query block qb (rows qb*block .. +block-1) lists key blocks col_idx[row_ptr[qb] ..
 *   row_ptr[qb+1]-1] in increasing order; a key block is listed iff some (i, j) in the block pair
 *   is allowed.  mask_id[e] is -1 when every pair of the block is allowed, else the index of
 *   its element mask: masks + mask_id * (block*block/32) u32 words, bit (r*block + cc) set iff
 *   (qb*block + r, kb*block + cc) is allowed, words little-endian.  Rows or columns past n are
 *   never set.  Identical masks are stored once per head kind.  The CSR of a head kind is built
 *   on its first export (the kernels run the execution frames, not this view), so the first call
 *   can take time at long n; ST_ERR_OOM if it does not fit in host memory. */
ST_API st_status_t st_layout_export(const st_layout_t *layout, int32_t head, const int32_t **row_ptr,
                             const int32_t **col_idx, const int32_t **mask_id,
                             const uint32_t **masks, int32_t *n_qblk, int32_t *nnz,
                             int32_t *n_masks);

/* Per batch element figures of the execution plan (host only).  Errors: ST_ERR_INVALID_ARG
 * (NULL argument), ST_ERR_UNSUPPORTED (a layout the kernels cannot run has no plan). */
typedef struct {
    int64_t fwd_items;      /* forward work items (query tiles over all heads and passes) */
    int64_t exec_tiles;     /* active 128 x 128 tile pairs the kernels compute */
    int64_t bwd_items;      /* backward work items (key tiles over all heads and passes) */
    int64_t allowed_pairs;  /* sum over heads and rows of |A(h, i)| */
    int32_t passes;         /* 1, or 2 for merged strided heads (band part, then grid part) */
    int32_t split_passes;   /* passes with a key tile whose query run is split over several CTAs
                               (each adds one short summing launch to the backward pass) */
    int32_t dq_direct_heads; /* heads whose every query tile is read by one backward item: their
                                dQ is written by st_attn_bwd_main, not accumulated */
    int32_t reserved;       /* 0 */
} st_layout_info_t;
ST_API st_status_t st_layout_info(const st_layout_t *layout, st_layout_info_t *info);

/* Host enumeration of the keys row i of head `head` attends in the execution frames (the same
 * frame and interval rules the kernels use), increasing, written to keys[0 .. *count-1];
 * keys must hold n entries.  For tests of the execution plan against the set definitions.
 * Errors: ST_ERR_INVALID_ARG (NULL pointer, head or i out of range), ST_ERR_UNSUPPORTED (a
 * layout the kernels cannot run has no plan). */
ST_API st_status_t st_layout_exec_row(const st_layout_t *layout, int32_t head, int64_t i, int64_t *keys,
                               int64_t *count);

/* Synchronise `stream` and report (and clear) the layout's device error word:
 * ST_ERR_DEVICE_TIMEOUT if a kernel's bounded wait gave up since the last check. */
ST_API st_status_t st_layout_check(st_layout_t *layout, st_stream_t stream);

/* Diagnostic of the failure path: launches one warp on `stream` whose single bounded wait is on
 * an mbarrier that nothing completes, so it gives up after the kernels' wait limit (1 s) and
 * records the timeout in the layout's device error word, as a stalled kernel pipeline would.
 * The next st_layout_check then returns ST_ERR_DEVICE_TIMEOUT (and clears the word); the CUDA
 * context stays usable.  Lets a caller test its error handling without a real fault.
 * Errors: ST_ERR_INVALID_ARG (NULL layout, or the current device is not the layout's),
 * ST_ERR_NOT_UPLOADED, ST_ERR_CUDA (launch failed). */
ST_API st_status_t st_selftest_wait_timeout(st_layout_t *layout, st_stream_t stream);

/* Release the layout's host tables and device buffers (NULL is a no-op).  Work already enqueued
 * that uses the layout must have completed. */
ST_API void st_layout_destroy(st_layout_t *layout);

/* Workspace (device bytes, 256-byte aligned) the calls below need.  0 for a NULL argument or a
 * descriptor whose sizes are invalid (non-positive, or batch x heads x n above 2^40 rows). */
ST_API size_t st_attn_fwd_workspace_bytes(const st_desc_t *desc, const st_layout_t *layout);
ST_API size_t st_attn_bwd_workspace_bytes(const st_desc_t *desc, const st_layout_t *layout);

/* Forward pass.  q, k, v: inputs; o: output; lse: [batch, heads, n] fp32 output.
 * Launches the fused tcgen05 attention kernel (one pass, or two for merged strided heads whose
 * second pass merges by log-sum-exp into the first pass's O and lse).
 * The workspace (st_attn_fwd_workspace_bytes, never 0) starts with the work-unit counters of the
 * persistent kernel, zeroed on `stream` by every call: calls that run at the same time need
 * separate workspaces.  fp32 I/O adds the bf16 copies of q, k and v after them.
 * Errors (nothing enqueued): ST_ERR_INVALID_ARG (NULL pointer; descriptor sizes, heads or n not
 * the layout's; the current device is not the layout's), ST_ERR_UNSUPPORTED (row widths or a
 * layout the kernels do not handle), ST_ERR_ALIGNMENT, ST_ERR_NOT_UPLOADED, ST_ERR_WORKSPACE;
 * ST_ERR_CUDA if a launch fails. */
ST_API st_status_t st_attn_fwd(const void *q, const void *k, const void *v, const st_layout_t *layout,
                        void *o, float *lse, void *workspace, size_t workspace_bytes,
                        const st_desc_t *desc, st_stream_t stream);

/* Backward pass with recomputation ("Sparse Transformers 深度解读报告" §3.4): attention
 * probabilities are rebuilt from q, k and the saved lse.  o, dO: forward output and its
 * gradient; dq, dk, dv: outputs (every element written; keys no query reads get 0).
 * The workspace holds the fp32 dQ accumulator and the per-row D_i = dO_i . O_i.
 * Errors as for st_attn_fwd. */
ST_API st_status_t st_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                        const float *lse, const void *dO, const st_layout_t *layout, void *dq,
                        void *dk, void *dv, void *workspace, size_t workspace_bytes,
                        const st_desc_t *desc, st_stream_t stream);

/* The three phases st_attn_bwd runs, callable one by one on the same stream (in this order,
 * with the same workspace) to time or overlap them:
 *   st_attn_bwd_prepare  D_i = dO_i . O_i into the workspace, zero the fp32 dQ accumulator, and
 *                        zero dK/dV of heads whose keys are not all written by the main phase
 *   st_attn_bwd_main     the recomputing tcgen05 kernel: dK, dV written, dQ accumulated -- or,
 *                        for a head whose every query tile is read by a single key tile (the
 *                        fixed pattern's same-block head with l = 128), written to dq directly
 *   st_attn_bwd_finish   dQ accumulator -> dq (output dtype) for the other heads
 * Arguments as for st_attn_bwd; errors as for st_attn_bwd. */
ST_API st_status_t st_attn_bwd_prepare(const void *o, const void *dO, const st_layout_t *layout,
                                       void *dk, void *dv, void *workspace,
                                       size_t workspace_bytes, const st_desc_t *desc,
                                       st_stream_t stream);
ST_API st_status_t st_attn_bwd_main(const void *q, const void *k, const void *v, const float *lse,
                                    const void *dO, const st_layout_t *layout, void *dq, void *dk,
                                    void *dv,
                                    void *workspace, size_t workspace_bytes,
                                    const st_desc_t *desc, st_stream_t stream);
ST_API st_status_t st_attn_bwd_finish(const st_layout_t *layout, void *dq, void *workspace,
                                      size_t workspace_bytes, const st_desc_t *desc,
                                      st_stream_t stream);

/* Backward pass for callers that cannot allocate device memory (no counterpart in the paper:
 * this is a deployment convenience).  A plug-in inside a host application that owns every device
 * allocation, or code that must not pay cudaMalloc's implicit synchronisation, can call this
 * instead of st_attn_bwd: same arguments and results, but no workspace argument -- the scratch
 * (fp32 dQ accumulator and D_i) lives in a fixed array of ST_NOALLOC_SCRATCH_BYTES that is part of
 * the library's device image, held on every GPU that loads the library until the process exits.
 * Nothing is allocated (no cudaMalloc, cudaFree or allocating library call).
 *   - The first call on a device looks up the array's device address (once per device, with
 *     that device current); make that first call before any stream capture.  The address is
 *     tied to the device's context: after a cudaDeviceReset the next call looks it up again
 *     (that call too should come before any stream capture).
 *   - The limit: a call is accepted when st_attn_bwd_workspace_bytes(desc, layout) <=
 *     ST_NOALLOC_SCRATCH_BYTES; larger problems are rejected with ST_ERR_WORKSPACE before
 *     anything is enqueued.  The workspace grows with batch * heads * n and also holds the
 *     partial dK/dV of split key tiles and, for fp32 I/O, bf16 copies of the inputs, so the row
 *     count alone is only an upper bound: with bf16 I/O and no split key tiles, batch * heads * n
 *     up to about 129,000 rows.
 *   - All calls on a device share the array; each call re-initialises what it reads, but calls
 *     whose work overlaps on the GPU (other streams, other threads) race on it. */
#define ST_NOALLOC_SCRATCH_BYTES (32u << 20)
ST_API st_status_t st_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                                       const float *lse, const void *dO,
                                       const st_layout_t *layout, void *dq, void *dk, void *dv,
                                       const st_desc_t *desc, st_stream_t stream);

/* Decode step ("长序列为何不必让每个 token 看见全部历史？…" §11: incremental inference brings one new
 * query row per step, Q_LEN = 1, against the key/value cache including the new position).
 * For every (batch, head): the query row q[b, h] at sequence position pos attends to its allowed
 * set A(h, pos) among the cache rows 0..pos -- by the set definitions exactly row pos of
 * st_attn_fwd on the full sequence.  Scores and the softmax are computed in fp32 ("Sparse
 * Transformers 深度解读报告" §3.6: query-key products in fp32 when sampling).
 *   q:        [batch, heads, 64] (desc->dtype)
 *   k_cache,
 *   v_cache:  [batch, heads, n, 64], n = the layout's n (the cache capacity); rows past pos are
 *             not read
 *   o:        [batch, heads, 64] output (desc->dtype);  lse: [batch, heads] fp32 output (natural
 *             log; -inf for a row with no allowed key, whose o is 0)
 *   workspace: st_attn_decode_workspace_bytes (a chunk counter per (batch, head), then the per-chunk
 *             partial results), 256-byte aligned; the call zeroes the counters (one memset on
 *             `stream`) and launches one kernel, whose last chunk of each row combines the row's
 *             chunks, so calls that share a workspace must not overlap on the GPU
 * desc is the full-sequence descriptor (its n is the cache capacity).  The layout need not be
 * uploaded: the kernels read only the per-head set kinds, passed by value.  Errors:
 * ST_ERR_INVALID_ARG (NULL pointers, pos outside [0, n), heads or n not the layout's),
 * ST_ERR_UNSUPPORTED (d != 64, more than 64 heads, a row with over 4,194,240 allowed keys),
 * ST_ERR_ALIGNMENT, ST_ERR_WORKSPACE,
 * ST_ERR_CUDA. */
ST_API size_t st_attn_decode_workspace_bytes(const st_desc_t *desc, const st_layout_t *layout);
ST_API st_status_t st_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                                  const st_layout_t *layout, int64_t pos, void *o, float *lse,
                                  void *workspace, size_t workspace_bytes, const st_desc_t *desc,
                                  st_stream_t stream);

/* Host enumeration of the cache rows the decode step reads for head `head` at position pos,
 * increasing, written to keys[0 .. *count-1]; keys must hold pos + 1 entries.  For tests of the
 * decode step's key sets against the set definitions. */
ST_API st_status_t st_decode_row_keys(const st_layout_t *layout, int32_t head, int64_t pos,
                                      int64_t *keys, int64_t *count);

/* Static description of a status code. */
ST_API const char *st_status_string(st_status_t status);

/* Library version string. */
ST_API const char *st_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ST_ATTN_H */
