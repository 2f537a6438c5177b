/*
 * dsa.h - C ABI of the DeepSeek Sparse Attention (DSA) forward path on
 * NVIDIA B200 (sm_100a).
 *
 * The method (page "DeepseekV3.2 拆解", section "核心组件"):
 *   lightning indexer   I[t,s] = sum_{j=1..H^I} w[t,j] * ReLU(q[t,j] . k[s])
 *                       over FP8 indexer queries/keys ("闪电索引器", eq. I_{t,s});
 *   token selection     S_t = Top-k(I[t,:]), k = 2048 in the deployed model
 *                       ("细粒度 Token 选择机制" and the complexity table row
 *                       "DSA 核心注意力");
 *   core attention      u_t = Attn(h_t, {c_s : s in S_t}) over the MLA latent
 *                       rows c_s (eq. u_t); the latent is 576 wide = 512
 *                       value dims + 64 decoupled-RoPE dims (page "DeepSeek
 *                       architecture", section 1.1, "4.5 d_h l" per token).
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer, allocated and owned by the
 *     caller. No call allocates device memory and the library keeps no
 *     caller pointer after a call returns. The one exception to "no library
 *     memory" is static: the 16 MiB scratch array of
 *     dsa_sparse_attn_noalloc, which every GPU that loads the library holds
 *     until the process exits.
 *   - Per-device facts (kernel attributes, the SM count, the scratch array's
 *     address) are looked up on first use and cached for the process. Do
 *     not use the library across a cudaDeviceReset (or any teardown of the
 *     device's primary context): the cached state would be stale.
 *   - Every call is asynchronous on the caller's CUDA stream (`stream`, a
 *     cudaStream_t passed as void*; NULL = legacy default stream). No call
 *     synchronises except dsa_check(). Inside dsa_forward[_ex], the top-k
 *     and attention kernels that follow a score kernel are programmatic
 *     dependent launches (they may start their set-up while the kernel
 *     before them finishes, and wait for it before reading its output); the
 *     first kernel of every call is an ordinary launch, so every call is
 *     ordered after the caller's earlier work on the stream as usual.
 *   - Argument errors are detected on the host BEFORE any launch and reported
 *     by the return value; dsa_last_error() gives a one-line reason.
 *   - Device-side failures (a bounded wait that ran out) set a per-device
 *     error word that dsa_check() reads and clears. Kernels never trap.
 *   - Scales (q_scale, k_scale) must be finite and > 0 (amax/448, or 1 for an
 *     all-zero row); the kernels rely on ReLU(a*x) = a*ReLU(x) for a > 0.
 *   - Validity: key s is visible to query row i of sequence b iff
 *       s <= q_pos0[b] + i  and  s < kv_len[b].
 *     q_pos0 / kv_len are device int32 [batch] arrays, or NULL for
 *     q_pos0 = 0 (prefill from position 0) and kv_len = n_kv.
 *     Decode: n_q = 1 and q_pos0[b] = kv_len[b] - 1.
 *   - Supported shapes (others return DSA_ERR_UNSUPPORTED):
 *       (idx_heads, idx_dim) in {(64, 128), (4, 32)};
 *       (heads, qk_dim, v_dim) in {(128, 576, 512), (8, 64, 64)};
 *       1 <= topk; n_q, n_kv >= 1; batch >= 1.
 */
#ifndef DSA_B200_DSA_H_
#define DSA_B200_DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, row range, ...      */
  DSA_ERR_UNSUPPORTED = 2,  /* shape outside the compiled tile set         */
  DSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required  */
  DSA_ERR_CUDA = 4,         /* a CUDA runtime call failed                  */
  DSA_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out          */
  DSA_ERR_NO_DEVICE = 6     /* no sm_100 device is current                 */
} dsa_status;

typedef enum { DSA_OUT_F32 = 0, DSA_OUT_BF16 = 1 } dsa_out_dtype;

typedef enum { DSA_SCORES_ALL = 0, DSA_SCORES_VISIBLE_ONLY = 1 } dsa_scores_flags;

typedef enum {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_ATTN = 2,
  DSA_OP_FORWARD = 3,
  DSA_OP_INDEXER_KL = 4
} dsa_op;

typedef struct {
  int32_t batch;          /* B                                              */
  int32_t n_q;            /* query rows per sequence (T)                    */
  int32_t n_kv;           /* key / latent rows per sequence (S)             */
  int32_t idx_heads;      /* H^I, indexer heads                             */
  int32_t idx_dim;        /* d^I, indexer head dim (bytes per fp8 row)      */
  int32_t topk;           /* k                                              */
  int32_t heads;          /* H, attention query heads (share one latent)    */
  int32_t qk_dim;         /* D_qk, dims of q and of the latent row          */
  int32_t v_dim;          /* D_v, value dims = the first v_dim latent dims  */
  float softmax_scale;    /* logits = softmax_scale * q . c                 */
} dsa_shape;

/*
 * Where the keys and the query positions of a call live. Every call below
 * has an _ex variant that takes a `const dsa_layout*` right after the shape;
 * NULL (and the plain call) means contiguous caches and consecutive rows.
 *
 * Paged caches (the PagedAttention layout, page "DeepSeek-V3 MoE blog",
 * section 4.1): with block_table set, the key inputs k_fp8, k_scale and kv
 * are POOLS of pool_rows rows, and logical key s of sequence b is pool row
 *     block_table[b * max_pages + s / page_size] * page_size + s % page_size.
 * Indices (dsa_topk's output, dsa_sparse_attn's input) stay logical key
 * positions. Every page that kv_len[b] (or n_kv) reaches must be mapped. A
 * page outside [0, pool_rows / page_size) is not read: its keys count as
 * zero vectors, and the next dsa_check() returns DSA_ERR_INVALID_ARG.
 *
 * Explicit query positions: with row_pos set, query row i of sequence b sits
 * at absolute position row_pos[b * n_q + i] (visibility: s <= row_pos and
 * s < kv_len), instead of q_pos0[b] + i. This lets the query rows of one
 * prefill be split over several calls or GPUs in any grouping; the fused
 * indexer treats every 4 consecutive rows of the call as one tile group, so
 * keep rows of nearby positions together and in increasing order for speed
 * (any order is correct).
 */
typedef struct {
  const int32_t* row_pos;      /* [B, n_q] device int32, or NULL               */
  const int32_t* block_table;  /* [B, max_pages] device int32, or NULL         */
  int32_t max_pages;           /* row stride of block_table,
                                  >= ceil(n_kv / page_size)                    */
  int32_t page_size;           /* keys per page: power of two in [128, 65536]  */
  int64_t pool_rows;           /* rows of the key pools: a multiple of
                                  page_size, below 2^31 - 256                  */
} dsa_layout;

/*
 * Indexer scores (page "DeepseekV3.2 拆解", eq. I_{t,s}), materialised.
 *   q_fp8   [B, n_q, H^I, d^I] e4m3fn codes     q_scale [B, n_q, H^I] fp32
 *   w       [B, n_q, H^I] fp32 head weights
 *   k_fp8   [B, n_kv, d^I] e4m3fn codes         k_scale [B, n_kv] fp32
 *   rows [row_begin, row_end) of every sequence are scored:
 *   scores  [B, row_end-row_begin, n_kv] fp32; invisible keys get -inf,
 *           unless flags has DSA_SCORES_VISIBLE_ONLY: then only the visible
 *           keys of each row are written (what dsa_topk reads) and the rest
 *           of the buffer is left as it was.
 *   I[t,s] = k_scale[s] * sum_j (w[t,j] q_scale[t,j]) ReLU(q8[t,j] . k8[s]),
 *   the dot products exact-product / fp32-accumulated on the tensor cores.
 */
dsa_status dsa_indexer_scores(const dsa_shape* shape, const uint8_t* q_fp8,
                              const float* q_scale, const float* w,
                              const uint8_t* k_fp8, const float* k_scale,
                              const int32_t* q_pos0, const int32_t* kv_len,
                              int32_t row_begin, int32_t row_end,
                              int32_t flags, float* scores, void* stream);
dsa_status dsa_indexer_scores_ex(const dsa_shape* shape, const dsa_layout* layout,
                                 const uint8_t* q_fp8, const float* q_scale, const float* w,
                                 const uint8_t* k_fp8, const float* k_scale,
                                 const int32_t* q_pos0, const int32_t* kv_len,
                                 int32_t row_begin, int32_t row_end, int32_t flags,
                                 float* scores, void* stream);

/*
 * Per-row FP8 quantisation of the indexer inputs (page "DeepseekV3.2 拆解",
 * section "闪电索引器": the indexer computes in FP8). For each row r of dim
 * values: scale[r] = amax_r / 448 (1 when the row is all zero), and
 * codes[r, d] = E4M3(clamp(x[r, d] / scale[r], -448, 448)) rounded to
 * nearest even (saturating, sign of zero kept). scale and x / scale are
 * fp32 IEEE operations, so the codes are reproducible bit for bit.
 *   x      [rows, dim] bf16 (raw bits)   (2 * dim / 32 -byte aligned)
 *   codes  [rows, dim] e4m3fn codes      (dim / 32 -byte aligned)
 *   scales [rows] fp32
 * The indexer's q_fp8 / q_scale are the rows of [B, T, H^I, d^I] (one scale
 * per token and head) and k_fp8 / k_scale those of [B, S, d^I]. dim must be
 * 32, 64 or 128 (DSA_ERR_UNSUPPORTED otherwise); rows = 0 launches nothing.
 */
dsa_status dsa_quantize_e4m3(int64_t rows, int32_t dim, const uint16_t* x, uint8_t* codes,
                             float* scales, void* stream);

/*
 * Indexer scores and top-k selection in one kernel (page "DeepseekV3.2 拆解",
 * section "闪电索引器", eq. I_{t,s}, and section "细粒度 Token 选择机制",
 * eq. u_t). Inputs and row range as dsa_indexer_scores; the score of each
 * (row, key) pair is computed exactly as dsa_indexer_scores computes it but
 * is never written to memory: each row keeps its candidates in shared memory
 * and only the selection leaves the GPU's SMs.
 *   indices [B, row_end-row_begin, topk] int32, as dsa_topk writes them:
 *           min(m, topk) distinct key indices of the m visible keys (the
 *           largest scores, ties to the lower index), then -1 padding, in
 *           unspecified order within a row.
 *   Supported: idx_heads = 64, idx_dim = 128, topk <= 2048; otherwise
 *   DSA_ERR_UNSUPPORTED before any launch (use dsa_indexer_scores + dsa_topk).
 *   No workspace. dsa_forward uses this kernel whenever the shape is
 *   supported and there are at least as many 4-row query groups as SMs.
 */
dsa_status dsa_indexer_topk(const dsa_shape* shape, const uint8_t* q_fp8,
                            const float* q_scale, const float* w,
                            const uint8_t* k_fp8, const float* k_scale,
                            const int32_t* q_pos0, const int32_t* kv_len,
                            int32_t row_begin, int32_t row_end, int32_t* indices,
                            void* stream);
dsa_status dsa_indexer_topk_ex(const dsa_shape* shape, const dsa_layout* layout,
                               const uint8_t* q_fp8, const float* q_scale, const float* w,
                               const uint8_t* k_fp8, const float* k_scale,
                               const int32_t* q_pos0, const int32_t* kv_len,
                               int32_t row_begin, int32_t row_end, int32_t* indices,
                               void* stream);

/*
 * Top-k selection per score row (page "DeepseekV3.2 拆解", eq. u_t: keep the
 * k keys with the largest I[t,s]).
 *   scores  [B, row_end-row_begin, n_kv] fp32 (as written by
 *           dsa_indexer_scores for the same rows); only the visible keys of
 *           each row are read.
 *   indices [B, row_end-row_begin, topk] int32. A row with m visible keys
 *           gets min(m, topk) distinct key indices, then -1 padding. Among
 *           equal scores the lower key index wins. The order of the
 *           selected indices within a row is unspecified.
 *   No workspace is needed (ws may be NULL, ws_bytes 0).
 */
dsa_status dsa_topk(const dsa_shape* shape, const float* scores,
                    int32_t row_begin, int32_t row_end,
                    const int32_t* q_pos0, const int32_t* kv_len,
                    int32_t* indices, void* ws, size_t ws_bytes, void* stream);
/* Only layout->row_pos matters here (scores are logical key positions). */
dsa_status dsa_topk_ex(const dsa_shape* shape, const dsa_layout* layout, const float* scores,
                       int32_t row_begin, int32_t row_end,
                       const int32_t* q_pos0, const int32_t* kv_len,
                       int32_t* indices, void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse MQA attention over the selected latent rows (eq. u_t).
 *   q       [B, n_q, H, D_qk] bf16
 *   kv      [B, n_kv, D_qk] bf16 latent rows; K = kv[s, :D_qk],
 *           V = kv[s, :D_v], shared by all H heads
 *   indices [B, n_q, topk] int32 key indices into kv of the same sequence,
 *           -1 = empty slot (skipped). Indices outside [0, n_kv) are treated
 *           as empty.
 *   out     [B, n_q, H, D_v] fp32 or bf16 (out_dtype)
 *   lse     [B, n_q, H] fp32 natural-log sum of exp of the logits, or NULL.
 *   p = softmax(softmax_scale * q . K) over the row's slots, out = p V.
 *   A row with no valid slot gets out = 0 and lse = -inf.
 *   Workspace: dsa_workspace_size(shape, DSA_OP_SPARSE_ATTN) bytes (split-K
 *   partials for short query counts), 256-byte aligned.
 */
dsa_status dsa_sparse_attn(const dsa_shape* shape, const uint16_t* q,
                           const uint16_t* kv, const int32_t* indices,
                           void* out, int32_t out_dtype, float* lse,
                           void* ws, size_t ws_bytes, void* stream);
/* Only layout->block_table (and its sizes) matters here. */
dsa_status dsa_sparse_attn_ex(const dsa_shape* shape, const dsa_layout* layout,
                              const uint16_t* q, const uint16_t* kv, const int32_t* indices,
                              void* out, int32_t out_dtype, float* lse,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * dsa_sparse_attn without a caller-provided workspace. The paper has no
 * counterpart: this entry point exists for callers that cannot call
 * cudaMalloc - code whose device memory belongs to another framework's
 * allocator, or a latency-critical decode loop that must not pay for (or
 * synchronise on) an allocation - and so cannot hand in the split-K
 * workspace that dsa_sparse_attn asks for when only a few query rows run.
 *
 * The split-K partials live in a static device array inside the library
 * (16 MiB; every GPU that loads the library holds it until the process
 * exits). Arguments, layouts and results are those of dsa_sparse_attn.
 *   - Returns DSA_ERR_WORKSPACE, before any launch, when the shape's split-K
 *     partials need more than 16 MiB (dsa_workspace_size(shape,
 *     DSA_OP_SPARSE_ATTN) > 16 MiB); use dsa_sparse_attn for those.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first
 *     call before any stream capture.
 *   - Every call shares the one array and it keeps the last call's
 *     contents; each call writes every partial it reads, so nothing needs
 *     clearing. Calls that overlap on the GPU (different streams, or other
 *     host threads) race on it: serialise them.
 *   - It allocates no device or host memory.
 */
dsa_status dsa_sparse_attn_noalloc(const dsa_shape* shape, const uint16_t* q,
                                   const uint16_t* kv, const int32_t* indices,
                                   void* out, int32_t out_dtype, float* lse,
                                   void* stream);

/*
 * The whole path for all n_q rows: indexer -> top-k -> sparse attention
 * (page "DeepseekV3.2 拆解", eq. I_{t,s} and eq. u_t).
 *   Indexer inputs as dsa_indexer_scores, attention inputs as
 *   dsa_sparse_attn. indices_out [B, n_q, topk] receives the selection
 *   (required). Workspace: dsa_workspace_size(shape, DSA_OP_FORWARD) bytes,
 *   256-byte aligned; ws may be NULL when that is 0.
 *   Plan: when dsa_indexer_topk supports the shape and there are at least
 *   as many 4-row query groups as SMs (prefill), the indexer and the top-k
 *   are one launch and no score is stored (workspace: only the attention's
 *   split-K partials, usually none). Otherwise (decode, other shapes) the
 *   score kernel and dsa_topk run per chunk of dsa_forward_chunk_rows()
 *   rows, through a score buffer in the workspace.
 */
dsa_status dsa_forward(const dsa_shape* shape, const uint8_t* q_fp8,
                       const float* q_scale, const float* w,
                       const uint8_t* k_fp8, const float* k_scale,
                       const int32_t* q_pos0, const int32_t* kv_len,
                       const uint16_t* q, const uint16_t* kv,
                       int32_t* indices_out, void* out, int32_t out_dtype,
                       float* lse, void* ws, size_t ws_bytes, void* stream);
dsa_status dsa_forward_ex(const dsa_shape* shape, const dsa_layout* layout,
                          const uint8_t* q_fp8, const float* q_scale, const float* w,
                          const uint8_t* k_fp8, const float* k_scale,
                          const int32_t* q_pos0, const int32_t* kv_len,
                          const uint16_t* q, const uint16_t* kv,
                          int32_t* indices_out, void* out, int32_t out_dtype,
                          float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Indexer warm-up loss and its gradient (page "DeepseekV3.2 拆解", section
 * "预训练策略 / 密集预热阶段": with the main model frozen, the indexer is
 * trained to follow the dense attention distribution,
 *     L^I = sum_t KL(p_{t,:} || Softmax(I_{t,:}))).
 *   p_{t,:}   the main attention's dense causal softmax of query row t over
 *             its visible keys (softmax_scale * q . kv over all qk_dim
 *             dims), averaged over the H heads;
 *   I_{t,:}   the indexer scores of dsa_indexer_scores over the same keys.
 *   Inputs:   the indexer inputs of dsa_indexer_scores (all n_q rows) and the
 *             attention inputs q [B, n_q, H, D_qk], kv [B, n_kv, D_qk] bf16.
 *   Outputs (fp32, written in full):
 *     loss [B, n_q]          KL of each row (sum them for L^I);
 *     dw   [B, n_q, H^I]     dL/dw;
 *     dq   [B, n_q, H^I, d^I] dL/dq^ with q^ = code * q_scale (the FP8
 *                            encoding passes the gradient through);
 *     dk   [B, n_kv, d^I]    dL/dk^ with k^ = code * k_scale (zero for keys
 *                            no row sees).
 *   p on the tensor cores (bf16, fp32 accumulate); the loss rows and the
 *   gradient sums in fp32. The ReLU mask [q^ . k^ > 0] is the sign of the
 *   tensor-core dot product (exact products, fp32 sum).
 *   Workspace: dsa_workspace_size(shape, DSA_OP_INDEXER_KL) bytes (16 per
 *   (row, key) of a row chunk), 256-byte aligned. Contiguous caches only.
 */
dsa_status dsa_indexer_kl(const dsa_shape* shape, const uint8_t* q_fp8,
                          const float* q_scale, const float* w,
                          const uint8_t* k_fp8, const float* k_scale,
                          const int32_t* q_pos0, const int32_t* kv_len,
                          const uint16_t* q, const uint16_t* kv,
                          float* loss, float* dw, float* dq, float* dk,
                          void* ws, size_t ws_bytes, void* stream);

/* Rows per indexer/top-k step that dsa_forward uses for this shape. With
 * the fused plan it is n_q (one dsa_indexer_topk launch over all rows, no
 * score storage). Otherwise the scores of `rows` query rows (rows * n_kv
 * fp32 per sequence) are the only score storage, so the L x L matrix is
 * never held at once; a caller that composes the path from the stage calls
 * gets the same launches by scoring [r, r + rows) with
 * DSA_SCORES_VISIBLE_ONLY and selecting from it. */
dsa_status dsa_forward_chunk_rows(const dsa_shape* shape, int32_t* rows);

/* The plan dsa_forward takes for this shape, for callers that compose the
 * path from the stage calls (or time its kernels one by one):
 *   *fused       1 when the indexer and the top-k run as one
 *                dsa_indexer_topk launch over all rows, else 0 (score kernel
 *                + dsa_topk per chunk of *chunk_rows rows);
 *   *chunk_rows  as dsa_forward_chunk_rows;
 *   *attn_splits split-K factor of the attention (1 = no partials, else a
 *                combine kernel follows the attention kernel).
 * Host-only; a shape outside the compiled set returns its error. */
dsa_status dsa_forward_plan(const dsa_shape* shape, int32_t* fused, int32_t* chunk_rows,
                            int32_t* attn_splits);

/* Workspace bytes an op needs for this shape (0 if none). Returns status. */
dsa_status dsa_workspace_size(const dsa_shape* shape, int32_t op,
                              size_t* bytes);

/* Synchronises `stream`, then returns DSA_ERR_CUDA for a pending CUDA error,
 * DSA_ERR_TIMEOUT if a kernel's bounded wait ran out since the last check,
 * DSA_ERR_INVALID_ARG if a kernel met a block-table page outside its pool
 * (the error word is cleared), else DSA_OK. */
dsa_status dsa_check(void* stream);

/* Static description of a status code. */
const char* dsa_status_string(dsa_status status);

/* Reason for the last non-OK status returned on this host thread. */
const char* dsa_last_error(void);

/* Library version, e.g. "0.1.0". */
const char* dsa_version(void);

/*
 * Failure-detection self-test (the paper has no counterpart). Launches one
 * small kernel that waits, with the same bounded wait every kernel uses, on
 * a barrier that nothing completes; after limit_ms milliseconds (1..10000)
 * the wait gives up, sets the device error word and the kernel exits
 * normally. The next dsa_check() on the stream returns DSA_ERR_TIMEOUT (and
 * clears the word); the context stays usable. Nothing faults or traps.
 */
dsa_status dsa_selftest_wait_timeout(uint32_t limit_ms, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_DSA_H_ */
