/*
 * pa.h -- C ABI of libpa.so: ProxyAttn-style block-sparse prefill attention
 * on NVIDIA B200 (sm_100a).
 *
 * The method (ProxyAttn blog, HIT; "4. ProxyAttn method"):
 *   Step 1  head pooling -> token-level proxy scores max-pooled to 128x128
 *           blocks -> ranking of the KV blocks of every query block;
 *   Step 2  a per-head budget estimated from the last query block, combined
 *           with the shared ranking into a block-sparse mask that drives a
 *           FlashAttention-style kernel.
 * Each call below is one of those steps; pa_prefill chains them.
 *
 * Conventions shared by every call
 * --------------------------------
 * Tensors.  q is [B][N][H][d], k and v are [B][N][Hkv][d], o is [B][N][H][d],
 *   all bf16, addressed with pa_strides (element strides of the batch, token
 *   and head dimensions); d is contiguous.  Base pointers must be 16-byte
 *   aligned and every stride a multiple of 8 elements (16 bytes).
 *   Proxies q_proxy/k_proxy are contiguous bf16 [B][G][N][d]; with a
 *   query-row stride r > 1 (see pa_budget.score_stride) q_proxy holds only
 *   the scored rows, [B][G][N/r][d].
 *   Block scores and ranked lists are [B][G][T] with nb = N/128,
 *   T = nb(nb+1)/2 and query block qb's row starting at tri(qb) = qb(qb+1)/2
 *   (entries tri(qb)+0 .. tri(qb)+qb).  With shape->non_causal = 1 every row
 *   holds all nb blocks: T = nb*nb, row qb at qb*nb ("tri(qb)" below then
 *   reads qb*nb, "j <= i" holds for every key and "qb+1" blocks read nb).
 * Heads.  kv(h) = floor(h*Hkv/H) (GQA), grp(h) = floor(h*G/H) (proxy group).
 * Memory.  Every pointer is a device pointer owned by the caller unless a
 *   comment says otherwise.  The library allocates no device memory; calls
 *   that need scratch take a caller-provided workspace (pa_workspace_size).
 * Streams.  Every call is asynchronous on `stream` (a cudaStream_t; 0 is the
 *   legacy default stream).  Argument errors are returned synchronously before
 *   anything is launched; a failed launch returns PA_ERR_CUDA.  Problems found
 *   on the device (a wait that timed out, an index out of range) are recorded
 *   in a device status word read by pa_get_device_status.
 * Threads.  Calls are reentrant; concurrent calls on different streams are
 *   independent except for the shared device status word.
 * Supported.  block = 128, d in {64, 128}, N % 128 == 0, 1 <= N/128 <= 4096,
 *   H % Hkv == 0, H % G == 0, H <= 128, B >= 1.  Others: PA_ERR_UNSUPPORTED.
 * Environment.
 *   PA_WAIT_TIMEOUT_MS  bound, in ms, of every wait inside the kernels
 *                       (default 2000; read once, at the first launch); a
 *                       wait that runs out records PA_ERR_TIMEOUT and the
 *                       kernel abandons its work.
 *   PA_NVTX=1           (read once) every launch, and pa_prefill /
 *                       pa_prefill_varlen as a whole, is wrapped in an NVTX
 *                       range named after its stage ("pa.pool_heads",
 *                       "pa.block_scores", "pa.head_mass", "pa.rank",
 *                       "pa.budget", "pa.block_sparse_attn", "pa.xattn_mask",
 *                       "pa.prefill", "pa.prefill_varlen") for profilers that
 *                       group kernels by range.  Off by default.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 3

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

typedef struct CUstream_st *pa_stream_t; /* same type as cudaStream_t */

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad stride, gamma out of (0,1], ... */
    PA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set above */
    PA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than pa_workspace_size */
    PA_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed */
    PA_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out (kernel abandoned its work) */
    PA_ERR_DEVICE_BOUNDS = 6, /* device: a block index outside 0..qb was met in a list */
    PA_ERR_DEVICE_NONFINITE = 7 /* device: a block score or head mass was NaN/inf */
} pa_status;

typedef struct pa_shape {
    int32_t batch;        /* B */
    int32_t seqlen;       /* N, multiple of 128 */
    int32_t num_q_heads;  /* H */
    int32_t num_kv_heads; /* Hkv, divides H */
    int32_t head_dim;     /* d: 64 or 128 */
    int32_t block;        /* must be 128 */
    int32_t num_groups;   /* G proxy groups, divides H */
    int32_t non_causal;   /* 0: causal prefill (query i attends keys j <= i);
                             1: every query attends every key (bidirectional,
                             e.g. diffusion transformers; XAttention blog,
                             video generation).  Non-causal block scores and
                             ranked lists hold all nb blocks per query block:
                             [B][G][nb*nb], row qb at qb*nb. */
} pa_shape;

typedef struct pa_strides {
    int64_t b, s, h;      /* element strides of the batch, token and head dims */
} pa_strides;

typedef enum pa_budget_mode {
    PA_BUDGET_DYNAMIC = 0,        /* per-head gamma budget from the last query block */
    PA_BUDGET_FIXED_FRACTION = 1, /* ceil(frac_permille * (qb+1) / 1000) blocks per row */
    PA_BUDGET_ALL = 2             /* every causal block (dense causal attention) */
} pa_budget_mode;

typedef struct pa_budget {
    int32_t mode;          /* pa_budget_mode */
    float gamma;           /* DYNAMIC: softmax-mass threshold in (0, 1] */
    int32_t frac_permille; /* FIXED_FRACTION: 1..1000 */
    int32_t score_stride;  /* query-row stride r of the block scores: 0 or 1
                              scores every row; 2, 4 or 8 scores only rows
                              i with i mod r == r-1 (pa_block_scores_strided).
                              Used by pa_prefill and pa_workspace_size. */
    float skip_threshold;  /* BLASST block skip in the attention of pa_prefill
                              (pa_block_sparse_attn_skip): lambda in [0, 1],
                              0 = off */
} pa_budget;

/* Mask buffers written by pa_build_mask / pa_prefill (device, caller-owned).
 *   rank   int32 [B][G][T]  ranked list of each query block:
 *                           [0, qb, then blocks 1..qb-1 by (score desc, index asc)]
 *   cnt    int32 [B][H][nb] blocks head h visits in query block qb: the first
 *                           cnt entries of its group's list
 *   budget int32 [B][H]     per-head budget k_h (= cnt at the last query block)
 *   mass   float [B][H][nb] last-block softmax mass per KV block (DYNAMIC mode;
 *                           may be NULL in the other modes) */
typedef struct pa_mask {
    int32_t *rank;
    int32_t *cnt;
    int32_t *budget;
    float *mass;
} pa_mask;

/* Bytes of workspace pa_prefill needs for this shape and budget (it is also
 * enough for pa_build_mask).  Returns 0 for an invalid or unsupported shape.
 * The workspace is scratch: its contents need no initialisation and are
 * meaningless after the call.  Two calls in flight at once need two
 * workspaces. */
PA_API size_t pa_workspace_size(const pa_shape *shape, const pa_budget *budget);

/* Step 1, "Head Pooling" (ProxyAttn blog, 4. ProxyAttn method, Step 1):
 *   q_proxy[b][g][i][:] = mean over the q heads h of group g of q[b][i][h][:]
 *   k_proxy[b][g][j][:] = mean over the same q heads h of k[b][j][kv(h)][:]
 * Sums run in fp64 over ascending h, the quotient is rounded to bf16 (round to
 * nearest even).  q_proxy, k_proxy: contiguous bf16 [B][G][N][d]. */
PA_API pa_status pa_pool_heads(const pa_shape *shape,
                        const void *q, pa_strides q_strides,
                        const void *k, pa_strides k_strides,
                        void *q_proxy, void *k_proxy, pa_stream_t stream);

/* Step 1, "Score Estimation" (ProxyAttn blog, 4. ProxyAttn method, Step 1;
 * block size from "2. Background: why block-wise"): the QK product of the
 * proxies fused with 128x128 max pooling.  For every (b, g, qb, kb <= qb):
 *   scores[b][g][tri(qb)+kb] = max over i in block qb, j in block kb, j <= i of
 *                              (q_proxy[i] . k_proxy[j]) / sqrt(d)
 * bf16 tensor-core products, fp32 accumulation; token scores never reach
 * memory.  scores: fp32 [B][G][T]. */
PA_API pa_status pa_block_scores(const pa_shape *shape,
                          const void *q_proxy, const void *k_proxy,
                          float *scores, pa_stream_t stream);

/* Step 1 with a query-row stride r in {1, 2, 4, 8} (ProxyAttn blog,
 * "5. Experiments", estimation cost: the pages credit a sequence-level
 * "sliding skip" for keeping the estimate cheap but do not define it; here it
 * is read as scoring only every r-th query row).  The scored rows of a block
 * are i with i mod r == r-1, the last row of each window of r rows.
 *   pa_pool_heads_strided: as pa_pool_heads, but q_proxy is [B][G][N/r][d]
 *     and its row t is the proxy of query row i = t*r + r-1; k_proxy is the
 *     full [B][G][N][d].
 *   pa_block_scores_strided: as pa_block_scores from those proxies, with the
 *     max over the scored rows i of block qb only:
 *       scores[b][g][tri(qb)+kb] = max over i in block qb, i mod r == r-1,
 *                                  j in block kb, j <= i of (q_p[i].k_p[j])/sqrt(d)
 * r = 1 is exactly pa_pool_heads / pa_block_scores.  Other r: PA_ERR_INVALID_ARG. */
PA_API pa_status pa_pool_heads_strided(const pa_shape *shape, int32_t score_stride,
                                       const void *q, pa_strides q_strides,
                                       const void *k, pa_strides k_strides,
                                       void *q_proxy, void *k_proxy, pa_stream_t stream);

PA_API pa_status pa_block_scores_strided(const pa_shape *shape, int32_t score_stride,
                                         const void *q_proxy, const void *k_proxy,
                                         float *scores, pa_stream_t stream);

/* Step 1 "Block Ranking" + Step 2 "dynamic budget" (ProxyAttn blog,
 * 4. ProxyAttn method; the threshold rule is XAttention's find_blocks,
 * XAttention blog 2.2):
 *  - rank: per (b, g, qb) the list [0, qb, then 1..qb-1 by (score desc,
 *    lower index first)] of the scores from pa_block_scores;
 *  - mass (DYNAMIC): for each head h, the exact softmax (scale 1/sqrt(d), causal)
 *    of the last 128 query rows of q against all keys of kv(h); mass[b][h][kb]
 *    = mean over those rows of the probability falling in KV block kb;
 *  - budget: DYNAMIC: with m_fx = rint(mass * 2^40), g_fx = rint(gamma * 2^40),
 *    k_h = smallest k >= |F| (|F| = 2, or 1 when nb = 1) such that the first k
 *    entries of the last row's list carry sum m_fx >= g_fx, else nb;
 *    cnt[b][h][qb] = clamp(ceil(k_h (qb+1) / nb), |F_qb|, qb+1)
 *    (non-causal: every row has nb blocks, cnt = clamp(k_h, |F_qb|, nb)).
 *    FIXED_FRACTION: cnt = clamp(ceil(p (qb+1) / 1000), |F_qb|, qb+1)
 *    (non-causal: ceil(p nb / 1000)).
 *    ALL: cnt = qb+1.  budget = cnt at qb = nb-1.
 * q and k are only read in DYNAMIC mode (may be NULL otherwise).  ws: device
 * workspace of ws_bytes >= pa_workspace_size(shape, budget). */
PA_API pa_status pa_build_mask(const pa_shape *shape, const pa_budget *budget,
                        const float *scores,
                        const void *q, pa_strides q_strides,
                        const void *k, pa_strides k_strides,
                        const pa_mask *out, void *ws, size_t ws_bytes,
                        pa_stream_t stream);

/* pa_build_mask without a workspace argument.  The paper has no counterpart:
 * this entry point exists for callers that cannot hand the library any device
 * scratch memory -- for example a plugin interface whose per-call hook
 * receives no workspace pointer, or a runtime that reserved all device memory
 * up front and does not let the libraries it hosts call cudaMalloc.
 * Same arguments, results and errors as pa_build_mask, minus ws/ws_bytes.
 * Its scratch is a 16 MiB array inside the library (device memory held by
 * every GPU that loads libpa.so until the process exits), so DYNAMIC mode
 * supports batch * num_q_heads * (seqlen/128) <= 16384 (e.g. 32 heads up to
 * 64K tokens); larger shapes return PA_ERR_UNSUPPORTED with that limit in
 * pa_last_error().  The other modes need no scratch.  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress, with that
 * device current); make that first call before any stream capture.  The
 * address is kept for the life of the process, so the device must not be
 * reset (cudaDeviceReset, or a primary context released and created again)
 * after that first call.  The call allocates nothing.  All calls on a device share the one array, so two calls
 * whose kernels overlap on the GPU (different streams, no ordering between
 * them) race on it; calls ordered on one stream are safe.  No contents carry
 * over between calls: each call writes every scratch byte it reads. */
PA_API pa_status pa_build_mask_noalloc(const pa_shape *shape, const pa_budget *budget,
                                       const float *scores,
                                       const void *q, pa_strides q_strides,
                                       const void *k, pa_strides k_strides,
                                       const pa_mask *out, pa_stream_t stream);

/* The block-sparse mask "fed to FlashAttention" (ProxyAttn blog, end of
 * 4. ProxyAttn method; attention formula of "2. Background"): for every
 * (b, h, qb) with list L = rank[b][grp(h)][tri(qb) ..] and n = cnt[b][h][qb],
 *   o[b][i][h] = sum_j softmax_j(softmax_scale * q_i . k_j) v_j
 * over the keys j of blocks L[0..n-1] with j <= i (i in block qb).
 * bf16 tensor-core products, fp32 softmax and accumulation, P rounded to bf16
 * for the PV product.  lse (nullable): fp32 [B][H][N], natural-log
 * log-sum-exp of the scaled logits of each row.  List entries outside 0..qb
 * are skipped and flagged PA_ERR_DEVICE_BOUNDS; lists must not repeat a block.
 * o must not overlap q, k or v. */
PA_API pa_status pa_block_sparse_attn(const pa_shape *shape,
                               const void *q, pa_strides q_strides,
                               const void *k, pa_strides k_strides,
                               const void *v, pa_strides v_strides,
                               const int32_t *rank, const int32_t *cnt,
                               float softmax_scale,
                               void *o, pa_strides o_strides, float *lse,
                               pa_stream_t stream);

/* pa_block_sparse_attn with BLASST's running-max block skip (BLASST,
 * introduction and "3.1 pruning attention with the running max": a block
 * whose scores all lie far below the running maximum contributes almost
 * nothing after the softmax, so its exponentials and its V product are
 * skipped).  The rule's own text is cut off on the pages; as implemented:
 * the blocks of (b, h, qb) are visited in ascending block index; with M_i the
 * running max of row i's scaled logits over the blocks visited before, a
 * block after the first is skipped when for every row i of the query block
 *     max_{j in block, j <= i} softmax_scale * q_i . k_j  <  M_i + ln(lambda)
 * and the output is the softmax attention over the keys of the blocks kept
 * (lse likewise).  skip_threshold = lambda in [0, 1]; 0 never skips and runs
 * exactly pa_block_sparse_attn.  The comparison runs in fp32 on the tensor
 * core's fp32 logits, so a block within rounding of the threshold may be
 * decided either way.  skipped (nullable): uint8 [B][H][T]; the kernel writes
 * 1 at tri(qb)+kb for every block it skips and leaves other entries as they
 * are (zero it first).  K and V of a skipped block are still loaded: the
 * loads are issued ahead of the decision. */
PA_API pa_status pa_block_sparse_attn_skip(const pa_shape *shape,
                                           const void *q, pa_strides q_strides,
                                           const void *k, pa_strides k_strides,
                                           const void *v, pa_strides v_strides,
                                           const int32_t *rank, const int32_t *cnt,
                                           float softmax_scale, float skip_threshold,
                                           void *o, pa_strides o_strides, float *lse,
                                           uint8_t *skipped, pa_stream_t stream);

/* XAttention's estimator (XAttention blog, 2.1 "importance prediction",
 * 2.2 "threshold block selection" and its block-selection algorithm), a second
 * way to build the mask that pa_block_sparse_attn consumes.  Per head h (one
 * list per head: pass the result to pa_block_sparse_attn with a shape whose
 * num_groups = num_q_heads), stride S in {4, 8, 16}:
 *   z[R][c] = sum_{t<S} q[R*S + S-1-t] . k[c*S + t] / (sqrt(d) * S)
 * for strided rows R and columns c (the antidiagonal sum of each S x S
 * sub-block of the score map); each row R is softmax-normalised over c <= R
 * (the causal mask at the sub-block level, a reading: the algorithm shows none);
 *   mass[b][h][tri(qb)+kb] = (S/128) * sum over the 128/S rows R of block qb
 *                            of the probability in block kb's 128/S columns;
 *   rank[b][h][tri(qb) ..]  = blocks 0..qb by (mass desc, lower index first);
 *   cnt[b][h][qb]           = find_blocks: the shortest prefix of that list
 *                            whose masses sum to >= tau (sums in 2^-40 fixed
 *                            point, tau taken as the fp32 value), else qb+1.
 * No block is forced into the set.  bf16 tensor-core products with fp32
 * accumulation; mass (nullable) fp32.  ws: device workspace of
 * ws_bytes >= pa_xattn_workspace_size(shape, S); tau in (0, 1].  The shape's
 * num_groups is not used.  Non-causal shapes (shape->non_causal = 1; the
 * pages' video-generation use) take every strided column, c < N/S, and
 * rows of all nb blocks. */
PA_API size_t pa_xattn_workspace_size(const pa_shape *shape, int32_t stride);

PA_API pa_status pa_xattn_mask(const pa_shape *shape, int32_t stride, float tau,
                               const void *q, pa_strides q_strides,
                               const void *k, pa_strides k_strides,
                               int32_t *rank, int32_t *cnt, float *mass,
                               void *ws, size_t ws_bytes, pa_stream_t stream);

/* The whole path: pa_pool_heads -> pa_block_scores -> pa_build_mask ->
 * pa_block_sparse_attn with softmax_scale = 1/sqrt(d) (the strided pooling
 * and scores when budget->score_stride > 1; the block skip when
 * budget->skip_threshold > 0).  The proxies and block
 * scores live in the workspace; the mask is written to *mask_out (all four
 * buffers required in DYNAMIC mode, mass may be NULL otherwise). */
PA_API pa_status pa_prefill(const pa_shape *shape, const pa_budget *budget,
                     const void *q, pa_strides q_strides,
                     const void *k, pa_strides k_strides,
                     const void *v, pa_strides v_strides,
                     void *o, pa_strides o_strides,
                     const pa_mask *mask_out, void *ws, size_t ws_bytes,
                     pa_stream_t stream);

/* Variable-length batch (the pages' workloads are one sequence per layer
 * call; this is the packed form serving frameworks use): num_seqs sequences
 * packed along the token axis of q, k, v, o ([1][total][heads][d] with the
 * usual strides).  cu_seqlens is a HOST array of num_seqs+1 token offsets:
 * cu_seqlens[0] = 0, every length cu_seqlens[s+1] - cu_seqlens[s] a positive
 * multiple of 128 (at most 4096 blocks), cu_seqlens[num_seqs] =
 * shape->seqlen; shape->batch must be 1.  Sequence s is exactly the
 * single-sequence problem of pa_prefill on its tokens (no attention across
 * sequences), run in order on `stream`, all sequences reusing one workspace of
 * pa_workspace_size_varlen bytes (the longest sequence's).  The mask buffers
 * are packed by sequence, with nb_s = len_s/128 and T_s the entries of one
 * (b, g) row set (nb_s(nb_s+1)/2, or nb_s^2 non-causal):
 *   rank   sequence s at element offset G * sum_{s'<s} T_s', laid out [G][T_s]
 *   cnt    at H * sum_{s'<s} nb_s', [H][nb_s];  mass likewise (DYNAMIC)
 *   budget at H * s, [H]
 * Errors as pa_prefill; a malformed cu_seqlens is PA_ERR_INVALID_ARG (or
 * PA_ERR_UNSUPPORTED for a length outside the supported set).  0 from
 * pa_workspace_size_varlen means invalid arguments. */
PA_API size_t pa_workspace_size_varlen(const pa_shape *shape, const pa_budget *budget,
                                       int32_t num_seqs, const int32_t *cu_seqlens);

PA_API pa_status pa_prefill_varlen(const pa_shape *shape, const pa_budget *budget,
                                   int32_t num_seqs, const int32_t *cu_seqlens,
                                   const void *q, pa_strides q_strides,
                                   const void *k, pa_strides k_strides,
                                   const void *v, pa_strides v_strides,
                                   void *o, pa_strides o_strides,
                                   const pa_mask *mask_out, void *ws, size_t ws_bytes,
                                   pa_stream_t stream);

/* Synchronises `stream`, then returns the device status word of the current
 * device (PA_OK, PA_ERR_TIMEOUT, PA_ERR_DEVICE_BOUNDS or PA_ERR_DEVICE_NONFINITE:
 * the first problem any
 * kernel recorded since the last clear) and, if `clear` is nonzero, resets it.
 * The word is shared by every stream of the device. */
PA_API pa_status pa_get_device_status(pa_stream_t stream, int clear);

/* Diagnostic for failure detection, with no counterpart on the pages: launches
 * one warp that waits on a device barrier nothing ever completes, bounded by
 * timeout_us (1..1000000).  The wait gives up, records PA_ERR_TIMEOUT in the
 * device status word and the kernel returns normally -- the same path every
 * bounded wait in the other kernels takes -- so a caller can check that a
 * timed-out wait is reported (pa_get_device_status) and leaves the context
 * usable, without faulting or hanging the GPU. */
PA_API pa_status pa_selftest_wait_timeout(uint32_t timeout_us, pa_stream_t stream);

/* Static description of a status code. */
PA_API const char *pa_status_string(pa_status status);

/* Thread-local text of the last error a call on this thread returned
 * (empty if none). */
PA_API const char *pa_last_error(void);

/* PA_ABI_VERSION of the loaded library. */
PA_API int32_t pa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
