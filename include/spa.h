/*
 * spa.h -- C ABI of libspa.so: query-aware sparse attention over a long KV cache,
 * hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * The path: score every cached key cheaply (low-rank r=16 index keys, or a second-order
 * Taylor score of 64-token blocks), select a support by top-k or by a sort-free
 * histogram top-p threshold, always keeping the attention sink and the local window,
 * then recompute exact softmax attention on the gathered K/V rows only.
 *
 * Passages (page title, section):
 *   "Full Attention Strikes Back" (RTPurbo) Methodology 1 (sink + sliding window),
 *     2 (r=16 low-rank indexer before RoPE), 3 (dynamic top-p), 5 (sort-free
 *     histogram threshold, bandwidth-optimised sparse decode).
 *   "Oracle-Guided Sparse Prefill" 2.1 (top-k support, sparse recompute with the
 *     original Q/K/V, b_sel = 1 or 64), 2.2 (head-collapsed indexer).
 *   "SPLA" 2.1 (Taylor block score with diagonal covariance).
 *
 * Conventions shared by every entry point
 *   - bf16 tensors are passed as their 16-bit patterns (uint16_t); all tensors are
 *     dense, row-major, in the layouts stated per argument, on the current CUDA device.
 *     bf16 input pointers must be 16-byte aligned.
 *   - The caller owns all memory.  The library allocates nothing on the device.
 *     Entry points that need scratch take a workspace (ws, ws_bytes) sized by the
 *     matching spa_*_workspace_bytes() call.  A workspace must be zero-filled once
 *     before its first use (cudaMemset); every call leaves it ready for the next one.
 *     Calls that share a workspace must not overlap on the GPU.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call is
 *     asynchronous: the returned status covers argument/shape validation and launch
 *     errors only.  Conditions found on the device (a support larger than its
 *     capacity) are OR-ed into a status word at the head of the workspace and read
 *     with spa_read_device_status().
 *   - Supports (idx) are ascending and duplicate-free.  Entries at and beyond
 *     min(count[u], cap) of a row are left untouched.
 *   - Scores are binary32.  Equal scores rank by ascending position.
 *   - No CPU fallback exists: an unsupported shape returns SPA_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef SPA_H
#define SPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum spa_status {
    SPA_OK = 0,
    SPA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, p outside (0, 1], ... */
    SPA_ERR_UNSUPPORTED_SHAPE = 2,   /* head dim, index dim, group size or alignment not supported */
    SPA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the spa_*_workspace_bytes() figure */
    SPA_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed (spa_last_cuda_error) */
    SPA_ERR_TIMEOUT = 5,             /* device: a bounded wait gave up (that call's results are undefined) */
    SPA_ERR_CAPACITY = 6             /* device: a support held more than cap entries (count[u] > cap) */
} spa_status;

typedef enum spa_collapse {
    SPA_COLLAPSE_NONE = 0,       /* one support per query head: U = B * Hq */
    SPA_COLLAPSE_GROUP_MEAN = 1  /* one support per kv head, scored for the mean of its G query heads: U = B * Hkv */
} spa_collapse;

typedef enum spa_score_kind {
    SPA_SCORE_LOWRANK = 0,      /* s_n = scale * qhat . Kidx_n (r = 16) */
    SPA_SCORE_TAYLOR_BLOCK = 1, /* s_b = log t_b, t_b = mean_h exp(q'_h . mean_b)(1 + 1/2 sum_i q'_hi^2 var_bi), q' = scale * q */
    SPA_SCORE_MINMAX_BLOCK = 2, /* s_b = mean_h sum_i max(q'_hi min_bi, q'_hi max_bi): the largest logit in the block's channel box */
    SPA_SCORE_MEAN_BLOCK = 3    /* s_b = mean_h q'_h . mean_b (first-order, mean pooling) */
} spa_score_kind;

/* OR-ed into a block score kind of spa_index_scores: the statistics are bf16 bit patterns
 * (spa_block_stats_bf16 / spa_block_minmax_bf16) instead of fp32; half the bytes. */
#define SPA_STATS_BF16 0x100

typedef enum spa_select_kind {
    SPA_SELECT_TOPK = 0,
    SPA_SELECT_TOPP = 1
} spa_select_kind;

/* Human-readable name of a status code (static string). */
const char* spa_status_string(int status);

/* Text of the last CUDA error seen by this library in the calling thread ("" if none). */
const char* spa_last_cuda_error(void);

/* Test hook of the failure-detection path (the method pages have no counterpart): every wait
 * inside the kernels is bounded and, when its bound runs out, raises SPA_ERR_TIMEOUT in the
 * device status word and leaves the kernel in a defined state.  With a bit set, the next
 * launches of that kernel arm their completion barrier for an arrival that is never issued
 * (nothing is left in flight), use a short bound, and so take that path:
 *   SPA_TEST_STALL_SELECT_LOAD  the selection's bulk load of its chunk of scores; the CTA
 *                               then reads the scores from global memory, so its results
 *                               stay those of a normal run;
 *   SPA_TEST_STALL_PREFILL_MMA  the tcgen05 prefill's first S = Q K^T; the CTA writes no
 *                               output and frees its tensor memory.
 * Process-wide; bits = 0 restores normal launches.  Returns SPA_ERR_INVALID_ARG for unknown
 * bits.  Not for production use. */
#define SPA_TEST_STALL_SELECT_LOAD 1
#define SPA_TEST_STALL_PREFILL_MMA 2
spa_status spa_test_stall(int bits);

/* ABI version of this header: 6 (spa_decode_args gained local_units in 2, the RLA fields in 3;
 * the min-max and mean block scores and spa_block_minmax came in 4; bf16 statistics in 5;
 * spa_select_static_status in 6). */
int spa_abi_version(void);

/* ------------------------------------------------------------------------------------
 * a1. Block statistics ("SPLA" 2.1: first- and second-order block statistics, the
 * covariance replaced by its diagonal).
 *   K     [B, Hkv, N, d] bf16 keys.
 *   mean  [B, Hkv, N / block, d] fp32 out: mean of each full block of `block` tokens.
 *   var   [B, Hkv, N / block, d] fp32 out: population variance (divided by `block`).
 * A trailing partial block (N % block tokens) is not an output.  d in {64, 128};
 * block in {32, 64, 128}.
 */
spa_status spa_block_stats(const uint16_t* K, int B, int Hkv, int N, int d, int block,
                           float* mean, float* var, void* stream);

/* Per-block channel minimum and maximum of K (min/max pooling, the block proxy "SPLA" 1
 * compares against; the statistics of token-to-page selection, "The Sparse Frontier"):
 *   mn, mx [B, Hkv, N / block, d] fp32 out, exact.  Full blocks only; shapes as
 *   spa_block_stats. */
spa_status spa_block_minmax(const uint16_t* K, int B, int Hkv, int N, int d, int block,
                            float* mn, float* mx, void* stream);

/* The same statistics stored as bf16 bit patterns (round to nearest even of the fp32 values;
 * the variance is taken about the fp32 mean; minima and maxima are exact), for scoring with
 * SPA_STATS_BF16 at half the bytes. */
spa_status spa_block_stats_bf16(const uint16_t* K, int B, int Hkv, int N, int d, int block,
                                uint16_t* mean, uint16_t* var, void* stream);
spa_status spa_block_minmax_bf16(const uint16_t* K, int B, int Hkv, int N, int d, int block,
                                 uint16_t* mn, uint16_t* mx, void* stream);

/* ------------------------------------------------------------------------------------
 * a2/a3. Index scores, one row of M scores per selection unit.
 * kind = SPA_SCORE_LOWRANK ("RTPurbo" Methodology 2, head collapse "Oracle-Guided
 * Sparse Prefill" 2.2):
 *   q     [B, Hq, r] bf16 index queries (the projected, pre-RoPE queries), r = dim = 16
 *   keys  [B, Hkv, M, r] bf16 index keys
 *   var   NULL
 *   s[u, n] = scale * qhat_u . keys[b, g, n], where qhat_u is query head h's index query
 *   (collapse NONE, u = b*Hq + h, g = h / G) or the mean of the G index queries of kv
 *   head g (collapse GROUP_MEAN, u = b*Hkv + g; heads summed in order, divided by G).
 * kind = SPA_SCORE_TAYLOR_BLOCK ("SPLA" 2.1):
 *   q     [B, Hq, d] bf16 queries, d = dim in {64, 128}
 *   keys  [B, Hkv, M, d] fp32 block means (M blocks), var [B, Hkv, M, d] fp32 block variances
 *   s[u, b] = log t, t = exp(q'.mean_b) * (1 + 1/2 sum_i q'_i^2 var_bi), q' = scale * q,
 *   with t averaged over the G heads of kv head g (GROUP_MEAN) or per head (NONE).  The
 *   log keeps the score finite for any input; it ranks blocks exactly as t does.
 * kind = SPA_SCORE_MINMAX_BLOCK: keys = block minima, var = block maxima (spa_block_minmax);
 *   s[u, b] = sum_i max(q'_i min_bi, q'_i max_bi), q' = scale * q, scale > 0; averaged
 *   over the G heads under GROUP_MEAN.
 * kind = SPA_SCORE_MEAN_BLOCK: keys = block means, var NULL (not read);
 *   s[u, b] = q' . mean_b; averaged over the G heads under GROUP_MEAN.
 * kind | SPA_STATS_BF16 (block kinds only): keys and var are bf16 bit patterns.
 * scores [U, M] fp32 out.  G = Hq / Hkv must be an integer, G <= 16.
 */
spa_status spa_index_scores(int kind, const void* q, const void* keys, const void* var,
                            int B, int Hq, int Hkv, int M, int dim, int collapse, float scale,
                            float* scores, void* stream);

/* ------------------------------------------------------------------------------------
 * a5/a6. Exact top-k ("Oracle-Guided Sparse Prefill" 2.1) united with the forced sink
 * and window ("RTPurbo" Methodology 1).
 *   scores   [U, M] fp32 (row stride M); unit_len NULL or [U] int32: unit u scores only
 *            its first unit_len[u] <= M entries (L_u = unit_len[u], else M).
 *   The ranking runs over all L_u positions (score desc, position asc); the best k are
 *   kept, then positions [0, sink) and [L_u - window, L_u) are added.
 *   idx      [U, cap] int32 out (ascending); count [U] int32 out (support size; when it
 *            exceeds cap only cap entries are written and SPA_ERR_CAPACITY is flagged).
 *   ws       >= spa_select_workspace_bytes(U, M).
 * The threshold is found by three shared-memory radix-histogram passes over the
 * order-preserving 32-bit keys of the scores (11 + 11 + 10 bits), run by a thread-block
 * cluster per unit; the result is exact.
 */
spa_status spa_select_topk(const float* scores, const int32_t* unit_len, int U, int M, int k,
                           int sink, int window, int32_t* idx, int32_t* count, int cap,
                           void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * a4-a6. Dynamic top-p ("RTPurbo" Methodology 3, sort-free histogram threshold of
 * Methodology 5), united with the sink and window.
 *   With m = max score and e_n = exp(s_n - m), the ranked part is the shortest prefix
 *   of the rank order whose mass reaches p * sum_n e_n (reach = >=); then [0, sink)
 *   and [L_u - window, L_u) are added.  Masses are accumulated as 64-bit fixed-point
 *   integers (e_n scaled by 2^40), so the cut is exact for those masses and independent
 *   of thread order.  0 < p <= 1; L_u <= 2^23.
 *   index_mass [U] fp32 out (optional): mass of the whole support over the total mass.
 * Other arguments as spa_select_topk.
 */
spa_status spa_select_topp(const float* scores, const int32_t* unit_len, int U, int M, float p,
                           int sink, int window, int32_t* idx, int32_t* count, int cap,
                           float* index_mass, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of spa_select_topk / spa_select_topp. */
size_t spa_select_workspace_bytes(int U, int M);

/* ------------------------------------------------------------------------------------
 * Top-p selection that needs no workspace from its caller.  The method pages have no
 * counterpart: this is an interface addition for callers that cannot allocate device
 * memory when they call -- for instance an inference server that reserves all device
 * memory at start-up and forbids allocation on the request path, or a plug-in whose host
 * framework owns every device buffer.
 * Arguments and results are those of spa_select_topp without (ws, ws_bytes).  The
 * scratch (a status word and the level-0 histograms of up to SPA_SELECT_STATIC_MAX_UNITS
 * units, about 960 KiB) is a fixed array in the library's device memory, held by every GPU
 * that loads the library until the process exits.  U > SPA_SELECT_STATIC_MAX_UNITS returns
 * SPA_ERR_UNSUPPORTED_SHAPE.  The first call on a device looks up the array's device
 * address with cudaGetSymbolAddress (with that device current) and caches it; make that
 * first call before any stream capture.  Each call clears the part of the array it uses
 * (cudaMemsetAsync on `stream`) and allocates nothing.  All calls share the one array:
 * calls that overlap on the GPU (other streams, other host threads on the same device)
 * race, and the caller must serialise them.  A support larger than cap shows as
 * count[u] > cap and as SPA_ERR_CAPACITY in the array's status word, which
 * spa_select_static_status reads back.
 */
#define SPA_SELECT_STATIC_MAX_UNITS 16
spa_status spa_select_topp_static(const float* scores, const int32_t* unit_len, int U, int M, float p,
                                  int sink, int window, int32_t* idx, int32_t* count, int cap,
                                  float* index_mass, void* stream);

/* Status word of spa_select_topp_static's fixed scratch (the same interface addition; the
 * method pages have no counterpart): synchronises `stream`, copies the word (sticky OR of
 * (1 << SPA_ERR_*) raised on the device: SPA_ERR_CAPACITY, SPA_ERR_TIMEOUT) to *bits and,
 * if reset != 0, clears it.  Every spa_select_topp_static call starts from a cleared word,
 * so the word describes the last call; read it before the next one.  Allocates nothing.
 * Returns SPA_OK, SPA_ERR_INVALID_ARG (bits NULL) or SPA_ERR_CUDA. */
spa_status spa_select_static_status(void* stream, uint32_t* bits, int reset);

/* ------------------------------------------------------------------------------------
 * a7/a8. Exact softmax attention on the gathered support ("Oracle-Guided Sparse
 * Prefill" 2.1: recompute with the original Q, K, V restricted to the support;
 * "RTPurbo" Methodology 5: bandwidth-optimised sparse decode).
 *   q      [B, Hq, d] bf16 decode queries; K, V [B, Hkv, N, d] bf16 cache.
 *   idx    [U, cap] int32 supports, count [U]: rows of unit u are the first
 *          min(count[u], cap) entries; entry i covers cache rows
 *          [idx*unit_tokens, idx*unit_tokens + unit_tokens).
 *   collapse NONE: U = B*Hq, unit (b, h) serves query head h of kv head h/G.
 *   collapse GROUP_MEAN: U = B*Hkv, unit (b, g) serves the G query heads of kv head g.
 *   out    [B, Hq, d] bf16 out; out_f32 [B, Hq, d] fp32 out (optional);
 *   lse    [B, Hq] fp32 out (optional): log sum_rows exp(sm_scale * q . k_row).
 *   An empty support gives out = 0 and lse = -inf.
 * Split-KV over all SMs: every CTA takes an equal share of all units' rows, gathers
 * them with cp.async and runs an fp32 online softmax on tensor-core tiles.  A CTA that
 * holds a whole unit writes its output; a unit split over several CTAs leaves one
 * partial (o, m, l) per CTA, and a second kernel, one CTA per (unit, head), merges them
 * in a fixed order (log-sum-exp combine).  d in {64, 128}; G <= 16 for GROUP_MEAN.
 * ws >= spa_attend_workspace_bytes.
 */
spa_status spa_sparse_attend(const uint16_t* q, const uint16_t* K, const uint16_t* V,
                             int B, int Hq, int Hkv, int N, int d,
                             const int32_t* idx, const int32_t* count, int cap, int collapse,
                             int unit_tokens, float sm_scale,
                             uint16_t* out, float* out_f32, float* lse,
                             void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of spa_sparse_attend (depends on the current device's SM count). */
size_t spa_attend_workspace_bytes(int B, int Hq, int Hkv, int d, int collapse);

/* ------------------------------------------------------------------------------------
 * Fused decode step: scores (a2 or a3) -> selection (a4-a6) -> attention (a7/a8) in one
 * call, with the scores kept in the workspace.
 */
typedef struct spa_decode_args {
    int score_kind;          /* spa_score_kind */
    int select_kind;         /* spa_select_kind */
    int collapse;            /* spa_collapse */
    int B, Hq, Hkv, N, d;
    int r;                   /* index dim (LOWRANK), 16 */
    int block;               /* tokens per scored unit: 1 (LOWRANK) or the block size (block kinds) */
    const uint16_t* q;       /* [B, Hq, d] */
    const uint16_t* q_idx;   /* [B, Hq, r] (LOWRANK) */
    const uint16_t* K;       /* [B, Hkv, N, d] */
    const uint16_t* V;       /* [B, Hkv, N, d] */
    const uint16_t* Kidx;    /* [B, Hkv, N, r] (LOWRANK) */
    const void* bmean;       /* [B, Hkv, N / block, d]: TAYLOR and MEAN block means; MINMAX block minima (fp32, or bf16 with stats_bf16) */
    const void* bvar;        /* [B, Hkv, N / block, d]: TAYLOR block variances; MINMAX block maxima; MEAN unused */
    float score_scale;       /* LOWRANK: index-score scale; block kinds: q' = score_scale * q */
    float sm_scale;          /* softmax scale of the exact attention */
    int topk;                /* SPA_SELECT_TOPK */
    float topp;              /* SPA_SELECT_TOPP */
    int sink, window;        /* forced leading / trailing scored units */
    int32_t* idx;            /* [U, cap] out */
    int32_t* count;          /* [U] out */
    int cap;
    float* index_mass;       /* [U] out, optional (top-p) */
    uint16_t* out;           /* [B, Hq, d] out */
    float* out_f32;          /* optional */
    float* lse;              /* optional */
    /* Head-wise routing ("Full Attention Strikes Back" (RTPurbo), Methodology 1: local heads
     * attend through a sliding window with an attention sink, retrieval heads through the
     * dynamic sparse selection).  local_units[u] != 0 makes unit u local: it is not scored
     * (GROUP_MEAN: its index keys are not read) and its support is [0, sink) and
     * [M - window, M) only; its index_mass is 0.  NULL: every unit is a retrieval unit.
     * [U] bytes, device memory, read-only. */
    const uint8_t* local_units;
    /* Residual linear attention ("SPLA", sections 2.2-2.3): the rows a support leaves out
     * are condensed by linear attention with the feature map phi(x) = exp(x) (every
     * component), and the output becomes
     *   out = exact sparse attention + gamma * o_rla / sqrt(mean_j o_rla[j]^2 + eps),
     *   o_rla = (phi(q)^T S - sum_sel w v) / (phi(q) . z - sum_sel w),  w = phi(q) . phi(k),
     * where sum_sel runs over the gathered rows (the same tiles the exact attention reads;
     * the left-out rows are never read) and (S, z) is the state of all N rows
     * (spa_rla_state).  o_rla = 0 when the support covers every row.  lse stays the exact
     * attention's.  The subtraction assumes supports without repeated rows and loses
     * precision when the left-out rows carry a tiny share of sum w; binary32 overflows once
     * q[i] + k[i] exceeds about 88 for some component i.
     * rla_state NULL: off (the fields below are not read).  Device memory, fp32, read-only:
     *   rla_state [B, Hkv, d, d]: S[i][j] = sum_n exp(k_n[i]) v_n[j] over rows [0, N);
     *   rla_z     [B, Hkv, d]:    z[i]    = sum_n exp(k_n[i]);
     *   rla_gamma [Hq, d]:        RMSNorm scale of the RLA output, per query head. */
    const float* rla_state;
    const float* rla_z;
    const float* rla_gamma;
    float rla_eps;           /* RMSNorm epsilon, >= 0 */
    int stats_bf16;          /* block kinds: bmean / bvar are bf16 bit patterns (spa_block_*_bf16), else fp32 */
    /* Kernel path (spa_decode_path).  SPA_DECODE_AUTO (the default) and SPA_DECODE_SEPARATE
     * run scoring, selection and attention as separate kernels.  SPA_DECODE_FUSED runs
     * low-rank, head-collapsed decodes (d = 128, G <= 8, 16384 <= N <= 2^23, no local_units,
     * no RLA) as one persistent dataflow kernel, in which every unit's selection chain runs
     * beside the other units' HBM streams, plus a combine kernel (other decodes fall back to
     * the separate kernels).  Supports are identical on both paths; the fused path sums the
     * attention in the order its CTAs claimed the rows, so its outputs may differ between
     * runs in the last bits of fp32.  A workspace serves one path: zero it again before
     * using it with the other. */
    int kernel_path;
} spa_decode_args;

typedef enum spa_decode_path {
    SPA_DECODE_AUTO = 0,
    SPA_DECODE_SEPARATE = 1,
    SPA_DECODE_FUSED = 2
} spa_decode_path;

spa_status spa_decode(const spa_decode_args* a, void* ws, size_t ws_bytes, void* stream);
size_t spa_decode_workspace_bytes(const spa_decode_args* a);

/* The path spa_decode takes for these arguments: SPA_DECODE_FUSED when it runs the fused
 * persistent kernel, SPA_DECODE_SEPARATE otherwise (host-side, no GPU work; -1 for NULL). */
int spa_decode_path_taken(const spa_decode_args* a);

/* spa_decode that also records four caller-created cudaEvent_t on `stream`: events[0]
 * before the scoring kernel, events[1] after it, events[2] after the selection kernel and
 * events[3] after the attention kernel, so a caller can time each kernel inside a real step.
 * On the fused path events[0] precedes the persistent kernel, events[1] and events[2] both
 * follow it and events[3] follows the combine kernel. */
spa_status spa_decode_timed(const spa_decode_args* a, void* ws, size_t ws_bytes, void* stream,
                            void* const* events);

/* ------------------------------------------------------------------------------------
 * RLA state ("SPLA", section 2.2): adds rows [n0, n1) of every (batch, kv head) of the
 * cache into the linear-attention state with the feature map phi(x) = exp(x):
 *   S[bg][i][j] += sum_{n0 <= n < n1} exp(K[bg][n][i]) * V[bg][n][j],
 *   z[bg][i]    += sum_{n0 <= n < n1} exp(K[bg][n][i]).
 * Zero S and z and call it with [0, N) after a prefill, then with [N, N + 1) for each
 * appended token.  K, V [B, Hkv, N, d] bf16 (16-byte aligned); S [B, Hkv, d, d] and
 * z [B, Hkv, d] fp32, device memory, read and written.  Runs on tensor cores with phi(k)
 * carried as two bf16 terms (about 16 significant bits) and fp32 accumulation; the
 * order of summation is fixed, so equal calls give equal bits.  d in {64, 128};
 * 0 <= n0 <= n1 <= N; B * Hkv <= 65535.  n0 == n1 or B == 0 does nothing.
 */
spa_status spa_rla_state(const uint16_t* K, const uint16_t* V, int B, int Hkv, int N, int d, int n0, int n1,
                         float* S, float* z, void* stream);

/* ------------------------------------------------------------------------------------
 * a9. Selection-block-shared sparse prefill ("Oracle-Guided Sparse Prefill" 2.1 with
 * b_sel = bq = 64: one support for 64 consecutive queries; 2.2: head-collapsed indexer).
 * One chunk of T queries at positions q_start .. q_start + T - 1 of a single sequence,
 * against the causal cache of N tokens (the chunk's own keys included).  For query block
 * b (positions t0 = q_start + b*bq ...) and kv head g, unit u = b * Hkv + g:
 *   index query = mean over the block's bq queries and the G heads of g of q_idx;
 *   support     = exact top-k of score_scale * index_query . Kidx[g][n] over n < t0,
 *                 united with the sink [0, sink) (written to idx[u], ascending);
 *   out[t][h]   = softmax(sm_scale * q K^T) V over the support plus the block's own
 *                 positions [t0, t] (causal), for every query t of the block and head h of g.
 * Attention runs on tcgen05 tensor cores with TMEM accumulators.  Requires d = 128,
 * bq = 64, G = Hq / Hkv even, T a multiple of bq with T / bq <= 128, q_start + T <= N,
 * cap >= min(N, topk + sink), sm_scale > 0.  ws >= spa_prefill_workspace_bytes.
 */
typedef struct spa_prefill_args {
    int T, Hq, Hkv, N, d, r;
    int q_start;
    int bq;                   /* queries per shared support: 64 */
    const uint16_t* Q;        /* [T, Hq, d] */
    const uint16_t* q_idx;    /* [T, Hq, r] */
    const uint16_t* K;        /* [Hkv, N, d] */
    const uint16_t* V;        /* [Hkv, N, d] */
    const uint16_t* Kidx;     /* [Hkv, N, r] */
    float score_scale;
    float sm_scale;
    int topk, sink;
    int32_t* idx;             /* [U, cap] out, U = (T / bq) * Hkv */
    int32_t* count;           /* [U] out */
    int cap;
    uint16_t* out;            /* [T, Hq, d] out */
    float* out_f32;           /* optional, [T, Hq, d]; 16-byte aligned */
} spa_prefill_args;

spa_status spa_prefill_shared(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream);
size_t spa_prefill_workspace_bytes(const spa_prefill_args* a);
/* spa_prefill_shared that also records two caller-created cudaEvent_t on `stream`: events[0]
 * right before the tcgen05 attention kernel and events[1] right after it, so a caller can time
 * that kernel inside a real step.  SPA_ERR_INVALID_ARG if events or either event is NULL. */
spa_status spa_prefill_shared_timed(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream,
                                    void* const* events);

/* ------------------------------------------------------------------------------------
 * Per-query sparse prefill ("Oracle-Guided Sparse Prefill" 2.1 with b_sel = 1: every query
 * has its own support; 2.2: head-collapsed indexer).  Same arguments as spa_prefill_shared
 * with bq = 1.  For query t of the chunk (position q_start + t) and kv head g, unit
 * u = t * Hkv + g:
 *   index query = mean of q_idx over the G heads of g;
 *   support     = exact top-k of score_scale * index_query . Kidx[g][n] over n < q_start + t,
 *                 united with the sink [0, sink), ascending in idx[u], count[u] entries;
 *   idx[u][count[u]] = q_start + t (the query's own position, which the attention also reads);
 *   out[t][h]   = softmax(sm_scale * q K^T) V over the support and the own position.
 * One query per support leaves no dense contraction: the path is the decode's scorer,
 * selection and split-KV gather attention on K/V shared by all queries of the chunk.
 * Requires d in {64, 128}, r = 16, G <= 16, q_start + T <= N, T * Hkv <= 8192 and
 * cap >= min(N, topk + sink) + 1.  The workspace holds one score row of N per unit
 * (T * Hkv * N * 4 bytes): chunk long prefills.  ws >= spa_prefill_per_query_workspace_bytes.
 */
spa_status spa_prefill_per_query(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream);
size_t spa_prefill_per_query_workspace_bytes(const spa_prefill_args* a);

/* ------------------------------------------------------------------------------------
 * Permuted block-sparse prefill ("Sparser Block-Sparse Attention via Token Permutation"
 * (PBS-Attn), sections 1-4) of a causal sequence of T tokens: queries and keys at positions
 * 0 .. T-1.  Per kv head g:
 *   importance[g][n] = mean, over the last query block's b queries and the G heads of g, of
 *                      their causal softmax probability softmax(sm_scale * q . k)[n]
 *                      (0 for keys after a query); fp32;
 *   perm[g][s0 + i]  = inside each segment [s0, s0 + S) (the last may be shorter), the keys'
 *                      original positions sorted by descending importance, equal importance by
 *                      ascending position;
 * per query block j (queries [t0, t0 + b), t0 = j * b, segment start seg0 = t0 / S * S) and kv
 * head g, unit u = j * Hkv + g:
 *   the key blocks are the blocks of b consecutive permuted keys in segments 0 .. seg0/S - 1,
 *   scored sm_scale * qbar . kbar (qbar: mean of the block's b x G queries; kbar: mean of the
 *   key block; mean pooling); the top-k blocks (score desc, block asc) are kept, none forced;
 *   idx[u]  = the kept blocks' original positions, ascending (count[u] = kept blocks * b);
 *   out[t][h] = softmax(sm_scale * q K^T) V over the support, the own segment's keys
 *              [seg0, t0) and the block's own positions up to t (causal), on tcgen05.
 * Queries are not permuted, so no inverse permutation of the output is needed.
 * Requires d = 128, b = 64, G = Hq / Hkv even and <= 8, T and S multiples of b, S <= 8192,
 * topk * b <= 8192, cap >= topk * b, sm_scale > 0.  ws >= spa_pbs_workspace_bytes.
 */
typedef struct spa_pbs_args {
    int T, Hq, Hkv, d;
    int b;                    /* block size: 64 */
    int S;                    /* segment size */
    int topk;                 /* key blocks kept per query block */
    float sm_scale;
    const uint16_t* Q;        /* [T, Hq, d] */
    const uint16_t* K;        /* [Hkv, T, d] */
    const uint16_t* V;        /* [Hkv, T, d] */
    float* importance;        /* [Hkv, T] out (optional) */
    int32_t* perm;            /* [Hkv, T] out */
    int32_t* idx;             /* [U, cap] out, U = (T / b) * Hkv */
    int32_t* count;           /* [U] out */
    int cap;
    uint16_t* out;            /* [T, Hq, d] out */
    float* out_f32;           /* optional, [T, Hq, d]; 16-byte aligned */
} spa_pbs_args;

spa_status spa_pbs_prefill(const spa_pbs_args* a, void* ws, size_t ws_bytes, void* stream);
size_t spa_pbs_workspace_bytes(const spa_pbs_args* a);
/* spa_pbs_prefill with two caller-created cudaEvent_t recorded on `stream` around the tcgen05
 * attention kernel (events[0] before, events[1] after).  SPA_ERR_INVALID_ARG if events or
 * either event is NULL. */
spa_status spa_pbs_prefill_timed(const spa_pbs_args* a, void* ws, size_t ws_bytes, void* stream,
                                 void* const* events);

/* ------------------------------------------------------------------------------------
 * Device status word of a workspace (sticky OR of SPA_ERR_* bits as (1 << code)).
 * Synchronises `stream`, copies the word to *bits and, if reset != 0, clears it.
 * Returns SPA_OK or SPA_ERR_CUDA.
 */
spa_status spa_read_device_status(void* ws, void* stream, uint32_t* bits, int reset);

#ifdef __cplusplus
}
#endif

#endif /* SPA_H */
