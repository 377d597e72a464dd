// Plain, slow, fp64 CPU oracle for query-aware sparse attention over a long KV cache.
//
// TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU-baseline
// leg use this library.  It shares no code, header, table or helper with the CUDA
// library; both sides meet only in the seeded inputs.
//
// Every routine works on ONE unit (one batch entry and one kv head, or one query
// head) at a time, in double precision, and follows the definitions on the method
// pages literally: no blocking, fusion or reordering beyond what a definition states.
// bf16 inputs are widened exactly to double.
//
// Passages followed (page title, section):
//   [RTP-2]  "Full Attention Strikes Back" (RTPurbo), Methodology 2: r=16 low-rank
//            projector on q and k, relevance scored in that subspace.
//   [RTP-3]  RTPurbo, Methodology 3: dynamic top-p -- accumulate attention mass in
//            the low-rank space until the cumulative threshold p is reached.
//   [RTP-1]  RTPurbo, Methodology 1: local heads keep an attention sink and a sliding
//            window; every support here keeps both.
//   [OGS-2.1] "Oracle-Guided Sparse Prefill", section 2.1: head-averaged attention
//            mass P_{l,t}; top-k support; attention recomputed with the original
//            Q, K, V restricted to the support; b_sel = 1 or 64.
//   [OGS-2.2] same page, section 2.2: head-collapsed indexer, one shared scoring
//            channel per GQA group.
//   [SPLA-2.1] "SPLA", section 2.1: block score exp(q^T kbar)(1 + 1/2 q^T Cov(k) q)
//            with Cov(k) replaced by its diagonal.
//   [SPLA-2.2] "SPLA", section 2.2: residual linear attention (RLA) over the blocks the
//            selection left out, with the parameter-free feature map phi(x) = exp(x); its
//            IO form subtracts linear attention over the selected rows from linear
//            attention over all rows, so the left-out rows are never read.
//   [SPLA-2.3] same page, section 2.3: the output is the exact sparse attention plus the
//            RLA output passed through an RMSNorm whose scale is the only new parameter.
//   [SPLA-1] "SPLA", section 1: the block proxies it improves on -- min/max pooling and
//            plain mean pooling of a block's keys.
//   [SF-4]   "The Sparse Frontier", decoding findings: token-to-page selection over a full
//            KV cache (Quest) for decode.
//   [PBS-1]  "Sparser Block-Sparse Attention via Token Permutation" (PBS-Attn), section 1:
//            attention is invariant to a joint permutation of the key-value pairs.
//   [PBS-2]  same page, section 2: keys are permuted only inside contiguous segments of
//            S tokens, so causality between segments is kept.
//   [PBS-3]  same page, section 3: the global importance of a key is the mean-pooled
//            attention it receives from the last query block; inside each segment keys are
//            sorted by descending importance; queries keep their order.
//   [PBS-4]  same page, section 4: blocks of the permuted keys are selected by a
//            mean-pooled block score, then attention runs over the selected blocks.
//
// Parity pins (tests/test_oracle.py): dense attention and masked attention against
// torch's fp64 scaled_dot_product_attention, top-k against numpy's lexsort, top-p
// against brute force over all subsets, block statistics against numpy mean/var,
// the Taylor score's zero-variance identity and fourth-order agreement on
// axis-symmetric blocks, the prefill path against dense causal attention, and the
// residual linear attention's subtraction form against its direct definition, its
// closed forms (zero query, one left-out row) and brute-force Python loops, and the
// permuted block-sparse prefill against dense causal attention (full budget), the
// segment-local causal attention (empty budget), its invariance to a shuffle of the
// key-value pairs inside segments, and a planted cluster of scattered heavy hitters.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

namespace {

inline double widen_bf16(uint16_t h) {
    uint32_t u = static_cast<uint32_t>(h) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

// Order of positions by score, highest first; equal scores by ascending position
// (the tie-break shared by top-k and top-p).
std::vector<int64_t> rank_order(const double* s, int64_t M) {
    std::vector<int64_t> order(M);
    std::iota(order.begin(), order.end(), int64_t{0});
    std::sort(order.begin(), order.end(), [s](int64_t a, int64_t b) {
        if (s[a] != s[b]) return s[a] > s[b];
        return a < b;
    });
    return order;
}

// Forced positions [RTP-1]: the sink [0, sink) and the window [M - window, M).
void mark_forced(std::vector<char>& keep, int64_t M, int64_t sink, int64_t window) {
    for (int64_t n = 0; n < std::min(sink, M); ++n) keep[n] = 1;
    for (int64_t n = std::max<int64_t>(0, M - window); n < M; ++n) keep[n] = 1;
}

int64_t emit_ascending(const std::vector<char>& keep, int32_t* idx) {
    int64_t c = 0;
    for (int64_t n = 0; n < static_cast<int64_t>(keep.size()); ++n)
        if (keep[n]) idx[c++] = static_cast<int32_t>(n);
    return c;
}

}  // namespace

extern "C" {

int orc_abi_version() { return 5; }

// a1 -- per-block mean and diagonal (population) variance of K [SPLA-2.1].
// K: [N, d] bf16 of one (batch, kv head); only the nb = N / block full blocks count.
// mean, var: [nb, d].  Variance divides by the block size: the score is an
// expectation over the block's own tokens.
void orc_block_stats(const uint16_t* K, int64_t N, int d, int block, double* mean, double* var) {
    const int64_t nb = N / block;
    std::vector<double> acc(d);
    for (int64_t b = 0; b < nb; ++b) {
        std::fill(acc.begin(), acc.end(), 0.0);
        for (int t = 0; t < block; ++t)
            for (int i = 0; i < d; ++i) acc[i] += widen_bf16(K[(b * block + t) * d + i]);
        for (int i = 0; i < d; ++i) mean[b * d + i] = acc[i] / block;
        std::fill(acc.begin(), acc.end(), 0.0);
        for (int t = 0; t < block; ++t)
            for (int i = 0; i < d; ++i) {
                const double e = widen_bf16(K[(b * block + t) * d + i]) - mean[b * d + i];
                acc[i] += e * e;
            }
        for (int i = 0; i < d; ++i) var[b * d + i] = acc[i] / block;
    }
}

// a2 -- low-rank index scores [RTP-2], head-collapsed when asked [OGS-2.2].
// qidx: [G, r] bf16 index queries of the G query heads sharing this kv head;
// kidx: [N, r] bf16 index keys.
// collapse = 0: out [G, N], out[h, n] = scale * qidx_h . kidx_n
// collapse = 1: out [N], scored with the mean index query over the G heads
//               (heads summed in order 0..G-1, then divided by G), which is the
//               average of the G heads' scores.
void orc_lowrank_scores(const uint16_t* qidx, int G, const uint16_t* kidx, int64_t N, int r,
                        int collapse, double scale, double* out) {
    const int nq = collapse ? 1 : G;
    std::vector<double> qv(static_cast<size_t>(nq) * r, 0.0);
    if (collapse) {
        for (int h = 0; h < G; ++h)
            for (int j = 0; j < r; ++j) qv[j] += widen_bf16(qidx[h * r + j]);
        for (int j = 0; j < r; ++j) qv[j] /= G;
    } else {
        for (int h = 0; h < G; ++h)
            for (int j = 0; j < r; ++j) qv[h * r + j] = widen_bf16(qidx[h * r + j]);
    }
    for (int h = 0; h < nq; ++h)
        for (int64_t n = 0; n < N; ++n) {
            double dot = 0.0;
            for (int j = 0; j < r; ++j) dot += qv[h * r + j] * widen_bf16(kidx[n * r + j]);
            out[h * N + n] = scale * dot;
        }
}

// a3 -- second-order Taylor block score with diagonal covariance [SPLA-2.1]:
//   t_{h,b} = exp(q'_h . kbar_b) * (1 + 1/2 * sum_i q'_{h,i}^2 var_{b,i}),  q' = scale * q.
// q: [G, d] bf16; mean, var: [nb, d].
// collapse = 0: out [G, nb]; collapse = 1: out [nb] = mean over the G heads of t_{h,b}.
void orc_taylor_scores(const uint16_t* q, int G, const double* mean, const double* var, int64_t nb,
                       int d, double scale, int collapse, double* out) {
    std::vector<double> qp(static_cast<size_t>(G) * d);
    for (int h = 0; h < G; ++h)
        for (int i = 0; i < d; ++i) qp[h * d + i] = scale * widen_bf16(q[h * d + i]);
    for (int64_t b = 0; b < nb; ++b) {
        double sum_heads = 0.0;
        for (int h = 0; h < G; ++h) {
            double lin = 0.0, quad = 0.0;
            for (int i = 0; i < d; ++i) {
                lin += qp[h * d + i] * mean[b * d + i];
                quad += qp[h * d + i] * qp[h * d + i] * var[b * d + i];
            }
            const double t = std::exp(lin) * (1.0 + 0.5 * quad);
            if (collapse) sum_heads += t;
            else out[h * nb + b] = t;
        }
        if (collapse) out[b] = sum_heads / G;
    }
}

// Positions sorted by (score desc, position asc); order: [M].
void orc_rank_order(const double* s, int64_t M, int64_t* order) {
    const std::vector<int64_t> o = rank_order(s, M);
    std::copy(o.begin(), o.end(), order);
}

// a5/a6 -- exact top-k [OGS-2.1] united with the forced sink and window [RTP-1].
// The ranking runs over all M positions; the k best (ties by ascending position) are
// kept, then the sink [0, sink) and window [M - window, M) are added.  idx receives
// the support in ascending order (room for min(M, k + sink + window) entries).
// Returns the support size.
int64_t orc_select_topk(const double* s, int64_t M, int64_t k, int64_t sink, int64_t window,
                        int32_t* idx) {
    const std::vector<int64_t> order = rank_order(s, M);
    std::vector<char> keep(M, 0);
    for (int64_t i = 0; i < std::min(k, M); ++i) keep[order[i]] = 1;
    mark_forced(keep, M, sink, window);
    return emit_ascending(keep, idx);
}

// a4-a6 -- dynamic top-p [RTP-3] united with the forced sink and window [RTP-1].
// pi_n = exp(s_n - m) / Z is the softmax of the scores over all M positions
// (m = max score, Z summed in rank order).  The ranked part is the shortest prefix of
// the rank order whose cumulative mass reaches p * Z ("reaches" read as >=).  The
// sink and window are then added.  idx receives the ascending support (room for M).
// index_mass (optional) = sum of pi_n over the whole support; cut (optional) = length
// of the ranked prefix.  Requires 0 < p <= 1; returns -1 otherwise.
int64_t orc_select_topp(const double* s, int64_t M, double p, int64_t sink, int64_t window,
                        int32_t* idx, double* index_mass, int64_t* cut) {
    if (!(p > 0.0 && p <= 1.0) || M <= 0) return -1;
    const std::vector<int64_t> order = rank_order(s, M);
    const double m = s[order[0]];
    std::vector<double> e(M);
    double Z = 0.0;
    for (int64_t i = 0; i < M; ++i) {
        e[i] = std::exp(s[order[i]] - m);
        Z += e[i];
    }
    const double target = p * Z;
    int64_t c = 0;
    double cum = 0.0;
    while (c < M) {
        cum += e[c];
        ++c;
        if (cum >= target) break;
    }
    std::vector<char> keep(M, 0);
    for (int64_t i = 0; i < c; ++i) keep[order[i]] = 1;
    mark_forced(keep, M, sink, window);
    if (index_mass) {
        double kept = 0.0;
        for (int64_t n = 0; n < M; ++n)
            if (keep[n]) kept += std::exp(s[n] - m);
        *index_mass = kept / Z;
    }
    if (cut) *cut = c;
    return emit_ascending(keep, idx);
}

// a7/a8 -- exact softmax attention recomputed on a support [OGS-2.1].
// q: [G, d] bf16 (the query heads that share this support); K, V: [N, d] bf16 rows of
// one kv head.  The support lists cnt entries; entry i stands for the rows
// [idx[i] * unit_tokens, idx[i] * unit_tokens + unit_tokens) (unit_tokens = 1 for
// token supports, the block size for block supports), in any order.
// out: [G, d]; lse: [G], lse_h = log sum_{rows} exp(sm_scale * q_h . k_row).
// An empty support gives out = 0 and lse = -inf.
void orc_sparse_attention(const uint16_t* q, int G, const uint16_t* K, const uint16_t* V, int64_t N,
                          int d, const int32_t* idx, int64_t cnt, int unit_tokens, double sm_scale,
                          double* out, double* lse) {
    std::vector<int64_t> rows;
    rows.reserve(static_cast<size_t>(cnt) * unit_tokens);
    for (int64_t i = 0; i < cnt; ++i)
        for (int t = 0; t < unit_tokens; ++t) {
            const int64_t row = static_cast<int64_t>(idx[i]) * unit_tokens + t;
            if (row >= 0 && row < N) rows.push_back(row);
        }
    std::vector<double> logit(rows.size());
    for (int h = 0; h < G; ++h) {
        double* o = out + static_cast<int64_t>(h) * d;
        std::fill(o, o + d, 0.0);
        if (rows.empty()) {
            if (lse) lse[h] = -std::numeric_limits<double>::infinity();
            continue;
        }
        double mx = -std::numeric_limits<double>::infinity();
        for (size_t j = 0; j < rows.size(); ++j) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i)
                dot += widen_bf16(q[h * d + i]) * widen_bf16(K[rows[j] * d + i]);
            logit[j] = sm_scale * dot;
            mx = std::max(mx, logit[j]);
        }
        double Z = 0.0;
        for (size_t j = 0; j < rows.size(); ++j) {
            const double w = std::exp(logit[j] - mx);
            Z += w;
            for (int i = 0; i < d; ++i) o[i] += w * widen_bf16(V[rows[j] * d + i]);
        }
        for (int i = 0; i < d; ++i) o[i] /= Z;
        if (lse) lse[h] = mx + std::log(Z);
    }
}

// Dense head-averaged attention distribution P [OGS-2.1]:
// P[n] = (1/G) sum_h softmax_n(sm_scale * q_h . k_n) over all N rows.  Used for the
// captured-mass metric sum_{n in S} P[n]; with G = 1 it is one head's distribution.
void orc_dense_probs(const uint16_t* q, int G, const uint16_t* K, int64_t N, int d, double sm_scale,
                     double* P) {
    std::fill(P, P + N, 0.0);
    std::vector<double> logit(N);
    for (int h = 0; h < G; ++h) {
        double mx = -std::numeric_limits<double>::infinity();
        for (int64_t n = 0; n < N; ++n) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += widen_bf16(q[h * d + i]) * widen_bf16(K[n * d + i]);
            logit[n] = sm_scale * dot;
            mx = std::max(mx, logit[n]);
        }
        double Z = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            logit[n] = std::exp(logit[n] - mx);
            Z += logit[n];
        }
        for (int64_t n = 0; n < N; ++n) P[n] += logit[n] / Z / G;
    }
}

// a9 -- selection-block-shared sparse prefill for one (query block, kv head) unit
// [OGS-2.1 b_sel = bq, OGS-2.2 head-collapsed indexer].
// qblk: [bq, G, d] bf16 queries of the block (positions t0 .. t0+bq-1) for the G query
// heads of the kv head; qidx_blk: [bq, G, r] their index queries.  K, V: [N, d];
// kidx: [N, r] of the kv head.
// 1. index query = mean of qidx_blk over the bq queries and G heads (summed in
//    (query, head) order, divided by bq*G);
// 2. scores s_n = idx_scale * index_query . kidx_n over the candidates n in [0, t0)
//    (rounded to binary32 when rank_f32 != 0, the precision a binary32 ranking sees);
// 3. support = exact top-k of those scores united with the sink [0, sink)
//    (written ascending to support, room for min(t0, k + sink)); returns its size;
//    the ranked scores are copied to scores_out [t0] when it is not null;
// 4. each query t0+i and head h attends, with the original q/K/V, to the support
//    plus its own block's causal prefix [t0, t0+i]: out [bq, G, d].
int64_t orc_prefill_unit(const uint16_t* qblk, const uint16_t* qidx_blk, int bq, int G, int d, int r,
                         const uint16_t* K, const uint16_t* V, const uint16_t* kidx, int64_t N,
                         int64_t t0, double idx_scale, int64_t k, int64_t sink, double sm_scale,
                         int rank_f32, int32_t* support, double* out, double* scores_out) {
    if (t0 < 0 || t0 + bq > N) return -1;
    std::vector<double> qhat(r, 0.0);
    for (int i = 0; i < bq; ++i)
        for (int h = 0; h < G; ++h)
            for (int j = 0; j < r; ++j) qhat[j] += widen_bf16(qidx_blk[(i * G + h) * r + j]);
    for (int j = 0; j < r; ++j) qhat[j] /= static_cast<double>(bq) * G;
    std::vector<double> s(t0);
    for (int64_t n = 0; n < t0; ++n) {
        double dot = 0.0;
        for (int j = 0; j < r; ++j) dot += qhat[j] * widen_bf16(kidx[n * r + j]);
        s[n] = idx_scale * dot;
        if (rank_f32) s[n] = static_cast<double>(static_cast<float>(s[n]));
    }
    if (scores_out) std::copy(s.begin(), s.end(), scores_out);
    const int64_t cnt = t0 > 0 ? orc_select_topk(s.data(), t0, k, sink, 0, support) : 0;

    std::vector<int32_t> rows(support, support + cnt);
    for (int i = 0; i < bq; ++i) {
        rows.resize(cnt);
        for (int j = 0; j <= i; ++j) rows.push_back(static_cast<int32_t>(t0 + j));
        for (int h = 0; h < G; ++h)
            orc_sparse_attention(qblk + (static_cast<int64_t>(i) * G + h) * d, 1, K, V, N, d, rows.data(),
                                 static_cast<int64_t>(rows.size()), 1, sm_scale,
                                 out + (static_cast<int64_t>(i) * G + h) * d, nullptr);
    }
    return cnt;
}

// ---------------------------------------------------------------- residual linear attention
// Rows of a support (selection units idx[0..cnt) of unit_tokens rows each), kept in
// [0, N), in the order they are gathered.
static std::vector<int64_t> support_rows(const int32_t* idx, int64_t cnt, int unit_tokens, int64_t N) {
    std::vector<int64_t> rows;
    for (int64_t i = 0; i < cnt; ++i)
        for (int t = 0; t < unit_tokens; ++t) {
            const int64_t row = static_cast<int64_t>(idx[i]) * unit_tokens + t;
            if (row >= 0 && row < N) rows.push_back(row);
        }
    return rows;
}

// Linear-attention weight of row n for query q [SPLA-2.2]: phi(q) . phi(k_n) with phi = exp
// applied to every component.
static double rla_weight(const uint16_t* q, const uint16_t* K, int64_t n, int d) {
    double w = 0.0;
    for (int i = 0; i < d; ++i) w += std::exp(widen_bf16(q[i])) * std::exp(widen_bf16(K[n * d + i]));
    return w;
}

// RLA state of rows [n0, n1) [SPLA-2.2]: S[i][j] = sum_n exp(k_n[i]) v_n[j], z[i] = sum_n exp(k_n[i]).
void orc_rla_state(const uint16_t* K, const uint16_t* V, int d, int64_t n0, int64_t n1, double* S, double* z) {
    std::fill(S, S + static_cast<int64_t>(d) * d, 0.0);
    std::fill(z, z + d, 0.0);
    for (int64_t n = n0; n < n1; ++n)
        for (int i = 0; i < d; ++i) {
            const double f = std::exp(widen_bf16(K[n * d + i]));
            z[i] += f;
            for (int j = 0; j < d; ++j) S[static_cast<int64_t>(i) * d + j] += f * widen_bf16(V[n * d + j]);
        }
}

// RLA output by its definition [SPLA-2.2]: normalised linear attention of every query head
// over the rows of [0, N) that the support leaves out,
//   o = sum_{n not in S} w_n v_n / sum_{n not in S} w_n,   w_n = phi(q) . phi(k_n);
// o = 0 when the support covers every row.  q [G, d]; o [G, d].
void orc_rla_direct(const uint16_t* q, int G, const uint16_t* K, const uint16_t* V, int64_t N, int d,
                    const int32_t* idx, int64_t cnt, int unit_tokens, double* o) {
    std::vector<char> in_support(static_cast<size_t>(N), 0);
    for (int64_t row : support_rows(idx, cnt, unit_tokens, N)) in_support[static_cast<size_t>(row)] = 1;
    for (int h = 0; h < G; ++h) {
        double* oh = o + static_cast<int64_t>(h) * d;
        std::fill(oh, oh + d, 0.0);
        double den = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            if (in_support[static_cast<size_t>(n)]) continue;
            const double w = rla_weight(q + static_cast<int64_t>(h) * d, K, n, d);
            den += w;
            for (int j = 0; j < d; ++j) oh[j] += w * widen_bf16(V[n * d + j]);
        }
        if (den > 0.0)
            for (int j = 0; j < d; ++j) oh[j] /= den;
    }
}

// RLA output in the pages' IO form [SPLA-2.2]: the global linear attention of the state
// (S, z) over all rows minus the linear attention over the gathered support rows, taken for
// numerator and normaliser alike: o = (phi(q)^T S - sum_sel w v) / (phi(q) . z - sum_sel w).
// o = 0 when the support covers every row.  Equal to orc_rla_direct for a support without
// repeated rows.
void orc_rla_subtract(const uint16_t* q, int G, const uint16_t* K, const uint16_t* V, int64_t N, int d,
                      const int32_t* idx, int64_t cnt, int unit_tokens, const double* S, const double* z,
                      double* o) {
    const std::vector<int64_t> rows = support_rows(idx, cnt, unit_tokens, N);
    for (int h = 0; h < G; ++h) {
        const uint16_t* qh = q + static_cast<int64_t>(h) * d;
        double* oh = o + static_cast<int64_t>(h) * d;
        std::vector<double> num(d, 0.0);
        double den = 0.0;
        for (int i = 0; i < d; ++i) {
            const double f = std::exp(widen_bf16(qh[i]));
            den += f * z[i];
            for (int j = 0; j < d; ++j) num[j] += f * S[static_cast<int64_t>(i) * d + j];
        }
        for (int64_t n : rows) {
            const double w = rla_weight(qh, K, n, d);
            den -= w;
            for (int j = 0; j < d; ++j) num[j] -= w * widen_bf16(V[n * d + j]);
        }
        const bool covered = static_cast<int64_t>(rows.size()) >= N;
        for (int j = 0; j < d; ++j) oh[j] = covered ? 0.0 : num[j] / den;
    }
}

// RMSNorm with scale [SPLA-2.3]: y = gamma * x / sqrt(mean(x^2) + eps), x [d].
void orc_rms_norm(const double* x, int d, const double* gamma, double eps, double* y) {
    double ms = 0.0;
    for (int j = 0; j < d; ++j) ms += x[j] * x[j];
    ms /= d;
    const double inv = 1.0 / std::sqrt(ms + eps);
    for (int j = 0; j < d; ++j) y[j] = gamma[j] * x[j] * inv;
}

// ---------------------------------------------------------------- PBS-Attn prefill
// Global importance of every key [PBS-3]: the mean, over the bl queries of the last query
// block (positions t_last0 ...) and the G query heads sharing the kv head, of their causal
// softmax probabilities softmax_n(sm_scale * q . k_n), n <= t (0 for keys after t).
// Qlast [bl, G, d] bf16; K [T, d] bf16; imp [T] out.
void orc_pbs_importance(const uint16_t* Qlast, int bl, int G, int64_t t_last0, const uint16_t* K, int64_t T,
                        int d, double sm_scale, double* imp) {
    std::fill(imp, imp + T, 0.0);
    std::vector<double> logit(static_cast<size_t>(T));
    for (int i = 0; i < bl; ++i)
        for (int h = 0; h < G; ++h) {
            const uint16_t* q = Qlast + (static_cast<int64_t>(i) * G + h) * d;
            const int64_t t = std::min(t_last0 + i, T - 1);
            double mx = -std::numeric_limits<double>::infinity();
            for (int64_t n = 0; n <= t; ++n) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += widen_bf16(q[c]) * widen_bf16(K[n * d + c]);
                logit[static_cast<size_t>(n)] = sm_scale * dot;
                mx = std::max(mx, logit[static_cast<size_t>(n)]);
            }
            double Z = 0.0;
            for (int64_t n = 0; n <= t; ++n) Z += std::exp(logit[static_cast<size_t>(n)] - mx);
            for (int64_t n = 0; n <= t; ++n)
                imp[n] += std::exp(logit[static_cast<size_t>(n)] - mx) / Z / (static_cast<double>(bl) * G);
        }
}

// Intra-segment key order [PBS-2, PBS-3]: inside each segment [j S, min((j + 1) S, T)) the
// keys sorted by descending importance, equal importance by ascending position.
// perm[p] = original position of the key at permuted position p.
void orc_pbs_permutation(const double* imp, int64_t T, int64_t S, int32_t* perm) {
    for (int64_t s0 = 0; s0 < T; s0 += S) {
        const int64_t len = std::min(S, T - s0);
        const std::vector<int64_t> order = rank_order(imp + s0, len);
        for (int64_t p = 0; p < len; ++p) perm[s0 + p] = static_cast<int32_t>(s0 + order[static_cast<size_t>(p)]);
    }
}

// One (query block, kv head) of the permuted block-sparse prefill [PBS-1..4].
// Qblk [b, G, d] bf16: the block's queries at positions t0 .. t0 + b - 1 (t0 a multiple of
// b, S a multiple of b) for the G heads of the kv head; K, V [T, d] bf16; perm from
// orc_pbs_permutation.  The query block lies in segment j = t0 / S.  Candidates are the
// blocks of b consecutive permuted keys in segments 0 .. j - 1; block c scores
// sm_scale * qbar . kbar_c, qbar the mean of the block's b x G queries and kbar_c the mean
// of the block's keys (mean pooling); the k best (score desc, block asc) are selected.
// support [min(k, candidates) * b] out: the original positions of the selected keys,
// ascending; returns their number.  out [b, G, d]: for query t and head h, softmax
// attention over the support and the keys [j S, t] of its own segment (causal by original
// position; the diagonal segment is never skipped).
int64_t orc_pbs_prefill_unit(const uint16_t* Qblk, int b, int G, int d, int64_t t0, const uint16_t* K,
                             const uint16_t* V, int64_t T, const int32_t* perm, int64_t S, int64_t k,
                             double sm_scale, int32_t* support, double* out) {
    if (b <= 0 || S % b != 0 || t0 % b != 0 || t0 + b > T) return -1;
    const int64_t seg0 = t0 / S * S;
    const int64_t nc = seg0 / b;                       // candidate blocks
    std::vector<double> qbar(d, 0.0);
    for (int i = 0; i < b; ++i)
        for (int h = 0; h < G; ++h)
            for (int c = 0; c < d; ++c) qbar[c] += widen_bf16(Qblk[(static_cast<int64_t>(i) * G + h) * d + c]);
    for (int c = 0; c < d; ++c) qbar[c] /= static_cast<double>(b) * G;
    std::vector<double> score(static_cast<size_t>(nc));
    for (int64_t blk = 0; blk < nc; ++blk) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) {
            double kbar = 0.0;
            for (int64_t p = blk * b; p < (blk + 1) * b; ++p) kbar += widen_bf16(K[static_cast<int64_t>(perm[p]) * d + c]);
            dot += qbar[c] * (kbar / b);
        }
        score[static_cast<size_t>(blk)] = sm_scale * dot;
    }
    const std::vector<int64_t> order = rank_order(score.data(), nc);
    const int64_t nsel = std::min<int64_t>(std::max<int64_t>(k, 0), nc);
    std::vector<int32_t> rows;
    for (int64_t r = 0; r < nsel; ++r)
        for (int64_t p = order[static_cast<size_t>(r)] * b; p < (order[static_cast<size_t>(r)] + 1) * b; ++p)
            rows.push_back(perm[p]);
    std::sort(rows.begin(), rows.end());
    std::copy(rows.begin(), rows.end(), support);
    const int64_t n_sup = static_cast<int64_t>(rows.size());
    for (int i = 0; i < b; ++i) {
        const int64_t t = t0 + i;
        std::vector<int32_t> all(rows);
        for (int64_t n = seg0; n <= t; ++n) all.push_back(static_cast<int32_t>(n));
        for (int h = 0; h < G; ++h) {
            const int64_t qi = static_cast<int64_t>(i) * G + h;
            orc_sparse_attention(Qblk + qi * d, 1, K, V, T, d, all.data(), static_cast<int64_t>(all.size()), 1,
                                 sm_scale, out + qi * d, nullptr);
        }
    }
    return n_sup;
}

// ---------------------------------------------------------------- first-order block proxies
// Per-block channel minimum and maximum of K [SPLA-1] (full blocks only, like a1).
// K [N, d] bf16; mn, mx [N / block, d] out.
void orc_block_minmax(const uint16_t* K, int64_t N, int d, int block, double* mn, double* mx) {
    const int64_t nb = N / block;
    for (int64_t b = 0; b < nb; ++b)
        for (int c = 0; c < d; ++c) {
            double lo = std::numeric_limits<double>::infinity(), hi = -lo;
            for (int64_t n = b * block; n < (b + 1) * block; ++n) {
                lo = std::min(lo, widen_bf16(K[n * d + c]));
                hi = std::max(hi, widen_bf16(K[n * d + c]));
            }
            mn[b * d + c] = lo;
            mx[b * d + c] = hi;
        }
}

// Min-max page score [SPLA-1, SF-4]: the largest scale * q . k over every k inside the
// block's channel box [mn, mx], s_{h,b} = scale * sum_i max(q_i mn_{b,i}, q_i mx_{b,i}); an
// upper bound of every key's logit in the block.  q [G, d] bf16; collapse = 0: out [G, nb];
// collapse = 1: out [nb] = mean over the G heads.
void orc_minmax_scores(const uint16_t* q, int G, const double* mn, const double* mx, int64_t nb, int d,
                       double scale, int collapse, double* out) {
    for (int64_t b = 0; b < nb; ++b) {
        double acc = 0.0;
        for (int h = 0; h < G; ++h) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) {
                const double qc = widen_bf16(q[h * d + c]);
                s += std::max(qc * mn[b * d + c], qc * mx[b * d + c]);
            }
            s *= scale;
            if (collapse) acc += s; else out[h * nb + b] = s;
        }
        if (collapse) out[b] = acc / G;
    }
}

// Mean-pooling block score [SPLA-1, PBS-4]: s_{h,b} = scale * q_h . kbar_b (the first-order
// term of the Taylor score).  mean [nb, d]; collapse as orc_minmax_scores.
void orc_mean_scores(const uint16_t* q, int G, const double* mean, int64_t nb, int d, double scale, int collapse,
                     double* out) {
    for (int64_t b = 0; b < nb; ++b) {
        double acc = 0.0;
        for (int h = 0; h < G; ++h) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += widen_bf16(q[h * d + c]) * mean[b * d + c];
            s *= scale;
            if (collapse) acc += s; else out[h * nb + b] = s;
        }
        if (collapse) out[b] = acc / G;
    }
}

// ---------------------------------------------------------------- bf16 storage
// Round-to-nearest-even of doubles to bf16 bit patterns (8 significant bits), directly from
// double, for statistics stored in bf16.  Finite inputs within the bf16 range.
void orc_round_bf16(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        const double v = x[i];
        if (v == 0.0) {
            out[i] = std::signbit(v) ? 0x8000u : 0u;
            continue;
        }
        int e;
        std::frexp(std::fabs(v), &e);                 // |v| = m * 2^e, m in [0.5, 1)
        const double ulp = std::ldexp(1.0, std::max(e - 8, -133));   // spacing of bf16 values near |v|
        const double q = std::fabs(v) / ulp;          // exact: a power-of-two scaling
        double r = std::floor(q);
        const double frac = q - r;
        if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
        const float f = static_cast<float>(std::copysign(r * ulp, v));   // exact in binary32
        uint32_t u;
        std::memcpy(&u, &f, sizeof u);
        out[i] = static_cast<uint16_t>(u >> 16);
    }
}

}  // extern "C"
