// Per-query sparse prefill ("Oracle-Guided Sparse Prefill" 2.1 with b_sel = 1: every query
// has its own support).
//
// For query t of the chunk (absolute position q_start + t) and kv head g, unit u = t*Hkv + g:
//   index query = mean of q_idx over the G heads of g (the head-collapsed indexer, 2.2);
//   support     = exact top-k of score_scale * index_query . Kidx[g][n] over n < q_start + t,
//                 united with the sink [0, sink);
//   out[t][h]   = softmax(sm_scale * q K^T) V over the support and the query's own position.
//
// With one query per support there is no dense contraction to put on tcgen05: every unit is a
// decode step over its own rows.  The path is the decode's: the low-rank scorer with one key
// set shared by all queries of the chunk, the exact top-k with a candidate length per unit,
// and the split-KV gather attention (also on shared K/V) after the own position is appended.
#include "internal.cuh"

namespace spa {
namespace {

// candidate length of unit u: the keys before its query
__global__ void pq_lengths_kernel(int32_t* __restrict__ unit_len, int U, int Hkv, int q_start) {
    pdl_enter();
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u < U) unit_len[u] = q_start + u / Hkv;
}

// the query's own position after its support: the rows the attention reads
__global__ void pq_own_row_kernel(int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                                  int32_t* __restrict__ count_att, int U, int Hkv, int cap, int q_start) {
    pdl_enter();
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= U) return;
    int c = count[u];
    c = c < 0 ? 0 : (c > cap - 1 ? cap - 1 : c);
    idx[size_t(u) * cap + c] = q_start + u / Hkv;
    count_att[u] = c + 1;
}

struct PqLayout {
    size_t unit_len, count_att, scores, hist, attend, total;
};

PqLayout pq_layout(int T, int Hq, int Hkv, int N, int d) {
    const int U = T * Hkv;
    PqLayout l{};
    size_t o = 0;
    l.unit_len = o; o += align_up(size_t(U) * 4, 256);
    l.count_att = o; o += align_up(size_t(U) * 4, 256);
    l.scores = o; o += align_up(size_t(U) * N * 4, 256);
    l.hist = o; o += hist0_bytes(U);
    l.attend = o; o += attend_scratch_bytes(U, Hq / Hkv, d);
    l.total = o;
    return l;
}

}  // namespace
}  // namespace spa

using namespace spa;

extern "C" size_t spa_prefill_per_query_workspace_bytes(const spa_prefill_args* a) {
    if (!a || a->T < 0 || a->Hkv <= 0 || a->Hq <= 0 || a->Hq % a->Hkv != 0 || a->N < 0) return 0;
    return kWsHeader + pq_layout(a->T, a->Hq, a->Hkv, a->N, a->d).total;
}

extern "C" spa_status spa_prefill_per_query(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream) {
    if (!a || !ws) return SPA_ERR_INVALID_ARG;
    if (a->T < 0 || a->N <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->q_start < 0 ||
        a->topk < 0 || a->sink < 0 || a->cap < 0)
        return SPA_ERR_INVALID_ARG;
    if (a->bq != 1) return SPA_ERR_INVALID_ARG;
    if (a->T == 0) return SPA_OK;
    if (!a->Q || !a->q_idx || !a->K || !a->V || !a->Kidx || !a->idx || !a->count || !a->out)
        return SPA_ERR_INVALID_ARG;
    const int G = a->Hq / a->Hkv;
    if ((a->d != 64 && a->d != 128) || a->r != 16 || G > 16 || a->q_start + a->T > a->N)
        return SPA_ERR_UNSUPPORTED_SHAPE;
    const long long U = (long long)a->T * a->Hkv;
    if (U > 8192) return SPA_ERR_UNSUPPORTED_SHAPE;   // the attention's unit table
    // room for the support and the own position
    if (a->cap < (a->topk + a->sink < a->N ? a->topk + a->sink : a->N) + 1) return SPA_ERR_INVALID_ARG;
    if (!aligned16(a->Q) || !aligned16(a->q_idx) || !aligned16(a->K) || !aligned16(a->V) || !aligned16(a->Kidx) ||
        !aligned16(a->out))
        return SPA_ERR_UNSUPPORTED_SHAPE;
    if (ws_bytes < spa_prefill_per_query_workspace_bytes(a)) return SPA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const PqLayout l = pq_layout(a->T, a->Hq, a->Hkv, a->N, a->d);
    uint8_t* w = static_cast<uint8_t*>(ws);
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    uint8_t* b = w + kWsHeader;
    int32_t* unit_len = reinterpret_cast<int32_t*>(b + l.unit_len);
    int32_t* count_att = reinterpret_cast<int32_t*>(b + l.count_att);
    float* scores = reinterpret_cast<float*>(b + l.scores);
    const Hist0 hist = hist0_carve(b + l.hist, int(U));
    uint8_t* attend_ws = b + l.attend;

    const int nU = int(U);
    SPA_CUDA_TRY(launch_pdl(pq_lengths_kernel, dim3((nU + 255) / 256), dim3(256), 0, st, unit_len, nU, a->Hkv,
                            a->q_start));
    // index scores of every key for every query (the keys past a query are never ranked)
    spa_status s = launch_lowrank_scores(a->q_idx, a->Kidx, a->T, a->Hq, a->Hkv, a->N, SPA_COLLAPSE_GROUP_MEAN,
                                         a->score_scale, scores, nullptr, false, st, nullptr, true);
    if (s != SPA_OK) return s;
    // exact top-k over each query's candidates, united with the sink
    SelectParams sp{hist, scores, unit_len, nU, a->N, a->topk, 0.f, a->sink, 0, a->idx, a->count, a->cap,
                    nullptr, status};
    if ((s = launch_hist0(sp, false, st)) != SPA_OK) return s;
    if ((s = launch_select(sp, false, st)) != SPA_OK) return s;
    SPA_CUDA_TRY(launch_pdl(pq_own_row_kernel, dim3((nU + 255) / 256), dim3(256), 0, st, a->idx,
                            static_cast<const int32_t*>(a->count), count_att, nU, a->Hkv, a->cap, a->q_start));
    // exact attention over the support and the own position, K and V shared by all queries
    AttendParams ap{};
    ap.q = a->Q;
    ap.K = a->K;
    ap.V = a->V;
    ap.B = a->T;
    ap.Hq = a->Hq;
    ap.Hkv = a->Hkv;
    ap.N = a->N;
    ap.d = a->d;
    ap.idx = a->idx;
    ap.count = count_att;
    ap.cap = a->cap;
    ap.collapse = SPA_COLLAPSE_GROUP_MEAN;
    ap.unit_tokens = 1;
    ap.sm_scale = a->sm_scale;
    ap.out = a->out;
    ap.out_f32 = a->out_f32;
    ap.lse = nullptr;
    ap.status = status;
    ap.kv_shared = 1;
    ap.unit_ctas = reinterpret_cast<int*>(attend_ws);
    ap.partials = reinterpret_cast<float*>(attend_ws + align_up(size_t(nU) * 8, 256));
    return launch_attend(ap, st);
}
