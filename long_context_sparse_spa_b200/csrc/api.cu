// Host side of the C ABI declared in include/spa.h: argument validation, workspace
// layout and kernel launches.  No entry point allocates device memory.
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>
#include <string>
#include <vector>

#include "internal.cuh"

namespace spa {

namespace {
thread_local std::string g_last_cuda_error;
std::atomic<int> g_test_stall{0};
std::mutex g_info_mu;
std::vector<DeviceInfo> g_info;
}  // namespace

int test_stall_bits() { return g_test_stall.load(std::memory_order_relaxed); }

spa_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = std::string(cudaGetErrorName(e)) + ": " + cudaGetErrorString(e);
    return SPA_ERR_CUDA;
}

const DeviceInfo& device_info() {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_info_mu);
    if (int(g_info.size()) <= dev) g_info.resize(dev + 1);
    DeviceInfo& d = g_info[dev];
    if (d.device < 0) {
        cudaDeviceProp prop{};
        if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) {
            d.num_sms = prop.multiProcessorCount;
            d.max_smem_optin = int(prop.sharedMemPerBlockOptin);
            d.cc_major = prop.major;
            d.cc_minor = prop.minor;
        } else {
            d.num_sms = 148;
            d.max_smem_optin = 232448;
        }
        d.device = dev;
    }
    return d;
}

namespace {
std::mutex g_memo_mu;
struct AttrKey {
    int dev;
    const void* func;
    int attr;
    bool operator<(const AttrKey& o) const {
        return std::tie(dev, func, attr) < std::tie(o.dev, o.func, o.attr);
    }
};
struct OccKey {
    int dev;
    const void* func;
    int threads;
    size_t smem;
    bool operator<(const OccKey& o) const {
        return std::tie(dev, func, threads, smem) < std::tie(o.dev, o.func, o.threads, o.smem);
    }
};
std::map<AttrKey, int> g_attr;
std::map<OccKey, int> g_occ;
}  // namespace

cudaError_t set_func_attr(const void* func, cudaFuncAttribute attr, int value) {
    int dev = 0;
    cudaGetDevice(&dev);
    const AttrKey key{dev, func, int(attr)};
    {
        std::lock_guard<std::mutex> lk(g_memo_mu);
        auto it = g_attr.find(key);
        if (it != g_attr.end() && it->second == value) return cudaSuccess;
    }
    const cudaError_t e = cudaFuncSetAttribute(func, attr, value);
    std::lock_guard<std::mutex> lk(g_memo_mu);
    if (e == cudaSuccess) g_attr[key] = value;
    else g_attr.erase(key);
    return e;
}

int occupancy_blocks(const void* func, int threads, size_t smem) {
    int dev = 0;
    cudaGetDevice(&dev);
    const OccKey key{dev, func, threads, smem};
    {
        std::lock_guard<std::mutex> lk(g_memo_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) return it->second;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess) {
        cudaGetLastError();
        return 0;   // not memoised: the query may succeed once the attributes allow this size
    }
    if (n <= 0) return 0;   // not memoised either (an attribute may still be below this size)
    std::lock_guard<std::mutex> lk(g_memo_mu);
    if (g_occ.size() > 4096) g_occ.clear();
    g_occ[key] = n;
    return n;
}

namespace {

inline bool bad_dims(int B, int Hq, int Hkv) { return B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0; }

// scores per unit of a decode: tokens, or blocks for the block score kinds
int decode_units_m(const spa_decode_args* a) {
    const bool block_kind = a->score_kind == SPA_SCORE_TAYLOR_BLOCK || a->score_kind == SPA_SCORE_MINMAX_BLOCK ||
                            a->score_kind == SPA_SCORE_MEAN_BLOCK;
    return block_kind ? a->N / (a->block > 0 ? a->block : 1) : a->N;
}

size_t decode_scores_bytes(const spa_decode_args* a) {
    const int U = a->collapse == SPA_COLLAPSE_GROUP_MEAN ? a->B * a->Hkv : a->B * a->Hq;
    return align_up(size_t(U) * size_t(decode_units_m(a)) * 4, 256);
}

}  // namespace
}  // namespace spa

using namespace spa;

extern "C" {

const char* spa_status_string(int s) {
    switch (s) {
        case SPA_OK: return "SPA_OK";
        case SPA_ERR_INVALID_ARG: return "SPA_ERR_INVALID_ARG";
        case SPA_ERR_UNSUPPORTED_SHAPE: return "SPA_ERR_UNSUPPORTED_SHAPE";
        case SPA_ERR_WORKSPACE_TOO_SMALL: return "SPA_ERR_WORKSPACE_TOO_SMALL";
        case SPA_ERR_CUDA: return "SPA_ERR_CUDA";
        case SPA_ERR_TIMEOUT: return "SPA_ERR_TIMEOUT";
        case SPA_ERR_CAPACITY: return "SPA_ERR_CAPACITY";
        default: return "SPA_ERR_UNKNOWN";
    }
}

const char* spa_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

spa_status spa_test_stall(int bits) {
    if (bits & ~(SPA_TEST_STALL_SELECT_LOAD | SPA_TEST_STALL_PREFILL_MMA)) return SPA_ERR_INVALID_ARG;
    g_test_stall.store(bits, std::memory_order_relaxed);
    return SPA_OK;
}

int spa_abi_version(void) { return 7; }

// shared checks of the block-statistics entries; SPA_OK with *noop set when there is nothing to do
static spa_status check_stats_args(const uint16_t* K, int B, int Hkv, int N, int d, int block, const void* a,
                                   const void* b, bool* noop) {
    *noop = false;
    if (B < 0 || Hkv <= 0 || N < 0 || block <= 0) return SPA_ERR_INVALID_ARG;
    if (B == 0 || N / block == 0) {
        *noop = true;
        return SPA_OK;
    }
    if (!K || !a || !b) return SPA_ERR_INVALID_ARG;
    if ((d != 64 && d != 128) || (block != 32 && block != 64 && block != 128)) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(K) || !aligned16(a) || !aligned16(b)) return SPA_ERR_UNSUPPORTED_SHAPE;
    return SPA_OK;
}

spa_status spa_block_stats(const uint16_t* K, int B, int Hkv, int N, int d, int block, float* mean, float* var,
                           void* stream) {
    bool noop;
    const spa_status s = check_stats_args(K, B, Hkv, N, d, block, mean, var, &noop);
    if (s != SPA_OK || noop) return s;
    return launch_block_stats(K, B, Hkv, N, d, block, mean, var, false, static_cast<cudaStream_t>(stream));
}

spa_status spa_block_stats_bf16(const uint16_t* K, int B, int Hkv, int N, int d, int block, uint16_t* mean,
                                uint16_t* var, void* stream) {
    bool noop;
    const spa_status s = check_stats_args(K, B, Hkv, N, d, block, mean, var, &noop);
    if (s != SPA_OK || noop) return s;
    return launch_block_stats(K, B, Hkv, N, d, block, mean, var, true, static_cast<cudaStream_t>(stream));
}

spa_status spa_block_minmax(const uint16_t* K, int B, int Hkv, int N, int d, int block, float* mn, float* mx,
                            void* stream) {
    bool noop;
    const spa_status s = check_stats_args(K, B, Hkv, N, d, block, mn, mx, &noop);
    if (s != SPA_OK || noop) return s;
    return launch_block_minmax(K, B, Hkv, N, d, block, mn, mx, false, static_cast<cudaStream_t>(stream));
}

spa_status spa_block_minmax_bf16(const uint16_t* K, int B, int Hkv, int N, int d, int block, uint16_t* mn,
                                 uint16_t* mx, void* stream) {
    bool noop;
    const spa_status s = check_stats_args(K, B, Hkv, N, d, block, mn, mx, &noop);
    if (s != SPA_OK || noop) return s;
    return launch_block_minmax(K, B, Hkv, N, d, block, mn, mx, true, static_cast<cudaStream_t>(stream));
}

// block score kinds other than low-rank, with their statistics' requirements
static spa_status check_block_kind(int kind, const void* a, const void* b, float scale) {
    if (!a || (kind != SPA_SCORE_MEAN_BLOCK && !b)) return SPA_ERR_INVALID_ARG;
    if (kind == SPA_SCORE_MINMAX_BLOCK && !(scale > 0.f)) return SPA_ERR_INVALID_ARG;
    if (!aligned16(a) || (b && !aligned16(b))) return SPA_ERR_UNSUPPORTED_SHAPE;
    return SPA_OK;
}

static bool is_block_kind(int kind) {
    return kind == SPA_SCORE_TAYLOR_BLOCK || kind == SPA_SCORE_MINMAX_BLOCK || kind == SPA_SCORE_MEAN_BLOCK;
}

spa_status spa_index_scores(int kind, const void* q, const void* keys, const void* var, int B, int Hq, int Hkv,
                            int M, int dim, int collapse, float scale, float* scores, void* stream) {
    const bool stats_bf16 = (kind & SPA_STATS_BF16) != 0;
    kind &= ~SPA_STATS_BF16;
    if (stats_bf16 && !is_block_kind(kind)) return SPA_ERR_INVALID_ARG;
    if (bad_dims(B, Hq, Hkv) || M < 0) return SPA_ERR_INVALID_ARG;
    if (collapse != SPA_COLLAPSE_NONE && collapse != SPA_COLLAPSE_GROUP_MEAN) return SPA_ERR_INVALID_ARG;
    if (B == 0 || M == 0) return SPA_OK;
    if (!q || !keys || !scores) return SPA_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (G > 16) return SPA_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == SPA_SCORE_LOWRANK) {
        if (dim != 16) return SPA_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(q) || !aligned16(keys)) return SPA_ERR_UNSUPPORTED_SHAPE;
        return launch_lowrank_scores(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(keys), B, Hq, Hkv,
                                     M, collapse, scale, scores, nullptr, false, st);
    }
    if (is_block_kind(kind)) {
        spa_status s = check_block_kind(kind, keys, var, scale);
        if (s != SPA_OK) return s;
        if (dim != 64 && dim != 128) return SPA_ERR_UNSUPPORTED_SHAPE;
        return launch_taylor_scores(static_cast<const uint16_t*>(q), keys, var, B, Hq, Hkv, M, dim, collapse, scale,
                                    scores, st, nullptr, kind, stats_bf16);
    }
    return SPA_ERR_INVALID_ARG;
}

size_t spa_select_workspace_bytes(int U, int M) {
    (void)M;
    return U < 0 ? 0 : kWsHeader + select_scratch_bytes(U);
}

static spa_status select_common(const float* scores, const int32_t* unit_len, int U, int M, int sink, int window,
                                int32_t* idx, int32_t* count, int cap, void* ws, size_t ws_bytes) {
    if (U < 0 || M < 0 || sink < 0 || window < 0 || cap < 0) return SPA_ERR_INVALID_ARG;
    if (U > 65535) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (U == 0) return SPA_OK;
    if (!scores || !idx || !count || !ws) return SPA_ERR_INVALID_ARG;
    if (ws_bytes < spa_select_workspace_bytes(U, M)) return SPA_ERR_WORKSPACE_TOO_SMALL;
    (void)unit_len;
    return SPA_OK;
}

spa_status spa_select_topk(const float* scores, const int32_t* unit_len, int U, int M, int k, int sink, int window,
                           int32_t* idx, int32_t* count, int cap, void* ws, size_t ws_bytes, void* stream) {
    spa_status s = select_common(scores, unit_len, U, M, sink, window, idx, count, cap, ws, ws_bytes);
    if (s != SPA_OK || U == 0) return s;
    if (k < 0) return SPA_ERR_INVALID_ARG;
    SelectParams p{hist0_carve(static_cast<uint8_t*>(ws) + kWsHeader, U), scores, unit_len, U, M, k, 0.f, sink,
                   window, idx, count, cap, nullptr, static_cast<uint32_t*>(ws)};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_hist0(p, false, st);
    if (s != SPA_OK) return s;
    return launch_select(p, false, st);
}

spa_status spa_select_topp(const float* scores, const int32_t* unit_len, int U, int M, float p, int sink,
                           int window, int32_t* idx, int32_t* count, int cap, float* index_mass, void* ws,
                           size_t ws_bytes, void* stream) {
    spa_status s = select_common(scores, unit_len, U, M, sink, window, idx, count, cap, ws, ws_bytes);
    if (s != SPA_OK || U == 0) return s;
    if (!(p > 0.f && p <= 1.f)) return SPA_ERR_INVALID_ARG;
    if (M > (1 << 23)) return SPA_ERR_UNSUPPORTED_SHAPE;
    SelectParams sp{hist0_carve(static_cast<uint8_t*>(ws) + kWsHeader, U), scores, unit_len, U, M, 0, p, sink,
                    window, idx, count, cap, index_mass, static_cast<uint32_t*>(ws)};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_hist0(sp, true, st);
    if (s != SPA_OK) return s;
    return launch_select(sp, true, st);
}

size_t spa_attend_workspace_bytes(int B, int Hq, int Hkv, int d, int collapse) {
    if (bad_dims(B, Hq, Hkv)) return 0;
    const int U = collapse == SPA_COLLAPSE_GROUP_MEAN ? B * Hkv : B * Hq;
    const int nh = collapse == SPA_COLLAPSE_GROUP_MEAN ? Hq / Hkv : 1;
    return kWsHeader + attend_scratch_bytes(U, nh, d);
}

static spa_status attend_params(const uint16_t* q, const uint16_t* K, const uint16_t* V, int B, int Hq, int Hkv,
                                int N, int d, const int32_t* idx, const int32_t* count, int cap, int collapse,
                                int unit_tokens, float sm_scale, uint16_t* out, float* out_f32, float* lse,
                                void* ws, size_t ws_bytes, AttendParams& p) {
    if (bad_dims(B, Hq, Hkv) || N < 0 || cap < 0 || unit_tokens <= 0) return SPA_ERR_INVALID_ARG;
    if (collapse != SPA_COLLAPSE_NONE && collapse != SPA_COLLAPSE_GROUP_MEAN) return SPA_ERR_INVALID_ARG;
    if (!q || !K || !V || !idx || !count || !out || !ws) return SPA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (collapse == SPA_COLLAPSE_GROUP_MEAN && Hq / Hkv > 16) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V)) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (ws_bytes < spa_attend_workspace_bytes(B, Hq, Hkv, d, collapse)) return SPA_ERR_WORKSPACE_TOO_SMALL;
    const int U = collapse == SPA_COLLAPSE_GROUP_MEAN ? B * Hkv : B * Hq;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p = AttendParams{};
    p.q = q; p.K = K; p.V = V;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.d = d;
    p.idx = idx; p.count = count; p.cap = cap; p.collapse = collapse; p.unit_tokens = unit_tokens;
    p.sm_scale = sm_scale; p.out = out; p.out_f32 = out_f32; p.lse = lse;
    p.status = reinterpret_cast<uint32_t*>(w);
    p.unit_ctas = reinterpret_cast<int*>(w + kWsHeader);
    p.partials = reinterpret_cast<float*>(w + kWsHeader + align_up(size_t(U) * 8, 256));
    return SPA_OK;
}

spa_status spa_sparse_attend(const uint16_t* q, const uint16_t* K, const uint16_t* V, int B, int Hq, int Hkv, int N,
                             int d, const int32_t* idx, const int32_t* count, int cap, int collapse,
                             int unit_tokens, float sm_scale, uint16_t* out, float* out_f32, float* lse, void* ws,
                             size_t ws_bytes, void* stream) {
    if (B == 0) return SPA_OK;
    AttendParams p;
    spa_status s = attend_params(q, K, V, B, Hq, Hkv, N, d, idx, count, cap, collapse, unit_tokens, sm_scale, out,
                                 out_f32, lse, ws, ws_bytes, p);
    if (s != SPA_OK) return s;
    return launch_attend(p, static_cast<cudaStream_t>(stream));
}

size_t spa_decode_workspace_bytes(const spa_decode_args* a) {
    if (!a || bad_dims(a->B, a->Hq, a->Hkv)) return 0;
    const int U = a->collapse == SPA_COLLAPSE_GROUP_MEAN ? a->B * a->Hkv : a->B * a->Hq;
    const size_t separate = kWsHeader + decode_scores_bytes(a) + select_scratch_bytes(U) +
                            attend_scratch_bytes(U, a->collapse == SPA_COLLAPSE_GROUP_MEAN ? a->Hq / a->Hkv : 1, a->d);
    if (a->kernel_path == SPA_DECODE_FUSED && a->N >= 0 && fused_decode_supported(a)) {
        const size_t fused = kWsHeader + fused_scratch_bytes(a);
        return fused > separate ? fused : separate;
    }
    return separate;
}

static spa_status decode_impl(const spa_decode_args* a, void* ws, size_t ws_bytes, void* stream,
                              void* const* events);

int spa_decode_path_taken(const spa_decode_args* a) {
    if (!a) return -1;
    return a->kernel_path == SPA_DECODE_FUSED && !bad_dims(a->B, a->Hq, a->Hkv) && fused_decode_supported(a)
               ? SPA_DECODE_FUSED
               : SPA_DECODE_SEPARATE;
}

spa_status spa_decode(const spa_decode_args* a, void* ws, size_t ws_bytes, void* stream) {
    return decode_impl(a, ws, ws_bytes, stream, nullptr);
}

spa_status spa_decode_timed(const spa_decode_args* a, void* ws, size_t ws_bytes, void* stream,
                            void* const* events) {
    if (!events) return SPA_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i)
        if (!events[i]) return SPA_ERR_INVALID_ARG;
    return decode_impl(a, ws, ws_bytes, stream, events);
}

static spa_status decode_impl(const spa_decode_args* a, void* ws, size_t ws_bytes, void* stream,
                              void* const* events) {
    if (!a || !ws) return SPA_ERR_INVALID_ARG;
    if (bad_dims(a->B, a->Hq, a->Hkv) || a->N < 0) return SPA_ERR_INVALID_ARG;
    if (a->B == 0) return SPA_OK;
    if (ws_bytes < spa_decode_workspace_bytes(a)) return SPA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool group = a->collapse == SPA_COLLAPSE_GROUP_MEAN;
    if (!group && a->collapse != SPA_COLLAPSE_NONE) return SPA_ERR_INVALID_ARG;
    const int U = group ? a->B * a->Hkv : a->B * a->Hq;
    const bool taylor = is_block_kind(a->score_kind);   // block scores (Taylor, min-max or mean)
    if (!taylor && a->score_kind != SPA_SCORE_LOWRANK) return SPA_ERR_INVALID_ARG;
    const int block = taylor ? a->block : 1;
    if (block <= 0 || (!taylor && a->block > 1)) return SPA_ERR_INVALID_ARG;
    const int M = a->N / block;
    if (U > 65535) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (a->select_kind == SPA_SELECT_TOPP) {
        if (!(a->topp > 0.f && a->topp <= 1.f)) return SPA_ERR_INVALID_ARG;
        if (M > (1 << 23)) return SPA_ERR_UNSUPPORTED_SHAPE;
    } else if (a->select_kind == SPA_SELECT_TOPK) {
        if (a->topk < 0) return SPA_ERR_INVALID_ARG;
    } else {
        return SPA_ERR_INVALID_ARG;
    }
    if (a->sink < 0 || a->window < 0 || a->cap < 0) return SPA_ERR_INVALID_ARG;
    if (taylor) {
        const spa_status sb = check_block_kind(a->score_kind, a->bmean, a->bvar, a->score_scale);
        if (sb != SPA_OK) return sb;
        if (a->d != 64 && a->d != 128) return SPA_ERR_UNSUPPORTED_SHAPE;
    } else {
        if (!a->q_idx || !a->Kidx) return SPA_ERR_INVALID_ARG;
        if (a->r != 16) return SPA_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(a->q_idx) || !aligned16(a->Kidx)) return SPA_ERR_UNSUPPORTED_SHAPE;
    }

    if (a->kernel_path != SPA_DECODE_AUTO && a->kernel_path != SPA_DECODE_SEPARATE && a->kernel_path != SPA_DECODE_FUSED)
        return SPA_ERR_INVALID_ARG;

    uint8_t* w = static_cast<uint8_t*>(ws);
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    if (a->kernel_path == SPA_DECODE_FUSED && fused_decode_supported(a)) {
        // the persistent dataflow kernel; the pointer and alignment checks are the attention's
        AttendParams chk;
        spa_status s = attend_params(a->q, a->K, a->V, a->B, a->Hq, a->Hkv, a->N, a->d, a->idx, a->count, a->cap,
                                     a->collapse, 1, a->sm_scale, a->out, a->out_f32, a->lse, ws, size_t(-1), chk);
        if (s != SPA_OK) return s;
        return launch_fused_decode(a, w + kWsHeader, status, st, events);
    }
    float* scores = reinterpret_cast<float*>(w + kWsHeader);
    const Hist0 hist = hist0_carve(w + kWsHeader + decode_scores_bytes(a), U);
    uint8_t* attend_ws = w + kWsHeader + decode_scores_bytes(a) + select_scratch_bytes(U);
    const bool topp = a->select_kind == SPA_SELECT_TOPP;
    // the level-0 selection histogram is built inside the scoring kernel when it produces
    // one score row per kv head (low-rank, GROUP_MEAN); otherwise by a histogram kernel
    const bool fused_hist = !taylor && group;

    // attention parameters first: they validate q/K/V/idx/out and carve the workspace
    AttendParams ap;
    spa_status s = attend_params(a->q, a->K, a->V, a->B, a->Hq, a->Hkv, a->N, a->d, a->idx, a->count, a->cap,
                                 a->collapse, block, a->sm_scale, a->out, a->out_f32, a->lse, ws,
                                 size_t(-1), ap);
    if (s != SPA_OK) return s;
    ap.unit_ctas = reinterpret_cast<int*>(attend_ws);
    ap.partials = reinterpret_cast<float*>(attend_ws + align_up(size_t(U) * 8, 256));
    if (a->rla_state) {
        if (!a->rla_z || !a->rla_gamma || !(a->rla_eps >= 0.f)) return SPA_ERR_INVALID_ARG;
        ap.rla_S = a->rla_state;
        ap.rla_z = a->rla_z;
        ap.rla_gamma = a->rla_gamma;
        ap.rla_eps = a->rla_eps;
    }

    auto mark = [&](int i) -> spa_status {
        if (events) SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st));
        return SPA_OK;
    };

    // 1. scores
    if ((s = mark(0)) != SPA_OK) return s;
    if (taylor) {
        s = launch_taylor_scores(a->q, a->bmean, a->bvar, a->B, a->Hq, a->Hkv, M, a->d, a->collapse,
                                 a->score_scale, scores, st, a->local_units, a->score_kind, a->stats_bf16 != 0);
    } else {
        s = launch_lowrank_scores(a->q_idx, a->Kidx, a->B, a->Hq, a->Hkv, M, a->collapse, a->score_scale, scores,
                                  fused_hist ? &hist : nullptr, topp, st, a->local_units);
    }
    if (s != SPA_OK) return s;

    // 2. selection
    SelectParams sp{hist, scores, nullptr, U, M, a->topk, a->topp, a->sink, a->window, a->idx, a->count, a->cap,
                    a->index_mass, status, a->local_units};
    if (!fused_hist && (s = launch_hist0(sp, topp, st)) != SPA_OK) return s;
    if ((s = mark(1)) != SPA_OK) return s;
    s = launch_select(sp, topp, st);
    if (s != SPA_OK) return s;
    if ((s = mark(2)) != SPA_OK) return s;

    // 3. attention on the gathered rows
    s = launch_attend(ap, st);
    if (s != SPA_OK) return s;
    return mark(3);
}

size_t spa_prefill_workspace_bytes(const spa_prefill_args* a) {
    if (!a || a->bq <= 0 || a->Hkv <= 0 || a->T < 0 || a->N < 0) return 0;
    const int U = (a->T / a->bq) * a->Hkv;
    return kWsHeader + prefill_scratch_bytes(U, a->N);
}

spa_status spa_rla_state(const uint16_t* K, const uint16_t* V, int B, int Hkv, int N, int d, int n0, int n1,
                         float* S, float* z, void* stream) {
    if (B < 0 || Hkv <= 0 || N < 0 || n0 < 0 || n1 < n0 || n1 > N) return SPA_ERR_INVALID_ARG;
    if (B == 0 || n0 == n1) return SPA_OK;
    if (!K || !V || !S || !z) return SPA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(K) || !aligned16(V) || !aligned16(S) || !aligned16(z)) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (size_t(B) * Hkv > 65535) return SPA_ERR_UNSUPPORTED_SHAPE;
    return launch_rla_state(K, V, B * Hkv, N, d, n0, n1, S, z, static_cast<cudaStream_t>(stream));
}

static spa_status prefill_impl(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream,
                               void* const* events) {
    if (!a || !ws) return SPA_ERR_INVALID_ARG;
    if (a->T < 0 || a->N <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->bq <= 0 ||
        a->q_start < 0 || a->topk < 0 || a->sink < 0 || a->cap < 0 || !(a->sm_scale > 0.f))
        return SPA_ERR_INVALID_ARG;
    if (a->T == 0) return SPA_OK;
    if (!a->Q || !a->q_idx || !a->K || !a->V || !a->Kidx || !a->idx || !a->count || !a->out)
        return SPA_ERR_INVALID_ARG;
    const int G = a->Hq / a->Hkv;
    if (a->d != 128 || a->r != 16 || a->bq != 64 || G % 2 != 0 || G > 16 || a->T % a->bq != 0 ||
        a->T / a->bq > 128 || a->q_start + a->T > a->N)
        return SPA_ERR_UNSUPPORTED_SHAPE;
    if (a->cap < (a->topk + a->sink < a->N ? a->topk + a->sink : a->N)) return SPA_ERR_INVALID_ARG;
    if (!aligned16(a->Q) || !aligned16(a->q_idx) || !aligned16(a->K) || !aligned16(a->V) || !aligned16(a->Kidx) ||
        !aligned16(a->out) || (a->out_f32 && !aligned16(a->out_f32)))
        return SPA_ERR_UNSUPPORTED_SHAPE;
    if (ws_bytes < spa_prefill_workspace_bytes(a)) return SPA_ERR_WORKSPACE_TOO_SMALL;
    return launch_prefill(a, ws, static_cast<cudaStream_t>(stream), events);
}

spa_status spa_prefill_shared(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream) {
    return prefill_impl(a, ws, ws_bytes, stream, nullptr);
}

spa_status spa_prefill_shared_timed(const spa_prefill_args* a, void* ws, size_t ws_bytes, void* stream,
                                    void* const* events) {
    if (!events || !events[0] || !events[1]) return SPA_ERR_INVALID_ARG;
    return prefill_impl(a, ws, ws_bytes, stream, events);
}

spa_status spa_read_device_status(void* ws, void* stream, uint32_t* bits, int reset) {
    if (!ws || !bits) return SPA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SPA_CUDA_TRY(cudaMemcpyAsync(bits, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, st));
    SPA_CUDA_TRY(cudaStreamSynchronize(st));
    if (reset) {
        SPA_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(uint32_t), st));
        SPA_CUDA_TRY(cudaStreamSynchronize(st));
    }
    return SPA_OK;
}

}  // extern "C"
