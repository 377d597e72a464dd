// Permuted block-sparse prefill: "Sparser Block-Sparse Attention via Token Permutation"
// (PBS-Attn), sections 1-4, for a causal prefill of T tokens.
//
//   1. importance (section 3): for every kv head g and key n, the mean over the last query
//      block's b queries and the G heads of g of their causal softmax probability of n
//      (keys after a query count 0 for it): two passes over the keys -- per-row max and sum,
//      then the probabilities summed per key in a fixed order;
//   2. permutation (sections 2-3): inside each segment of S keys, keys sorted by descending
//      importance, equal importance by ascending position (a bitonic sort of 64-bit keys);
//   3. block selection (section 4): each query block j (b queries, segment seg0 = j*b/S*S) and
//      kv head g scores the blocks of b consecutive permuted keys in the segments before its
//      own with sm_scale * qbar . kbar (mean pooling of the block's b x G queries and of the
//      block's keys); the top-k blocks (score desc, block asc) are kept, no block is forced;
//   4. attention: the selected keys (original positions, ascending), the own segment's keys
//      before the block, [seg0, t0), and the block's causal diagonal -- the row set of the
//      selection-block-shared prefill -- on the tcgen05 attention kernel.  Queries are not
//      permuted, so no inverse permutation of the output is needed.
//
// Steps 1-3 are CUDA-core kernels (the importance pass is a b*G x T x d contraction done once
// per prefill); step 3's top-k is the library's exact selection with a per-unit candidate
// length.
#include "internal.cuh"

namespace spa {
namespace {

constexpr int kPbThreads = 256;
constexpr int kPbKeys = 128;       // keys per CTA in the importance passes
constexpr int kPbRows = 256;       // query rows held in shared memory at once
constexpr int kPbD = 128;
constexpr float kPbLog2e = 1.4426950408889634f;

struct PbsParams {
    const uint16_t* Q;   // [T, Hq, d]
    const uint16_t* K;   // [Hkv, T, d]
    int T, Hq, Hkv, G, b, S, R, ntiles, nblk;
    float sm_scale;
    float* rm;           // [Hkv][ntiles][R] per-tile row max (log2 units)
    float* rl;           // [Hkv][ntiles][R] per-tile row sum
    float* M;            // [Hkv][R]
    float* L;            // [Hkv][R]
    float* imp;          // [Hkv][T]
    int32_t* perm;       // [Hkv][T]
    float* kbar;         // [Hkv][nblk][d]
    float* qbar;         // [nblk][Hkv][d]
    float* scores;       // [U][nblk]
    int32_t* unit_len;   // [U]
    const int32_t* bidx; // [U][topk] selected blocks
    const int32_t* bcount;
    int topk;
    int32_t* idx;        // [U][cap] support (original positions, ascending)
    int32_t* count;
    int cap;
    int32_t* aidx;       // [U][acap] rows of the attention: support, then [seg0, t0)
    int32_t* acount;
    int acap;
};

__device__ __forceinline__ float bf(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

// Stage the key tile [n0, n0 + kPbKeys) of kv head g (fp32, zero past T) and rows [rc, rc +
// kPbRows) of the last query block (transposed: qT[c][r], zero past R) in shared memory.
__device__ void pb_stage(const PbsParams& p, int g, int n0, int rc, float* ks, float* qT) {
    for (int i = threadIdx.x; i < kPbKeys * kPbD; i += kPbThreads) {
        const int k = i / kPbD, c = i - k * kPbD, n = n0 + k;
        ks[i] = n < p.T ? bf(p.K[(size_t(g) * p.T + n) * kPbD + c]) : 0.f;
    }
    for (int i = threadIdx.x; i < kPbRows * kPbD; i += kPbThreads) {
        const int rr = i % kPbRows, c = i / kPbRows, r = rc + rr;
        float v = 0.f;
        if (r < p.R) {
            const int qi = p.T - p.b + r / p.G, h = r % p.G;
            v = bf(p.Q[(size_t(qi) * p.Hq + g * p.G + h) * kPbD + c]);
        }
        qT[c * kPbRows + rr] = v;
    }
}

// scaled logit (log2 units) of staged row rr and staged key k, channels in ascending order
__device__ __forceinline__ float pb_logit(const float* qT, const float* ks, int rr, int k, float sl2) {
    float dot = 0.f;
    const float4* k4 = reinterpret_cast<const float4*>(ks + k * kPbD);
#pragma unroll 8
    for (int c4 = 0; c4 < kPbD / 4; ++c4) {
        const float4 kv = k4[c4];
        dot = fmaf(qT[(4 * c4 + 0) * kPbRows + rr], kv.x, dot);
        dot = fmaf(qT[(4 * c4 + 1) * kPbRows + rr], kv.y, dot);
        dot = fmaf(qT[(4 * c4 + 2) * kPbRows + rr], kv.z, dot);
        dot = fmaf(qT[(4 * c4 + 3) * kPbRows + rr], kv.w, dot);
    }
    return dot * sl2;
}

// pass 1: per key tile, every row's max and sum of exp2 over the tile's keys it may see
__global__ void __launch_bounds__(kPbThreads) pbs_rowstats_kernel(PbsParams p) {
    pdl_enter();
    extern __shared__ __align__(16) float pbs_smem[];
    float* ks = pbs_smem;
    float* qT = pbs_smem + kPbKeys * kPbD;
    const int g = blockIdx.y, kt = blockIdx.x;
    const int n0 = kt * kPbKeys, n1 = min(p.T, n0 + kPbKeys);
    const float sl2 = p.sm_scale * kPbLog2e;
    for (int rc = 0; rc < p.R; rc += kPbRows) {
        __syncthreads();
        pb_stage(p, g, n0, rc, ks, qT);
        __syncthreads();
        const int r = rc + threadIdx.x;
        if (r >= p.R) continue;
        const int t_row = p.T - p.b + r / p.G;
        const int kend = min(n1, t_row + 1);
        float m = -INFINITY, l = 0.f;
        for (int n = n0; n < kend; ++n) {
            const float x = pb_logit(qT, ks, threadIdx.x, n - n0, sl2);
            const float mn = fmaxf(m, x);
            l = l * exp2f(m - mn) + exp2f(x - mn);
            m = mn;
        }
        p.rm[(size_t(g) * p.ntiles + kt) * p.R + r] = m;
        p.rl[(size_t(g) * p.ntiles + kt) * p.R + r] = l;
    }
}

// every row's max and sum over all tiles (tile order)
__global__ void __launch_bounds__(kPbThreads) pbs_rowcombine_kernel(PbsParams p) {
    pdl_enter();
    const int g = blockIdx.y;
    const int r = blockIdx.x * kPbThreads + threadIdx.x;
    if (r >= p.R) return;
    float M = -INFINITY;
    for (int t = 0; t < p.ntiles; ++t) M = fmaxf(M, p.rm[(size_t(g) * p.ntiles + t) * p.R + r]);
    float L = 0.f;
    for (int t = 0; t < p.ntiles; ++t) {
        const float m = p.rm[(size_t(g) * p.ntiles + t) * p.R + r];
        if (m != -INFINITY) L += p.rl[(size_t(g) * p.ntiles + t) * p.R + r] * exp2f(m - M);
    }
    p.M[size_t(g) * p.R + r] = M;
    p.L[size_t(g) * p.R + r] = L;
}

// pass 2: importance of the tile's keys: sum over rows of exp2(x - M_r) / L_r, divided by R;
// rows are summed within a warp in lane order, then over warps and row chunks in order
__global__ void __launch_bounds__(kPbThreads) pbs_importance_kernel(PbsParams p) {
    pdl_enter();
    extern __shared__ __align__(16) float pbs_smem[];
    float* ks = pbs_smem;
    float* qT = pbs_smem + kPbKeys * kPbD;
    float* part = qT + kPbD * kPbRows;   // [warps][kPbKeys]
    const int g = blockIdx.y, kt = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n0 = kt * kPbKeys, n1 = min(p.T, n0 + kPbKeys);
    const float sl2 = p.sm_scale * kPbLog2e;
    float acc = 0.f;   // thread k < kPbKeys: the running sum of key n0 + k
    for (int rc = 0; rc < p.R; rc += kPbRows) {
        __syncthreads();
        pb_stage(p, g, n0, rc, ks, qT);
        __syncthreads();
        const int r = rc + threadIdx.x;
        const bool live = r < p.R;
        const int t_row = live ? p.T - p.b + r / p.G : -1;
        const float Mr = live ? p.M[size_t(g) * p.R + r] : 0.f;
        const float inv_l = live ? 1.f / p.L[size_t(g) * p.R + r] : 0.f;
        for (int k = 0; k < n1 - n0; ++k) {
            const int n = n0 + k;
            float pr = 0.f;
            if (live && n <= t_row) pr = exp2f(pb_logit(qT, ks, threadIdx.x, k, sl2) - Mr) * inv_l;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) pr += __shfl_xor_sync(0xffffffffu, pr, off);
            if (lane == 0) part[warp * kPbKeys + k] = pr;
        }
        __syncthreads();
        if (threadIdx.x < kPbKeys) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < kPbThreads / 32; ++w) s += part[w * kPbKeys + threadIdx.x];
            acc += s;
        }
    }
    if (threadIdx.x < n1 - n0) p.imp[size_t(g) * p.T + n0 + threadIdx.x] = acc / float(p.R);
}

// sort each segment by (importance desc, position asc): bitonic sort of 64-bit keys
__global__ void __launch_bounds__(1024) pbs_sort_kernel(PbsParams p) {
    pdl_enter();
    extern __shared__ __align__(16) unsigned long long sk[];
    const int g = blockIdx.y, s0 = blockIdx.x * p.S;
    const int len = min(p.S, p.T - s0);
    int P = 1;
    while (P < len) P <<= 1;
    for (int i = threadIdx.x; i < P; i += blockDim.x) {
        unsigned long long key = ~0ull;
        if (i < len) {
            const uint32_t ik = score_key(p.imp[size_t(g) * p.T + s0 + i]);
            key = (static_cast<unsigned long long>(~ik) << 32) | uint32_t(s0 + i);
        }
        sk[i] = key;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const bool up = (i & k) == 0;
                    const unsigned long long a = sk[i], c = sk[ixj];
                    if ((a > c) == up) {
                        sk[i] = c;
                        sk[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < len; i += blockDim.x) p.perm[size_t(g) * p.T + s0 + i] = int32_t(sk[i] & 0xffffffffu);
}

// z = 0: kbar of permuted key block blockIdx.x; z = 1: qbar of query block blockIdx.x (mean over
// its b queries and G heads, in (query, head) order); one thread per channel
__global__ void __launch_bounds__(kPbD) pbs_means_kernel(PbsParams p) {
    pdl_enter();
    const int blk = blockIdx.x, g = blockIdx.y, c = threadIdx.x;
    float s = 0.f;
    if (blockIdx.z == 0) {
        const int32_t* pm = p.perm + size_t(g) * p.T + size_t(blk) * p.b;
        for (int i = 0; i < p.b; ++i) s += bf(p.K[(size_t(g) * p.T + pm[i]) * kPbD + c]);
        p.kbar[(size_t(g) * p.nblk + blk) * kPbD + c] = s / float(p.b);
    } else {
        for (int i = 0; i < p.b; ++i)
            for (int h = 0; h < p.G; ++h) s += bf(p.Q[(size_t(blk * p.b + i) * p.Hq + g * p.G + h) * kPbD + c]);
        p.qbar[(size_t(blk) * p.Hkv + g) * kPbD + c] = s / float(p.b * p.G);
    }
}

// block scores of unit u = j * Hkv + g over the permuted blocks before its own segment
__global__ void __launch_bounds__(kPbThreads) pbs_scores_kernel(PbsParams p) {
    pdl_enter();
    const int u = blockIdx.x, j = u / p.Hkv, g = u - j * p.Hkv;
    const int seg0 = (j * p.b) / p.S * p.S;
    const int nc = seg0 / p.b;
    __shared__ float qb[kPbD];
    if (threadIdx.x < kPbD) qb[threadIdx.x] = p.qbar[(size_t(j) * p.Hkv + g) * kPbD + threadIdx.x];
    if (threadIdx.x == 0) p.unit_len[u] = nc;
    __syncthreads();
    for (int c = threadIdx.x; c < nc; c += kPbThreads) {
        const float4* kb = reinterpret_cast<const float4*>(p.kbar + (size_t(g) * p.nblk + c) * kPbD);
        float dot = 0.f;
#pragma unroll 8
        for (int d4 = 0; d4 < kPbD / 4; ++d4) {
            const float4 v = kb[d4];
            dot = fmaf(qb[4 * d4 + 0], v.x, dot);
            dot = fmaf(qb[4 * d4 + 1], v.y, dot);
            dot = fmaf(qb[4 * d4 + 2], v.z, dot);
            dot = fmaf(qb[4 * d4 + 3], v.w, dot);
        }
        p.scores[size_t(u) * p.nblk + c] = p.sm_scale * dot;
    }
}

// selected blocks -> their keys' original positions, ascending (support); the attention's
// rows are the support followed by the own segment's keys before the block, [seg0, t0)
__global__ void __launch_bounds__(kPbThreads) pbs_expand_kernel(PbsParams p) {
    pdl_enter();
    extern __shared__ __align__(16) uint32_t pos[];
    const int u = blockIdx.x, j = u / p.Hkv, g = u - j * p.Hkv;
    const int t0 = j * p.b, seg0 = t0 / p.S * p.S;
    int nb = p.bcount[u];
    nb = nb < 0 ? 0 : (nb > p.topk ? p.topk : nb);
    const int n = nb * p.b;
    int P = 1;
    while (P < n) P <<= 1;
    for (int i = threadIdx.x; i < P; i += kPbThreads) {
        uint32_t v = 0xffffffffu;
        if (i < n) {
            const int blk = p.bidx[size_t(u) * p.topk + i / p.b];
            v = uint32_t(p.perm[size_t(g) * p.T + size_t(blk) * p.b + (i % p.b)]);
        }
        pos[i] = v;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int i = threadIdx.x; i < P; i += kPbThreads) {
                const int ixj = i ^ jj;
                if (ixj > i) {
                    const bool up = (i & k) == 0;
                    const uint32_t a = pos[i], c = pos[ixj];
                    if ((a > c) == up) {
                        pos[i] = c;
                        pos[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < n; i += kPbThreads) {
        p.idx[size_t(u) * p.cap + i] = int32_t(pos[i]);
        p.aidx[size_t(u) * p.acap + i] = int32_t(pos[i]);
    }
    for (int i = threadIdx.x; i < t0 - seg0; i += kPbThreads) p.aidx[size_t(u) * p.acap + n + i] = seg0 + i;
    if (threadIdx.x == 0) {
        p.count[u] = n;
        p.acount[u] = n + (t0 - seg0);
    }
}

struct PbsLayout {
    size_t rm, rl, M, L, imp, perm, kbar, qbar, scores, unit_len, hist, bidx, bcount, aidx, acount, total;
};

PbsLayout pbs_layout(const spa_pbs_args* a) {
    const int G = a->Hq / a->Hkv, R = a->b * G, ntiles = (a->T + kPbKeys - 1) / kPbKeys, nblk = a->T / a->b;
    const int U = nblk * a->Hkv;
    const int topk = a->topk > 0 ? a->topk : 1;
    PbsLayout l{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += align_up(bytes, 256);
        return at;
    };
    l.rm = take(size_t(a->Hkv) * ntiles * R * 4);
    l.rl = take(size_t(a->Hkv) * ntiles * R * 4);
    l.M = take(size_t(a->Hkv) * R * 4);
    l.L = take(size_t(a->Hkv) * R * 4);
    l.imp = take(size_t(a->Hkv) * a->T * 4);
    l.perm = take(size_t(a->Hkv) * a->T * 4);
    l.kbar = take(size_t(a->Hkv) * nblk * kPbD * 4);
    l.qbar = take(size_t(nblk) * a->Hkv * kPbD * 4);
    l.scores = take(size_t(U) * nblk * 4);
    l.unit_len = take(size_t(U) * 4);
    l.hist = o;
    o += hist0_bytes(U);
    l.bidx = take(size_t(U) * topk * 4);
    l.bcount = take(size_t(U) * 4);
    l.aidx = take(size_t(U) * (size_t(topk) * a->b + a->S) * 4);
    l.acount = take(size_t(U) * 4);
    l.total = o;
    return l;
}

bool pbs_shape_ok(const spa_pbs_args* a) {
    const int G = a->Hq / a->Hkv;
    return a->d == kPbD && a->b == 64 && G % 2 == 0 && G <= 8 && a->T % a->b == 0 && a->S % a->b == 0 &&
           a->S <= 8192 && size_t(a->topk) * a->b <= 8192;
}

}  // namespace
}  // namespace spa

using namespace spa;

extern "C" size_t spa_pbs_workspace_bytes(const spa_pbs_args* a) {
    if (!a || a->T <= 0 || a->Hkv <= 0 || a->Hq <= 0 || a->Hq % a->Hkv != 0 || a->b <= 0 || a->S <= 0 ||
        a->topk < 0)
        return 0;
    return kWsHeader + pbs_layout(a).total;
}

static spa_status pbs_impl(const spa_pbs_args* a, void* ws, size_t ws_bytes, void* stream, void* const* events) {
    if (!a || !ws) return SPA_ERR_INVALID_ARG;
    if (a->T <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->b <= 0 || a->S <= 0 || a->topk < 0 ||
        a->cap < 0 || !(a->sm_scale > 0.f))
        return SPA_ERR_INVALID_ARG;
    if (!a->Q || !a->K || !a->V || !a->perm || !a->idx || !a->count || !a->out) return SPA_ERR_INVALID_ARG;
    if (!pbs_shape_ok(a)) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (a->cap < a->topk * a->b) return SPA_ERR_INVALID_ARG;
    if (!aligned16(a->Q) || !aligned16(a->K) || !aligned16(a->V) || !aligned16(a->out) ||
        (a->out_f32 && !aligned16(a->out_f32)))
        return SPA_ERR_UNSUPPORTED_SHAPE;
    if (ws_bytes < spa_pbs_workspace_bytes(a)) return SPA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const PbsLayout l = pbs_layout(a);
    uint8_t* w = static_cast<uint8_t*>(ws);
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    uint8_t* b = w + kWsHeader;
    const int G = a->Hq / a->Hkv;
    const int nblk = a->T / a->b;
    const int U = nblk * a->Hkv;
    const int topk = a->topk > 0 ? a->topk : 1;
    PbsParams p{};
    p.Q = a->Q;
    p.K = a->K;
    p.T = a->T;
    p.Hq = a->Hq;
    p.Hkv = a->Hkv;
    p.G = G;
    p.b = a->b;
    p.S = a->S;
    p.R = a->b * G;
    p.ntiles = (a->T + kPbKeys - 1) / kPbKeys;
    p.nblk = nblk;
    p.sm_scale = a->sm_scale;
    p.rm = reinterpret_cast<float*>(b + l.rm);
    p.rl = reinterpret_cast<float*>(b + l.rl);
    p.M = reinterpret_cast<float*>(b + l.M);
    p.L = reinterpret_cast<float*>(b + l.L);
    p.imp = a->importance ? a->importance : reinterpret_cast<float*>(b + l.imp);
    p.perm = a->perm;
    p.kbar = reinterpret_cast<float*>(b + l.kbar);
    p.qbar = reinterpret_cast<float*>(b + l.qbar);
    p.scores = reinterpret_cast<float*>(b + l.scores);
    p.unit_len = reinterpret_cast<int32_t*>(b + l.unit_len);
    int32_t* bidx = reinterpret_cast<int32_t*>(b + l.bidx);
    int32_t* bcount = reinterpret_cast<int32_t*>(b + l.bcount);
    p.bidx = bidx;
    p.bcount = bcount;
    p.topk = topk;
    p.idx = a->idx;
    p.count = a->count;
    p.cap = a->cap;
    p.acap = topk * a->b + a->S;
    p.aidx = reinterpret_cast<int32_t*>(b + l.aidx);
    p.acount = reinterpret_cast<int32_t*>(b + l.acount);

    // 1. importance
    const size_t smem1 = size_t(kPbKeys) * kPbD * 4 + size_t(kPbD) * kPbRows * 4;
    const size_t smem2 = smem1 + size_t(kPbThreads / 32) * kPbKeys * 4;
    SPA_CUDA_TRY(cudaFuncSetAttribute(pbs_rowstats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem1)));
    SPA_CUDA_TRY(cudaFuncSetAttribute(pbs_importance_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem2)));
    SPA_CUDA_TRY(launch_pdl(pbs_rowstats_kernel, dim3(p.ntiles, a->Hkv), dim3(kPbThreads), smem1, st, p));
    SPA_CUDA_TRY(launch_pdl(pbs_rowcombine_kernel, dim3((p.R + kPbThreads - 1) / kPbThreads, a->Hkv),
                            dim3(kPbThreads), 0, st, p));
    SPA_CUDA_TRY(launch_pdl(pbs_importance_kernel, dim3(p.ntiles, a->Hkv), dim3(kPbThreads), smem2, st, p));
    // 2. permutation inside segments
    int P = 1;
    while (P < a->S) P <<= 1;
    SPA_CUDA_TRY(cudaFuncSetAttribute(pbs_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(P * 8)));
    SPA_CUDA_TRY(launch_pdl(pbs_sort_kernel, dim3((a->T + a->S - 1) / a->S, a->Hkv), dim3(1024), size_t(P) * 8, st, p));
    // 3. block means, block scores, top-k blocks
    SPA_CUDA_TRY(launch_pdl(pbs_means_kernel, dim3(nblk, a->Hkv, 2), dim3(kPbD), 0, st, p));
    SPA_CUDA_TRY(launch_pdl(pbs_scores_kernel, dim3(U), dim3(kPbThreads), 0, st, p));
    SelectParams sp{hist0_carve(b + l.hist, U), p.scores, p.unit_len, U, nblk, a->topk, 0.f, 0, 0, bidx, bcount,
                    topk, nullptr, status};
    spa_status s = launch_hist0(sp, false, st);
    if (s != SPA_OK) return s;
    if ((s = launch_select(sp, false, st)) != SPA_OK) return s;
    // 4. rows of the attention, then the tcgen05 attention
    int Pe = 1;
    while (Pe < topk * a->b) Pe <<= 1;
    SPA_CUDA_TRY(cudaFuncSetAttribute(pbs_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Pe * 4)));
    SPA_CUDA_TRY(launch_pdl(pbs_expand_kernel, dim3(U), dim3(kPbThreads), size_t(Pe) * 4, st, p));
    PrefillAttendParams pp{a->Q, a->K, a->V, p.aidx, p.acount, p.acap, a->Hq, a->Hkv, a->T, a->b, 0, a->sm_scale,
                           a->out, a->out_f32, status};
    return launch_prefill_attend(pp, U, st, events);
}

extern "C" spa_status spa_pbs_prefill(const spa_pbs_args* a, void* ws, size_t ws_bytes, void* stream) {
    return pbs_impl(a, ws, ws_bytes, stream, nullptr);
}

extern "C" spa_status spa_pbs_prefill_timed(const spa_pbs_args* a, void* ws, size_t ws_bytes, void* stream,
                                            void* const* events) {
    if (!events || !events[0] || !events[1]) return SPA_ERR_INVALID_ARG;
    return pbs_impl(a, ws, ws_bytes, stream, events);
}
