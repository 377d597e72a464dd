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
// Step 1 is a b*G x T x d contraction and runs on tcgen05 (two passes: row statistics, then the
// probabilities' column sums); steps 2-3 are CUDA-core kernels: the block scores as a tiled
// product of the block means, the top-k as a per-unit bitonic sort of (score, block) keys (a
// unit has at most T / b candidates), and the support as a bitmap of positions compacted in
// ascending order.
#include "internal.cuh"
#include "tc.cuh"

namespace spa {
namespace {

constexpr int kPbThreads = 256;
constexpr int kPbKeys = 128;       // keys per importance tile
constexpr int kPbD = 128;
constexpr float kPbLog2e = 1.4426950408889634f;

struct PbsParams {
    const uint16_t* Q;   // [T, Hq, d]
    const uint16_t* K;   // [Hkv, T, d]
    int T, Hq, Hkv, G, b, S, R, ntiles, nblk;
    float sm_scale;
    float* rm;           // [Hkv][ntiles][R] per-chunk row max (log2 units); ntiles = the chunk count
    float* rl;           // [Hkv][ntiles][R] per-chunk row sum
    float* M;            // [Hkv][R]
    float* L;            // [Hkv][R]
    float* imp;          // [Hkv][T]
    int32_t* perm;       // [Hkv][T]
    float* kbar;         // [Hkv][nblk][d]
    float* qbar;         // [nblk][Hkv][d]
    float* scores;       // [U][nblk]
    int32_t* bidx;       // [U][topk] selected blocks
    int32_t* bcount;
    int topk;
    int32_t* idx;        // [U][cap] support (original positions, ascending)
    int32_t* count;
    int cap;
    int32_t* aidx;       // [U][acap] rows of the attention: support, then [seg0, t0)
    int32_t* acount;
    int acap;
};

__device__ __forceinline__ float bf(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

// ---------------------------------------------------------------------------- importance
// The importance passes are R x T x d contractions (R = b * G rows of the last query block
// against every key of the kv head) and run on tcgen05: S = Q_last K_tile^T into TMEM, one
// 128 x 128 MMA tile per 128 rows, one thread per row.  R = 128 * NMT rows are staged once
// (row r: query T - b + r / G, head r % G); a CTA then walks a chunk of kImTiles key tiles with
// double-buffered cp.async.
//   PASS 0: per row, the max and sum of 2^(sm_scale log2e s) over the chunk's keys the row may
//           see (keys after its query count nothing) -> rm / rl [g][chunk][r];
//   PASS 1: per key, sum over rows of 2^(sm_scale log2e s - M_r) / L_r (M, L: the combined row
//           statistics).  A warp sums its 32 rows per column with a transposing butterfly of
//           shuffles (five steps over each half of the tile, the live columns halving at each),
//           the warps are then added in order, so the sum is in a fixed order.
constexpr int kImTiles = 16;              // key tiles of 128 per CTA
constexpr uint32_t kImSpinLimit = 1u << 22;

// One step of a transposing butterfly over a warp: each lane holds 2 HF live columns of its
// row; it keeps the half selected by (lane & MK), adds its partner's copy of that half, and hands
// the other half to the partner.  Five steps from 64 columns leave every lane with the warp's
// sums of 2 columns.
template <int HF, int MK>
__device__ __forceinline__ void bfly_step(float (&v)[64], int lane) {
    const bool up = (lane & MK) != 0;
#pragma unroll
    for (int i = 0; i < HF; ++i) {
        const float send = up ? v[i] : v[HF + i];
        const float keep = up ? v[HF + i] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, MK);
    }
}

template <int NMT>
struct __align__(1024) ImShared {
    uint8_t q[NMT][tc::kTileBytes];
    uint8_t k[2][tc::kTileBytes];
    uint64_t bar;
    uint32_t tmem_base;
    float colsum[4 * NMT][128];           // PASS 1: per-warp column sums of a tile
};

template <int NMT, int PASS>
__global__ void __launch_bounds__(128 * NMT, 1) pbs_importance_tc_kernel(PbsParams p, uint32_t* status) {
    using namespace tc;
    pdl_enter();
    extern __shared__ __align__(1024) uint8_t dyn[];
    ImShared<NMT>& sh = *reinterpret_cast<ImShared<NMT>*>(dyn);
    constexpr int R = 128 * NMT, NT = 128 * NMT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y, chunk = blockIdx.x;
    const int n_all = (p.T + 127) / 128;
    const int t_begin = chunk * kImTiles, t_end = min(n_all, t_begin + kImTiles);
    const int r = tid;                                          // this thread's row
    const int t_row = p.T - p.b + r / p.G;                      // its query position
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t col_off = uint32_t(warp >> 2) * 128;         // TMEM columns of its operand tile
    const float sl2 = p.sm_scale * kPbLog2e;
    constexpr uint32_t kId = idesc_bf16(128, 128, false);

    constexpr uint32_t kCols = NMT <= 1 ? 128 : (NMT <= 2 ? 256 : 512);   // a power of 2
    if (warp == 0) tmem_alloc(&sh.tmem_base, kCols);
    if (tid == 0) {
        mbar_init(&sh.bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    // Q rows, then the first key tile, in one cp.async group
    for (int i = tid; i < R * 16; i += NT) {
        const int row = i >> 4, c = i & 15;
        const size_t q = size_t(p.T - p.b + row / p.G) * p.Hq + size_t(g) * p.G + row % p.G;
        cp_async16(smem_u32(sh.q[row >> 7]) + tile_off(row & 127, c), p.Q + q * kPbD + c * 8, true);
    }
    auto issue = [&](int t) {
        if (t < t_end) {
            for (int i = tid; i < 128 * 16; i += NT) {
                const int kr = i >> 4, c = i & 15, n = t * 128 + kr;
                const bool ok = n < p.T;
                cp_async16(smem_u32(sh.k[t & 1]) + tile_off(kr, c), p.K + (ok ? (size_t(g) * p.T + n) * kPbD + c * 8 : 0),
                           ok);
            }
        }
        cp_async_commit();
    };
    issue(t_begin);
    const float Mr = PASS == 1 ? p.M[size_t(g) * R + r] : 0.f;
    const float inv_l = PASS == 1 ? 1.f / p.L[size_t(g) * R + r] : 0.f;
    float m = -INFINITY, l = 0.f;
    uint32_t phase = 0;
    bool my_to = false, pending = false, stopped = false;
    uint32_t tmem = 0;
    for (int t = t_begin; t < t_end; ++t) {
        issue(t + 1);                                           // the next tile's buffer was read by S(t - 1)
        cp_async_wait_group<1>();                               // tile t (and Q) landed
        fence_async_smem();
        tc_fence_before();
        stopped = __syncthreads_or(my_to) != 0;                 // also: S(t - 1) and colsum read by everyone
        tc_fence_after();
        if (stopped) break;
        tmem = sh.tmem_base;
        if (tid == 0) {
#pragma unroll
            for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = uint32_t((kk >> 2) * kSlab + (kk & 3) * 32);
                    umma_bf16(tmem + mt * 128, sw128_desc(smem_u32(sh.q[mt]) + off, 16, 1024),
                              sw128_desc(smem_u32(sh.k[t & 1]) + off, 16, 1024), kId, kk > 0);
                }
            umma_commit(&sh.bar);
        }
        pending = true;
        {
            uint32_t it = 0;
            bool done = true;
            while (!mbar_try_wait(&sh.bar, phase))
                if (++it >= kImSpinLimit) {
                    done = false;
                    my_to = true;
                    break;
                }
            if (done) {
                pending = false;
                phase ^= 1u;
            }
        }
        stopped = __syncthreads_or(my_to) != 0;                 // every thread takes the same path
        tc_fence_after();
        if (stopped) break;
        // this row's 128 logits of the tile, in two halves of 64 columns
        const int n0 = t * 128;
        const int lim = min(p.T - 1, t_row) - n0;               // keys c <= lim are seen by this row
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float v[64];
            {
                float w[32];
                tmem_ld32(tmem + col_off + lane_off + hh * 64, w);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = w[i];
                tmem_ld32(tmem + col_off + lane_off + hh * 64 + 32, w);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[32 + i] = w[i];
            }
            const int lh = lim - hh * 64;
            if (PASS == 0) {
                float tmax = -INFINITY;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    v[c] = c <= lh ? v[c] * sl2 : -INFINITY;
                    tmax = fmaxf(tmax, v[c]);
                }
                if (tmax != -INFINITY) {
                    const float mn = fmaxf(m, tmax);
                    float add = 0.f;
#pragma unroll
                    for (int c = 0; c < 64; ++c) add += exp2f(v[c] - mn);
                    l = l * exp2f(m - mn) + add;
                    m = mn;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) v[c] = c <= lh ? exp2f(fmaf(v[c], sl2, -Mr)) * inv_l : 0.f;
                bfly_step<32, 16>(v, lane);
                bfly_step<16, 8>(v, lane);
                bfly_step<8, 4>(v, lane);
                bfly_step<4, 2>(v, lane);
                bfly_step<2, 1>(v, lane);
                // this lane now holds the warp's sums of columns c0, c0 + 1 of the half
                const int c0 = ((lane >> 4) & 1) * 32 + ((lane >> 3) & 1) * 16 + ((lane >> 2) & 1) * 8 +
                               ((lane >> 1) & 1) * 4 + (lane & 1) * 2;
                sh.colsum[warp][hh * 64 + c0] = v[0];
                sh.colsum[warp][hh * 64 + c0 + 1] = v[1];
            }
        }
        tc_fence_before();
        if (PASS == 1) {
            __syncthreads();
            if (tid < 128 && n0 + tid < p.T) {
                float tot = 0.f;
#pragma unroll
                for (int w = 0; w < 4 * NMT; ++w) tot += sh.colsum[w][tid];
                p.imp[size_t(g) * p.T + n0 + tid] = tot / float(R);
            }
        }
    }
    cp_async_wait_all();
    tc_fence_before();
    const bool good = __syncthreads_or(my_to) == 0;
    if (PASS == 0 && good) {
        p.rm[(size_t(g) * p.ntiles + chunk) * R + r] = m;
        p.rl[(size_t(g) * p.ntiles + chunk) * R + r] = l;
    }
    if (!good && tid == 0) raise_status(status, SPA_ERR_TIMEOUT);
    // an MMA that was not seen to complete may still be running: wait once more (bounded) and
    // free the tensor memory only when nothing is owed
    if (pending) {
        uint32_t it = 0;
        while (!mbar_try_wait(&sh.bar, phase) && ++it < kImSpinLimit) {
        }
        pending = it >= kImSpinLimit;
    }
    if (warp == 0 && !__any_sync(0xffffffffu, pending)) {
        tc_fence_after();
        tmem_dealloc(sh.tmem_base, kCols);
    }
}

// every row's max and sum over all chunks (chunk order)
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
// its b queries and G heads, in (query, head) order); one thread per channel.  The block's 64
// permuted positions are staged in shared memory first; loads are then issued eight at a time
// and the sums keep their sequential order.
__global__ void __launch_bounds__(kPbD) pbs_means_kernel(PbsParams p) {
    pdl_enter();
    __shared__ int32_t pm[64];
    const int blk = blockIdx.x, g = blockIdx.y, c = threadIdx.x;
    float s = 0.f;
    if (blockIdx.z == 0) {
        if (c < p.b) pm[c] = p.perm[size_t(g) * p.T + size_t(blk) * p.b + c];   // b = 64
        __syncthreads();
        const uint16_t* kg = p.K + size_t(g) * p.T * kPbD + c;
        for (int i = 0; i < p.b; i += 8) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = bf(kg[size_t(pm[i + e]) * kPbD]);
#pragma unroll
            for (int e = 0; e < 8; ++e) s += v[e];
        }
        p.kbar[(size_t(g) * p.nblk + blk) * kPbD + c] = s / float(p.b);
    } else {
        // rows (query i, head h) in (i, h) order; b * G is a multiple of 8
        const uint16_t* qb = p.Q + (size_t(blk) * p.b * p.Hq + size_t(g) * p.G) * kPbD + c;
        int i = 0, h = 0;
        for (int f = 0; f < p.b * p.G; f += 8) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[e] = bf(qb[(size_t(i) * p.Hq + h) * kPbD]);
                if (++h == p.G) {
                    h = 0;
                    ++i;
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) s += v[e];
        }
        p.qbar[(size_t(blk) * p.Hkv + g) * kPbD + c] = s / float(p.b * p.G);
    }
}

// Block scores sm_scale * qbar . kbar over the permuted blocks before each query block's own
// segment.  CTA per (kv head g, kPbJ consecutive query blocks): their qbar rows sit in shared
// memory; each thread takes key blocks c = tid, tid + 256, ..., loads kbar[c] once and forms the
// dots with every query block of the tile that has c among its candidates.  Each dot runs over
// the channels in ascending order.
constexpr int kPbJ = 32;
__global__ void __launch_bounds__(kPbThreads) pbs_scores_kernel(PbsParams p) {
    pdl_enter();
    __shared__ __align__(16) float qs[kPbJ][kPbD];
    const int g = blockIdx.y, j0 = blockIdx.x * kPbJ;
    const int nj = min(kPbJ, p.nblk - j0);
    for (int i = threadIdx.x; i < nj * kPbD; i += kPbThreads)
        qs[i / kPbD][i % kPbD] = p.qbar[(size_t(j0 + i / kPbD) * p.Hkv + g) * kPbD + i % kPbD];
    __syncthreads();
    const int nc_max = ((j0 + nj - 1) * p.b) / p.S * p.S / p.b;   // the tile's largest candidate count
    for (int c = threadIdx.x; c < nc_max; c += kPbThreads) {
        float4 kb[kPbD / 4];
        const float4* k4 = reinterpret_cast<const float4*>(p.kbar + (size_t(g) * p.nblk + c) * kPbD);
#pragma unroll
        for (int d4 = 0; d4 < kPbD / 4; ++d4) kb[d4] = k4[d4];
        for (int jj = 0; jj < nj; ++jj) {
            const int j = j0 + jj;
            if (c >= (j * p.b) / p.S * p.S / p.b) continue;
            const float4* q4 = reinterpret_cast<const float4*>(qs[jj]);
            float dot = 0.f;
#pragma unroll
            for (int d4 = 0; d4 < kPbD / 4; ++d4) {
                const float4 q = q4[d4];
                dot = fmaf(q.x, kb[d4].x, dot);
                dot = fmaf(q.y, kb[d4].y, dot);
                dot = fmaf(q.z, kb[d4].z, dot);
                dot = fmaf(q.w, kb[d4].w, dot);
            }
            p.scores[size_t(j * p.Hkv + g) * p.nblk + c] = p.sm_scale * dot;
        }
    }
}

// Block top-k of unit u: its nc candidate scores sorted by (score desc, block asc) with a
// bitonic sort of 64-bit keys in shared memory; the first min(k, nc) blocks are kept.
__global__ void __launch_bounds__(kPbThreads) pbs_topk_kernel(PbsParams p, int k) {
    pdl_enter();
    extern __shared__ __align__(16) unsigned long long tk[];
    const int u = blockIdx.x, j = u / p.Hkv;
    const int nc = (j * p.b) / p.S * p.S / p.b;
    int P = 1;
    while (P < nc) P <<= 1;
    for (int i = threadIdx.x; i < P; i += kPbThreads) {
        unsigned long long key = ~0ull;
        if (i < nc) {
            const uint32_t sk = score_key(p.scores[size_t(u) * p.nblk + i]);
            key = (static_cast<unsigned long long>(~sk) << 32) | uint32_t(i);
        }
        tk[i] = key;
    }
    __syncthreads();
    for (int kk = 2; kk <= P; kk <<= 1) {
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            for (int i = threadIdx.x; i < P; i += kPbThreads) {
                const int ixj = i ^ jj;
                if (ixj > i) {
                    const bool up = (i & kk) == 0;
                    const unsigned long long a = tk[i], c = tk[ixj];
                    if ((a > c) == up) {
                        tk[i] = c;
                        tk[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    const int kept = k < nc ? k : nc;
    for (int i = threadIdx.x; i < kept; i += kPbThreads) p.bidx[size_t(u) * p.topk + i] = int32_t(tk[i] & 0xffffffffu);
    if (threadIdx.x == 0) p.bcount[u] = kept;
}

// selected blocks -> their keys' original positions, ascending (the support): the positions are
// marked in a bitmap of [0, seg0) in shared memory (the blocks lie in earlier segments and the
// permutation stays inside segments) and compacted in order; the attention's rows are the
// support followed by the own segment's keys before the block, [seg0, t0)
__global__ void __launch_bounds__(kPbThreads) pbs_expand_kernel(PbsParams p) {
    pdl_enter();
    extern __shared__ __align__(16) uint32_t bits[];
    __shared__ int wsum[kPbThreads / 32];
    const int u = blockIdx.x, j = u / p.Hkv, g = u - j * p.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = j * p.b, seg0 = t0 / p.S * p.S;
    int nb = p.bcount[u];
    nb = nb < 0 ? 0 : (nb > p.topk ? p.topk : nb);
    const int n = nb * p.b;
    const int nw = (seg0 + 31) / 32;
    for (int i = tid; i < nw; i += kPbThreads) bits[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kPbThreads) {
        const int blk = p.bidx[size_t(u) * p.topk + i / p.b];
        const int pos = p.perm[size_t(g) * p.T + size_t(blk) * p.b + (i % p.b)];
        if (pos >= 0 && pos < seg0) atomicOr(&bits[pos >> 5], 1u << (pos & 31));
    }
    __syncthreads();
    // thread t owns words [t W, t W + W): count, exclusive scan over threads, then write in order
    const int W = (nw + kPbThreads - 1) / kPbThreads;
    const int w0 = min(nw, tid * W), w1 = min(nw, w0 + W);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += x;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int base = incl - cnt;
    for (int w = 0; w < warp; ++w) base += wsum[w];
    int total = 0;
    for (int w = 0; w < kPbThreads / 32; ++w) total += wsum[w];
    int32_t* out_i = p.idx + size_t(u) * p.cap;
    int32_t* out_a = p.aidx + size_t(u) * p.acap;
    for (int w = w0; w < w1; ++w) {
        uint32_t x = bits[w];
        while (x) {
            const int bit = __ffs(x) - 1;
            x &= x - 1;
            out_i[base] = w * 32 + bit;
            out_a[base] = w * 32 + bit;
            ++base;
        }
    }
    for (int i = tid; i < t0 - seg0; i += kPbThreads) out_a[total + i] = seg0 + i;
    if (tid == 0) {
        p.count[u] = total;
        p.acount[u] = total + (t0 - seg0);
    }
}

struct PbsLayout {
    size_t rm, rl, M, L, imp, perm, kbar, qbar, scores, bidx, bcount, aidx, acount, total;
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

    // 1. importance (tcgen05): row statistics per key chunk, combined per row, then the column sums
    const int nchunk = (p.ntiles + kImTiles - 1) / kImTiles;
    p.ntiles = nchunk;                                        // rm / rl hold one record per chunk
    const int nmt = p.R / 128;
#define SPA_PB_IMP(NMT)                                                                                         \
    if (nmt == NMT) {                                                                                           \
        const size_t sm = sizeof(ImShared<NMT>);                                                                \
        SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(pbs_importance_tc_kernel<NMT, 0>),            \
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)));                     \
        SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(pbs_importance_tc_kernel<NMT, 1>),            \
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)));                     \
        SPA_CUDA_TRY(launch_pdl(pbs_importance_tc_kernel<NMT, 0>, dim3(nchunk, a->Hkv), dim3(128 * NMT), sm, st,  \
                                p, status));                                                                    \
        SPA_CUDA_TRY(launch_pdl(pbs_rowcombine_kernel, dim3((p.R + kPbThreads - 1) / kPbThreads, a->Hkv),        \
                                dim3(kPbThreads), 0, st, p));                                                   \
        SPA_CUDA_TRY(launch_pdl(pbs_importance_tc_kernel<NMT, 1>, dim3(nchunk, a->Hkv), dim3(128 * NMT), sm, st,  \
                                p, status));                                                                    \
    }
    SPA_PB_IMP(1) else SPA_PB_IMP(2) else SPA_PB_IMP(3) else SPA_PB_IMP(4) else return SPA_ERR_UNSUPPORTED_SHAPE;
#undef SPA_PB_IMP
    // 2. permutation inside segments
    int P = 1;
    while (P < a->S) P <<= 1;
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(pbs_sort_kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(P * 8)));
    SPA_CUDA_TRY(launch_pdl(pbs_sort_kernel, dim3((a->T + a->S - 1) / a->S, a->Hkv), dim3(1024), size_t(P) * 8, st, p));
    // 3. block means, block scores, top-k blocks
    SPA_CUDA_TRY(launch_pdl(pbs_means_kernel, dim3(nblk, a->Hkv, 2), dim3(kPbD), 0, st, p));
    SPA_CUDA_TRY(launch_pdl(pbs_scores_kernel, dim3((nblk + kPbJ - 1) / kPbJ, a->Hkv), dim3(kPbThreads), 0, st, p));
    int Pk = 1;
    while (Pk < nblk) Pk <<= 1;
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(pbs_topk_kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(Pk * 8)));
    SPA_CUDA_TRY(launch_pdl(pbs_topk_kernel, dim3(U), dim3(kPbThreads), size_t(Pk) * 8, st, p, a->topk));
    // 4. rows of the attention, then the tcgen05 attention
    const size_t bitmap = size_t((a->T + 31) / 32) * 4;
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(pbs_expand_kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(bitmap)));
    SPA_CUDA_TRY(launch_pdl(pbs_expand_kernel, dim3(U), dim3(kPbThreads), bitmap, st, p));
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
