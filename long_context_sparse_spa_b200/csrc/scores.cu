// Streaming score kernels: low-rank index scores ("Full Attention Strikes Back"
// (RTPurbo), Methodology 2; head collapse per "Oracle-Guided Sparse Prefill" 2.2),
// Taylor block scores and block statistics ("SPLA" 2.1).
//
// All three are HBM-bound streams with a few flops per byte: they are written for
// coalesced 128-bit loads, enough bytes in flight per SM and grids sized in multiples
// of the SM count.  Reductions run in a fixed order, so results are bit-reproducible.
#include "internal.cuh"

namespace spa {
namespace {

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ============================================================================ low-rank
// One work item = (kv unit, chunk of at most kLrChunk rows).  Two lanes share a 32-byte index-key
// row: each loads one 16-byte half (8 bf16) and the halves are joined with one
// warp shuffle.  Each thread keeps kLrUnroll rows of loads in flight.
// With HIST (one score per row, GROUP_MEAN), the CTA also histograms its scores into the
// level-0 selection histogram (shared-memory bins flushed to global with integer atomics,
// so the result does not depend on the order of accumulation).
constexpr int kLrThreads = 256;
constexpr int kLrUnroll = 8;
// At most 4080 rows per item: each 32-bit half of an item's fixed-point bin masses takes at most
// 2^20 per row (masses are at most 2^40), so no half can overflow below 4096 rows.
constexpr int kLrChunk = 4080;

template <int NQ, bool HIST, bool MASS>
__global__ void __launch_bounds__(kLrThreads)
lowrank_scores_kernel(const uint16_t* __restrict__ qidx, const uint4* __restrict__ kidx, int Hq, int Hkv,
                      int M, float scale, float* __restrict__ scores, int chunks_per_unit, int chunk_rows, int n_items,
                      Hist0 hist, const uint8_t* __restrict__ local, int kv_shared) {
    pdl_enter();
    const int G = Hq / Hkv;
    const int half = threadIdx.x & 1;          // which 8 of the 16 index dims this lane holds
    const int pair = threadIdx.x >> 1;         // row slot within a pass
    constexpr int kRowsPerPass = kLrThreads / 2;
    constexpr int kHb = HIST ? kHistBins : 1;
    __shared__ __align__(16) uint32_t h_cnt[kHb];
    __shared__ __align__(16) uint32_t h_mhi[MASS ? kHb : 1];
    __shared__ __align__(16) uint32_t h_mlo[MASS ? kHb : 1];
    __shared__ uint32_t h_max;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int kvu = item / chunks_per_unit;        // b * Hkv + g
        const int chunk = item - kvu * chunks_per_unit;
        const int b = kvu / Hkv, g = kvu - b * Hkv;
        if (NQ == 1 && local && local[kvu]) continue;  // a local unit is not scored (uniform per CTA)
        if (HIST) {
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            for (int i = threadIdx.x; i < kHistBins / 4; i += kLrThreads) {
                reinterpret_cast<uint4*>(h_cnt)[i] = z4;
                if (MASS) reinterpret_cast<uint4*>(h_mhi)[i] = reinterpret_cast<uint4*>(h_mlo)[i] = z4;
            }
            if (threadIdx.x == 0) h_max = 0;
            __syncthreads();
        }
        uint32_t my_max = 0;

        // Index query (8 dims of it) per query vector, fp32.
        float qv[NQ][8];
        const uint16_t* qbase = qidx + (size_t(b) * Hq + size_t(g) * G) * 16 + half * 8;
        if (NQ == 1) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int h = 0; h < G; ++h) {             // heads summed in order 0..G-1
                const uint4 w = *reinterpret_cast<const uint4*>(qbase + size_t(h) * 16);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[2 * j] += bf_lo(ws[j]);
                    acc[2 * j + 1] += bf_hi(ws[j]);
                }
            }
            const float fg = float(G);
#pragma unroll
            for (int j = 0; j < 8; ++j) qv[0][j] = acc[j] / fg;
        } else {
#pragma unroll
            for (int h = 0; h < NQ; ++h) {
                const uint4 w = *reinterpret_cast<const uint4*>(qbase + size_t(h) * 16);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    qv[h][2 * j] = bf_lo(ws[j]);
                    qv[h][2 * j + 1] = bf_hi(ws[j]);
                }
            }
        }

        const int n0 = chunk * chunk_rows;
        const int n1 = min(M, n0 + chunk_rows);
        // kv_shared: one key set [Hkv][M] serves every batch row (per-query prefill)
        const uint4* krow = kidx + size_t(kv_shared ? g : kvu) * M * 2 + half;
        float* out_base = NQ == 1 ? scores + size_t(kvu) * M : scores + (size_t(b) * Hq + size_t(g) * G) * M;

        // every lane runs the same number of passes (the shuffle below needs the whole warp),
        // rows past the chunk are masked
        for (int pb = n0; pb < n1; pb += kRowsPerPass * kLrUnroll) {
            const int nb = pb + pair;
            uint4 w[kLrUnroll];
#pragma unroll
            for (int i = 0; i < kLrUnroll; ++i) {
                const int n = nb + i * kRowsPerPass;
                w[i] = n < n1 ? __ldg(krow + size_t(n) * 2) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < kLrUnroll; ++i) {
                const int n = nb + i * kRowsPerPass;
                const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
                for (int h = 0; h < NQ; ++h) {
                    float part = 0.f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        part = fmaf(qv[h][2 * j], bf_lo(ws[j]), part);
                        part = fmaf(qv[h][2 * j + 1], bf_hi(ws[j]), part);
                    }
                    const float other = __shfl_xor_sync(0xffffffffu, part, 1);
                    const float dot = half ? other + part : part + other;   // low half + high half
                    if (!half && n < n1) {
                        const float sc = scale * dot;
                        out_base[size_t(h) * M + n] = sc;
                        if (HIST) {
                            const uint32_t key = score_key(sc);
                            const uint32_t bin = key >> 21;
                            my_max = max(my_max, key);
                            atomicAdd(&h_cnt[bin], 1u);
                            if (MASS) {
                                // the 41-bit fixed-point mass as two 32-bit halves (20 low
                                // bits, the rest high): with <= kLrChunk < 4096 rows per work
                                // item neither half can overflow
                                const unsigned long long e = fixed_mass(sc, bin_top_score(bin));
                                atomicAdd(&h_mhi[bin], uint32_t(e >> 20));
                                atomicAdd(&h_mlo[bin], uint32_t(e & 0xfffffu));
                            }
                        }
                    }
                }
            }
        }
        if (HIST) {
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, off));
            if ((threadIdx.x & 31) == 0) atomicMax(&h_max, my_max);
            __syncthreads();
            uint32_t* gc = hist.cnt + size_t(kvu) * kHistBins;
            unsigned long long* gm = hist.mass + size_t(kvu) * kHistBins;
            for (int i4 = threadIdx.x; i4 < kHistBins / 4; i4 += kLrThreads) {   // four bins at a time
                const uint4 c4 = reinterpret_cast<const uint4*>(h_cnt)[i4];
                if ((c4.x | c4.y | c4.z | c4.w) == 0) continue;
                const uint32_t c[4] = {c4.x, c4.y, c4.z, c4.w};
                uint32_t mh[4] = {0, 0, 0, 0}, ml[4] = {0, 0, 0, 0};
                if (MASS) {
                    const uint4 h4 = reinterpret_cast<const uint4*>(h_mhi)[i4];
                    const uint4 l4 = reinterpret_cast<const uint4*>(h_mlo)[i4];
                    mh[0] = h4.x; mh[1] = h4.y; mh[2] = h4.z; mh[3] = h4.w;
                    ml[0] = l4.x; ml[1] = l4.y; ml[2] = l4.z; ml[3] = l4.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (!c[j]) continue;
                    atomicAdd(gc + 4 * i4 + j, c[j]);
                    if (MASS) atomicAdd(gm + 4 * i4 + j, (static_cast<unsigned long long>(mh[j]) << 20) + ml[j]);
                }
            }
            if (threadIdx.x == 0) atomicMax(hist.max_key + kvu, h_max);
            __syncthreads();
        }
    }
}

// ============================================================================ block scores
// One work item = (kv unit, chunk of kTyChunk blocks).  Eight lanes share a block: each
// holds D/8 dims of the block statistics (float4 loads) and the per-head partial sums for
// the G heads are joined by three xor-shuffles.  q' = scale * q lives in shared memory.
//   KIND_TAYLOR ("SPLA" 2.1): stats (mean, var); a_h = q'_h . mean, c_h = sum q'_h^2 var,
//                 score log t (t averaged over the heads under GROUP_MEAN).
//   KIND_MINMAX (min/max pooling, "SPLA" 1; token-to-page selection, "The Sparse
//                 Frontier"): stats (min, max); a_h = sum_i max(q'_i min_i, q'_i max_i),
//                 the largest logit inside the block's channel box.
//   KIND_MEAN   (mean pooling, "SPLA" 1, PBS-Attn 4): stats (mean); a_h = q'_h . mean.
//   Under GROUP_MEAN the min-max and mean scores are averaged over the G heads.
// SBF16: the statistics are stored as bf16 (8-byte loads of four values) instead of fp32.
constexpr int kTyThreads = 256;
constexpr int kTyChunk = 256;
constexpr int KIND_TAYLOR = 0, KIND_MINMAX = 1, KIND_MEAN = 2;

// four statistics at position f4 (in units of four values) of a row starting at base
template <bool SBF16>
__device__ __forceinline__ float4 load_stats4(const void* p, size_t base, int f4) {
    if constexpr (SBF16) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(p) + base + f4);
        return make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
    } else {
        return __ldg(reinterpret_cast<const float4*>(p) + base + f4);
    }
}

template <int D, int G, int KIND, bool SBF16>
__global__ void __launch_bounds__(kTyThreads)
taylor_scores_kernel(const uint16_t* __restrict__ q, const void* __restrict__ mean, const void* __restrict__ var,
                     int Hq, int Hkv, int M, int collapse, float scale, float* __restrict__ scores,
                     int chunks_per_unit, int n_items, const uint8_t* __restrict__ local) {
    pdl_enter();
    __shared__ float qs[G][D];
    constexpr int kPer = D / 8;          // dims per lane
    constexpr int kVec = kPer / 4;       // float4 loads per lane per tensor
    const int lane8 = threadIdx.x & 7;
    const int slot = threadIdx.x >> 3;   // block slot within a pass
    constexpr int kSlots = kTyThreads / 8;
    int cur_kvu = -1;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int kvu = item / chunks_per_unit;
        const int chunk = item - kvu * chunks_per_unit;
        const int b = kvu / Hkv, g = kvu - b * Hkv;
        // a local unit (GROUP_MEAN: one unit per kv head) is not scored (uniform per CTA)
        if (collapse == SPA_COLLAPSE_GROUP_MEAN && local && local[kvu]) continue;
        if (kvu != cur_kvu) {
            __syncthreads();
            for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
                const uint16_t h = q[(size_t(b) * Hq + size_t(g) * G + i / D) * D + (i % D)];
                qs[i / D][i % D] = scale * __uint_as_float(uint32_t(h) << 16);
            }
            __syncthreads();
            cur_kvu = kvu;
        }
        const int b0 = chunk * kTyChunk;
        const int b1 = min(M, b0 + kTyChunk);
        for (int pass = b0; pass < b1; pass += kSlots) {   // same trip count for every lane
            const int blk = pass + slot;
            const bool live = blk < b1;
            float a[G], c[G];
#pragma unroll
            for (int h = 0; h < G; ++h) a[h] = c[h] = 0.f;
            if (live) {
                const size_t base = (size_t(kvu) * M + blk) * (D / 4);
#pragma unroll
                for (int v = 0; v < kVec; ++v) {
                    // lane8 owns dims {4*(lane8 + 8*v) .. +3}: 8 lanes read 128 contiguous bytes
                    const int f4 = lane8 + 8 * v;
                    const float4 mu = load_stats4<SBF16>(mean, base, f4);
                    const float4 vr = KIND == KIND_MEAN ? make_float4(0.f, 0.f, 0.f, 0.f)
                                                        : load_stats4<SBF16>(var, base, f4);
                    const float mus[4] = {mu.x, mu.y, mu.z, mu.w};
                    const float vrs[4] = {vr.x, vr.y, vr.z, vr.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 4 * f4 + e;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float qp = qs[h][i];
                            if (KIND == KIND_MINMAX) {
                                a[h] += fmaxf(qp * mus[e], qp * vrs[e]);
                            } else {
                                a[h] = fmaf(qp, mus[e], a[h]);
                                if (KIND == KIND_TAYLOR) c[h] = fmaf(qp * qp, vrs[e], c[h]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int off = 4; off >= 1; off >>= 1) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    a[h] += __shfl_xor_sync(0xffffffffu, a[h], off);
                    c[h] += __shfl_xor_sync(0xffffffffu, c[h], off);
                }
            }
            if (!live) continue;
            if (KIND != KIND_TAYLOR) {
                if (collapse == SPA_COLLAPSE_GROUP_MEAN) {
                    if (lane8 == 0) {
                        float acc = 0.f;
#pragma unroll
                        for (int h = 0; h < G; ++h) acc += a[h];
                        scores[size_t(kvu) * M + blk] = acc / float(G);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        if ((h & 7) == lane8) scores[(size_t(b) * Hq + size_t(g) * G + h) * M + blk] = a[h];
                }
                continue;
            }
            if (collapse == SPA_COLLAPSE_GROUP_MEAN) {
                if (lane8 == 0) {
                    float mx = a[0];
#pragma unroll
                    for (int h = 1; h < G; ++h) mx = fmaxf(mx, a[h]);
                    float acc = 0.f;
#pragma unroll
                    for (int h = 0; h < G; ++h) acc += expf(a[h] - mx) * (1.f + 0.5f * c[h]);
                    scores[size_t(kvu) * M + blk] = mx + logf(acc / float(G));
                }
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h)
                    if ((h & 7) == lane8)
                        scores[(size_t(b) * Hq + size_t(g) * G + h) * M + blk] = a[h] + log1pf(0.5f * c[h]);
            }
        }
    }
}

// ============================================================================ block stats
// One CTA of 128 threads per 64-token (or 32/128) block at a time: thread t holds 8
// dims (one 16-byte chunk) of BLOCK*D/1024 rows in registers, so the two passes (mean,
// then squared deviations) read HBM once.
// store one statistic: fp32, or its bf16 rounding (round to nearest even)
template <bool OBF16>
__device__ __forceinline__ void store_stat(void* p, size_t i, float v) {
    if constexpr (OBF16) {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        reinterpret_cast<__nv_bfloat16*>(p)[i] = h;
    } else {
        reinterpret_cast<float*>(p)[i] = v;
    }
}

template <int D, int BLOCK, bool OBF16>
__global__ void __launch_bounds__(128)
block_stats_kernel(const uint4* __restrict__ K, int n_blocks, int nb_per_unit, int N, void* __restrict__ mean,
                   void* __restrict__ var) {
    pdl_enter();
    constexpr int DV = D / 8;                 // 16-byte chunks per row
    constexpr int PH = 128 / DV;              // row phases
    constexpr int RPT = BLOCK / PH;           // rows per thread
    static_assert(RPT * PH == BLOCK, "block must be a multiple of the row phases");
    __shared__ float red[PH][D];
    __shared__ float mu_s[D];
    const int c = threadIdx.x % DV;
    const int ph = threadIdx.x / DV;

    for (int blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
        const int unit = blk / nb_per_unit;
        const int j = blk - unit * nb_per_unit;
        const uint4* base = K + (size_t(unit) * N + size_t(j) * BLOCK) * DV + c;
        uint4 w[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) w[i] = __ldg(base + size_t(ph + i * PH) * DV);
        float s[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) s[e] = 0.f;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s[2 * e] += bf_lo(ws[e]);
                s[2 * e + 1] += bf_hi(ws[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[ph][c * 8 + e] = s[e];
        __syncthreads();
        if (threadIdx.x < D) {
            float t = 0.f;
#pragma unroll
            for (int p = 0; p < PH; ++p) t += red[p][threadIdx.x];
            const float m = t / float(BLOCK);
            mu_s[threadIdx.x] = m;                 // the deviations use the fp32 mean
            store_stat<OBF16>(mean, size_t(blk) * D + threadIdx.x, m);
        }
        __syncthreads();
        float mv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { mv[e] = mu_s[c * 8 + e]; s[e] = 0.f; }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float d0 = bf_lo(ws[e]) - mv[2 * e];
                const float d1 = bf_hi(ws[e]) - mv[2 * e + 1];
                s[2 * e] = fmaf(d0, d0, s[2 * e]);
                s[2 * e + 1] = fmaf(d1, d1, s[2 * e + 1]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[ph][c * 8 + e] = s[e];
        __syncthreads();
        if (threadIdx.x < D) {
            float t = 0.f;
#pragma unroll
            for (int p = 0; p < PH; ++p) t += red[p][threadIdx.x];
            store_stat<OBF16>(var, size_t(blk) * D + threadIdx.x, t / float(BLOCK));
        }
        __syncthreads();
    }
}

// Per-block channel minimum and maximum of K (min/max pooling, "SPLA" 1): the loads of
// block_stats_kernel, one pass, exact (bf16 values are exact in fp32).
template <int D, int BLOCK, bool OBF16>
__global__ void __launch_bounds__(128)
block_minmax_kernel(const uint4* __restrict__ K, int n_blocks, int nb_per_unit, int N, void* __restrict__ mn,
                    void* __restrict__ mx) {
    pdl_enter();
    constexpr int DV = D / 8;
    constexpr int PH = 128 / DV;
    constexpr int RPT = BLOCK / PH;
    static_assert(RPT * PH == BLOCK, "block must be a multiple of the row phases");
    __shared__ float rlo[PH][D], rhi[PH][D];
    const int c = threadIdx.x % DV;
    const int ph = threadIdx.x / DV;

    for (int blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
        const int unit = blk / nb_per_unit;
        const int j = blk - unit * nb_per_unit;
        const uint4* base = K + (size_t(unit) * N + size_t(j) * BLOCK) * DV + c;
        uint4 w[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) w[i] = __ldg(base + size_t(ph + i * PH) * DV);
        float lo[8], hi[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { lo[e] = INFINITY; hi[e] = -INFINITY; }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                lo[2 * e] = fminf(lo[2 * e], bf_lo(ws[e]));
                hi[2 * e] = fmaxf(hi[2 * e], bf_lo(ws[e]));
                lo[2 * e + 1] = fminf(lo[2 * e + 1], bf_hi(ws[e]));
                hi[2 * e + 1] = fmaxf(hi[2 * e + 1], bf_hi(ws[e]));
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            rlo[ph][c * 8 + e] = lo[e];
            rhi[ph][c * 8 + e] = hi[e];
        }
        __syncthreads();
        if (threadIdx.x < D) {
            float l = INFINITY, h = -INFINITY;
#pragma unroll
            for (int p = 0; p < PH; ++p) {
                l = fminf(l, rlo[p][threadIdx.x]);
                h = fmaxf(h, rhi[p][threadIdx.x]);
            }
            store_stat<OBF16>(mn, size_t(blk) * D + threadIdx.x, l);   // exact: bf16 values
            store_stat<OBF16>(mx, size_t(blk) * D + threadIdx.x, h);
        }
        __syncthreads();
    }
}

int grid_for(int items, int per_sm) {
    const int cap = device_info().num_sms * per_sm;
    return items < cap ? (items > 0 ? items : 1) : cap;
}

// Rows per work item of the low-rank scorer, at most kLrChunk.  The grid is made a whole number
// of waves of the CTAs the SMs hold at once: the fewest waves for which items of at most
// kLrChunk rows cover every unit, with every unit cut into the same number of items.  A partial
// last wave (1024 items of 2048 rows for 592 resident CTAs at a 128K-token cache) leaves most of
// the SMs idle while it runs.  Short caches are cut into items of at least min_rows rows (a
// histogram item clears and flushes 2048 bins).
template <typename Kern>
int lr_chunk_rows(Kern kern, int units, int M, int min_rows) {
    const int sms = device_info().num_sms;
    int per_sm = occupancy_blocks(reinterpret_cast<const void*>(kern), kLrThreads, 0);
    if (per_sm <= 0) per_sm = 1;
    const long long resident = (long long)per_sm * sms;
    const long long fewest = (long long)units * ((M + kLrChunk - 1) / kLrChunk);   // items at kLrChunk rows
    const long long waves = (fewest + resident - 1) / resident;
    const long long per_unit = (waves * resident + units - 1) / units;             // items per unit
    int rows = int((M + per_unit - 1) / per_unit);
    rows = (rows + 15) / 16 * 16;
    rows = rows < min_rows ? min_rows : rows;
    return rows > kLrChunk ? kLrChunk : rows;
}

}  // namespace

spa_status launch_lowrank_scores(const uint16_t* qidx, const uint16_t* kidx, int B, int Hq, int Hkv, int M,
                                 int collapse, float scale, float* scores, const Hist0* hist, bool with_mass,
                                 cudaStream_t st, const uint8_t* local, bool kv_shared) {
    const int G = Hq / Hkv;
    const int units = B * Hkv;
    const uint4* k4 = reinterpret_cast<const uint4*>(kidx);
    const Hist0 h = hist ? *hist : Hist0{nullptr, nullptr, nullptr};
    if (collapse == SPA_COLLAPSE_GROUP_MEAN) {
        auto kern = hist && with_mass ? lowrank_scores_kernel<1, true, true>
                                      : (hist ? lowrank_scores_kernel<1, true, false> : lowrank_scores_kernel<1, false, false>);
        const int rows = lr_chunk_rows(kern, units, M, hist ? 1024 : 256);
        const int chunks = (M + rows - 1) / rows;
        const int items = units * chunks;
        SPA_CUDA_TRY(launch_pdl(kern, dim3(grid_for(items, 32)), dim3(kLrThreads), 0, st, qidx, k4, Hq, Hkv, M, scale,
                                scores, chunks, rows, items, h, local, kv_shared ? 1 : 0));
    } else {
        if (hist) return SPA_ERR_INVALID_ARG;
        switch (G) {
#define SPA_LR_CASE(n)                                                                                          \
    case n: {                                                                                                   \
        const int rows = lr_chunk_rows(lowrank_scores_kernel<n, false, false>, units, M, 256);                 \
        const int chunks = (M + rows - 1) / rows;                                                              \
        const int items = units * chunks;                                                                      \
        SPA_CUDA_TRY(launch_pdl(lowrank_scores_kernel<n, false, false>, dim3(grid_for(items, 32)), dim3(kLrThreads), \
                                0, st, qidx, k4, Hq, Hkv, M, scale, scores, chunks, rows, items, h, nullptr,     \
                                kv_shared ? 1 : 0));                                                           \
        break;                                                                                                 \
    }
            SPA_LR_CASE(1) SPA_LR_CASE(2) SPA_LR_CASE(4) SPA_LR_CASE(8) SPA_LR_CASE(16)
#undef SPA_LR_CASE
            default: return SPA_ERR_UNSUPPORTED_SHAPE;
        }
    }
    return SPA_OK;
}

spa_status launch_taylor_scores(const uint16_t* q, const void* mean, const void* var, int B, int Hq, int Hkv,
                                int M, int d, int collapse, float scale, float* scores, cudaStream_t st,
                                const uint8_t* local, int kind, bool stats_bf16) {
    const int G = Hq / Hkv;
    const int chunks = (M + kTyChunk - 1) / kTyChunk;
    const int items = B * Hkv * chunks;
    const int grid = grid_for(items, 8);
#define SPA_TY_LAUNCH(D, GG, KD, SB)                                                                          \
    SPA_CUDA_TRY(launch_pdl(taylor_scores_kernel<D, GG, KD, SB>, dim3(grid), dim3(kTyThreads), 0, st, q, mean, var, \
                            Hq, Hkv, M, collapse, scale, scores, chunks, items, local))
#define SPA_TY_KIND(D, GG, SB)                                                                                \
    if (kind == SPA_SCORE_MINMAX_BLOCK) SPA_TY_LAUNCH(D, GG, KIND_MINMAX, SB);                                 \
    else if (kind == SPA_SCORE_MEAN_BLOCK) SPA_TY_LAUNCH(D, GG, KIND_MEAN, SB);                                \
    else SPA_TY_LAUNCH(D, GG, KIND_TAYLOR, SB);
#define SPA_TY_CASE(D, GG)                                                                                    \
    if (d == D && G == GG) {                                                                                 \
        if (stats_bf16) { SPA_TY_KIND(D, GG, true) } else { SPA_TY_KIND(D, GG, false) }                       \
        return SPA_OK;                                                                                       \
    }
    SPA_TY_CASE(64, 1) SPA_TY_CASE(64, 2) SPA_TY_CASE(64, 4) SPA_TY_CASE(64, 8) SPA_TY_CASE(64, 16)
    SPA_TY_CASE(128, 1) SPA_TY_CASE(128, 2) SPA_TY_CASE(128, 4) SPA_TY_CASE(128, 8) SPA_TY_CASE(128, 16)
#undef SPA_TY_CASE
#undef SPA_TY_KIND
#undef SPA_TY_LAUNCH
    return SPA_ERR_UNSUPPORTED_SHAPE;
}

spa_status launch_block_minmax(const uint16_t* K, int B, int Hkv, int N, int d, int block, void* mn, void* mx,
                               bool out_bf16, cudaStream_t st) {
    const int nb = N / block;
    const int n_blocks = B * Hkv * nb;
    if (n_blocks == 0) return SPA_OK;
    const int grid = grid_for(n_blocks, 16);
    const uint4* k4 = reinterpret_cast<const uint4*>(K);
#define SPA_MM_CASE(D, BL)                                                                              \
    if (d == D && block == BL) {                                                                       \
        if (out_bf16)                                                                                  \
            SPA_CUDA_TRY(launch_pdl(block_minmax_kernel<D, BL, true>, dim3(grid), dim3(128), 0, st, k4,  \
                                    n_blocks, nb, N, mn, mx));                                         \
        else                                                                                           \
            SPA_CUDA_TRY(launch_pdl(block_minmax_kernel<D, BL, false>, dim3(grid), dim3(128), 0, st, k4, \
                                    n_blocks, nb, N, mn, mx));                                         \
        return SPA_OK;                                                                                 \
    }
    SPA_MM_CASE(64, 32) SPA_MM_CASE(64, 64) SPA_MM_CASE(64, 128)
    SPA_MM_CASE(128, 32) SPA_MM_CASE(128, 64) SPA_MM_CASE(128, 128)
#undef SPA_MM_CASE
    return SPA_ERR_UNSUPPORTED_SHAPE;
}

spa_status launch_block_stats(const uint16_t* K, int B, int Hkv, int N, int d, int block, void* mean,
                              void* var, bool out_bf16, cudaStream_t st) {
    const int nb = N / block;
    const int n_blocks = B * Hkv * nb;
    if (n_blocks == 0) return SPA_OK;
    const int grid = grid_for(n_blocks, 16);
    const uint4* k4 = reinterpret_cast<const uint4*>(K);
#define SPA_BS_CASE(D, BL)                                                                              \
    if (d == D && block == BL) {                                                                       \
        if (out_bf16)                                                                                  \
            SPA_CUDA_TRY(launch_pdl(block_stats_kernel<D, BL, true>, dim3(grid), dim3(128), 0, st, k4,   \
                                    n_blocks, nb, N, mean, var));                                      \
        else                                                                                           \
            SPA_CUDA_TRY(launch_pdl(block_stats_kernel<D, BL, false>, dim3(grid), dim3(128), 0, st, k4,  \
                                    n_blocks, nb, N, mean, var));                                      \
        return SPA_OK;                                                                                 \
    }
    SPA_BS_CASE(64, 32) SPA_BS_CASE(64, 64) SPA_BS_CASE(64, 128)
    SPA_BS_CASE(128, 32) SPA_BS_CASE(128, 64) SPA_BS_CASE(128, 128)
#undef SPA_BS_CASE
    return SPA_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace spa
