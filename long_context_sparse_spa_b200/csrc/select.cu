// Exact top-k and sort-free histogram top-p selection with the forced sink and window.
//
// "Full Attention Strikes Back" (RTPurbo), Methodology 3 (dynamic top-p: accumulate
// mass until the cumulative threshold p) and 5 (sort-free histogram thresholding);
// "Oracle-Guided Sparse Prefill" 2.1 (top-k support); RTPurbo Methodology 1 (sink and
// sliding window kept).
//
// One thread-block cluster of C CTAs selects one unit's support.  Each CTA owns a
// contiguous chunk of the unit's scores, converted to order-preserving 32-bit keys and
// held in shared memory when they fit (re-read from global/L2 otherwise).  The
// threshold key is found by three radix-histogram levels over the key bits (11, 11 and
// 10 bits):
//   1. every CTA histograms (count, mass) of its elements that match the prefix so far;
//   2. each CTA sums the peers' histograms for the bins it owns (distributed shared
//      memory, fixed peer order);
//   3. every CTA reads the merged bins and scans them from the top, finding the bin
//      where the cumulative count (top-k) or mass (top-p) reaches the target.
// After the last level the threshold key tau and the quota q of elements equal to tau
// (taken by ascending position) are exact.  Compaction then walks the chunk in
// ascending order per warp (ballot + popc prefix sums) and writes the support in
// ascending order at offsets from a cluster-wide prefix of the CTA counts.
//
// Top-p masses are e_n = exp(s_n - m) scaled by 2^40 and rounded to 64-bit integers,
// so every sum is exact and independent of thread order; the cut is the shortest
// prefix with sum >= ceil(p * Z).
#include <cooperative_groups.h>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace spa {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxCluster = 8;
constexpr float kMassScale = 1099511627776.0f;   // 2^40

using u64 = unsigned long long;

struct SelShared {
    uint32_t hist_cnt[kBins];     // local histogram of the current level
    u64 hist_mass[kBins];
    uint32_t mrg_cnt[kBins];      // merged histogram of the bins this CTA owns
    u64 mrg_mass[kBins];
    uint32_t warp_u32[kSelWarps];
    u64 warp_u64[kSelWarps];
    uint32_t cta_max_key;         // published to peers
    uint32_t cta_sel;             // selected count of this CTA (published)
    u64 cta_fmass;                // mass of forced-only elements (published)
    // result of a level scan
    uint32_t found_bin;
    uint32_t found_above_cnt;
    u64 found_above_mass;
    uint32_t found_cnt;
    u64 total_mass;
};

__device__ __forceinline__ u64 mass_of(uint32_t key, float m) {
    return __float2ull_rn(expf(key_score(key) - m) * kMassScale);
}

// Block-wide exclusive scan of (a, b) in thread order; returns the exclusive prefix and
// writes the block totals.
__device__ __forceinline__ void block_exscan(uint32_t a, u64 b, uint32_t& ea, u64& eb, uint32_t& ta, u64& tb,
                                             SelShared& sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t ia = a;
    u64 ib = b;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t xa = __shfl_up_sync(0xffffffffu, ia, off);
        const u64 xb = __shfl_up_sync(0xffffffffu, ib, off);
        if (lane >= off) { ia += xa; ib += xb; }
    }
    if (lane == 31) { sh.warp_u32[warp] = ia; sh.warp_u64[warp] = ib; }
    __syncthreads();
    uint32_t wa = 0, sa = 0;
    u64 wb = 0, sb = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        const uint32_t va = sh.warp_u32[w];
        const u64 vb = sh.warp_u64[w];
        if (w < warp) { wa += va; wb += vb; }
        sa += va; sb += vb;
    }
    ea = wa + ia - a;
    eb = wb + ib - b;
    ta = sa;
    tb = sb;
    __syncthreads();   // warp_* may be reused by the caller's next scan
}

template <bool TOPP>
__global__ void __launch_bounds__(kSelThreads, 1)
select_kernel(SelectParams p, int chunk, int resident) {
    cg::cluster_group cluster = cg::this_cluster();
    const int C = int(cluster.num_blocks());
    const int rank = int(cluster.block_rank());
    const int u = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ __align__(16) uint8_t dyn[];
    SelShared& sh = *reinterpret_cast<SelShared*>(dyn);
    uint32_t* keys = reinterpret_cast<uint32_t*>(dyn + align_up(sizeof(SelShared), 16));

    const int L = p.unit_len ? min(max(p.unit_len[u], 0), p.M) : p.M;
    const int lo = min(L, rank * chunk);
    const int hi = min(L, lo + chunk);
    const int n = hi - lo;
    const float* srow = p.scores + size_t(u) * p.M + lo;

    auto key_at = [&](int i) -> uint32_t { return resident ? keys[i] : score_key(__ldg(srow + i)); };

    // ---- keys into shared memory, local maximum
    uint32_t kmax = 0;
    for (int i = tid; i < n; i += kSelThreads) {
        const uint32_t k = score_key(__ldg(srow + i));
        if (resident) keys[i] = k;
        kmax = max(kmax, k);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    if (lane == 0) sh.warp_u32[warp] = kmax;
    __syncthreads();
    if (tid == 0) {
        uint32_t m = 0;
        for (int w = 0; w < kSelWarps; ++w) m = max(m, sh.warp_u32[w]);
        sh.cta_max_key = m;
    }

    // ---- mode
    // select_all: every position is selected (top-k with k >= L).
    // select_none: only forced positions (top-k with k <= 0).
    bool select_all = false, select_none = false;
    if (!TOPP) {
        select_all = p.topk >= L;
        select_none = p.topk <= 0;
    }
    cluster.sync();   // cta_max_key visible; keys resident

    float m = 0.f;
    if (TOPP) {
        uint32_t gmax = 0;
        for (int r = 0; r < C; ++r) gmax = max(gmax, *cluster.map_shared_rank(&sh.cta_max_key, r));
        m = key_score(gmax);
    }

    uint32_t tau = 0, q = 0;              // threshold key, tie quota
    uint32_t bin_last = 0;                // level-3 bin of tau (its local count = ties here)
    u64 Z = 0, T = 0, cum_mass = 0, E_tau = 0;
    uint32_t cum_cnt = 0;
    const bool thresholded = L > 0 && !select_all && !select_none;

    if (thresholded) {
        uint32_t prefix = 0;
        for (int level = 0; level < 3; ++level) {
            const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
            const int nb = level == 2 ? 1024 : 2048;
            const int pshift = shift + (level == 2 ? 10 : 11);   // bits above this level
            for (int i = tid; i < nb; i += kSelThreads) {
                sh.hist_cnt[i] = 0;
                if (TOPP) sh.hist_mass[i] = 0;
            }
            __syncthreads();
            for (int i = tid; i < n; i += kSelThreads) {
                const uint32_t k = key_at(i);
                if (level == 0 || (k >> pshift) == prefix) {
                    const uint32_t bin = (k >> shift) & uint32_t(nb - 1);
                    atomicAdd(&sh.hist_cnt[bin], 1u);
                    if (TOPP) atomicAdd(&sh.hist_mass[bin], mass_of(k, m));
                }
            }
            cluster.sync();   // local histograms complete
            const int per_owner = nb / C;
            for (int bin = rank * per_owner + tid; bin < (rank + 1) * per_owner; bin += kSelThreads) {
                uint32_t c = 0;
                u64 ms = 0;
                for (int r = 0; r < C; ++r) {
                    c += *cluster.map_shared_rank(&sh.hist_cnt[bin], r);
                    if (TOPP) ms += *cluster.map_shared_rank(&sh.hist_mass[bin], r);
                }
                sh.mrg_cnt[bin] = c;
                if (TOPP) sh.mrg_mass[bin] = ms;
            }
            cluster.sync();   // merged slices complete

            // scan the merged bins from the top (thread t owns descending positions)
            const int per = nb / kSelThreads;
            uint32_t vc[4];
            u64 vm[4];
            uint32_t sc = 0;
            u64 sm = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                vc[j] = 0; vm[j] = 0;
                if (j < per) {
                    const int bin = nb - 1 - (tid * per + j);
                    const int owner = bin / per_owner;
                    vc[j] = *cluster.map_shared_rank(&sh.mrg_cnt[bin], owner);
                    if (TOPP) vm[j] = *cluster.map_shared_rank(&sh.mrg_mass[bin], owner);
                    sc += vc[j];
                    sm += vm[j];
                }
            }
            uint32_t ec, tc;
            u64 em, tm;
            block_exscan(sc, sm, ec, em, tc, tm, sh);
            if (level == 0 && TOPP) {
                Z = tm;
                const double t = ceil(double(p.topp) * double(Z));
                T = t >= double(Z) ? Z : (t < 1.0 ? 1ull : u64(t));
            }
            uint32_t ac = cum_cnt + ec;
            u64 am = cum_mass + em;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j < per) {
                    bool hit;
                    if (TOPP) hit = am < T && am + vm[j] >= T;
                    else hit = ac < uint32_t(p.topk) && ac + vc[j] >= uint32_t(p.topk);
                    if (hit) {
                        sh.found_bin = uint32_t(nb - 1 - (tid * per + j));
                        sh.found_above_cnt = ac;
                        sh.found_above_mass = am;
                        sh.found_cnt = vc[j];
                    }
                    ac += vc[j];
                    am += vm[j];
                }
            }
            __syncthreads();
            const uint32_t fb = sh.found_bin;
            prefix = (prefix << (level == 2 ? 10 : 11)) | fb;
            cum_cnt = sh.found_above_cnt;
            cum_mass = sh.found_above_mass;
            if (level == 2) {
                bin_last = fb;
                tau = prefix;
                const uint32_t cnt_tau = sh.found_cnt;
                if (TOPP) {
                    E_tau = mass_of(tau, m);
                    const u64 need = T - cum_mass;
                    u64 qq = E_tau ? (need + E_tau - 1) / E_tau : u64(cnt_tau);
                    if (qq < 1) qq = 1;
                    if (qq > cnt_tau) qq = cnt_tau;
                    q = uint32_t(qq);
                } else {
                    q = uint32_t(p.topk) - cum_cnt;
                }
            }
            __syncthreads();   // found_* may be rewritten by the next level
        }
    }

    // ---- ties before this CTA (each CTA's level-3 local count of tau, peers in order)
    uint32_t ties_before_cta = 0;
    if (thresholded)
        for (int r = 0; r < rank; ++r) ties_before_cta += *cluster.map_shared_rank(&sh.hist_cnt[bin_last], r);

    // ---- compaction: warp w walks [w*seg, w*seg+seg) of the chunk in ascending order
    const int seg = ((n + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
    const int w0 = min(n, warp * seg), w1 = min(n, w0 + seg);
    const int window_lo = L - p.window;
    auto forced = [&](int pos) { return pos < p.sink || pos >= window_lo; };

    // pass 1: ties per warp -> ties before each warp
    uint32_t wties = 0;
    if (thresholded)
        for (int i0 = w0; i0 < w1; i0 += 32) {
            const int i = i0 + lane;
            const bool tie = i < w1 && key_at(i) == tau;
            wties += __popc(__ballot_sync(0xffffffffu, tie));
        }
    if (lane == 0) sh.warp_u32[warp] = wties;
    __syncthreads();
    uint32_t ties_before = ties_before_cta;
    for (int w = 0; w < warp; ++w) ties_before += sh.warp_u32[w];
    __syncthreads();
    const int64_t q_warp = int64_t(q) - int64_t(ties_before);

    const unsigned lt_mask = (1u << lane) - 1u;
    auto walk = [&](bool write, uint32_t base, uint32_t& nsel, u64& fmass) {
        uint32_t run_tie = 0;
        nsel = 0;
        fmass = 0;
        for (int i0 = w0; i0 < w1; i0 += 32) {
            const int i = i0 + lane;
            const bool live = i < w1;
            const uint32_t k = live ? key_at(i) : 0u;
            const int pos = lo + i;
            bool top = false, tie = false;
            if (select_all) top = live;
            else if (thresholded) {
                top = live && k > tau;
                tie = live && k == tau;
            }
            const unsigned tb = __ballot_sync(0xffffffffu, tie);
            if (tie) top = int64_t(run_tie + __popc(tb & lt_mask)) < q_warp;
            run_tie += __popc(tb);
            const bool f = live && forced(pos);
            const bool sel = top || f;
            if (TOPP && f && !top) fmass += mass_of(k, m);
            const unsigned sb = __ballot_sync(0xffffffffu, sel);
            if (write && sel) {
                const uint32_t at = base + nsel + __popc(sb & lt_mask);
                if (at < uint32_t(p.cap)) p.idx[size_t(u) * p.cap + at] = pos;
            }
            nsel += __popc(sb);
        }
    };

    // pass 2: counts per warp
    uint32_t nsel;
    u64 fmass;
    walk(false, 0, nsel, fmass);
    if (TOPP) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) fmass += __shfl_xor_sync(0xffffffffu, fmass, off);
    }
    if (lane == 0) { sh.warp_u32[warp] = nsel; sh.warp_u64[warp] = fmass; }
    __syncthreads();
    uint32_t sel_before_warp = 0;
    for (int w = 0; w < warp; ++w) sel_before_warp += sh.warp_u32[w];
    if (tid == 0) {
        uint32_t t = 0;
        u64 fm = 0;
        for (int w = 0; w < kSelWarps; ++w) { t += sh.warp_u32[w]; fm += sh.warp_u64[w]; }
        sh.cta_sel = t;
        sh.cta_fmass = fm;
    }
    cluster.sync();   // CTA counts visible to peers
    uint32_t sel_before_cta = 0, total = 0;
    u64 fmass_total = 0;
    for (int r = 0; r < C; ++r) {
        const uint32_t c = *cluster.map_shared_rank(&sh.cta_sel, r);
        if (r < rank) sel_before_cta += c;
        total += c;
        if (TOPP) fmass_total += *cluster.map_shared_rank(&sh.cta_fmass, r);
    }

    // pass 3: write
    walk(true, sel_before_cta + sel_before_warp, nsel, fmass);

    if (rank == 0 && tid == 0) {
        p.count[u] = int32_t(total);
        if (total > uint32_t(p.cap)) raise_status(p.status, SPA_ERR_CAPACITY);
        if (TOPP && p.index_mass) {
            const u64 top_mass = thresholded ? cum_mass + u64(q) * E_tau : 0ull;
            p.index_mass[u] = Z ? float(double(top_mass + fmass_total) / double(Z)) : 0.f;
        }
    }
    cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

struct SelectConfig {
    int C;
    int chunk;
    int resident;
    size_t smem;
};

SelectConfig choose(int U, int M) {
    const DeviceInfo& di = device_info();
    SelectConfig c{};
    int C = 1;
    while (C < kMaxCluster && U * C < di.num_sms) C *= 2;
    while (C > 1 && (M + C - 1) / C < 1024) C /= 2;
    c.C = C;
    c.chunk = (M + C - 1) / C;
    const size_t fixed = align_up(sizeof(SelShared), 16);
    const size_t budget = size_t(di.max_smem_optin) - fixed;
    c.resident = size_t(c.chunk) * 4 <= budget;
    c.smem = fixed + (c.resident ? size_t(c.chunk) * 4 : 0);
    return c;
}

template <bool TOPP>
spa_status launch_t(const SelectParams& p, cudaStream_t st) {
    const SelectConfig c = choose(p.U, p.M);
    static_assert(kBins % (kMaxCluster * 1) == 0, "bins split across the cluster");
    SPA_CUDA_TRY(cudaFuncSetAttribute(select_kernel<TOPP>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(c.smem)));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(c.C, p.U, 1);
    cfg.blockDim = dim3(kSelThreads, 1, 1);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SPA_CUDA_TRY(cudaLaunchKernelEx(&cfg, select_kernel<TOPP>, p, c.chunk, c.resident));
    return SPA_OK;
}

}  // namespace

spa_status launch_select(const SelectParams& p, bool topp, cudaStream_t st) {
    return topp ? launch_t<true>(p, st) : launch_t<false>(p, st);
}

}  // namespace spa
