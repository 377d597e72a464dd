// Exact top-k and sort-free histogram top-p selection with the forced sink and window.
//
// "Full Attention Strikes Back" (RTPurbo), Methodology 3 (dynamic top-p: accumulate
// mass until the cumulative threshold p) and 5 (sort-free histogram thresholding);
// "Oracle-Guided Sparse Prefill" 2.1 (top-k support); RTPurbo Methodology 1 (sink and
// sliding window kept).
//
// The scores are mapped to order-preserving 32-bit keys and the threshold key is found by
// a radix descent over the key bits in three levels (11, 11 and 10 bits):
//   level 0: a histogram of the top 11 bits, with counts and 64-bit fixed-point masses,
//            built while the scores are produced (fused scoring kernel) or by
//            hist0_kernel; every bin's masses are taken relative to the largest score the
//            bin can hold, so the sums are exact integers independent of thread order and
//            need no knowledge of the maximum.  The crossing bin B0 -- where the cumulative
//            count reaches k, or the cumulative mass (scaled to the unit's maximum, fp64,
//            fixed order) reaches p times the total -- is found by one block scan.
//   levels 1, 2: one thread-block cluster of C CTAs per unit.  Each CTA holds a contiguous
//            chunk of the unit's scores in shared memory (512 threads), or streams it from L2
//            on every level when it is too long for shared memory (1024 threads); only
//            elements of B0 are histogrammed (masses relative to the same bin reference, so
//            they sum exactly to the level-0 mass of B0).  The CTAs add their nonzero bins to
//            the unit's merged histogram in global memory with integer reductions (order-free),
//            meet at one cluster barrier and scan the merged bins from the top; a lone CTA
//            (C = 1) scans its own shared histogram.
// The result is the threshold key tau and the quota q of elements equal to tau, taken in
// ascending position.  Compaction walks each warp's slice of the chunk in ascending order
// (ballot + popc prefix) and packs the selected positions in place in shared memory; a
// block scan and a cluster-wide prefix of the CTA counts give every list its offset in the
// ascending support, and the lists are copied out coalesced.
#include <map>
#include <mutex>
#include <tuple>

#include <cooperative_groups.h>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace spa {
namespace {

// Threads per selection CTA: 512 when the chunk is resident in shared memory, 1024 when it is
// streamed from L2 on every level (twice the loads in flight; measured on B200 at 1M scores per
// unit in clusters of 16: 111 -> 86 us).  Resident chunks are faster with 512.
constexpr int kSelThreadsResident = 512;
constexpr int kSelThreadsStream = 1024;
constexpr int kMaxSelWarps = kSelThreadsStream / 32;
constexpr int kBins = 2048;
constexpr int kMaxCluster = 16;   // 16 is a non-portable cluster size, allowed on sm_100
constexpr double kInvMassScale = 1.0 / 1099511627776.0;   // 2^-40

using u64 = unsigned long long;

// A CTA's local histogram sums fixed-point masses (< 2^41) in three 14-bit parts with 32-bit
// shared atomics (a 64-bit shared atomic is several times slower); a part cannot overflow while
// the chunk holds at most kPartSafe scores, longer chunks use 64-bit sums (aliased storage).
constexpr int kPartSafe = 1 << 18;
constexpr uint32_t kLoadSpinLimit = 1u << 24;   // bounded polls of the chunk-load barrier
constexpr int kBulkPiece = 32768;               // bytes per bulk copy of the chunk load

struct SelShared {
    uint32_t hist_cnt[kBins];     // local histogram of the current level (levels 1 and 2)
    uint32_t hist_part[3][kBins];
    uint32_t warp_u32[kMaxSelWarps];
    u64 warp_u64[kMaxSelWarps];
    double warp_f64[kMaxSelWarps];
    uint32_t sel_of[kMaxCluster];   // selected count of every CTA of the cluster (pushed by each)
    double fmass_of[kMaxCluster];   // mass of every CTA's forced-only elements (pushed by each)
    u64 load_bar;                   // completion of the chunk's bulk copy
    uint32_t found_bin;
    uint32_t found_above_cnt;
    u64 found_above_mass;
    double found_above_f64;
    uint32_t found_cnt;
    Level0Shared l0;
};

// Block-wide exclusive scan of (a, b) in thread order over NW warps; totals returned too.
// Fixed order.
template <int NW, typename TB>
__device__ __forceinline__ void block_exscan(uint32_t a, TB b, uint32_t& ea, TB& eb, uint32_t& ta, TB& tb,
                                             uint32_t* wa_s, TB* wb_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t ia = a;
    TB ib = b;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t xa = __shfl_up_sync(0xffffffffu, ia, off);
        const TB xb = __shfl_up_sync(0xffffffffu, ib, off);
        if (lane >= off) { ia += xa; ib += xb; }
    }
    if (lane == 31) { wa_s[warp] = ia; wb_s[warp] = ib; }
    __syncthreads();
    uint32_t wa = 0, sa = 0;
    TB wb = 0, sb = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const uint32_t va = wa_s[w];
        const TB vb = wb_s[w];
        if (w < warp) { wa += va; wb += vb; }
        sa += va; sb += vb;
    }
    ea = wa + ia - a;
    eb = wb + ib - b;
    ta = sa;
    tb = sb;
    __syncthreads();
}

// ============================================================================ level-0 histogram
// One work item = (unit, chunk of 4096 scores); shared-memory bins flushed with integer
// atomics into the unit's histogram.  When rows are 16-byte aligned (M a multiple of 4) every
// thread issues its four float4 loads at once; the bins are cleared and scanned four at a time.
constexpr int kH0Threads = 256;
constexpr int kH0Chunk = 4096;

template <bool MASS>
__global__ void __launch_bounds__(kH0Threads)
hist0_kernel(SelectParams p, int chunks_per_unit, int n_items) {
    pdl_enter();
    __shared__ __align__(16) uint32_t h_cnt[kBins];
    __shared__ __align__(16) u64 h_mass[MASS ? kBins : 2];
    __shared__ uint32_t h_max;
    const bool vec = (p.M & 3) == 0 && (reinterpret_cast<uintptr_t>(p.scores) & 15) == 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int u = item / chunks_per_unit;
        const int chunk = item - u * chunks_per_unit;
        const int L = p.unit_len ? min(max(p.unit_len[u], 0), p.M) : p.M;
        const int n0 = chunk * kH0Chunk, n1 = min(L, n0 + kH0Chunk);
        if (n0 >= n1 || (p.local && p.local[u])) continue;   // local units are not selected from
        const uint4 z4 = make_uint4(0, 0, 0, 0);
        for (int i = threadIdx.x; i < kBins / 4; i += kH0Threads) {
            reinterpret_cast<uint4*>(h_cnt)[i] = z4;
            if (MASS) {
                reinterpret_cast<uint4*>(h_mass)[2 * i] = z4;
                reinterpret_cast<uint4*>(h_mass)[2 * i + 1] = z4;
            }
        }
        if (threadIdx.x == 0) h_max = 0;
        __syncthreads();
        uint32_t my_max = 0;
        const float* row = p.scores + size_t(u) * p.M;
        auto add = [&](float s) {
            const uint32_t key = score_key(s);
            const uint32_t bin = key >> 21;
            my_max = max(my_max, key);
            atomicAdd(&h_cnt[bin], 1u);
            if (MASS) atomicAdd(&h_mass[bin], fixed_mass(s, bin_top_score(bin)));
        };
        if (vec && n1 - n0 == kH0Chunk) {
            const float4* r4 = reinterpret_cast<const float4*>(row + n0);
            float4 v[kH0Chunk / 4 / kH0Threads];
#pragma unroll
            for (int j = 0; j < kH0Chunk / 4 / kH0Threads; ++j) v[j] = __ldg(r4 + threadIdx.x + j * kH0Threads);
#pragma unroll
            for (int j = 0; j < kH0Chunk / 4 / kH0Threads; ++j) {
                add(v[j].x);
                add(v[j].y);
                add(v[j].z);
                add(v[j].w);
            }
        } else {
            for (int n = n0 + threadIdx.x; n < n1; n += kH0Threads) add(__ldg(row + n));
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, off));
        if ((threadIdx.x & 31) == 0) atomicMax(&h_max, my_max);
        __syncthreads();
        for (int i4 = threadIdx.x; i4 < kBins / 4; i4 += kH0Threads) {   // four bins at a time
            const uint4 c4 = reinterpret_cast<const uint4*>(h_cnt)[i4];
            if ((c4.x | c4.y | c4.z | c4.w) == 0) continue;
            const uint32_t c[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (!c[j]) continue;
                atomicAdd(p.hist.cnt + size_t(u) * kBins + 4 * i4 + j, c[j]);
                if (MASS) atomicAdd(p.hist.mass + size_t(u) * kBins + 4 * i4 + j, h_mass[4 * i4 + j]);
            }
        }
        if (threadIdx.x == 0) atomicMax(p.hist.max_key + u, h_max);
        __syncthreads();
    }
}

// ============================================================================ selection
template <bool TOPP, int NT>
__global__ void __launch_bounds__(NT, 1024 / NT)
select_kernel(SelectParams p, int chunk, int resident_launch) {
    constexpr int kSelThreads = NT;
    constexpr int kSelWarps = NT / 32;
    constexpr int kPerMax = 2048 / NT;   // histogram bins per thread in a scan
    pdl_enter();
    cg::cluster_group cluster = cg::this_cluster();
    const int C = int(cluster.num_blocks());
    const int rank = int(cluster.block_rank());
    const bool solo = C == 1;
    const int u = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ __align__(16) uint8_t dyn[];
    SelShared& sh = *reinterpret_cast<SelShared*>(dyn);
    float* sv = reinterpret_cast<float*>(dyn + align_up(sizeof(SelShared), 16));   // resident chunk

    const int L = p.unit_len ? min(max(p.unit_len[u], 0), p.M) : p.M;
    const int lo = min(L, rank * chunk);
    const int hi = min(L, lo + chunk);
    const int n = hi - lo;
    const float* srow = p.scores + size_t(u) * p.M + lo;

    // ---- the chunk into shared memory: bulk asynchronous copies when the row slice is
    // 16-byte aligned (they run while the level-0 scan below executes), else plain loads
    const int n16 = (reinterpret_cast<uintptr_t>(srow) & 15) == 0 ? (n & ~3) : 0;
    const bool bulk = resident_launch && n16 > 0;
    // the test hook stalls the chunk load: the barrier expects bytes no copy delivers
    const bool stall = (p.test_stall & SPA_TEST_STALL_SELECT_LOAD) != 0;
    const uint32_t spin_limit = stall ? 1024u : kLoadSpinLimit;
    const uint32_t bar = uint32_t(__cvta_generic_to_shared(&sh.load_bar));
    if (bulk) {
        if (tid == 0) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(bar));
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // the init precedes the copies
            const uint32_t bytes = uint32_t(n16) * 4u;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
            const uint32_t dst = uint32_t(__cvta_generic_to_shared(sv));
            for (uint32_t off = 0; off < (stall ? 0u : bytes); off += kBulkPiece) {
                const uint32_t piece = min(uint32_t(kBulkPiece), bytes - off);
                asm volatile(
                    "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                        dst + off),
                    "l"(reinterpret_cast<const uint8_t*>(srow) + off), "r"(piece), "r"(bar)
                    : "memory");
            }
        }
        for (int j = n16 + tid; j < n; j += kSelThreads) sv[j] = __ldg(srow + j);
    } else if (resident_launch) {
        for (int j = tid; j < n; j += kSelThreads) sv[j] = __ldg(srow + j);
    }
    // bounded poll of the chunk-load barrier
    auto poll_chunk = [&](uint32_t limit) -> bool {
        uint32_t ok = 0;
        for (uint32_t it = 0; !ok; ++it) {
            asm volatile(
                "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n selp.u32 %0, 1, 0, q;\n}\n"
                : "=r"(ok)
                : "r"(bar)
                : "memory");
            if (!ok && it >= limit) return false;
        }
        return true;
    };
    // Once the chunk has arrived, every warp sees it (barrier).  If the bulk copy has not
    // landed within the bound, the CTA raises SPA_ERR_TIMEOUT and stops using its shared copy
    // of the chunk: it reads the scores from global memory instead (the streaming path), so
    // the result stays correct and nothing reads a half-written chunk.
    int resident = resident_launch;
    bool chunk_ok = true;
    auto wait_chunk = [&]() {
        const bool ok = !bulk || poll_chunk(spin_limit);
        chunk_ok = __syncthreads_and(ok ? 1 : 0) != 0;
        if (!chunk_ok) {
            if (tid == 0) raise_status(p.status, SPA_ERR_TIMEOUT);
            resident = 0;
        }
    };
    auto val_at = [&](int i) -> float { return resident ? sv[i] : __ldg(srow + i); };

    // a local unit (head-wise routing) keeps its sink and window only
    const bool local = p.local && p.local[u];
    bool select_all = false, select_none = local;
    if (!TOPP) {
        select_all = !local && p.topk >= L;
        select_none = local || p.topk <= 0;
    }
    const bool thresholded = L > 0 && !select_all && !select_none;

    // ---- level 0: crossing bin B0 from the unit's histogram (same result in every CTA)
    const uint32_t* hc = p.hist.cnt + size_t(u) * kBins;
    const u64* hm = p.hist.mass + size_t(u) * kBins;
    const uint32_t max_key = p.hist.max_key[u];
    const float m = key_score(max_key);
    double Z = 0.0, T = 0.0;
    uint32_t b0 = max_key >> 21, cum_cnt0 = 0;
    double cum_mass0 = 0.0;
    if (thresholded) {
        const Level0 l0 = level0_crossing(hc, hm, max_key, TOPP, p.topp, p.topk, sh.l0);
        b0 = l0.bin;
        cum_cnt0 = l0.above_cnt;
        cum_mass0 = l0.above_mass;
        if (TOPP) {
            Z = l0.Z;
            T = double(p.topp) * Z;
        }
    }
    const float r0 = bin_top_score(b0);                       // mass reference inside B0
    const double scale0 = TOPP ? kInvMassScale * exp(double(r0) - double(m)) : 0.0;
    // Thread 0 initialised the chunk barrier: level 0's block barriers order that before every
    // thread's first poll; a unit without level 0 (all or none selected) needs this one.
    if (bulk && !thresholded) __syncthreads();
    wait_chunk();

    // ---- levels 1 and 2 inside B0
    uint32_t tau = 0, q = 0, cnt_tau = 0, bin_last = 0;
    u64 cum_in = 0, E_tau = 0;          // mass above tau inside B0 (fixed point, relative to r0)
    if (thresholded) {
        uint32_t target_cnt = 0;
        u64 target_mass = 0;
        if (TOPP) {
            const double need = (T - cum_mass0) / (scale0 > 0.0 ? scale0 : 1.0);
            const u64 hb = __ldcg(hm + b0);
            u64 t = need <= 1.0 ? 1ull : (need >= double(hb) ? hb : u64(ceil(need)));
            target_mass = t < 1 ? 1 : t;
        } else {
            target_cnt = uint32_t(p.topk) - cum_cnt0;
        }
        uint32_t prefix = b0;
        uint32_t cum_c = 0;
        u64 cum_m = 0;
        for (int level = 1; level <= 2; ++level) {
            const int shift = level == 1 ? 10 : 0;
            const int nb = level == 1 ? 2048 : 1024;
            const int pshift = level == 1 ? 21 : 10;
            const bool wide = n > kPartSafe;
            u64* hist_wide = reinterpret_cast<u64*>(&sh.hist_part[0][0]);
            for (int i = tid; i < nb; i += kSelThreads) {
                sh.hist_cnt[i] = 0;
                if (TOPP) {
                    if (wide) {
                        hist_wide[i] = 0;
                    } else {
                        sh.hist_part[0][i] = 0;
                        sh.hist_part[1][i] = 0;
                        sh.hist_part[2][i] = 0;
                    }
                }
            }
            __syncthreads();
            auto add = [&](float s) {
                const uint32_t k = score_key(s);
                if ((k >> pshift) == prefix) {
                    const uint32_t bin = (k >> shift) & uint32_t(nb - 1);
                    atomicAdd(&sh.hist_cnt[bin], 1u);
                    if (TOPP) {
                        const u64 m = fixed_mass(s, r0);
                        if (wide) {
                            atomicAdd(&hist_wide[bin], m);
                        } else {
                            atomicAdd(&sh.hist_part[0][bin], uint32_t(m) & 0x3fffu);
                            atomicAdd(&sh.hist_part[1][bin], uint32_t(m >> 14) & 0x3fffu);
                            atomicAdd(&sh.hist_part[2][bin], uint32_t(m >> 28));
                        }
                    }
                }
            };
            if (resident) {
                const int n4 = n >> 2;
                const float4* v4 = reinterpret_cast<const float4*>(sv);
                for (int i = tid; i < n4; i += kSelThreads) {
                    const float4 v = v4[i];
                    add(v.x); add(v.y); add(v.z); add(v.w);
                }
                for (int i = (n4 << 2) + tid; i < n; i += kSelThreads) add(sv[i]);
            } else if ((reinterpret_cast<uintptr_t>(srow) & 15) == 0) {
                // streaming chunk (too long for shared memory): four float4 loads in flight
                const int n4 = n >> 2;
                const float4* s4 = reinterpret_cast<const float4*>(srow);
                int i = tid;
                for (; i + 3 * kSelThreads < n4; i += 4 * kSelThreads) {
                    float4 v[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] = __ldg(s4 + i + j * kSelThreads);
#pragma unroll
                    for (int j = 0; j < 4; ++j) { add(v[j].x); add(v[j].y); add(v[j].z); add(v[j].w); }
                }
                for (; i < n4; i += kSelThreads) {
                    const float4 v = __ldg(s4 + i);
                    add(v.x); add(v.y); add(v.z); add(v.w);
                }
                for (int j = (n4 << 2) + tid; j < n; j += kSelThreads) add(__ldg(srow + j));
            } else {
                for (int i = tid; i < n; i += kSelThreads) add(__ldg(srow + i));
            }
            __syncthreads();
            auto local_mass = [&](int i) -> u64 {
                return wide ? hist_wide[i]
                            : u64(sh.hist_part[0][i]) + (u64(sh.hist_part[1][i]) << 14) +
                                  (u64(sh.hist_part[2][i]) << 28);
            };
            // the unit's merged histogram.  A lone CTA's shared histogram already is the merged
            // one; in a cluster every CTA adds its nonzero bins with global reductions (integer
            // sums: the result does not depend on their order)
            const int goff = level == 1 ? 0 : kBins;
            uint32_t* gcnt = p.hist.lvl_cnt + size_t(u) * kLvlBins + goff;
            u64* gmass = p.hist.lvl_mass + size_t(u) * kLvlBins + goff;
            if (!solo) {
                for (int i = tid; i < nb; i += kSelThreads) {
                    const uint32_t c = sh.hist_cnt[i];
                    if (c) {
                        atomicAdd(gcnt + i, c);
                        if (TOPP) atomicAdd(gmass + i, local_mass(i));
                    }
                }
                cluster.sync();   // every CTA's reductions are performed (release / acquire at cluster scope)
            }

            const int per = nb / kSelThreads;    // bins per thread, descending
            uint32_t vc[kPerMax];
            u64 vm[kPerMax];
            uint32_t sc = 0;
            u64 sm = 0;
#pragma unroll
            for (int j = 0; j < kPerMax; ++j) {
                vc[j] = 0; vm[j] = 0;
                if (j < per) {
                    const int bin = nb - 1 - (tid * per + j);
                    if (solo) {
                        vc[j] = sh.hist_cnt[bin];
                        if (TOPP) vm[j] = local_mass(bin);
                    } else {
                        vc[j] = __ldcg(gcnt + bin);
                        if (TOPP) vm[j] = __ldcg(gmass + bin);
                    }
                    sc += vc[j];
                    sm += vm[j];
                }
            }
            uint32_t ec, tc;
            u64 em, tm;
            block_exscan<kSelWarps, u64>(sc, sm, ec, em, tc, tm, sh.warp_u32, sh.warp_u64);
            if (tid == 0) {   // defaults if rounding left no crossing: the last non-empty bin
                sh.found_bin = 0;
                sh.found_above_cnt = cum_c;
                sh.found_above_mass = cum_m;
                sh.found_cnt = 0;
            }
            __syncthreads();
            uint32_t ac = cum_c + ec;
            u64 am = cum_m + em;
#pragma unroll
            for (int j = 0; j < kPerMax; ++j) {
                if (j < per) {
                    const bool hit = TOPP ? (am < target_mass && am + vm[j] >= target_mass)
                                          : (ac < target_cnt && ac + vc[j] >= target_cnt);
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
            prefix = (prefix << (level == 1 ? 11 : 10)) | fb;
            cum_c = sh.found_above_cnt;
            cum_m = sh.found_above_mass;
            if (level == 2) {
                bin_last = fb;
                tau = prefix;
                cnt_tau = sh.found_cnt;
                cum_in = cum_m;
                if (TOPP) {
                    E_tau = fixed_mass(key_score(tau), r0);
                    const u64 need = target_mass > cum_m ? target_mass - cum_m : 0;
                    u64 qq = E_tau ? (need + E_tau - 1) / E_tau : u64(cnt_tau);
                    if (qq < 1) qq = 1;
                    if (qq > cnt_tau) qq = cnt_tau;
                    q = uint32_t(qq);
                } else {
                    q = target_cnt - cum_c;
                    if (q > cnt_tau) q = cnt_tau;
                }
            }
            __syncthreads();
        }
    }

    // ---- compaction: warp w owns [w*seg, w*seg + seg) of the chunk, walked in ascending order
    const int seg = ((n + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
    const int w0 = min(n, warp * seg), w1 = min(n, w0 + seg);
    const int window_lo = L - p.window;
    const unsigned lt_mask = (1u << lane) - 1u;
    // whether this warp's slice holds a forced position (sink or window)
    const bool fx_slice = w0 < w1 && (lo + w0 < p.sink || lo + w1 > window_lo);

    // ties before each warp are needed only when the quota splits the run of equal keys
    int64_t q_warp = int64_t(q);
    const bool split_ties = thresholded && q < cnt_tau;
    if (split_ties) {
        uint32_t before = 0;
        for (int r = 0; r < rank; ++r) before += *cluster.map_shared_rank(&sh.hist_cnt[bin_last], r);
        uint32_t wt = 0;
        for (int g0 = w0; g0 < w1; g0 += 256) {
            float vals[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = g0 + 32 * j + lane;
                vals[j] = i < w1 ? val_at(i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = g0 + 32 * j + lane;
                wt += __popc(__ballot_sync(0xffffffffu, i < w1 && score_key(vals[j]) == tau));
            }
        }
        if (lane == 0) sh.warp_u32[warp] = wt;
        __syncthreads();
        for (int w = 0; w < warp; ++w) before += sh.warp_u32[w];
        __syncthreads();
        q_warp = int64_t(q) - int64_t(before);
    }

    // one ascending walk: selected positions of warp w are packed at sv[w0 ...] in place
    // (resident chunk), or only counted (streaming chunk, written by a second walk)
    auto walk = [&](bool pack, bool write, uint32_t base, uint32_t& nsel, double& fmass) {
        uint32_t run_tie = 0;
        nsel = 0;
        fmass = 0.0;
        int* packed = reinterpret_cast<int*>(sv);
        constexpr int kAhead = 8;     // groups of 32 scores loaded ahead (streaming chunk)
        for (int g0 = w0; g0 < w1; g0 += 32 * kAhead) {
            float vals[kAhead];
#pragma unroll
            for (int j = 0; j < kAhead; ++j) {
                const int i = g0 + 32 * j + lane;
                vals[j] = i < w1 ? val_at(i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kAhead; ++j) {
                const int i0 = g0 + 32 * j;
                if (i0 >= w1) break;                      // warp-uniform
                const int i = i0 + lane;
                const bool live = i < w1;
                const float s = vals[j];
                const uint32_t k = score_key(s);
                const int pos = lo + i;
                bool top = false, tie = false;
                if (select_all) top = live;
                else if (thresholded) {
                    top = live && k > tau;
                    tie = live && k == tau;
                }
                const unsigned tb = __ballot_sync(0xffffffffu, tie);
                if (tie) top = !split_ties || int64_t(run_tie + __popc(tb & lt_mask)) < q_warp;
                run_tie += __popc(tb);
                const bool f = fx_slice && live && (pos < p.sink || pos >= window_lo);
                const bool sel = top || f;
                if (TOPP && __any_sync(0xffffffffu, f && !top) && f && !top) fmass += exp(double(s) - double(m));
                const unsigned sb = __ballot_sync(0xffffffffu, sel);
                if (sel) {
                    const uint32_t at = nsel + __popc(sb & lt_mask);
                    if (pack) packed[w0 + at] = pos;     // at <= i: never overtakes the reads
                    if (write && base + at < uint32_t(p.cap)) p.idx[size_t(u) * p.cap + base + at] = pos;
                }
                nsel += __popc(sb);
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) fmass += __shfl_xor_sync(0xffffffffu, fmass, off);
    };

    // common case: resident chunk and no tie split.  Lane l of a step owns the four
    // consecutive elements [4l, 4l + 4) of a 128-element run; a warp inclusive scan of the
    // per-lane counts gives the packed offsets (ascending order is lane-major).
    auto walk4 = [&](uint32_t& nsel_out, double& fmass_out) {
        uint32_t ns = 0;
        double fm = 0.0;
        int* packed = reinterpret_cast<int*>(sv);
        for (int i0 = w0; i0 < w1; i0 += 128) {
            const int i = i0 + 4 * lane;
            float v[4];
            if (i + 3 < w1) {
                const float4 t = *reinterpret_cast<const float4*>(sv + i);
                v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[j] = i + j < w1 ? sv[i + j] : 0.f;
            }
            uint32_t flags = 0, fx = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool live = i + j < w1;
                const int pos = lo + i + j;
                const bool top = live && (select_all || (thresholded && score_key(v[j]) >= tau));
                const bool f = fx_slice && live && (pos < p.sink || pos >= window_lo);
                fx |= uint32_t(f && !top) << j;
                flags |= uint32_t(top || f) << j;
            }
            if (TOPP && __any_sync(0xffffffffu, fx != 0)) {   // forced-only elements are few
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (fx >> j & 1u) fm += exp(double(v[j]) - double(m));
            }
            const uint32_t cnt = __popc(flags);
            uint32_t incl = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t x = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += x;
            }
            uint32_t at = ns + incl - cnt;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (flags >> j & 1u) packed[w0 + at++] = lo + i + j;   // never overtakes the reads
            ns += __shfl_sync(0xffffffffu, incl, 31);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) fm += __shfl_xor_sync(0xffffffffu, fm, off);
        nsel_out = ns;
        fmass_out = fm;
    };

    uint32_t nsel;
    double fmass;
    // the vector walk needs 16-byte aligned warp slices of the resident chunk
    const bool fast = resident && !split_ties && (seg % 4 == 0);
    if (fast) {
        __syncwarp();
        walk4(nsel, fmass);
    } else {
        walk(resident != 0, false, 0, nsel, fmass);
    }
    if (lane == 0) { sh.warp_u32[warp] = nsel; sh.warp_f64[warp] = fmass; }
    __syncthreads();
    uint32_t sel_before_warp = 0;
    for (int w = 0; w < warp; ++w) sel_before_warp += sh.warp_u32[w];
    if (tid < C) {   // this CTA's totals, pushed into every CTA of the cluster
        uint32_t t = 0;
        double fm = 0.0;
        for (int w = 0; w < kSelWarps; ++w) { t += sh.warp_u32[w]; fm += sh.warp_f64[w]; }
        SelShared& peer = *cluster.map_shared_rank(&sh, tid);
        peer.sel_of[rank] = t;
        peer.fmass_of[rank] = fm;
    }
    // the counts are in place; every CTA is past its reads of the histograms and of its peers'
    // shared memory, so after this barrier no CTA touches another's
    cluster.sync();
    uint32_t sel_before_cta = 0, total = 0;
    double fmass_total = 0.0;
    for (int r = 0; r < C; ++r) {
        const uint32_t c = sh.sel_of[r];
        if (r < rank) sel_before_cta += c;
        total += c;
        if (TOPP) fmass_total += sh.fmass_of[r];
    }
    const uint32_t base = sel_before_cta + sel_before_warp;
    if (resident) {
        const int* packed = reinterpret_cast<const int*>(sv);
        for (uint32_t j = lane; j < nsel; j += 32)
            if (base + j < uint32_t(p.cap)) p.idx[size_t(u) * p.cap + base + j] = packed[w0 + j];
    } else {
        walk(false, true, base, nsel, fmass);
    }

    // a chunk load that gave up: wait once more (bounded) so that a late copy lands before
    // the CTA exits (a copy still in flight after that bound is the one hazard left)
    if (!chunk_ok && bulk) poll_chunk(spin_limit);
    if (rank == 0) {
        // the unit's level-0 histogram is consumed: clear it for the next producer
        for (int i = tid; i < kBins; i += kSelThreads) {
            p.hist.cnt[size_t(u) * kBins + i] = 0;
            p.hist.mass[size_t(u) * kBins + i] = 0;
        }
        // (a lone CTA never wrote the level 1 and 2 bins)
        if (!solo) {
            for (int i = tid; i < kLvlBins; i += kSelThreads) {
                p.hist.lvl_cnt[size_t(u) * kLvlBins + i] = 0;
                p.hist.lvl_mass[size_t(u) * kLvlBins + i] = 0;
            }
        }
        if (tid == 0) {
            p.hist.max_key[u] = 0;
            p.count[u] = int32_t(total);
            if (total > uint32_t(p.cap)) raise_status(p.status, SPA_ERR_CAPACITY);
            if (TOPP && p.index_mass) {
                double top = 0.0;
                if (thresholded) top = cum_mass0 + double(cum_in + u64(q) * E_tau) * scale0;
                p.index_mass[u] = Z > 0.0 ? float((top + fmass_total) / Z) : 0.f;
            }
        }
    }
    // no barrier here: after the count barrier no CTA reads or writes another's shared memory
}

struct SelectConfig {
    int C;
    int chunk;
    int resident;
    size_t smem;
    int nt;   // threads per CTA
};

template <bool TOPP, int NT>
int max_active_clusters(int C, size_t smem) {
    // cached per (device, C, smem bucket)
    static thread_local int cache_dev = -1;
    static thread_local int cache[kMaxCluster + 1][4];
    const DeviceInfo& di = device_info();
    if (cache_dev != di.device) {
        for (auto& row : cache)
            for (int& v : row) v = -1;
        cache_dev = di.device;
    }
    const int bucket = smem <= 48 * 1024 ? 0 : (smem <= 113 * 1024 ? 1 : (smem <= 160 * 1024 ? 2 : 3));
    int& v = cache[C][bucket];
    if (v < 0) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(C, 1, 1);
        cfg.blockDim = dim3(NT, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, select_kernel<TOPP, NT>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        v = n;
    }
    return v;
}

// Cluster size C for U units of M scores.  A configuration runs ceil(U / concurrent units)
// waves of CTAs that each scan M / C scores plus a fixed cost (level-0 resolution, barriers,
// histogram merges) worth about kSelFixed scores; a chunk too long for shared memory streams
// from L2 on every level (kSelStreamCost per score).  The cheapest estimate wins, ties to the
// larger cluster; C > 1 needs at least 2048 scores per CTA.  kSelFixed was fitted on B200 to the
// selection of 512 units of about 30K scores timed with clusters of 2, 4 and 8 (90, 136 and 230
// us); when every unit's cluster fits in one wave the choice is the largest C.
constexpr double kSelFixed = 40960.0;
constexpr double kSelStreamCost = 3.0;
template <bool TOPP>
using SelectKernel = void (*)(SelectParams, int, int);

template <bool TOPP>
SelectKernel<TOPP> select_kernel_for(int nt) {
    return nt == kSelThreadsStream ? select_kernel<TOPP, kSelThreadsStream> : select_kernel<TOPP, kSelThreadsResident>;
}

template <bool TOPP>
SelectConfig choose(int U, int M) {
    // memoised per (device, U, M): the choice depends on nothing else
    static std::mutex memo_mu;
    static std::map<std::tuple<int, int, int>, SelectConfig> memo;
    const DeviceInfo& di = device_info();
    const std::tuple<int, int, int> key{di.device, U, M};
    {
        std::lock_guard<std::mutex> lk(memo_mu);
        auto it = memo.find(key);
        if (it != memo.end()) return it->second;
    }
    const size_t fixed = align_up(sizeof(SelShared), 16);
    SelectConfig best{};
    best.C = 0;
    double best_cost = 0.0;
    for (int C = kMaxCluster; C >= 1; C /= 2) {
        if (C > 1 && (M + C - 1) / C < 2048) continue;
        const int chunk = ((M + C - 1) / C + 3) / 4 * 4;
        size_t smem = fixed + size_t(chunk) * 4;
        int resident = 1;
        if (smem > size_t(di.max_smem_optin)) {
            resident = 0;
            smem = fixed;
        }
        const int nt = resident ? kSelThreadsResident : kSelThreadsStream;
        const SelectKernel<TOPP> kern = select_kernel_for<TOPP>(nt);
        set_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        set_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        int active = 0;   // units whose CTAs run at once
        if (C > 1) {
            active = resident ? max_active_clusters<TOPP, kSelThreadsResident>(C, smem)
                              : max_active_clusters<TOPP, kSelThreadsStream>(C, smem);
        } else {
            int per_sm = occupancy_blocks(reinterpret_cast<const void*>(kern), nt, smem);
            if (per_sm <= 0) per_sm = 1;
            active = per_sm * di.num_sms;
        }
        if (active <= 0) continue;
        const double waves = double((U + active - 1) / active);
        const double cost = waves * (double(chunk) * (resident ? 1.0 : kSelStreamCost) + kSelFixed);
        if (best.C == 0 || cost < best_cost) {
            best = SelectConfig{C, chunk, resident, smem, nt};
            best_cost = cost;
        }
    }
    if (best.C == 0) best = SelectConfig{1, M, 0, fixed, kSelThreadsStream};
    std::lock_guard<std::mutex> lk(memo_mu);
    if (memo.size() > 4096) memo.clear();
    memo[key] = best;
    return best;
}

template <bool TOPP>
spa_status launch_t(const SelectParams& p0, cudaStream_t st) {
    SelectParams p = p0;
    p.test_stall = test_stall_bits();
    const SelectConfig c = choose<TOPP>(p.U, p.M);
    const SelectKernel<TOPP> kern = select_kernel_for<TOPP>(c.nt);
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(c.smem)));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(c.C, p.U, 1);
    cfg.blockDim = dim3(c.nt, 1, 1);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_enter()
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    SPA_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, p, c.chunk, c.resident));
    return SPA_OK;
}

}  // namespace

size_t select_scratch_bytes(int U) { return hist0_bytes(U); }

spa_status launch_hist0(const SelectParams& p, bool with_mass, cudaStream_t st) {
    const int chunks = (p.M + kH0Chunk - 1) / kH0Chunk;
    const int items = p.U * chunks;
    if (items == 0) return SPA_OK;
    const int cap = device_info().num_sms * 8;
    const int grid = items < cap ? items : cap;
    if (with_mass) SPA_CUDA_TRY(launch_pdl(hist0_kernel<true>, dim3(grid), dim3(kH0Threads), 0, st, p, chunks, items));
    else SPA_CUDA_TRY(launch_pdl(hist0_kernel<false>, dim3(grid), dim3(kH0Threads), 0, st, p, chunks, items));
    return SPA_OK;
}

spa_status launch_select(const SelectParams& p, bool topp, cudaStream_t st) {
    return topp ? launch_t<true>(p, st) : launch_t<false>(p, st);
}

}  // namespace spa
