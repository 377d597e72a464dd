// Fused decode step as one persistent dataflow kernel: low-rank index scores, exact top-p /
// top-k threshold selection with the sink and window, compaction, and exact attention on the
// gathered rows, for head-collapsed units (one support per kv head, G <= 8 query heads,
// d = 128), followed by a small log-sum-exp combine kernel.
//
// "Full Attention Strikes Back" (RTPurbo), Methodology 2 (r = 16 index keys), 3 (dynamic
// top-p), 5 (sort-free histogram threshold, bandwidth-optimised sparse decode);
// "Oracle-Guided Sparse Prefill" 2.1 (exact attention recomputed on the support) and 2.2
// (head-collapsed indexer); RTPurbo Methodology 1 (sink and local window kept).
//
// Why one kernel.  The step moves two HBM streams -- every index key once, then the selected
// K/V rows -- and between them sits the selection, which moves almost no bytes but is a chain
// of dependent steps.  Run as separate kernels the chain leaves HBM idle; here every unit
// (sequence, kv head) advances through its own chain while other units stream:
//
//   S  (unit, 2048 keys)  scores into the workspace and the level-0 histogram (counts and
//                         fixed-point masses of the top 11 key bits); the CTA that finishes
//                         a unit's last S task resolves level 0 (the crossing bin B0);
//   C  (unit, 8192 pos.)  counts the positions above B0 and appends the members of B0 to the
//                         unit's candidate list; the CTA that finishes the last C task
//                         resolves levels 1 and 2 on the candidates (threshold key tau, the
//                         quota of ties at tau, the position cut that takes those ties in
//                         ascending order), the per-range support counts and offsets, the
//                         support size and the index mass;
//   K  (unit, 8192 pos.)  writes the range's support positions, ascending, at its offset; the
//                         CTA that finishes the last K task publishes the unit for gathering;
//   G  (unit, 128 rows)   gathers 16 support rows per warp and runs the exact online-softmax
//                         attention of the unit's G query heads on tensor cores.
//
// S, C and K tasks are claimed from one queue in a fixed, unit-staggered order (the C and K
// tasks of a unit come a few units of S tasks after its own S tasks, so their inputs are
// normally complete when they are claimed); G chunks are claimed per published unit.  Every
// wait is on a task claimed earlier by a running CTA, so the kernel cannot deadlock even when
// not all CTAs are resident; every wait is also bounded: on expiry the kernel raises
// SPA_ERR_TIMEOUT, sets an abort flag and every CTA returns.  Half the CTAs prefer queue
// tasks, half prefer gather chunks, so the selection chains progress while the gathers run.
//
// Selection arithmetic is that of the cluster selection kernel (select.cu): order-preserving
// 32-bit keys, three radix levels of 11, 11 and 10 bits, exact 64-bit fixed-point masses
// (2^40 scale, relative to the largest score of B0), ties at tau taken in ascending position.
//
// Attention per 16-row tile (mma.sync m16n8k16, bf16 in, fp32 accumulate), transposed so the
// keys fill the 16-row side: S^T = K Q^T with K loaded straight from global memory into the
// A-fragment registers (each lane reads 64 contiguous bytes of its two rows per load; the
// head dimension is permuted consistently in K and Q), online softmax per head, P^T moved to
// the B layout with movmatrix, O^T += V^T P^T with V staged by cp.async in a two-stage
// per-warp ring and read with transposing ldmatrix.  P is carried as bf16 hi + lo.  A CTA
// accumulates every chunk it takes of a unit and, when the unit is exhausted, merges its
// warps and appends one (o, m, l) record per head; the combine kernel merges the records.
// Partial sums are therefore taken in the order the chunks were claimed: the output can
// differ from run to run in the last bits of fp32 (the support cannot).
#include "internal.cuh"
#include "warp_mma.cuh"

namespace spa {
namespace {

constexpr int kFThreads = 256;
constexpr int kFWarps = kFThreads / 32;
constexpr int kD = 128;                 // head dim
constexpr int kSRows = 2048;            // keys per S task
constexpr int kRRows = 8192;            // positions per C / K task
constexpr int kCandSmem = 8192;         // candidates held in shared memory by the level-1/2 pass
constexpr int kBins = kHistBins;        // 2048
constexpr uint32_t kWaitLimit = 1u << 21;   // polls (about 0.1-0.3 s) before a wait gives up
constexpr double kInvMass = 1.0 / 1099511627776.0;   // 2^-40
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

enum : uint32_t { MODE_THRESH = 0, MODE_ALL = 1, MODE_NONE = 2 };
enum : int { T_NONE = 0, T_S = 1, T_C = 2, T_K = 3, T_G = 4, T_DONE = 5 };

using u64 = unsigned long long;

struct __align__(16) FCounters {
    uint32_t s_head;       // next S task (unit-major order)
    uint32_t exit_count;
    uint32_t abort;
    uint32_t pub[3];       // units published to the C, K and G stages
};

// per-unit state; counters are reset by the last CTA to leave the fused kernel (nrec and
// comb_done by the combine kernel, which reads the records)
struct __align__(128) FUnit {
    uint32_t s_done;
    uint32_t next[3];      // claim cursors: C and K ranges, G tiles
    uint32_t done[2];      // finished C and K ranges
    uint32_t cand_n;
    uint32_t ntiles;       // 16-row gather tiles of the support (capped at cap rows)
    uint32_t nrec, comb_done;
    // level 0
    uint32_t mode, b0, cum_cnt0, max_key;
    uint32_t target_cnt;
    u64 target_mass;
    double cum_mass0, Z, scale0;
    // levels 1-2
    uint32_t tau, tie_cut, total;
};

struct FusedParams {
    const uint16_t* qidx;   // [B, Hq, 16]
    const uint4* kidx;      // [B, Hkv, N, 16] as 16-byte halves
    const uint16_t* q;      // [B, Hq, d]
    const uint16_t* K;      // [B, Hkv, N, d]
    const uint16_t* V;
    int B, Hq, Hkv, N, G;
    float score_scale, sm_scale;
    int topp_mode, topk;
    float topp;
    int sink, window;
    int32_t* idx;
    int32_t* count;
    int cap;
    float* index_mass;
    uint16_t* out;
    float* out_f32;
    float* lse;
    uint32_t* status;
    // workspace
    FCounters* ctr;
    FUnit* unit;            // [U]
    uint32_t* order;        // [3][U]: unit published in each slot of the C, K and G stages
    uint32_t* ready;        // [3][U]: slot filled
    uint32_t* rng_above;    // [U][NR]
    uint32_t* rng_off;      // [U][NR + 1]
    float* scores;          // [U][N]
    Hist0 hist;             // level-0 histograms
    uint2* cand;            // [U][N] (position, score bits)
    float* rec;             // [U][G][n_ctas][d + 2]
    int U, nS, NR, n_ctas;
    int n_sel;              // CTAs that run S, C and K tasks only (never gather)
    int M;                  // scores per unit (N for token scores, N / block for block scores)
    const uint8_t* local;   // [U] or null: local units (head-wise routing) keep sink + window only
};

// ---------------------------------------------------------------- memory-order helpers
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

// a unit enters the next stage of its chain (C = 0, K = 1, G = 2): its slot is taken, the
// unit written, then the slot released
__device__ __forceinline__ void publish(const FusedParams& p, int stage, int u) {
    const uint32_t slot = atomicAdd(&p.ctr->pub[stage], 1u);
    p.order[stage * p.U + slot] = uint32_t(u);
    __threadfence();
    st_release(p.ready + stage * p.U + slot, 1u);
}

// ---------------------------------------------------------------- shared memory
struct FShared {
    uint32_t wu32[kFWarps];
    double wf64[kFWarps];
    u64 wu64[kFWarps];
    uint32_t rsel[1024];               // per-range support counts of one unit (levels 1-2 pass)
    int task, tu, tc;                  // broadcast of the claimed task
    int flag, gslot;
    uint32_t found_bin, found_above_cnt, found_cnt;
    u64 found_above_mass;
    double found_above_f64;
    uint32_t vmask[kFWarps][2];
    Level0Shared l0;
    // last, so kernels that need none of it can allocate only the fields above; 128-byte
    // aligned (cp.async and ldmatrix need 16-byte aligned rows)
    union alignas(128) {
        struct {                       // S task: level-0 histogram of the task's keys
            uint32_t cnt[kBins];
            uint32_t mhi[kBins];
            uint32_t mlo[kBins];
        } s;
        struct {                       // levels 1-2: local histograms and the candidates
            uint32_t cnt[kBins];
            uint32_t part[3][kBins];
            uint2 cand[kCandSmem];
        } d;
        struct {                       // K task: packed positions of the range
            int32_t pos[kRRows];
        } k;
        struct {                       // G: per-warp V ring and the warps' parked states
            uint8_t ring[kFWarps][2][16 * kD * 2];
            float park[kFWarps][8][kD];
            float pm[kFWarps][8];
            float pl[kFWarps][8];
        } g;
    };
};
static_assert(offsetof(FShared, s) % 128 == 0, "the cp.async / ldmatrix ring needs 16-byte aligned rows");

// Block-wide exclusive scan of (a, b) in thread order, with totals.  Fixed order.
template <typename TB>
__device__ __forceinline__ void bscan(uint32_t a, TB b, uint32_t& ea, TB& eb, uint32_t& ta, TB& tb, uint32_t* wa,
                                      TB* wb) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t ia = a;
    TB ib = b;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t xa = __shfl_up_sync(0xffffffffu, ia, off);
        const TB xb = __shfl_up_sync(0xffffffffu, ib, off);
        if (lane >= off) { ia += xa; ib += xb; }
    }
    if (lane == 31) { wa[warp] = ia; wb[warp] = ib; }
    __syncthreads();
    uint32_t sa = 0, pa = 0;
    TB sb = 0, pb = 0;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) {
        const uint32_t va = wa[w];
        const TB vb = wb[w];
        if (w < warp) { pa += va; pb += vb; }
        sa += va; sb += vb;
    }
    ea = pa + ia - a;
    eb = pb + ib - b;
    ta = sa;
    tb = sb;
    __syncthreads();
}

__device__ __forceinline__ float bflo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bfhi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------- S: scores + level 0
// One key row per thread (32 bytes: two 16-byte loads), the 8 rows of a thread loaded before
// any is used.  The dot product runs in the order of the separate scoring kernel (dims 0-7
// and 8-15 as two fma chains, then added), so both paths produce the same scores.  The
// histogram is built with shared-memory atomics (a warp's 32 scores fall in about 20
// distinct bins, so conflicts are few).
__device__ void task_s(const FusedParams& p, FShared& sh, int u, int chunk) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int b = u / p.Hkv, g = u - b * p.Hkv;
    const int M = p.N;
    const int n0 = chunk * kSRows, n1 = min(M, n0 + kSRows);
    const uint4* krow = p.kidx + size_t(u) * M * 2;
    constexpr int kPer = kSRows / kFThreads;   // 8 rows per thread
    uint4 w[kPer][2];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int n = n0 + tid + i * kFThreads;
        if (n < n1) {
            w[i][0] = __ldg(krow + size_t(n) * 2);
            w[i][1] = __ldg(krow + size_t(n) * 2 + 1);
        } else {
            w[i][0] = w[i][1] = make_uint4(0, 0, 0, 0);
        }
    }
    for (int i = tid; i < kBins; i += kFThreads) {
        sh.s.cnt[i] = 0;
        sh.s.mhi[i] = 0;
        sh.s.mlo[i] = 0;
    }
    // index query: mean over the G heads (summed in order), all 16 dims
    float qv[16];
    {
#pragma unroll
        for (int j = 0; j < 16; ++j) qv[j] = 0.f;
        const uint4* qb = reinterpret_cast<const uint4*>(p.qidx + (size_t(b) * p.Hq + size_t(g) * p.G) * 16);
        for (int h = 0; h < p.G; ++h) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint4 v = __ldg(qb + 2 * h + hh);
                const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    qv[8 * hh + 2 * j] += bflo(ws[j]);
                    qv[8 * hh + 2 * j + 1] += bfhi(ws[j]);
                }
            }
        }
        const float fg = float(p.G);
#pragma unroll
        for (int j = 0; j < 16; ++j) qv[j] = qv[j] / fg;
    }
    __syncthreads();
    float* srow = p.scores + size_t(u) * M;
    uint32_t my_max = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int n = n0 + tid + i * kFThreads;
        const bool live = n < n1;
        float half_dot[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t ws[4] = {w[i][hh].x, w[i][hh].y, w[i][hh].z, w[i][hh].w};
            float part = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                part = fmaf(qv[8 * hh + 2 * j], bflo(ws[j]), part);
                part = fmaf(qv[8 * hh + 2 * j + 1], bfhi(ws[j]), part);
            }
            half_dot[hh] = part;
        }
        const float sc = p.score_scale * (half_dot[0] + half_dot[1]);
        const uint32_t key = score_key(sc);
        const uint32_t bin = key >> 21;
        if (live) {
            srow[n] = sc;
            my_max = max(my_max, key);
            atomicAdd(&sh.s.cnt[bin], 1u);
            if (p.topp_mode) {
                // 41-bit fixed-point mass as two halves; <= 2048 keys per task cannot overflow
                const u64 e = fixed_mass(sc, bin_top_score(bin));
                atomicAdd(&sh.s.mhi[bin], uint32_t(e >> 20));
                atomicAdd(&sh.s.mlo[bin], uint32_t(e & 0xfffffu));
            }
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, off));
    if (lane == 0) atomicMax(p.hist.max_key + u, my_max);
    __syncthreads();
    uint32_t* gc = p.hist.cnt + size_t(u) * kBins;
    u64* gm = p.hist.mass + size_t(u) * kBins;
    for (int i = tid; i < kBins; i += kFThreads) {
        const uint32_t c = sh.s.cnt[i];
        if (c) {
            atomicAdd(gc + i, c);
            if (p.topp_mode) atomicAdd(gm + i, (u64(sh.s.mhi[i]) << 20) + sh.s.mlo[i]);
        }
    }
}

// ---------------------------------------------------------------- D0: level 0 of unit u
__device__ void resolve_level0(const FusedParams& p, FShared& sh, int u, bool pub) {
    const int tid = threadIdx.x;
    FUnit& U = p.unit[u];
    const int L = p.M;
    uint32_t mode = MODE_THRESH;
    if (p.local && p.local[u]) mode = MODE_NONE;
    else if (!p.topp_mode) {
        if (p.topk >= L) mode = MODE_ALL;
        else if (p.topk <= 0) mode = MODE_NONE;
    }
    const uint32_t* hc = p.hist.cnt + size_t(u) * kBins;
    const u64* hm = p.hist.mass + size_t(u) * kBins;
    const uint32_t max_key = __ldcg(p.hist.max_key + u);
    const float m = key_score(max_key);
    if (mode == MODE_THRESH) {
        const Level0 l0 = level0_crossing(hc, hm, max_key, p.topp_mode != 0, p.topp, p.topk, sh.l0);
        if (tid == 0) {
            const uint32_t b0 = l0.bin;
            const float r0 = bin_top_score(b0);
            const double scale0 = p.topp_mode ? kInvMass * exp(double(r0) - double(m)) : 0.0;
            const double T = double(p.topp) * l0.Z;
            U.b0 = b0;
            U.cum_cnt0 = l0.above_cnt;
            U.cum_mass0 = l0.above_mass;
            U.Z = l0.Z;
            U.scale0 = scale0;
            if (p.topp_mode) {
                const double need = (T - l0.above_mass) / (scale0 > 0.0 ? scale0 : 1.0);
                const u64 hb = __ldcg(hm + b0);
                u64 t = need <= 1.0 ? 1ull : (need >= double(hb) ? hb : u64(ceil(need)));
                U.target_mass = t < 1 ? 1 : t;
                U.target_cnt = 0;
            } else {
                U.target_mass = 0;
                U.target_cnt = uint32_t(p.topk) - l0.above_cnt;
            }
        }
    }
    if (tid == 0) {
        U.mode = mode;
        U.max_key = max_key;
    }
    __syncthreads();
    // the histogram is consumed: clear it for the next call
    for (int i = tid; i < kBins; i += kFThreads) {
        p.hist.cnt[size_t(u) * kBins + i] = 0;
        p.hist.mass[size_t(u) * kBins + i] = 0;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        p.hist.max_key[u] = 0;
        if (pub) {
            __threadfence();
            publish(p, 0, u);
        }
    }
}

// ---------------------------------------------------------------- C: counts and candidates
__device__ void task_c(const FusedParams& p, FShared& sh, int u, int r) {
    const int tid = threadIdx.x, lane = tid & 31;
    FUnit& U = p.unit[u];
    const uint32_t mode = __ldcg(&U.mode), b0 = __ldcg(&U.b0);
    const int M = p.M;
    const int n0 = r * kRRows, n1 = min(M, n0 + kRRows);
    const float* srow = p.scores + size_t(u) * M;
    uint2* cand = p.cand + size_t(u) * M;
    uint32_t above = 0;
    if (mode == MODE_ALL) {
        above = tid == 0 ? uint32_t(n1 - n0) : 0u;
    } else if (mode == MODE_THRESH) {
        // groups of 4 scores per thread, all 8 groups loaded before any is used (n0 is a
        // multiple of 4; the row start is 16-byte aligned when N is a multiple of 4, else
        // scalar loads)
        const bool vec = (M & 3) == 0;
        constexpr int kSteps = kRRows / (4 * kFThreads);   // 8
        float vv[kSteps][4];
#pragma unroll
        for (int k = 0; k < kSteps; ++k) {
            const int i = n0 + k * 4 * kFThreads + 4 * tid;
            if (vec && i + 3 < n1) {
                const float4 t = __ldcg(reinterpret_cast<const float4*>(srow + i));
                vv[k][0] = t.x; vv[k][1] = t.y; vv[k][2] = t.z; vv[k][3] = t.w;
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) vv[k][j] = i + j < n1 ? __ldcg(srow + i + j) : -INFINITY;
            }
        }
#pragma unroll
        for (int k = 0; k < kSteps; ++k) {
            const int i = n0 + k * 4 * kFThreads + 4 * tid;
            const float* v = vv[k];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool live = i + j < n1;
                const uint32_t key = score_key(v[j]);
                const uint32_t bin = key >> 21;
                above += uint32_t(live && bin > b0);
                const bool isc = live && bin == b0;
                const unsigned bal = __ballot_sync(0xffffffffu, isc);
                if (bal) {
                    uint32_t slot = 0;
                    if (lane == 0) slot = atomicAdd(&U.cand_n, uint32_t(__popc(bal)));
                    slot = __shfl_sync(0xffffffffu, slot, 0);
                    if (isc) cand[slot + __popc(bal & ((1u << lane) - 1u))] = make_uint2(uint32_t(i + j), key);
                }
            }
        }
    }
    uint32_t e, t;
    u64 e2, t2;
    bscan<u64>(above, 0ull, e, e2, t, t2, sh.wu32, sh.wu64);
    if (tid == 0) p.rng_above[size_t(u) * p.NR + r] = t;
}

// ---------------------------------------------------------------- D1: levels 1-2 of unit u
// candidate i of the unit (from shared memory when they fit)
__device__ __forceinline__ uint2 cand_at(const FusedParams& p, const FShared& sh, int u, bool in_smem, uint32_t i) {
    return in_smem ? sh.d.cand[i] : __ldcg(p.cand + size_t(u) * p.M + i);
}

__device__ void resolve_levels12(const FusedParams& p, FShared& sh, int u, bool pub) {
    const int tid = threadIdx.x;
    FUnit& U = p.unit[u];
    const uint32_t mode = __ldcg(&U.mode);
    const int L = p.M;
    const bool is_local = p.local && p.local[u];
    const uint32_t nc = __ldcg(&U.cand_n);
    const bool in_smem = nc <= uint32_t(kCandSmem);
    if (in_smem) {
        const uint2* src = p.cand + size_t(u) * p.M;
        for (uint32_t i0 = 0; i0 < nc; i0 += 8 * kFThreads) {
            uint2 t[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t i = i0 + k * kFThreads + tid;
                t[k] = i < nc ? __ldcg(src + i) : make_uint2(0, 0);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t i = i0 + k * kFThreads + tid;
                if (i < nc) sh.d.cand[i] = t[k];
            }
        }
    }
    const uint32_t b0 = __ldcg(&U.b0);
    const float r0 = bin_top_score(b0);
    const float m = key_score(__ldcg(&U.max_key));
    uint32_t tau = 0xffffffffu, q = 0, cnt_tau = 0, tie_cut = 0x7fffffffu;
    u64 cum_in = 0, E_tau = 0;
    if (mode == MODE_THRESH) {
        const u64 target_mass = __ldcg(&U.target_mass);
        const uint32_t target_cnt = __ldcg(&U.target_cnt);
        uint32_t prefix = b0, cum_c = 0;
        u64 cum_m = 0;
        for (int level = 1; level <= 2; ++level) {
            const int shift = level == 1 ? 10 : 0;
            const int nb = level == 1 ? 2048 : 1024;
            const int pshift = level == 1 ? 21 : 10;
            // masses (< 2^41 each) are summed in three 14-bit parts with 32-bit shared atomics,
            // which cannot overflow below 2^18 candidates; more candidates use 64-bit sums
            // (aliased on the parts)
            const bool wide = nc > (1u << 18);
            u64* hw = reinterpret_cast<u64*>(&sh.d.part[0][0]);
            for (int i = tid; i < nb; i += kFThreads) {
                sh.d.cnt[i] = 0;
                if (wide) hw[i] = 0;
                else sh.d.part[0][i] = sh.d.part[1][i] = sh.d.part[2][i] = 0;
            }
            __syncthreads();
            for (uint32_t i = tid; i < nc; i += kFThreads) {
                const uint2 cd = cand_at(p, sh, u, in_smem, i);
                const uint32_t k = cd.y;
                if ((k >> pshift) == prefix) {
                    const uint32_t bin = (k >> shift) & uint32_t(nb - 1);
                    atomicAdd(&sh.d.cnt[bin], 1u);
                    if (p.topp_mode) {
                        const u64 e = fixed_mass(key_score(k), r0);
                        if (wide) {
                            atomicAdd(&hw[bin], e);
                        } else {
                            atomicAdd(&sh.d.part[0][bin], uint32_t(e) & 0x3fffu);
                            atomicAdd(&sh.d.part[1][bin], uint32_t(e >> 14) & 0x3fffu);
                            atomicAdd(&sh.d.part[2][bin], uint32_t(e >> 28));
                        }
                    }
                }
            }
            __syncthreads();
            const int per = nb / kFThreads;   // 8 or 4 bins per thread, descending
            uint32_t vc[8];
            u64 vm[8];
            uint32_t sc = 0;
            u64 sm = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                vc[j] = 0; vm[j] = 0;
                if (j < per) {
                    const int bin = nb - 1 - (tid * per + j);
                    vc[j] = sh.d.cnt[bin];
                    if (p.topp_mode)
                        vm[j] = wide ? hw[bin]
                                     : u64(sh.d.part[0][bin]) + (u64(sh.d.part[1][bin]) << 14) +
                                           (u64(sh.d.part[2][bin]) << 28);
                    sc += vc[j];
                    sm += vm[j];
                }
            }
            if (tid == 0) {   // defaults if rounding left no crossing: the last bin
                sh.found_bin = 0;
                sh.found_above_cnt = cum_c;
                sh.found_above_mass = cum_m;
                sh.found_cnt = 0;
            }
            uint32_t ec, tc;
            u64 em, tm;
            bscan<u64>(sc, sm, ec, em, tc, tm, sh.wu32, sh.wu64);
            uint32_t ac = cum_c + ec;
            u64 am = cum_m + em;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < per) {
                    const bool hit = p.topp_mode ? (am < target_mass && am + vm[j] >= target_mass)
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
                tau = prefix;
                cnt_tau = sh.found_cnt;
                cum_in = cum_m;
                if (p.topp_mode) {
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
        // ties at tau are taken in ascending position: when the quota splits them, the cut is
        // the smallest position P with #(ties at positions <= P) >= q (binary search)
        if (q < cnt_tau) {
            int lo = -1, hi = L - 1;   // count(lo) < q <= count(hi)
            while (hi - lo > 1) {
                const int mid = (lo + hi) / 2;
                uint32_t c = 0;
                for (uint32_t i = tid; i < nc; i += kFThreads) {
                    const uint2 cd = cand_at(p, sh, u, in_smem, i);
                    c += uint32_t(cd.y == tau && int(cd.x) <= mid);
                }
                uint32_t e1, t1;
                u64 e2, t2;
                bscan<u64>(c, 0ull, e1, e2, t1, t2, sh.wu32, sh.wu64);
                if (t1 >= q) hi = mid; else lo = mid;
            }
            tie_cut = uint32_t(hi);
        }
    }
    // per-range support counts: above B0 (from the C tasks), the candidates at or above the
    // threshold, and the forced positions (sink, window) the threshold did not take
    for (int r = tid; r < p.NR; r += kFThreads) sh.rsel[r] = __ldcg(p.rng_above + size_t(u) * p.NR + r);
    __syncthreads();
    if (mode == MODE_THRESH) {
        for (uint32_t i = tid; i < nc; i += kFThreads) {
            const uint2 cd = cand_at(p, sh, u, in_smem, i);
            if (cd.y > tau || (cd.y == tau && cd.x <= tie_cut)) atomicAdd(&sh.rsel[cd.x / kRRows], 1u);
        }
    }
    double fmass = 0.0;
    {
        const int s_end = min(p.sink, L);
        const int w_beg = max(s_end, L - p.window);
        const int nf = s_end + (L - w_beg);
        const float* srow = p.scores + size_t(u) * p.M;
        for (int j = tid; j < nf; j += kFThreads) {
            const int pos = j < s_end ? j : w_beg + (j - s_end);
            const float s = __ldcg(srow + pos);
            const uint32_t k = score_key(s);
            bool taken;
            if (mode == MODE_ALL) taken = true;
            else if (mode == MODE_NONE) taken = false;
            else taken = k > tau || (k == tau && uint32_t(pos) <= tie_cut);
            if (!taken) {
                atomicAdd(&sh.rsel[pos / kRRows], 1u);
                if (p.topp_mode && !is_local) fmass += exp(double(s) - double(m));
            }
        }
    }
    __syncthreads();
    // offsets: exclusive prefix over the ranges (NR <= 1024: four per thread)
    uint32_t loc[4], lsum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = tid * 4 + j;
        loc[j] = r < p.NR ? sh.rsel[r] : 0u;
        lsum += loc[j];
    }
    uint32_t eo, total;
    double efm, tfm;
    bscan<double>(lsum, fmass, eo, efm, total, tfm, sh.wu32, sh.wf64);
    {
        uint32_t o = eo;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = tid * 4 + j;
            if (r < p.NR) p.rng_off[size_t(u) * (p.NR + 1) + r] = o;
            o += loc[j];
        }
        if (tid == 0) p.rng_off[size_t(u) * (p.NR + 1) + p.NR] = total;
    }
    if (tid == 0) {
        U.tau = tau;
        U.tie_cut = tie_cut;
        U.total = total;
        const uint32_t rows = min(total, uint32_t(p.cap));
        U.ntiles = (rows + 15) / 16;
        p.count[u] = int32_t(total);
        if (total > uint32_t(p.cap)) raise_status(p.status, SPA_ERR_CAPACITY);
        if (p.topp_mode && p.index_mass) {
            double top = 0.0;
            if (mode == MODE_THRESH) top = __ldcg(&U.cum_mass0) + double(cum_in + u64(q) * E_tau) * __ldcg(&U.scale0);
            const double Z = __ldcg(&U.Z);
            p.index_mass[u] = Z > 0.0 && !is_local ? float((top + tfm) / Z) : 0.f;
        }
        U.cand_n = 0;   // consumed
        if (pub) {
            __threadfence();
            publish(p, 1, u);
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------- K: compaction of a range
__device__ void task_k(const FusedParams& p, FShared& sh, int u, int r) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    FUnit& U = p.unit[u];
    const uint32_t mode = __ldcg(&U.mode), tau = __ldcg(&U.tau), tie_cut = __ldcg(&U.tie_cut);
    const int L = p.M;
    const int n0 = r * kRRows, n1 = min(L, n0 + kRRows);
    const float* srow = p.scores + size_t(u) * L;
    const int window_lo = L - p.window;
    // warp w walks [w * kRRows / 8, ...) of the range in steps of 128 (four per lane)
    constexpr int kSeg = kRRows / kFWarps;   // 1024
    const int w0 = n0 + warp * kSeg, w1 = min(n1, w0 + kSeg);
    const bool vec = (L & 3) == 0;
    uint32_t ns = 0;
    int32_t* packed = sh.k.pos + warp * kSeg;
    constexpr int kSteps = kSeg / 128;   // 8 steps of 128 positions, loaded before any is used
    float vv[kSteps][4];
#pragma unroll
    for (int k = 0; k < kSteps; ++k) {
        const int i = w0 + k * 128 + 4 * lane;
        if (vec && i + 3 < w1) {
            const float4 t = __ldcg(reinterpret_cast<const float4*>(srow + i));
            vv[k][0] = t.x; vv[k][1] = t.y; vv[k][2] = t.z; vv[k][3] = t.w;
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) vv[k][j] = i + j < w1 ? __ldcg(srow + i + j) : 0.f;
        }
    }
#pragma unroll
    for (int k = 0; k < kSteps; ++k) {
        const int i0 = w0 + k * 128;
        if (i0 >= w1) break;                       // warp-uniform
        const int i = i0 + 4 * lane;
        const float* v = vv[k];
        uint32_t flags = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int pos = i + j;
            const bool live = pos < w1;
            const uint32_t key = score_key(v[j]);
            bool sel;
            if (mode == MODE_ALL) sel = true;
            else if (mode == MODE_NONE) sel = false;
            else sel = key > tau || (key == tau && uint32_t(pos) <= tie_cut);
            sel = live && (sel || pos < p.sink || pos >= window_lo);
            flags |= uint32_t(sel) << j;
        }
        const uint32_t c = __popc(flags);
        uint32_t incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += x;
        }
        uint32_t at = ns + incl - c;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (flags >> j & 1u) packed[at++] = i + j;
        ns += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sh.wu32[warp] = ns;
    __syncthreads();
    uint32_t before = __ldcg(p.rng_off + size_t(u) * (p.NR + 1) + r);
    for (int w = 0; w < warp; ++w) before += sh.wu32[w];
    int32_t* dst = p.idx + size_t(u) * p.cap;
    for (uint32_t j = lane; j < ns; j += 32) {
        const uint32_t o = before + j;
        if (o < uint32_t(p.cap)) dst[o] = packed[j];
    }
}

// ---------------------------------------------------------------- G: gather + attention
struct GState {
    float m[2], l[2];       // heads 2cq, 2cq + 1 (log2 units)
    float acc[8][4];        // O^T: dims 16dt + gq (+8) x heads 2cq (+1)
    uint32_t qb[8][2];      // Q^T B fragments, permuted head dimension
};

// B fragments of Q^T for unit u: lane (gq, cq) holds head gq, dims 32t + 8cq + [0, 8) of load t,
// which serve k-steps 2t (words 0, 1) and 2t + 1 (words 2, 3) -- the same permutation as K.
__device__ __forceinline__ void g_init(const FusedParams& p, int u, GState& st) {
    const int lane = threadIdx.x & 31, gq = lane >> 2, cq = lane & 3;
    const int b = u / p.Hkv, g = u - b * p.Hkv;
    const bool v = gq < p.G;
    const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.Hq + size_t(g) * p.G + (v ? gq : 0)) * kD);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const uint4 w = v ? __ldg(qrow + 4 * t + cq) : make_uint4(0, 0, 0, 0);
        st.qb[2 * t][0] = w.x; st.qb[2 * t][1] = w.y;
        st.qb[2 * t + 1][0] = w.z; st.qb[2 * t + 1][1] = w.w;
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) { st.m[e] = -INFINITY; st.l[e] = 0.f; }
#pragma unroll
    for (int dt = 0; dt < 8; ++dt) st.acc[dt][0] = st.acc[dt][1] = st.acc[dt][2] = st.acc[dt][3] = 0.f;
}

__device__ void g_flush(const FusedParams& p, FShared& sh, int u, GState& st);

// Support rows of gather tile t (lane l & 15 holds row l & 15; -1 past the support)
__device__ __forceinline__ int g_row(const int32_t* idx_u, int rows, int t, int& nval) {
    const int lane = threadIdx.x & 31;
    const int base = t * 16;
    nval = max(0, min(16, rows - base));
    return (lane & 15) < nval ? __ldcg(idx_u + base + (lane & 15)) : -1;
}

// Issue the loads of a tile: K rows gq and gq + 8 straight into A fragments (64 contiguous
// bytes per lane and row), V rows into the ring stage by cp.async (16-byte chunks, row-swizzled).
__device__ __forceinline__ void g_issue(const FusedParams& p, size_t kv0, int myrow, uint4 (&ka)[4], uint4 (&kb)[4],
                                        uint32_t vbase) {
    const int lane = threadIdx.x & 31, gq = lane >> 2, cq = lane & 3;
    const int ra = __shfl_sync(0xffffffffu, myrow, gq), rb = __shfl_sync(0xffffffffu, myrow, gq + 8);
    const uint4* pa = reinterpret_cast<const uint4*>(p.K + (kv0 + size_t(ra < 0 ? 0 : ra)) * kD);
    const uint4* pb = reinterpret_cast<const uint4*>(p.K + (kv0 + size_t(rb < 0 ? 0 : rb)) * kD);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        ka[t] = ra >= 0 ? __ldg(pa + 4 * t + cq) : make_uint4(0, 0, 0, 0);
        kb[t] = rb >= 0 ? __ldg(pb + 4 * t + cq) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rr = 2 * i + (lane >> 4), ch = lane & 15;
        const int row = __shfl_sync(0xffffffffu, myrow, rr);
        const bool ok = row >= 0;
        const uint16_t* src = p.V + (ok ? (kv0 + size_t(row)) * kD + ch * 8 : 0);
        cp_async16(vbase + (rr * 16 + (ch ^ (rr & 7))) * 16, src, ok);
    }
    cp_commit();
}

// The gather of unit u by this CTA: every warp claims 16-row tiles of the unit's support from
// the unit's cursor until none is left, keeping one tile's loads in flight while it computes
// the previous one (tiles are claimed two ahead, their row indices read one ahead).  The CTA
// then merges its warps and appends one record per head (none if it found no tile).
__device__ void g_stretch(const FusedParams& p, FShared& sh, int u) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gq = lane >> 2;
    GState st;
    g_init(p, u, st);
    const float sl2 = p.sm_scale * kLog2e;
    FUnit& U = p.unit[u];
    const int ntiles = int(__ldcg(&U.ntiles));
    const int rows = int(min(__ldcg(&U.total), uint32_t(p.cap)));
    const int32_t* idx_u = p.idx + size_t(u) * p.cap;
    const size_t kv0 = size_t(u) * size_t(p.N);
    auto claim = [&]() -> int {
        uint32_t t = 0;
        if (lane == 0) t = atomicAdd(&U.next[2], 1u);
        return int(__shfl_sync(0xffffffffu, t, 0));
    };
    int t0 = claim();
    int t1 = t0 < ntiles ? claim() : ntiles;
    int nval0 = 0;
    int row0 = t0 < ntiles ? g_row(idx_u, rows, t0, nval0) : -1;
    uint4 ka[4], kb[4];
    int stage = 0;
    bool did = false;
    if (nval0 > 0) g_issue(p, kv0, row0, ka, kb, smem_u32(sh.g.ring[warp][stage]));
    while (t0 < ntiles) {
        uint32_t t2 = 0;
        if (lane == 0 && t1 < ntiles) t2 = atomicAdd(&U.next[2], 1u);   // consumed after this tile
        int nval1 = 0, row1 = -1;
        if (t1 < ntiles) row1 = g_row(idx_u, rows, t1, nval1);
        if (nval0 > 0) {
            did = true;
            const uint32_t vbase = smem_u32(sh.g.ring[warp][stage]);
            // S^T = K Q^T
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t a0[4] = {ka[t].x, kb[t].x, ka[t].y, kb[t].y};
                mma16816(s, a0, st.qb[2 * t][0], st.qb[2 * t][1]);
                const uint32_t a1[4] = {ka[t].z, kb[t].z, ka[t].w, kb[t].w};
                mma16816(s, a1, st.qb[2 * t + 1][0], st.qb[2 * t + 1][1]);
            }
            // the next tile's loads go out now (the K registers are free)
            const bool issued = nval1 > 0;
            if (issued) g_issue(p, kv0, row1, ka, kb, smem_u32(sh.g.ring[warp][stage ^ 1]));
            // online softmax per head (column); keys gq, gq + 8 here, reduced over gq by xor
            const bool v0 = gq < nval0, v1 = gq + 8 < nval0;
            float alpha[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float x0 = v0 ? s[e] * sl2 : -INFINITY;
                const float x1 = v1 ? s[2 + e] * sl2 : -INFINITY;
                float tm = fmaxf(x0, x1);
                tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
                tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
                tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
                const float mn = fmaxf(st.m[e], tm);
                const float mref = mn == -INFINITY ? 0.f : mn;
                alpha[e] = exp2f(st.m[e] - mref);
                st.m[e] = mn;
                const float p0 = exp2f(x0 - mref), p1 = exp2f(x1 - mref);
                s[e] = p0;
                s[2 + e] = p1;
                st.l[e] = st.l[e] * alpha[e] + p0 + p1;
            }
#pragma unroll
            for (int dt = 0; dt < 8; ++dt) {
                st.acc[dt][0] *= alpha[0];
                st.acc[dt][1] *= alpha[1];
                st.acc[dt][2] *= alpha[0];
                st.acc[dt][3] *= alpha[1];
            }
            uint32_t bh[2], bl[2];
            {
                uint32_t h0, l0, h1, l1;
                split_bf16(s[0], s[1], h0, l0);     // key gq,     heads 2cq, 2cq + 1
                split_bf16(s[2], s[3], h1, l1);     // key gq + 8
                bh[0] = movm_t(h0); bh[1] = movm_t(h1);
                bl[0] = movm_t(l0); bl[1] = movm_t(l1);
            }
            if (issued) cp_wait<1>(); else cp_wait<0>();
            __syncwarp();
            // O^T += V^T P^T
#pragma unroll
            for (int dt = 0; dt < 8; ++dt) {
                const int mat = lane >> 3;
                const int rr = (mat >> 1) * 8 + (lane & 7);
                const int ch = 2 * dt + (mat & 1);
                uint32_t a[4];
                ldsm_x4_t(vbase + (rr * 16 + (ch ^ (rr & 7))) * 16, a[0], a[1], a[2], a[3]);
                mma16816(st.acc[dt], a, bh[0], bh[1]);
                mma16816(st.acc[dt], a, bl[0], bl[1]);
            }
            __syncwarp();   // this stage may be refilled
        } else if (nval1 > 0) {
            g_issue(p, kv0, row1, ka, kb, smem_u32(sh.g.ring[warp][stage ^ 1]));
        }
        const int t2v = t1 < ntiles ? int(__shfl_sync(0xffffffffu, t2, 0)) : ntiles;
        t0 = t1;
        t1 = t2v;
        nval0 = nval1;
        stage ^= 1;
    }
    cp_wait<0>();
    if (__syncthreads_or(did ? 1 : 0)) g_flush(p, sh, u, st);
}

// merge the warps' states of unit u and append one record per head
__device__ void g_flush(const FusedParams& p, FShared& sh, int u, GState& st) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gq = lane >> 2, cq = lane & 3;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        st.l[e] += __shfl_xor_sync(0xffffffffu, st.l[e], 4);
        st.l[e] += __shfl_xor_sync(0xffffffffu, st.l[e], 8);
        st.l[e] += __shfl_xor_sync(0xffffffffu, st.l[e], 16);
    }
    __syncthreads();   // the rings are no longer read
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int hd = 2 * cq + e;
        if (gq == 0) {
            sh.g.pm[warp][hd] = st.m[e];
            sh.g.pl[warp][hd] = st.l[e];
        }
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
            sh.g.park[warp][hd][dt * 16 + gq] = st.acc[dt][e];
            sh.g.park[warp][hd][dt * 16 + gq + 8] = st.acc[dt][2 + e];
        }
    }
    if (tid == 0) {
        const uint32_t slot = atomicAdd(&p.unit[u].nrec, 1u);
        // at most one record per (CTA, unit); a count left over from an interrupted call
        // must not push a record out of its buffer
        if (slot >= uint32_t(p.n_ctas)) raise_status(p.status, SPA_ERR_TIMEOUT);
        sh.flag = slot < uint32_t(p.n_ctas) ? int(slot) : -1;
    }
    __syncthreads();
    const int slot = sh.flag;
    const int nh = p.G;
    for (int i = tid; slot >= 0 && i < nh * kD; i += kFThreads) {
        const int hd = i / kD, col = i - hd * kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) M = fmaxf(M, sh.g.pm[w][hd]);
        const float Mr = M == -INFINITY ? 0.f : M;
        float Lsum = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) {
            const float sc = exp2f(sh.g.pm[w][hd] - Mr);
            Lsum += sh.g.pl[w][hd] * sc;
            O += sh.g.park[w][hd][col] * sc;
        }
        float* rec = p.rec + ((size_t(u) * nh + hd) * p.n_ctas + slot) * (kD + 2);
        rec[col] = O;
        if (col == 0) {
            rec[kD] = M;
            rec[kD + 1] = Lsum;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------- the persistent kernel
__global__ void __launch_bounds__(kFThreads, 2) decode_fused_kernel(FusedParams p) {
    pdl_enter();
    extern __shared__ __align__(128) uint8_t dyn[];
    FShared& sh = *reinterpret_cast<FShared*>(dyn);
    const int tid = threadIdx.x;
    const uint32_t n_s = uint32_t(p.U) * uint32_t(p.nS);
    const bool sel_only = int(blockIdx.x) < p.n_sel;
    // choice state, kept by thread 0: the next slot of each stage this CTA looks at
    int slot[3] = {0, 0, 0};
    bool s_done = false;
    uint32_t idle = 0;   // consecutive rounds without a task (bounded like every wait)

    while (true) {
        // ---- choose a task: C and K ranges of published units first (they unlock the
        // gathers), then S tasks, then gather tiles; nothing is ever claimed before it is ready
        if (tid == 0) {
            int task = T_NONE, tu = 0, tc = 0;
            for (int sg = 0; sg < 2 && task == T_NONE; ++sg) {
                while (slot[sg] < p.U) {
                    if (!ld_acquire(p.ready + sg * p.U + slot[sg])) break;
                    const int u = int(__ldcg(p.order + sg * p.U + slot[sg]));
                    const uint32_t c = atomicAdd(&p.unit[u].next[sg], 1u);
                    if (c < uint32_t(p.NR)) {
                        task = sg == 0 ? T_C : T_K;
                        tu = u;
                        tc = int(c);
                        break;
                    }
                    ++slot[sg];
                }
            }
            if (task == T_NONE && !s_done) {
                const uint32_t t = atomicAdd(&p.ctr->s_head, 1u);
                if (t < n_s) {
                    task = T_S;
                    tu = int(t / uint32_t(p.nS));
                    tc = int(t % uint32_t(p.nS));
                } else {
                    s_done = true;
                }
            }
            if (task == T_NONE && !sel_only) {
                while (slot[2] < p.U) {
                    if (!ld_acquire(p.ready + 2 * p.U + slot[2])) break;
                    const int u = int(__ldcg(p.order + 2 * p.U + slot[2]));
                    if (__ldcg(&p.unit[u].next[2]) < __ldcg(&p.unit[u].ntiles)) {
                        task = T_G;
                        tu = u;
                        break;
                    }
                    ++slot[2];
                }
            }
            if (task == T_NONE) {
                if (s_done && slot[0] >= p.U && slot[1] >= p.U && (sel_only || slot[2] >= p.U)) {
                    task = T_DONE;
                } else if (ld_acquire(&p.ctr->abort)) {
                    task = T_DONE;
                } else if (++idle >= kWaitLimit) {
                    raise_status(p.status, SPA_ERR_TIMEOUT);
                    atomicExch(&p.ctr->abort, 1u);
                    task = T_DONE;
                }
            } else {
                idle = 0;
            }
            sh.task = task; sh.tu = tu; sh.tc = tc;
        }
        __syncthreads();
        const int task = sh.task, u = sh.tu, c = sh.tc;
        __syncthreads();
        if (task == T_DONE) break;
        if (task == T_NONE) {
            __nanosleep(256);
            continue;
        }
        if (task == T_G) {
            g_stretch(p, sh, u);
            continue;
        }
        FUnit& U = p.unit[u];
        if (task == T_S) {
            task_s(p, sh, u, c);
            __threadfence();
            __syncthreads();
            if (tid == 0) sh.flag = atomicAdd(&U.s_done, 1u) == uint32_t(p.nS - 1);
            __syncthreads();
            if (sh.flag) {
                __threadfence();
                resolve_level0(p, sh, u, true);   // publishes the unit's C ranges
            }
            __syncthreads();
        } else if (task == T_C) {
            task_c(p, sh, u, c);
            __threadfence();
            __syncthreads();
            if (tid == 0) sh.flag = atomicAdd(&U.done[0], 1u) == uint32_t(p.NR - 1);
            __syncthreads();
            if (sh.flag) {
                __threadfence();
                resolve_levels12(p, sh, u, true);   // publishes the unit's K ranges
            }
            __syncthreads();
        } else {
            task_k(p, sh, u, c);
            __threadfence();
            __syncthreads();
            if (tid == 0 && atomicAdd(&U.done[1], 1u) == uint32_t(p.NR - 1)) {
                __threadfence();
                publish(p, 2, u);   // the support is complete: gather
            }
            __syncthreads();
        }
    }

    // ---- the last CTA out resets the counters for the next call
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        sh.flag = atomicAdd(&p.ctr->exit_count, 1u) == gridDim.x - 1 ? 1 : 0;
    }
    __syncthreads();
    if (sh.flag) {
        __threadfence();
        const bool aborted = __ldcg(&p.ctr->abort) != 0;
        for (int u = tid; u < p.U; u += kFThreads) {
            FUnit& U = p.unit[u];
            U.s_done = 0;
            U.next[0] = U.next[1] = U.next[2] = 0;
            U.done[0] = U.done[1] = 0;
            U.cand_n = 0;
            p.ready[u] = p.ready[p.U + u] = p.ready[2 * p.U + u] = 0;
            if (aborted) p.hist.max_key[u] = 0;
        }
        if (aborted)
            for (size_t i = tid; i < size_t(p.U) * kBins; i += kFThreads) {
                p.hist.cnt[i] = 0;
                p.hist.mass[i] = 0;
            }
        __syncthreads();
        if (tid == 0) {
            p.ctr->s_head = 0;
            p.ctr->pub[0] = p.ctr->pub[1] = p.ctr->pub[2] = 0;
            p.ctr->abort = 0;
            __threadfence();
            p.ctr->exit_count = 0;
        }
    }
}

// ---------------------------------------------------------------- combine
// grid (U, G, 4): column quarter q of (unit, head).  The records are merged in slot order:
// 8 record groups x 32 columns per CTA, every load of a group's records issued in batches of
// 4 before use, then a fixed-order sum over the groups.  The last CTA of a unit resets the
// unit's record count.
constexpr int kCombQ = 4;
__global__ void __launch_bounds__(256) fused_combine_kernel(FusedParams p) {
    pdl_enter();
    constexpr int REC = kD + 2;
    constexpr int QC = kD / kCombQ;   // 32 columns
    const int u = blockIdx.x, hd = blockIdx.y, qt = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
    FUnit& U = p.unit[u];
    const int nrec = min(int(__ldcg(&U.nrec)), p.n_ctas);
    __shared__ float s_red[8], sL[8], sO[8][QC];
    const float* base = p.rec + ((size_t(u) * p.G + hd) * p.n_ctas) * REC;
    float mx = -INFINITY;
    for (int r = tid; r < nrec; r += 256) mx = fmaxf(mx, __ldcg(base + size_t(r) * REC + kD));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) s_red[grp] = mx;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, s_red[w]);
    const float Mr = M == -INFINITY ? 0.f : M;
    const int col = qt * QC + lane;
    float L = 0.f, O = 0.f;
    for (int r0 = grp; r0 < nrec; r0 += 4 * 8) {
        float o[4], m[4], l[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = r0 + k * 8;
            const float* rec = base + size_t(r) * REC;
            o[k] = r < nrec ? __ldcg(rec + col) : 0.f;
            m[k] = r < nrec ? __ldcg(rec + kD) : -INFINITY;
            l[k] = r < nrec ? __ldcg(rec + kD + 1) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float sc = exp2f(m[k] - Mr);
            L += l[k] * sc;
            O += o[k] * sc;
        }
    }
    if (lane == 0) sL[grp] = L;
    sO[grp][lane] = O;
    __syncthreads();
    if (tid == 0 && atomicAdd(&U.comb_done, 1u) == uint32_t(p.G * kCombQ - 1)) {
        U.nrec = 0;
        U.comb_done = 0;
    }
    if (tid >= QC) return;
    float Lt = 0.f, Ot = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        Lt += sL[g];
        Ot += sO[g][tid];
    }
    const int b = u / p.Hkv, g = u - b * p.Hkv;
    const size_t row = size_t(b) * p.Hq + size_t(g) * p.G + hd;
    const int c = qt * QC + tid;
    const float val = Lt > 0.f ? Ot / Lt : 0.f;
    const __nv_bfloat16 bv = __float2bfloat16_rn(val);
    p.out[row * kD + c] = *reinterpret_cast<const uint16_t*>(&bv);
    if (p.out_f32) p.out_f32[row * kD + c] = val;
    if (p.lse && qt == 0 && tid == 0) p.lse[row] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
}

size_t fused_smem() { return sizeof(FShared); }

int fused_ctas() {
    static thread_local int dev = -1, ctas = 0;
    const DeviceInfo& di = device_info();
    if (dev != di.device) {
        int per_sm = 0;
        set_func_attr(reinterpret_cast<const void*>(decode_fused_kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                      int(fused_smem()));
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel, kFThreads, fused_smem()) !=
                cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            per_sm = 1;
        }
        ctas = di.num_sms * (per_sm < 2 ? per_sm : 2);
        dev = di.device;
    }
    return ctas;
}

struct FusedLayout {
    size_t counters, units, order, ready, above, off, scores, hist, cand, rec, total;
};

FusedLayout fused_layout(int U, int N, int G, int n_ctas) {
    const int NR = (N + kRRows - 1) / kRRows;
    FusedLayout l{};
    size_t o = 0;
    l.counters = o; o += align_up(sizeof(FCounters), 256);
    l.units = o; o += align_up(size_t(U) * sizeof(FUnit), 256);
    l.order = o; o += align_up(size_t(3) * U * 4, 256);
    l.ready = o; o += align_up(size_t(3) * U * 4, 256);
    l.above = o; o += align_up(size_t(U) * NR * 4, 256);
    l.off = o; o += align_up(size_t(U) * (NR + 1) * 4, 256);
    l.scores = o; o += align_up(size_t(U) * N * 4, 256);
    l.hist = o; o += hist0_bytes(U);
    l.cand = o; o += align_up(size_t(U) * N * 8, 256);
    l.rec = o; o += align_up(size_t(U) * G * n_ctas * (kD + 2) * 4, 256);
    l.total = o;
    return l;
}

}  // namespace

bool fused_decode_supported(const spa_decode_args* a) {
    if (a->score_kind != SPA_SCORE_LOWRANK || a->collapse != SPA_COLLAPSE_GROUP_MEAN) return false;
    if (a->local_units || a->rla_state || a->block > 1) return false;
    if (a->d != kD || a->r != 16) return false;
    const int G = a->Hq / a->Hkv;
    if (G < 1 || G > 8) return false;
    // long caches only: below this the separate kernels are as fast
    if (a->N < 16384 || a->N > (1 << 23)) return false;
    return a->B * a->Hkv <= 4096;
}

size_t fused_scratch_bytes(const spa_decode_args* a) {
    const int U = a->B * a->Hkv;
    return fused_layout(U, a->N, a->Hq / a->Hkv, fused_ctas()).total;
}

spa_status launch_fused_decode(const spa_decode_args* a, void* ws_after_header, uint32_t* status, cudaStream_t st,
                               void* const* events) {
    const int U = a->B * a->Hkv;
    const int G = a->Hq / a->Hkv;
    const int n_ctas = fused_ctas();
    const FusedLayout l = fused_layout(U, a->N, G, n_ctas);
    uint8_t* w = static_cast<uint8_t*>(ws_after_header);
    FusedParams p{};
    p.qidx = a->q_idx;
    p.kidx = reinterpret_cast<const uint4*>(a->Kidx);
    p.q = a->q; p.K = a->K; p.V = a->V;
    p.B = a->B; p.Hq = a->Hq; p.Hkv = a->Hkv; p.N = a->N; p.G = G;
    p.M = a->N;
    p.score_scale = a->score_scale; p.sm_scale = a->sm_scale;
    p.topp_mode = a->select_kind == SPA_SELECT_TOPP;
    p.topk = a->topk; p.topp = a->topp;
    p.sink = a->sink; p.window = a->window;
    p.idx = a->idx; p.count = a->count; p.cap = a->cap; p.index_mass = a->index_mass;
    p.out = a->out; p.out_f32 = a->out_f32; p.lse = a->lse;
    p.status = status;
    p.ctr = reinterpret_cast<FCounters*>(w + l.counters);
    p.unit = reinterpret_cast<FUnit*>(w + l.units);
    p.order = reinterpret_cast<uint32_t*>(w + l.order);
    p.ready = reinterpret_cast<uint32_t*>(w + l.ready);
    p.rng_above = reinterpret_cast<uint32_t*>(w + l.above);
    p.rng_off = reinterpret_cast<uint32_t*>(w + l.off);
    p.scores = reinterpret_cast<float*>(w + l.scores);
    p.hist = hist0_carve(w + l.hist, U);
    p.cand = reinterpret_cast<uint2*>(w + l.cand);
    p.rec = reinterpret_cast<float*>(w + l.rec);
    p.U = U;
    p.nS = (a->N + kSRows - 1) / kSRows;
    p.NR = (a->N + kRRows - 1) / kRRows;
    p.n_ctas = n_ctas;
    // a few CTAs never gather, so the selection chains of the last units are not held up
    // behind gather tiles
    p.n_sel = U < 16 ? U : 16;
    if (p.NR > 1024) return SPA_ERR_UNSUPPORTED_SHAPE;
    const size_t smem = fused_smem();
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(decode_fused_kernel),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    if (events) SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[0]), st));
    SPA_CUDA_TRY(launch_pdl(decode_fused_kernel, dim3(n_ctas), dim3(kFThreads), smem, st, p));
    if (events) {
        SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[1]), st));
        SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[2]), st));
    }
    SPA_CUDA_TRY(launch_pdl(fused_combine_kernel, dim3(U, G, kCombQ), dim3(256), 0, st, p));
    if (events) SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[3]), st));
    return SPA_OK;
}

}  // namespace spa
