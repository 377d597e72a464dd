// Internal declarations shared by the translation units of libspa.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>

#include "../../include/spa.h"

namespace spa {

// ------------------------------------------------------------------ workspace header
// Every workspace starts with a 256-byte header; word 0 is the device status word
// (OR of 1 << SPA_ERR_* raised on the device).
constexpr size_t kWsHeader = 256;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ device facts
struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    int max_smem_optin = 0;   // bytes of dynamic shared memory a CTA may opt in to
    int cc_major = 0, cc_minor = 0;
};
// Cached per device; safe to call from several host threads.
const DeviceInfo& device_info();

// Kernel attributes and occupancy queries are driver calls of microseconds each, made with the
// same values on every launch; both are memoised per device (safe from several host threads).
// set_func_attr calls cudaFuncSetAttribute only when the value differs from the last one set.
cudaError_t set_func_attr(const void* func, cudaFuncAttribute attr, int value);
// CTAs of func per SM at this block size and dynamic shared memory (0 if the query fails).
int occupancy_blocks(const void* func, int threads, size_t smem);

// Records the CUDA error (thread-local text for spa_last_cuda_error) and maps it to a status.
spa_status cuda_fail(cudaError_t e);

#define SPA_CUDA_TRY(expr)                          \
    do {                                            \
        cudaError_t _e = (expr);                    \
        if (_e != cudaSuccess) return cuda_fail(_e); \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ order-preserving keys
// Maps a binary32 score to a uint32 whose unsigned order is the numeric order of the
// scores (negatives reversed, sign bit flipped for non-negatives).
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// ------------------------------------------------------------------ level-0 selection histogram
// Per unit: 2048 bins over the top 11 bits of the score keys.  Each bin holds its count
// and a 64-bit fixed-point mass sum_n round(2^40 exp(s_n - r_b)), where r_b is the largest
// score a key of bin b can hold, so the sums need no knowledge of the unit's maximum and
// are exact integers whatever the order of accumulation; plus the unit's largest key.
// Producers (the fused scoring kernel, or the histogram kernel) add into it; the selection
// kernel reads it and zeroes it again for the next call, likewise the finer levels' merged
// histograms it keeps beside it.
constexpr int kHistBins = 2048;
constexpr float kMassScale = 1099511627776.0f;   // 2^40

struct Hist0 {
    uint32_t* cnt;                 // [U][2048]
    unsigned long long* mass;      // [U][2048]
    uint32_t* max_key;             // [U]
    // the selection kernel's merged level-1 (2048 bins) and level-2 (1024 bins) histograms
    uint32_t* lvl_cnt;             // [U][3072]
    unsigned long long* lvl_mass;  // [U][3072]
};
constexpr int kLvlBins = 3072;
inline size_t hist0_bytes(int U) {
    return align_up(size_t(U) * kHistBins * 4, 256) + align_up(size_t(U) * kHistBins * 8, 256) +
           align_up(size_t(U) * 4, 256) + align_up(size_t(U) * kLvlBins * 4, 256) +
           align_up(size_t(U) * kLvlBins * 8, 256);
}
inline Hist0 hist0_carve(void* base, int U) {
    uint8_t* b = static_cast<uint8_t*>(base);
    Hist0 h;
    h.cnt = reinterpret_cast<uint32_t*>(b);
    b += align_up(size_t(U) * kHistBins * 4, 256);
    h.mass = reinterpret_cast<unsigned long long*>(b);
    b += align_up(size_t(U) * kHistBins * 8, 256);
    h.max_key = reinterpret_cast<uint32_t*>(b);
    b += align_up(size_t(U) * 4, 256);
    h.lvl_cnt = reinterpret_cast<uint32_t*>(b);
    b += align_up(size_t(U) * kLvlBins * 4, 256);
    h.lvl_mass = reinterpret_cast<unsigned long long*>(b);
    return h;
}
// largest score a key of level-0 bin b can hold (bin 2047 holds only +inf/NaN patterns)
__device__ __forceinline__ float bin_top_score(uint32_t b) {
    return b >= 2047u ? 3.402823466e38f : key_score(((b + 1u) << 21) - 1u);
}
// round(2^40 e^(s - ref)) for s <= ref, with the MUFU exponential (about 2^-22 relative; the
// level-0 and in-bin masses of every kernel use this one function, so they agree exactly)
__device__ __forceinline__ unsigned long long fixed_mass(float s, float ref) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"((s - ref) * 1.4426950408889634f));
    return __float2ull_rn(e * kMassScale);
}

// ------------------------------------------------------------------ level-0 crossing bin
// Shared by the cluster selection kernel and the fused decode kernel, so both take the same
// decision from the same histogram: the first 256 threads of the block own 256 groups of 8
// bins (descending from the top bin), every sum runs in a fixed order independent of the
// block size (within a group, then a warp scan over the groups, then the warps in order).
// Top-p: the crossing bin is the first (from the top) where the cumulative mass
// sum_b mass_b * 2^-40 * exp(r_b - m) reaches p * Z; should fp64 rounding keep every
// cumulative sum below p * Z, the lowest non-empty bin is taken (everything is needed).
// Top-k: the first bin where the cumulative count reaches k (exact).
struct Level0Shared {
    uint32_t wc[8];
    double wm[8];
    uint32_t bin, above_cnt, bmin, hit;
    uint32_t fb_above_cnt;
    double above_mass, fb_above_mass;
};
struct Level0 {
    uint32_t bin, above_cnt;
    double above_mass, Z;
};
// blockDim.x >= 256 and a multiple of 32; every thread of the block must call it
__device__ inline Level0 level0_crossing(const uint32_t* hc, const unsigned long long* hm, uint32_t max_key, bool topp,
                                         float p, int k, Level0Shared& sh) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float m = key_score(max_key);
    const bool act = tid < 256;
    uint32_t vc[8];
    unsigned long long mb[8];
    double vm[8];
    uint32_t gc = 0;
    double gm = 0.0;
    // every load of the thread is issued before any is used
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int bin = 2047 - (tid * 8 + j);
        vc[j] = act ? __ldcg(hc + bin) : 0u;
        mb[j] = act && topp ? __ldcg(hm + bin) : 0ull;
    }
    if (tid == 0) {
        sh.bin = max_key >> 21;
        sh.above_cnt = 0;
        sh.above_mass = 0.0;
        sh.bmin = 2048u;
        sh.hit = 0;
        sh.fb_above_cnt = 0;
        sh.fb_above_mass = 0.0;
    }
    __syncthreads();
    uint32_t my_min = 2048u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int bin = 2047 - (tid * 8 + j);
        vm[j] = mb[j] ? double(mb[j]) * (1.0 / 1099511627776.0) * exp(double(bin_top_score(bin)) - double(m)) : 0.0;
        if (vc[j]) my_min = min(my_min, uint32_t(bin));
        gc += vc[j];
        gm += vm[j];
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) my_min = min(my_min, __shfl_xor_sync(0xffffffffu, my_min, off));
    if (lane == 0 && my_min < 2048u) atomicMin(&sh.bmin, my_min);
    // inclusive scan over the groups of this warp, in group order
    uint32_t ic = gc;
    double im = gm;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t xc = __shfl_up_sync(0xffffffffu, ic, off);
        const double xm = __shfl_up_sync(0xffffffffu, im, off);
        if (lane >= off) { ic += xc; im += xm; }
    }
    if (act && lane == 31) { sh.wc[warp] = ic; sh.wm[warp] = im; }
    __syncthreads();
    uint32_t pc = 0, tc = 0;
    double pm = 0.0, tm = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        if (w < warp) { pc += sh.wc[w]; pm += sh.wm[w]; }
        tc += sh.wc[w];
        tm += sh.wm[w];
    }
    const double T = double(p) * tm;
    uint32_t ac = pc + ic - gc;
    double am = pm + im - gm;
    if (act) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t bin = uint32_t(2047 - (tid * 8 + j));
            const bool hit = topp ? (am < T && am + vm[j] >= T) : (ac < uint32_t(k) && ac + vc[j] >= uint32_t(k));
            if (hit) {
                sh.bin = bin;
                sh.above_cnt = ac;
                sh.above_mass = am;
                sh.hit = 1;
            }
            if (bin == sh.bmin) {   // bmin is final here (set before the barrier above)
                sh.fb_above_cnt = ac;
                sh.fb_above_mass = am;
            }
            ac += vc[j];
            am += vm[j];
        }
    }
    __syncthreads();
    Level0 r;
    if (!sh.hit && topp && sh.bmin < 2048u) {
        r.bin = sh.bmin;
        r.above_cnt = sh.fb_above_cnt;
        r.above_mass = sh.fb_above_mass;
    } else {
        r.bin = sh.bin;
        r.above_cnt = sh.above_cnt;
        r.above_mass = sh.above_mass;
    }
    r.Z = tm;
    __syncthreads();
    return r;
}

__device__ __forceinline__ void raise_status(uint32_t* status, int code) {
    if (status) atomicOr(status, 1u << code);
}

// ------------------------------------------------------------------ programmatic dependent launch
// Every kernel of the library is launched with programmatic stream serialization, so the
// hardware may schedule it while the previous kernel of the stream is still draining.  Its
// first statement waits until that kernel has completed and its memory is visible (a no-op
// when there is none), and then lets the next kernel be scheduled likewise: dependents
// become launchable only once every CTA of this grid has started, so CTAs waiting here never
// hold back a CTA of the grid they wait for.
__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ launchers
// scores.cu
// hist (optional, GROUP_MEAN only): also accumulate the level-0 histogram of the scores;
// with_mass adds the fixed-point masses (top-p), else counts only.
// local (optional, GROUP_MEAN): [B * Hkv] flags of units that are not scored (head-wise routing)
// kv_shared: the key set [Hkv][M] is shared by every batch row (per-query prefill), else [B][Hkv][M]
spa_status launch_lowrank_scores(const uint16_t* qidx, const uint16_t* kidx, int B, int Hq, int Hkv, int M,
                                 int collapse, float scale, float* scores, const Hist0* hist, bool with_mass,
                                 cudaStream_t st, const uint8_t* local = nullptr, bool kv_shared = false);
// kind: SPA_SCORE_TAYLOR_BLOCK (mean, var), SPA_SCORE_MINMAX_BLOCK (min, max) or
// SPA_SCORE_MEAN_BLOCK (mean; var not read); stats_bf16: the statistics are bf16, else fp32
spa_status launch_taylor_scores(const uint16_t* q, const void* mean, const void* var, int B, int Hq, int Hkv,
                                int M, int d, int collapse, float scale, float* scores, cudaStream_t st,
                                const uint8_t* local = nullptr, int kind = SPA_SCORE_TAYLOR_BLOCK,
                                bool stats_bf16 = false);
// out_bf16: write the statistics as bf16 (round to nearest even), else fp32
spa_status launch_block_stats(const uint16_t* K, int B, int Hkv, int N, int d, int block, void* mean,
                              void* var, bool out_bf16, cudaStream_t st);
spa_status launch_block_minmax(const uint16_t* K, int B, int Hkv, int N, int d, int block, void* mn, void* mx,
                               bool out_bf16, cudaStream_t st);

// select.cu
struct SelectParams {
    Hist0 hist;        // level-0 histogram (filled by launch_hist0 or the fused scorer)
    const float* scores;
    const int32_t* unit_len;
    int U, M;
    int topk;          // SPA_SELECT_TOPK
    float topp;        // SPA_SELECT_TOPP
    int sink, window;
    int32_t* idx;
    int32_t* count;
    int cap;
    float* index_mass;
    uint32_t* status;
    const uint8_t* local;   // [U] or null: local units (head-wise routing) select only sink + window
    int test_stall;         // SPA_TEST_STALL_* bits armed by spa_test_stall (test hook), else 0
};
spa_status launch_hist0(const SelectParams& p, bool with_mass, cudaStream_t st);
spa_status launch_select(const SelectParams& p, bool topp, cudaStream_t st);
size_t select_scratch_bytes(int U);

// rla.cu: adds rows [n0, n1) of every (batch, kv head) into S [B*Hkv][d][d] and z [B*Hkv][d]
spa_status launch_rla_state(const uint16_t* K, const uint16_t* V, int BH, int N, int d, int n0, int n1, float* S,
                            float* z, cudaStream_t st);

// prefill.cu
size_t prefill_scratch_bytes(int U, int N);
// events (optional, 2): recorded on st right before and right after the attention kernel
spa_status launch_prefill(const spa_prefill_args* a, void* ws, cudaStream_t st, void* const* events = nullptr);
// The tcgen05 attention of 64-query blocks: unit u = block * Hkv + g attends, for each of its 64
// queries (positions q_start + block * 64 + i) and G heads, to the rows idx[u][0 .. count[u])
// and to the block's own positions up to the query (causal).  d = 128, G even.
struct PrefillAttendParams {
    const uint16_t* Q;     // [T, Hq, d]
    const uint16_t* K;     // [Hkv, N, d]
    const uint16_t* V;
    const int32_t* idx;    // [U, cap]
    const int32_t* count;  // [U]
    int cap;
    int Hq, Hkv, N, bq, q_start;
    float sm_scale;
    uint16_t* out;         // [T, Hq, d]
    float* out_f32;
    uint32_t* status;
    int test_stall;        // SPA_TEST_STALL_* bits (test hook), else 0
};
spa_status launch_prefill_attend(const PrefillAttendParams& pp, int U, cudaStream_t st,
                                 void* const* events = nullptr);

// The test hook's armed bits (spa_test_stall), read by the launchers.
int test_stall_bits();

// fused.cu: the persistent dataflow decode (low-rank, head-collapsed, d = 128, G <= 8)
bool fused_decode_supported(const spa_decode_args* a);
size_t fused_scratch_bytes(const spa_decode_args* a);
// events (optional, 4): before the fused kernel, after it (twice), after the combine kernel
spa_status launch_fused_decode(const spa_decode_args* a, void* ws_after_header, uint32_t* status, cudaStream_t st,
                               void* const* events);

// attend.cu
struct AttendParams {
    const uint16_t* q;
    const uint16_t* K;
    const uint16_t* V;
    int B, Hq, Hkv, N, d;
    const int32_t* idx;
    const int32_t* count;
    int cap;
    int collapse;
    int unit_tokens;
    float sm_scale;
    uint16_t* out;
    float* out_f32;
    float* lse;
    // workspace pieces
    int* unit_ctas;    // [U][2]: first and last CTA of a unit split over several CTAs, else -1
    float* partials;   // [(U + grid) * heads_per_unit * (d + 2)]; the RLA partials follow
    uint32_t* status;
    // kv_shared: K and V are [Hkv, N, d], shared by every batch row (per-query prefill)
    int kv_shared;
    // residual linear attention (null rla_S: off): state S [B*Hkv][d][d], z [B*Hkv][d],
    // RMSNorm scale gamma [Hq][d] and epsilon
    const float* rla_S;
    const float* rla_z;
    const float* rla_gamma;
    float rla_eps;
};
size_t attend_scratch_bytes(int U, int heads_per_unit, int d);   // unit CTA ranges + partials
int attend_grid();
spa_status launch_attend(const AttendParams& p, cudaStream_t st);

}  // namespace spa
