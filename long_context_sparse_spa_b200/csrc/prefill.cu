// Selection-block-shared sparse prefill ("Oracle-Guided Sparse Prefill" 2.1, b_sel = 64:
// one support for 64 consecutive queries; 2.2: head-collapsed indexer).
//
// For each block of bq = 64 queries at positions t0 .. t0+63 and each kv head g:
//   1. the index query is the mean of the block's index queries over its 64 queries and
//      the G query heads of g (prefill_qhat_kernel);
//   2. every candidate key n < t0 is scored against it (prefill_scores_kernel: one CTA
//      scores a chunk of keys of one kv head for all query blocks at once, so each index
//      key is read once);
//   3. the support is the exact top-k of those scores united with the sink [0, sink)
//      (the top-k selection kernels, with per-unit candidate length t0);
//   4. every query row (query t0 + i, head h of g) attends with the original Q, K, V to
//      the support plus its own block's causal prefix [t0, t0 + i] (prefill_attend_kernel).
//
// Step 4 is a dense contraction (64 queries x G heads share each support) and runs on the
// 5th-generation tensor cores: tcgen05.mma with operands in shared memory (128-byte
// swizzled, one 128-byte line per row of 64 bf16), fp32 accumulators in tensor memory
// (TMEM), issued by one thread and completed through mbarriers.  One CTA owns 128 query
// rows (two heads x 64 queries).  Keys are processed in tiles of 128 gathered rows
// (cp.async, bounds-checked) plus the diagonal tile of the block's own 64 positions, in one
// pass with an online softmax (see the attention section below).
#include "internal.cuh"
#include "tc.cuh"

namespace spa {
namespace {
using namespace tc;

constexpr int kPfRows = 128;          // query rows per CTA (tensor-core M)
constexpr int kPfKeys = 128;          // keys per tile (tensor-core N of S, K of P V)
constexpr uint32_t kSpinLimit = 1u << 22;   // bounded mbarrier polls before giving up
constexpr float kLog2e = 1.4426950408889634f;

// ============================================================================ index query
// qhat[u][0..15] (fp32) = mean over the block's bq queries and G heads of q_idx; also
// unit_len[u] = t0, the number of candidate keys.  One CTA per unit: thread j takes the rows
// (query, head) = j, j + 256, ... (in (query, head) order) as two 16-byte loads each, and the
// partial sums are added in a fixed tree (lanes, then warps in order), so the result does not
// depend on scheduling.
__global__ void __launch_bounds__(256)
prefill_qhat_kernel(const uint16_t* __restrict__ qidx, int Hq, int Hkv, int bq, int q_start,
                    float* __restrict__ qhat, int32_t* __restrict__ unit_len, int U) {
    pdl_enter();
    __shared__ float part[8][16];
    const int u = blockIdx.x;
    if (u >= U) return;
    const int blk = u / Hkv, g = u - blk * Hkv;
    const int G = Hq / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = 0.f;
    for (int j = tid; j < bq * G; j += 256) {
        const int i = j / G, h = j - i * G;
        const uint4* row = reinterpret_cast<const uint4*>(qidx + (size_t(blk * bq + i) * Hq + g * G + h) * 16);
        const uint4 w0 = __ldg(row), w1 = __ldg(row + 1);
        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            acc[2 * k] += __uint_as_float(ws[k] << 16);
            acc[2 * k + 1] += __uint_as_float(ws[k] & 0xffff0000u);
        }
    }
#pragma unroll
    for (int c = 0; c < 16; ++c)
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], off);
    if (lane == 0)
#pragma unroll
        for (int c = 0; c < 16; ++c) part[warp][c] = acc[c];
    __syncthreads();
    if (tid < 16) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += part[w][tid];
        qhat[u * 16 + tid] = t / float(bq * G);
    }
    if (tid == 0) unit_len[u] = q_start + blk * bq;
}

// ============================================================================ scores
// grid (key chunks, Hkv); each thread scores one key against the index queries of every
// query block of its kv head (kept in shared memory); keys at or after a block's t0 are
// not scored for it.
constexpr int kPsThreads = 256;
constexpr int kPsMaxBlocks = 128;
__global__ void __launch_bounds__(kPsThreads)
prefill_scores_kernel(const float* __restrict__ qhat, const int32_t* __restrict__ unit_len,
                      const uint4* __restrict__ kidx, int Hkv, int N, int n_blocks, float scale,
                      float* __restrict__ scores) {
    pdl_enter();
    __shared__ float qs[kPsMaxBlocks][16];
    __shared__ int t0s[kPsMaxBlocks];
    const int g = blockIdx.y;
    for (int i = threadIdx.x; i < n_blocks * 16; i += kPsThreads) {
        const int blk = i / 16;
        qs[blk][i & 15] = qhat[(blk * Hkv + g) * 16 + (i & 15)];
        if ((i & 15) == 0) t0s[blk] = unit_len[blk * Hkv + g];
    }
    __syncthreads();
    const int n = blockIdx.x * kPsThreads + threadIdx.x;
    if (n >= N) return;
    const uint4 w0 = __ldg(kidx + (size_t(g) * N + n) * 2), w1 = __ldg(kidx + (size_t(g) * N + n) * 2 + 1);
    const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float k[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        k[2 * j] = __uint_as_float(ws[j] << 16);
        k[2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
    }
    for (int blk = 0; blk < n_blocks; ++blk) {
        if (n >= t0s[blk]) continue;
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) dot = fmaf(qs[blk][j], k[j], dot);
        scores[size_t(blk * Hkv + g) * N + n] = scale * dot;
    }
}

// ============================================================================ attention
// One pass with an online softmax, pipelined.
//   * 8 warps.  Warp w reads TMEM lanes 32 (w % 4) .. +31 (its 32 query rows) and owns key
//     columns 64 (w / 4) .. +63 of every S tile.  Each (row, column half) keeps its own running
//     maximum m, sum l and output accumulator (O_a over the first 64 keys of every tile, O_b over
//     the last 64), so the softmax exchanges nothing between threads until the epilogue merges
//     the halves: O = (2^(m_a - m) O_a + 2^(m_b - m) O_b) / (2^(m_a - m) l_a + 2^(m_b - m) l_b).
//   * A half's maximum moves (and its O is rescaled through TMEM) only when a tile's maximum
//     exceeds it by more than kRescaleLog2, so P = 2^(S - m) <= 2^kRescaleLog2; the result is the
//     same softmax for any such m.  P enters the MMA as bf16 hi + lo (two MMAs), ~16 bits.
//   * S is double-buffered in TMEM: S(t+1) = Q K(t+1)^T runs on the tensor cores while the
//     threads turn S(t) into P(t), and O += P(t) V(t) runs while they read S(t+1).
//   * K and V tiles are double-buffered in shared memory and gathered one tile ahead: K of tile
//     t+2 as soon as S(t) has consumed its buffer, V of tile t+1 as soon as P(t-1) V(t-1) has.
//     Every thread commits one cp.async group per gather point, empty or not, so the group
//     counts of the waits are the same in every iteration.
// TMEM columns: S buffers 0..127 and 128..255, O_a 256..383, O_b 384..511.
constexpr int kPfSoft = 256;               // warps 0-7: gathers and softmax
constexpr int kPfThreads = kPfSoft + 32;   // + warp 8, whose lane 0 issues the MMAs
constexpr float kRescaleLog2 = 8.f;

// (the operand tiles sit at multiples of 32 KB from the 1024-byte aligned start of dynamic shared
// memory, as the 128-byte swizzle needs; the struct itself is not padded to 1024 bytes, which
// keeps it under the 227 KB a CTA may use)
struct PfShared {
    uint8_t q[kTileBytes];
    uint8_t k[2][kTileBytes];
    uint8_t v[2][kTileBytes];
    uint8_t p_hi[kTileBytes];   // the epilogue reuses it for the halves' (m, l)
    uint8_t p_lo[kTileBytes];
    uint64_t bar_s, bar_o;      // completion of the S MMAs / of the P V MMAs (tcgen05.commit)
    uint64_t k_ready;           // the 256 softmax threads: the next tile's keys are in place (and S read)
    uint64_t p_ready;           // the 256 softmax threads: P(t) stored and V(t) in place
    uint32_t tmem_base;
    uint32_t n_s, n_o;          // commits the issuer made on bar_s / bar_o
    uint32_t valid[4][kPfKeys / 32];   // bit c: key c of tile t (slot t % 4) is attended
    int rows[4][kPfKeys];              // cache rows of tile t's keys (slot t % 4), -1 for none
};
static_assert(sizeof(PfShared) <= 227 * 1024, "prefill attention: shared memory over the per-CTA limit");

// paired fp32 arithmetic (one instruction for two lanes of a 64-bit register pair)
__device__ __forceinline__ void ffma2(float& r0, float& r1, float a0, float a1, float b0, float b1, float c0, float c1) {
    asm("{\n .reg .b64 a, b, c, d;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n mov.b64 c, {%6, %7};\n"
        " fma.rn.f32x2 d, a, b, c;\n mov.b64 {%0, %1}, d;\n}\n"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n .reg .b64 a, b, d;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n add.f32x2 d, a, b;\n"
        " mov.b64 {%0, %1}, d;\n}\n"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// named barrier 1 of the 256 softmax threads (the issuing warp never joins it)
__device__ __forceinline__ void soft_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
// the same barrier, returning the OR of v over the 256 threads
__device__ __forceinline__ bool soft_sync_or(bool v) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
                 : "=r"(r)
                 : "r"(uint32_t(v))
                 : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// grid (U, G / 2): one CTA per (unit, pair of query heads); 288 threads.  Warps 0-7 gather and run
// the softmax; lane 0 of warp 8 issues every MMA.  The two sides meet only at mbarriers: the
// softmax warps arrive on k_ready once the next tile's keys have landed (and the S buffer they
// overwrite was read) and on p_ready once P(t) is stored and V(t) has landed; the issuer waits
// on those and the softmax warps on the MMAs' commits.  So an MMA issue that waits for room in the
// tensor core's queue delays no softmax warp, and the softmax warps share one named barrier per
// tile (row staging, and the decision to stop after a bounded wait gave up).
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_attend_kernel(PrefillAttendParams p) {
    pdl_enter();
    extern __shared__ __align__(1024) uint8_t dyn[];
    PfShared& sh = *reinterpret_cast<PfShared*>(dyn);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool issuer_warp = warp == kPfSoft / 32;
    const int u = blockIdx.x, pair = blockIdx.y;
    const int blk = u / p.Hkv, g = u - blk * p.Hkv;
    const int G = p.Hq / p.Hkv;
    const int t0 = p.q_start + blk * p.bq;
    int n_sup = p.count[u];
    n_sup = n_sup < 0 ? 0 : (n_sup > p.cap ? p.cap : n_sup);
    const int n_gather = (n_sup + kPfKeys - 1) / kPfKeys;
    const int n_tiles = n_gather + 1;                          // + the diagonal tile
    const int32_t* sup = p.idx + size_t(u) * p.cap;
    const size_t kv0 = size_t(g) * p.N;

    // softmax role: query row r (TMEM lane) and key-column half
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int r = quad * 32 + lane, qi = r & 63;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;

    if (warp == 0) tmem_alloc(&sh.tmem_base, 512);
    if (tid == 0) {
        mbar_init(&sh.bar_s, 1);
        mbar_init(&sh.bar_o, 1);
        mbar_init(&sh.k_ready, kPfSoft);
        mbar_init(&sh.p_ready, kPfSoft);
        sh.n_s = 0;
        sh.n_o = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }

    // cache row of key rr of tile t, or -1 (outside the support, or out of range)
    auto key_row = [&](int t, int rr) -> int {
        if (t < n_gather) {
            const int e = t * kPfKeys + rr;
            if (e >= n_sup) return -1;
            const int n = __ldg(sup + e);
            return (n >= 0 && n < p.N) ? n : -1;
        }
        const int n = t0 + rr;                                 // the diagonal tile: the block's own keys
        return (rr < p.bq && n < p.N) ? n : -1;
    };
    // tile t's cache rows and key mask into slot t % 4 (threads 0..127, one key each); the value
    // comes from a register loaded earlier, so the load's latency is not waited for here
    auto stage_rows = [&](int t, int row) {
        if (t < n_tiles && warp < 4) {
            sh.rows[t & 3][tid] = row;
            const uint32_t b = __ballot_sync(0xffffffffu, row >= 0);
            if (lane == 0) sh.valid[t & 3][warp] = b;
        }
    };
    // 128 rows x 16 chunks of 16 bytes; softmax thread tid copies chunk tid % 16 of rows tid / 16 + 16 j
    auto gather = [&](const uint16_t* src, uint8_t* dst, int t) {
        const int c = tid & 15;
#pragma unroll
        for (int j = 0; j < kPfKeys / 16; ++j) {
            const int rr = j * 16 + (tid >> 4);
            const int row = sh.rows[t & 3][rr];
            const bool ok = row >= 0;
            cp_async16(smem_u32(dst) + tile_off(rr, c), src + (ok ? (kv0 + size_t(row)) * 128 + c * 8 : 0), ok);
        }
    };
    auto gather_k = [&](int t) {
        if (t < n_tiles) gather(p.K, sh.k[t & 1], t);
        cp_async_commit();
    };
    auto gather_v = [&](int t) {
        if (t < n_tiles) gather(p.V, sh.v[t & 1], t);
        cp_async_commit();
    };

    // the test hook stalls the first S = Q K^T: its completion barrier waits for an MMA that
    // is never issued, so the bounded waits run out with nothing in flight
    const bool stall = (p.test_stall & SPA_TEST_STALL_PREFILL_MMA) != 0;
    const uint32_t spin_limit = stall ? 1024u : kSpinLimit;
    const float sl2 = p.sm_scale * kLog2e;
    constexpr uint32_t kIdS = idesc_bf16(kPfRows, kPfKeys, false);
    constexpr uint32_t kIdO = idesc_bf16(kPfRows, 128, true);

    tc_fence_before();
    __syncthreads();                                           // barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const uint32_t t_oa = tmem + 256;

    // bounded wait on a barrier phase; on expiry this thread's flag is set
    bool my_to = false;
    auto wait_bar = [&](uint64_t* bar, uint32_t& ph) -> bool {
        uint32_t it = 0;
        while (!mbar_try_wait(bar, ph)) {
            if (++it >= spin_limit) {
                my_to = true;
                return false;
            }
        }
        ph ^= 1u;
        tc_fence_after();
        return true;
    };

    uint32_t seen_s = 0, seen_o = 0;       // completions of bar_s / bar_o this thread observed
    uint32_t ph_s = 0, ph_o = 0;
    float m_run = -INFINITY, l_run = 0.f;

    if (issuer_warp) {
        if (lane == 0) {
            // Operand descriptors, built once: a k-step moves the start address, the descriptor's
            // low 14 bits (address / 16, below 2^14 for any shared-memory address), one 64-bit add.
            const uint64_t d_q = sw128_desc(smem_u32(sh.q), 16, 1024);
            const uint64_t d_k0 = sw128_desc(smem_u32(sh.k[0]), 16, 1024), d_k1 = sw128_desc(smem_u32(sh.k[1]), 16, 1024);
            const uint64_t d_v0 = sw128_desc(smem_u32(sh.v[0]), kSlab, 1024);
            const uint64_t d_v1 = sw128_desc(smem_u32(sh.v[1]), kSlab, 1024);
            const uint64_t d_ph = sw128_desc(smem_u32(sh.p_hi), 16, 1024), d_pl = sw128_desc(smem_u32(sh.p_lo), 16, 1024);
            auto issue_s = [&](int t) {                        // S(t) = Q K(t)^T into S buffer t % 2
                const uint32_t d = tmem + uint32_t(t & 1) * 128;
                const uint64_t dk = (t & 1) ? d_k1 : d_k0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = uint64_t(((kk >> 2) * kSlab + (kk & 3) * 32) >> 4);
                    umma_bf16(d, d_q + off, dk + off, kIdS, kk > 0);
                }
                umma_commit(&sh.bar_s);
            };
            auto issue_pv = [&](int t) {                       // O_a += P[:, 0:64] V(t)[0:64], O_b += the rest
                const uint64_t dv = (t & 1) ? d_v1 : d_v0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t d = t_oa + uint32_t(kk >> 2) * 128;
                    const uint64_t aoff = uint64_t(((kk >> 2) * kSlab + (kk & 3) * 32) >> 4);
                    const uint64_t bv = dv + uint64_t((kk * 2048) >> 4);
                    umma_bf16(d, d_ph + aoff, bv, kIdO, (t > 0 || (kk & 3) > 0) ? 1u : 0u);
                    umma_bf16(d, d_pl + aoff, bv, kIdO, 1u);
                }
                umma_commit(&sh.bar_o);
            };
            // S(t + 1) is issued before P(t) V(t): the softmax of tile t + 1 needs it first
            uint32_t pk = 0, pp = 0;
            bool live = wait_bar(&sh.k_ready, pk);             // Q and tile 0's keys
            if (live && !stall) {
                issue_s(0);
                sh.n_s = 1;
            }
            for (int t = 0; live && t < n_tiles; ++t) {
                if (t + 1 < n_tiles) {
                    if (!wait_bar(&sh.k_ready, pk)) break;
                    issue_s(t + 1);
                    sh.n_s = uint32_t(t + 2);
                }
                if (!wait_bar(&sh.p_ready, pp)) break;
                issue_pv(t);
                sh.n_o = uint32_t(t + 1);
            }
        }
    } else {
        // Q tile (row rr: head 2 pair + rr / 64, query rr % 64 of the block), in K(0)'s group
#pragma unroll
        for (int j = 0; j < kPfRows / 16; ++j) {
            const int rr = j * 16 + (tid >> 4), c = tid & 15;
            const size_t qrow = size_t(blk * p.bq + (rr & 63)) * p.Hq + g * G + 2 * pair + rr / 64;
            cp_async16(smem_u32(sh.q) + tile_off(rr, c), p.Q + qrow * 128 + c * 8, true);
        }
        // rows of tiles 0..2; tile t + 3 is staged during iteration t
#pragma unroll
        for (int t = 0; t < 3; ++t) stage_rows(t, tid < kPfKeys ? key_row(t, tid) : -1);
        soft_sync();
        gather_k(0);
        gather_k(1);
        gather_v(0);
        cp_async_wait_group<2>();                              // Q and K(0)
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.k_ready);
        const uint32_t t_my_o = t_oa + uint32_t(half) * 128 + lane_off;

        for (int t = 0; t < n_tiles; ++t) {
            // S(t) is complete: its K buffer takes tile t + 2 (ok is made warp-uniform: the
            // stores below hold warp votes)
            bool ok = !my_to && wait_bar(&sh.bar_s, ph_s);
            if (ok) ++seen_s;
            ok = __all_sync(0xffffffffu, ok);
            if (ok) gather_k(t + 2);
            else cp_async_commit();
            cp_async_wait_group<2>();                          // K(t + 1) has landed
            if (ok && t + 1 < n_tiles) {                       // ... for the issuer's S(t + 1)
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&sh.k_ready);
            }
            // rows of tile t + 3: the load is issued now and stored before the next barrier
            const int row_pf = (tid < kPfKeys && t + 3 < n_tiles) ? key_row(t + 3, tid) : -1;

            bool rescale = false;
            float alpha = 1.f;
            // this thread's 64 logits of S(t) are read from TMEM twice, 32 at a time: for the
            // tile's maximum now, and for P after P(t-1) V(t-1) is complete (the issuer rewrites
            // the buffer only after this thread's next arrival on k_ready)
            const uint32_t ta = tmem + uint32_t(t & 1) * 128 + uint32_t(half) * 64 + lane_off;
            const uint32_t vm0 = sh.valid[t & 3][2 * half], vm1 = sh.valid[t & 3][2 * half + 1];
            // masked keys become -inf.  A full tile of support keys (every tile but the last partial
            // one and the diagonal) needs no mask: the test is warp-uniform
            const bool full = t < n_gather && (vm0 & vm1) == 0xffffffffu;
            const int causal = t < n_gather ? kPfKeys : qi - half * 64;   // diagonal tile: key c <= qi
            auto logits32 = [&](int q2, float (&v)[32]) {
                tmem_ld32(ta + uint32_t(q2) * 32, v);
                if (!full) {
                    const uint32_t vm = q2 ? vm1 : vm0;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const bool valid = ((vm >> i) & 1u) && q2 * 32 + i <= causal;
                        v[i] = valid ? v[i] : -INFINITY;
                    }
                }
            };
            if (ok) {
                // tile maximum in four independent chains, then in log2 units (sm_scale > 0)
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    float v[32];
                    logits32(q2, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], v[i]);
                }
                const float tmax = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
                if (tmax > m_run + kRescaleLog2) {             // also the first finite maximum
                    alpha = ex2_approx(m_run - tmax);
                    rescale = m_run != -INFINITY;               // O of this half holds nonzero terms
                    m_run = tmax;
                    l_run *= alpha;
                }
            }

            // P(t-1) V(t-1) is complete: P, O and its V buffer are free
            bool ok2 = ok && (t == 0 || wait_bar(&sh.bar_o, ph_o));
            if (ok2 && t > 0) ++seen_o;
            ok2 = __all_sync(0xffffffffu, ok2);
            if (ok2) {
                // tcgen05.ld / st are warp-collective: a warp rescales when any of its rows needs
                // it, the other rows by 1
                if (__any_sync(0xffffffffu, rescale)) {
                    const float a = rescale ? alpha : 1.f;
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        float v[32];
                        tmem_ld32(t_my_o + cb * 32, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= a;
                        tmem_st32(t_my_o + cb * 32, v);
                    }
                    tmem_wait_st();
                }
                // P = 2^(sl2 s - m) as bf16 hi + lo, stored 8 keys at a time (masked keys give
                // 2^-inf = 0; while no key has been seen m is -inf and every logit is -inf, so the
                // reference 0 gives P = 0)
                const float mu = m_run == -INFINITY ? 0.f : m_run;
                const uint32_t ph = smem_u32(sh.p_hi), pl = smem_u32(sh.p_lo);
                float add4[4] = {0.f, 0.f, 0.f, 0.f};   // two pairs of running sums
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    float s[32];
                    logits32(q2, s);
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int i = c4 * 8 + 2 * j;
                            float x0, x1;
                            ffma2(x0, x1, s[i], s[i + 1], sl2, sl2, -mu, -mu);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const int a = (j & 1) * 2;
                            fadd2(add4[a], add4[a + 1], add4[a], add4[a + 1], p0, p1);
                            const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                            const float2 hf = __bfloat1622float2(h);
                            float r0, r1;
                            fadd2(r0, r1, p0, p1, -hf.x, -hf.y);
                            const __nv_bfloat162 lo = __floats2bfloat162_rn(r0, r1);
                            hw[j] = *reinterpret_cast<const uint32_t*>(&h);
                            lw[j] = *reinterpret_cast<const uint32_t*>(&lo);
                        }
                        const uint32_t off = tile_off(r, half * 8 + q2 * 4 + c4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(ph + off), "r"(hw[0]),
                                     "r"(hw[1]), "r"(hw[2]), "r"(hw[3]));
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(pl + off), "r"(lw[0]),
                                     "r"(lw[1]), "r"(lw[2]), "r"(lw[3]));
                    }
                }
                tc_fence_before();
                l_run += (add4[0] + add4[1]) + (add4[2] + add4[3]);
                gather_v(t + 1);
            } else {
                cp_async_commit();
            }
            stage_rows(t + 3, row_pf);                         // slot of tile t - 1, no longer read
            cp_async_wait_group<2>();                          // V(t) has landed
            if (ok2) {                                         // ... for the issuer's P(t) V(t)
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&sh.p_ready);
            }
            if (soft_sync_or(my_to)) break;                    // staged rows visible; a give-up stops all
        }
        // the last P V
        if (!my_to && wait_bar(&sh.bar_o, ph_o)) ++seen_o;
    }

    // ---- epilogue: every thread's copies have landed; the halves' (m, l) meet in shared memory
    cp_async_wait_all();
    tc_fence_before();
    const bool good = __syncthreads_or(my_to) == 0;
    float* ex = reinterpret_cast<float*>(sh.p_hi);            // [half][m | l][row]
    if (good && !issuer_warp) {
        ex[half * 256 + r] = m_run;
        ex[half * 256 + 128 + r] = l_run;
    }
    __syncthreads();
    tc_fence_after();
    if (good && !issuer_warp) {
        const float ma = ex[r], la = ex[128 + r], mb = ex[256 + r], lb = ex[384 + r];
        const float m = fmaxf(ma, mb);
        float sa = 0.f, sb = 0.f;
        if (m != -INFINITY) {
            const float ea = exp2f(ma - m), eb = exp2f(mb - m);
            const float l = la * ea + lb * eb;
            if (l > 0.f) {
                sa = ea / l;
                sb = eb / l;
            }
        }
        // this thread writes output columns 64 half .. 64 half + 63 of row r
        const size_t qrow = size_t(blk * p.bq + qi) * p.Hq + g * G + 2 * pair + r / 64;
        uint16_t* orow = p.out + qrow * 128 + half * 64;
        float* frow = p.out_f32 ? p.out_f32 + qrow * 128 + half * 64 : nullptr;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float va[16], vb[16];
            tmem_ld16(t_oa + uint32_t(half * 64 + cb * 16) + lane_off, va);
            tmem_ld16(t_oa + 128 + uint32_t(half * 64 + cb * 16) + lane_off, vb);
#pragma unroll
            for (int i = 0; i < 16; i += 8) {
                float o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) o[k] = va[i + k] * sa + vb[i + k] * sb;
                uint32_t w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * k], o[2 * k + 1]);
                    w[k] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(orow + cb * 16 + i) = make_uint4(w[0], w[1], w[2], w[3]);
                if (frow) {
                    *reinterpret_cast<float4*>(frow + cb * 16 + i) = make_float4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<float4*>(frow + cb * 16 + i + 4) = make_float4(o[4], o[5], o[6], o[7]);
                }
            }
        }
    } else if (!good && tid == 0) {
        raise_status(p.status, SPA_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    // commits the issuer made that warp 0 has not seen complete (at most one per barrier, as the
    // issuer waits for the softmax warps' hand-off before each): wait once more (bounded); TMEM is
    // freed only when nothing is owed (a CTA that exits holding TMEM is the remaining hazard of a
    // wait that never completes)
    if (warp == 0) {
        bool owed = false;
        if (sh.n_s > seen_s) {
            uint32_t it = 0;
            while (!mbar_try_wait(&sh.bar_s, ph_s) && ++it < spin_limit) {
            }
            owed = owed || it >= spin_limit;
        }
        if (sh.n_o > seen_o) {
            uint32_t it = 0;
            while (!mbar_try_wait(&sh.bar_o, ph_o) && ++it < spin_limit) {
            }
            owed = owed || it >= spin_limit;
        }
        if (!__any_sync(0xffffffffu, owed)) {
            tc_fence_after();
            tmem_dealloc(tmem, 512);
        }
    }
}

}  // namespace

size_t prefill_scratch_bytes(int U, int N) {
    return align_up(size_t(U) * 16 * 4, 256) + align_up(size_t(U) * 4, 256) + align_up(size_t(U) * N * 4, 256) +
           hist0_bytes(U);
}

spa_status launch_prefill(const spa_prefill_args* a, void* ws, cudaStream_t st, void* const* events) {
    const int n_blocks = a->T / a->bq;
    const int U = n_blocks * a->Hkv;
    uint8_t* w = static_cast<uint8_t*>(ws);
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    w += kWsHeader;
    float* qhat = reinterpret_cast<float*>(w);
    w += align_up(size_t(U) * 16 * 4, 256);
    int32_t* unit_len = reinterpret_cast<int32_t*>(w);
    w += align_up(size_t(U) * 4, 256);
    float* scores = reinterpret_cast<float*>(w);
    w += align_up(size_t(U) * a->N * 4, 256);
    const Hist0 hist = hist0_carve(w, U);

    SPA_CUDA_TRY(launch_pdl(prefill_qhat_kernel, dim3(U), dim3(256), 0, st, a->q_idx, a->Hq, a->Hkv, a->bq,
                            a->q_start, qhat, unit_len, U));
    SPA_CUDA_TRY(launch_pdl(prefill_scores_kernel, dim3((a->N + kPsThreads - 1) / kPsThreads, a->Hkv), dim3(kPsThreads),
                            0, st, qhat, unit_len, reinterpret_cast<const uint4*>(a->Kidx), a->Hkv, a->N, n_blocks,
                            a->score_scale, scores));
    SelectParams sp{hist, scores, unit_len, U, a->N, a->topk, 0.f, a->sink, 0, a->idx, a->count, a->cap,
                    nullptr, status};
    spa_status s = launch_hist0(sp, false, st);
    if (s != SPA_OK) return s;
    s = launch_select(sp, false, st);
    if (s != SPA_OK) return s;

    PrefillAttendParams pp{a->Q, a->K, a->V, a->idx, a->count, a->cap, a->Hq, a->Hkv, a->N, a->bq, a->q_start,
                           a->sm_scale, a->out, a->out_f32, status};
    return launch_prefill_attend(pp, U, st, events);
}

spa_status launch_prefill_attend(const PrefillAttendParams& pp0, int U, cudaStream_t st, void* const* events) {
    PrefillAttendParams pp = pp0;
    pp.test_stall = test_stall_bits();
    const size_t smem = sizeof(PfShared);
    SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(prefill_attend_kernel),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    if (events) SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[0]), st));
    SPA_CUDA_TRY(launch_pdl(prefill_attend_kernel, dim3(U, pp.Hq / pp.Hkv / 2), dim3(kPfThreads), smem, st, pp));
    if (events) SPA_CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[1]), st));
    return SPA_OK;
}

}  // namespace spa
