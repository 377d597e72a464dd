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
// (TMEM), issued by one thread and completed through an mbarrier.  One CTA owns 128 query
// rows (two heads x 64 queries).  Keys are processed in tiles of 128 gathered rows
// (cp.async, bounds-checked) plus the diagonal tile of the block's own 64 positions.
// Two passes: pass 1 accumulates each row's max m and sum l from S = Q K^T; pass 2
// recomputes S, forms the normalised P = exp(S - m) / l as the sum of two bf16 terms
// and accumulates O += P V (two MMAs), so no rescaling of O is needed.
#include "internal.cuh"

namespace spa {
namespace {

constexpr int kPfRows = 128;          // query rows per CTA (tensor-core M)
constexpr int kPfKeys = 128;          // keys per tile (tensor-core N of S, K of P V)
constexpr int kPfThreads = 128;       // one thread per query row / TMEM lane
constexpr int kSlab = kPfRows * 128;  // bytes of one 64-column slab of a 128-row operand
constexpr int kTileBytes = 2 * kSlab; // 128 rows x 128 bf16
constexpr uint32_t kSpinLimit = 1u << 22;   // bounded mbarrier polls before giving up
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(slot)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols));
}
// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format, version 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}
// Instruction descriptor of kind::f16: fp32 D, bf16 A and B, A K-major, B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) |
           (uint32_t(M >> 4) << 24);
}

// byte offset of 16-byte chunk c (0..15) of row r in a 128-row, two-slab operand tile
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
    return uint32_t((c >> 3) * kSlab + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// ============================================================================ index query
// qhat[u][0..15] (fp32) = mean over the block's bq queries and G heads of q_idx, summed in
// (query, head) order; also unit_len[u] = t0, the number of candidate keys.
__global__ void prefill_qhat_kernel(const uint16_t* __restrict__ qidx, int Hq, int Hkv, int bq, int q_start,
                                    float* __restrict__ qhat, int32_t* __restrict__ unit_len, int U) {
    pdl_enter();
    const int u = blockIdx.x * (blockDim.x / 16) + threadIdx.x / 16;
    const int dim = threadIdx.x & 15;
    if (u >= U) return;
    const int blk = u / Hkv, g = u - blk * Hkv;
    const int G = Hq / Hkv;
    float acc = 0.f;
    for (int i = 0; i < bq; ++i)
        for (int h = 0; h < G; ++h)
            acc += __uint_as_float(uint32_t(qidx[(size_t(blk * bq + i) * Hq + g * G + h) * 16 + dim]) << 16);
    qhat[u * 16 + dim] = acc / float(bq * G);
    if (dim == 0) unit_len[u] = q_start + blk * bq;
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
struct __align__(1024) PfShared {
    uint8_t q[kTileBytes];
    uint8_t k[kTileBytes];
    uint8_t v[kTileBytes];
    uint8_t p_hi[kTileBytes];
    uint8_t p_lo[kTileBytes];
    uint64_t bar;
    uint32_t tmem_base;
    int rows[kPfKeys];     // cache rows of the current key tile (-1: none)
    int timed_out;
};

// grid (U, G / 2): one CTA per (unit, pair of query heads); 128 threads.
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_attend_kernel(PrefillAttendParams p) {
    pdl_enter();
    extern __shared__ __align__(1024) uint8_t dyn[];
    PfShared& sh = *reinterpret_cast<PfShared*>(dyn);
    const int tid = threadIdx.x, warp = tid >> 5;
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

    // this thread's query row: head 2*pair + tid/64, query tid%64 of the block
    const int hh = 2 * pair + tid / 64, qi = tid & 63;
    const int head = g * G + hh;
    const size_t qrow = size_t(blk * p.bq + qi) * p.Hq + head;

    if (warp == 0) tmem_alloc(&sh.tmem_base, 256);
    if (tid == 0) {
        mbar_init(&sh.bar, 1);
        sh.timed_out = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    // Q tile: row r = tid
#pragma unroll
    for (int c = 0; c < 16; ++c)
        cp_async16(smem_u32(sh.q) + tile_off(tid, c), p.Q + qrow * 128 + c * 8, true);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const uint32_t t_s = tmem, t_o = tmem + 128;                 // S at columns 0..127, O at 128..255
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    uint32_t phase = 0;
    // the test hook stalls the first S = Q K^T: its completion barrier waits for an MMA that
    // is never issued, so the bounded wait runs out with nothing in flight
    const bool stall = (p.test_stall & SPA_TEST_STALL_PREFILL_MMA) != 0;
    const uint32_t spin_limit = stall ? 1024u : kSpinLimit;
    bool pending = false;   // an MMA commit issued and not yet observed (uniform over the CTA)
    const float sl2 = p.sm_scale * kLog2e;
    constexpr uint32_t kIdS = idesc_bf16(kPfRows, kPfKeys, false);
    constexpr uint32_t kIdO = idesc_bf16(kPfRows, 128, true);

    // gather the keys (and values) of tile t into shared memory; returns the number of valid keys
    auto load_tile = [&](int t, bool with_v) {
        __syncthreads();   // previous readers of rows/k/v are done
        {
            const int r = tid;
            int row = -1;
            if (t < n_gather) {
                const int e = t * kPfKeys + r;
                if (e < n_sup) {
                    const int n = sup[e];
                    row = (n >= 0 && n < p.N) ? n : -1;
                }
            } else if (r < p.bq) {
                row = t0 + r;                                  // diagonal tile: the block's own keys
                if (row >= p.N) row = -1;
            }
            sh.rows[r] = row;
        }
        __syncthreads();
        // 128 rows x 16 chunks per tensor; thread tid copies chunk (tid & 15) of rows tid/16 + 8j
        for (int j = 0; j < kPfKeys / 8; ++j) {
            const int r = j * 8 + (tid >> 4), c = tid & 15;
            const int row = sh.rows[r];
            const bool ok = row >= 0;
            const size_t src = ok ? (kv0 + size_t(row)) * 128 + c * 8 : 0;
            cp_async16(smem_u32(sh.k) + tile_off(r, c), p.K + src, ok);
            if (with_v) cp_async16(smem_u32(sh.v) + tile_off(r, c), p.V + src, ok);
        }
        cp_async_wait_all();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };
    // S = Q K^T into TMEM columns 0..127; every thread waits for completion
    auto mma_s = [&]() -> bool {
        pending = !stall;
        if (tid == 0 && !stall) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = uint32_t((kk >> 2) * kSlab + (kk & 3) * 32);
                const uint64_t a = sw128_desc(smem_u32(sh.q) + off, 16, 1024);
                const uint64_t b = sw128_desc(smem_u32(sh.k) + off, 16, 1024);
                umma_bf16(t_s, a, b, kIdS, kk > 0);
            }
            umma_commit(&sh.bar);
        }
        return true;
    };
    // bounded wait for the outstanding commit; on expiry the CTA stops (every later step checks
    // sh.timed_out) and the commit stays owed, so TMEM is not freed under a running MMA
    auto wait_mma = [&]() {
        uint32_t it = 0;
        while (!mbar_try_wait(&sh.bar, phase)) {
            if (++it >= spin_limit) {
                atomicExch(&sh.timed_out, 1);
                return;
            }
        }
        pending = false;
        phase ^= 1u;
        tc_fence_after();
    };
    // this thread's row of S (scaled to log2 units, masked); key c of tile t
    auto row_logits = [&](int t, float (&s)[kPfKeys]) {
#pragma unroll
        for (int cb = 0; cb < kPfKeys / 32; ++cb) {
            float v[32];
            tmem_ld32(t_s + lane_off + cb * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int c = cb * 32 + i;
                const bool valid = sh.rows[c] >= 0 && (t < n_gather || c <= qi);
                s[c] = valid ? v[i] * sl2 : -INFINITY;
            }
        }
    };

    // a bounded wait that gave up ends both passes for every thread at the same point
    auto stop = [&]() -> bool {
        __syncthreads();
        return sh.timed_out != 0;
    };

    // ---- pass 1: row max m and sum l
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < n_tiles; ++t) {
        load_tile(t, false);
        mma_s();
        wait_mma();
        if (stop()) break;
        float s[kPfKeys];
        row_logits(t, s);
        float tm = -INFINITY;
#pragma unroll
        for (int c = 0; c < kPfKeys; ++c) tm = fmaxf(tm, s[c]);
        const float mn = fmaxf(m, tm);
        if (mn != -INFINITY) {
            float add = 0.f;
#pragma unroll
            for (int c = 0; c < kPfKeys; ++c) add += exp2f(s[c] - mn);
            l = l * exp2f(m - mn) + add;
            m = mn;
        }
        tc_fence_before();
    }
    const float inv_l = l > 0.f ? 1.f / l : 0.f;

    // ---- pass 2: O = sum_t P_t V_t with P = exp2(S - m) / l as bf16 hi + lo
    for (int t = 0; t < n_tiles && !sh.timed_out; ++t) {
        load_tile(t, true);
        mma_s();
        wait_mma();
        if (stop()) break;
        float s[kPfKeys];
        row_logits(t, s);
        const uint32_t ph = smem_u32(sh.p_hi), pl = smem_u32(sh.p_lo);
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float p0 = m == -INFINITY ? 0.f : exp2f(s[c8 * 8 + 2 * j] - m) * inv_l;
                const float p1 = m == -INFINITY ? 0.f : exp2f(s[c8 * 8 + 2 * j + 1] - m) * inv_l;
                const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                const float2 hf = __bfloat1622float2(h);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                hw[j] = *reinterpret_cast<const uint32_t*>(&h);
                lw[j] = *reinterpret_cast<const uint32_t*>(&lo);
            }
            const uint32_t off = tile_off(tid, c8);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(ph + off), "r"(hw[0]), "r"(hw[1]),
                         "r"(hw[2]), "r"(hw[3]));
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(pl + off), "r"(lw[0]), "r"(lw[1]),
                         "r"(lw[2]), "r"(lw[3]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t aoff = uint32_t((kk >> 2) * kSlab + (kk & 3) * 32);
                const uint64_t bh = sw128_desc(smem_u32(sh.v) + kk * 2048, kSlab, 1024);
                umma_bf16(t_o, sw128_desc(ph + aoff, 16, 1024), bh, kIdO, (t > 0 || kk > 0) ? 1u : 0u);
                umma_bf16(t_o, sw128_desc(pl + aoff, 16, 1024), bh, kIdO, 1u);
            }
            umma_commit(&sh.bar);
        }
        pending = true;
        wait_mma();       // O ready; P, K and V may be overwritten
        tc_fence_before();
        if (stop()) break;
    }

    // ---- epilogue: this thread's output row from TMEM
    __syncthreads();
    if (!sh.timed_out) {
        uint16_t* orow = p.out + qrow * 128;
        float* frow = p.out_f32 ? p.out_f32 + qrow * 128 : nullptr;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float v[32];
            tmem_ld32(t_o + lane_off + cb * 32, v);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float a = l > 0.f ? v[i] : 0.f, b = l > 0.f ? v[i + 1] : 0.f;
                const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                *reinterpret_cast<__nv_bfloat162*>(orow + cb * 32 + i) = h;
                if (frow) {
                    frow[cb * 32 + i] = a;
                    frow[cb * 32 + i + 1] = b;
                }
            }
        }
    } else if (tid == 0) {
        raise_status(p.status, SPA_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    // after a give-up, an issued MMA may still be running: wait once more (bounded); TMEM is
    // freed only when no commit is owed (a CTA that exits holding TMEM is the remaining hazard
    // of a wait that never completes)
    if (pending) {
        uint32_t it = 0;
        while (!mbar_try_wait(&sh.bar, phase) && ++it < spin_limit) {
        }
        pending = it >= spin_limit;
    }
    if (warp == 0 && !pending) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

size_t prefill_scratch_bytes(int U, int N) {
    return align_up(size_t(U) * 16 * 4, 256) + align_up(size_t(U) * 4, 256) + align_up(size_t(U) * N * 4, 256) +
           hist0_bytes(U);
}

spa_status launch_prefill(const spa_prefill_args* a, void* ws, cudaStream_t st) {
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

    SPA_CUDA_TRY(launch_pdl(prefill_qhat_kernel, dim3((U + 15) / 16), dim3(256), 0, st, a->q_idx, a->Hq, a->Hkv, a->bq,
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
    return launch_prefill_attend(pp, U, st);
}

spa_status launch_prefill_attend(const PrefillAttendParams& pp0, int U, cudaStream_t st) {
    PrefillAttendParams pp = pp0;
    pp.test_stall = test_stall_bits();
    const size_t smem = sizeof(PfShared);
    SPA_CUDA_TRY(cudaFuncSetAttribute(prefill_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    SPA_CUDA_TRY(launch_pdl(prefill_attend_kernel, dim3(U, pp.Hq / pp.Hkv / 2), dim3(kPfThreads), smem, st, pp));
    return SPA_OK;
}

}  // namespace spa
