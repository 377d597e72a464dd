// Exact softmax attention on the gathered support: split-KV flash-decode with a
// log-sum-exp combine.
//
// "Oracle-Guided Sparse Prefill" 2.1: attention is recomputed with the original Q, K, V
// restricted to the selected support; "Full Attention Strikes Back" (RTPurbo),
// Methodology 5: bandwidth-optimised sparse decode.
//
// Work split: every unit (one support) has R_u gathered rows, cut into tiles of 16
// rows.  The tiles of all units form one list, split evenly over all CTAs (two per SM),
// so every SM streams the same number of K/V bytes whatever the support sizes.  Inside
// a CTA the four warps take a unit's tiles round-robin; each warp gathers its tiles
// with cp.async (16-byte copies, bounds-checked, zero-filled when the index is out of
// range) into a private multi-stage ring in shared memory.
//
// Math per 16-row tile, on tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   S = Q K^T with the unit's query heads as the 16 rows of Q (G <= 16 heads; unused
//   rows are zero), an fp32 online softmax per head (exp2 with the log2(e) factor folded
//   into the scale), then O += P V.  P is carried as the sum of two bf16 terms (hi + lo)
//   so that the product keeps about 16 bits of each weight.  The rows of a GQA group
//   share every K/V row loaded, which is why the step is a small dense contraction: on
//   CUDA cores its 8 flops per byte would bound the kernel well below HBM speed.
//
// At the end of its share of a unit a CTA merges its warps' (m, l, o) in shared memory.
// A CTA holding a whole unit writes the output; otherwise it stores a partial (o, m, l),
// and a second kernel, one CTA per (unit, head) with eight warps splitting the unit's
// partials, merges them in a fixed order (log-sum-exp combine) and writes the output.
#include "internal.cuh"

namespace spa {
namespace {

constexpr int kAtThreads = 128;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kRows = 16;           // rows per tile (the mma N-extent of the score tile)
constexpr int kStages = 3;          // cp.async ring depth per warp
constexpr int kMaxUnits = 8192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// p ~= hi + lo with hi = bf16(p), lo = bf16(p - hi)
__device__ __forceinline__ void split_bf16(float p0, float p1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

struct UnitGeom {
    int b, h0, nh;        // batch, first query head, query heads served
    size_t kv;            // row offset of the unit's kv head in K/V
    int rows;             // gathered rows R_u
};

__device__ __forceinline__ UnitGeom unit_geom(const AttendParams& p, int u, int nh) {
    UnitGeom g;
    const int G = p.Hq / p.Hkv;
    if (p.collapse == SPA_COLLAPSE_GROUP_MEAN) {
        g.b = u / p.Hkv;
        const int kvh = u - g.b * p.Hkv;
        g.h0 = kvh * G;
        g.kv = (size_t(g.b) * p.Hkv + kvh) * size_t(p.N);
    } else {
        g.b = u / p.Hq;
        g.h0 = u - g.b * p.Hq;
        g.kv = (size_t(g.b) * p.Hkv + g.h0 / G) * size_t(p.N);
    }
    g.nh = nh;
    int c = p.count[u];
    c = c < 0 ? 0 : (c > p.cap ? p.cap : c);
    g.rows = c * p.unit_tokens;
    return g;
}

template <int D>
struct Tile {
    static constexpr int CPR = D / 8;                 // 16-byte chunks per row
    static constexpr int PPR = 2 * CPR;               // chunk copies per row (K and V)
    static constexpr int RPI = 32 / PPR;              // rows per warp-wide copy instruction
    static constexpr int BYTES = 2 * kRows * D * 2;   // K and V of 16 rows
    static constexpr int KSTEPS = D / 16;
    static constexpr int NT = D / 8;                  // 8-wide output column tiles
};

// owner CTA of tile x when TT tiles are split over G CTAs as [TT*c/G, TT*(c+1)/G)
__device__ __forceinline__ int tile_owner(long long x, long long TT, int G) {
    return int(((x + 1) * G - 1) / TT);
}

template <int D>
__global__ void __launch_bounds__(kAtThreads, 2)
attend_kernel(AttendParams p, int U, int nh) {
    using TL = Tile<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    int* s_prefix = reinterpret_cast<int*>(smem);                            // [U + 1]
    uint8_t* ring = smem + align_up(size_t(U + 1) * 4, 128);
    __shared__ uint32_t s_vmask[kAtWarps][kStages];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, cq = lane & 3;   // mma fragment coordinates
    uint8_t* my_ring = ring + size_t(warp) * kStages * TL::BYTES;

    // ---- tile prefix over units
    int running = 0;
    for (int base = 0; base < U; base += kAtThreads) {
        const int u = base + tid;
        int t = 0;
        if (u < U) {
            int c = p.count[u];
            c = c < 0 ? 0 : (c > p.cap ? p.cap : c);
            t = (c * p.unit_tokens + kRows - 1) / kRows;
        }
        int incl = t;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += x;
        }
        __shared__ int s_wsum[kAtWarps];
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int before = running;
        for (int w = 0; w < warp; ++w) before += s_wsum[w];
        if (u < U) s_prefix[u] = before + incl - t;
        int tot = 0;
        for (int w = 0; w < kAtWarps; ++w) tot += s_wsum[w];
        running += tot;
        __syncthreads();
    }
    if (tid == 0) s_prefix[U] = running;
    __syncthreads();
    const long long TT = running;
    const int cta = blockIdx.x;
    // Tiles are split over G = min(grid, TT) CTAs so that every range is non-empty (the
    // partial accounting counts CTAs); the rest only serve empty supports.
    const int G = int(TT < (long long)gridDim.x ? TT : (long long)gridDim.x);

    // ---- empty supports: out = 0, lse = -inf
    for (int u = cta; u < U; u += gridDim.x) {
        if (s_prefix[u + 1] != s_prefix[u]) continue;
        const UnitGeom ug = unit_geom(p, u, nh);
        for (int i = tid; i < nh * D; i += kAtThreads) {
            const size_t o = (size_t(ug.b) * p.Hq + ug.h0 + i / D) * D + (i % D);
            p.out[o] = 0;
            if (p.out_f32) p.out_f32[o] = 0.f;
            if (p.lse && i % D == 0) p.lse[size_t(ug.b) * p.Hq + ug.h0 + i / D] = -INFINITY;
        }
    }

    // CTA range of every unit, for the combine kernel: (first, last) CTA, or (-1, -1)
    // when one CTA (or none) produced the whole output
    if (cta == 0) {
        for (int v = tid; v < U; v += kAtThreads) {
            int lo = -1, hi = -1;
            if (s_prefix[v + 1] > s_prefix[v]) {
                lo = tile_owner(s_prefix[v], TT, G);
                hi = tile_owner(s_prefix[v + 1] - 1, TT, G);
                if (lo == hi) lo = hi = -1;
            }
            p.unit_ctas[2 * v] = lo;
            p.unit_ctas[2 * v + 1] = hi;
        }
    }
    if (cta >= G) return;
    const long long t0 = TT * cta / G, t1 = TT * (cta + 1) / G;

    // first unit of the range: last u with prefix[u] <= t0 (empty units are skipped)
    int u;
    {
        int lo_u = 0, hi_u = U;   // prefix[lo_u] <= t0 < prefix[hi_u]
        while (hi_u - lo_u > 1) {
            const int mid = (lo_u + hi_u) >> 1;
            if (s_prefix[mid] <= t0) lo_u = mid; else hi_u = mid;
        }
        u = lo_u;
    }
    const float sl2 = p.sm_scale * kLog2e;
    long long x = t0;
    while (x < t1) {
        while (s_prefix[u + 1] <= x) ++u;
        const long long seg_end = min(t1, (long long)s_prefix[u + 1]);
        const int a = int(x - s_prefix[u]);
        const int bnd = int(seg_end - s_prefix[u]);
        const int tiles_u = s_prefix[u + 1] - s_prefix[u];
        const UnitGeom ug = unit_geom(p, u, nh);

        // Q fragments (rows = query heads of the unit; rows >= nh are zero)
        uint32_t qa[TL::KSTEPS][4];
        {
            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
            const size_t r0 = size_t(ug.b) * p.Hq + ug.h0 + gq;
            const bool v0 = gq < nh, v1 = gq + 8 < nh;
#pragma unroll
            for (int kk = 0; kk < TL::KSTEPS; ++kk) {
                const int col = kk * 16 + 2 * cq;
                qa[kk][0] = v0 ? __ldg(q32 + (r0 * D + col) / 2) : 0u;
                qa[kk][1] = v1 ? __ldg(q32 + ((r0 + 8) * D + col) / 2) : 0u;
                qa[kk][2] = v0 ? __ldg(q32 + (r0 * D + col + 8) / 2) : 0u;
                qa[kk][3] = v1 ? __ldg(q32 + ((r0 + 8) * D + col + 8) / 2) : 0u;
            }
        }

        // warp's tiles: a + warp, a + warp + 4, ...
        const int first = a + warp;
        const int n_my = first < bnd ? (bnd - first + kAtWarps - 1) / kAtWarps : 0;
        const int32_t* idx_u = p.idx + size_t(u) * p.cap;
        const int T = p.unit_tokens;

        auto issue = [&](int j, int stage) {
            const int tile = first + j * kAtWarps;
            const int r = tile * kRows + (lane & 15);
            long long row = -1;
            if (r < ug.rows) {
                const int e = T == 1 ? r : r / T;
                const long long n = (long long)idx_u[e] * T + (T == 1 ? 0 : r - e * T);
                if (n >= 0 && n < p.N) row = n;
            }
            const uint32_t vm = __ballot_sync(0xffffffffu, row >= 0) & 0xffffu;
            if (lane == 0) s_vmask[warp][stage] = vm;
            uint8_t* st = my_ring + size_t(stage) * TL::BYTES;
            const uint32_t kbase = smem_u32(st), vbase = kbase + kRows * D * 2;
#pragma unroll
            for (int i = 0; i < kRows / TL::RPI; ++i) {
                const int rr = i * TL::RPI + lane / TL::PPR;       // row within the tile
                const int part = lane % TL::PPR;
                const long long gr = __shfl_sync(0xffffffffu, row, rr);
                const bool isv = part >= TL::CPR;
                const int c = isv ? part - TL::CPR : part;
                const bool ok = gr >= 0;
                const uint16_t* src = (isv ? p.V : p.K) + (ok ? (ug.kv + size_t(gr)) * D + c * 8 : 0);
                const uint32_t dst = (isv ? vbase : kbase) + (rr * TL::CPR + (c ^ (rr & 7))) * 16;
                cp_async16(dst, src, ok);
            }
        };

        float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
        float acc[TL::NT][4];
#pragma unroll
        for (int i = 0; i < TL::NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

#pragma unroll
        for (int j = 0; j < kStages - 1; ++j) {
            if (j < n_my) issue(j, j);
            cp_commit();
        }
        for (int j = 0; j < n_my; ++j) {
            const int jn = j + kStages - 1;
            if (jn < n_my) issue(jn, jn % kStages);
            cp_commit();
            cp_wait<kStages - 1>();
            __syncwarp();
            const int stage = j % kStages;
            const uint8_t* st = my_ring + size_t(stage) * TL::BYTES;
            const uint32_t kbase = smem_u32(st), vbase = kbase + kRows * D * 2;
            const uint32_t vm = s_vmask[warp][stage];

            // S = Q K^T (two 8-key column tiles)
            float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < TL::KSTEPS; ++kk) {
                const int mat = lane >> 3;
                const int rr = (mat >> 1) * 8 + (lane & 7);
                const int c = 2 * kk + (mat & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + (rr * TL::CPR + (c ^ (rr & 7))) * 16, b0, b1, b2, b3);
                mma16816(s[0], qa[kk], b0, b1);
                mma16816(s[1], qa[kk], b2, b3);
            }
            // scale, mask, online softmax (rows gq and gq + 8)
            float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = nt * 8 + 2 * cq + (e & 1);
                    const float v = ((vm >> key) & 1u) ? s[nt][e] * sl2 : -INFINITY;
                    s[nt][e] = v;
                    tmax[e >> 1] = fmaxf(tmax[e >> 1], v);
                }
            float alpha[2], mref[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
                tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
                const float mn = fmaxf(m_r[h], tmax[h]);
                mref[h] = mn == -INFINITY ? 0.f : mn;
                alpha[h] = exp2f(m_r[h] - mref[h]);
                m_r[h] = mn;
            }
            float rs[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pv = exp2f(s[nt][e] - mref[e >> 1]);
                    s[nt][e] = pv;
                    rs[e >> 1] += pv;
                }
            l_r[0] = l_r[0] * alpha[0] + rs[0];
            l_r[1] = l_r[1] * alpha[1] + rs[1];
#pragma unroll
            for (int i = 0; i < TL::NT; ++i) {
                acc[i][0] *= alpha[0]; acc[i][1] *= alpha[0];
                acc[i][2] *= alpha[1]; acc[i][3] *= alpha[1];
            }
            uint32_t ph[4], pl[4];
            split_bf16(s[0][0], s[0][1], ph[0], pl[0]);
            split_bf16(s[0][2], s[0][3], ph[1], pl[1]);
            split_bf16(s[1][0], s[1][1], ph[2], pl[2]);
            split_bf16(s[1][2], s[1][3], ph[3], pl[3]);
            // O += P V
#pragma unroll
            for (int n2 = 0; n2 < TL::NT / 2; ++n2) {
                const int mat = lane >> 3;
                const int rr = (mat & 1) * 8 + (lane & 7);
                const int c = 2 * n2 + (mat >> 1);
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(vbase + (rr * TL::CPR + (c ^ (rr & 7))) * 16, v0, v1, v2, v3);
                mma16816(acc[2 * n2], ph, v0, v1);
                mma16816(acc[2 * n2], pl, v0, v1);
                mma16816(acc[2 * n2 + 1], ph, v2, v3);
                mma16816(acc[2 * n2 + 1], pl, v2, v3);
            }
            __syncwarp();   // this stage may be refilled after the next wait
        }
        cp_wait<0>();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_r[h] += __shfl_xor_sync(0xffffffffu, l_r[h], 1);
            l_r[h] += __shfl_xor_sync(0xffffffffu, l_r[h], 2);
        }

        // ---- merge the warps: each warp parks (m, l, o) in its own ring
        __syncthreads();
        float* wbuf = reinterpret_cast<float*>(my_ring);      // m[16], l[16], o[16][D]
        if (cq == 0) {
            wbuf[gq] = m_r[0]; wbuf[gq + 8] = m_r[1];
            wbuf[16 + gq] = l_r[0]; wbuf[16 + gq + 8] = l_r[1];
        }
#pragma unroll
        for (int i = 0; i < TL::NT; ++i) {
            const int col = i * 8 + 2 * cq;
            wbuf[32 + gq * D + col] = acc[i][0];
            wbuf[32 + gq * D + col + 1] = acc[i][1];
            wbuf[32 + (gq + 8) * D + col] = acc[i][2];
            wbuf[32 + (gq + 8) * D + col + 1] = acc[i][3];
        }
        __syncthreads();
        const bool whole = a == 0 && bnd == tiles_u;
        const int slot = u + cta;
        float* part = p.partials + size_t(slot) * nh * (D + 2);
        for (int i = tid; i < nh * D; i += kAtThreads) {
            const int row = i / D, col = i - row * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kAtWarps; ++w)
                M = fmaxf(M, reinterpret_cast<const float*>(ring + size_t(w) * kStages * TL::BYTES)[row]);
            const float Mr = M == -INFINITY ? 0.f : M;
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < kAtWarps; ++w) {
                const float* wb = reinterpret_cast<const float*>(ring + size_t(w) * kStages * TL::BYTES);
                const float sc = exp2f(wb[row] - Mr);
                L += wb[16 + row] * sc;
                O += wb[32 + row * D + col] * sc;
            }
            if (whole) {
                const size_t o = (size_t(ug.b) * p.Hq + ug.h0 + row) * D + col;
                const float val = L > 0.f ? O / L : 0.f;
                const __nv_bfloat16 bv = __float2bfloat16_rn(val);
                p.out[o] = *reinterpret_cast<const uint16_t*>(&bv);
                if (p.out_f32) p.out_f32[o] = val;
                if (p.lse && col == 0)
                    p.lse[size_t(ug.b) * p.Hq + ug.h0 + row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
            } else {
                part[row * (D + 2) + col] = O;
                if (col == 0) {
                    part[row * (D + 2) + D] = M;
                    part[row * (D + 2) + D + 1] = L;
                }
            }
        }
        __syncthreads();   // rings are reused by the next segment
        x = seg_end;
    }
}

// Log-sum-exp combine of the partials of every unit split over several CTAs.
// grid (U, heads per unit), 256 threads: warp w merges partials c_lo + w, c_lo + w + 8, ...
// online (running max, rescaled sums); the eight warp results are merged in warp order.
template <int D>
__global__ void __launch_bounds__(256)
combine_kernel(AttendParams p, int nh) {
    constexpr int CPL = D / 32;    // columns per lane
    const int u = blockIdx.x, row = blockIdx.y;
    const int c_lo = p.unit_ctas[2 * u], c_hi = p.unit_ctas[2 * u + 1];
    if (c_lo < 0 || row >= nh) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float M = -INFINITY, L = 0.f, O[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) O[j] = 0.f;
    for (int c = c_lo + warp; c <= c_hi; c += 8) {
        const float* pp = p.partials + (size_t(u + c) * nh + row) * (D + 2);
        const float m = __ldcg(pp + D), l = __ldcg(pp + D + 1);
        float v[CPL];
#pragma unroll
        for (int j = 0; j < CPL; ++j) v[j] = __ldcg(pp + lane * CPL + j);
        const float Mn = fmaxf(M, m);
        if (Mn == -INFINITY) continue;
        const float a = exp2f(M - Mn), b = exp2f(m - Mn);
        L = L * a + l * b;
#pragma unroll
        for (int j = 0; j < CPL; ++j) O[j] = O[j] * a + v[j] * b;
        M = Mn;
    }
    __shared__ float sM[8], sL[8], sO[8][D];
    if (lane == 0) { sM[warp] = M; sL[warp] = L; }
#pragma unroll
    for (int j = 0; j < CPL; ++j) sO[warp][lane * CPL + j] = O[j];
    __syncthreads();
    if (warp != 0) return;
    float Mt = -INFINITY;
    for (int w = 0; w < 8; ++w) Mt = fmaxf(Mt, sM[w]);
    const float Mr = Mt == -INFINITY ? 0.f : Mt;
    float Lt = 0.f, Ot[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) Ot[j] = 0.f;
    for (int w = 0; w < 8; ++w) {
        const float sc = exp2f(sM[w] - Mr);
        Lt += sL[w] * sc;
#pragma unroll
        for (int j = 0; j < CPL; ++j) Ot[j] += sO[w][lane * CPL + j] * sc;
    }
    const UnitGeom ug = unit_geom(p, u, nh);
    const size_t ob = (size_t(ug.b) * p.Hq + ug.h0 + row) * D;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const float val = Lt > 0.f ? Ot[j] / Lt : 0.f;
        const __nv_bfloat16 bv = __float2bfloat16_rn(val);
        p.out[ob + lane * CPL + j] = *reinterpret_cast<const uint16_t*>(&bv);
        if (p.out_f32) p.out_f32[ob + lane * CPL + j] = val;
    }
    if (p.lse && lane == 0)
        p.lse[size_t(ug.b) * p.Hq + ug.h0 + row] = Lt > 0.f ? (Mt + log2f(Lt)) * kLn2 : -INFINITY;
}

template <int D>
size_t attend_smem(int U) {
    return align_up(size_t(U + 1) * 4, 128) + size_t(kAtWarps) * kStages * Tile<D>::BYTES;
}

}  // namespace

int attend_grid() { return device_info().num_sms * 2; }

size_t attend_scratch_bytes(int U, int heads_per_unit, int d) {
    const size_t meta = align_up(size_t(U) * 8, 256);
    const size_t partials = size_t(U + attend_grid()) * heads_per_unit * (d + 2) * 4;
    return meta + align_up(partials, 256);
}

spa_status launch_attend(const AttendParams& p, cudaStream_t st) {
    const int G = p.Hq / p.Hkv;
    const int U = p.collapse == SPA_COLLAPSE_GROUP_MEAN ? p.B * p.Hkv : p.B * p.Hq;
    const int nh = p.collapse == SPA_COLLAPSE_GROUP_MEAN ? G : 1;
    if (U > kMaxUnits || nh > 16) return SPA_ERR_UNSUPPORTED_SHAPE;
    const int grid = attend_grid();
    if (p.d == 128) {
        const size_t sm = attend_smem<128>(U);
        SPA_CUDA_TRY(cudaFuncSetAttribute(attend_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)));
        attend_kernel<128><<<grid, kAtThreads, sm, st>>>(p, U, nh);
        SPA_CUDA_TRY(cudaGetLastError());
        combine_kernel<128><<<dim3(U, nh), 256, 0, st>>>(p, nh);
    } else if (p.d == 64) {
        const size_t sm = attend_smem<64>(U);
        SPA_CUDA_TRY(cudaFuncSetAttribute(attend_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)));
        attend_kernel<64><<<grid, kAtThreads, sm, st>>>(p, U, nh);
        SPA_CUDA_TRY(cudaGetLastError());
        combine_kernel<64><<<dim3(U, nh), 256, 0, st>>>(p, nh);
    } else {
        return SPA_ERR_UNSUPPORTED_SHAPE;
    }
    SPA_CUDA_TRY(cudaGetLastError());
    return SPA_OK;
}

}  // namespace spa
