// Exact softmax attention on the gathered support: split-KV flash-decode with a
// log-sum-exp combine.
//
// "Oracle-Guided Sparse Prefill" 2.1: attention is recomputed with the original Q, K, V
// restricted to the selected support; "Full Attention Strikes Back" (RTPurbo),
// Methodology 5: bandwidth-optimised sparse decode.
//
// Work split: every unit (one support) has R_u gathered rows, cut into tiles of 16
// rows.  The tiles of all units form one list, split evenly over all CTAs (two per SM),
// so every SM streams about the same number of K/V bytes whatever the support sizes; each
// unit is charged a fixed segment cost on top of its tiles, so that a CTA whose share spans
// several units (and pays their start-up and merge) gets fewer tiles.  Inside
// a CTA the four warps take a unit's tiles round-robin; each warp gathers its tiles
// with cp.async (16-byte copies, bounds-checked, zero-filled when the index is out of
// range) into a private multi-stage ring in shared memory.
//
// Math per 16-row tile, on tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate),
// in transposed form so that the gathered keys, not the few query heads, fill the
// 16-row side of the tensor-core tile:
//   S^T = K Q^T      16 keys x 8 heads per head tile (the group's G <= 16 heads, padded to 8);
//   fp32 online softmax per head (column), exp2 with log2(e) folded into the scale;
//   P^T is moved into the B-operand layout by two 8x8 transposes (movmatrix);
//   O^T += V^T P^T   V^T read with transposing ldmatrix; d = 128 rows x 8 heads.
// P is carried as the sum of two bf16 terms (hi + lo) so the product keeps about 16 bits
// of each weight.  The heads of a GQA group share every K/V row loaded, which is why the
// step is a small dense contraction: on CUDA cores its 8 flops per byte would bound the
// kernel well below HBM speed.  Row indices are fetched one tile ahead of their gather.
//
// At the end of its share of a unit a CTA merges its warps' (m, l, o) in shared memory.
// A CTA holding a whole unit writes the output; otherwise it stores a partial (o, m, l),
// and a second kernel, one CTA per (unit, head) with eight warps splitting the unit's
// partials, merges them in a fixed order (log-sum-exp combine) and writes the output.
#include "internal.cuh"
#include "warp_mma.cuh"

namespace spa {
namespace {

constexpr int kAtThreads = 128;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kRows = 16;           // rows per tile (the mma N-extent of the score tile)
constexpr int kStages = 3;          // cp.async ring depth per warp
constexpr int kMaxUnits = 8192;
constexpr int kWinTiles = 128;      // tiles whose row indices are staged in shared memory at once
// Fixed cost of a segment (one unit's share of a CTA's range) in tiles: draining the gathers,
// the merge of the warps, the partial's store, the next unit's query and index loads and the
// refill of the rings.  Measured on B200 at 5-8 us per extra segment against about 0.5 us per
// tile of a CTA (10-16 tiles), and charged as 20 tiles at the head of every non-empty unit when
// the tiles are split over the CTAs, so that a CTA whose range crosses unit boundaries gets
// fewer tiles (8, 12 and 20 were timed: 20 was the fastest or level on every decode workload).
constexpr int kSegCost = 20;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct UnitGeom {
    int b, h0, nh;        // batch, first query head, query heads served
    int bh;               // batch * Hkv + kv head
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
        g.bh = g.b * p.Hkv + kvh;
        g.kv = size_t(p.kv_shared ? kvh : g.bh) * size_t(p.N);
    } else {
        g.b = u / p.Hq;
        g.h0 = u - g.b * p.Hq;
        g.bh = g.b * p.Hkv + g.h0 / G;
        g.kv = size_t(p.kv_shared ? g.h0 / G : g.bh) * size_t(p.N);
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

// owner CTA of (weighted) tile x when TT tiles are split over G CTAs as [TT*c/G, TT*(c+1)/G)
__device__ __forceinline__ int tile_owner(long long x, long long TT, int G) {
    return int(((x + 1) * G - 1) / TT);
}

// RLA: also accumulate, per head, the linear attention of the gathered rows with phi = exp
// ("SPLA", section 2.2): W^T = phi(K) phi(Q)^T on the same K fragments as S^T, and
// Olin^T += V^T W^T on the same V fragments as O^T; every unit then leaves partials for the
// combine kernel, which forms the residual term.
template <int D, int NH8, bool RLA>
__global__ void __launch_bounds__(kAtThreads, 2)
attend_kernel(AttendParams p, int U, int nh) {
    pdl_enter();
    using TL = Tile<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    int* s_prefix = reinterpret_cast<int*>(smem);                            // [U + 1]
    int* s_rows = reinterpret_cast<int*>(smem + align_up(size_t(U + 1) * 4, 128));   // [kWinTiles * 16]
    uint8_t* ring = smem + align_up(size_t(U + 1) * 4, 128) + size_t(kWinTiles) * kRows * 4;
    __shared__ uint32_t s_vmask[kAtWarps][kStages];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, cq = lane & 3;   // mma fragment coordinates (row group, column pair)
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
            if (t > 0) t += kSegCost;   // the unit's tiles, weighted by the fixed cost of a segment
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
    // Weighted tiles are split over G = min(grid, TT) CTAs so that every range is non-empty;
    // the rest only serve empty supports.  A range may hold only a unit's cost share: the CTA
    // then produces nothing for that unit, and the combine kernel takes the unit's partials
    // from the CTAs that own its first to its last real tile.
    const int G = int(TT < (long long)gridDim.x ? TT : (long long)gridDim.x);

    // ---- empty supports: out = 0, lse = -inf
    for (int u = cta; !RLA && u < U; u += gridDim.x) {   // (with RLA the combine kernel writes them)
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
                lo = tile_owner(s_prefix[v] + kSegCost, TT, G);   // owner of the first real tile
                hi = tile_owner(s_prefix[v + 1] - 1, TT, G);
                if (lo == hi && !RLA) lo = hi = -1;
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
        // the unit's weighted range is its segment cost, then its tiles: [a, bnd) are real tiles
        const int a = max(int(x - s_prefix[u]) - kSegCost, 0);
        const int bnd = max(int(seg_end - s_prefix[u]) - kSegCost, 0);
        const int tiles_u = s_prefix[u + 1] - s_prefix[u] - kSegCost;
        if (a >= bnd) {   // only the cost share of the unit (uniform over the CTA)
            x = seg_end;
            continue;
        }
        const UnitGeom ug = unit_geom(p, u, nh);

        // Q^T as the B operand of S^T = K Q^T: b0/b1 of k-step kk, head tile nt hold
        // q[head 8nt + gq][16kk + 2cq (+1)] and [16kk + 8 + 2cq (+1)]; heads >= nh are zero.
        uint32_t qb[TL::KSTEPS][NH8][2];
        {
            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
#pragma unroll
            for (int nt = 0; nt < NH8; ++nt) {
                const int hd = nt * 8 + gq;
                const bool v = hd < nh;
                const size_t r0 = size_t(ug.b) * p.Hq + ug.h0 + hd;
#pragma unroll
                for (int kk = 0; kk < TL::KSTEPS; ++kk) {
                    const int col = kk * 16 + 2 * cq;
                    qb[kk][nt][0] = v ? __ldg(q32 + (r0 * D + col) / 2) : 0u;
                    qb[kk][nt][1] = v ? __ldg(q32 + (r0 * D + col + 8) / 2) : 0u;
                }
            }
        }

        // RLA: phi(Q)^T as B operand, exp of the same elements as qb, hi + lo bf16; zero for
        // absent heads
        uint32_t qfh[RLA ? TL::KSTEPS : 1][NH8][2], qfl[RLA ? TL::KSTEPS : 1][NH8][2];
        if constexpr (RLA) {
#pragma unroll
            for (int nt = 0; nt < NH8; ++nt)
#pragma unroll
                for (int kk = 0; kk < TL::KSTEPS; ++kk)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool v = nt * 8 + gq < nh;
                        const float2 f = bf16x2_to_float2(qb[kk][nt][e]);
                        split_bf16(v ? expf(f.x) : 0.f, v ? expf(f.y) : 0.f, qfh[kk][nt][e], qfl[kk][nt][e]);
                    }
        }

        const int32_t* idx_u = p.idx + size_t(u) * p.cap;
        const int T = p.unit_tokens;
        auto issue = [&](long long row, int stage) {
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

        // online-softmax state of heads 8nt + 2cq + e (e = 0, 1); l is this thread's partial sum
        float m_r[NH8][2], l_r[NH8][2];
        float acc[TL::KSTEPS][NH8][4];      // O^T: d-tile x head tile, rows d = 16dt + gq (+8)
        float lin[RLA ? TL::KSTEPS : 1][NH8][4], den_r[NH8][2];   // RLA: Olin^T and sum of weights
        int nval = 0;                                             // RLA: rows gathered in [0, N)
#pragma unroll
        for (int nt = 0; nt < NH8; ++nt) {
            m_r[nt][0] = m_r[nt][1] = -INFINITY;
            l_r[nt][0] = l_r[nt][1] = 0.f;
            den_r[nt][0] = den_r[nt][1] = 0.f;
#pragma unroll
            for (int dt = 0; dt < (RLA ? TL::KSTEPS : 1); ++dt)
                lin[dt][nt][0] = lin[dt][nt][1] = lin[dt][nt][2] = lin[dt][nt][3] = 0.f;
#pragma unroll
            for (int dt = 0; dt < TL::KSTEPS; ++dt) acc[dt][nt][0] = acc[dt][nt][1] = acc[dt][nt][2] = acc[dt][nt][3] = 0.f;
        }

        for (int wt0 = a; wt0 < bnd; wt0 += kWinTiles) {
        const int wt1 = min(bnd, wt0 + kWinTiles);
        // cache rows of the window's tiles, staged once with coalesced index loads (-1: none)
        __syncthreads();
        for (int i = tid; i < (wt1 - wt0) * kRows; i += kAtThreads) {
            const int r = wt0 * kRows + i;
            int v = -1;
            if (r < ug.rows) {
                const int e = T == 1 ? r : r / T;
                const long long n = (long long)__ldg(idx_u + e) * T + (T == 1 ? 0 : r - e * T);
                v = (n >= 0 && n < p.N) ? int(n) : -1;
            }
            s_rows[i] = v;
        }
        __syncthreads();
        // warp's tiles of the window: wt0 + warp, wt0 + warp + 4, ...
        const int first = wt0 + warp;
        const int n_my = first < wt1 ? (wt1 - first + kAtWarps - 1) / kAtWarps : 0;
        auto fetch = [&](int j) -> long long {
            return j < n_my ? (long long)s_rows[(first - wt0 + j * kAtWarps) * kRows + (lane & 15)] : -1ll;
        };
#pragma unroll
        for (int j = 0; j < kStages - 1; ++j) {
            if (j < n_my) issue(fetch(j), j);
            cp_commit();
        }
        for (int j = 0; j < n_my; ++j) {
            const int jn = j + kStages - 1;
            if (jn < n_my) issue(fetch(jn), jn % kStages);
            cp_commit();
            cp_wait<kStages - 1>();
            __syncwarp();
            const int stage = j % kStages;
            const uint8_t* st = my_ring + size_t(stage) * TL::BYTES;
            const uint32_t kbase = smem_u32(st), vbase = kbase + kRows * D * 2;
            const uint32_t vm = s_vmask[warp][stage];

            // S^T = K Q^T: 16 keys x 8 heads per head tile
            float s[NH8][4], w[RLA ? NH8 : 1][4];
#pragma unroll
            for (int nt = 0; nt < NH8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int nt = 0; nt < (RLA ? NH8 : 1); ++nt) w[nt][0] = w[nt][1] = w[nt][2] = w[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < TL::KSTEPS; ++kk) {
                const int mat = lane >> 3;
                const int rr = (mat & 1) * 8 + (lane & 7);
                const int c = 2 * kk + (mat >> 1);
                uint32_t a[4];
                ldsm_x4(kbase + (rr * TL::CPR + (c ^ (rr & 7))) * 16, a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NH8; ++nt) mma16816(s[nt], a, qb[kk][nt][0], qb[kk][nt][1]);
                if constexpr (RLA) {
                    // W^T += phi(K) phi(Q)^T, both factors as hi + lo (the lo * lo term dropped)
                    uint32_t fh[4], fl[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 kf = bf16x2_to_float2(a[i]);
                        split_bf16(expf(kf.x), expf(kf.y), fh[i], fl[i]);
                    }
#pragma unroll
                    for (int nt = 0; nt < NH8; ++nt) {
                        mma16816(w[nt], fh, qfh[kk][nt][0], qfh[kk][nt][1]);
                        mma16816(w[nt], fl, qfh[kk][nt][0], qfh[kk][nt][1]);
                        mma16816(w[nt], fh, qfl[kk][nt][0], qfl[kk][nt][1]);
                    }
                }
            }
            // mask, scale; per-head max over the 16 keys (keys gq, gq + 8 here; xor over gq)
            const bool kv0 = (vm >> gq) & 1u, kv1 = (vm >> (gq + 8)) & 1u;
            // RLA: masked weights (zero-filled rows would weigh phi(q) . 1), their sums, and
            // W^T moved into the B-operand layout like P^T
            uint32_t wh[RLA ? NH8 : 1][2], wl[RLA ? NH8 : 1][2];
            if constexpr (RLA) {
                nval += __popc(vm);
#pragma unroll
                for (int nt = 0; nt < NH8; ++nt) {
                    const float w00 = kv0 ? w[nt][0] : 0.f, w01 = kv0 ? w[nt][1] : 0.f;
                    const float w10 = kv1 ? w[nt][2] : 0.f, w11 = kv1 ? w[nt][3] : 0.f;
                    den_r[nt][0] += w00 + w10;
                    den_r[nt][1] += w01 + w11;
                    uint32_t h0, l0, h1, l1;
                    split_bf16(w00, w01, h0, l0);
                    split_bf16(w10, w11, h1, l1);
                    wh[nt][0] = movm_t(h0); wh[nt][1] = movm_t(h1);
                    wl[nt][0] = movm_t(l0); wl[nt][1] = movm_t(l1);
                }
            }
            uint32_t bh[NH8][2], bl[NH8][2];
#pragma unroll
            for (int nt = 0; nt < NH8; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float x0 = kv0 ? s[nt][e] * sl2 : -INFINITY;       // key gq
                    const float x1 = kv1 ? s[nt][2 + e] * sl2 : -INFINITY;   // key gq + 8
                    float tm = fmaxf(x0, x1);
                    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
                    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
                    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
                    const float mn = fmaxf(m_r[nt][e], tm);
                    const float mref = mn == -INFINITY ? 0.f : mn;
                    const float alpha = exp2f(m_r[nt][e] - mref);
                    m_r[nt][e] = mn;
                    const float p0 = exp2f(x0 - mref), p1 = exp2f(x1 - mref);
                    s[nt][e] = p0;
                    s[nt][2 + e] = p1;
                    l_r[nt][e] = l_r[nt][e] * alpha + p0 + p1;
#pragma unroll
                    for (int dt = 0; dt < TL::KSTEPS; ++dt) {
                        acc[dt][nt][e] *= alpha;
                        acc[dt][nt][2 + e] *= alpha;
                    }
                }
                // P^T into B-operand layout: transpose the two 8x8 (key x head) blocks
                uint32_t h0, l0, h1, l1;
                split_bf16(s[nt][0], s[nt][1], h0, l0);     // key gq,     heads 2cq, 2cq+1
                split_bf16(s[nt][2], s[nt][3], h1, l1);     // key gq + 8
                bh[nt][0] = movm_t(h0); bh[nt][1] = movm_t(h1);
                bl[nt][0] = movm_t(l0); bl[nt][1] = movm_t(l1);
            }
            // O^T += V^T P^T  (P as hi + lo bf16 terms)
#pragma unroll
            for (int dt = 0; dt < TL::KSTEPS; ++dt) {
                const int mat = lane >> 3;
                const int rr = (mat >> 1) * 8 + (lane & 7);
                const int c = 2 * dt + (mat & 1);
                uint32_t a[4];
                ldsm_x4_t(vbase + (rr * TL::CPR + (c ^ (rr & 7))) * 16, a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NH8; ++nt) {
                    mma16816(acc[dt][nt], a, bh[nt][0], bh[nt][1]);
                    mma16816(acc[dt][nt], a, bl[nt][0], bl[nt][1]);
                    if constexpr (RLA) {
                        mma16816(lin[dt][nt], a, wh[nt][0], wh[nt][1]);
                        mma16816(lin[dt][nt], a, wl[nt][0], wl[nt][1]);
                    }
                }
            }
            __syncwarp();   // this stage may be refilled after the next wait
        }
        cp_wait<0>();
        }   // window
#pragma unroll
        for (int nt = 0; nt < NH8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                l_r[nt][e] += __shfl_xor_sync(0xffffffffu, l_r[nt][e], 4);
                l_r[nt][e] += __shfl_xor_sync(0xffffffffu, l_r[nt][e], 8);
                l_r[nt][e] += __shfl_xor_sync(0xffffffffu, l_r[nt][e], 16);
                if constexpr (RLA) {
                    den_r[nt][e] += __shfl_xor_sync(0xffffffffu, den_r[nt][e], 4);
                    den_r[nt][e] += __shfl_xor_sync(0xffffffffu, den_r[nt][e], 8);
                    den_r[nt][e] += __shfl_xor_sync(0xffffffffu, den_r[nt][e], 16);
                }
            }

        // ---- merge the warps: each warp parks (m, l, o) in its own ring
        __syncthreads();
        float* wbuf = reinterpret_cast<float*>(my_ring);      // m[16], l[16], o[16][D]
#pragma unroll
        for (int nt = 0; nt < NH8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hd = nt * 8 + 2 * cq + e;
                if (gq == 0) {
                    wbuf[hd] = m_r[nt][e];
                    wbuf[16 + hd] = l_r[nt][e];
                }
#pragma unroll
                for (int dt = 0; dt < TL::KSTEPS; ++dt) {
                    wbuf[32 + hd * D + dt * 16 + gq] = acc[dt][nt][e];
                    wbuf[32 + hd * D + dt * 16 + gq + 8] = acc[dt][nt][2 + e];
                }
            }
        if (NH8 == 1 && lane < 8) {     // heads 8..15 absent: empty state
            wbuf[8 + lane] = -INFINITY;
            wbuf[24 + lane] = 0.f;
        }
        // RLA: den[16] at kDen, the warp's row count at kNval, Olin[16][D] at kLin
        constexpr int kDen = 32 + 16 * D, kNval = kDen + 16, kLin = kDen + 32;
        if constexpr (RLA) {
#pragma unroll
            for (int nt = 0; nt < NH8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int hd = nt * 8 + 2 * cq + e;
                    if (gq == 0) wbuf[kDen + hd] = den_r[nt][e];
#pragma unroll
                    for (int dt = 0; dt < TL::KSTEPS; ++dt) {
                        wbuf[kLin + hd * D + dt * 16 + gq] = lin[dt][nt][e];
                        wbuf[kLin + hd * D + dt * 16 + gq + 8] = lin[dt][nt][2 + e];
                    }
                }
            if (lane == 0) wbuf[kNval] = float(nval);
        }
        __syncthreads();
        const bool whole = !RLA && a == 0 && bnd == tiles_u;
        const int slot = u + cta;
        const size_t n_slots = size_t(U) + gridDim.x;
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
                float* part = p.partials + (size_t(row) * n_slots + slot) * (D + 2);
                part[col] = O;
                if (col == 0) {
                    part[D] = M;
                    part[D + 1] = L;
                }
                if constexpr (RLA) {     // (Olin, sum of weights, rows) of this CTA's share
                    float* rp = p.partials + (size_t(nh) * n_slots + size_t(row) * n_slots + slot) * (D + 2);
                    float Lin = 0.f, Den = 0.f, Nv = 0.f;
#pragma unroll
                    for (int w = 0; w < kAtWarps; ++w) {
                        const float* wb = reinterpret_cast<const float*>(ring + size_t(w) * kStages * TL::BYTES);
                        Lin += wb[kLin + row * D + col];
                        Den += wb[kDen + row];
                        Nv += wb[kNval];
                    }
                    rp[col] = Lin;
                    if (col == 0) {
                        rp[D] = Den;
                        rp[D + 1] = Nv;
                    }
                }
            }
        }
        __syncthreads();   // rings are reused by the next segment
        x = seg_end;
    }
}

// Log-sum-exp combine of the partials of every unit split over several CTAs.
// grid (U, heads per unit), 256 threads.  Partials are stored head-major, so the records
// (o[D], m, l) of one (unit, head) are contiguous: they are staged into shared memory in
// chunks with every load of a thread issued at once, then merged against the unit's
// maximum M with a fixed assignment of records to thread groups and a fixed-order sum.
// A unit of at most kCombRecs records (every unit of a 2-CTA-per-SM grid split over at most
// 128 CTAs) is staged in one round and takes M from the staged records, so its only global
// round trip is that one; longer units first read every record's m, then stage in chunks.
constexpr int kCombRecs = 128;   // records staged per chunk (dynamic shared memory)

//
// RLA: every unit, empty ones included, is finished here.  With the unit's sums of Olin,
// weights and rows over its CTAs, the residual linear attention of head h is
//   o_rla = (phi(q)^T S - Olin) / (phi(q) . z - sum w),   0 when the rows cover the cache,
// and the output is the exact attention plus gamma * o_rla / sqrt(mean(o_rla^2) + eps)
// ("SPLA", sections 2.2-2.3).
template <int D, bool RLA>
__global__ void __launch_bounds__(256)
combine_kernel(AttendParams p, int nh, int n_slots) {
    pdl_enter();
    constexpr int REC = D + 2;
    constexpr int PAIRS = D / 2;                 // float2 columns
    constexpr int GROUPS = 256 / PAIRS;          // record groups
    constexpr int LOADS = (kCombRecs * REC / 2 + 255) / 256;
    const int u = blockIdx.x, row = blockIdx.y;
    const int c_lo = p.unit_ctas[2 * u], c_hi = p.unit_ctas[2 * u + 1];
    if ((!RLA && c_lo < 0) || row >= nh) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_c = c_lo < 0 ? 0 : c_hi - c_lo + 1;
    const size_t first = size_t(row) * n_slots + u + (c_lo < 0 ? 0 : c_lo);
    const float* base = p.partials + first * REC;

    extern __shared__ __align__(16) float st[];   // [kCombRecs][REC]
    __shared__ float s_red[8];
    __shared__ float sL[GROUPS], sO[GROUPS][D];
    // the unit's maximum m over its records, as seen by every thread
    auto block_max = [&](float mx) -> float {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) s_red[warp] = mx;
        __syncthreads();
        float r = -INFINITY;
#pragma unroll
        for (int w = 0; w < 8; ++w) r = fmaxf(r, s_red[w]);
        return r;
    };
    const bool one_round = n_c <= kCombRecs;
    float M = -INFINITY;
    if (!one_round) {
        float mx = -INFINITY;
        for (int c = tid; c < n_c; c += 256) mx = fmaxf(mx, __ldcg(base + size_t(c) * REC + D));
        M = block_max(mx);
    }

    const int pair = tid % PAIRS, grp = tid / PAIRS;
    float L = 0.f, O0 = 0.f, O1 = 0.f;
    for (int c0 = 0; c0 < n_c; c0 += kCombRecs) {
        const int nr = min(kCombRecs, n_c - c0);
        const int n2 = nr * REC / 2;                     // float2 count (REC is even)
        const float2* src = reinterpret_cast<const float2*>(base + size_t(c0) * REC);
        float2 t[LOADS];
#pragma unroll
        for (int k = 0; k < LOADS; ++k) {
            const int i = tid + k * 256;
            t[k] = i < n2 ? __ldcg(src + i) : make_float2(0.f, 0.f);
        }
        __syncthreads();   // previous chunk consumed
#pragma unroll
        for (int k = 0; k < LOADS; ++k) {
            const int i = tid + k * 256;
            if (i < n2) reinterpret_cast<float2*>(st)[i] = t[k];
        }
        __syncthreads();
        if (one_round) M = block_max(tid < nr ? st[tid * REC + D] : -INFINITY);   // nr <= kCombRecs <= 256
        const float Mr = M == -INFINITY ? 0.f : M;
        for (int r = grp; r < nr; r += GROUPS) {
            const float* rec = st + r * REC;
            const float sc = exp2f(rec[D] - Mr);
            L += rec[D + 1] * sc;
            const float2 o = reinterpret_cast<const float2*>(rec)[pair];
            O0 += o.x * sc;
            O1 += o.y * sc;
        }
    }
    if (pair == 0) sL[grp] = L;
    sO[grp][2 * pair] = O0;
    sO[grp][2 * pair + 1] = O1;
    __syncthreads();
    if (!RLA && tid >= D) return;
    const bool act = tid < D;
    float Lt = 0.f, Ot = 0.f;
    if (act) {
#pragma unroll
        for (int g = 0; g < GROUPS; ++g) {
            Lt += sL[g];
            Ot += sO[g][tid];
        }
    }
    const UnitGeom ug = unit_geom(p, u, nh);
    const size_t o = (size_t(ug.b) * p.Hq + ug.h0 + row) * D + tid;
    float val = Lt > 0.f ? Ot / Lt : 0.f;
    if constexpr (RLA) {
        __shared__ float s_phq[D], s_sq[8];
        const float* rbase = p.partials + (size_t(nh) * n_slots + first) * REC;
        float lin = 0.f, den = 0.f, nval = 0.f;
        if (act) {
            for (int c = 0; c < n_c; ++c) {           // fixed order over the unit's CTAs
                const float* rec = rbase + size_t(c) * REC;
                lin += __ldcg(rec + tid);
                den += __ldcg(rec + D);
                nval += __ldcg(rec + D + 1);
            }
            s_phq[tid] = expf(__uint_as_float(uint32_t(p.q[o]) << 16));
        }
        __syncthreads();
        float num_all = 0.f, den_all = 0.f;
        if (act) {
            const float* Sb = p.rla_S + size_t(ug.bh) * D * D;
            const float* zb = p.rla_z + size_t(ug.bh) * D;
#pragma unroll 8
            for (int i = 0; i < D; ++i) {
                num_all += s_phq[i] * __ldg(Sb + size_t(i) * D + tid);
                den_all += s_phq[i] * __ldg(zb + i);
            }
        }
        const float orla = act && nval < float(p.N) ? (num_all - lin) / (den_all - den) : 0.f;
        float sq = orla * orla;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        if (lane == 0) s_sq[warp] = sq;
        __syncthreads();
        if (!act) return;
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < D / 32; ++w) tot += s_sq[w];
        val += __ldg(p.rla_gamma + size_t(ug.h0 + row) * D + tid) * orla / sqrtf(tot / D + p.rla_eps);
    }
    const __nv_bfloat16 bv = __float2bfloat16_rn(val);
    p.out[o] = *reinterpret_cast<const uint16_t*>(&bv);
    if (p.out_f32) p.out_f32[o] = val;
    if (p.lse && tid == 0)
        p.lse[size_t(ug.b) * p.Hq + ug.h0 + row] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
}

template <int D>
size_t attend_smem(int U) {
    return align_up(size_t(U + 1) * 4, 128) + size_t(kWinTiles) * kRows * 4 +
           size_t(kAtWarps) * kStages * Tile<D>::BYTES;
}

}  // namespace

int attend_grid() { return device_info().num_sms * 2; }

size_t attend_scratch_bytes(int U, int heads_per_unit, int d) {
    const size_t meta = align_up(size_t(U) * 8, 256);
    // exact partials (o, m, l), then the RLA partials (Olin, sum of weights, rows)
    const size_t partials = 2 * size_t(U + attend_grid()) * heads_per_unit * (d + 2) * 4;
    return meta + align_up(partials, 256);
}

spa_status launch_attend(const AttendParams& p, cudaStream_t st) {
    const int G = p.Hq / p.Hkv;
    const int U = p.collapse == SPA_COLLAPSE_GROUP_MEAN ? p.B * p.Hkv : p.B * p.Hq;
    const int nh = p.collapse == SPA_COLLAPSE_GROUP_MEAN ? G : 1;
    if (U > kMaxUnits || nh > 16) return SPA_ERR_UNSUPPORTED_SHAPE;
    const int grid = attend_grid();
    const bool rla = p.rla_S != nullptr;
#define SPA_AT_CASE(DD, H8, R)                                                                                   \
    if (p.d == DD && (nh + 7) / 8 == H8 && rla == R) {                                                          \
        const size_t sm = attend_smem<DD>(U);                                                                   \
        SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(attend_kernel<DD, H8, R>),                     \
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)));                     \
        SPA_CUDA_TRY(launch_pdl(attend_kernel<DD, H8, R>, dim3(grid), dim3(kAtThreads), sm, st, p, U, nh));      \
        const size_t cs = size_t(kCombRecs) * (DD + 2) * 4;                                                    \
        SPA_CUDA_TRY(set_func_attr(reinterpret_cast<const void*>(combine_kernel<DD, R>),                        \
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(cs)));                     \
        SPA_CUDA_TRY(launch_pdl(combine_kernel<DD, R>, dim3(U, nh), dim3(256), cs, st, p, nh, U + grid));         \
        return SPA_OK;                                                                                          \
    }
    SPA_AT_CASE(128, 1, false) SPA_AT_CASE(128, 2, false) SPA_AT_CASE(64, 1, false) SPA_AT_CASE(64, 2, false)
    SPA_AT_CASE(128, 1, true) SPA_AT_CASE(128, 2, true) SPA_AT_CASE(64, 1, true) SPA_AT_CASE(64, 2, true)
#undef SPA_AT_CASE
    return SPA_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace spa
