// State of the residual linear attention ("SPLA", section 2.2).
//
// RLA is linear attention with the parameter-free feature map phi(x) = exp(x), applied
// to every component.  Its recurrent state per (batch, kv head) is
//   S = sum_n phi(k_n) v_n^T   [d x d]     and     z = sum_n phi(k_n)   [d],
// and the decode step reads it to form the global term phi(q)^T S / phi(q) . z, from which
// the attention kernel subtracts the linear attention over the rows it gathered.  This file
// adds rows [n0, n1) of every (batch, kv head) into (S, z): the whole cache once after a
// prefill, then each appended token.
//
// S is a dense contraction over the rows, phi(K)^T V, so it runs on tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate).  phi(k) is evaluated in fp32 and carried
// as the sum of two bf16 terms (hi + lo, about 16 significant bits); V is bf16 already and
// enters exactly.  z is summed from the fp32 values.
//
// Grid: (d / 32 column slabs of V, B * Hkv).  A CTA of 8 warps streams the rows of its
// (batch, kv head) through a 4-stage cp.async ring of 32-row stages (K rows whole, 32
// columns of V).  Warp w takes features [d/4 * (w % 4), d/4 * (w % 4 + 1)) of the 16-row
// half w / 4 of every stage; the two halves' sums are added in a fixed order at the end,
// then added into S, so a call is deterministic.
#include "internal.cuh"
#include "warp_mma.cuh"

namespace spa {
namespace {

constexpr int kStThreads = 256;
constexpr int kSlab = 32;           // V columns per CTA
constexpr int kStageRows = 32;      // rows per ring stage: one 16-row tile per half
constexpr int kStStages = 4;

template <int D>
struct StTile {
    static constexpr int KCH = D / 8;                          // 16-byte chunks per K row
    static constexpr int KBYTES = kStageRows * D * 2;
    static constexpr int VBYTES = kStageRows * kSlab * 2;      // 4 chunks per row
    static constexpr int BYTES = KBYTES + VBYTES;
    static constexpr int FPW = D / 4;                          // features per warp
    static constexpr int MT = FPW / 16;                        // 16-feature m-tiles per warp
};

// byte offset of chunk ch of stage row r (XOR swizzles keep ldmatrix free of bank conflicts)
template <int D>
__device__ __forceinline__ uint32_t k_off(int r, int ch) {
    return uint32_t(r * StTile<D>::KCH + (ch ^ (r & 7))) * 16;
}
__device__ __forceinline__ uint32_t v_off(int r, int ch) { return uint32_t(r * 4 + (ch ^ ((r >> 1) & 3))) * 16; }

template <int D>
__global__ void __launch_bounds__(kStThreads)
rla_state_kernel(const uint16_t* __restrict__ K, const uint16_t* __restrict__ V, int N, int n0, int n1,
                 float* __restrict__ S, float* __restrict__ z) {
    pdl_enter();
    using TL = StTile<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int fg = warp & 3, half = warp >> 2;
    const int g = lane >> 2, c = lane & 3;
    const int slab = blockIdx.x;
    const size_t bh = blockIdx.y;
    const uint16_t* Kb = K + bh * size_t(N) * D;
    const uint16_t* Vb = V + bh * size_t(N) * D + slab * kSlab;
    const int n_stages = (n1 - n0 + kStageRows - 1) / kStageRows;

    auto issue = [&](int t, int stage) {
        const uint32_t kb = smem_u32(smem + size_t(stage) * TL::BYTES), vb = kb + TL::KBYTES;
        const int r0 = n0 + t * kStageRows;
        for (int i = tid; i < kStageRows * TL::KCH; i += kStThreads) {
            const int r = i / TL::KCH, ch = i % TL::KCH;
            const bool ok = r0 + r < n1;
            cp_async16(kb + k_off<D>(r, ch), Kb + (ok ? size_t(r0 + r) * D + ch * 8 : 0), ok);
        }
        if (tid < kStageRows * 4) {
            const int r = tid >> 2, ch = tid & 3;
            const bool ok = r0 + r < n1;
            cp_async16(vb + v_off(r, ch), Vb + (ok ? size_t(r0 + r) * D + ch * 8 : 0), ok);
        }
    };

    float acc[TL::MT][4][4];          // m-tile x n-tile x C fragment
    float zs[TL::MT][2];              // features f0 + g and f0 + 8 + g of each m-tile
#pragma unroll
    for (int mt = 0; mt < TL::MT; ++mt) {
        zs[mt][0] = zs[mt][1] = 0.f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
    }

#pragma unroll
    for (int j = 0; j < kStStages - 1; ++j) {
        if (j < n_stages) issue(j, j);
        cp_commit();
    }
    for (int t = 0; t < n_stages; ++t) {
        if (t + kStStages - 1 < n_stages) issue(t + kStStages - 1, (t + kStStages - 1) % kStStages);
        cp_commit();
        cp_wait<kStStages - 1>();
        __syncthreads();
        const uint32_t kb = smem_u32(smem + size_t(t % kStStages) * TL::BYTES), vb = kb + TL::KBYTES;
        const int rfirst = n0 + t * kStageRows + half * 16;     // first row of this warp's tile
        // rows 2c, 2c + 1 (fragment registers 0, 1) and 2c + 8, 2c + 9 (registers 2, 3)
        const bool ok0 = rfirst + 2 * c < n1, ok1 = rfirst + 2 * c + 1 < n1;
        const bool ok2 = rfirst + 2 * c + 8 < n1, ok3 = rfirst + 2 * c + 9 < n1;
        const int mat = lane >> 3;

        // B = V[16 rows x 8 columns] per n-tile, through transposing ldmatrix
        uint32_t bv[4][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = half * 16 + (mat & 1) * 8 + (lane & 7);
            ldsm_x4_t(vb + v_off(r, 2 * h + (mat >> 1)), bv[2 * h][0], bv[2 * h][1], bv[2 * h + 1][0],
                      bv[2 * h + 1][1]);
        }
        // A = phi(K)^T [16 features x 16 rows] per m-tile
#pragma unroll
        for (int mt = 0; mt < TL::MT; ++mt) {
            const int f0 = fg * TL::FPW + mt * 16;
            const int r = half * 16 + (mat >> 1) * 8 + (lane & 7);
            uint32_t a[4], ah[4], al[4];
            ldsm_x4_t(kb + k_off<D>(r, f0 / 8 + (mat & 1)), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 kf = bf16x2_to_float2(a[i]);
                const float e0 = expf(kf.x), e1 = expf(kf.y);
                split_bf16(e0, e1, ah[i], al[i]);
                const bool va = i < 2 ? ok0 : ok2, vb2 = i < 2 ? ok1 : ok3;
                zs[mt][i & 1] += (va ? e0 : 0.f) + (vb2 ? e1 : 0.f);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                mma16816(acc[mt][nt], ah, bv[nt][0], bv[nt][1]);
                mma16816(acc[mt][nt], al, bv[nt][0], bv[nt][1]);
            }
        }
        __syncthreads();   // the stage is refilled by the next iteration
    }
    cp_wait<0>();
    __syncthreads();

    // z: sum over the four lanes of a row group, then over the halves
#pragma unroll
    for (int mt = 0; mt < TL::MT; ++mt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            zs[mt][e] += __shfl_xor_sync(0xffffffffu, zs[mt][e], 1);
            zs[mt][e] += __shfl_xor_sync(0xffffffffu, zs[mt][e], 2);
        }
    float* red = reinterpret_cast<float*>(smem);       // [4 warps][MT * 18][32]
    constexpr int PER = TL::MT * 18;
    if (half == 1) {
#pragma unroll
        for (int mt = 0; mt < TL::MT; ++mt) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[(fg * PER + mt * 18 + nt * 4 + i) * 32 + lane] = acc[mt][nt][i];
            red[(fg * PER + mt * 18 + 16) * 32 + lane] = zs[mt][0];
            red[(fg * PER + mt * 18 + 17) * 32 + lane] = zs[mt][1];
        }
    }
    __syncthreads();
    if (half == 1) return;
    float* Sb = S + bh * size_t(D) * D;
#pragma unroll
    for (int mt = 0; mt < TL::MT; ++mt) {
        const int f = fg * TL::FPW + mt * 16 + g;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const float* o = red + (fg * PER + mt * 18 + nt * 4) * 32 + lane;
            const int col = slab * kSlab + nt * 8 + 2 * c;
            float2* p0 = reinterpret_cast<float2*>(Sb + size_t(f) * D + col);
            float2* p1 = reinterpret_cast<float2*>(Sb + size_t(f + 8) * D + col);
            float2 v0 = *p0, v1 = *p1;
            v0.x += acc[mt][nt][0] + o[0];
            v0.y += acc[mt][nt][1] + o[32];
            v1.x += acc[mt][nt][2] + o[64];
            v1.y += acc[mt][nt][3] + o[96];
            *p0 = v0;
            *p1 = v1;
        }
        if (slab == 0 && c == 0) {
            z[bh * D + f] += zs[mt][0] + red[(fg * PER + mt * 18 + 16) * 32 + lane];
            z[bh * D + f + 8] += zs[mt][1] + red[(fg * PER + mt * 18 + 17) * 32 + lane];
        }
    }
}

}  // namespace

spa_status launch_rla_state(const uint16_t* K, const uint16_t* V, int BH, int N, int d, int n0, int n1, float* S,
                            float* z, cudaStream_t st) {
    if (BH == 0 || n1 <= n0) return SPA_OK;
    if (BH > 65535) return SPA_ERR_UNSUPPORTED_SHAPE;
    if (d == 128) {
        SPA_CUDA_TRY(launch_pdl(rla_state_kernel<128>, dim3(128 / kSlab, BH), dim3(kStThreads),
                                size_t(kStStages) * StTile<128>::BYTES, st, K, V, N, n0, n1, S, z));
        return SPA_OK;
    }
    if (d == 64) {
        SPA_CUDA_TRY(launch_pdl(rla_state_kernel<64>, dim3(64 / kSlab, BH), dim3(kStThreads),
                                size_t(kStStages) * StTile<64>::BYTES, st, K, V, N, n0, n1, S, z));
        return SPA_OK;
    }
    return SPA_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace spa
