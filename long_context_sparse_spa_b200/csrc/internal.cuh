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

__device__ __forceinline__ void raise_status(uint32_t* status, int code) {
    if (status) atomicOr(status, 1u << code);
}

// ------------------------------------------------------------------ launchers
// scores.cu
spa_status launch_lowrank_scores(const uint16_t* qidx, const uint16_t* kidx, int B, int Hq, int Hkv, int M,
                                 int collapse, float scale, float* scores, int* zero_ptr, int zero_count,
                                 cudaStream_t st);
spa_status launch_taylor_scores(const uint16_t* q, const float* mean, const float* var, int B, int Hq, int Hkv,
                                int M, int d, int collapse, float scale, float* scores, int* zero_ptr,
                                int zero_count, cudaStream_t st);
spa_status launch_block_stats(const uint16_t* K, int B, int Hkv, int N, int d, int block, float* mean,
                              float* var, cudaStream_t st);

// select.cu
struct SelectParams {
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
};
spa_status launch_select(const SelectParams& p, bool topp, cudaStream_t st);

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
    int* tickets;      // [U], zero on entry; left zero on exit
    float* partials;   // [(U + grid) * heads_per_unit * (d + 2)]
    uint32_t* status;
};
size_t attend_scratch_bytes(int U, int heads_per_unit, int d);   // tickets + partials
int attend_grid();
spa_status launch_attend(const AttendParams& p, cudaStream_t st);

}  // namespace spa
