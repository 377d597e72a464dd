// Top-p selection for callers that cannot hand the library a workspace.
//
// spa_select_topp needs scratch (a status word and the per-unit level-0 histogram) that
// its caller allocates.  Some callers cannot allocate device memory when they call: an
// inference server that reserves all device memory at start-up and forbids allocation on
// the request path, or a plug-in whose host framework owns every device buffer.
// spa_select_topp_static serves them: its scratch is a file-scope __device__ array of
// fixed size, resident on every GPU that loads the library until the process exits.
//
// Host code must not pass the array's name to a kernel (on the host it names a host-side
// stand-in, not device memory); the device address is obtained once per device with
// cudaGetSymbolAddress and cached.
#include <mutex>
#include <vector>

#include "internal.cuh"

namespace spa {
namespace {

constexpr int kStaticUnits = SPA_SELECT_STATIC_MAX_UNITS;
constexpr size_t kStaticHistBytes =
    ((size_t(kStaticUnits) * kHistBins * 4 + 255) / 256) * 256 +
    ((size_t(kStaticUnits) * kHistBins * 8 + 255) / 256) * 256 +
    ((size_t(kStaticUnits) * 4 + 255) / 256) * 256 +
    ((size_t(kStaticUnits) * kLvlBins * 4 + 255) / 256) * 256 +
    ((size_t(kStaticUnits) * kLvlBins * 8 + 255) / 256) * 256;
constexpr size_t kStaticScratchBytes = kWsHeader + kStaticHistBytes;

// status word (first 256 bytes) + level-0 histogram of up to kStaticUnits units
__device__ __align__(256) unsigned char g_select_scratch[kStaticScratchBytes];

std::mutex g_mu;
std::vector<void*> g_addr;   // device address of g_select_scratch per device ordinal

// Device address of the scratch array on the current device; set up on the first call
// made with that device current.
spa_status scratch_address(void** out) {
    int dev = 0;
    SPA_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(g_mu);
    if (int(g_addr.size()) <= dev) g_addr.resize(dev + 1, nullptr);
    if (!g_addr[dev]) {
        void* p = nullptr;
        SPA_CUDA_TRY(cudaGetSymbolAddress(&p, g_select_scratch));
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return SPA_OK;
}

}  // namespace
}  // namespace spa

using namespace spa;

extern "C" spa_status spa_select_topp_static(const float* scores, const int32_t* unit_len, int U, int M, float p,
                                             int sink, int window, int32_t* idx, int32_t* count, int cap,
                                             float* index_mass, void* stream) {
    if (U < 0 || M < 0 || sink < 0 || window < 0 || cap < 0) return SPA_ERR_INVALID_ARG;
    if (U > kStaticUnits) return SPA_ERR_UNSUPPORTED_SHAPE;    // beyond the fixed scratch
    if (U == 0) return SPA_OK;
    if (!scores || !idx || !count) return SPA_ERR_INVALID_ARG;
    if (!(p > 0.f && p <= 1.f)) return SPA_ERR_INVALID_ARG;
    if (M > (1 << 23)) return SPA_ERR_UNSUPPORTED_SHAPE;
    void* scratch = nullptr;
    spa_status s = scratch_address(&scratch);
    if (s != SPA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: start from a zero status word and
    // zero histograms (the part this call uses)
    const size_t used = kWsHeader + hist0_bytes(U);   // never above kStaticScratchBytes (U <= kStaticUnits)
    SPA_CUDA_TRY(cudaMemsetAsync(scratch, 0, used, st));
    uint8_t* w = static_cast<uint8_t*>(scratch);
    SelectParams sp{hist0_carve(w + kWsHeader, U), scores, unit_len, U, M, 0, p, sink, window, idx, count, cap,
                    index_mass, reinterpret_cast<uint32_t*>(w)};
    s = launch_hist0(sp, true, st);
    if (s != SPA_OK) return s;
    return launch_select(sp, true, st);
}

// Status word of the fixed scratch: the select kernel ORs SPA_ERR_TIMEOUT / SPA_ERR_CAPACITY
// into it.  Copied with one cudaMemcpyAsync on the caller's stream (and cleared with one
// cudaMemsetAsync if asked); nothing is allocated.
extern "C" spa_status spa_select_static_status(void* stream, uint32_t* bits, int reset) {
    if (!bits) return SPA_ERR_INVALID_ARG;
    void* scratch = nullptr;
    spa_status s = scratch_address(&scratch);
    if (s != SPA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SPA_CUDA_TRY(cudaMemcpyAsync(bits, scratch, sizeof(uint32_t), cudaMemcpyDeviceToHost, st));
    SPA_CUDA_TRY(cudaStreamSynchronize(st));
    if (reset) {
        SPA_CUDA_TRY(cudaMemsetAsync(scratch, 0, sizeof(uint32_t), st));
        SPA_CUDA_TRY(cudaStreamSynchronize(st));
    }
    return SPA_OK;
}
