// moe_permute_noalloc: the S2 permutation for callers that cannot allocate.
//
// Some callers only hold the buffers they were handed: an operator invoked from
// another runtime's launch hook with nothing but input and output pointers, or a
// serving loop with a fixed memory plan in which cudaMalloc (which also
// synchronises the device) is not allowed after start-up. moe_permute asks such a
// caller for a workspace it cannot provide. This variant keeps that workspace in
// a file-scope device array instead, so the caller passes inputs and outputs only.
//
// The array is a fixed kNoAllocScratchBytes on every GPU that loads the library
// and stays allocated until the process exits. Host code cannot use the array's
// name as a device address (it denotes a host-side shadow), so the device address
// is looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on that device.
#include <mutex>

#include "internal.h"

namespace moe {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB per device

static __device__ __align__(256) unsigned char g_permute_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_ids, const float* topk_w, int T, int topk,
                                            int E, int B, const int32_t* replica_src, const void* x, int H,
                                            int32_t* cu_seqlens, int32_t* perm_token, float* perm_w,
                                            int32_t* inv_perm, void* x_perm, int M_alloc,
                                            moe_stream_t stream) {
    if (T < 0 || topk < 1 || E < 1 || B < 0 || topk > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts || E + B > kMaxRows || topk > kMaxTopk) return MOE_ERR_UNSUPPORTED;
    if (B > 0 && !replica_src) return MOE_ERR_INVALID_ARG;
    if (!cu_seqlens) return MOE_ERR_INVALID_ARG;
    // the scratch these sizes need must fit in the fixed array
    if (kErrBytes + permute_ws_layout(T, topk, E, B).bytes > kNoAllocScratchBytes)
        return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (x_perm) {
        if (!x || H <= 0 || M_alloc < T * topk) return MOE_ERR_INVALID_ARG;
        if (H % 8 || (reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u))
            return MOE_ERR_ALIGNMENT;
    }
    if (T > 0 && (!topk_ids || !perm_token || !perm_w || !inv_perm)) return MOE_ERR_INVALID_ARG;
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
    char* w = static_cast<char*>(base);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the error word must start at zero; every other scratch byte is written before it is read
    if (cudaMemsetAsync(w, 0, sizeof(DevError), st) != cudaSuccess) return MOE_ERR_CUDA;
    cudaError_t e = launch_permute(topk_ids, topk_w, T, topk, E, B, replica_src, cu_seqlens, perm_token, perm_w,
                                   inv_perm, reinterpret_cast<DevError*>(w), w + kErrBytes, st, false);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (x_perm) e = launch_gather(0, x, H, perm_token, T * topk, x_perm, nullptr, nullptr, st, true);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The device-detected status of the last moe_permute_noalloc call on the current device
// (its error word lives in the scratch array): waits for the stream, reads the word and
// clears it. Allocates nothing.
extern "C" moe_status_t moe_permute_noalloc_status(moe_stream_t stream) {
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    DevError h{0, 0};
    if (cudaMemcpy(&h, base, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (h.code != 0) {
        if (cudaMemset(base, 0, sizeof(h)) != cudaSuccess) return MOE_ERR_CUDA;
        return static_cast<moe_status_t>(h.code);
    }
    return MOE_OK;
}
