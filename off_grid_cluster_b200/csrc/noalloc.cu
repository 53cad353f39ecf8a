// noalloc.cu -- acl_cluster_attn_bwd_noalloc: the attention backward with its scratch in
// a fixed device array owned by the library, for callers that cannot allocate device
// memory themselves (for example code running inside a framework that forbids
// allocations on its hot path, or a runtime that only hands out pre-registered buffers).
//
// The scratch is a file-scope __device__ array of ACL_NOALLOC_ATTN_WS_BYTES.  Every GPU
// that loads the library keeps it for the life of the process.  Host code cannot pass the
// array's name to a kernel (on the host it is only a stand-in for the symbol), so the
// device address is looked up once per device with cudaGetSymbolAddress, with that
// device current, and cached.
#include <mutex>

#include "../../include/acl.h"
#include "internal.h"

namespace {

__device__ __align__(256) uint8_t g_attn_bwd_scratch[ACL_NOALLOC_ATTN_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_bwd_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" acl_status acl_cluster_attn_bwd_noalloc(
    const acl_bf16* Q, const acl_bf16* K, const acl_bf16* V, const float* coords,
    const int32_t* clusters, const int32_t* nbr, const float* bias_coef, int B, int N, int H,
    int D, int C, int M, float scale, const acl_bf16* O, const acl_bf16* dO, const float* lse,
    acl_bf16* dQ, acl_bf16* dK, acl_bf16* dV, float* dbias_coef, acl_stream_t stream) {
    const size_t need = acl_cluster_attn_workspace(B, N, H, C, M);
    if (need == 0) return ACL_ERR_INVALID_ARG;
    if (need > ACL_NOALLOC_ATTN_WS_BYTES) return ACL_ERR_UNSUPPORTED;
    // the scratch address is the current device's: a stream of another device is refused
    if (stream) {
        int dev = 0, sdev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) != cudaSuccess)
            return ACL_ERR_CUDA;
        if (sdev != dev) return ACL_ERR_INVALID_ARG;
    }
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return ACL_ERR_CUDA;
    return acl_cluster_attn_bwd(Q, K, V, coords, clusters, nbr, bias_coef, B, N, H, D, C, M, scale,
                                O, dO, lse, dQ, dK, dV, dbias_coef, scratch,
                                ACL_NOALLOC_ATTN_WS_BYTES, stream);
}
