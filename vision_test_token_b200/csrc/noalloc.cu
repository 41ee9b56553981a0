// noalloc.cu -- ttt_forward_linear_noalloc: the linear-head forward for callers that cannot allocate
// device memory (see include/ttt.h).  It runs the same kernels as ttt_forward_linear; the scratch
// that the caller would otherwise pass as a workspace lives in one fixed-size array that the library
// owns on every device that loads it.
#include <mutex>

#include "ttt_internal.h"

namespace ttt {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

// Library-owned scratch.  In host code this name is only a stand-in for the device array: its
// device address is fetched with cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device (looked up on the first use per device).
static ttt_status noalloc_scratch(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_launch(e);
    if (dev < 0 || dev >= kMaxDevices) return TTT_ERR_UNSUPPORTED;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return check_launch(e);
        if (!p) return TTT_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return TTT_OK;
}

}  // namespace ttt

using namespace ttt;

extern "C" ttt_status ttt_forward_linear_noalloc(const void* Q, const void* K, const void* V, const float* W0,
                                                 void* Z, float eta, const ttt_shape* s, float* W1_out,
                                                 void* stream) {
    const size_t need = ttt_workspace_bytes(TTT_HEAD_LINEAR, s);
    if (need == 0)   // invalid shape: report the precise reason
        return validate_call(TTT_HEAD_LINEAR, Q, K, V, W0, nullptr, Z, eta, s, nullptr, 0, 0, stream);
    if (need > kNoAllocScratchBytes) return TTT_ERR_WORKSPACE;
    void* ws = nullptr;
    ttt_status st = noalloc_scratch(&ws);
    if (st != TTT_OK) return st;
    st = validate_call(TTT_HEAD_LINEAR, Q, K, V, W0, nullptr, Z, eta, s, ws, kNoAllocScratchBytes, need, stream);
    if (st != TTT_OK) return st;
    // The scratch keeps the previous call's contents: clear the words that must start at zero.
    const cudaError_t e = cudaMemsetAsync(ws, 0, linear_ws_control_bytes(*s), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return check_launch(e);
    return ttt_forward_linear(Q, K, V, W0, Z, eta, s, ws, kNoAllocScratchBytes, W1_out, stream);
}
