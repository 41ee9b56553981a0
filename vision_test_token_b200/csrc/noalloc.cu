// noalloc.cu -- ttt_forward_linear_noalloc and ttt_noalloc_status: the linear-head forward for callers
// that cannot allocate device memory (see include/ttt.h).  It runs the same kernels as
// ttt_forward_linear; the scratch that the caller would otherwise pass as a workspace lives in one
// fixed-size array that the library owns on every device that loads it.
#include <mutex>

#include "ttt_internal.h"

namespace ttt {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

// Library-owned scratch.  In host code this name is only a stand-in for the device array: its
// device address is fetched with cudaGetSymbolAddress, with the device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of the scratch on the current device.  It is looked up on the first use per device
// and again whenever the device's current context differs from the one the address was taken in
// (after a cudaDeviceReset the module is loaded anew and the old address is stale).
ttt_status noalloc_scratch(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_launch(e);
    if (dev < 0 || dev >= kMaxDevices) return TTT_ERR_UNSUPPORTED;
    CtxGetCurrentFn get = ctx_get_current();
    CUcontext ctx = nullptr;
    if (!get || get(&ctx) != CUDA_SUCCESS) return TTT_ERR_CUDA;
    if (!ctx) {
        // no context is current yet: the runtime's first call on the device creates it
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return check_launch(e);
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return TTT_ERR_CUDA;
    }
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    static CUcontext addr_ctx[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || addr_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return check_launch(e);
        if (!p) return TTT_ERR_CUDA;
        addr[dev] = p;
        addr_ctx[dev] = ctx;
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
    Call c;
    st = prepare_linear(Q, K, V, W0, Z, eta, s, ws, kNoAllocScratchBytes, W1_out, stream, &c);
    if (st != TTT_OK) return st;
    // The scratch keeps the previous call's contents: clear the control words that must start at
    // zero.  The error word (the first kWsHeader bytes) is kept, so that a wait that ran out in an
    // earlier call is still reported by ttt_noalloc_status.
    const size_t ctl = linear_ws_control_bytes(*s);
    if (ctl > kWsHeader) {
        const cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(ws) + kWsHeader, 0, ctl - kWsHeader,
                                              static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return check_launch(e);
    }
    return launch_linear(c);
}

extern "C" ttt_status ttt_noalloc_status(void* stream) {
    void* ws = nullptr;
    const ttt_status st = noalloc_scratch(&ws);
    if (st != TTT_OK) return st;
    return read_error_word(ws, stream);
}
