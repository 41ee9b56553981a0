// selftest.cu -- exercises the failure-detection path of the library without a GPU fault: one kernel
// waits, with a short bound, on a workspace word that nothing sets.  When the bound runs out it takes
// the same steps as every wait in the layer kernels (raise the CTA's abort flag, OR kErrTimeout into
// the workspace error word, return), so that ttt_workspace_status reports TTT_ERR_TIMEOUT.
#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {

// Workspace word 1 (in the 256-byte header): the flag the self-test waits on.  Nothing writes it.
constexpr size_t kSelftestFlagWord = 1;

__global__ void selftest_wait(const uint32_t* flag, uint32_t* err, unsigned long long limit_ns) {
    __shared__ int abort_flag;
    if (threadIdx.x == 0) abort_flag = 0;
    __syncthreads();
    const Abort ab{&abort_flag, err};
    if (threadIdx.x != 0) return;
    const unsigned long long t0 = global_timer_ns();
    while (ld_acquire_gpu(flag) == 0u) {
        __nanosleep(1000);
        if (global_timer_ns() - t0 > limit_ns) {
            ab.raise();
            return;
        }
    }
}

}  // namespace ttt

using namespace ttt;

extern "C" ttt_status ttt_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned long long limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > 1000000000ull) return TTT_ERR_INVALID_ARG;
    if (!ws) {                       // the no-alloc entry point's array: reported by ttt_noalloc_status
        const ttt_status st = noalloc_scratch(&ws);
        if (st != TTT_OK) return st;
        ws_bytes = kWsHeader;
    }
    if (ws_bytes < kWsHeader) return TTT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % 256) return TTT_ERR_ALIGNMENT;
    uint32_t* words = static_cast<uint32_t*>(ws);
    selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(words + kSelftestFlagWord, words, limit_ns);
    return check_launch(cudaGetLastError());
}
