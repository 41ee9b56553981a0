// ttt_internal.h -- host-side interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ttt.h"

namespace ttt {

// Workspace header: every workspace starts with kWsHeader bytes; word 0 is the device error word.
constexpr size_t kWsHeader = 256;
// Bit set in the error word when a bounded device-side wait gave up.
constexpr uint32_t kErrTimeout = 1u;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Validated, flattened description of one call.
struct Call {
    const void* Q;
    const void* K;
    const void* V;
    void* Z;
    const float* W0;     // linear / conv weights, or MLP Wa
    const float* W0b;    // MLP Wb
    float* W1_out;       // linear / conv updated weights, or MLP Wa_out (nullable)
    float* W1b_out;      // MLP Wb_out (nullable)
    float eta;
    int batch, heads, H, W, N, d, hidden;
    long long bs, hs;    // element strides
    int dtype;           // ttt_dtype
    int loss;            // ttt_loss
    uint8_t* ws;
    size_t ws_bytes;
    cudaStream_t stream;
    int num_sms;             // SMs the call may spread its work over
    int overlap_previous;    // launch as a programmatic dependent of the preceding kernel in the stream
    uint8_t* err_ws;         // workspace whose error word the kernels report to (nullptr: ws itself)
    int* grid_out;           // nullable: the launch writes the number of CTAs it launched
    unsigned long long wait_ns;   // bound of every device-side wait of the launch (ns)
};

// The library-owned array of ttt_forward_linear_noalloc on the current device (its first 256 bytes
// are a workspace header).
ttt_status noalloc_scratch(void** out);

// Bound of the device-side waits of every launch (ns), process-wide (ttt_set_wait_limit).
unsigned long long wait_limit_ns();

// Encodes a rank-4 bf16 tensor map over [batch][heads][N][64] with a 64 x box_rows box,
// 128-byte swizzle, zero fill out of bounds.  Returns false on failure.
bool make_tmap_tokens(CUtensorMap* m, const void* base, const Call& c, int box_rows);
// Rank-5 tensor map over [batch][heads][H][W][64] (the token grid), no swizzle, zero fill out of bounds,
// box = 64 channels x box_cols x box_rows of one unit.  Element type from c.dtype.
bool make_tmap_grid(CUtensorMap* m, const void* base, const Call& c, int box_cols, int box_rows);
// As make_tmap_grid, bf16 with 128-byte swizzle (a box of 64 channels is one 128-byte swizzled row
// per position, the layout of a K-major tensor-core operand).
bool make_tmap_grid_sw128(CUtensorMap* m, const void* base, const Call& c, int box_cols, int box_rows);
// Rank-2 bf16 tensor map over a contiguous [rows][cols] matrix with a cols x box_rows box (cols*2 = 128).
bool make_tmap_matrix(CUtensorMap* m, const void* base, long long rows, int cols, int box_rows);

size_t linear_ws_bytes(const ttt_shape& s);
// Bytes at the start of a linear workspace that must be zero before a call (the rest is written
// before it is read).
size_t linear_ws_control_bytes(const ttt_shape& s);
ttt_status launch_linear(const Call& c);

size_t dwconv_ws_bytes(const ttt_shape& s);
// Bytes at the start of a conv workspace that must be zero before a call (every call leaves them zero).
size_t dwconv_ws_control_bytes(const ttt_shape& s);
ttt_status launch_dwconv(const Call& c);

// Full 3x3 conv head (bf16, L2 loss).
size_t conv3x3_ws_bytes(const ttt_shape& s);
ttt_status launch_conv3x3(const Call& c);

size_t mlp_ws_bytes(const ttt_shape& s);
ttt_status launch_mlp(const Call& c);

// Backward pass of the linear head.
size_t linear_backward_ws_bytes(const ttt_shape& s);
size_t linear_backward_ws_control_bytes(const ttt_shape& s);
ttt_status launch_linear_backward(const Call& c, const void* dZ, void* dQ, void* dK, void* dV, float* dW0_out,
                                  float* deta_out);

// Backward pass of the depthwise-conv head.
size_t dwconv_backward_ws_bytes(const ttt_shape& s);
ttt_status launch_dwconv_backward(const Call& c, const void* dZ, void* dQ, void* dK, void* dV, float* dW0_out,
                                  float* deta_out);

// Backward pass of the MLP head (s: the validated shape, for the workspace layout).
size_t mlp_backward_ws_bytes(const ttt_shape& s);
ttt_status launch_mlp_backward(const Call& c, const ttt_shape& s, const void* dZ, void* dQ, void* dK, void* dV,
                               float* dWa_out, float* dWb_out, float* deta_out);

// Mini-batch linear head (its workspace is the error word only): batch_tokens >= 1, mode
// TTT_MB_PREFIX or TTT_MB_EPOCH.
ttt_status launch_linear_minibatch(const Call& c, int batch_tokens, int mode);

// Full synchronous validation of a call (the checks every entry point runs before launching).
ttt_status validate_call(int kind, const void* Q, const void* K, const void* V, const float* W0, const float* W0b,
                         void* Z, float eta, const ttt_shape* s, void* ws, size_t ws_bytes, size_t need, void* stream);

// The validation of ttt_forward_linear (shape, pointers, workspace of ws_bytes, W1_out) into *c.
ttt_status prepare_linear(const void* Q, const void* K, const void* V, const float* W0, void* Z, float eta,
                          const ttt_shape* s, void* ws, size_t ws_bytes, float* W1_out, void* stream, Call* c);

// Synchronises `stream`, reads the error word at the start of device buffer ws; a recorded timeout
// is cleared and reported as TTT_ERR_TIMEOUT.
ttt_status read_error_word(void* ws, void* stream);

// Records a launch error in the library's sticky error and maps it to a status.
ttt_status check_launch(cudaError_t e);

}  // namespace ttt
