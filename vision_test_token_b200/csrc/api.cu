// api.cu -- the C ABI of libttt.so (declared in include/ttt.h): argument validation, tensor-map
// encoding, workspace helpers and error reporting.  The kernels live in linear.cu, dwconv.cu and
// mlp.cu; nothing here computes.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "ttt_internal.h"

namespace ttt {

static std::atomic<int> g_sticky{0};   // first asynchronous CUDA error seen (as cudaError_t)
static std::atomic<unsigned long long> g_wait_ns{1000000000ull};   // bound of each device-side wait

unsigned long long wait_limit_ns() { return g_wait_ns.load(); }

ttt_status check_launch(cudaError_t e) {
    if (e == cudaSuccess) return TTT_OK;
    int expected = 0;
    g_sticky.compare_exchange_strong(expected, (int)e);
    return TTT_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime, so no -lcuda is needed)
// ------------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_tmap_tokens(CUtensorMap* m, const void* base, const Call& c, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const long long esz = 2;   // bf16
    // Strides of unused dimensions (size 1) still have to be valid multiples of 16 bytes.
    const long long hs = (c.heads > 1) ? c.hs : (long long)c.N * c.d;
    const long long bs = (c.batch > 1) ? c.bs : hs * c.heads;
    cuuint64_t dims[4] = {(cuuint64_t)c.d, (cuuint64_t)c.N, (cuuint64_t)c.heads, (cuuint64_t)c.batch};
    cuuint64_t strides[3] = {(cuuint64_t)(c.d * esz), (cuuint64_t)(hs * esz), (cuuint64_t)(bs * esz)};
    cuuint32_t box[4] = {(cuuint32_t)c.d, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_grid(CUtensorMap* m, const void* base, const Call& c, int box_cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const long long esz = (c.dtype == TTT_BF16) ? 2 : 4;
    const long long hs = (c.heads > 1) ? c.hs : (long long)c.N * c.d;
    const long long bs = (c.batch > 1) ? c.bs : hs * c.heads;
    cuuint64_t dims[5] = {(cuuint64_t)c.d, (cuuint64_t)c.W, (cuuint64_t)c.H, (cuuint64_t)c.heads, (cuuint64_t)c.batch};
    cuuint64_t strides[4] = {(cuuint64_t)(c.d * esz), (cuuint64_t)((long long)c.W * c.d * esz), (cuuint64_t)(hs * esz),
                             (cuuint64_t)(bs * esz)};
    cuuint32_t box[5] = {(cuuint32_t)c.d, (cuuint32_t)box_cols, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, (c.dtype == TTT_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_grid_sw128(CUtensorMap* m, const void* base, const Call& c, int box_cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const long long esz = 2;   // bf16
    const long long hs = (c.heads > 1) ? c.hs : (long long)c.N * c.d;
    const long long bs = (c.batch > 1) ? c.bs : hs * c.heads;
    cuuint64_t dims[5] = {(cuuint64_t)c.d, (cuuint64_t)c.W, (cuuint64_t)c.H, (cuuint64_t)c.heads, (cuuint64_t)c.batch};
    cuuint64_t strides[4] = {(cuuint64_t)(c.d * esz), (cuuint64_t)((long long)c.W * c.d * esz), (cuuint64_t)(hs * esz),
                             (cuuint64_t)(bs * esz)};
    cuuint32_t box[5] = {(cuuint32_t)c.d, (cuuint32_t)box_cols, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_matrix(CUtensorMap* m, const void* base, long long rows, int cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------------------------------
// Validation
// ------------------------------------------------------------------------------------------------
static ttt_status check_shape(int kind, const ttt_shape* s) {
    if (!s) return TTT_ERR_INVALID_ARG;
    if (s->batch < 1 || s->heads < 1 || s->H < 1 || s->W < 1 || s->d < 1) return TTT_ERR_INVALID_ARG;
    if ((long long)s->H * s->W > (1LL << 30)) return TTT_ERR_INVALID_ARG;
    if (s->dtype != TTT_FP32 && s->dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if (s->batch_stride < 0 || s->head_stride < 0 || s->max_sms < 0) return TTT_ERR_INVALID_ARG;
    if (s->loss != TTT_LOSS_L2 && s->loss != TTT_LOSS_DOT) return TTT_ERR_INVALID_ARG;
    if ((long long)s->batch * s->heads > (1LL << 24)) return TTT_ERR_INVALID_ARG;
    if (s->d != 64) return TTT_ERR_UNSUPPORTED;
    if (kind == TTT_HEAD_CONV3X3) {
        if (s->dtype != TTT_BF16) return TTT_ERR_UNSUPPORTED;
        if (s->loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    }
    if (kind == TTT_HEAD_MLP_BACKWARD) {
        if (s->hidden < 64 || s->hidden % 64 != 0) return TTT_ERR_INVALID_ARG;
        if (s->hidden > 256) return TTT_ERR_UNSUPPORTED;
        if (s->loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    }
    if (kind == TTT_HEAD_MLP) {
        if (s->hidden < 64 || s->hidden % 64 != 0) return TTT_ERR_INVALID_ARG;
        if (s->hidden > 256) return TTT_ERR_UNSUPPORTED;
        if (s->dtype != TTT_BF16) return TTT_ERR_UNSUPPORTED;
        if (s->loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    }
    const long long N = (long long)s->H * s->W;
    const long long span = N * s->d;
    if (s->heads > 1 && s->head_stride < span) return TTT_ERR_INVALID_ARG;          // heads may not overlap
    if (s->batch > 1 && s->batch_stride < (long long)(s->heads - 1) * s->head_stride + span)
        return TTT_ERR_INVALID_ARG;                                                   // images may not overlap
    const int align_elems = (s->dtype == TTT_BF16) ? 8 : 4;                         // 16 bytes
    if ((s->heads > 1 && s->head_stride % align_elems) || (s->batch > 1 && s->batch_stride % align_elems))
        return TTT_ERR_ALIGNMENT;
    return TTT_OK;
}

static bool is_device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();   // clear the non-sticky error
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

static long long extent_bytes(const ttt_shape* s) {   // bytes spanned by one Q/K/V/Z view
    const long long esz = (s->dtype == TTT_BF16) ? 2 : 4;
    const long long N = (long long)s->H * s->W;
    return ((long long)(s->batch - 1) * s->batch_stride + (long long)(s->heads - 1) * s->head_stride + N * s->d) * esz;
}

static bool overlaps(const void* a, const void* b, long long n) {
    const char* x = static_cast<const char*>(a);
    const char* y = static_cast<const char*>(b);
    return x < y + n && y < x + n;
}

static ttt_status prepare(int kind, const void* Q, const void* K, const void* V, const float* W0, const float* W0b,
                          void* Z, float eta, const ttt_shape* s, void* ws, size_t ws_bytes, size_t need,
                          void* stream, Call* c) {
    ttt_status st = check_shape(kind, s);
    if (st != TTT_OK) return st;
    if (!Q || !K || !V || !W0 || !Z || ((kind == TTT_HEAD_MLP || kind == TTT_HEAD_MLP_BACKWARD) && !W0b))
        return TTT_ERR_INVALID_ARG;
    if (!std::isfinite(eta)) return TTT_ERR_INVALID_ARG;
    if (need > 0 && (!ws || ws_bytes < need)) return TTT_ERR_WORKSPACE;   // need 0: the call takes no workspace
    for (const void* p : {Q, K, V, (const void*)Z})
        if (reinterpret_cast<uintptr_t>(p) % 16) return TTT_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(W0) % 16 || (W0b && reinterpret_cast<uintptr_t>(W0b) % 16) ||
        (ws && reinterpret_cast<uintptr_t>(ws) % 256))
        return TTT_ERR_ALIGNMENT;
    const long long ext = extent_bytes(s);
    if (overlaps(Z, Q, ext) || overlaps(Z, K, ext) || overlaps(Z, V, ext)) return TTT_ERR_INVALID_ARG;
    for (const void* p : {Q, K, V, (const void*)Z, (const void*)W0})
        if (!is_device_ptr(p)) return TTT_ERR_INVALID_ARG;
    if (ws && !is_device_ptr(ws)) return TTT_ERR_INVALID_ARG;
    if (W0b && !is_device_ptr(W0b)) return TTT_ERR_INVALID_ARG;

    int sticky = g_sticky.load();
    if (sticky != 0) return TTT_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return check_launch(cudaGetLastError());
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return check_launch(cudaGetLastError());

    c->Q = Q; c->K = K; c->V = V; c->Z = Z;
    c->W0 = W0; c->W0b = W0b;
    c->W1_out = nullptr; c->W1b_out = nullptr;
    c->eta = eta;
    c->batch = s->batch; c->heads = s->heads; c->H = s->H; c->W = s->W;
    c->N = s->H * s->W; c->d = s->d; c->hidden = s->hidden;
    c->hs = (s->heads > 1) ? s->head_stride : (long long)c->N * s->d;
    c->bs = (s->batch > 1) ? s->batch_stride : c->hs * s->heads;
    c->dtype = s->dtype;
    c->loss = s->loss;
    c->ws = static_cast<uint8_t*>(ws);
    c->ws_bytes = ws_bytes;
    c->stream = static_cast<cudaStream_t>(stream);
    c->num_sms = (s->max_sms > 0 && s->max_sms < sms) ? s->max_sms : sms;
    c->overlap_previous = 0;
    c->err_ws = nullptr;
    c->grid_out = nullptr;
    c->wait_ns = wait_limit_ns();
    return TTT_OK;
}

ttt_status validate_call(int kind, const void* Q, const void* K, const void* V, const float* W0, const float* W0b,
                         void* Z, float eta, const ttt_shape* s, void* ws, size_t ws_bytes, size_t need, void* stream) {
    Call c;
    return prepare(kind, Q, K, V, W0, W0b, Z, eta, s, ws, ws_bytes, need, stream, &c);
}

ttt_status prepare_linear(const void* Q, const void* K, const void* V, const float* W0, void* Z, float eta,
                          const ttt_shape* s, void* ws, size_t ws_bytes, float* W1_out, void* stream, Call* c) {
    const size_t need = (check_shape(TTT_HEAD_LINEAR, s) == TTT_OK) ? linear_ws_bytes(*s) : 0;
    ttt_status st = prepare(TTT_HEAD_LINEAR, Q, K, V, W0, nullptr, Z, eta, s, ws, ws_bytes, need, stream, c);
    if (st != TTT_OK) return st;
    if (W1_out && (reinterpret_cast<uintptr_t>(W1_out) % 16 || !is_device_ptr(W1_out))) return TTT_ERR_INVALID_ARG;
    c->W1_out = W1_out;
    return TTT_OK;
}

ttt_status read_error_word(void* ws, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return check_launch(e);
    if (word & kErrTimeout) {
        const uint32_t zero = 0;
        e = cudaMemcpyAsync(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return check_launch(e);
        return TTT_ERR_TIMEOUT;
    }
    return TTT_OK;
}

}  // namespace ttt

// ------------------------------------------------------------------------------------------------
// extern "C" entry points
// ------------------------------------------------------------------------------------------------
using namespace ttt;

extern "C" {

size_t ttt_workspace_bytes(int kind, const ttt_shape* s) {
    if (check_shape(kind, s) != TTT_OK) return 0;
    switch (kind) {
        case TTT_HEAD_LINEAR: return linear_ws_bytes(*s);
        case TTT_HEAD_DWCONV: return dwconv_ws_bytes(*s);
        case TTT_HEAD_MLP: return mlp_ws_bytes(*s);
        case TTT_HEAD_LINEAR_BACKWARD: return linear_backward_ws_bytes(*s);
        case TTT_HEAD_CONV3X3: return conv3x3_ws_bytes(*s);
        case TTT_HEAD_DWCONV_BACKWARD: return dwconv_backward_ws_bytes(*s);
        case TTT_HEAD_MLP_BACKWARD: return mlp_backward_ws_bytes(*s);
        default: return 0;
    }
}

ttt_status ttt_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < kWsHeader) return TTT_ERR_WORKSPACE;
    if (!is_device_ptr(ws)) return TTT_ERR_INVALID_ARG;
    return check_launch(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

ttt_status ttt_workspace_status(void* ws, void* stream) {
    if (!ws) return TTT_ERR_WORKSPACE;
    if (!is_device_ptr(ws)) return TTT_ERR_INVALID_ARG;
    return read_error_word(ws, stream);
}

ttt_status ttt_forward_linear(const void* Q, const void* K, const void* V, const float* W0, void* Z, float eta,
                              const ttt_shape* s, void* ws, size_t ws_bytes, float* W1_out, void* stream) {
    Call c;
    const ttt_status st = prepare_linear(Q, K, V, W0, Z, eta, s, ws, ws_bytes, W1_out, stream, &c);
    if (st != TTT_OK) return st;
    return launch_linear(c);
}

ttt_status ttt_forward_dwconv(const void* Q, const void* K, const void* V, const float* W0, void* Z, float eta,
                              const ttt_shape* s, void* ws, size_t ws_bytes, float* W1_out, void* stream) {
    Call c;
    const size_t need = (check_shape(TTT_HEAD_DWCONV, s) == TTT_OK) ? dwconv_ws_bytes(*s) : 0;
    ttt_status st = prepare(TTT_HEAD_DWCONV, Q, K, V, W0, nullptr, Z, eta, s, ws, ws_bytes, need, stream, &c);
    if (st != TTT_OK) return st;
    if (W1_out && (reinterpret_cast<uintptr_t>(W1_out) % 16 || !is_device_ptr(W1_out))) return TTT_ERR_INVALID_ARG;
    c.W1_out = W1_out;
    return launch_dwconv(c);
}

ttt_status ttt_forward_conv3x3(const void* Q, const void* K, const void* V, const float* W0, void* Z, float eta,
                               const ttt_shape* s, void* ws, size_t ws_bytes, float* W1_out, void* stream) {
    Call c;
    const size_t need = (check_shape(TTT_HEAD_CONV3X3, s) == TTT_OK) ? conv3x3_ws_bytes(*s) : 0;
    ttt_status st = prepare(TTT_HEAD_CONV3X3, Q, K, V, W0, nullptr, Z, eta, s, ws, ws_bytes, need, stream, &c);
    if (st != TTT_OK) return st;
    if (W1_out && (reinterpret_cast<uintptr_t>(W1_out) % 16 || !is_device_ptr(W1_out))) return TTT_ERR_INVALID_ARG;
    c.W1_out = W1_out;
    return launch_conv3x3(c);
}

ttt_status ttt_forward_mlp(const void* Q, const void* K, const void* V, const float* Wa, const float* Wb, void* Z,
                           float eta, const ttt_shape* s, void* ws, size_t ws_bytes, float* Wa_out, float* Wb_out,
                           void* stream) {
    Call c;
    const size_t need = (check_shape(TTT_HEAD_MLP, s) == TTT_OK) ? mlp_ws_bytes(*s) : 0;
    ttt_status st = prepare(TTT_HEAD_MLP, Q, K, V, Wa, Wb, Z, eta, s, ws, ws_bytes, need, stream, &c);
    if (st != TTT_OK) return st;
    for (float* o : {Wa_out, Wb_out})
        if (o && (reinterpret_cast<uintptr_t>(o) % 16 || !is_device_ptr(o))) return TTT_ERR_INVALID_ARG;
    c.W1_out = Wa_out;
    c.W1b_out = Wb_out;
    return launch_mlp(c);
}

ttt_status ttt_forward_linear_minibatch(const void* Q, const void* K, const void* V, const float* W0, void* Z,
                                        float eta, const ttt_shape* s, int batch_tokens, int mode, void* ws,
                                        size_t ws_bytes, float* W1_out, void* stream) {
    ttt_status st = check_shape(TTT_HEAD_LINEAR, s);
    if (st != TTT_OK) return st;
    if (batch_tokens < 1 || (mode != TTT_MB_PREFIX && mode != TTT_MB_EPOCH)) return TTT_ERR_INVALID_ARG;
    if (s->loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    Call c;
    st = prepare(TTT_HEAD_LINEAR, Q, K, V, W0, nullptr, Z, eta, s, ws, ws_bytes, kWsHeader, stream, &c);
    if (st != TTT_OK) return st;
    if (W1_out && (reinterpret_cast<uintptr_t>(W1_out) % 16 || !is_device_ptr(W1_out))) return TTT_ERR_INVALID_ARG;
    c.W1_out = W1_out;
    return launch_linear_minibatch(c, batch_tokens, mode);
}

static ttt_status backward_common(int kind, const void* Q, const void* K, const void* V, const float* W0,
                                  const float* W0b, const void* dZ, float eta, const ttt_shape* s, void* ws,
                                  size_t ws_bytes, void* dQ, void* dK, void* dV, float* dW0_out, float* dW0b_out,
                                  float* deta_out, void* stream) {
    ttt_status st = check_shape(kind, s);
    if (st != TTT_OK) return st;
    if (s->loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    if (!dZ || !dK || !dV) return TTT_ERR_INVALID_ARG;
    Call c;
    const size_t need = (kind == TTT_HEAD_LINEAR_BACKWARD) ? linear_backward_ws_bytes(*s)
                        : (kind == TTT_HEAD_DWCONV_BACKWARD) ? dwconv_backward_ws_bytes(*s)
                                                             : mlp_backward_ws_bytes(*s);
    // Q, K, V, the weights, the workspace and dQ (as the output Z: apart from Q, K and V)
    st = prepare(kind, Q, K, V, W0, W0b, dQ, eta, s, ws, ws_bytes, need, stream, &c);
    if (st != TTT_OK) return st;
    for (const void* p : {dZ, (const void*)dK, (const void*)dV}) {
        if (reinterpret_cast<uintptr_t>(p) % 16) return TTT_ERR_ALIGNMENT;
        if (!is_device_ptr(p)) return TTT_ERR_INVALID_ARG;
    }
    const long long ext = extent_bytes(s);
    const void* ins[] = {Q, K, V, dZ};
    const void* outs[] = {dQ, dK, dV};
    for (const void* o : outs)
        for (const void* in : ins)
            if (overlaps(o, in, ext)) return TTT_ERR_INVALID_ARG;
    if (overlaps(dQ, dK, ext) || overlaps(dQ, dV, ext) || overlaps(dK, dV, ext)) return TTT_ERR_INVALID_ARG;
    for (float* o : {dW0_out, dW0b_out})
        if (o && (reinterpret_cast<uintptr_t>(o) % 16 || !is_device_ptr(o))) return TTT_ERR_INVALID_ARG;
    if (deta_out && (reinterpret_cast<uintptr_t>(deta_out) % 4 || !is_device_ptr(deta_out))) return TTT_ERR_INVALID_ARG;
    if (kind == TTT_HEAD_LINEAR_BACKWARD) return launch_linear_backward(c, dZ, dQ, dK, dV, dW0_out, deta_out);
    if (kind == TTT_HEAD_DWCONV_BACKWARD) return launch_dwconv_backward(c, dZ, dQ, dK, dV, dW0_out, deta_out);
    return launch_mlp_backward(c, *s, dZ, dQ, dK, dV, dW0_out, dW0b_out, deta_out);
}

ttt_status ttt_backward_linear(const void* Q, const void* K, const void* V, const float* W0, const void* dZ,
                               float eta, const ttt_shape* s, void* ws, size_t ws_bytes, void* dQ, void* dK,
                               void* dV, float* dW0_out, float* deta_out, void* stream) {
    return backward_common(TTT_HEAD_LINEAR_BACKWARD, Q, K, V, W0, nullptr, dZ, eta, s, ws, ws_bytes, dQ, dK, dV,
                           dW0_out, nullptr, deta_out, stream);
}

ttt_status ttt_backward_dwconv(const void* Q, const void* K, const void* V, const float* W0, const void* dZ,
                               float eta, const ttt_shape* s, void* ws, size_t ws_bytes, void* dQ, void* dK,
                               void* dV, float* dW0_out, float* deta_out, void* stream) {
    return backward_common(TTT_HEAD_DWCONV_BACKWARD, Q, K, V, W0, nullptr, dZ, eta, s, ws, ws_bytes, dQ, dK, dV,
                           dW0_out, nullptr, deta_out, stream);
}

ttt_status ttt_backward_mlp(const void* Q, const void* K, const void* V, const float* Wa, const float* Wb,
                            const void* dZ, float eta, const ttt_shape* s, void* ws, size_t ws_bytes, void* dQ,
                            void* dK, void* dV, float* dWa_out, float* dWb_out, float* deta_out, void* stream) {
    return backward_common(TTT_HEAD_MLP_BACKWARD, Q, K, V, Wa, Wb, dZ, eta, s, ws, ws_bytes, dQ, dK, dV, dWa_out,
                           dWb_out, deta_out, stream);
}

constexpr double kConvHeadWeight = 2.0;

// The layer call works on two head ranges of one [B][heads][N][d] view: heads [0, nl) linear, heads
// [nl, heads) depthwise conv.  Its workspace is the linear workspace followed by the conv workspace.
static void layer_shapes(const ttt_shape* s, int conv_heads, ttt_shape* lin, ttt_shape* conv) {
    *lin = *s;
    *conv = *s;
    lin->heads = s->heads - conv_heads;
    conv->heads = conv_heads;
}

static size_t layer_lin_ws(const ttt_shape& lin) {
    return lin.heads > 0 ? align_up(linear_ws_bytes(lin), 256) : 0;
}

size_t ttt_layer_workspace_bytes(const ttt_shape* s, int conv_heads) {
    if (check_shape(TTT_HEAD_LINEAR, s) != TTT_OK || conv_heads < 0 || conv_heads > s->heads) return 0;
    ttt_shape lin, conv;
    layer_shapes(s, conv_heads, &lin, &conv);
    return layer_lin_ws(lin) + (conv.heads > 0 ? dwconv_ws_bytes(conv) : 0);
}

ttt_status ttt_forward_layer(const void* Q, const void* K, const void* V, const float* W0_lin, const float* W0_conv,
                             void* Z, float eta, const ttt_shape* s, int conv_heads, void* ws, size_t ws_bytes,
                             float* W1_lin_out, float* W1_conv_out, void* stream) {
    ttt_status st = check_shape(TTT_HEAD_LINEAR, s);
    if (st != TTT_OK) return st;
    if (conv_heads < 0 || conv_heads > s->heads) return TTT_ERR_INVALID_ARG;
    ttt_shape lin, conv;
    layer_shapes(s, conv_heads, &lin, &conv);
    const size_t lin_ws = layer_lin_ws(lin);
    const size_t need = ttt_layer_workspace_bytes(s, conv_heads);
    // the whole view first (pointers, alignment, Z apart from Q/K/V over all heads), then each range
    Call whole;
    st = prepare(TTT_HEAD_LINEAR, Q, K, V, lin.heads ? W0_lin : W0_conv, nullptr, Z, eta, s, ws, ws_bytes, need,
                 stream, &whole);
    if (st != TTT_OK) return st;
    for (float* o : {W1_lin_out, W1_conv_out})
        if (o && (reinterpret_cast<uintptr_t>(o) % 16 || !is_device_ptr(o))) return TTT_ERR_INVALID_ARG;
    Call cl, cc;
    const long long esz = (s->dtype == TTT_BF16) ? 2 : 4;
    const long long off = (long long)lin.heads * whole.hs * esz;    // bytes from head 0 to head nl
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    if (lin.heads) {
        st = prepare(TTT_HEAD_LINEAR, Q, K, V, W0_lin, nullptr, Z, eta, &lin, w8, lin_ws, linear_ws_bytes(lin),
                     stream, &cl);
        if (st != TTT_OK) return st;
        cl.W1_out = W1_lin_out;
    }
    if (conv.heads) {
        auto shift = [&](const void* p) { return static_cast<const void*>(static_cast<const uint8_t*>(p) + off); };
        st = prepare(TTT_HEAD_DWCONV, shift(Q), shift(K), shift(V), W0_conv, nullptr,
                     const_cast<void*>(shift(Z)), eta, &conv, w8 + lin_ws, ws_bytes - lin_ws, dwconv_ws_bytes(conv),
                     stream, &cc);
        if (st != TTT_OK) return st;
        cc.W1_out = W1_conv_out;
        cc.err_ws = w8;                                              // one error word for the layer
        // the conv kernel queues behind the linear kernel and takes the SMs it leaves free; as its
        // CTAs finish, the rest of the conv grid takes over the SMs the linear kernel releases
        cc.overlap_previous = lin.heads ? 1 : 0;
    }
    if (lin.heads && conv.heads) {
        // The linear kernel gets a share of the SMs in proportion to its heads' work, counting a conv
        // head as kConvHeadWeight linear heads (a conv head's FMA work per token is about that much
        // more SM time than a linear head's tensor-core streaming); the conv kernel takes the rest.
        const double wl = (double)lin.heads, wc = kConvHeadWeight * conv.heads;
        cl.num_sms = std::max(1, (int)((double)whole.num_sms * wl / (wl + wc)));
    }
    int lin_grid = 0;
    cl.grid_out = &lin_grid;
    if (lin.heads && (st = launch_linear(cl)) != TTT_OK) return st;
    // The conv kernel is queued behind the linear kernel as a programmatic dependent and sized for
    // the SMs the linear grid leaves free; with none left, it takes the whole device and its CTAs
    // start as the linear CTAs finish.
    if (conv.heads && lin.heads && lin_grid > 0 && lin_grid < whole.num_sms) cc.num_sms = whole.num_sms - lin_grid;
    if (conv.heads) st = launch_dwconv(cc);
    return st;
}

const char* ttt_status_string(ttt_status st) {
    switch (st) {
        case TTT_OK: return "TTT_OK";
        case TTT_ERR_INVALID_ARG: return "TTT_ERR_INVALID_ARG";
        case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED";
        case TTT_ERR_ALIGNMENT: return "TTT_ERR_ALIGNMENT";
        case TTT_ERR_WORKSPACE: return "TTT_ERR_WORKSPACE";
        case TTT_ERR_CUDA: return "TTT_ERR_CUDA";
        case TTT_ERR_TIMEOUT: return "TTT_ERR_TIMEOUT";
    }
    return "TTT_ERR_UNKNOWN";
}

ttt_status ttt_last_error(void) { return g_sticky.load() ? TTT_ERR_CUDA : TTT_OK; }

ttt_status ttt_set_wait_limit(unsigned long long limit_ns) {
    if (limit_ns == 0 || limit_ns > 1000000000ull) return TTT_ERR_INVALID_ARG;
    g_wait_ns.store(limit_ns);
    return TTT_OK;
}

int ttt_version(void) { return 200; }

}  // extern "C"
