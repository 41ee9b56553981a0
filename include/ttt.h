/*
 * ttt.h -- C ABI of libttt.so: the forward pass of the ViT^3 test-time-training (TTT) token-mixing
 * layer on NVIDIA B200 (sm_100a).
 *
 * The operation (one "unit" = one image b and one head h; N = H*W tokens of width d):
 *   The unit's key/value pairs are a small training set.  An inner model f(.;W) takes ONE
 *   full-batch, non-causal gradient step of the L2 reconstruction loss over all N pairs,
 *       L(W)  = (1/N) sum_n || f(k_n; W) - v_n ||^2,        W1 = W0 - eta * dL/dW (W0),
 *   and every query is read out through the updated model:  z_n = f(q_n; W1).
 *   The shape's `loss` field selects the dot-product inner loss instead (see ttt_loss).
 *   Sources, by page title and section:
 *     "CVPR 2026 Oral | 清華+阿里發布ViT3" (press article): section 序列建模的新視角 (keys and values
 *       as a dataset, reconstruction by gradient descent, readout on the queries); Observation 2,
 *       Fig. 3 (one full-batch step, B = N); Observations 4 and 6, Fig. 5 (MLP and depthwise-conv
 *       inner models).
 *     "Vision-TTT: Efficient and Expressive Visual Representation Learning with Test-Time
 *       Training" (paper notes): section 关键设计 1 (L2 loss ||W x_K - x_V||^2, gradient
 *       2 (W x_K - x_V) x_K^T, readout z = W x_Q, one d x d state per head).
 *   The gradient is the mean over the N pairs (factor 2/N); the pages print a per-token gradient
 *   and leave the batch normalisation open.
 *
 * Data layout (all entry points):
 *   Q, K, V, Z   element (b, h, n, c) at  b*batch_stride + h*head_stride + n*d + c   (elements of
 *                the call's dtype); token n sits at grid position (n / W, n % W).  Rows of d
 *                features are contiguous; batch_stride and head_stride let one call work on a
 *                sub-range of heads of a larger [B][heads_total][N][d] buffer.
 *   Weights are fp32, contiguous, one set per head shared by every image of the batch.
 *
 * Conventions:
 *   - Device pointers only (Q, K, V, weights, Z, workspace, optional outputs); host pointers are
 *     rejected with TTT_ERR_INVALID_ARG.  The caller owns every buffer; the library never
 *     allocates, frees or synchronises.  All work is queued on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream) and the call returns before it completes.
 *   - Inputs are read-only.  Z must not overlap Q, K or V.
 *   - Validation is synchronous: on any error nothing is launched.  Errors raised while the
 *     kernels run are sticky CUDA errors (reported by the next call, or by ttt_last_error), or a
 *     device-side wait that ran out (reported by ttt_workspace_status).
 *   - d must be 64.  Q, K, V, Z must be 16-byte aligned and batch_stride, head_stride multiples of
 *     8 (bf16) or 4 (fp32) elements.
 *   - The workspace (size from ttt_workspace_bytes) must be zero-filled once after allocation
 *     (ttt_workspace_init); every successful call leaves it ready for the next one.  Calls that
 *     may run at the same time need distinct workspaces.
 *   - Results are deterministic: the same inputs on the same device give bitwise-equal outputs.
 *   - Arithmetic: bf16 inputs are multiplied exactly and accumulated in fp32; the updated weights
 *     are formed in fp32 and rounded once to bf16 for the readout; Z is rounded to the input dtype.
 *     fp32 inputs are computed in fp32 throughout.
 */
#ifndef TTT_H
#define TTT_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TTT_OK = 0,
    TTT_ERR_INVALID_ARG = 1,   /* null/host pointer, bad size, overlap, non-finite eta */
    TTT_ERR_UNSUPPORTED = 2,   /* a valid request this build does not implement (e.g. d != 64) */
    TTT_ERR_ALIGNMENT = 3,     /* pointer or stride alignment rule broken */
    TTT_ERR_WORKSPACE = 4,     /* workspace missing or smaller than ttt_workspace_bytes() */
    TTT_ERR_CUDA = 5,          /* a CUDA runtime error (launch failure or a sticky earlier error) */
    TTT_ERR_TIMEOUT = 6        /* a device-side wait gave up (see ttt_workspace_status) */
} ttt_status;

typedef enum { TTT_FP32 = 0, TTT_BF16 = 1 } ttt_dtype;

typedef enum {
    TTT_HEAD_LINEAR = 0,
    TTT_HEAD_DWCONV = 1,
    TTT_HEAD_MLP = 2,
    TTT_HEAD_LINEAR_BACKWARD = 3,  /* the workspace of ttt_backward_linear */
    TTT_HEAD_CONV3X3 = 4,          /* the workspace of ttt_forward_conv3x3 */
    TTT_HEAD_DWCONV_BACKWARD = 5,  /* the workspace of ttt_backward_dwconv */
    TTT_HEAD_MLP_BACKWARD = 6      /* the workspace of ttt_backward_mlp */
} ttt_head_kind;

/* Inner loss of the one-step training.
 *   TTT_LOSS_L2:  L(W) = (1/N) sum_n || f(k_n; W) - v_n ||^2  (the formulas of each entry point below).
 *   TTT_LOSS_DOT: L(W) = -(1/N) sum_n < f(k_n; W), v_n >, the dot-product loss of the ViT^3 recipe
 *     (press article, section ViT3：視覺測試時訓練模型: one full-batch step, learning rate 1.0,
 *     dot-product loss; the pages do not print the loss, this is its plain reading).  Its gradient
 *     has no residual and does not depend on W0:
 *       linear:  W1 = W0 + eta (1/N) sum_n v_n k_n^T   (= W0 + eta C / N; the Gram term drops out)
 *       conv:    W1[c][a][b] = W0[c][a][b] + eta (1/N) sum_{y,x} V[c,y,x] K[c,y+a-1,x+b-1]
 *     The MLP head does not implement it (TTT_ERR_UNSUPPORTED). */
typedef enum { TTT_LOSS_L2 = 0, TTT_LOSS_DOT = 1 } ttt_loss;

typedef struct {
    int batch;               /* images B >= 1 */
    int heads;               /* heads handled by this call >= 1 */
    int H, W;                /* token grid; N = H*W >= 1 */
    int d;                   /* head width; must be 64 */
    int hidden;              /* MLP hidden width (multiple of 64, <= 256); ignored by other heads */
    long long batch_stride;  /* elements between consecutive images in Q, K, V, Z */
    long long head_stride;   /* elements between consecutive heads in Q, K, V, Z */
    int dtype;               /* ttt_dtype of Q, K, V and Z */
    int max_sms;             /* SMs the call may spread its work over; 0 = the whole device.  Two calls
                                that run at the same time on two streams (e.g. the linear heads and the
                                conv heads of one layer) each take a share, so that neither waits for
                                SMs the other holds.  It may change how sums are split over CTAs, hence
                                the rounding; results are bitwise reproducible for a fixed value. */
    int loss;                /* ttt_loss of the inner training step (0 = TTT_LOSS_L2) */
} ttt_shape;

/* Bytes of device workspace that a call of head kind `kind` with shape `s` needs (0 on an invalid
 * shape).  Depends only on the shape, not on the device. */
size_t ttt_workspace_bytes(int kind, const ttt_shape* s);

/* Zero-fill a workspace on `stream` (call once after allocating it). */
ttt_status ttt_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reports whether a kernel that used `ws` gave up a bounded device-side
 * wait (TTT_ERR_TIMEOUT, and the flag is cleared) or finished normally (TTT_OK). */
ttt_status ttt_workspace_status(void* ws, void* stream);

/* Linear inner model f(x) = W x, W in R^{d x d}.
 *   Computes per unit  G = sum_n k_n k_n^T,  C = sum_n v_n k_n^T   (fp32),
 *   W1 = W0 - eta * (2/N) * (W0 G - C)   and   z_n = W1 q_n
 *   (TTT_LOSS_DOT: W1 = W0 + eta * (1/N) * C; G is not used).
 *   W0:     [heads][d][d] fp32 (W0[i][j] maps input feature j to output feature i).
 *   W1_out: optional (NULL = not written) [batch][heads][d][d] fp32, the updated weights.
 */
ttt_status ttt_forward_linear(const void* Q, const void* K, const void* V, const float* W0,
                              void* Z, float eta, const ttt_shape* s, void* ws, size_t ws_bytes,
                              float* W1_out, void* stream);

/* 3x3 depthwise-convolution inner model over the H x W grid (press article, Observation 6 and
 * Fig. 5 part 3; one head of ViT^3 uses it): cross-correlation, zero padding, stride 1, no bias,
 * one kernel per feature channel c:
 *   f(X;W)[c,y,x] = sum_{a,b=0..2} W[c][a][b] X[c, y+a-1, x+b-1].
 *   r = f(K;W0) - V;  g[c][a][b] = (2/N) sum_{y,x} r[c,y,x] K[c,y+a-1,x+b-1];  W1 = W0 - eta g;
 *   Z = f(Q;W1).   (TTT_LOSS_DOT: g[c][a][b] = -(1/N) sum_{y,x} V[c,y,x] K[c,y+a-1,x+b-1].)
 *   W0:     [heads][d][3][3] fp32.   W1_out: optional [batch][heads][d][3][3] fp32.
 *   The workspace holds per-(image, head) partial sums and counters (about 25 KB per unit at 78 x 78
 *   tokens); after a TTT_ERR_TIMEOUT it must be zero-filled again (ttt_workspace_init).
 */
ttt_status ttt_forward_dwconv(const void* Q, const void* K, const void* V, const float* W0,
                              void* Z, float eta, const ttt_shape* s, void* ws, size_t ws_bytes,
                              float* W1_out, void* stream);

/* Full 3x3 convolution inner model over the H x W grid (press article, Observation 6 and Fig. 5
 * part 3: the inner model implemented as a 3x3 convolution, beside the depthwise variant above):
 * cross-correlation, zero padding, stride 1, no bias, every output channel reading every input one:
 *   f(X;W)[c,y,x] = sum_{c'} sum_{a,b=0..2} W[c][c'][a][b] X[c', y+a-1, x+b-1].
 *   r = f(K;W0) - V;  g[c][c'][a][b] = (2/N) sum_{y,x} r[c,y,x] K[c', y+a-1, x+b-1];  W1 = W0 - eta g;
 *   Z = f(Q;W1).
 *   W0: [heads][d][d][3][3] fp32.  W1_out: optional [batch][heads][d][d][3][3] fp32.
 *   The three contractions (576 input features per position) run on the tensor cores with bf16
 *   operands and fp32 accumulation: W0 is rounded to bf16 for the residual, the residual is carried
 *   as two bf16 parts (about 16 significant bits), W1 is rounded once to bf16 for the readout.
 *   bf16 and TTT_LOSS_L2 only (fp32 or TTT_LOSS_DOT returns TTT_ERR_UNSUPPORTED).
 *   ws: ttt_workspace_bytes(TTT_HEAD_CONV3X3, s) bytes (per-CTA partial gradients of 144 KB each, and
 *   W0 and the updated weights as bf16 operand images); it needs no zero fill, every call writes what
 *   it reads.
 *   Work is split over CTAs in fixed ranges: results are bitwise reproducible for a fixed SM budget.
 */
ttt_status ttt_forward_conv3x3(const void* Q, const void* K, const void* V, const float* W0,
                               void* Z, float eta, const ttt_shape* s, void* ws, size_t ws_bytes,
                               float* W1_out, void* stream);

/* One-hidden-layer MLP inner model f(x) = Wb gelu_tanh(Wa x) (press article, Observation 4 and
 * Fig. 5 part 1: width ratio up to 4), gelu_tanh(u) = u/2 (1 + tanh(sqrt(2/pi)(u + 0.044715 u^3))).
 * Both matrices take one simultaneous step from the gradients at (Wa, Wb):
 *   h = Wa k, a = gelu(h), r = Wb a - v,
 *   Wb1 = Wb - eta (2/N) sum r a^T,   Wa1 = Wa - eta (2/N) sum [(Wb^T r) * gelu'(h)] k^T,
 *   z = Wb1 gelu(Wa1 q).
 *   Wa: [heads][hidden][d] fp32,  Wb: [heads][d][hidden] fp32.
 *   Wa_out / Wb_out: optional [batch][heads][hidden][d] / [batch][heads][d][hidden] fp32.
 *   bf16 and TTT_LOSS_L2 only (fp32 or TTT_LOSS_DOT returns TTT_ERR_UNSUPPORTED).
 */
ttt_status ttt_forward_mlp(const void* Q, const void* K, const void* V, const float* Wa,
                           const float* Wb, void* Z, float eta, const ttt_shape* s, void* ws,
                           size_t ws_bytes, float* Wa_out, float* Wb_out, void* stream);

/* Linear-head forward without a caller workspace.  The pages have no counterpart of this entry
 * point: it exists for callers that cannot allocate device memory themselves -- for example a plugin
 * inside a host framework that hands it only its input and output buffers and owns the allocator,
 * or code that runs under a fixed, pre-reserved memory budget and must not call cudaMalloc at run
 * time (cudaMalloc may synchronise the device and has no bounded latency).
 *   Same arguments, computation, results and validation errors as ttt_forward_linear, minus
 *   (ws, ws_bytes).
 *   Scratch: an 8 MiB array that the library holds on every device that loads it, until the process
 *   exits.  Shapes whose ttt_workspace_bytes(TTT_HEAD_LINEAR, s) exceeds 8 MiB are rejected with
 *   TTT_ERR_WORKSPACE (bf16 calls need only the 256-byte error word; fp32 calls need about
 *   5 MiB + 48 KiB per (image, head) unit, so fp32 calls above about 60 units are rejected).
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
 *   device current, and looks it up again when the device's context has changed (after a
 *   cudaDeviceReset); make that first call before any stream capture begins.
 *   Every call on a device shares that device's one array, which keeps the previous call's contents;
 *   each call clears the control words that must start at zero (a cudaMemsetAsync on `stream`)
 *   before its kernels run, and keeps the error word.  Calls whose work may overlap on the same GPU
 *   (other streams, other host threads) race on the array and must be serialised by the caller.
 *   A device-side wait that runs out is reported by ttt_noalloc_status (below), not by the call.
 *   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 */
ttt_status ttt_forward_linear_noalloc(const void* Q, const void* K, const void* V, const float* W0, void* Z,
                                      float eta, const ttt_shape* s, float* W1_out, void* stream);

/* The error word of the current device's ttt_forward_linear_noalloc scratch (no counterpart on the
 * pages either): synchronises `stream`, then reports TTT_ERR_TIMEOUT (and clears it) if a kernel of
 * an earlier noalloc call on this device gave up a bounded device-side wait -- its Z and W1_out are
 * then incomplete -- else TTT_OK.  Allocates nothing. */
ttt_status ttt_noalloc_status(void* stream);

/* Mini-batch variants of the linear head's inner training (mode: ttt_minibatch_mode).
 * The raster-ordered tokens are cut into consecutive mini-batches of batch_tokens tokens (the last
 * may be shorter); in every mini-batch the per-token gradients are taken at the weights W_s the
 * mini-batch starts from, G_t = 2 (W_s k_t - v_t) k_t^T.
 *   TTT_MB_PREFIX ("Vision-TTT" paper notes, section 关键设计 4, b = 16 there): inside a mini-batch
 *     W_t = W_s - eta * sum_{s <= t} G_s (a causal prefix sum, no 1/b) and z_t = W_t q_t; the next
 *     mini-batch starts from the last W_t.  batch_tokens = 1 is per-token sequential TTT.
 *   TTT_MB_EPOCH (press article, Observation 2 and Fig. 3: the dataset cut into 2, 3 or 4
 *     consecutive mini-batches, one update each): W <- W_s - eta * (2/|batch|) sum (W_s k_t - v_t) k_t^T
 *     per mini-batch, then z_n = W_final q_n for every token.  batch_tokens >= N gives the results of
 *     ttt_forward_linear up to rounding.
 * Computed in fp32 from bf16 or fp32 inputs (Z rounded to the input dtype).
 *   ws: a workspace of at least 256 bytes, zero-filled once (ttt_workspace_init); its error word
 *   reports a device-side wait that ran out (ttt_workspace_status).
 *   W0: [heads][d][d] fp32.  W1_out: optional [batch][heads][d][d] fp32, the weights after the last
 *   mini-batch.  s->loss must be TTT_LOSS_L2 (else TTT_ERR_UNSUPPORTED); s->max_sms bounds the SMs.
 * Errors: TTT_ERR_INVALID_ARG for batch_tokens < 1 or an unknown mode, and as ttt_forward_linear. */
typedef enum { TTT_MB_PREFIX = 0, TTT_MB_EPOCH = 1 } ttt_minibatch_mode;
ttt_status ttt_forward_linear_minibatch(const void* Q, const void* K, const void* V, const float* W0,
                                        void* Z, float eta, const ttt_shape* s, int batch_tokens, int mode,
                                        void* ws, size_t ws_bytes, float* W1_out, void* stream);

/* Backward pass of the full-batch linear head (L2 loss): the outer gradient through the inner update
 * that trains the layer end to end (press article, Observation 1).  With s = 2 eta / N and the
 * forward of ttt_forward_linear, for the upstream gradient dZ of Z:
 *   dW1 = sum dz q^T,  dq = W1^T dz,  dC = s dW1,  dG = -s W0^T dW1,
 *   dv = dC k,  dk = dC^T v + (dG + dG^T) k,  dW0 = dW1 (I - s G),
 *   deta = -(2/N) sum_ij dW1_ij (W0 G - C)_ij.
 *   dZ: same layout and dtype as Q.  dQ, dK, dV: outputs, same layout and dtype as Q; they may not
 *   overlap Q, K, V, dZ or one another.
 *   dW0_out: optional [heads][d][d] fp32, summed over the images of each head in image order.
 *   deta_out: optional, one fp32, summed over every (image, head) unit in index order.
 *   ws: ttt_workspace_bytes(TTT_HEAD_LINEAR_BACKWARD, s) bytes, zero-filled once
 *   (ttt_workspace_init); it holds per-unit partial sums and matrices.
 * fp32 inputs: computed in fp32 throughout.  bf16 inputs (tensor cores): the token sums G, C, dW1 are
 * exact products accumulated in fp32, the unit matrices are formed in fp32, and the per-token maps
 * multiply by them split into two bf16 parts (about 16 significant bits).  Outputs are rounded to the
 * input dtype; deterministic.  s->loss must be TTT_LOSS_L2 (else TTT_ERR_UNSUPPORTED). */
ttt_status ttt_backward_linear(const void* Q, const void* K, const void* V, const float* W0, const void* dZ,
                               float eta, const ttt_shape* s, void* ws, size_t ws_bytes, void* dQ, void* dK,
                               void* dV, float* dW0_out, float* deta_out, void* stream);

/* Backward pass of the 3x3 depthwise-conv head (L2 loss; the head of ttt_forward_dwconv), the outer
 * gradient through its inner step (press article, Observation 1).  Per channel c, taps t with shifts
 * s_t = (a-1, b-1), dg = -eta dW1, and positions q - s_t outside the grid contributing nothing:
 *   dW1_t = sum_p dZ_p Q_{p+s_t},          dQ_q = sum_t W1_t dZ_{q-s_t},
 *   dr_p = (2/N) sum_t dg_t K_{p+s_t},     dV_p = -dr_p,
 *   dK_q = (2/N) sum_t dg_t r_{q-s_t} + sum_t W0_t dr_{q-s_t}   (r = f(K;W0) - V),
 *   dW0_t = dW1_t + sum_p dr_p K_{p+s_t},  deta = -sum_t dW1_t g_t.
 *   Layouts, outputs and rules as ttt_backward_linear: dQ, dK, dV like Q; dW0_out optional
 *   [heads][d][3][3] fp32 summed over the images of each head in image order; deta_out optional, summed
 *   over every unit in index order.  ws: ttt_workspace_bytes(TTT_HEAD_DWCONV_BACKWARD, s) bytes (per-tile
 *   partial sums and per-unit coefficients; needs no zero fill).  fp32 arithmetic from bf16 or fp32
 *   inputs; deterministic.  s->loss must be TTT_LOSS_L2 (else TTT_ERR_UNSUPPORTED). */
ttt_status ttt_backward_dwconv(const void* Q, const void* K, const void* V, const float* W0, const void* dZ,
                               float eta, const ttt_shape* s, void* ws, size_t ws_bytes, void* dQ, void* dK,
                               void* dV, float* dW0_out, float* deta_out, void* stream);

/* Backward pass of the MLP head (L2 loss; the head of ttt_forward_mlp), the outer gradient through its
 * inner step (press article, Observation 1).  With s = 2/N, per key token h = Wa k, a = gelu(h),
 * D = gelu'(h), r = Wb a - v, b = Wb^T r, e = b * D, the step gWb = s sum r a^T, gWa = s sum e k^T,
 * Wa1 = Wa - eta gWa, Wb1 = Wb - eta gWb, and per query token hq = Wa1 q, aq = gelu(hq):
 *   readout: dWb1 = sum dz aq^T, dhq = (Wb1^T dz) * gelu'(hq), dq = Wa1^T dhq, dWa1 = sum dhq q^T;
 *   update:  dgWa = -eta dWa1, dgWb = -eta dWb1, and per key token de = s dgWa k, db = de * D,
 *            dD = de * b, dr = s dgWb a + Wb db, da = s dgWb^T r + Wb^T dr, dh = da * D + dD * gelu''(h),
 *            dk = s dgWa^T e + Wa^T dh, dv = -dr, dWa += dh k^T, dWb += dr a^T + r db^T;
 *   dWa_out = sum over images of (dWa1 + dWa), dWb_out likewise, deta = -sum dWa1 * gWa - sum dWb1 * gWb
 *   summed over every unit.
 *   Wa: [heads][hidden][d], Wb: [heads][d][hidden] fp32; dWa_out / dWb_out optional, same shapes.
 *   dQ, dK, dV like Q.  hidden a multiple of 64 up to 256; bf16 or fp32 inputs, fp32 arithmetic;
 *   ws: ttt_workspace_bytes(TTT_HEAD_MLP_BACKWARD, s) bytes (needs no zero fill); deterministic.
 *   s->loss must be TTT_LOSS_L2 (else TTT_ERR_UNSUPPORTED). */
ttt_status ttt_backward_mlp(const void* Q, const void* K, const void* V, const float* Wa, const float* Wb,
                            const void* dZ, float eta, const ttt_shape* s, void* ws, size_t ws_bytes, void* dQ,
                            void* dK, void* dV, float* dWa_out, float* dWb_out, float* deta_out, void* stream);

/* A layer whose heads [0, heads - conv_heads) are linear heads and whose last conv_heads heads are
 * depthwise-conv heads (ViT^3 keeps one conv head among its linear heads: press article,
 * Observation 6), over one [batch][heads][N][d] view described by s (s->heads = all heads):
 * ttt_forward_linear on the first range and ttt_forward_dwconv on the second, with the same results.
 * Both kernels run at the same time: the linear kernel is given a share of the SMs in proportion to
 * its heads' work (a conv head counting as two linear heads); the conv kernel is queued behind it as
 * a programmatic dependent, starts as soon as every linear CTA is resident and runs on the SMs the
 * linear kernel leaves free (its work split for that many CTAs).  The call is complete on `stream`
 * when both kernels are.  Results equal those of the two separate calls given the same SM budgets
 * (linear: its share; conv: the SMs left to it).  s->loss applies to both ranges.
 *   W0_lin: [heads - conv_heads][d][d], W0_conv: [conv_heads][d][3][3] (each may be NULL when its
 *   range is empty).  W1_lin_out / W1_conv_out: optional, as in the two calls above.
 *   ws: ttt_layer_workspace_bytes(s, conv_heads) bytes, zero-filled once (ttt_workspace_init); its
 *   error word is the one ttt_workspace_status reads.
 */
size_t ttt_layer_workspace_bytes(const ttt_shape* s, int conv_heads);
ttt_status ttt_forward_layer(const void* Q, const void* K, const void* V, const float* W0_lin,
                             const float* W0_conv, void* Z, float eta, const ttt_shape* s, int conv_heads,
                             void* ws, size_t ws_bytes, float* W1_lin_out, float* W1_conv_out, void* stream);

/* Self-test of the failure-detection path (no fault is involved): launches one kernel on `stream`
 * that waits, for at most limit_ns nanoseconds (1 .. 1e9), on a word of the workspace header that
 * nothing sets, and then takes the steps every bounded wait of the layer kernels takes when it runs
 * out: it records TTT_ERR_TIMEOUT in the workspace error word and returns.  ttt_workspace_status(ws)
 * then reports TTT_ERR_TIMEOUT (and clears it).  ws: any workspace of at least 256 bytes that is
 * zero-filled (ttt_workspace_init); it must not be in use by another call.  ws = NULL: the
 * library-owned array of ttt_forward_linear_noalloc on the current device (ws_bytes is ignored), whose
 * timeout ttt_noalloc_status then reports.
 * Errors: TTT_ERR_WORKSPACE (ws too small), TTT_ERR_ALIGNMENT, TTT_ERR_INVALID_ARG. */
ttt_status ttt_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned long long limit_ns, void* stream);

/* Bound, in nanoseconds (1 .. 1e9; 1e9 at load), of every device-side wait of the kernels launched
 * by later calls in this process (a wait on a tile, on a partner warp or on another CTA's result).
 * A wait that runs out records TTT_ERR_TIMEOUT in the call's workspace error word and the kernel
 * returns; no fault is involved.  Shortening it is meant for tests of that failure path.  Returns
 * TTT_ERR_INVALID_ARG outside the range. */
ttt_status ttt_set_wait_limit(unsigned long long limit_ns);

/* Human-readable name of a status code (static string). */
const char* ttt_status_string(ttt_status st);

/* The first asynchronous CUDA error seen by the library in this process, if any (TTT_ERR_CUDA), else
 * TTT_OK.  Does not synchronise. */
ttt_status ttt_last_error(void);

/* ABI version (major*100 + minor). */
int ttt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H */
