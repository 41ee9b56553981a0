/*
 * ttt_oracle.c -- plain fp64 CPU oracle for the ViT^3 test-time-training (TTT) layer: its forward
 * pass, the variants of its inner training, and the backward pass of its linear head.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this file or the
 * library built from it.  Only the test suite, the package smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (one "unit" = one image b and one head h; N = H*W tokens of width d):
 *   The token sequence is treated as a small dataset of (key -> value) pairs.  An inner model f(.;W)
 *   is trained on it by ONE full-batch, non-causal gradient step of the L2 reconstruction loss
 *       L(W) = (1/N) * sum_n || f(k_n; W) - v_n ||^2
 *   and the updated model is then applied to every query:  z_n = f(q_n; W1),  W1 = W0 - eta*dL/dW(W0).
 *   Sources (pages on ViT^3 / vision TTT, cited by title and section):
 *     - "CVPR 2026 Oral | 清華+阿里發布ViT3" (press article), section 序列建模的新視角: keys and
 *       values form a dataset, the inner model learns to reconstruct v from k by gradient descent
 *       with e.g. an L2 loss, and the trained model is then applied to the queries.
 *     - same article, Observation 2 and Fig. 3: one full-batch (B = N) step over all pairs, with no
 *       ordering between tokens.
 *     - "Vision-TTT: Efficient and Expressive Visual Representation Learning with Test-Time
 *       Training" (paper notes), section 关键设计 1: the L2 loss ||W x_K - x_V||^2, its gradient
 *       2 (W x_K - x_V) x_K^T and the readout z = W x_Q, one d x d matrix per head.
 *     - press article, Observations 4 and 6 (Fig. 5 parts 1 and 3): the inner model may be a
 *       2-layer MLP (width ratio up to 4) or a 3x3 depthwise convolution over the token grid.
 *   Readings where the pages are silent (each also listed in the design notes of the repository):
 *     - the gradient is the MEAN over the N pairs (factor 2/N), not the sum;
 *     - the conv head is a cross-correlation with zero padding, stride 1, no bias, one 3x3 kernel
 *       per channel, tokens in raster order n = y*W + x, channel c = feature c of the head;
 *       the full 3x3 conv head (the article's other variant) has the same conventions with a
 *       d x d x 3 x 3 kernel, every output channel reading every input channel;
 *     - the MLP head is f(x) = Wb * gelu_tanh(Wa * x) with no biases, and both matrices take one
 *       simultaneous step from gradients evaluated at the initial weights.
 *     - the dot-product inner loss of the ViT3 recipe (press article, section on the ViT3 model;
 *       the loss itself is not printed) is the negative mean inner product of prediction and value,
 *       L(W) = -(1/N) sum_n <f(k_n; W), v_n>.
 *     - the mini-batch variants take every in-batch gradient at the weights the mini-batch starts
 *       from; inside a batch the notes' prefix sum carries no 1/b, while the press article's
 *       B = N/k ablation takes one step of each batch's mean loss and reads out with the final
 *       weights;
 *     - the backward pass differentiates the full-batch linear, depthwise-conv and MLP steps;
 *       W0 and eta are shared by every unit, so their gradients are summed (over images, over units).
 *
 * Memory layout of every array (contiguous, row-major, fp64):
 *   Q, K, V, Z : [B][heads][N][d]     (token n, feature c at ((b*heads + h)*N + n)*d + c)
 *   linear W   : [heads][d][d]        W[i][j] maps input feature j to output feature i
 *   conv W     : [heads][d][3][3]     W[c][a][b] multiplies the input at offset (a-1, b-1)
 *   dense conv W: [heads][d][d][3][3] W[c][c'][a][b] maps input channel c' at offset (a-1, b-1)
 *                                     to output channel c
 *   mlp Wa     : [heads][hidden][d],  Wb : [heads][d][hidden]
 *   updated weights are returned per unit: [B][heads][...]
 *
 * Every routine is written as the definition states it: explicit loops, no blocking, no reordering.
 * Units are independent; OpenMP only distributes whole units over threads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* ------------------------------------------------------------------------------------------ */
/* Linear inner model f(x) = W x.                                                               */
/* ------------------------------------------------------------------------------------------ */

/* One unit, per-pair form: grad = (2/N) sum_n (W0 k_n - v_n) k_n^T  (Vision-TTT notes, 关键设计 1,
 * the gradient G_t summed over all pairs and divided by N); W1 = W0 - eta*grad; z_n = W1 q_n. */
static int linear_unit_pairs(int N, int d, const double* Q, const double* K, const double* V,
                             const double* W0, double eta, double* W1, double* Z)
{
    double* grad = (double*)calloc((size_t)d * d, sizeof(double));
    double* r = (double*)malloc((size_t)d * sizeof(double));
    if (!grad || !r) { free(grad); free(r); return ORACLE_ERR_NOMEM; }
    for (int n = 0; n < N; ++n) {
        const double* k = K + (size_t)n * d;
        const double* v = V + (size_t)n * d;
        for (int i = 0; i < d; ++i) {           /* residual r = W0 k - v */
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += W0[(size_t)i * d + j] * k[j];
            r[i] = s - v[i];
        }
        for (int i = 0; i < d; ++i)             /* grad += r k^T */
            for (int j = 0; j < d; ++j) grad[(size_t)i * d + j] += r[i] * k[j];
    }
    const double scale = 2.0 / (double)N;
    for (int i = 0; i < d * d; ++i) W1[i] = W0[i] - eta * scale * grad[i];
    for (int n = 0; n < N; ++n) {                /* readout z = W1 q */
        const double* q = Q + (size_t)n * d;
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += W1[(size_t)i * d + j] * q[j];
            Z[(size_t)n * d + i] = s;
        }
    }
    free(grad); free(r);
    return ORACLE_OK;
}

/* One unit, Gram form: G = sum_n k_n k_n^T, C = sum_n v_n k_n^T,
 * W1 = W0 - eta*(2/N)*(W0 G - C).  Algebraically the same step as the per-pair form
 * (sum_n (W0 k_n - v_n) k_n^T = W0 G - C); kept as a second, independent routine. */
static int linear_unit_gram(int N, int d, const double* Q, const double* K, const double* V,
                            const double* W0, double eta, double* W1, double* Z)
{
    double* G = (double*)calloc((size_t)d * d, sizeof(double));
    double* C = (double*)calloc((size_t)d * d, sizeof(double));
    if (!G || !C) { free(G); free(C); return ORACLE_ERR_NOMEM; }
    for (int n = 0; n < N; ++n) {
        const double* k = K + (size_t)n * d;
        const double* v = V + (size_t)n * d;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) {
                G[(size_t)i * d + j] += k[i] * k[j];
                C[(size_t)i * d + j] += v[i] * k[j];
            }
    }
    const double scale = 2.0 / (double)N;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) {
            double wg = 0.0;
            for (int m = 0; m < d; ++m) wg += W0[(size_t)i * d + m] * G[(size_t)m * d + j];
            W1[(size_t)i * d + j] = W0[(size_t)i * d + j] - eta * scale * (wg - C[(size_t)i * d + j]);
        }
    for (int n = 0; n < N; ++n) {
        const double* q = Q + (size_t)n * d;
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += W1[(size_t)i * d + j] * q[j];
            Z[(size_t)n * d + i] = s;
        }
    }
    free(G); free(C);
    return ORACLE_OK;
}

static int linear_batch(int gram, int B, int heads, int N, int d, const double* Q, const double* K,
                        const double* V, const double* W0, double eta, double* W1, double* Z,
                        int nthreads)
{
    if (B < 0 || heads < 0 || N < 1 || d < 1 || !Q || !K || !V || !W0 || !W1 || !Z)
        return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int h = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        int s = gram ? linear_unit_gram(N, d, Q + off, K + off, V + off, W0 + (size_t)h * d * d,
                                        eta, W1 + (size_t)u * d * d, Z + off)
                     : linear_unit_pairs(N, d, Q + off, K + off, V + off, W0 + (size_t)h * d * d,
                                         eta, W1 + (size_t)u * d * d, Z + off);
        if (s != ORACLE_OK) {
#pragma omp atomic write
            status = s;
        }
    }
    return status;
}

int oracle_linear(int B, int heads, int N, int d, const double* Q, const double* K, const double* V,
                  const double* W0, double eta, double* W1, double* Z, int nthreads)
{
    return linear_batch(0, B, heads, N, d, Q, K, V, W0, eta, W1, Z, nthreads);
}

int oracle_linear_gram(int B, int heads, int N, int d, const double* Q, const double* K,
                       const double* V, const double* W0, double eta, double* W1, double* Z,
                       int nthreads)
{
    return linear_batch(1, B, heads, N, d, Q, K, V, W0, eta, W1, Z, nthreads);
}

/* ------------------------------------------------------------------------------------------ */
/* Linear inner model trained with the dot-product inner loss (press article, section            */
/* ViT3：視覺測試時訓練模型: ViT3's inner training is one full-batch step with a dot-product loss,  */
/* learning rate 1.0).  The pages do not print the loss; read as the negative mean inner product  */
/* of prediction and value,                                                                     */
/*     L(W) = -(1/N) sum_n <W k_n, v_n>,   dL/dW = -(1/N) sum_n v_n k_n^T,                        */
/*     W1 = W0 - eta dL/dW = W0 + (eta/N) sum_n v_n k_n^T,   z_n = W1 q_n.                        */
/* Its mixed second derivative d2L/dW dv is not zero (press article, Observation 1).  The update   */
/* does not depend on W0: there is no Gram term.                                                  */
/* ------------------------------------------------------------------------------------------ */

static int linear_dot_unit(int N, int d, const double* Q, const double* K, const double* V,
                           const double* W0, double eta, double* W1, double* Z)
{
    double* grad = (double*)calloc((size_t)d * d, sizeof(double));
    if (!grad) return ORACLE_ERR_NOMEM;
    for (int n = 0; n < N; ++n) {                /* grad -= v_n k_n^T */
        const double* k = K + (size_t)n * d;
        const double* v = V + (size_t)n * d;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) grad[(size_t)i * d + j] -= v[i] * k[j];
    }
    const double scale = 1.0 / (double)N;
    for (int i = 0; i < d * d; ++i) W1[i] = W0[i] - eta * scale * grad[i];
    for (int n = 0; n < N; ++n) {                /* readout z = W1 q */
        const double* q = Q + (size_t)n * d;
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += W1[(size_t)i * d + j] * q[j];
            Z[(size_t)n * d + i] = s;
        }
    }
    free(grad);
    return ORACLE_OK;
}

int oracle_linear_dot(int B, int heads, int N, int d, const double* Q, const double* K, const double* V,
                      const double* W0, double eta, double* W1, double* Z, int nthreads)
{
    if (B < 0 || heads < 0 || N < 1 || d < 1 || !Q || !K || !V || !W0 || !W1 || !Z) return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int h = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        int st = linear_dot_unit(N, d, Q + off, K + off, V + off, W0 + (size_t)h * d * d, eta,
                                 W1 + (size_t)u * d * d, Z + off);
        if (st != ORACLE_OK) {
#pragma omp atomic write
            status = st;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------------------------ */
/* Backward pass of the linear head (press article, Observation 1: the layer is trained end to   */
/* end through its inner step, the outer gradient flowing through the inner update).  Given the */
/* upstream gradient dZ of the forward above (L2 loss, full batch), the chain rule through       */
/*     G = sum k k^T,  C = sum v k^T,  W1 = W0 - s (W0 G - C),  z = W1 q,   s = 2 eta / N        */
/* gives                                                                                         */
/*     dW1 = sum dz q^T,   dq = W1^T dz,                                                          */
/*     dW0 = dW1 (I - s G),   dC = s dW1,   dG = -s W0^T dW1,                                     */
/*     dv = dC k,   dk = dC^T v + (dG + dG^T) k,   deta = -(2/N) sum_ij dW1_ij (W0 G - C)_ij.     */
/* W0 and eta are shared by every unit: dW0 is summed over the images of each head and deta over */
/* every unit, in index order.                                                                   */
/* ------------------------------------------------------------------------------------------ */

static int linear_backward_unit(int N, int d, const double* Q, const double* K, const double* V,
                                const double* W0, double eta, const double* dZ, double* dQ, double* dK,
                                double* dV, double* dW0, double* deta)
{
    const size_t dd = (size_t)d * d;
    double* buf = (double*)calloc(8 * dd, sizeof(double));
    if (!buf) return ORACLE_ERR_NOMEM;
    double *G = buf, *C = buf + dd, *dW1 = buf + 2 * dd, *W1 = buf + 3 * dd, *P = buf + 4 * dd;
    double *dC = buf + 5 * dd, *dG = buf + 6 * dd;
    const double s = 2.0 * eta / (double)N;
    for (int n = 0; n < N; ++n) {
        const double *k = K + (size_t)n * d, *v = V + (size_t)n * d, *q = Q + (size_t)n * d;
        const double* dz = dZ + (size_t)n * d;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) {
                G[(size_t)i * d + j] += k[i] * k[j];
                C[(size_t)i * d + j] += v[i] * k[j];
                dW1[(size_t)i * d + j] += dz[i] * q[j];
            }
    }
    for (int i = 0; i < d; ++i)                              /* P = W0 G - C,  W1 = W0 - s P */
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int m = 0; m < d; ++m) acc += W0[(size_t)i * d + m] * G[(size_t)m * d + j];
            P[(size_t)i * d + j] = acc - C[(size_t)i * d + j];
            W1[(size_t)i * d + j] = W0[(size_t)i * d + j] - s * P[(size_t)i * d + j];
        }
    double de = 0.0;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) {
            double acc = 0.0, g = 0.0;
            for (int m = 0; m < d; ++m) {
                acc += dW1[(size_t)i * d + m] * G[(size_t)m * d + j];   /* (dW1 G)_ij */
                g += W0[(size_t)m * d + i] * dW1[(size_t)m * d + j];    /* (W0^T dW1)_ij */
            }
            dW0[(size_t)i * d + j] += dW1[(size_t)i * d + j] - s * acc;
            dC[(size_t)i * d + j] = s * dW1[(size_t)i * d + j];
            dG[(size_t)i * d + j] = -s * g;
            de += dW1[(size_t)i * d + j] * P[(size_t)i * d + j];
        }
    *deta += -(2.0 / (double)N) * de;
    for (int n = 0; n < N; ++n) {
        const double *k = K + (size_t)n * d, *v = V + (size_t)n * d, *dz = dZ + (size_t)n * d;
        for (int j = 0; j < d; ++j) {
            double aq = 0.0, ak = 0.0, av = 0.0;
            for (int i = 0; i < d; ++i) {
                aq += W1[(size_t)i * d + j] * dz[i];                                   /* W1^T dz */
                ak += dC[(size_t)i * d + j] * v[i]                                     /* dC^T v */
                      + (dG[(size_t)j * d + i] + dG[(size_t)i * d + j]) * k[i];         /* (dG + dG^T) k */
                av += dC[(size_t)j * d + i] * k[i];                                    /* dC k */
            }
            dQ[(size_t)n * d + j] = aq;
            dK[(size_t)n * d + j] = ak;
            dV[(size_t)n * d + j] = av;
        }
    }
    free(buf);
    return ORACLE_OK;
}

/* dW0: [heads][d][d] (summed over images), deta: one value (summed over units).  Units run one at a
 * time per head in image order so that both sums have a fixed order; heads run in parallel. */
int oracle_linear_backward(int B, int heads, int N, int d, const double* Q, const double* K, const double* V,
                           const double* W0, double eta, const double* dZ, double* dQ, double* dK, double* dV,
                           double* dW0, double* deta, int nthreads)
{
    if (B < 0 || heads < 0 || N < 1 || d < 1 || !Q || !K || !V || !W0 || !dZ || !dQ || !dK || !dV || !dW0 ||
        !deta)
        return ORACLE_ERR_ARG;
    double* deta_h = (double*)calloc(heads > 0 ? (size_t)heads : 1, sizeof(double));
    if (!deta_h) return ORACLE_ERR_NOMEM;
    memset(dW0, 0, (size_t)heads * d * d * sizeof(double));
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int h = 0; h < heads; ++h) {
        for (int b = 0; b < B; ++b) {
            const size_t off = ((size_t)b * heads + h) * N * d;
            int st = linear_backward_unit(N, d, Q + off, K + off, V + off, W0 + (size_t)h * d * d, eta, dZ + off,
                                          dQ + off, dK + off, dV + off, dW0 + (size_t)h * d * d, &deta_h[h]);
            if (st != ORACLE_OK) {
#pragma omp atomic write
                status = st;
            }
        }
    }
    double total = 0.0;
    for (int h = 0; h < heads; ++h) total += deta_h[h];
    *deta = total;
    free(deta_h);
    return status;
}

/* ------------------------------------------------------------------------------------------ */
/* Linear inner model trained by mini-batch gradient descent over consecutive token batches.    */
/*   The tokens, in raster order, are cut into consecutive mini-batches of b tokens (the last     */
/*   may be shorter).  In every mini-batch the per-token gradients are taken at the weights W_s   */
/*   the mini-batch starts from:  G_t = 2 (W_s k_t - v_t) k_t^T  (L2 loss, the notes' G_t).       */
/*   mode 0, prefix ("Vision-TTT" paper notes, section 关键设计 4): inside a mini-batch the       */
/*     weights follow the causal prefix sum  W_t = W_s - eta * sum_{s<=t} G_s  and token t reads  */
/*     out z_t = W_t q_t; the next mini-batch starts from the last W_t.                          */
/*   mode 1, epoch (press article, Observation 2 and Fig. 3: the dataset cut into 2, 3 or 4       */
/*     consecutive mini-batches, one parameter update per mini-batch): every mini-batch takes    */
/*     one step of its mean L2 loss,  W <- W_s - eta (2/|batch|) sum_t (W_s k_t - v_t) k_t^T,    */
/*     and every query is read out with the weights after the last mini-batch.  With b >= N     */
/*     this is the full-batch step above.                                                       */
/* ------------------------------------------------------------------------------------------ */

static int linear_minibatch_unit(int N, int d, int b, int mode, const double* Q, const double* K,
                                 const double* V, const double* W0, double eta, double* W1, double* Z)
{
    double* Ws = (double*)malloc((size_t)d * d * sizeof(double));   /* weights at the batch start */
    double* Wt = (double*)malloc((size_t)d * d * sizeof(double));   /* running weights */
    double* R = (double*)malloc((size_t)b * d * sizeof(double));    /* residuals of the batch */
    if (!Ws || !Wt || !R) { free(Ws); free(Wt); free(R); return ORACLE_ERR_NOMEM; }
    memcpy(Ws, W0, (size_t)d * d * sizeof(double));
    for (int start = 0; start < N; start += b) {
        const int end = (start + b < N) ? start + b : N;
        const int nb = end - start;
        for (int t = start; t < end; ++t) {                 /* r_t = W_s k_t - v_t */
            const double* k = K + (size_t)t * d;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += Ws[(size_t)i * d + j] * k[j];
                R[(size_t)(t - start) * d + i] = acc - V[(size_t)t * d + i];
            }
        }
        memcpy(Wt, Ws, (size_t)d * d * sizeof(double));
        /* prefix: step -eta*G_t after each token; epoch: the batch mean, one step */
        const double step = (mode == 0) ? eta : eta / (double)nb;
        for (int t = start; t < end; ++t) {
            const double* k = K + (size_t)t * d;
            const double* r = R + (size_t)(t - start) * d;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) Wt[(size_t)i * d + j] -= step * 2.0 * r[i] * k[j];
            if (mode == 0) {                                 /* z_t = W_t q_t */
                const double* q = Q + (size_t)t * d;
                for (int i = 0; i < d; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < d; ++j) acc += Wt[(size_t)i * d + j] * q[j];
                    Z[(size_t)t * d + i] = acc;
                }
            }
        }
        memcpy(Ws, Wt, (size_t)d * d * sizeof(double));
    }
    if (mode == 1) {                                         /* readout with the final weights */
        for (int t = 0; t < N; ++t) {
            const double* q = Q + (size_t)t * d;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += Ws[(size_t)i * d + j] * q[j];
                Z[(size_t)t * d + i] = acc;
            }
        }
    }
    memcpy(W1, Ws, (size_t)d * d * sizeof(double));
    free(Ws); free(Wt); free(R);
    return ORACLE_OK;
}

int oracle_linear_minibatch(int B, int heads, int N, int d, int b, int mode, const double* Q,
                            const double* K, const double* V, const double* W0, double eta,
                            double* W1, double* Z, int nthreads)
{
    if (B < 0 || heads < 0 || N < 1 || d < 1 || b < 1 || (mode != 0 && mode != 1) || !Q || !K || !V ||
        !W0 || !W1 || !Z)
        return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int h = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        int st = linear_minibatch_unit(N, d, b, mode, Q + off, K + off, V + off, W0 + (size_t)h * d * d,
                                       eta, W1 + (size_t)u * d * d, Z + off);
        if (st != ORACLE_OK) {
#pragma omp atomic write
            status = st;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------------------------ */
/* 3x3 depthwise-convolution inner model over the H x W token grid                             */
/* (press article, Observation 6 and Fig. 5 part 3; ViT3 news article, 原則六 and section      */
/* 效果全面驗證: one head uses a 3x3 depthwise convolution).                                     */
/* ------------------------------------------------------------------------------------------ */

/* Value of channel c of a [N][d] token-major map at grid position (y, x); zero outside the grid. */
static double grid_at(const double* X, int Hg, int Wg, int d, int c, int y, int x)
{
    if (y < 0 || y >= Hg || x < 0 || x >= Wg) return 0.0;
    return X[((size_t)y * Wg + x) * d + c];
}

/* One unit.  f(X;W)[c,y,x] = sum_{a,b in 0..2} W[c][a][b] * X[c, y+a-1, x+b-1].
 * r = f(K;W0) - V;  g[c][a][b] = (2/N) sum_{y,x} r[c,y,x] * K[c, y+a-1, x+b-1];
 * W1 = W0 - eta*g;  Z = f(Q;W1). */
static int dwconv_unit(int Hg, int Wg, int d, const double* Q, const double* K, const double* V,
                       const double* W0, double eta, double* W1, double* Z)
{
    const int N = Hg * Wg;
    double* g = (double*)calloc((size_t)d * 9, sizeof(double));
    if (!g) return ORACLE_ERR_NOMEM;
    for (int c = 0; c < d; ++c) {
        const double* w = W0 + (size_t)c * 9;
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double f = 0.0;
                for (int a = 0; a < 3; ++a)
                    for (int b = 0; b < 3; ++b)
                        f += w[a * 3 + b] * grid_at(K, Hg, Wg, d, c, y + a - 1, x + b - 1);
                const double r = f - V[((size_t)y * Wg + x) * d + c];
                for (int a = 0; a < 3; ++a)
                    for (int b = 0; b < 3; ++b)
                        g[(size_t)c * 9 + a * 3 + b] += r * grid_at(K, Hg, Wg, d, c, y + a - 1, x + b - 1);
            }
    }
    const double scale = 2.0 / (double)N;
    for (int i = 0; i < d * 9; ++i) W1[i] = W0[i] - eta * scale * g[i];
    for (int c = 0; c < d; ++c) {
        const double* w = W1 + (size_t)c * 9;
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double f = 0.0;
                for (int a = 0; a < 3; ++a)
                    for (int b = 0; b < 3; ++b)
                        f += w[a * 3 + b] * grid_at(Q, Hg, Wg, d, c, y + a - 1, x + b - 1);
                Z[((size_t)y * Wg + x) * d + c] = f;
            }
    }
    free(g);
    return ORACLE_OK;
}

int oracle_dwconv(int B, int heads, int Hg, int Wg, int d, const double* Q, const double* K,
                  const double* V, const double* W0, double eta, double* W1, double* Z, int nthreads)
{
    if (B < 0 || heads < 0 || Hg < 1 || Wg < 1 || d < 1 || !Q || !K || !V || !W0 || !W1 || !Z)
        return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    const size_t N = (size_t)Hg * Wg;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int h = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        int s = dwconv_unit(Hg, Wg, d, Q + off, K + off, V + off, W0 + (size_t)h * d * 9, eta,
                            W1 + (size_t)u * d * 9, Z + off);
        if (s != ORACLE_OK) {
#pragma omp atomic write
            status = s;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------------------------ */
/* Full (dense) 3x3 convolution inner model over the token grid (press article, Observation 6   */
/* and Fig. 5 part 3: the inner model implemented as a 3x3 convolution or as a depthwise one).  */
/* ------------------------------------------------------------------------------------------ */

/* One unit.  f(X;W)[c,y,x] = sum_{c'} sum_{a,b in 0..2} W[c][c'][a][b] * X[c', y+a-1, x+b-1]
 * (every output channel reads every input channel; zero padding; no bias).
 * r = f(K;W0) - V;  g[c][c'][a][b] = (2/N) sum_{y,x} r[c,y,x] * K[c', y+a-1, x+b-1];
 * W1 = W0 - eta*g;  Z = f(Q;W1).  W: [d][d][3][3]. */
static int conv3x3_unit(int Hg, int Wg, int d, const double* Q, const double* K, const double* V,
                        const double* W0, double eta, double* W1, double* Z)
{
    const int N = Hg * Wg;
    double* g = (double*)calloc((size_t)d * d * 9, sizeof(double));
    if (!g) return ORACLE_ERR_NOMEM;
    for (int c = 0; c < d; ++c)
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double f = 0.0;
                for (int cp = 0; cp < d; ++cp)
                    for (int a = 0; a < 3; ++a)
                        for (int b = 0; b < 3; ++b)
                            f += W0[((size_t)c * d + cp) * 9 + a * 3 + b] * grid_at(K, Hg, Wg, d, cp, y + a - 1, x + b - 1);
                const double r = f - V[((size_t)y * Wg + x) * d + c];
                for (int cp = 0; cp < d; ++cp)
                    for (int a = 0; a < 3; ++a)
                        for (int b = 0; b < 3; ++b)
                            g[((size_t)c * d + cp) * 9 + a * 3 + b] += r * grid_at(K, Hg, Wg, d, cp, y + a - 1, x + b - 1);
            }
    const double scale = 2.0 / (double)N;
    for (size_t i = 0; i < (size_t)d * d * 9; ++i) W1[i] = W0[i] - eta * scale * g[i];
    for (int c = 0; c < d; ++c)
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double f = 0.0;
                for (int cp = 0; cp < d; ++cp)
                    for (int a = 0; a < 3; ++a)
                        for (int b = 0; b < 3; ++b)
                            f += W1[((size_t)c * d + cp) * 9 + a * 3 + b] * grid_at(Q, Hg, Wg, d, cp, y + a - 1, x + b - 1);
                Z[((size_t)y * Wg + x) * d + c] = f;
            }
    free(g);
    return ORACLE_OK;
}

int oracle_conv3x3(int B, int heads, int Hg, int Wg, int d, const double* Q, const double* K,
                   const double* V, const double* W0, double eta, double* W1, double* Z, int nthreads)
{
    if (B < 0 || heads < 0 || Hg < 1 || Wg < 1 || d < 1 || !Q || !K || !V || !W0 || !W1 || !Z)
        return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    const size_t N = (size_t)Hg * Wg;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int h = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        int s = conv3x3_unit(Hg, Wg, d, Q + off, K + off, V + off, W0 + (size_t)h * d * d * 9, eta,
                             W1 + (size_t)u * d * d * 9, Z + off);
        if (s != ORACLE_OK) {
#pragma omp atomic write
            status = s;
        }
    }
    return status;
}

/* Backward pass of the depthwise-conv head (press article, Observation 1: the outer gradient    */
/* flows through the inner step).  Per channel c, with taps t = (a, b), shifts s_t = (a-1, b-1),  */
/* K[c, p + s_t] zero outside the grid, and the forward                                          */
/*     r_p = sum_t W0_t K_{p+s_t} - V_p,   g_t = (2/N) sum_p r_p K_{p+s_t},   W1 = W0 - eta g,    */
/*     Z_p = sum_t W1_t Q_{p+s_t},                                                               */
/* the chain rule for the upstream gradient dZ gives, with dg = -eta dW1:                        */
/*     dW1_t = sum_p dZ_p Q_{p+s_t},          dQ_q = sum_t W1_t dZ_{q-s_t},                      */
/*     dr_p = (2/N) sum_t dg_t K_{p+s_t},     dV_p = -dr_p,                                      */
/*     dK_q = (2/N) sum_t dg_t r_{q-s_t} + sum_t W0_t dr_{q-s_t},                                 */
/*     dW0_t = dW1_t + sum_p dr_p K_{p+s_t},  deta = -sum_t dW1_t g_t                            */
/* (positions q - s_t outside the grid contribute nothing).  As for the linear head, dW0 is      */
/* summed over the images of each head and deta over every unit, in index order.                 */
static int dwconv_backward_unit(int Hg, int Wg, int d, const double* Q, const double* K, const double* V,
                                const double* W0, double eta, const double* dZ, double* dQ, double* dK,
                                double* dV, double* dW0, double* deta)
{
    const int N = Hg * Wg;
    double* r = (double*)malloc((size_t)N * sizeof(double));
    double* dr = (double*)malloc((size_t)N * sizeof(double));
    if (!r || !dr) { free(r); free(dr); return ORACLE_ERR_NOMEM; }
    const double scale = 2.0 / (double)N;
    double de = 0.0;
    for (int c = 0; c < d; ++c) {
        const double* w0 = W0 + (size_t)c * 9;
        double g[9] = {0}, dW1[9] = {0}, w1[9], dg[9];
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double f = 0.0;
                for (int t = 0; t < 9; ++t) f += w0[t] * grid_at(K, Hg, Wg, d, c, y + t / 3 - 1, x + t % 3 - 1);
                r[y * Wg + x] = f - V[((size_t)y * Wg + x) * d + c];
            }
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x)
                for (int t = 0; t < 9; ++t) {
                    g[t] += r[y * Wg + x] * grid_at(K, Hg, Wg, d, c, y + t / 3 - 1, x + t % 3 - 1);
                    dW1[t] += dZ[((size_t)y * Wg + x) * d + c] * grid_at(Q, Hg, Wg, d, c, y + t / 3 - 1, x + t % 3 - 1);
                }
        for (int t = 0; t < 9; ++t) {
            g[t] *= scale;
            w1[t] = w0[t] - eta * g[t];
            dg[t] = -eta * dW1[t];
            de += -dW1[t] * g[t];
        }
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double a = 0.0;
                for (int t = 0; t < 9; ++t) a += dg[t] * grid_at(K, Hg, Wg, d, c, y + t / 3 - 1, x + t % 3 - 1);
                dr[y * Wg + x] = scale * a;
            }
        double dw0[9];
        for (int t = 0; t < 9; ++t) dw0[t] = dW1[t];
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                const size_t o = ((size_t)y * Wg + x) * d + c;
                double aq = 0.0, ak = 0.0;
                for (int t = 0; t < 9; ++t) {
                    const int yy = y - (t / 3 - 1), xx = x - (t % 3 - 1);   /* q - s_t */
                    if (yy < 0 || yy >= Hg || xx < 0 || xx >= Wg) continue;
                    aq += w1[t] * dZ[((size_t)yy * Wg + xx) * d + c];
                    ak += scale * dg[t] * r[yy * Wg + xx] + w0[t] * dr[yy * Wg + xx];
                }
                dQ[o] = aq;
                dK[o] = ak;
                dV[o] = -dr[y * Wg + x];
                for (int t = 0; t < 9; ++t) dw0[t] += dr[y * Wg + x] * grid_at(K, Hg, Wg, d, c, y + t / 3 - 1, x + t % 3 - 1);
            }
        for (int t = 0; t < 9; ++t) dW0[(size_t)c * 9 + t] += dw0[t];
    }
    *deta += de;
    free(r);
    free(dr);
    return ORACLE_OK;
}

/* dW0: [heads][d][3][3] (summed over images), deta: one value (summed over units), as for the
 * linear head's backward. */
int oracle_dwconv_backward(int B, int heads, int Hg, int Wg, int d, const double* Q, const double* K,
                           const double* V, const double* W0, double eta, const double* dZ, double* dQ,
                           double* dK, double* dV, double* dW0, double* deta, int nthreads)
{
    if (B < 0 || heads < 0 || Hg < 1 || Wg < 1 || d < 1 || !Q || !K || !V || !W0 || !dZ || !dQ || !dK || !dV ||
        !dW0 || !deta)
        return ORACLE_ERR_ARG;
    const size_t N = (size_t)Hg * Wg;
    double* deta_h = (double*)calloc(heads > 0 ? (size_t)heads : 1, sizeof(double));
    if (!deta_h) return ORACLE_ERR_NOMEM;
    memset(dW0, 0, (size_t)heads * d * 9 * sizeof(double));
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int h = 0; h < heads; ++h) {
        for (int b = 0; b < B; ++b) {
            const size_t off = ((size_t)b * heads + h) * N * d;
            int st = dwconv_backward_unit(Hg, Wg, d, Q + off, K + off, V + off, W0 + (size_t)h * d * 9, eta, dZ + off,
                                          dQ + off, dK + off, dV + off, dW0 + (size_t)h * d * 9, &deta_h[h]);
            if (st != ORACLE_OK) {
#pragma omp atomic write
                status = st;
            }
        }
    }
    double total = 0.0;
    for (int h = 0; h < heads; ++h) total += deta_h[h];
    *deta = total;
    free(deta_h);
    return status;
}

/* The conv inner model trained with the dot-product inner loss (press article, section
 * ViT3：視覺測試時訓練模型: the ViT3 recipe pairs the dot-product loss with a depthwise-conv inner
 * model).  Read as L(W) = -(1/N) sum_{c,y,x} f(K;W)[c,y,x] * V[c,y,x], whose gradient is
 *     g[c][a][b] = -(1/N) sum_{y,x} V[c,y,x] * K[c, y+a-1, x+b-1],
 * W1 = W0 - eta*g;  Z = f(Q;W1).  The update does not depend on W0. */
static int dwconv_dot_unit(int Hg, int Wg, int d, const double* Q, const double* K, const double* V,
                           const double* W0, double eta, double* W1, double* Z)
{
    const int N = Hg * Wg;
    double* g = (double*)calloc((size_t)d * 9, sizeof(double));
    if (!g) return ORACLE_ERR_NOMEM;
    for (int c = 0; c < d; ++c)
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                const double v = V[((size_t)y * Wg + x) * d + c];
                for (int a = 0; a < 3; ++a)
                    for (int b = 0; b < 3; ++b)
                        g[(size_t)c * 9 + a * 3 + b] -= v * grid_at(K, Hg, Wg, d, c, y + a - 1, x + b - 1);
            }
    const double scale = 1.0 / (double)N;
    for (int i = 0; i < d * 9; ++i) W1[i] = W0[i] - eta * scale * g[i];
    for (int c = 0; c < d; ++c) {
        const double* w = W1 + (size_t)c * 9;
        for (int y = 0; y < Hg; ++y)
            for (int x = 0; x < Wg; ++x) {
                double f = 0.0;
                for (int a = 0; a < 3; ++a)
                    for (int b = 0; b < 3; ++b)
                        f += w[a * 3 + b] * grid_at(Q, Hg, Wg, d, c, y + a - 1, x + b - 1);
                Z[((size_t)y * Wg + x) * d + c] = f;
            }
    }
    free(g);
    return ORACLE_OK;
}

int oracle_dwconv_dot(int B, int heads, int Hg, int Wg, int d, const double* Q, const double* K,
                      const double* V, const double* W0, double eta, double* W1, double* Z, int nthreads)
{
    if (B < 0 || heads < 0 || Hg < 1 || Wg < 1 || d < 1 || !Q || !K || !V || !W0 || !W1 || !Z)
        return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    const size_t N = (size_t)Hg * Wg;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int h = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        int s = dwconv_dot_unit(Hg, Wg, d, Q + off, K + off, V + off, W0 + (size_t)h * d * 9, eta,
                                W1 + (size_t)u * d * 9, Z + off);
        if (s != ORACLE_OK) {
#pragma omp atomic write
            status = s;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------------------------ */
/* One-hidden-layer MLP inner model f(x) = Wb * gelu_tanh(Wa * x)                              */
/* (press article, Observation 4 and Fig. 5 part 1: a 2-layer MLP inner model, width ratio r up */
/* to 4; ViT3 news article, 原則四: widening d -> 4d).  The activation is GELU (tanh form).     */
/* ------------------------------------------------------------------------------------------ */

/* GELU, tanh form (Hendrycks & Gimpel, "Gaussian Error Linear Units", the tanh approximation):
 *   gelu(u) = u/2 * (1 + tanh( sqrt(2/pi) * (u + 0.044715 u^3) )). */
double oracle_gelu_tanh(double u)
{
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * u * (1.0 + tanh(c * (u + 0.044715 * u * u * u)));
}

/* Exact derivative of the expression above:
 *   d/du = 1/2 (1 + t) + u/2 (1 - t^2) * c * (1 + 3*0.044715 u^2),   t = tanh(c (u + 0.044715 u^3)). */
double oracle_gelu_tanh_deriv(double u)
{
    const double c = sqrt(2.0 / M_PI);
    const double t = tanh(c * (u + 0.044715 * u * u * u));
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * c * (1.0 + 3.0 * 0.044715 * u * u);
}

/* One unit.  With h_n = Wa k_n, a_n = gelu(h_n), y_n = Wb a_n, r_n = y_n - v_n:
 *   dL/dWb = (2/N) sum_n r_n a_n^T
 *   dL/dWa = (2/N) sum_n [ (Wb^T r_n) * gelu'(h_n) ] k_n^T      (* = elementwise)
 *   Wa1 = Wa - eta dL/dWa,  Wb1 = Wb - eta dL/dWb   (both from gradients at the initial weights)
 *   z_n = Wb1 gelu(Wa1 q_n). */
static int mlp_unit(int N, int d, int hidden, const double* Q, const double* K, const double* V,
                    const double* Wa, const double* Wb, double eta, double* Wa1, double* Wb1,
                    double* Z)
{
    double* gA = (double*)calloc((size_t)hidden * d, sizeof(double));
    double* gB = (double*)calloc((size_t)d * hidden, sizeof(double));
    double* h = (double*)malloc((size_t)hidden * sizeof(double));
    double* a = (double*)malloc((size_t)hidden * sizeof(double));
    double* r = (double*)malloc((size_t)d * sizeof(double));
    double* dh = (double*)malloc((size_t)hidden * sizeof(double));
    if (!gA || !gB || !h || !a || !r || !dh) {
        free(gA); free(gB); free(h); free(a); free(r); free(dh);
        return ORACLE_ERR_NOMEM;
    }
    for (int n = 0; n < N; ++n) {
        const double* k = K + (size_t)n * d;
        const double* v = V + (size_t)n * d;
        for (int j = 0; j < hidden; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += Wa[(size_t)j * d + i] * k[i];
            h[j] = s;
            a[j] = oracle_gelu_tanh(s);
        }
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < hidden; ++j) s += Wb[(size_t)i * hidden + j] * a[j];
            r[i] = s - v[i];
        }
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < hidden; ++j) gB[(size_t)i * hidden + j] += r[i] * a[j];
        for (int j = 0; j < hidden; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += Wb[(size_t)i * hidden + j] * r[i];
            dh[j] = s * oracle_gelu_tanh_deriv(h[j]);
        }
        for (int j = 0; j < hidden; ++j)
            for (int i = 0; i < d; ++i) gA[(size_t)j * d + i] += dh[j] * k[i];
    }
    const double scale = 2.0 / (double)N;
    for (int i = 0; i < hidden * d; ++i) Wa1[i] = Wa[i] - eta * scale * gA[i];
    for (int i = 0; i < d * hidden; ++i) Wb1[i] = Wb[i] - eta * scale * gB[i];
    for (int n = 0; n < N; ++n) {
        const double* q = Q + (size_t)n * d;
        for (int j = 0; j < hidden; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += Wa1[(size_t)j * d + i] * q[i];
            a[j] = oracle_gelu_tanh(s);
        }
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < hidden; ++j) s += Wb1[(size_t)i * hidden + j] * a[j];
            Z[(size_t)n * d + i] = s;
        }
    }
    free(gA); free(gB); free(h); free(a); free(r); free(dh);
    return ORACLE_OK;
}

int oracle_mlp(int B, int heads, int N, int d, int hidden, const double* Q, const double* K,
               const double* V, const double* Wa, const double* Wb, double eta, double* Wa1,
               double* Wb1, double* Z, int nthreads)
{
    if (B < 0 || heads < 0 || N < 1 || d < 1 || hidden < 1 || !Q || !K || !V || !Wa || !Wb ||
        !Wa1 || !Wb1 || !Z)
        return ORACLE_ERR_ARG;
    const long units = (long)B * heads;
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long u = 0; u < units; ++u) {
        const int hh = (int)(u % heads);
        const size_t off = (size_t)u * N * d;
        const size_t wsz = (size_t)hidden * d;
        int s = mlp_unit(N, d, hidden, Q + off, K + off, V + off, Wa + hh * wsz, Wb + hh * wsz, eta,
                         Wa1 + (size_t)u * wsz, Wb1 + (size_t)u * wsz, Z + off);
        if (s != ORACLE_OK) {
#pragma omp atomic write
            status = s;
        }
    }
    return status;
}

/* Second derivative of gelu_tanh (needed by the MLP head's backward pass): with
 * t = tanh(c (u + a u^3)) and w = c (1 + 3 a u^2),  gelu'' = (1 - t^2) (w - u t w^2 + 3 a c u^2). */
double oracle_gelu_tanh_deriv2(double u)
{
    const double c = sqrt(2.0 / M_PI), a = 0.044715;
    const double t = tanh(c * (u + a * u * u * u));
    const double w = c * (1.0 + 3.0 * a * u * u);
    return (1.0 - t * t) * (w - u * t * w * w + 3.0 * a * c * u * u);
}

/* Backward pass of the MLP head (press article, Observation 1: the outer gradient flows through the */
/* inner step; the head: Observation 4).  With s = 2/N and, per key token,                         */
/*   h = Wa k, a = gelu(h), D = gelu'(h), r = Wb a - v, b = Wb^T r, e = b * D  (* elementwise),     */
/*   gWb = s sum r a^T, gWa = s sum e k^T, Wa1 = Wa - eta gWa, Wb1 = Wb - eta gWb,                 */
/* and per query token hq = Wa1 q, aq = gelu(hq), z = Wb1 aq, the chain rule for dZ gives          */
/*   readout:  dWb1 = sum dz aq^T,  dhq = (Wb1^T dz) * gelu'(hq),  dq = Wa1^T dhq,                 */
/*             dWa1 = sum dhq q^T;                                                               */
/*   update:   dgWa = -eta dWa1, dgWb = -eta dWb1, deta = -sum dWa1 * gWa - sum dWb1 * gWb,        */
/*             and per key token                                                                 */
/*             de = s dgWa k,  db = de * D,  dD = de * b,  dr = s dgWb a + Wb db,                   */
/*             da = s dgWb^T r + Wb^T dr,  dh = da * D + dD * gelu''(h),                          */
/*             dk = s dgWa^T e + Wa^T dh,  dv = -dr,                                              */
/*             dWa += dh k^T,  dWb += dr a^T + r db^T;                                           */
/*   dWa_total = dWa1 + dWa,  dWb_total = dWb1 + dWb.                                            */
/* Wa, Wb and eta are shared by every unit: dWa, dWb are summed over the images of each head and   */
/* deta over every unit, in index order.                                                         */
static int mlp_backward_unit(int N, int d, int hid, const double* Q, const double* K, const double* V,
                             const double* Wa, const double* Wb, double eta, const double* dZ, double* dQ,
                             double* dK, double* dV, double* dWa, double* dWb, double* deta)
{
    const size_t wsz = (size_t)hid * d;
    double* buf = (double*)calloc(8 * wsz + 12 * (size_t)hid, sizeof(double));
    if (!buf) return ORACLE_ERR_NOMEM;
    double *gA = buf, *gB = buf + wsz, *Wa1 = buf + 2 * wsz, *Wb1 = buf + 3 * wsz;
    double *dWa1 = buf + 4 * wsz, *dWb1 = buf + 5 * wsz, *dgA = buf + 6 * wsz, *dgB = buf + 7 * wsz;
    double* vec = buf + 8 * wsz;
    double *h = vec, *a = vec + hid, *D = vec + 2 * hid, *bb = vec + 3 * hid, *e = vec + 4 * hid;
    double *de = vec + 5 * hid, *db = vec + 6 * hid, *dD = vec + 7 * hid, *da = vec + 8 * hid, *dh = vec + 9 * hid;
    double r[256], dr[256], dz[256];
    if (d > 256) { free(buf); return ORACLE_ERR_ARG; }
    const double s = 2.0 / (double)N;
    /* (1) the inner step's gradients at (Wa, Wb) and the updated weights */
    for (int n = 0; n < N; ++n) {
        const double *k = K + (size_t)n * d, *v = V + (size_t)n * d;
        for (int j = 0; j < hid; ++j) {
            double t = 0.0;
            for (int i = 0; i < d; ++i) t += Wa[(size_t)j * d + i] * k[i];
            h[j] = t; a[j] = oracle_gelu_tanh(t); D[j] = oracle_gelu_tanh_deriv(t);
        }
        for (int i = 0; i < d; ++i) {
            double t = 0.0;
            for (int j = 0; j < hid; ++j) t += Wb[(size_t)i * hid + j] * a[j];
            r[i] = t - v[i];
        }
        for (int j = 0; j < hid; ++j) {
            double t = 0.0;
            for (int i = 0; i < d; ++i) t += Wb[(size_t)i * hid + j] * r[i];
            e[j] = t * D[j];
        }
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < hid; ++j) gB[(size_t)i * hid + j] += s * r[i] * a[j];
        for (int j = 0; j < hid; ++j)
            for (int i = 0; i < d; ++i) gA[(size_t)j * d + i] += s * e[j] * k[i];
    }
    for (size_t i = 0; i < wsz; ++i) { Wa1[i] = Wa[i] - eta * gA[i]; Wb1[i] = Wb[i] - eta * gB[i]; }
    /* (2) the readout */
    for (int n = 0; n < N; ++n) {
        const double* q = Q + (size_t)n * d;
        for (int i = 0; i < d; ++i) dz[i] = dZ[(size_t)n * d + i];
        for (int j = 0; j < hid; ++j) {
            double t = 0.0;
            for (int i = 0; i < d; ++i) t += Wa1[(size_t)j * d + i] * q[i];
            h[j] = t; a[j] = oracle_gelu_tanh(t); D[j] = oracle_gelu_tanh_deriv(t);
        }
        for (int j = 0; j < hid; ++j) {
            double t = 0.0;
            for (int i = 0; i < d; ++i) t += Wb1[(size_t)i * hid + j] * dz[i];
            dh[j] = t * D[j];
        }
        for (int i = 0; i < d; ++i) {
            double t = 0.0;
            for (int j = 0; j < hid; ++j) t += Wa1[(size_t)j * d + i] * dh[j];
            dQ[(size_t)n * d + i] = t;
        }
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < hid; ++j) dWb1[(size_t)i * hid + j] += dz[i] * a[j];
        for (int j = 0; j < hid; ++j)
            for (int i = 0; i < d; ++i) dWa1[(size_t)j * d + i] += dh[j] * q[i];
    }
    double dsum = 0.0;
    for (size_t i = 0; i < wsz; ++i) {
        dgA[i] = -eta * dWa1[i];
        dgB[i] = -eta * dWb1[i];
        dsum += -dWa1[i] * gA[i] - dWb1[i] * gB[i];
        dWa[i] += dWa1[i];
        dWb[i] += dWb1[i];
    }
    *deta += dsum;
    /* (3) through the inner step, per key token */
    for (int n = 0; n < N; ++n) {
        const double *k = K + (size_t)n * d, *v = V + (size_t)n * d;
        for (int j = 0; j < hid; ++j) {
            double t = 0.0;
            for (int i = 0; i < d; ++i) t += Wa[(size_t)j * d + i] * k[i];
            h[j] = t; a[j] = oracle_gelu_tanh(t); D[j] = oracle_gelu_tanh_deriv(t);
        }
        for (int i = 0; i < d; ++i) {
            double t = 0.0;
            for (int j = 0; j < hid; ++j) t += Wb[(size_t)i * hid + j] * a[j];
            r[i] = t - v[i];
        }
        for (int j = 0; j < hid; ++j) {
            double t = 0.0, u = 0.0;
            for (int i = 0; i < d; ++i) { t += Wb[(size_t)i * hid + j] * r[i]; u += dgA[(size_t)j * d + i] * k[i]; }
            bb[j] = t; e[j] = t * D[j];
            de[j] = s * u; db[j] = de[j] * D[j]; dD[j] = de[j] * t;
        }
        for (int i = 0; i < d; ++i) {
            double t = 0.0;
            for (int j = 0; j < hid; ++j) t += s * dgB[(size_t)i * hid + j] * a[j] + Wb[(size_t)i * hid + j] * db[j];
            dr[i] = t;
        }
        for (int j = 0; j < hid; ++j) {
            double t = 0.0;
            for (int i = 0; i < d; ++i) t += s * dgB[(size_t)i * hid + j] * r[i] + Wb[(size_t)i * hid + j] * dr[i];
            da[j] = t;
            dh[j] = t * D[j] + dD[j] * oracle_gelu_tanh_deriv2(h[j]);
        }
        for (int i = 0; i < d; ++i) {
            double t = 0.0;
            for (int j = 0; j < hid; ++j) t += s * dgA[(size_t)j * d + i] * e[j] + Wa[(size_t)j * d + i] * dh[j];
            dK[(size_t)n * d + i] = t;
            dV[(size_t)n * d + i] = -dr[i];
        }
        for (int j = 0; j < hid; ++j)
            for (int i = 0; i < d; ++i) dWa[(size_t)j * d + i] += dh[j] * k[i];
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < hid; ++j) dWb[(size_t)i * hid + j] += dr[i] * a[j] + r[i] * db[j];
    }
    free(buf);
    return ORACLE_OK;
}

/* dWa: [heads][hidden][d], dWb: [heads][d][hidden] (summed over images), deta: one value (summed over
 * units), as for the linear head's backward. */
int oracle_mlp_backward(int B, int heads, int N, int d, int hidden, const double* Q, const double* K,
                        const double* V, const double* Wa, const double* Wb, double eta, const double* dZ,
                        double* dQ, double* dK, double* dV, double* dWa, double* dWb, double* deta, int nthreads)
{
    if (B < 0 || heads < 0 || N < 1 || d < 1 || d > 256 || hidden < 1 || !Q || !K || !V || !Wa || !Wb || !dZ ||
        !dQ || !dK || !dV || !dWa || !dWb || !deta)
        return ORACLE_ERR_ARG;
    const size_t wsz = (size_t)hidden * d;
    double* deta_h = (double*)calloc(heads > 0 ? (size_t)heads : 1, sizeof(double));
    if (!deta_h) return ORACLE_ERR_NOMEM;
    memset(dWa, 0, (size_t)heads * wsz * sizeof(double));
    memset(dWb, 0, (size_t)heads * wsz * sizeof(double));
    int status = ORACLE_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int h = 0; h < heads; ++h) {
        for (int b = 0; b < B; ++b) {
            const size_t off = ((size_t)b * heads + h) * N * d;
            int st = mlp_backward_unit(N, d, hidden, Q + off, K + off, V + off, Wa + h * wsz, Wb + h * wsz, eta,
                                       dZ + off, dQ + off, dK + off, dV + off, dWa + h * wsz, dWb + h * wsz,
                                       &deta_h[h]);
            if (st != ORACLE_OK) {
#pragma omp atomic write
                status = st;
            }
        }
    }
    double total = 0.0;
    for (int h = 0; h < heads; ++h) total += deta_h[h];
    *deta = total;
    free(deta_h);
    return status;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
