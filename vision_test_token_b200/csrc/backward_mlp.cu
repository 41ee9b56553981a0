// backward_mlp.cu -- backward pass of the MLP head f(x) = Wb gelu_tanh(Wa x) (press article "CVPR 2026
// Oral | 清華+阿里發布ViT3", Observation 1: the outer gradient flows through the inner step; the head:
// Observation 4).  With s = 2/N and, per key token,
//     h = Wa k, a = gelu(h), D = gelu'(h), r = Wb a - v, b = Wb^T r, e = b * D        (* elementwise),
//     gWb = s sum r a^T,  gWa = s sum e k^T,  Wa1 = Wa - eta gWa,  Wb1 = Wb - eta gWb,
// and per query token hq = Wa1 q, aq = gelu(hq), z = Wb1 aq, the chain rule for dZ gives
//     readout: dWb1 = sum dz aq^T, dhq = (Wb1^T dz) * gelu'(hq), dq = Wa1^T dhq, dWa1 = sum dhq q^T;
//     update:  dgWa = -eta dWa1, dgWb = -eta dWb1, deta = -sum dWa1 * gWa - sum dWb1 * gWb, and per key
//              token de = s dgWa k, db = de * D, dD = de * b, dr = s dgWb a + Wb db,
//              da = s dgWb^T r + Wb^T dr, dh = da * D + dD * gelu''(h), dk = s dgWa^T e + Wa^T dh,
//              dv = -dr, dWa += dh k^T, dWb += dr a^T + r db^T;
//     dWa_total = dWa1 + dWa, dWb_total = dWb1 + dWb (summed over the images of each head), deta
//     summed over every unit.
//
// First path in plain fp32 FMA (hidden width <= 256, d = 64): every kernel takes (unit, chunk) CTAs
// of 256 threads and walks its chunk of tokens in tiles of TT = 4.  Hidden-indexed quantities give
// thread j hidden unit j (for the four tokens); d-indexed ones give thread (t, i) token t, channel i.
// The weights are read through L1 in the layout that makes each warp's read contiguous (transposed
// copies are written once per call), vectors of the tile live in shared memory, and every CTA keeps
// its share of the weight-gradient sums in registers (thread j: row j of the hidden x d sum, column j
// of the d x hidden one).  Partial sums go to per-(unit, chunk) slots; every sum over them has a fixed
// order, so results are bitwise reproducible.
//   mb_prep   transposed copies of Wa, Wb
//   mb_fwd    per chunk: partial gWa, gWb                 mb_merge1  per unit: g, Wa1, Wb1 (+ Wa1^T)
//   mb_read   per chunk: dq, partial dWa1, dWb1           mb_merge2  per unit: dgWa, dgWb (+ ^T), deta
//   mb_upd    per chunk: dk, dv, partial dWa, dWb         mb_final   per head: dWa, dWb; deta
#include <algorithm>
#include <cmath>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace mb2 {

constexpr int D = 64;
constexpr int HMAX = 256;
constexpr int TT = 4;                        // tokens per tile
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float ldx(const T* p);
template <>
__device__ __forceinline__ float ldx<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldx<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <typename T>
__device__ __forceinline__ void stx(T* p, float v);
template <>
__device__ __forceinline__ void stx<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void stx<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// gelu with the tanh approximation, its first and second derivatives (written from the formula
// u/2 (1 + tanh(c (u + a u^3))), c = sqrt(2/pi), a = 0.044715; tanh from the CUDA math library).
struct Gelu {
    float g, d1, d2;
};
__device__ __forceinline__ Gelu gelu3(float u) {
    const float c = 0.7978845608028654f, a = 0.044715f;
    const float t = tanhf(c * (u + a * u * u * u));
    const float w = c * (1.f + 3.f * a * u * u);
    Gelu r;
    r.g = 0.5f * u * (1.f + t);
    r.d1 = 0.5f * (1.f + t) + 0.5f * u * (1.f - t * t) * w;
    r.d2 = (1.f - t * t) * (w - u * t * w * w + 3.f * a * c * u * u);
    return r;
}

struct Params {
    int heads, N, hid, U, nch;               // units, chunks per unit
    long long bs, hs;
    float eta, s;                            // eta, 2/N
    const float* Wa;                         // [heads][hid][64]
    const float* Wb;                         // [heads][64][hid]
    float* WaT;                              // [heads][64][hid]
    float* WbT;                              // [heads][hid][64]
    float* part;                             // [U][nch][2][hid*64]: per-chunk sums (reused by each phase)
    float* g;                                // [U][2][hid*64]: gWa, gWb
    float* w1;                               // [U][3][hid*64]: Wa1, Wb1, Wa1^T
    float* dg;                               // [U][4][hid*64]: dgWa, dgWb, dgWa^T, dgWb^T
    float* dw1;                              // [U][2][hid*64]: dWa1, dWb1
    float* upd;                              // [U][nch][2][hid*64]: per-chunk dWa, dWb of the update path
    float* deta_u;                           // [U]
    float* dWa_out;                          // nullable [heads][hid][64]
    float* dWb_out;                          // nullable [heads][64][hid]
    float* deta_out;                         // nullable
};

__device__ __forceinline__ long long unit_off(const Params& p, int u) {
    return (long long)(u / p.heads) * p.bs + (long long)(u % p.heads) * p.hs;
}
__device__ __forceinline__ void chunk_range(const Params& p, int c, int& n0, int& n1) {
    n0 = (int)((long long)p.N * c / p.nch);
    n1 = (int)((long long)p.N * (c + 1) / p.nch);
}

// Per-CTA sums kept in registers: thread j < hid owns row j of a hid x 64 sum (ra) and column j of a
// 64 x hid sum (cb).  Written to a [2][hid*64] slot: [0] row-major hid x 64, [1] row-major 64 x hid.
__device__ __forceinline__ void store_sums(float* slot, int hid, int j, const float (&ra)[D], const float (&cb)[D]) {
    if (j >= hid) return;
#pragma unroll
    for (int i = 0; i < D; i += 4)
        *reinterpret_cast<float4*>(slot + (size_t)j * D + i) = make_float4(ra[i], ra[i + 1], ra[i + 2], ra[i + 3]);
#pragma unroll
    for (int i = 0; i < D; ++i) slot[(size_t)hid * D + (size_t)i * hid + j] = cb[i];
}

// sum_jj x[jj] * y[jj] over jj < n (x[jj] = px[jj * D], y in shared memory) as four interleaved
// partial sums, added in a fixed order: a dependency chain of n / 4 instead of n.
template <class LD>
__device__ __forceinline__ float dot_hidden(float init, const float* px, const float* y, int n, LD ld) {
    float a0 = init, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int jj = 0;
    for (; jj + 4 <= n; jj += 4) {
        a0 = fmaf(ld(px + (size_t)jj * D), y[jj], a0);
        a1 = fmaf(ld(px + (size_t)(jj + 1) * D), y[jj + 1], a1);
        a2 = fmaf(ld(px + (size_t)(jj + 2) * D), y[jj + 2], a2);
        a3 = fmaf(ld(px + (size_t)(jj + 3) * D), y[jj + 3], a3);
    }
    for (; jj < n; ++jj) a0 = fmaf(ld(px + (size_t)jj * D), y[jj], a0);
    return (a0 + a1) + (a2 + a3);
}
// sum_jj (s1 x1[jj] y1[jj] + x2[jj] y2[jj]) likewise (per term: the x2 product first, then x1's).
template <class LD1, class LD2>
__device__ __forceinline__ float dot_hidden2(float s1, const float* px1, const float* y1, LD1 ld1, const float* px2,
                                             const float* y2, LD2 ld2, int n) {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    int jj = 0;
    for (; jj + 4 <= n; jj += 4)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            a[q] = fmaf(s1 * ld1(px1 + (size_t)(jj + q) * D), y1[jj + q], fmaf(ld2(px2 + (size_t)(jj + q) * D), y2[jj + q], a[q]));
    for (; jj < n; ++jj) a[0] = fmaf(s1 * ld1(px1 + (size_t)jj * D), y1[jj], fmaf(ld2(px2 + (size_t)jj * D), y2[jj], a[0]));
    return (a[0] + a[1]) + (a[2] + a[3]);
}
__device__ __forceinline__ float ld_nc(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }

// ---- mb_prep: transposes of Wa, Wb ----------------------------------------------------------------
__global__ void mb_prep(const Params p) {
    pdl_launch_dependents();
    const size_t w = (size_t)p.hid * D;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < (size_t)p.heads * w;
         e += (size_t)gridDim.x * blockDim.x) {
        const size_t h = e / w, r = e % w;
        const int j = (int)(r / D), i = (int)(r % D);       // Wa[h][j][i]
        p.WaT[h * w + (size_t)i * p.hid + j] = p.Wa[e];
        const int i2 = (int)(r / p.hid), j2 = (int)(r % p.hid);   // Wb[h][i2][j2]
        p.WbT[h * w + (size_t)j2 * D + i2] = p.Wb[e];
    }
}

// ---- mb_fwd: gWa, gWb partials --------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
mb_fwd(const T* __restrict__ K, const T* __restrict__ V, const Params p) {
    __shared__ float kv[2][TT][D];                          // k, v of the tile
    __shared__ float av[3][TT][HMAX];                       // a, D, e
    __shared__ float rv[TT][D];
    const int u = blockIdx.x / p.nch, c = blockIdx.x % p.nch, h = u % p.heads;
    const int j = threadIdx.x, hid = p.hid;
    const int ti = threadIdx.x / D, ci = threadIdx.x % D;    // (token, channel) view
    pdl_launch_dependents();
    pdl_wait_primary();                                      // the transposes
    const long long off = unit_off(p, u);
    const size_t w = (size_t)hid * D;
    const float *Wa = p.Wa + h * w, *Wb = p.Wb + h * w, *WaT = p.WaT + h * w, *WbT = p.WbT + h * w;
    float ga[D], gb[D];
#pragma unroll
    for (int i = 0; i < D; ++i) ga[i] = gb[i] = 0.f;
    int n0, n1;
    chunk_range(p, c, n0, n1);
    for (int n = n0; n < n1; n += TT) {
        const int nt = min(TT, n1 - n);
        {
            const float kk = ti < nt ? ldx(K + off + (long long)(n + ti) * D + ci) : 0.f;
            const float vv = ti < nt ? ldx(V + off + (long long)(n + ti) * D + ci) : 0.f;
            kv[0][ti][ci] = kk;
            kv[1][ti][ci] = vv;
        }
        __syncthreads();
        if (j < hid) {                                       // h = Wa k  (WaT: contiguous in j)
            float hh[TT] = {0.f, 0.f, 0.f, 0.f};
            for (int i = 0; i < D; ++i) {
                const float wv = __ldg(WaT + (size_t)i * hid + j);
#pragma unroll
                for (int t = 0; t < TT; ++t) hh[t] = fmaf(wv, kv[0][t][i], hh[t]);
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const Gelu gl = gelu3(hh[t]);
                av[0][t][j] = t < nt ? gl.g : 0.f;
                av[1][t][j] = gl.d1;
            }
        }
        __syncthreads();
        {                                                    // r = Wb a - v  (WbT: contiguous in i)
            const float acc = dot_hidden(-kv[1][ti][ci], WbT + ci, av[0][ti], hid, ld_nc);
            rv[ti][ci] = ti < nt ? acc : 0.f;
        }
        __syncthreads();
        if (j < hid) {                                       // e = (Wb^T r) * D, then the sums
            float bb[TT] = {0.f, 0.f, 0.f, 0.f};
            for (int i = 0; i < D; ++i) {
                const float wv = __ldg(Wb + (size_t)i * hid + j);
#pragma unroll
                for (int t = 0; t < TT; ++t) bb[t] = fmaf(wv, rv[t][i], bb[t]);
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float e = bb[t] * av[1][t][j];
                const float a = av[0][t][j];
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    ga[i] = fmaf(e, kv[0][t][i], ga[i]);
                    gb[i] = fmaf(rv[t][i], a, gb[i]);
                }
            }
        }
        __syncthreads();
    }
    (void)Wa;
    store_sums(p.part + ((size_t)u * p.nch + c) * 2 * w, hid, j, ga, gb);
}

// ---- mb_merge1: per unit, g and W1 ----------------------------------------------------------------
__global__ void mb_merge1(const Params p) {
    const int u = blockIdx.x, h = u % p.heads;
    const size_t w = (size_t)p.hid * D;
    pdl_launch_dependents();
    pdl_wait_primary();
    for (size_t e = threadIdx.x; e < 2 * w; e += blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < p.nch; ++c) acc += __ldcg(p.part + ((size_t)u * p.nch + c) * 2 * w + e);
        const float gv = p.s * acc;
        p.g[(size_t)u * 2 * w + e] = gv;
        const float w0 = (e < w) ? __ldg(p.Wa + h * w + e) : __ldg(p.Wb + h * w + (e - w));
        const float w1 = w0 - p.eta * gv;
        p.w1[(size_t)u * 3 * w + e] = w1;
        if (e < w) {                                         // Wa1^T
            const int j = (int)(e / D), i = (int)(e % D);
            p.w1[(size_t)u * 3 * w + 2 * w + (size_t)i * p.hid + j] = w1;
        }
    }
}

// ---- mb_read: dq, dWa1, dWb1 partials -------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
mb_read(const T* __restrict__ Q, const T* __restrict__ dZ, T* __restrict__ dQ, const Params p) {
    __shared__ float qz[2][TT][D];                          // q, dz
    __shared__ float hv[2][TT][HMAX];                       // aq, dhq
    const int u = blockIdx.x / p.nch, c = blockIdx.x % p.nch;
    const int j = threadIdx.x, hid = p.hid;
    const int ti = threadIdx.x / D, ci = threadIdx.x % D;
    pdl_launch_dependents();
    pdl_wait_primary();                                      // W1
    const long long off = unit_off(p, u);
    const size_t w = (size_t)hid * D;
    const float *Wa1 = p.w1 + (size_t)u * 3 * w, *Wb1 = Wa1 + w, *Wa1T = Wa1 + 2 * w;
    float da[D], db[D];
#pragma unroll
    for (int i = 0; i < D; ++i) da[i] = db[i] = 0.f;
    int n0, n1;
    chunk_range(p, c, n0, n1);
    for (int n = n0; n < n1; n += TT) {
        const int nt = min(TT, n1 - n);
        qz[0][ti][ci] = ti < nt ? ldx(Q + off + (long long)(n + ti) * D + ci) : 0.f;
        qz[1][ti][ci] = ti < nt ? ldx(dZ + off + (long long)(n + ti) * D + ci) : 0.f;
        __syncthreads();
        if (j < hid) {
            float hq[TT] = {0.f, 0.f, 0.f, 0.f}, tz[TT] = {0.f, 0.f, 0.f, 0.f};
            for (int i = 0; i < D; ++i) {
                const float wa = __ldcg(Wa1T + (size_t)i * hid + j), wb = __ldcg(Wb1 + (size_t)i * hid + j);
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    hq[t] = fmaf(wa, qz[0][t][i], hq[t]);
                    tz[t] = fmaf(wb, qz[1][t][i], tz[t]);
                }
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const Gelu gl = gelu3(hq[t]);
                const float aq = t < nt ? gl.g : 0.f, dh = t < nt ? tz[t] * gl.d1 : 0.f;
                hv[0][t][j] = aq;
                hv[1][t][j] = dh;
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    da[i] = fmaf(dh, qz[0][t][i], da[i]);
                    db[i] = fmaf(qz[1][t][i], aq, db[i]);
                }
            }
        }
        __syncthreads();
        {                                                    // dq = Wa1^T dhq  (Wa1: contiguous in i)
            const float acc = dot_hidden(0.f, Wa1 + ci, hv[1][ti], hid, ld_cg);
            if (ti < nt) stx(dQ + off + (long long)(n + ti) * D + ci, acc);
        }
        __syncthreads();
    }
    store_sums(p.part + ((size_t)u * p.nch + c) * 2 * w, hid, j, da, db);
}

// ---- mb_merge2: per unit, dgWa, dgWb and the unit's deta term -------------------------------------
__global__ void __launch_bounds__(1024) mb_merge2(const Params p) {
    __shared__ float red[1024];
    const int u = blockIdx.x;
    const size_t w = (size_t)p.hid * D;
    pdl_launch_dependents();
    pdl_wait_primary();
    float de = 0.f;
    for (size_t e = threadIdx.x; e < 2 * w; e += blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < p.nch; ++c) acc += __ldcg(p.part + ((size_t)u * p.nch + c) * 2 * w + e);
        p.dw1[(size_t)u * 2 * w + e] = acc;
        const float dgv = -p.eta * acc;
        float* dg = p.dg + (size_t)u * 4 * w;
        dg[e] = dgv;
        if (e < w) {                                         // dgWa^T
            const int j = (int)(e / D), i = (int)(e % D);
            dg[2 * w + (size_t)i * p.hid + j] = dgv;
        } else {                                             // dgWb^T
            const int i = (int)((e - w) / p.hid), j = (int)((e - w) % p.hid);
            dg[3 * w + (size_t)j * D + i] = dgv;
        }
        de -= acc * __ldcg(p.g + (size_t)u * 2 * w + e);
    }
    red[threadIdx.x] = de;
    __syncthreads();
    if (threadIdx.x == 0) {                                  // threads in order
        float acc = 0.f;
        for (int t = 0; t < (int)blockDim.x; ++t) acc += red[t];
        p.deta_u[u] = acc;
    }
}

// ---- mb_upd: the update path per key token ---------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
mb_upd(const T* __restrict__ K, const T* __restrict__ V, T* __restrict__ dK, T* __restrict__ dV, const Params p) {
    __shared__ float kv[2][TT][D];                          // k, v
    __shared__ float av[6][TT][HMAX];                       // a, D, e, db, dh, (b)
    __shared__ float rv[2][TT][D];                          // r, dr
    const int u = blockIdx.x / p.nch, c = blockIdx.x % p.nch, h = u % p.heads;
    const int j = threadIdx.x, hid = p.hid;
    const int ti = threadIdx.x / D, ci = threadIdx.x % D;
    pdl_launch_dependents();
    pdl_wait_primary();                                      // dgWa, dgWb
    const long long off = unit_off(p, u);
    const size_t w = (size_t)hid * D;
    const float *Wa = p.Wa + h * w, *Wb = p.Wb + h * w, *WaT = p.WaT + h * w, *WbT = p.WbT + h * w;
    const float* dgb = p.dg + (size_t)u * 4 * w;
    const float *dgA = dgb, *dgB = dgb + w, *dgAT = dgb + 2 * w, *dgBT = dgb + 3 * w;
    const float s = p.s;
    float sa[D], sb[D];
#pragma unroll
    for (int i = 0; i < D; ++i) sa[i] = sb[i] = 0.f;
    int n0, n1;
    chunk_range(p, c, n0, n1);
    for (int n = n0; n < n1; n += TT) {
        const int nt = min(TT, n1 - n);
        kv[0][ti][ci] = ti < nt ? ldx(K + off + (long long)(n + ti) * D + ci) : 0.f;
        kv[1][ti][ci] = ti < nt ? ldx(V + off + (long long)(n + ti) * D + ci) : 0.f;
        __syncthreads();
        float hh[TT] = {0.f, 0.f, 0.f, 0.f}, d2[TT];
        if (j < hid) {                                       // h = Wa k; a, D
            for (int i = 0; i < D; ++i) {
                const float wv = __ldg(WaT + (size_t)i * hid + j);
#pragma unroll
                for (int t = 0; t < TT; ++t) hh[t] = fmaf(wv, kv[0][t][i], hh[t]);
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const Gelu gl = gelu3(hh[t]);
                av[0][t][j] = t < nt ? gl.g : 0.f;
                av[1][t][j] = gl.d1;
                d2[t] = gl.d2;
            }
        }
        __syncthreads();
        {                                                    // r = Wb a - v
            const float acc = dot_hidden(-kv[1][ti][ci], WbT + ci, av[0][ti], hid, ld_nc);
            rv[0][ti][ci] = ti < nt ? acc : 0.f;
        }
        __syncthreads();
        float dD[TT];
        if (j < hid) {                                       // b = Wb^T r, e = b D, de = s dgWa k, db, dD
            float bb[TT] = {0.f, 0.f, 0.f, 0.f}, dd[TT] = {0.f, 0.f, 0.f, 0.f};
            for (int i = 0; i < D; ++i) {
                const float wv = __ldg(Wb + (size_t)i * hid + j), gv = __ldcg(dgAT + (size_t)i * hid + j);
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    bb[t] = fmaf(wv, rv[0][t][i], bb[t]);
                    dd[t] = fmaf(gv, kv[0][t][i], dd[t]);
                }
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float Dv = av[1][t][j], de = s * dd[t];
                av[2][t][j] = bb[t] * Dv;                    // e
                av[3][t][j] = t < nt ? de * Dv : 0.f;        // db
                dD[t] = de * bb[t];
            }
        }
        __syncthreads();
        {                                                    // dr = s dgWb a + Wb db
            const float acc = dot_hidden2(s, dgBT + ci, av[0][ti], ld_cg, WbT + ci, av[3][ti], ld_nc, hid);
            rv[1][ti][ci] = ti < nt ? acc : 0.f;
            if (ti < nt) stx(dV + off + (long long)(n + ti) * D + ci, -acc);
        }
        __syncthreads();
        if (j < hid) {                                       // da = s dgWb^T r + Wb^T dr; dh; the sums
            float da[TT] = {0.f, 0.f, 0.f, 0.f};
            for (int i = 0; i < D; ++i) {
                const float gv = __ldcg(dgB + (size_t)i * hid + j), wv = __ldg(Wb + (size_t)i * hid + j);
#pragma unroll
                for (int t = 0; t < TT; ++t) da[t] = fmaf(s * gv, rv[0][t][i], fmaf(wv, rv[1][t][i], da[t]));
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float dh = t < nt ? da[t] * av[1][t][j] + dD[t] * d2[t] : 0.f;
                av[4][t][j] = dh;
                const float a = av[0][t][j], dbv = av[3][t][j];
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    sa[i] = fmaf(dh, kv[0][t][i], sa[i]);
                    sb[i] = fmaf(rv[1][t][i], a, fmaf(rv[0][t][i], dbv, sb[i]));
                }
            }
        }
        __syncthreads();
        {                                                    // dk = s dgWa^T e + Wa^T dh
            const float acc = dot_hidden2(s, dgA + ci, av[2][ti], ld_cg, Wa + ci, av[4][ti], ld_nc, hid);
            if (ti < nt) stx(dK + off + (long long)(n + ti) * D + ci, acc);
        }
        __syncthreads();
    }
    store_sums(p.upd + ((size_t)u * p.nch + c) * 2 * w, hid, j, sa, sb);
}

// ---- mb_final: per head, dWa and dWb; block 0 also deta -------------------------------------------
__global__ void mb_final(const Params p) {
    const int h = blockIdx.x;
    const size_t w = (size_t)p.hid * D;
    const int B = p.U / p.heads;
    pdl_wait_primary();
    for (size_t e = (size_t)blockIdx.y * blockDim.x + threadIdx.x; e < 2 * w; e += (size_t)gridDim.y * blockDim.x) {
        // images in order: per image dW1, then the image's chunk partials in order
        const float acc = nested_sum_in_order(
            B, p.nch, [&](int b) { return p.dw1 + (size_t)(b * p.heads + h) * 2 * w + e; },
            [&](int b, int c) { return p.upd + ((size_t)(b * p.heads + h) * p.nch + c) * 2 * w + e; });
        if (e < w) { if (p.dWa_out) p.dWa_out[h * w + e] = acc; }
        else if (p.dWb_out) p.dWb_out[h * w + (e - w)] = acc;
    }
    if (h == 0 && blockIdx.y == 0 && threadIdx.x == 0 && p.deta_out) {
        float acc = 0.f;
        for (int u = 0; u < p.U; ++u) acc += __ldcg(p.deta_u + u);
        *p.deta_out = acc;
    }
}

struct WsLayout {
    size_t WaT, WbT, part, g, w1, dg, dw1, upd, deta, total;
};
static int chunks_for(long long U, int N) {
    return (int)std::max<long long>(1, std::min<long long>((N + 63) / 64, (256 + U - 1) / U));
}
static WsLayout ws_layout(const ttt_shape& s) {
    const long long U = (long long)s.batch * s.heads;
    const size_t w = (size_t)s.hidden * D * 4;
    const int nch = chunks_for(U, s.H * s.W);
    WsLayout L;
    L.WaT = kWsHeader;
    L.WbT = align_up(L.WaT + (size_t)s.heads * w, 256);
    L.part = align_up(L.WbT + (size_t)s.heads * w, 256);
    L.g = align_up(L.part + (size_t)U * nch * 2 * w, 256);
    L.w1 = align_up(L.g + (size_t)U * 2 * w, 256);
    L.dg = align_up(L.w1 + (size_t)U * 3 * w, 256);
    L.dw1 = align_up(L.dg + (size_t)U * 4 * w, 256);
    L.upd = align_up(L.dw1 + (size_t)U * 2 * w, 256);
    L.deta = align_up(L.upd + (size_t)U * nch * 2 * w, 256);
    L.total = L.deta + (size_t)U * 4;
    return L;
}

template <typename T>
static ttt_status launch(const Call& c, const ttt_shape& sh, const void* dZ, void* dQ, void* dK, void* dV,
                         float* dWa_out, float* dWb_out, float* deta_out) {
    const WsLayout L = ws_layout(sh);
    if (c.ws_bytes < L.total) return TTT_ERR_WORKSPACE;
    Params p{};
    p.heads = c.heads; p.N = c.N; p.hid = c.hidden;
    p.U = c.batch * c.heads;
    p.nch = chunks_for(p.U, c.N);
    p.bs = c.bs; p.hs = c.hs;
    p.eta = c.eta; p.s = 2.0f / (float)c.N;
    p.Wa = c.W0; p.Wb = c.W0b;
    p.WaT = reinterpret_cast<float*>(c.ws + L.WaT);
    p.WbT = reinterpret_cast<float*>(c.ws + L.WbT);
    p.part = reinterpret_cast<float*>(c.ws + L.part);
    p.g = reinterpret_cast<float*>(c.ws + L.g);
    p.w1 = reinterpret_cast<float*>(c.ws + L.w1);
    p.dg = reinterpret_cast<float*>(c.ws + L.dg);
    p.dw1 = reinterpret_cast<float*>(c.ws + L.dw1);
    p.upd = reinterpret_cast<float*>(c.ws + L.upd);
    p.deta_u = reinterpret_cast<float*>(c.ws + L.deta);
    p.dWa_out = dWa_out; p.dWb_out = dWb_out; p.deta_out = deta_out;
    const T *Q = static_cast<const T*>(c.Q), *K = static_cast<const T*>(c.K), *V = static_cast<const T*>(c.V);
    const T* dz = static_cast<const T*>(dZ);
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.blockDim = dim3(kThreads);
    cfg.gridDim = dim3(std::max(1, std::min(c.num_sms, (int)((c.heads * (size_t)c.hidden * D + 255) / 256))));
    cfg.numAttrs = 0;
    ttt_status st = check_launch(cudaLaunchKernelEx(&cfg, mb_prep, p));
    cfg.numAttrs = 1;
    const dim3 chunks((unsigned)(p.U * p.nch)), units((unsigned)p.U);
    if (st == TTT_OK) { cfg.gridDim = chunks; st = check_launch(cudaLaunchKernelEx(&cfg, mb_fwd<T>, K, V, p)); }
    if (st == TTT_OK) { cfg.gridDim = units; st = check_launch(cudaLaunchKernelEx(&cfg, mb_merge1, p)); }
    if (st == TTT_OK) {
        cfg.gridDim = chunks;
        st = check_launch(cudaLaunchKernelEx(&cfg, mb_read<T>, Q, dz, static_cast<T*>(dQ), p));
    }
    if (st == TTT_OK) { cfg.gridDim = units; cfg.blockDim = dim3(1024); st = check_launch(cudaLaunchKernelEx(&cfg, mb_merge2, p)); }
    if (st == TTT_OK) {
        cfg.gridDim = chunks;
        cfg.blockDim = dim3(kThreads);
        st = check_launch(cudaLaunchKernelEx(&cfg, mb_upd<T>, K, V, static_cast<T*>(dK), static_cast<T*>(dV), p));
    }
    if (st == TTT_OK) {                                     // per head, the 2 hidden x d elements over 32 CTAs
        cfg.gridDim = dim3((unsigned)c.heads, 32u);
        st = check_launch(cudaLaunchKernelEx(&cfg, mb_final, p));
    }
    return st;
}

}  // namespace mb2

size_t mlp_backward_ws_bytes(const ttt_shape& s) { return mb2::ws_layout(s).total; }

ttt_status launch_mlp_backward(const Call& c, const ttt_shape& s, const void* dZ, void* dQ, void* dK, void* dV,
                               float* dWa_out, float* dWb_out, float* deta_out) {
    if (c.loss != TTT_LOSS_L2 || c.hidden > mb2::HMAX) return TTT_ERR_UNSUPPORTED;
    if (c.dtype == TTT_BF16) return mb2::launch<__nv_bfloat16>(c, s, dZ, dQ, dK, dV, dWa_out, dWb_out, deta_out);
    return mb2::launch<float>(c, s, dZ, dQ, dK, dV, dWa_out, dWb_out, deta_out);
}

}  // namespace ttt
