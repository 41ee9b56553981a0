// backward_conv.cu -- backward pass of the 3x3 depthwise-convolution head (press article "CVPR 2026
// Oral | 清華+阿里發布ViT3", Observation 1: the layer is trained end to end, the outer gradient flowing
// through the inner step; the head itself: Observation 6, Fig. 5 part 3).  Per channel c, taps t with
// grid shifts s_t = (a-1, b-1), K zero outside the grid, and the forward
//     r_p = sum_t W0_t K_{p+s_t} - V_p,   g_t = (2/N) sum_p r_p K_{p+s_t},   W1 = W0 - eta g,
//     Z_p = sum_t W1_t Q_{p+s_t},
// the chain rule for the upstream gradient dZ gives, with dg = -eta dW1:
//     dW1_t = sum_p dZ_p Q_{p+s_t},          dQ_q = sum_t W1_t dZ_{q-s_t},
//     dr_p = (2/N) sum_t dg_t K_{p+s_t},     dV_p = -dr_p,
//     dK_q = (2/N) sum_t dg_t r_{q-s_t} + sum_t W0_t dr_{q-s_t},
//     dW0_t = dW1_t + sum_p dr_p K_{p+s_t},  deta = -sum_t dW1_t g_t
// (positions q - s_t outside the grid contribute nothing).  W0 and eta are shared by every unit:
// dW0 is summed over the images of each head and deta over every unit, in index order.
//
// Not a contraction (no sharing across channels): fp32 FMA, lane l of a warp owning channels 2l and
// 2l+1, a 3 x 3 register window sliding along a grid row.  Four kernels on one stream, each a
// programmatic dependent of the one before; every sum has a fixed order, so the results are bitwise
// reproducible.  Positions are taken in tiles of 8 grid rows x 16 columns (warp w: row w of a tile).
// Each tile's inputs (with the margins its taps reach) are first staged in shared memory with all of
// their loads in flight, so that the per-position loops read no global memory.
//   cb_reduce    per tile: the partial sums sum_p r_p K_{p+s_t} and sum_p dZ_p Q_{p+s_t} (2 x 64 x 9)
//   cb_unit      per unit: the tile partials summed in tile order -> g, W1, dg, dW1 and the unit's
//                deta term
//   cb_map       per tile: r and dr on the tile and a one-position halo (shared memory), then dQ, dK,
//                dV for the tile's positions and the tile's partial sum_p dr_p K_{p+s_t}
//   cb_final     per (head, tap): dW0 = sum over images of (dW1 + the unit's map partials in tile
//                order), the images' terms formed in parallel; block 0 also sums deta over the units
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace cb {

constexpr int D = 64;
constexpr int TAPS = 9;
constexpr int kPart = D * TAPS;              // 576: one 64 x 9 sum, tap-major
constexpr int TR = 8, TC = 16;               // a tile: 8 rows x 16 columns
constexpr int HR = TR + 2, HC = TC + 2;      // the tile with a one-position halo
constexpr int kThreads = TR * 32;            // warp w: tile row w

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float2 ld(const __nv_bfloat16* p) {
        const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p));
        return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
    }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float2 v) {
        *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v.x, v.y);
    }
};
template <>
struct Elem<float> {
    static __device__ __forceinline__ float2 ld(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
    static __device__ __forceinline__ void st(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
};

struct Geo {
    int heads, H, W, N;
    int tiles_x, tpu;                        // tiles along x, per unit
    long long bs, hs;                        // element strides of Q/K/V/dZ and of the outputs
    int U;
    float eta, scale;                        // eta, 2/N
};

struct Params {
    Geo g;
    const float* W0;                         // [heads][64][9]
    float* red;                              // [U][tpu][2][576]: sum r K_t, sum dZ Q_t per tile
    float* coef;                             // [U][3][576]: W1, dg, dW1 per unit
    float* deta_u;                           // [U]
    float* mapp;                             // [U][tpu][576]: sum dr K_t per tile
    float* dW0_out;                          // nullable [heads][64][9]
    float* deta_out;                         // nullable, one float
};

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return ffma2(a, b, c); }

// Channel pair `lane` of X at grid position (y, x) of the unit at `base`; zero outside the grid.
template <typename T>
__device__ __forceinline__ float2 at(const T* base, const Geo& g, int y, int x, int lane) {
    if (y < 0 || y >= g.H || x < 0 || x >= g.W) return make_float2(0.f, 0.f);
    return Elem<T>::ld(base + ((long long)y * g.W + x) * D + 2 * lane);
}

__device__ __forceinline__ long long unit_off(const Geo& g, int u) {
    return (long long)(u / g.heads) * g.bs + (long long)(u % g.heads) * g.hs;
}

// The positions (y0 - MR .. y0 + TR - 1 + MR) x (x0 - MR .. x0 + TC - 1 + MR) of one unit's X, staged in
// shared memory as rows of 64 channels (zero outside the grid), with all of the 16-byte loads in
// flight before any is stored.
template <typename T, int MR>
__device__ __forceinline__ void stage_halo(T* dst, const T* base, const Geo& g, int y0, int x0) {
    constexpr int RW = TC + 2 * MR, CH = D * (int)sizeof(T) / 16;
    constexpr int TOT = (TR + 2 * MR) * RW * CH, PER = (TOT + kThreads - 1) / kThreads;
    uint4 v[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const int e = threadIdx.x + k * kThreads, pos = e / CH, ch = e % CH;
        const int y = y0 - MR + pos / RW, x = x0 - MR + pos % RW;
        v[k] = (e < TOT && y >= 0 && y < g.H && x >= 0 && x < g.W)
                   ? __ldg(reinterpret_cast<const uint4*>(base + ((long long)y * g.W + x) * D) + ch)
                   : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const int e = threadIdx.x + k * kThreads;
        if (e < TOT) reinterpret_cast<uint4*>(dst)[e] = v[k];
    }
}
// Channel pair `lane` at staged row r, column c of a region RW positions wide.
template <typename T>
__device__ __forceinline__ float2 sat(const T* st, int RW, int r, int c, int lane);
template <>
__device__ __forceinline__ float2 sat<__nv_bfloat16>(const __nv_bfloat16* st, int RW, int r, int c, int lane) {
    const uint32_t w = reinterpret_cast<const uint32_t*>(st + (r * RW + c) * D)[lane];
    return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
}
template <>
__device__ __forceinline__ float2 sat<float>(const float* st, int RW, int r, int c, int lane) {
    return reinterpret_cast<const float2*>(st + (r * RW + c) * D)[lane];
}
constexpr int KRW = TC + 4, ZRW = TC + 2;    // staged K (two-position margin), staged dZ (one)
constexpr int kMaxFinalImages = 64;          // images whose terms cb_final holds at a time

// ---- cb_reduce: one CTA per tile -----------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
cb_reduce(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ dZ,
          const Params p) {
    extern __shared__ uint8_t smem_raw[];
    float (*red)[2][kPart] = reinterpret_cast<float (*)[2][kPart]>(smem_raw);   // [TR][2][576]
    T* ks = reinterpret_cast<T*>(smem_raw + sizeof(float) * TR * 2 * kPart);    // [TR+2][TC+2][64] K
    T* qs = ks + (TR + 2) * ZRW * D;                                            // [TR+2][TC+2][64] Q
    T* vs = qs + (TR + 2) * ZRW * D;                                            // [TR][TC][64] V
    T* zs = vs + TR * TC * D;                                                   // [TR][TC][64] dZ
    const Geo& g = p.g;
    const int u = blockIdx.x / g.tpu, i = blockIdx.x % g.tpu;
    const int h = u % g.heads;
    const int x0 = (i % g.tiles_x) * TC, y0 = (i / g.tiles_x) * TR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    const long long off = unit_off(g, u);
    const T *Ku = K + off, *Vu = V + off, *Qu = Q + off, *dZu = dZ + off;
    stage_halo<T, 1>(ks, Ku, g, y0, x0);
    stage_halo<T, 1>(qs, Qu, g, y0, x0);
    stage_halo<T, 0>(vs, Vu, g, y0, x0);
    stage_halo<T, 0>(zs, dZu, g, y0, x0);
    __syncthreads();
    float2 w0[TAPS], sk[TAPS], zq[TAPS];
#pragma unroll
    for (int t = 0; t < TAPS; ++t) {
        w0[t] = make_float2(__ldg(p.W0 + ((size_t)h * D + 2 * lane) * TAPS + t),
                            __ldg(p.W0 + ((size_t)h * D + 2 * lane + 1) * TAPS + t));
        sk[t] = zq[t] = make_float2(0.f, 0.f);
    }
    const int y = y0 + warp;
    if (y < g.H) {
        const int xe = min(g.W, x0 + TC);
        float2 kw[3][3], qw[3][3];                           // [tap row][column x-1, x, x+1]
#pragma unroll
        for (int a = 0; a < 3; ++a) {                        // staged row warp + a is grid row y + a - 1
            kw[a][0] = sat<T>(ks, ZRW, warp + a, 0, lane); kw[a][1] = sat<T>(ks, ZRW, warp + a, 1, lane);
            qw[a][0] = sat<T>(qs, ZRW, warp + a, 0, lane); qw[a][1] = sat<T>(qs, ZRW, warp + a, 1, lane);
        }
        for (int x = x0; x < xe; ++x) {
#pragma unroll
            for (int a = 0; a < 3; ++a) {
                kw[a][2] = sat<T>(ks, ZRW, warp + a, x - x0 + 2, lane);
                qw[a][2] = sat<T>(qs, ZRW, warp + a, x - x0 + 2, lane);
            }
            const float2 v = sat<T>(vs, TC, warp, x - x0, lane), dz = sat<T>(zs, TC, warp, x - x0, lane);
            float2 r = make_float2(-v.x, -v.y);
#pragma unroll
            for (int t = 0; t < TAPS; ++t) r = fma2(w0[t], kw[t / 3][t % 3], r);
#pragma unroll
            for (int t = 0; t < TAPS; ++t) {
                sk[t] = fma2(r, kw[t / 3][t % 3], sk[t]);
                zq[t] = fma2(dz, qw[t / 3][t % 3], zq[t]);
            }
#pragma unroll
            for (int a = 0; a < 3; ++a) {
                kw[a][0] = kw[a][1]; kw[a][1] = kw[a][2];
                qw[a][0] = qw[a][1]; qw[a][1] = qw[a][2];
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TAPS; ++t) {
        *reinterpret_cast<float2*>(&red[warp][0][t * D + 2 * lane]) = sk[t];
        *reinterpret_cast<float2*>(&red[warp][1][t * D + 2 * lane]) = zq[t];
    }
    __syncthreads();
    float* dst = p.red + ((size_t)u * g.tpu + i) * 2 * kPart;
    for (int e = threadIdx.x; e < 2 * kPart; e += kThreads) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < TR; ++w) acc += (&red[w][0][0])[e];   // rows in order
        dst[e] = acc;
    }
}

// ---- cb_unit: one CTA per unit -------------------------------------------------------------------
__global__ void __launch_bounds__(kPart)
cb_unit(const Params p) {
    __shared__ float part[kPart];
    const Geo& g = p.g;
    const int u = blockIdx.x, e = threadIdx.x;                // e: tap-major (t, c)
    const int t = e / D, c = e % D, h = u % g.heads;
    pdl_launch_dependents();
    pdl_wait_primary();                                       // every tile partial is written
    const float* src = p.red + (size_t)u * g.tpu * 2 * kPart;
    const float sk = add_strided_in_order(0.f, src + e, 2 * kPart, g.tpu);
    const float zq = add_strided_in_order(0.f, src + kPart + e, 2 * kPart, g.tpu);
    const float w0 = __ldg(p.W0 + ((size_t)h * D + c) * TAPS + t);
    const float gr = g.scale * sk;                            // g_t = (2/N) sum r K_t
    float* cf = p.coef + (size_t)u * 3 * kPart;
    cf[e] = w0 - g.eta * gr;                                  // W1
    cf[kPart + e] = -g.eta * zq;                              // dg
    cf[2 * kPart + e] = zq;                                   // dW1
    part[e] = -zq * gr;
    __syncthreads();
    if (e == 0) {                                             // the unit's deta term, in element order
        float acc = 0.f;
        for (int j = 0; j < kPart; ++j) acc += part[j];
        p.deta_u[u] = acc;
    }
}

// ---- cb_map: one CTA per tile --------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
cb_map(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ dZ, T* __restrict__ dQ,
       T* __restrict__ dK, T* __restrict__ dV, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    float2* rs = reinterpret_cast<float2*>(smem_raw);          // [HR*HC][32] r at the halo tile
    float2* drs = rs + HR * HC * 32;                           // [HR*HC][32] dr
    float* red = reinterpret_cast<float*>(drs + HR * HC * 32); // [TR][576]
    T* ks = reinterpret_cast<T*>(red + TR * kPart);            // [TR+4][TC+4][64] K
    T* zs = ks + (TR + 4) * KRW * D;                           // [TR+2][TC+2][64] dZ
    const Geo& g = p.g;
    const int u = blockIdx.x / g.tpu, i = blockIdx.x % g.tpu;
    const int h = u % g.heads;
    const int x0 = (i % g.tiles_x) * TC, y0 = (i / g.tiles_x) * TR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    const long long off = unit_off(g, u);
    const T *Ku = K + off, *Vu = V + off, *dZu = dZ + off;
    stage_halo<T, 2>(ks, Ku, g, y0, x0);                      // inputs: loaded before the wait
    stage_halo<T, 1>(zs, dZu, g, y0, x0);
    float2 w0[TAPS];
#pragma unroll
    for (int t = 0; t < TAPS; ++t)
        w0[t] = make_float2(__ldg(p.W0 + ((size_t)h * D + 2 * lane) * TAPS + t),
                            __ldg(p.W0 + ((size_t)h * D + 2 * lane + 1) * TAPS + t));
    __syncthreads();
    pdl_wait_primary();                                       // W1, dg of the unit are formed
    const float* cf = p.coef + (size_t)u * 3 * kPart;
    float2 w1[TAPS], dgs[TAPS];                               // dgs = (2/N) dg
#pragma unroll
    for (int t = 0; t < TAPS; ++t) {
        w1[t] = __ldcg(reinterpret_cast<const float2*>(cf + t * D) + lane);
        const float2 dg = __ldcg(reinterpret_cast<const float2*>(cf + kPart + t * D) + lane);
        dgs[t] = make_float2(g.scale * dg.x, g.scale * dg.y);
    }
    // (1) r and dr at the tile and its halo (zero outside the grid); V six positions at a time, all
    //     six loads in flight
    for (int hr = warp; hr < HR; hr += TR) {
        const int y = y0 - 1 + hr;
        for (int hc0 = 0; hc0 < HC; hc0 += 6) {
            float2 v[6];
#pragma unroll
            for (int q = 0; q < 6; ++q) v[q] = at(Vu, g, y, x0 - 1 + hc0 + q, lane);
#pragma unroll
            for (int q = 0; q < 6; ++q) {
                const int hc = hc0 + q, x = x0 - 1 + hc;
                float2 r = make_float2(0.f, 0.f), dr = make_float2(0.f, 0.f);
                if (y >= 0 && y < g.H && x >= 0 && x < g.W) {
                    r = make_float2(-v[q].x, -v[q].y);
#pragma unroll
                    for (int t = 0; t < TAPS; ++t) {
                        const float2 k = sat<T>(ks, KRW, hr + t / 3, hc + t % 3, lane);
                        r = fma2(w0[t], k, r);
                        dr = fma2(dgs[t], k, dr);
                    }
                }
                rs[(hr * HC + hc) * 32 + lane] = r;
                drs[(hr * HC + hc) * 32 + lane] = dr;
            }
        }
    }
    __syncthreads();
    // (2) the tile's positions: dQ, dK, dV and sum dr K_t
    float2 acc[TAPS];
#pragma unroll
    for (int t = 0; t < TAPS; ++t) acc[t] = make_float2(0.f, 0.f);
    const int y = y0 + warp;
    if (y < g.H) {
        const int xe = min(g.W, x0 + TC);
        for (int x = x0; x < xe; ++x) {
            const int hr = warp + 1, hc = x - x0 + 1;          // this position in the halo tile
            float2 aq = make_float2(0.f, 0.f), ak = make_float2(0.f, 0.f);
#pragma unroll
            for (int t = 0; t < TAPS; ++t) {
                const int ay = t / 3 - 1, bx = t % 3 - 1;      // q - s_t
                aq = fma2(w1[t], sat<T>(zs, ZRW, warp + 1 - ay, x - x0 + 1 - bx, lane), aq);
                const int hidx = ((hr - ay) * HC + (hc - bx)) * 32 + lane;
                ak = fma2(dgs[t], rs[hidx], ak);
                ak = fma2(w0[t], drs[hidx], ak);
            }
            const float2 dr = drs[(hr * HC + hc) * 32 + lane];
#pragma unroll
            for (int t = 0; t < TAPS; ++t) acc[t] = fma2(dr, sat<T>(ks, KRW, warp + 1 + t / 3, x - x0 + 1 + t % 3, lane), acc[t]);
            const long long o = ((long long)y * g.W + x) * D + 2 * lane;
            Elem<T>::st(dQ + off + o, aq);
            Elem<T>::st(dK + off + o, ak);
            Elem<T>::st(dV + off + o, make_float2(-dr.x, -dr.y));
        }
    }
#pragma unroll
    for (int t = 0; t < TAPS; ++t) *reinterpret_cast<float2*>(&red[warp * kPart + t * D + 2 * lane]) = acc[t];
    __syncthreads();
    float* dst = p.mapp + ((size_t)u * g.tpu + i) * kPart;
    for (int e = threadIdx.x; e < kPart; e += kThreads) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < TR; ++w) a += red[w * kPart + e];
        dst[e] = a;
    }
}

// ---- cb_final: per (head, tap) 64 channels; block 0 also sums deta ---------------------------------
// dW0 = sum over images in order of (dW1 + the unit's tile partials in tile order).  Thread (c, b0)
// forms the per-image terms of images b0, b0 + 8, ... (each with its tile loads in flight), then
// thread c adds the images' terms in image order: the same sums, in the same order, as one thread
// walking the images.
constexpr int kFinalLanes = 8;
__global__ void __launch_bounds__(D * kFinalLanes)
cb_final(const Params p) {
    const Geo& g = p.g;
    __shared__ float img[kMaxFinalImages][D];
    __shared__ float dterms[kFinalLanes * D];
    const int h = blockIdx.x / TAPS, t = blockIdx.x % TAPS;
    const int c = threadIdx.x % D, b0 = threadIdx.x / D, e = t * D + c;
    pdl_wait_primary();
    const int B = g.U / g.heads;
    if (p.dW0_out) {
        for (int bc = 0; bc < B; bc += kMaxFinalImages) {
            const int nb = min(kMaxFinalImages, B - bc);
            for (int b = b0; b < nb; b += kFinalLanes) {
                const int u = (bc + b) * g.heads + h;
                img[b][c] = add_strided_in_order(__ldcg(p.coef + (size_t)u * 3 * kPart + 2 * kPart + e),   // dW1
                                                 p.mapp + (size_t)u * g.tpu * kPart + e, kPart, g.tpu);
            }
            __syncthreads();
            if (b0 == 0) {
                float acc = (bc == 0) ? 0.f : p.dW0_out[((size_t)h * D + c) * TAPS + t];
                for (int b = 0; b < nb; ++b) acc += img[b][c];
                p.dW0_out[((size_t)h * D + c) * TAPS + t] = acc;
            }
            __syncthreads();
        }
    }
    if (blockIdx.x == 0 && p.deta_out) {
        // the units' terms loaded by the whole block, summed in unit order
        float acc = 0.f;
        for (int u0 = 0; u0 < g.U; u0 += kFinalLanes * D) {
            const int n = min(kFinalLanes * D, g.U - u0);
            __syncthreads();
            if ((int)threadIdx.x < n) dterms[threadIdx.x] = __ldcg(p.deta_u + u0 + threadIdx.x);
            __syncthreads();
            if (threadIdx.x == 0)
                for (int k = 0; k < n; ++k) acc += dterms[k];
        }
        if (threadIdx.x == 0) *p.deta_out = acc;
    }
}

struct WsLayout {
    size_t red, coef, deta, mapp, total;
};
static WsLayout ws_layout(long long U, long long tpu) {
    WsLayout L;
    L.red = kWsHeader;
    L.coef = align_up(L.red + (size_t)U * tpu * 2 * kPart * 4, 256);
    L.deta = align_up(L.coef + (size_t)U * 3 * kPart * 4, 256);
    L.mapp = align_up(L.deta + (size_t)U * 4, 256);
    L.total = L.mapp + (size_t)U * tpu * kPart * 4;
    return L;
}

static long long tiles_per_unit(int H, int W) { return (long long)((W + TC - 1) / TC) * ((H + TR - 1) / TR); }

template <typename T>
static ttt_status launch(const Call& c, const void* dZ, void* dQ, void* dK, void* dV, float* dW0_out,
                         float* deta_out) {
    const long long U = (long long)c.batch * c.heads;
    const long long tpu = tiles_per_unit(c.H, c.W);
    if (U * tpu > (1LL << 31) - 1) return TTT_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(U, tpu);
    if (c.ws_bytes < L.total) return TTT_ERR_WORKSPACE;
    Params p{};
    p.g.heads = c.heads; p.g.H = c.H; p.g.W = c.W; p.g.N = c.N;
    p.g.tiles_x = (c.W + TC - 1) / TC;
    p.g.tpu = (int)tpu;
    p.g.bs = c.bs; p.g.hs = c.hs;
    p.g.U = (int)U;
    p.g.eta = c.eta;
    p.g.scale = 2.0f / (float)c.N;
    p.W0 = c.W0;
    p.red = reinterpret_cast<float*>(c.ws + L.red);
    p.coef = reinterpret_cast<float*>(c.ws + L.coef);
    p.deta_u = reinterpret_cast<float*>(c.ws + L.deta);
    p.mapp = reinterpret_cast<float*>(c.ws + L.mapp);
    p.dW0_out = dW0_out;
    p.deta_out = deta_out;
    const T *Q = static_cast<const T*>(c.Q), *K = static_cast<const T*>(c.K), *V = static_cast<const T*>(c.V);
    const T* dz = static_cast<const T*>(dZ);
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.gridDim = dim3((unsigned)(U * tpu));
    cfg.blockDim = dim3(kThreads);
    cfg.numAttrs = 0;
    const size_t smem_r = sizeof(float) * TR * 2 * kPart + ((size_t)2 * (TR + 2) * ZRW + 2 * TR * TC) * D * sizeof(T);
    cudaFuncSetAttribute(cb_reduce<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_r);
    cfg.dynamicSmemBytes = smem_r;
    ttt_status st = check_launch(cudaLaunchKernelEx(&cfg, cb_reduce<T>, Q, K, V, dz, p));
    if (st != TTT_OK) return st;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)U);
    cfg.blockDim = dim3(kPart);
    cfg.dynamicSmemBytes = 0;
    st = check_launch(cudaLaunchKernelEx(&cfg, cb_unit, p));
    if (st != TTT_OK) return st;
    const size_t smem = (size_t)2 * HR * HC * 32 * sizeof(float2) + (size_t)TR * kPart * sizeof(float) +
                        ((size_t)(TR + 4) * KRW + (size_t)(TR + 2) * ZRW) * D * sizeof(T);
    cudaFuncSetAttribute(cb_map<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cfg.gridDim = dim3((unsigned)(U * tpu));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    st = check_launch(cudaLaunchKernelEx(&cfg, cb_map<T>, K, V, dz, static_cast<T*>(dQ), static_cast<T*>(dK),
                                         static_cast<T*>(dV), p));
    if (st != TTT_OK) return st;
    cfg.gridDim = dim3((unsigned)(c.heads * TAPS));
    cfg.blockDim = dim3(D * kFinalLanes);
    cfg.dynamicSmemBytes = 0;
    return check_launch(cudaLaunchKernelEx(&cfg, cb_final, p));
}

}  // namespace cb

size_t dwconv_backward_ws_bytes(const ttt_shape& s) {
    const long long U = (long long)s.batch * s.heads;
    return cb::ws_layout(U, cb::tiles_per_unit(s.H, s.W)).total;
}

ttt_status launch_dwconv_backward(const Call& c, const void* dZ, void* dQ, void* dK, void* dV, float* dW0_out,
                                  float* deta_out) {
    if (c.loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    if (c.dtype == TTT_BF16) return cb::launch<__nv_bfloat16>(c, dZ, dQ, dK, dV, dW0_out, deta_out);
    return cb::launch<float>(c, dZ, dQ, dK, dV, dW0_out, deta_out);
}

}  // namespace ttt
