// backward.cu -- backward pass of the full-batch linear head (L2 loss), the outer gradient that the
// press article "CVPR 2026 Oral | 清華+阿里發布ViT3" (Observation 1) trains the layer with: the
// gradient flows through the inner update.  With s = 2 eta / N and the forward
//     G = sum k k^T,  C = sum v k^T,  W1 = W0 - s (W0 G - C),  z = W1 q,
// the upstream gradient dZ gives
//     dW1 = sum dz q^T,   dq = W1^T dz,   dC = s dW1,   dG = -s W0^T dW1,
//     dv = dC k,   dk = dC^T v + (dG + dG^T) k,   dW0 = dW1 (I - s G),
//     deta = -(2/N) sum_ij dW1_ij (W0 G - C)_ij,
// dW0 summed over the images of each head and deta over every unit.
//
// Three kernels, plain fp32 FMA (a first, exact-arithmetic path; the contractions are the same
// shapes as the forward's, so the tensor-core route of the forward applies to them):
//   lin_bwd_p1  static partition of 128-token tiles over CTAs; each CTA accumulates its share of
//               [G ; C ; dW1] (192 x 64) and writes it to a partial slot; the CTA that completes a
//               unit sums the unit's slots in slot order (deterministic) and forms W1, dC, dC^T,
//               dG + dG^T, the unit's dW0 and deta.
//   lin_bwd_p2  one CTA per 32 tokens (a programmatic dependent of p1): the four 64 x 64 matrices and
//               the tokens' dz, k, v rows in shared memory; 8 lanes per token compute its dq, dk, dv.
// The lanes that share a row of outputs take interleaved groups of 4 columns, so that their float4
// reads of shared memory are contiguous (no bank conflicts), and both kernels keep their shared
// memory under half an SM's, so that two CTAs share every SM.
//   lin_bwd_sum dW0 over images and deta over units, in index order.
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace bwd {

constexpr int D = 64;
constexpr int TOK = 128;                     // tokens per tile
constexpr int CHUNK = 32;                    // tokens staged in shared memory at a time (p1)
constexpr int P1_THREADS = 384;              // (row of [G ; C ; dW1], one of 2 interleaved column sets)
constexpr int P2_TOK = 32;                   // tokens per phase-2 CTA
constexpr int P2_LANES = 8;                  // lanes per token in phase 2
constexpr int P2_THREADS = P2_TOK * P2_LANES;
constexpr int kRows = 3 * D;                 // [G ; C ; dW1]
constexpr int kPartial = kRows * D;          // floats per partial slot
constexpr int kMats = 4;                     // W1, dC, dC^T, dG + dG^T per unit
constexpr int kMaxGrid = 320;               // phase-1 CTAs: two per SM
constexpr int MP = D + 4;                    // padded pitch of the 64 x 64 matrices in shared memory
constexpr int RP = D + 1;                    // padded pitch of token rows

template <typename E> struct Io;
template <> struct Io<float> {
    static __device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
    // 4 consecutive outputs (16-byte aligned)
    static __device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
        *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
    }
};
template <> struct Io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(p[0]); }
    // 4 consecutive outputs (8-byte aligned), rounded to bf16
    static __device__ __forceinline__ void st4(__nv_bfloat16* p, float a, float b, float c, float d) {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
    }
};

struct View {                                // element (u, n, c) of a [B][heads][N][64] view
    long long bs, hs;
    int heads;
    __device__ __forceinline__ size_t row(int u, int n) const {
        return (size_t)(u / heads) * bs + (size_t)(u % heads) * hs + (size_t)n * D;
    }
};

struct Partition {                           // CTA c owns tiles [start(c), start(c + 1))
    long long T;
    int G;
    __host__ __device__ long long start(int c) const { return (long long)c * T / G; }
    __host__ __device__ int cta_of(long long t) const { return (int)(((t + 1) * G - 1) / T); }
};

struct Params {
    const void *Q, *K, *V, *dZ;
    void *dQ, *dK, *dV;
    View view;
    int N, tpu, units;
    Partition part;
    float s, eta_grad_scale;                 // s = 2 eta / N; -(2/N)
    const float* W0;                         // [heads][64][64]
    unsigned* counters;                      // [units], zero between calls
    float* partials;                         // [(G + units)][192][64], slot = cta + unit
    float* mats;                             // [units][4][64][64]: W1, dC, dC^T, dG + dG^T
    float* dW0_unit;                         // [units][64][64]
    float* deta_unit;                        // [units]
    float* dW0_out;                          // nullable [heads][64][64]
    float* deta_out;                         // nullable, one float
};

// ------------------------------------------------------------------------------------------------
// phase 1: token sums and the per-unit merge
// ------------------------------------------------------------------------------------------------
struct P1Stage {                             // token chunk (the sums)
    float k[CHUNK][D], v[CHUNK][D], q[CHUNK][D], dz[CHUNK][D];
};
struct P1Merge {                             // the merge (the staging tiles are idle by then)
    float acc[kRows][D];                     // the unit's summed [G ; C ; dW1]
    float w0[D][MP];                         // W0 of the head
    float p[D][MP];                          // P = W0 G - C
};
struct P1Smem {
    union {
        P1Stage st;
        P1Merge mg;
    };
    float red[P1_THREADS / 32];
    int last;
};

template <typename E>
__device__ void merge_unit(const Params& p, P1Smem& s, int u, int slot0, int nslots) {
    const int tid = threadIdx.x;
    const int h = u % p.view.heads;
    // fixed-order sum of the unit's partial slots
    for (int e = tid; e < kPartial; e += P1_THREADS) {
        (&s.mg.acc[0][0])[e] = add_strided_in_order(0.f, p.partials + (size_t)slot0 * kPartial + e, kPartial, nslots);
    }
    for (int e = tid; e < D * D; e += P1_THREADS) s.mg.w0[e / D][e % D] = __ldg(p.W0 + (size_t)h * D * D + e);
    __syncthreads();
    const float (*G)[D] = s.mg.acc;          // rows 0..63
    const float (*C)[D] = s.mg.acc + D;      // rows 64..127
    const float (*dW1)[D] = s.mg.acc + 2 * D;   // rows 128..191
    const float (*w0)[MP] = s.mg.w0;
    float (*P)[MP] = s.mg.p;
    // P = W0 G - C (a warp's lanes take consecutive j: rows of G are read contiguously)
    for (int e = tid; e < D * D; e += P1_THREADS) {
        const int i = e / D, j = e % D;
        float a = 0.f;
#pragma unroll 8
        for (int m = 0; m < D; ++m) a = fmaf(w0[i][m], G[m][j], a);
        P[i][j] = a - C[i][j];
    }
    __syncthreads();
    float* M = p.mats + (size_t)u * kMats * D * D;
    float part = 0.f;
    for (int e = tid; e < D * D; e += P1_THREADS) {
        const int i = e / D, j = e % D;
        const float g = dW1[i][j];
        float dg = 0.f, dgt = 0.f, dwg = 0.f;
#pragma unroll 8
        for (int m = 0; m < D; ++m) {
            dg = fmaf(w0[m][i], dW1[m][j], dg);      // (W0^T dW1)_ij
            dgt = fmaf(w0[m][j], dW1[m][i], dgt);    // (W0^T dW1)_ji
            dwg = fmaf(dW1[i][m], G[m][j], dwg);     // (dW1 G)_ij
        }
        M[0 * D * D + e] = w0[i][j] - p.s * P[i][j];        // W1
        M[1 * D * D + e] = p.s * g;                         // dC
        M[2 * D * D + j * D + i] = p.s * g;                 // dC^T
        M[3 * D * D + e] = -p.s * (dg + dgt);               // dG + dG^T
        p.dW0_unit[(size_t)u * D * D + e] = g - p.s * dwg;  // dW0 of this unit
        part = fmaf(g, P[i][j], part);
    }
    // deta of the unit: fixed-order block sum
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) s.red[tid >> 5] = part;
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < P1_THREADS / 32; ++w) t += s.red[w];
        p.deta_unit[u] = p.eta_grad_scale * t;
    }
}

template <typename E>
__global__ void __launch_bounds__(P1_THREADS)
lin_bwd_p1(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    P1Smem& s = *reinterpret_cast<P1Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, c = blockIdx.x;
    const E* Kp = static_cast<const E*>(p.K);
    const E* Vp = static_cast<const E*>(p.V);
    const E* Qp = static_cast<const E*>(p.Q);
    const E* Zp = static_cast<const E*>(p.dZ);
    const int r = tid >> 1, j0 = (tid & 1) * 4;        // row of [G ; C ; dW1]; columns 8 c + j0 .. + 3
    pdl_launch_dependents();
    const long long t_begin = p.part.start(c), t_end = p.part.start(c + 1);
    long long t = t_begin;
    while (t < t_end) {
        const int u = (int)(t / p.tpu);
        const long long seg_end = min(t_end, (long long)(u + 1) * p.tpu);
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
        const int n_begin = (int)(t % p.tpu) * TOK;
        const int n_end = min(p.N, (int)((seg_end - (long long)u * p.tpu) * TOK));
        for (int n0 = n_begin; n0 < n_end; n0 += CHUNK) {
            for (int e = tid; e < CHUNK * D; e += P1_THREADS) {
                const int tk = e / D, cc = e % D, n = n0 + tk;
                const bool in = n < n_end;
                const size_t o = p.view.row(u, in ? n : 0) + cc;
                s.st.k[tk][cc] = in ? Io<E>::ld(Kp + o) : 0.f;
                s.st.v[tk][cc] = in ? Io<E>::ld(Vp + o) : 0.f;
                s.st.q[tk][cc] = in ? Io<E>::ld(Qp + o) : 0.f;
                s.st.dz[tk][cc] = in ? Io<E>::ld(Zp + o) : 0.f;
            }
            __syncthreads();
            for (int tk = 0; tk < CHUNK; ++tk) {
                const float x = (r < D) ? s.st.k[tk][r] : (r < 2 * D) ? s.st.v[tk][r - D] : s.st.dz[tk][r - 2 * D];
                const float* y = (r < 2 * D) ? s.st.k[tk] : s.st.q[tk];
#pragma unroll
                for (int cg = 0; cg < 8; ++cg) {
                    const float4 yv = *reinterpret_cast<const float4*>(y + 8 * cg + j0);
                    acc[4 * cg + 0] = fmaf(x, yv.x, acc[4 * cg + 0]);
                    acc[4 * cg + 1] = fmaf(x, yv.y, acc[4 * cg + 1]);
                    acc[4 * cg + 2] = fmaf(x, yv.z, acc[4 * cg + 2]);
                    acc[4 * cg + 3] = fmaf(x, yv.w, acc[4 * cg + 3]);
                }
            }
            __syncthreads();
        }
        float* dst = p.partials + (size_t)(c + u) * kPartial + (size_t)r * D + j0;
#pragma unroll
        for (int cg = 0; cg < 8; ++cg)
            *reinterpret_cast<float4*>(dst + 8 * cg) =
                make_float4(acc[4 * cg], acc[4 * cg + 1], acc[4 * cg + 2], acc[4 * cg + 3]);
        __threadfence();
        __syncthreads();
        const int cf = p.part.cta_of((long long)u * p.tpu), cl = p.part.cta_of((long long)(u + 1) * p.tpu - 1);
        if (tid == 0) {
            const unsigned old = atomicAdd(p.counters + u, 1u);
            s.last = (old + 1u == (unsigned)(cl - cf + 1)) ? 1 : 0;
        }
        __syncthreads();
        if (s.last) {
            __threadfence();
            merge_unit<E>(p, s, u, cf + u, cl - cf + 1);
            __threadfence();
            if (tid == 0) p.counters[u] = 0u;
        }
        __syncthreads();
        t = seg_end;
    }
}

// ------------------------------------------------------------------------------------------------
// phase 2: dq, dk, dv per token
// ------------------------------------------------------------------------------------------------
struct P2Smem {
    float m[kMats][D][D];                    // W1, dC, dC^T, dG + dG^T
    float dz[P2_TOK][RP], k[P2_TOK][RP], v[P2_TOK][RP];
};

template <typename E>
__global__ void __launch_bounds__(P2_THREADS)
lin_bwd_p2(const Params p, int tiles_per_unit) {
    extern __shared__ uint8_t smem_raw[];
    P2Smem& s = *reinterpret_cast<P2Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x;
    const long long tile = blockIdx.x;
    const int u = (int)(tile / tiles_per_unit), n0 = (int)(tile % tiles_per_unit) * P2_TOK;
    const E* Kp = static_cast<const E*>(p.K);
    const E* Vp = static_cast<const E*>(p.V);
    const E* Zp = static_cast<const E*>(p.dZ);
    for (int e = tid; e < P2_TOK * D; e += P2_THREADS) {
        const int tk = e / D, cc = e % D, n = n0 + tk;
        const bool in = n < p.N;
        const size_t o = p.view.row(u, in ? n : 0) + cc;
        s.dz[tk][cc] = in ? Io<E>::ld(Zp + o) : 0.f;
        s.k[tk][cc] = in ? Io<E>::ld(Kp + o) : 0.f;
        s.v[tk][cc] = in ? Io<E>::ld(Vp + o) : 0.f;
    }
    pdl_wait_primary();                      // the unit's matrices come from phase 1
    const float4* M4 = reinterpret_cast<const float4*>(p.mats + (size_t)u * kMats * D * D);
    float4* m4 = reinterpret_cast<float4*>(&s.m[0][0][0]);
    for (int e = tid; e < kMats * D * D / 4; e += P2_THREADS) m4[e] = __ldcg(M4 + e);
    __syncthreads();
    // token row of the CTA; output columns 32 h + 4 j4 .. + 3 for h = 0, 1
    const int row = tid / P2_LANES, j4 = (tid % P2_LANES) * 4;
    float gq[8], gk[8], gv[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) { gq[a] = 0.f; gk[a] = 0.f; gv[a] = 0.f; }
#pragma unroll 4
    for (int i = 0; i < D; ++i) {
        const float z = s.dz[row][i], kk = s.k[row][i], vv = s.v[row][i];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = 32 * h + j4, a = 4 * h;
            const float4 w1 = *reinterpret_cast<const float4*>(&s.m[0][i][c]);    // W1[i][.]
            const float4 dc = *reinterpret_cast<const float4*>(&s.m[1][i][c]);    // dC[i][.]
            const float4 dct = *reinterpret_cast<const float4*>(&s.m[2][i][c]);   // dC^T[i][.]
            const float4 dg = *reinterpret_cast<const float4*>(&s.m[3][i][c]);    // (dG + dG^T)[i][.]
            gq[a] = fmaf(w1.x, z, gq[a]); gq[a + 1] = fmaf(w1.y, z, gq[a + 1]);
            gq[a + 2] = fmaf(w1.z, z, gq[a + 2]); gq[a + 3] = fmaf(w1.w, z, gq[a + 3]);
            gk[a] = fmaf(dc.x, vv, fmaf(dg.x, kk, gk[a]));
            gk[a + 1] = fmaf(dc.y, vv, fmaf(dg.y, kk, gk[a + 1]));
            gk[a + 2] = fmaf(dc.z, vv, fmaf(dg.z, kk, gk[a + 2]));
            gk[a + 3] = fmaf(dc.w, vv, fmaf(dg.w, kk, gk[a + 3]));
            gv[a] = fmaf(dct.x, kk, gv[a]); gv[a + 1] = fmaf(dct.y, kk, gv[a + 1]);
            gv[a + 2] = fmaf(dct.z, kk, gv[a + 2]); gv[a + 3] = fmaf(dct.w, kk, gv[a + 3]);
        }
    }
    const int n = n0 + row;
    if (n < p.N) {
        const size_t o = p.view.row(u, n);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = 32 * h + j4, a = 4 * h;
            Io<E>::st4(static_cast<E*>(p.dQ) + o + c, gq[a], gq[a + 1], gq[a + 2], gq[a + 3]);
            Io<E>::st4(static_cast<E*>(p.dK) + o + c, gk[a], gk[a + 1], gk[a + 2], gk[a + 3]);
            Io<E>::st4(static_cast<E*>(p.dV) + o + c, gv[a], gv[a + 1], gv[a + 2], gv[a + 3]);
        }
    }
}

// ------------------------------------------------------------------------------------------------
// dW0 over images, deta over units (index order)
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
lin_bwd_sum(const Params p, int batch) {
    const int h = blockIdx.x, heads = p.view.heads;
    if (p.dW0_out) {
        for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
            float a = 0.f;
            for (int b = 0; b < batch; ++b) a += p.dW0_unit[((size_t)b * heads + h) * D * D + e];
            p.dW0_out[(size_t)h * D * D + e] = a;
        }
    }
    if (p.deta_out && h == 0 && threadIdx.x == 0) {
        float a = 0.f;
        for (int u = 0; u < p.units; ++u) a += p.deta_unit[u];
        *p.deta_out = a;
    }
}

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
struct WsLayout {
    size_t counters, partials, mats, dw0, deta, total;
};

static WsLayout ws_layout(long long units) {
    WsLayout L;
    L.counters = kWsHeader;
    L.partials = align_up(L.counters + (size_t)units * sizeof(unsigned), 1024);
    L.mats = align_up(L.partials + (size_t)(kMaxGrid + units) * kPartial * sizeof(float), 1024);
    L.dw0 = align_up(L.mats + (size_t)units * kMats * D * D * sizeof(float), 1024);
    L.deta = align_up(L.dw0 + (size_t)units * D * D * sizeof(float), 256);
    L.total = align_up(L.deta + (size_t)units * sizeof(float), 256);
    return L;
}

template <typename E>
static ttt_status launch(const Call& c, const void* dZ, void* dQ, void* dK, void* dV, float* dW0_out,
                         float* deta_out) {
    const long long units = (long long)c.batch * c.heads;
    const int tpu = (c.N + TOK - 1) / TOK;
    const WsLayout L = ws_layout(units);
    Params p{};
    p.Q = c.Q; p.K = c.K; p.V = c.V; p.dZ = dZ;
    p.dQ = dQ; p.dK = dK; p.dV = dV;
    p.view = View{c.bs, c.hs, c.heads};
    p.N = c.N;
    p.tpu = tpu;
    p.units = (int)units;
    const long long T = units * tpu;
    const int G = (int)std::max<long long>(1, std::min<long long>(std::min(2 * c.num_sms, kMaxGrid), T));
    p.part = Partition{T, G};
    p.s = c.eta * (2.0f / (float)c.N);
    p.eta_grad_scale = -2.0f / (float)c.N;
    p.W0 = c.W0;
    p.counters = reinterpret_cast<unsigned*>(c.ws + L.counters);
    p.partials = reinterpret_cast<float*>(c.ws + L.partials);
    p.mats = reinterpret_cast<float*>(c.ws + L.mats);
    p.dW0_unit = reinterpret_cast<float*>(c.ws + L.dw0);
    p.deta_unit = reinterpret_cast<float*>(c.ws + L.deta);
    p.dW0_out = dW0_out;
    p.deta_out = deta_out;

    const size_t sm1 = sizeof(P1Smem) + 128, sm2 = sizeof(P2Smem) + 128;
    cudaFuncSetAttribute(lin_bwd_p1<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    cudaFuncSetAttribute(lin_bwd_p2<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    lin_bwd_p1<E><<<G, P1_THREADS, sm1, c.stream>>>(p);
    ttt_status st = check_launch(cudaGetLastError());
    if (st != TTT_OK) return st;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    const int tiles2 = (c.N + P2_TOK - 1) / P2_TOK;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(units * tiles2));
    cfg.blockDim = dim3(P2_THREADS);
    cfg.dynamicSmemBytes = sm2;
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    st = check_launch(cudaLaunchKernelEx(&cfg, lin_bwd_p2<E>, p, tiles2));
    if (st != TTT_OK || (!dW0_out && !deta_out)) return st;
    lin_bwd_sum<<<c.heads, 256, 0, c.stream>>>(p, c.batch);
    return check_launch(cudaGetLastError());
}

}  // namespace bwd

size_t linear_backward_ws_bytes(const ttt_shape& s) {
    return bwd::ws_layout((long long)s.batch * s.heads).total;
}

size_t linear_backward_ws_control_bytes(const ttt_shape& s) {
    return bwd::ws_layout((long long)s.batch * s.heads).partials;
}

ttt_status launch_linear_backward(const Call& c, const void* dZ, void* dQ, void* dK, void* dV, float* dW0_out,
                                  float* deta_out) {
    if (c.dtype == TTT_BF16) return bwd::launch<__nv_bfloat16>(c, dZ, dQ, dK, dV, dW0_out, deta_out);
    return bwd::launch<float>(c, dZ, dQ, dK, dV, dW0_out, deta_out);
}

}  // namespace ttt
