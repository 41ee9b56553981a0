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
// bf16 runs on the tensor cores (lin_bwd_p1_tc, lin_bwd_merge_tc, lin_bwd_p2_tc below: the token sums
// and the per-token maps are the forward's contraction shapes).  fp32 keeps three plain fp32 FMA
// kernels, for fp32 accuracy:
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
#include <type_traits>

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
    float* deta_unit;                        // [deta_terms]: per unit (fp32), per merge CTA (bf16)
    int deta_terms;
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
// Four CTAs per head, one float4 of dW0 per thread, the images' terms eight at a time in flight.
__global__ void __launch_bounds__(256)
lin_bwd_sum(const Params p, int batch) {
    const int h = blockIdx.x >> 2, heads = p.view.heads;
    const int e4 = (blockIdx.x & 3) * 256 + (int)threadIdx.x;        // float4 of the head's 64 x 64
    pdl_wait_primary();                      // launched as a programmatic dependent of phase 2
    if (p.dW0_out) {
        const float4* src = reinterpret_cast<const float4*>(p.dW0_unit) + (size_t)h * (D * D / 4) + e4;
        const size_t stride = (size_t)heads * (D * D / 4);
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int b0 = 0; b0 < batch; b0 += 8) {
            float4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = b0 + q < batch ? __ldcg(src + (size_t)(b0 + q) * stride) : a;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (b0 + q < batch) { a.x += v[q].x; a.y += v[q].y; a.z += v[q].z; a.w += v[q].w; }
        }
        reinterpret_cast<float4*>(p.dW0_out + (size_t)h * D * D)[e4] = a;
    }
    if (p.deta_out && blockIdx.x == 0) {
        // the terms of deta loaded by the whole block (one round trip per 1024), summed in index order
        __shared__ float terms[1024];
        float acc = 0.f;
        for (int t0 = 0; t0 < p.deta_terms; t0 += 1024) {
            const int n = min(1024, p.deta_terms - t0);
            __syncthreads();
            for (int k = threadIdx.x; k < n; k += blockDim.x) terms[k] = __ldcg(p.deta_unit + t0 + k);
            __syncthreads();
            if (threadIdx.x == 0)
                for (int k = 0; k < n; ++k) acc += terms[k];
        }
        if (threadIdx.x == 0) *p.deta_out = acc;
    }
}

// ------------------------------------------------------------------------------------------------
// bf16 on the tensor cores (tcgen05, fp32 accumulation in tensor memory, tiles moved by TMA)
//   lin_bwd_p1_tc     static partition of 128-token tiles over one CTA per SM.  Per tile the four
//                     token boxes [K | V | dZ | Q] land in one 64 KB ring stage; two MMAs per
//                     16-token step accumulate [K | V]^T K (M = 128: the G rows, then the C rows)
//                     and [dZ | Q]^T Q (M = 128, of which the dZ rows are dW1).  At the end of each
//                     unit's run of tiles the accumulators go to the (CTA, unit) partial slot.
//   lin_bwd_merge_tc  1, 2 or 4 CTAs per unit (programmatic dependent of p1), each a share of the
//                     unit's rows: the slot sum, the unit's matrices as in merge_unit, and the four
//                     maps of phase 2 as bf16 hi + lo operand images (128-byte swizzled rows c, K = i).
//   lin_bwd_p2_tc     static partition of 128-token tiles over one CTA per SM (programmatic
//                     dependent of the merge): per tile the boxes dZ, K, V; dQ = dZ W1, dV = K dC^T,
//                     dK = V dC + K (dG + dG^T), each against the hi and lo image; the
//                     accumulators are drained to bf16 and stored by TMA.
// ------------------------------------------------------------------------------------------------
namespace tc {

constexpr int BOX = TOK * D * 2;             // one 128-token box of one tensor: 16 KB
constexpr int S1 = 3;                        // ring stages of p1 (four boxes each)
constexpr int S2 = 2;                        // ring stages of p2 (three boxes each)
constexpr int kImg = D * D * 2;              // one 64 x 64 bf16 operand image: 8 KB
constexpr int kImgs = 8;                     // W1^T, dC, dC^T, dG + dG^T, each hi and lo
constexpr int kThreads = 192;                // producer warp, MMA warp, four drain warps
constexpr uint32_t kIdescSum = idesc_bf16_f32(128, 64, true, true);     // D[m][n] = sum_tok A[tok][m] B[tok][n]
constexpr uint32_t kIdescMap = idesc_bf16_f32(128, 64, false, false);   // D[tok][c] = sum_i A[tok][i] B[c][i]

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// 16-byte chunk j (elements 8j .. 8j+7) of row `row` of a 128-byte swizzled operand image.
__device__ __forceinline__ uint32_t sw_off(int row, int j) { return (uint32_t)(row * 128 + ((j ^ (row & 7)) << 4)); }

struct TcParams {
    int tpu, heads;
    Partition part;
    float* partials;                         // [(G + units)][192][64]
    const uint8_t* imgs;                     // [units][kImgs][kImg] (p2)
    uint32_t* err;
    unsigned long long wait_ns;
};

// ---------------------------------------------------------------- p1
struct P1TcSmem {
    uint8_t ring[S1][4 * BOX];               // K, V, dZ, Q
    uint64_t full[S1], empty[S1];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain_bar;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ void p1_producer(P1TcSmem& s, const TcParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                            const CUtensorMap* tmZ, const CUtensorMap* tmQ, const Abort& ab) {
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    int st = 0; uint32_t ph = 0, issued = 0;
    for (long long t = t0; t < t1; ++t) {
        const int u = (int)(t / p.tpu), n0 = (int)(t % p.tpu) * TOK, h = u % p.heads, b = u / p.heads;
        if (!mbar_wait(&s.empty[st], ph ^ 1u, ab)) break;
        mbar_arrive_expect_tx(&s.full[st], 4 * BOX);
        uint8_t* dst = s.ring[st];
        tma_load_4d(dst + 0 * BOX, tmK, &s.full[st], 0, n0, h, b);
        tma_load_4d(dst + 1 * BOX, tmV, &s.full[st], 0, n0, h, b);
        tma_load_4d(dst + 2 * BOX, tmZ, &s.full[st], 0, n0, h, b);
        tma_load_4d(dst + 3 * BOX, tmQ, &s.full[st], 0, n0, h, b);
        ++issued;
        if (++st == S1) { st = 0; ph ^= 1u; }
    }
    for (uint32_t k = issued > (uint32_t)S1 ? issued - S1 : 0u; k < issued; ++k)
        mbar_drain(&s.full[k % S1], (k / S1) & 1u, ab.limit);
}

__device__ __forceinline__ void p1_mma(P1TcSmem& s, const TcParams& p, uint32_t tmem, const Abort& ab) {
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    int st = 0; uint32_t ph = 0, seg = 0;
    for (long long t = t0; t < t1;) {
        const int u = (int)(t / p.tpu);
        const long long se = min(t1, (long long)(u + 1) * p.tpu);
        const uint32_t ab2 = seg & 1u;
        if (!mbar_wait(&s.acc_empty[ab2], ((seg >> 1) & 1u) ^ 1u, ab)) return;
        tc_fence_after();
        const uint32_t d1 = tmem + ab2 * 128u, d2 = d1 + 64u;
        for (long long tt = t; tt < se; ++tt) {
            if (!mbar_wait(&s.full[st], ph, ab)) return;
            tc_fence_after();
            const uint32_t k = smem_u32(s.ring[st]), z = k + 2 * BOX;
#pragma unroll
            for (int kk = 0; kk < TOK / 16; ++kk) {
                const uint32_t acc = (tt == t && kk == 0) ? 0u : 1u;
                const uint64_t bk = sdesc_sw128(k + kk * 2048, BOX, 1024);
                mma_bf16_ss(d1, sdesc_sw128(k + kk * 2048, BOX, 1024), bk, kIdescSum, acc);   // [K | V]^T K
                mma_bf16_ss(d2, sdesc_sw128(z + kk * 2048, BOX, 1024),
                            sdesc_sw128(z + BOX + kk * 2048, BOX, 1024), kIdescSum, acc);     // [dZ | Q]^T Q
            }
            mma_commit(&s.empty[st]);
            if (++st == S1) { st = 0; ph ^= 1u; }
        }
        mma_commit(&s.acc_full[ab2]);
        ++seg;
        t = se;
    }
}

// Drain warps: TMEM lane r of the accumulators is row r of [G ; C] and (r < 64) row r of dW1.
__device__ __forceinline__ void p1_drain(P1TcSmem& s, const TcParams& p, uint32_t tmem, const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    uint32_t seg = 0;
    for (long long t = t0; t < t1;) {
        const int u = (int)(t / p.tpu);
        const long long se = min(t1, (long long)(u + 1) * p.tpu);
        const uint32_t ab2 = seg & 1u;
        const bool ok = mbar_wait(&s.acc_full[ab2], (seg >> 1) & 1u, ab);
        if (named_bar_or(1, 128, !ok)) break;
        __syncwarp();
        tc_fence_after();
        float g[4][16], w[4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld16(tmem + ab2 * 128u + (uint32_t)(j * 16) + lane_off, g[j]);
        if (q < 2) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(tmem + ab2 * 128u + 64u + (uint32_t)(j * 16) + lane_off, w[j]);
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s.acc_empty[ab2]);
        float* slot = p.partials + (size_t)(blockIdx.x + u) * kPartial;
        float4* d1 = reinterpret_cast<float4*>(slot + (size_t)r * D);
#pragma unroll
        for (int j = 0; j < 16; ++j) d1[j] = make_float4(g[j / 4][(j % 4) * 4], g[j / 4][(j % 4) * 4 + 1],
                                                         g[j / 4][(j % 4) * 4 + 2], g[j / 4][(j % 4) * 4 + 3]);
        if (q < 2) {
            float4* d2 = reinterpret_cast<float4*>(slot + (size_t)(2 * D + r) * D);
#pragma unroll
            for (int j = 0; j < 16; ++j) d2[j] = make_float4(w[j / 4][(j % 4) * 4], w[j / 4][(j % 4) * 4 + 1],
                                                             w[j / 4][(j % 4) * 4 + 2], w[j / 4][(j % 4) * 4 + 3]);
        }
        ++seg;
        t = se;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
lin_bwd_p1_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmQ, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    P1TcSmem& s = *reinterpret_cast<P1TcSmem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};
    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < S1; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
        mbar_init(&s.drain_bar, 1);
        fence_barrier_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmZ); prefetch_tmap(&tmQ);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 256); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    const uint32_t tmem = s.tmem_base;
    if (warp == 0) {
        if (lane == 0) p1_producer(s, p, &tmK, &tmV, &tmZ, &tmQ, ab);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            p1_mma(s, p, tmem, ab);
            mma_commit(&s.drain_bar);
            mbar_drain(&s.drain_bar, 0u, ab.limit);
        }
        __syncwarp();
    } else {
        p1_drain(s, p, tmem, ab);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------- merge
// SPLIT CTAs per unit (1, 2 or 4: as many as keep one CTA per SM), each 64 / SPLIT rows i of the
// unit's matrices; a thread takes 4 / SPLIT of those rows and four columns j0 .. j0+3 of the products
// P = W0 G - C, M = W0^T dW1 (row i and column i) and dW1 G:
//   W1 = W0 - s P,  dC = s dW1,  dG + dG^T = -s (M + M^T),  dW0 = dW1 - s dW1 G,
//   deta = -(2/N) sum dW1 * P  (per CTA: warp sums, then the warps in order; the CTAs' partials are
//   summed in index order by lin_bwd_sum).
constexpr int kMergeThreads = 256;
constexpr int kMaxSplit = 4;
// Dynamic shared memory of a merge CTA: more than half an SM's, so that the block scheduler places
// one merge CTA per SM (packed four to an SM they ran four times slower).
constexpr size_t kMergeSmem = 120 * 1024;
struct MergeTcSmem {
    float g[D][MP];                              // G, summed over the unit's slots
    float dw1[D][MP];                            // dW1
    float c[D][MP];                              // the CTA's rows of C
    float w0[D][MP];
    __nv_bfloat16 tr[4][D][D];                   // W1^T and dC^T (hi, lo): rows c, the CTA's K = i
    float red[kMergeThreads / 32];
};
static_assert(sizeof(MergeTcSmem) + 128 <= kMergeSmem, "merge shared memory");

// Elements K = k0 .. k0+3 of row `row` of an operand image pair (8-byte stores, k0 a multiple of 4).
__device__ __forceinline__ void put_hi_lo4(uint8_t* hi, int row, int k0, const float (&v)[4]) {
    float h[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        h[k] = __bfloat162float(__float2bfloat16_rn(v[k]));
        l[k] = v[k] - h[k];
    }
    const uint32_t off = sw_off(row, k0 / 8) + (uint32_t)(k0 % 8) * 2;
    *reinterpret_cast<uint2*>(hi + off) = make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
    *reinterpret_cast<uint2*>(hi + kImg + off) = make_uint2(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]));
}

// Row r (0 .. 143) of what a merge CTA sums: G rows 0..63, its 16 rows of C, then dW1 rows 0..63;
// returns the slot row and the shared-memory row.
template <int ROWS>
__device__ __forceinline__ void merge_row(MergeTcSmem& s, int r, int i0, int& slot_row, float*& dst) {
    if (r < D) { slot_row = r; dst = s.g[r]; }
    else if (r < D + ROWS) { slot_row = D + i0 + (r - D); dst = s.c[r - D]; }
    else { slot_row = 2 * D + (r - D - ROWS); dst = s.dw1[r - D - ROWS]; }
}

// The unit's matrices, then the operand images of phase 2, image x holding X[c][i]:
//   0/1 W1^T (dQ = dZ W1),  2/3 dC (dV = K dC^T),  4/5 dC^T (dK = V dC + ..),  6/7 dG + dG^T (symmetric),
// each rounded to bf16 (hi) with the rounding error rounded again (lo).
template <int SPLIT>
__global__ void __launch_bounds__(kMergeThreads, 1)
lin_bwd_merge_tc(const Params p, uint8_t* imgs) {
    constexpr int ROWS = D / SPLIT, RPT = ROWS / 16;     // rows per CTA, rows per thread
    extern __shared__ uint8_t smem_raw[];
    MergeTcSmem& s = *reinterpret_cast<MergeTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int u = blockIdx.x / SPLIT, i0 = (blockIdx.x % SPLIT) * ROWS;
    const int tid = threadIdx.x, h = u % p.view.heads;
    pdl_wait_primary();                      // every partial slot is written
    pdl_launch_dependents();
    const int cf = p.part.cta_of((long long)u * p.tpu), cl = p.part.cta_of((long long)(u + 1) * p.tpu - 1);
    const int nslots = cl - cf + 1;
    // the slot sums in slot order: three float4 per thread at a time, eight slots of each in flight
    constexpr int F4 = (2 * D + ROWS) * (D / 4);
    const float4* src = reinterpret_cast<const float4*>(p.partials + (size_t)(cf + u) * kPartial);
    for (int f0 = tid; f0 < F4; f0 += 3 * kMergeThreads) {
        float4 acc[3];
        size_t off[3];
#pragma unroll
        for (int g = 0; g < 3; ++g) {
            acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
            const int f = min(f0 + g * kMergeThreads, F4 - 1);
            int sr; float* d;
            merge_row<ROWS>(s, f / (D / 4), i0, sr, d);
            off[g] = (size_t)sr * (D / 4) + f % (D / 4);
        }
        for (int k0 = 0; k0 < nslots; k0 += 8) {
            float4 v[3][8];
#pragma unroll
            for (int g = 0; g < 3; ++g)
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    v[g][q] = k0 + q < nslots ? __ldcg(src + (size_t)(k0 + q) * (kPartial / 4) + off[g])
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int g = 0; g < 3; ++g)
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (k0 + q < nslots) {
                        acc[g].x += v[g][q].x; acc[g].y += v[g][q].y; acc[g].z += v[g][q].z; acc[g].w += v[g][q].w;
                    }
        }
#pragma unroll
        for (int g = 0; g < 3; ++g) {
            const int f = f0 + g * kMergeThreads;
            if (f < F4) {
                int sr; float* d;
                merge_row<ROWS>(s, f / (D / 4), i0, sr, d);
                *reinterpret_cast<float4*>(d + 4 * (f % (D / 4))) = acc[g];
            }
        }
    }
    const float4* w04 = reinterpret_cast<const float4*>(p.W0 + (size_t)h * D * D);
#pragma unroll
    for (int k = 0; k < D * D / 4 / kMergeThreads; ++k) {
        const int e = 4 * (tid + k * kMergeThreads);
        *reinterpret_cast<float4*>(&s.w0[e / D][e % D]) = __ldg(w04 + tid + k * kMergeThreads);
    }
    __syncthreads();
    const int a0 = (tid >> 4) * RPT, j0 = (tid & 15) * 4;     // rows i0 + a0 .. i0 + a0 + RPT - 1
    float P[RPT][4], Mr[RPT][4], Mc[RPT][4], WG[RPT][4];
#pragma unroll
    for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int b = 0; b < 4; ++b) { P[r][b] = 0.f; Mr[r][b] = 0.f; Mc[r][b] = 0.f; WG[r][b] = 0.f; }
#pragma unroll 4
    for (int m = 0; m < D; ++m) {
        const float4 g4 = *reinterpret_cast<const float4*>(&s.g[m][j0]);
        const float4 d4 = *reinterpret_cast<const float4*>(&s.dw1[m][j0]);
        const float4 w4 = *reinterpret_cast<const float4*>(&s.w0[m][j0]);
        const float gv[4] = {g4.x, g4.y, g4.z, g4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w}, wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = i0 + a0 + r;
            const float wim = s.w0[i][m], wmi = s.w0[m][i], dmi = s.dw1[m][i], dim = s.dw1[i][m];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                P[r][b] = fmaf(wim, gv[b], P[r][b]);       // (W0 G)[i][j]
                Mr[r][b] = fmaf(wmi, dv[b], Mr[r][b]);     // M[i][j] = sum_m W0[m][i] dW1[m][j]
                Mc[r][b] = fmaf(wv[b], dmi, Mc[r][b]);     // M[j][i]
                WG[r][b] = fmaf(dim, gv[b], WG[r][b]);     // (dW1 G)[i][j]
            }
        }
    }
    uint8_t* out = imgs + (size_t)u * kImgs * kImg;
    float part = 0.f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = i0 + a0 + r;
        float dc[4], dg[4], dw0[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int j = j0 + b;
            const float pij = P[r][b] - s.c[a0 + r][j], g = s.dw1[i][j];
            const float w1 = s.w0[i][j] - p.s * pij;
            dc[b] = p.s * g;
            dg[b] = -p.s * (Mr[r][b] + Mc[r][b]);
            dw0[b] = g - p.s * WG[r][b];
            part = fmaf(g, pij, part);
            // W1^T and dC^T (row c = j, K = i): staged, stored below as 16-byte chunks
            const __nv_bfloat16 wh = __float2bfloat16_rn(w1), ch = __float2bfloat16_rn(dc[b]);
            s.tr[0][j][i - i0] = wh;
            s.tr[1][j][i - i0] = __float2bfloat16_rn(w1 - __bfloat162float(wh));
            s.tr[2][j][i - i0] = ch;
            s.tr[3][j][i - i0] = __float2bfloat16_rn(dc[b] - __bfloat162float(ch));
        }
        put_hi_lo4(out + 2 * kImg, i, j0, dc);                // dC: row c = i, K = j
        put_hi_lo4(out + 6 * kImg, i, j0, dg);                // dG + dG^T: row c = i, K = j
        *reinterpret_cast<float4*>(p.dW0_unit + (size_t)u * D * D + (size_t)i * D + j0) =
            make_float4(dw0[0], dw0[1], dw0[2], dw0[3]);
    }
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) s.red[tid >> 5] = part;
    __syncthreads();
    // the staged chunks: images 0, 1 (W1^T hi, lo) and 4, 5 (dC^T hi, lo), rows c, chunks of K = i
    constexpr int CH = ROWS / 8;
    for (int e = tid; e < 4 * D * CH; e += kMergeThreads) {
        const int x = e / (D * CH), c = (e / CH) % D, k = e % CH;
        const int img = (x < 2) ? x : x + 2;
        *reinterpret_cast<uint4*>(out + (size_t)img * kImg + sw_off(c, i0 / 8 + k)) =
            *reinterpret_cast<const uint4*>(&s.tr[x][c][8 * k]);
    }
    if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kMergeThreads / 32; ++w) t += s.red[w];
        p.deta_unit[blockIdx.x] = p.eta_grad_scale * t;
    }
}

// ---------------------------------------------------------------- p2
struct P2TcSmem {
    uint8_t ring[S2][3 * BOX];               // dZ, K, V
    uint8_t img[kImgs][kImg];                // the unit's operand images
    uint8_t stage[3][BOX];                   // dQ, dK, dV of a tile as bf16, for the TMA stores
    uint64_t full[S2], empty[S2];
    uint64_t img_full, img_empty;
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain_bar;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool p2_load_imgs(P2TcSmem& s, const TcParams& p, int u, uint32_t& parts, const Abort& ab) {
    if (parts == 0) pdl_wait_primary();      // the merge kernel has written the images
    if (!mbar_wait(&s.img_empty, (parts & 1u) ^ 1u, ab)) return false;
    fence_proxy_async_global();
    mbar_arrive_expect_tx(&s.img_full, kImgs * kImg);
    bulk_g2s(s.img, p.imgs + (size_t)u * kImgs * kImg, kImgs * kImg, &s.img_full);
    ++parts;
    return true;
}

__device__ __forceinline__ void p2_producer(P2TcSmem& s, const TcParams& p, const CUtensorMap* tmZ, const CUtensorMap* tmK,
                                            const CUtensorMap* tmV, const Abort& ab) {
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    int st = 0; uint32_t ph = 0, issued = 0, parts = 0;
    int pending = -1;                        // unit whose images are not requested yet
    bool ok = true;
    for (long long t = t0; t < t1 && ok; ++t) {
        const int u = (int)(t / p.tpu), n0 = (int)(t % p.tpu) * TOK, h = u % p.heads, b = u / p.heads;
        if (t == t0) {
            pending = u;                     // the first tiles (inputs) load while the merge runs
        } else if (t % p.tpu == 0) {         // a new unit: its images, after the first unit's
            if (pending >= 0 && !(ok = p2_load_imgs(s, p, pending, parts, ab))) break;
            pending = -1;
            if (!(ok = p2_load_imgs(s, p, u, parts, ab))) break;
        }
        if (pending >= 0 && issued == (uint32_t)S2) {
            if (!(ok = p2_load_imgs(s, p, pending, parts, ab))) break;
            pending = -1;
        }
        if (!(ok = mbar_wait(&s.empty[st], ph ^ 1u, ab))) break;
        mbar_arrive_expect_tx(&s.full[st], 3 * BOX);
        uint8_t* dst = s.ring[st];
        tma_load_4d(dst + 0 * BOX, tmZ, &s.full[st], 0, n0, h, b);
        tma_load_4d(dst + 1 * BOX, tmK, &s.full[st], 0, n0, h, b);
        tma_load_4d(dst + 2 * BOX, tmV, &s.full[st], 0, n0, h, b);
        ++issued;
        if (++st == S2) { st = 0; ph ^= 1u; }
    }
    if (ok && pending >= 0) p2_load_imgs(s, p, pending, parts, ab);
    for (uint32_t k = issued > (uint32_t)S2 ? issued - S2 : 0u; k < issued; ++k)
        mbar_drain(&s.full[k % S2], (k / S2) & 1u, ab.limit);
    if (parts > 0) mbar_drain(&s.img_full, (parts - 1) & 1u, ab.limit);
}

__device__ __forceinline__ void p2_mma(P2TcSmem& s, const TcParams& p, uint32_t tmem, const Abort& ab) {
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    int st = 0; uint32_t ph = 0, parts = 0, n = 0;
    const uint32_t img = smem_u32(s.img);
    for (long long t = t0; t < t1; ++t, ++n) {
        if (t == t0 || t % p.tpu == 0) {
            if (!mbar_wait(&s.img_full, parts & 1u, ab)) return;
            ++parts;
        }
        const uint32_t ab2 = n & 1u;
        if (!mbar_wait(&s.acc_empty[ab2], ((n >> 1) & 1u) ^ 1u, ab)) return;
        if (!mbar_wait(&s.full[st], ph, ab)) return;
        tc_fence_after();
        const uint32_t z = smem_u32(s.ring[st]), k = z + BOX, v = z + 2 * BOX;
        const uint32_t dq = tmem + ab2 * 192u, dv = dq + 64u, dk = dq + 128u;
        // (A box, image pair, accumulator): dQ = dZ W1, dV = K dC^T, dK = V dC + K (dG + dG^T)
        const uint32_t a_of[4] = {z, k, v, k};
        const uint32_t d_of[4] = {dq, dv, dk, dk};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
            for (int hl = 0; hl < 2; ++hl) {
                const uint32_t bimg = img + (uint32_t)((2 * m + hl) * kImg);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16_ss(d_of[m], sdesc_sw128(a_of[m] + kk * 32, 16, 1024), sdesc_sw128(bimg + kk * 32, 16, 1024),
                                kIdescMap, (m == 3 || hl || kk) ? 1u : 0u);
            }
        }
        mma_commit(&s.empty[st]);
        mma_commit(&s.acc_full[ab2]);
        if (t + 1 == t1 || (t + 1) % p.tpu == 0) mma_commit(&s.img_empty);
        if (++st == S2) { st = 0; ph ^= 1u; }
    }
}

// Drain warps: TMEM lane r is token row r of the tile; each output goes to its staging box as bf16
// (128-byte swizzled rows, the TMA store's layout), then one TMA store per output.
__device__ __forceinline__ void p2_drain(P2TcSmem& s, const TcParams& p, uint32_t tmem, const CUtensorMap* tmdQ,
                                         const CUtensorMap* tmdK, const CUtensorMap* tmdV, const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3, r = q * 32 + lane;
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    uint32_t n = 0;
    for (long long t = t0; t < t1; ++t, ++n) {
        const int u = (int)(t / p.tpu), n0 = (int)(t % p.tpu) * TOK, h = u % p.heads, b = u / p.heads;
        const uint32_t ab2 = n & 1u;
        const bool ok = mbar_wait(&s.acc_full[ab2], (n >> 1) & 1u, ab);
        if (tid == 0 && n > 0) bulk_wait_read<0>();          // the previous tile's stores have read the staging boxes
        if (named_bar_or(1, 128, !ok)) break;
        __syncwarp();
        tc_fence_after();
#pragma unroll 1
        for (int o = 0; o < 3; ++o) {                         // dQ, dV, dK: accumulator columns 64 o
            float v[4][16];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(tmem + ab2 * 192u + (uint32_t)(64 * o + 16 * j) + lane_off, v[j]);
            tmem_ld_wait();
            uint8_t* dst = s.stage[o];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float* x = &v[j / 2][(j % 2) * 8];
                uint4 pk;
                pk.x = pack_bf16x2(x[0], x[1]); pk.y = pack_bf16x2(x[2], x[3]);
                pk.z = pack_bf16x2(x[4], x[5]); pk.w = pack_bf16x2(x[6], x[7]);
                *reinterpret_cast<uint4*>(dst + sw_off(r, j)) = pk;
            }
        }
        tc_fence_before();
        mbar_arrive(&s.acc_empty[ab2]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (tid == 0) {
            tma_store_4d(tmdQ, s.stage[0], 0, n0, h, b);
            tma_store_4d(tmdV, s.stage[1], 0, n0, h, b);
            tma_store_4d(tmdK, s.stage[2], 0, n0, h, b);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait<0>();
}

__global__ void __launch_bounds__(kThreads, 1)
lin_bwd_p2_tc(const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdQ,
              const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    P2TcSmem& s = *reinterpret_cast<P2TcSmem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};
    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < S2; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        mbar_init(&s.img_full, 1); mbar_init(&s.img_empty, 1);
        for (int i = 0; i < 2; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
        mbar_init(&s.drain_bar, 1);
        fence_barrier_init();
        prefetch_tmap(&tmZ); prefetch_tmap(&tmK); prefetch_tmap(&tmV);
        prefetch_tmap(&tmdQ); prefetch_tmap(&tmdK); prefetch_tmap(&tmdV);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();                 // lin_bwd_sum waits for this grid's completion itself
    const uint32_t tmem = s.tmem_base;
    if (warp == 0) {
        if (lane == 0) p2_producer(s, p, &tmZ, &tmK, &tmV, ab);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            p2_mma(s, p, tmem, ab);
            mma_commit(&s.drain_bar);
            mbar_drain(&s.drain_bar, 0u, ab.limit);
        }
        __syncwarp();
    } else {
        p2_drain(s, p, tmem, &tmdQ, &tmdK, &tmdV, ab);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
struct WsLayout {
    size_t counters, partials, mats, dw0, deta, imgs, total;
};

static WsLayout ws_layout(long long units) {
    WsLayout L;
    L.counters = kWsHeader;
    L.partials = align_up(L.counters + (size_t)units * sizeof(unsigned), 1024);
    L.mats = align_up(L.partials + (size_t)(kMaxGrid + units) * kPartial * sizeof(float), 1024);
    L.dw0 = align_up(L.mats + (size_t)units * kMats * D * D * sizeof(float), 1024);
    L.deta = align_up(L.dw0 + (size_t)units * D * D * sizeof(float), 256);
    L.imgs = align_up(L.deta + (size_t)units * tc::kMaxSplit * sizeof(float), 1024);
    L.total = L.imgs + (size_t)units * tc::kImgs * tc::kImg;
    return L;
}

// bf16: the tensor-core kernels, one CTA per SM for the two streaming phases.
static ttt_status launch_tc(const Call& c, Params p, const WsLayout& L) {
    using namespace tc;
    CUtensorMap tmK, tmV, tmZ, tmQ, tmdQ, tmdK, tmdV;
    if (!make_tmap_tokens(&tmK, c.K, c, TOK) || !make_tmap_tokens(&tmV, c.V, c, TOK) ||
        !make_tmap_tokens(&tmZ, p.dZ, c, TOK) || !make_tmap_tokens(&tmQ, c.Q, c, TOK) ||
        !make_tmap_tokens(&tmdQ, p.dQ, c, TOK) || !make_tmap_tokens(&tmdK, p.dK, c, TOK) ||
        !make_tmap_tokens(&tmdV, p.dV, c, TOK))
        return TTT_ERR_INVALID_ARG;
    const long long T = p.part.T;
    const int G = (int)std::max<long long>(1, std::min<long long>(std::min(c.num_sms, kMaxGrid), T));
    p.part = Partition{T, G};
    TcParams tp{};
    tp.tpu = p.tpu;
    tp.heads = c.heads;
    tp.part = p.part;
    tp.partials = p.partials;
    tp.imgs = c.ws + L.imgs;
    tp.err = reinterpret_cast<uint32_t*>(c.ws);
    tp.wait_ns = c.wait_ns;
    const size_t sm1 = sizeof(P1TcSmem) + 1024, sm2 = sizeof(P2TcSmem) + 1024;
    if (sm1 > 227 * 1024 || sm2 > 227 * 1024) return TTT_ERR_UNSUPPORTED;
    cudaFuncSetAttribute(lin_bwd_p1_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    cudaFuncSetAttribute(lin_bwd_merge_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMergeSmem);
    cudaFuncSetAttribute(lin_bwd_merge_tc<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMergeSmem);
    cudaFuncSetAttribute(lin_bwd_merge_tc<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMergeSmem);
    cudaFuncSetAttribute(lin_bwd_p2_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    lin_bwd_p1_tc<<<G, kThreads, sm1, c.stream>>>(tmK, tmV, tmZ, tmQ, tp);
    ttt_status st = check_launch(cudaGetLastError());
    if (st != TTT_OK) return st;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    // merge CTAs per unit: the most of 4, 2, 1 that keeps every merge CTA on an SM of its own
    const int split = (p.units * 4 <= c.num_sms) ? 4 : (p.units * 2 <= c.num_sms) ? 2 : 1;
    p.deta_terms = p.units * split;
    cfg.gridDim = dim3((unsigned)(p.units * split));
    cfg.blockDim = dim3(kMergeThreads);
    cfg.dynamicSmemBytes = kMergeSmem;
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    st = check_launch(split == 4 ? cudaLaunchKernelEx(&cfg, lin_bwd_merge_tc<4>, p, c.ws + L.imgs)
                      : split == 2 ? cudaLaunchKernelEx(&cfg, lin_bwd_merge_tc<2>, p, c.ws + L.imgs)
                                   : cudaLaunchKernelEx(&cfg, lin_bwd_merge_tc<1>, p, c.ws + L.imgs));
    if (st != TTT_OK) return st;
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sm2;
    st = check_launch(cudaLaunchKernelEx(&cfg, lin_bwd_p2_tc, tmZ, tmK, tmV, tmdQ, tmdK, tmdV, tp));
    if (st != TTT_OK || (!p.dW0_out && !p.deta_out)) return st;
    cfg.gridDim = dim3((unsigned)(c.heads * 4));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    return check_launch(cudaLaunchKernelEx(&cfg, lin_bwd_sum, p, c.batch));
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
    p.deta_terms = (int)units;
    p.dW0_out = dW0_out;
    p.deta_out = deta_out;
    if constexpr (std::is_same<E, __nv_bfloat16>::value) {
        return launch_tc(c, p, L);
    } else {
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
        lin_bwd_sum<<<c.heads * 4, 256, 0, c.stream>>>(p, c.batch);
        return check_launch(cudaGetLastError());
    }
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
