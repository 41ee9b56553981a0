// mlp.cu -- one-hidden-layer MLP inner model of the TTT layer, f(x) = Wb gelu_tanh(Wa x), hidden
// width 256 = 4d (press article "CVPR 2026 Oral | 清華+阿里發布ViT3", Observation 4 and Fig. 5 part 1:
// an MLP inner model whose width ratio goes up to 4).  One full-batch step of the L2 loss on both
// matrices (gradients taken at the initial weights), then the readout:
//     h = Wa k, a = gelu(h), y = Wb a, r = y - v
//     gWb = sum_n r a^T,  gWa = sum_n [(Wb^T r) * gelu'(h)] k^T
//     Wa1 = Wa - eta (2/N) gWa,  Wb1 = Wb - eta (2/N) gWb,  z = Wb1 gelu(Wa1 q)
// gelu_tanh(u) = u/2 (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))) (the tanh form of Hendrycks & Gimpel).
//
// Every product is a dense contraction and runs on tcgen05 (bf16 operands, fp32 accumulation in
// tensor memory).  A unit is owned by a cluster of two CTAs, each taking half of the tokens (one CTA
// per unit, persistent over units, when there are more units than SM pairs).  A CTA has a TMA
// producer warp and 8 compute warps: tid 0 issues the MMAs, and the two warps of each tensor-memory
// lane quarter split every elementwise pass's columns (GELU in packed half precision).  Per 128-token
// tile of phase 1:
//   H  = K Wa^T            M=128 tokens, N=256, K=64       -> TMEM cols 256..511
//   A  = gelu(H) (bf16, shared memory), gelu'(H) packed bf16x2 back into TMEM cols 256..383
//   Y  = A Wb^T            M=128, N=64, K=256             -> TMEM cols 384..447
//   R  = Y - V (bf16, shared memory)
//   gWb^T += A^T R         M=256 (two 128-row halves), N=64, K=128 tokens (MN-major operands)
//   dA = R Wb              M=128, N=128 per hidden half, K=64     -> TMEM cols 384..511
//   dH = dA * gelu'(H) (bf16, shared memory, over A)
//   gWa  += dH^T K         M=256 (two halves), N=64, K=128 tokens
// The accumulators gWb^T and gWa stay in TMEM cols 0..255 across the CTA's tiles.  Then the two
// CTAs exchange partial gradients over distributed shared memory: CTA `rank` owns hidden half `rank`,
// adds the peer's partial for it (two terms: the same sum in either order), forms that half of Wa1
// and Wb1 in fp32 (optionally written out) and stores the bf16 operands into both CTAs' shared
// memory.  Phase 2 streams the CTA's Q tiles: H' = Q Wa1^T, A' = gelu(H'), Z = A' Wb1^T, stored
// with TMA.
// The same shared-memory buffers serve as K-major operands of one product and MN-major operands of
// another (both use the 128-byte swizzled layout TMA writes), so nothing is transposed.
#include <algorithm>

#include <cuda_fp16.h>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace mlp {

constexpr int D = 64;
constexpr int HID = 256;
constexpr int TOK = 128;
constexpr int TILE = TOK * D * 2;           // 16 KB bf16 tile
constexpr int STAGES = 2;                   // each holds a K tile + V tile, or a Q tile
constexpr int THREADS = 288;                // warp 0: TMA producer, warps 1..8: MMA + elementwise
constexpr int kCT = 256;                    // compute threads: two warps per tensor-memory lane quarter
constexpr float kGeluC = 0.7978845608028654f;   // sqrt(2 / pi)
constexpr float kGeluA = 0.044715f;

constexpr uint32_t kIdH = idesc_bf16_f32(128, 256, false, false);
constexpr uint32_t kIdY = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t kIdG = idesc_bf16_f32(128, 64, true, true);
constexpr uint32_t kIdDA = idesc_bf16_f32(128, 128, false, true);

struct Params {
    int U, heads, N, tpu;
    int CS;                                 // CTAs per unit (a cluster): 1 or 2
    float eta_scale;                        // eta * 2 / N
    const float* Wa;                        // [heads][256][64]
    const float* Wb;                        // [heads][64][256]
    float* Wa_out;                          // nullable [units][256][64]
    float* Wb_out;                          // nullable [units][64][256]
    uint32_t* err;
    unsigned long long wait_ns;     // bound of every device-side wait
};

struct Smem {
    uint8_t stage[STAGES][2 * TILE];        // K | V tiles, or a Q tile (1024-aligned)
    uint8_t act[4][TOK * 128];              // A (then dH): [token][hidden], 4 panels of 64 hidden
    uint8_t wa[HID * 128];                  // Wa (bf16): rows = hidden, 64 d per row
    uint8_t wb[4][D * 128];                 // Wb (bf16): rows = d, 4 panels of 64 hidden
    uint8_t rz[TOK * 128];                  // R tile (phase 1), Z staging (phase 2)
    uint64_t full[STAGES], empty[STAGES];
    uint64_t mma_bar;
    uint64_t free_bar;                      // the peer has finished phase 1: its act and weights may be written
    uint64_t xbar;                          // the peer's partial gradients for my hidden half have arrived
    uint64_t wbar;                          // the peer's half of the updated weight operands has arrived
    uint32_t tmem_base;
    int abort_flag;
};

__host__ __device__ __forceinline__ int split_lo(int n, int r, int parts) { return (int)((long long)n * r / parts); }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Byte offset of element (row, col) in a 128-byte swizzled panel of 64 bf16 per row.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + ((col & 7) << 1));
}

// gelu(u) and its derivative, from t = tanh(c (u + a u^3)):
//     gelu(u) = u/2 (1 + t),   gelu'(u) = (1 + t)/2 + u/2 (1 - t^2) c (1 + 3 a u^2),
// evaluated on a pair of values in packed half precision (10-bit mantissa, finer than
// the bf16 the results are rounded to), returned as packed bf16 pairs: about half the instructions
// of the fp32 form.
__device__ __forceinline__ __half2 tanh_fast_h2(__half2 x) {
    uint32_t y;
    asm("tanh.approx.f16x2 %0, %1;" : "=r"(y) : "r"(*reinterpret_cast<const uint32_t*>(&x)));
    return *reinterpret_cast<const __half2*>(&y);
}
__device__ __forceinline__ uint32_t h2_to_bf16x2(__half2 v) {
    const float2 f = __half22float2(v);
    return pack_bf16x2(f.x, f.y);
}
__device__ __forceinline__ void gelu_and_grad2(float u0, float u1, uint32_t& g, uint32_t& dg) {
    const __half2 one = __float2half2_rn(1.f), half = __float2half2_rn(0.5f);
    const __half2 u = __floats2half2_rn(u0, u1);
    const __half2 u2 = __hmul2(u, u);
    const __half2 t = tanh_fast_h2(__hmul2(__float2half2_rn(kGeluC), __hfma2(__hmul2(__float2half2_rn(kGeluA), u2), u, u)));
    const __half2 opt = __hadd2(one, t);
    g = h2_to_bf16x2(__hmul2(__hmul2(half, u), opt));
    const __half2 omt2 = __hfma2(__hneg2(t), t, one);                            // 1 - t^2
    const __half2 poly = __hfma2(__float2half2_rn(3.f * kGeluA), u2, one);      // 1 + 3 a u^2
    dg = h2_to_bf16x2(__hfma2(__hmul2(__hmul2(__float2half2_rn(0.5f * kGeluC), u), omt2), poly, __hmul2(half, opt)));
}
__device__ __forceinline__ uint32_t gelu_only2(float u0, float u1) {
    const __half2 u = __floats2half2_rn(u0, u1);
    const __half2 t = tanh_fast_h2(__hmul2(__float2half2_rn(kGeluC),
                                           __hfma2(__hmul2(__float2half2_rn(kGeluA), __hmul2(u, u)), u, u)));
    return h2_to_bf16x2(__hmul2(__hmul2(__float2half2_rn(0.5f), u), __hadd2(__float2half2_rn(1.f), t)));
}

__global__ void __launch_bounds__(THREADS, 1)
mlp_fused(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
          const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmZ, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        mbar_init(&s.mma_bar, 1);
        mbar_init(&s.free_bar, 1);
        mbar_init(&s.xbar, kCT);
        mbar_init(&s.wbar, kCT);
        fence_barrier_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmQ); prefetch_tmap(&tmZ);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every CTA's barriers exist before its peer arrives on them
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    const uint32_t tmem = s.tmem_base;
    const bool multi = p.CS > 1;
    const int rank = multi ? (int)cluster_ctarank() : 0;
    const int cid = multi ? (int)cluster_id_x() : (int)blockIdx.x;
    const int ncl = multi ? (int)cluster_count_x() : (int)gridDim.x;
    const int t0 = split_lo(p.tpu, rank, p.CS), t1 = split_lo(p.tpu, rank + 1, p.CS);   // this CTA's tiles

    if (warp == 0) {                                           // TMA producer
        if (lane == 0) {
            int st = 0; uint32_t ph = 0;
            for (int u = cid; u < p.U; u += ncl) {
                const int b = u / p.heads, h = u % p.heads;
                for (int t = t0; t < t1; ++t) {
                    if (!mbar_wait(&s.empty[st], ph ^ 1u, ab)) return;
                    mbar_arrive_expect_tx(&s.full[st], 2 * TILE);
                    tma_load_4d(s.stage[st], &tmK, &s.full[st], 0, t * TOK, h, b);
                    tma_load_4d(s.stage[st] + TILE, &tmV, &s.full[st], 0, t * TOK, h, b);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
                for (int t = t0; t < t1; ++t) {
                    if (!mbar_wait(&s.empty[st], ph ^ 1u, ab)) return;
                    mbar_arrive_expect_tx(&s.full[st], TILE);
                    tma_load_4d(s.stage[st], &tmQ, &s.full[st], 0, t * TOK, h, b);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
            }
        }
        __syncwarp();                                          // the warp reaches the block barrier converged
    } else {
        // ---------------------------------------------------------------------------------------
        // warps 1..8: tid 0 issues the MMAs, all 256 threads do the elementwise work.  Thread tid
        // reads and writes accumulator row r (its TMEM lane): a token (or a hidden unit); the two
        // warps of a lane quarter take the two halves (hw) of each elementwise pass's columns.
        // ---------------------------------------------------------------------------------------
        const int tid = threadIdx.x - 32;
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int hw = (warp - 1) >> 2;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t sact = smem_u32(s.act[0]), swa = smem_u32(s.wa), swb = smem_u32(s.wb[0]), srz = smem_u32(s.rz);
        uint32_t mph = 0;                                       // mma_bar phase
        int st = 0; uint32_t ph = 0;
        int zn = 0;
        bool failed = false;

        // issue-and-wait helper state
        auto mma_sync = [&](bool& ok) {
            if (tid == 0) mma_commit(&s.mma_bar);
            ok = mbar_wait(&s.mma_bar, mph, ab);
            mph ^= 1u;
            if (named_bar_or(1, kCT, !ok)) return false;
            __syncwarp();
            tc_fence_after();
            return true;
        };

        uint32_t k = 0;                                         // units done (phase of the exchange barriers)
        for (int u = cid; u < p.U && !failed; u += ncl, ++k) {
            const int bi = u / p.heads, h = u % p.heads;
            // ---- Wa, Wb of the head -> bf16 operands (coalesced float4 loads: consecutive threads read
            //      consecutive 16-byte pieces of a row)
            {
                // all 16 of a thread's float4 of each matrix in flight before any is converted
                const float4* Wa4 = reinterpret_cast<const float4*>(p.Wa + (size_t)h * HID * D);
                const float4* Wb4 = reinterpret_cast<const float4*>(p.Wb + (size_t)h * D * HID);
                constexpr int F4 = HID * D / 4 / kCT;
                float4 v[F4];
#pragma unroll
                for (int i = 0; i < F4; ++i) v[i] = __ldg(Wa4 + i * kCT + tid);
#pragma unroll
                for (int i = 0; i < F4; ++i) {                             // Wa: row = hidden unit, 16 float4 a row
                    const int f = i * kCT + tid, row = f >> 4, col = (f & 15) * 4;
                    *reinterpret_cast<uint2*>(s.wa + sw_off(row, col)) =
                        make_uint2(pack_bf16x2(v[i].x, v[i].y), pack_bf16x2(v[i].z, v[i].w));
                }
#pragma unroll
                for (int i = 0; i < F4; ++i) v[i] = __ldg(Wb4 + i * kCT + tid);
#pragma unroll
                for (int i = 0; i < F4; ++i) {                             // Wb: row = d, 64 float4 a row
                    const int f = i * kCT + tid, d = f >> 6, col = (f & 63) * 4;
                    *reinterpret_cast<uint2*>(s.wb[col / 64] + sw_off(d, col % 64)) =
                        make_uint2(pack_bf16x2(v[i].x, v[i].y), pack_bf16x2(v[i].z, v[i].w));
                }
                fence_proxy_async_smem();
                named_bar_sync(1, kCT);
            }
            // ---- phase 1 over this CTA's tiles
            for (int t = t0; t < t1 && !failed; ++t) {
                bool ok = mbar_wait(&s.full[st], ph, ab);
                if (named_bar_or(1, kCT, !ok)) { failed = true; break; }
                const uint32_t sK = smem_u32(s.stage[st]);
                const uint8_t* vtile = s.stage[st] + TILE;
                // H = K Wa^T
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16_ss(tmem + 256u, sdesc_sw128(sK + kk * 32, 16, 1024), sdesc_sw128(swa + kk * 32, 16, 1024),
                                    kIdH, kk > 0 ? 1u : 0u);
                }
                if (!mma_sync(ok)) { failed = true; break; }
                // A = gelu(H) -> act (bf16); gelu'(H) packed bf16x2 -> TMEM cols 256 + hid/2.  Half hw
                // takes the 64-hidden chunks 2 hw and 2 hw + 1; the packed gelu' overwrites H columns
                // the other half may still read, so it is written back after a barrier
                uint32_t gp[2][2][16];
#pragma unroll
                for (int ci = 0; ci < 2; ++ci) {
                    const int c = 2 * hw + ci;                         // 64 hidden units per chunk
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float hv[16];
                        tmem_ld16(tmem + 256u + (uint32_t)(c * 64 + j * 16) + lane_off, hv);
                        tmem_ld_wait();
                        uint32_t aw[8];
#pragma unroll
                        for (int e = 0; e < 16; e += 2) gelu_and_grad2(hv[e], hv[e + 1], aw[e / 2], gp[ci][j / 2][(j % 2) * 8 + e / 2]);
                        *reinterpret_cast<uint4*>(s.act[c] + sw_off(r, j * 16)) = make_uint4(aw[0], aw[1], aw[2], aw[3]);
                        *reinterpret_cast<uint4*>(s.act[c] + sw_off(r, j * 16 + 8)) = make_uint4(aw[4], aw[5], aw[6], aw[7]);
                    }
                }
                tc_fence_before();
                named_bar_sync(1, kCT);                                // every H column has been read
                tc_fence_after();
#pragma unroll
                for (int ci = 0; ci < 2; ++ci) {
                    const int c = 2 * hw + ci;
                    tmem_st16(tmem + 256u + (uint32_t)(c * 32) + lane_off, gp[ci][0]);
                    tmem_st16(tmem + 256u + (uint32_t)(c * 32 + 16) + lane_off, gp[ci][1]);
                }
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(1, kCT);
                // Y = A Wb^T
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < HID / 16; ++kk)
                        mma_bf16_ss(tmem + 384u, sdesc_sw128(sact + (kk / 4) * (TOK * 128) + (kk % 4) * 32, 16, 1024),
                                    sdesc_sw128(swb + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024), kIdY,
                                    kk > 0 ? 1u : 0u);
                }
                if (!mma_sync(ok)) { failed = true; break; }
                // R = Y - V -> rz (bf16); half hw takes columns 32 hw .. 32 hw + 31
                {
                    float yv[2][16];
#pragma unroll
                    for (int j = 0; j < 2; ++j) tmem_ld16(tmem + 384u + (uint32_t)(hw * 32 + j * 16) + lane_off, yv[j]);
                    tmem_ld_wait();
#pragma unroll
                    for (int cc = 0; cc < 32; cc += 8) {
                        const int c = hw * 32 + cc;
                        const uint4 vv = *reinterpret_cast<const uint4*>(vtile + sw_off(r, c));
                        const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
                        float rr[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            rr[2 * e] = yv[cc / 16][(cc % 16) + 2 * e] - bf16lo_to_f32(vw[e]);
                            rr[2 * e + 1] = yv[cc / 16][(cc % 16) + 2 * e + 1] - bf16hi_to_f32(vw[e]);
                        }
                        uint4 pk;
                        pk.x = pack_bf16x2(rr[0], rr[1]); pk.y = pack_bf16x2(rr[2], rr[3]);
                        pk.z = pack_bf16x2(rr[4], rr[5]); pk.w = pack_bf16x2(rr[6], rr[7]);
                        *reinterpret_cast<uint4*>(s.rz + sw_off(r, c)) = pk;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(1, kCT);
                // gWb^T += A^T R (two hidden halves) and dA_0 = R Wb (hidden 0..127)
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                        for (int kk = 0; kk < TOK / 16; ++kk)
                            mma_bf16_ss(tmem + (uint32_t)(hb * 64),
                                        sdesc_sw128(sact + (2 * hb) * (TOK * 128) + kk * 2048, TOK * 128, 1024),
                                        sdesc_sw128(srz + kk * 2048, 0, 1024), kIdG, (t > t0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16_ss(tmem + 384u, sdesc_sw128(srz + kk * 32, 16, 1024),
                                    sdesc_sw128(swb + kk * 2048, D * 128, 1024), kIdDA, kk > 0 ? 1u : 0u);
                }
                if (!mma_sync(ok)) { failed = true; break; }
                // dH = dA * gelu'(H) for both hidden halves -> act (A is no longer needed)
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    if (half == 1) {
                        if (tid == 0) {
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_bf16_ss(tmem + 384u, sdesc_sw128(srz + kk * 32, 16, 1024),
                                            sdesc_sw128(swb + 2 * (D * 128) + kk * 2048, D * 128, 1024), kIdDA,
                                            kk > 0 ? 1u : 0u);
                        }
                        if (!mma_sync(ok)) { failed = true; break; }
                    }
                    {
                        const int c = hw;                                // 64 hidden units per chunk
                        const int panel = half * 2 + c;
#pragma unroll
                        for (int sub = 0; sub < 2; ++sub) {              // 32 hidden units at a time
                            float da[2][16];
                            float gq[16];
#pragma unroll
                            for (int j = 0; j < 2; ++j)
                                tmem_ld16(tmem + 384u + (uint32_t)(c * 64 + sub * 32 + j * 16) + lane_off, da[j]);
                            tmem_ld16(tmem + 256u + (uint32_t)(half * 64 + c * 32 + sub * 16) + lane_off, gq);
                            tmem_ld_wait();
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                float dh[8];
#pragma unroll
                                for (int i = 0; i < 8; i += 2) {
                                    const uint32_t w = __float_as_uint(gq[(e + i) / 2]);
                                    dh[i] = da[(e + i) / 16][(e + i) % 16] * bf16lo_to_f32(w);
                                    dh[i + 1] = da[(e + i + 1) / 16][(e + i + 1) % 16] * bf16hi_to_f32(w);
                                }
                                uint4 pk;
                                pk.x = pack_bf16x2(dh[0], dh[1]); pk.y = pack_bf16x2(dh[2], dh[3]);
                                pk.z = pack_bf16x2(dh[4], dh[5]); pk.w = pack_bf16x2(dh[6], dh[7]);
                                *reinterpret_cast<uint4*>(s.act[panel] + sw_off(r, sub * 32 + e)) = pk;
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    named_bar_sync(1, kCT);
                }
                if (failed) break;
                // gWa += dH^T K (two hidden halves); frees the K/V stage when done
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                        for (int kk = 0; kk < TOK / 16; ++kk)
                            mma_bf16_ss(tmem + 128u + (uint32_t)(hb * 64),
                                        sdesc_sw128(sact + (2 * hb) * (TOK * 128) + kk * 2048, TOK * 128, 1024),
                                        sdesc_sw128(sK + kk * 2048, 0, 1024), kIdG, (t > t0 || kk > 0) ? 1u : 0u);
                    mma_commit(&s.empty[st]);
                }
                if (!mma_sync(ok)) { failed = true; break; }
                if (++st == STAGES) { st = 0; ph ^= 1u; }
            }
            if (failed) break;
            // ---- update: Wa1 = Wa - eta (2/N) gWa, Wb1 = Wb - eta (2/N) gWb.  With a 2-CTA cluster, CTA
            //      `rank` owns hidden half `rank` (hidden units 128 rank + r): it receives the peer's
            //      partial gradients for that half, forms that half of Wa1 (rows) and Wb1 (columns),
            //      and writes the bf16 operands into its own and the peer's shared memory.  One CTA
            //      (no cluster) owns both halves.
            {
                const bool has = t1 > t0;                             // this CTA accumulated any tile
                const int peer = rank ^ 1;
                float* recv = reinterpret_cast<float*>(s.act[0]);     // [2][128][64]: gWa, gWb^T of my half
                // recv element (m, row, col): float4 chunk swizzled by the row (conflict-free stores)
                auto roff = [](int m, int row, int col) {
                    return (uint32_t)(((m * 128 + row) * 64 + ((((col >> 2) ^ (row & 15))) << 2) + (col & 3)) * 4);
                };
                bool ok = true;
                if (multi) {
                    // (1) my phase 1 is over: the peer may now write my act and weight operands
                    if (tid == 0) mbar_arrive_remote(map_to_rank(smem_u32(&s.free_bar), (uint32_t)peer));
                    // (2) and the peer's phase 1 is over
                    ok = mbar_wait_cluster(&s.free_bar, k & 1u, ab);
                    if (named_bar_or(1, kCT, !ok)) { failed = true; break; }
                    tc_fence_after();
                    // (3) push my partials for the peer's half into the peer's act
                    const int ob = peer;
                    const uint32_t rb = map_to_rank(smem_u32(recv), (uint32_t)peer);
#pragma unroll 1
                    for (int j = 2 * hw; j < 2 * hw + 2; ++j) {
                        float ga[16], gb[16];
                        tmem_ld16(tmem + 128u + (uint32_t)(ob * 64 + j * 16) + lane_off, ga);
                        tmem_ld16(tmem + (uint32_t)(ob * 64 + j * 16) + lane_off, gb);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; e += 4) {
                            const uint4 va = has ? make_uint4(__float_as_uint(ga[e]), __float_as_uint(ga[e + 1]),
                                                              __float_as_uint(ga[e + 2]), __float_as_uint(ga[e + 3]))
                                                 : make_uint4(0u, 0u, 0u, 0u);
                            const uint4 vb = has ? make_uint4(__float_as_uint(gb[e]), __float_as_uint(gb[e + 1]),
                                                              __float_as_uint(gb[e + 2]), __float_as_uint(gb[e + 3]))
                                                 : make_uint4(0u, 0u, 0u, 0u);
                            st_cluster_v4(rb + roff(0, r, j * 16 + e), va);
                            st_cluster_v4(rb + roff(1, r, j * 16 + e), vb);
                        }
                    }
                    mbar_arrive_remote(map_to_rank(smem_u32(&s.xbar), (uint32_t)peer));   // after my stores
                    // (4) the peer's partials for my half
                    ok = mbar_wait_cluster(&s.xbar, k & 1u, ab);
                    if (named_bar_or(1, kCT, !ok)) { failed = true; break; }
                }
                const float* Wa = p.Wa + (size_t)h * HID * D;
                const float* Wb = p.Wb + (size_t)h * D * HID;
                const uint32_t pwa = multi ? map_to_rank(swa, (uint32_t)peer) : 0u;
                const uint32_t pwb = multi ? map_to_rank(swb, (uint32_t)peer) : 0u;
#pragma unroll 1
                for (int hb = multi ? rank : 0; hb < (multi ? rank + 1 : 2); ++hb) {
                    const int hid = hb * 128 + r;
                    const int c0 = hw * 32;                           // this half's 32 columns
                    // the initial weights of this thread's entries, all loads in flight at once
                    float4 wa0[8];
                    float wb0[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) wa0[i] = __ldg(reinterpret_cast<const float4*>(Wa + (size_t)hid * D + c0) + i);
#pragma unroll
                    for (int dd = 0; dd < 32; ++dd) wb0[dd] = __ldg(Wb + (size_t)(c0 + dd) * HID + hid);
                    float ga[2][16], gb[2][16];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        tmem_ld16(tmem + 128u + (uint32_t)(hb * 64 + c0 + j * 16) + lane_off, ga[j]);
                        tmem_ld16(tmem + (uint32_t)(hb * 64 + c0 + j * 16) + lane_off, gb[j]);
                    }
                    tmem_ld_wait();
                    if (!has) {
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int e = 0; e < 16; ++e) { ga[j][e] = 0.f; gb[j][e] = 0.f; }
                    }
                    if (multi) {                                      // + the peer's partial (two terms: any order)
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                ga[j][e] += *reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(recv) + roff(0, r, c0 + j * 16 + e));
                                gb[j][e] += *reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(recv) + roff(1, r, c0 + j * 16 + e));
                            }
                    }
#pragma unroll
                    for (int cc = 0; cc < 32; cc += 8) {
                        const int c = c0 + cc;
                        float w[8];
                        const float4 w0a = wa0[cc / 4], w0b = wa0[cc / 4 + 1];
                        const float w0[8] = {w0a.x, w0a.y, w0a.z, w0a.w, w0b.x, w0b.y, w0b.z, w0b.w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            w[e] = w0[e] - p.eta_scale * ga[(cc + e) / 16][(cc + e) % 16];
                            if (p.Wa_out) p.Wa_out[((size_t)u * HID + hid) * D + c + e] = w[e];
                        }
                        uint4 pk;
                        pk.x = pack_bf16x2(w[0], w[1]); pk.y = pack_bf16x2(w[2], w[3]);
                        pk.z = pack_bf16x2(w[4], w[5]); pk.w = pack_bf16x2(w[6], w[7]);
                        *reinterpret_cast<uint4*>(s.wa + sw_off(hid, c)) = pk;
                        if (multi) st_cluster_v4(pwa + sw_off(hid, c), pk);
                    }
#pragma unroll
                    for (int dd = 0; dd < 32; ++dd) {
                        const int d = c0 + dd;
                        const float w = wb0[dd] - p.eta_scale * gb[dd / 16][dd % 16];
                        if (p.Wb_out) p.Wb_out[((size_t)u * D + d) * HID + hid] = w;
                        const __nv_bfloat16 wb16 = __float2bfloat16_rn(w);
                        const uint32_t off = (uint32_t)((hid / 64) * (D * 128)) + sw_off(d, hid % 64);
                        *reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(s.wb[0]) + off) = wb16;
                        // hidden units 2i, 2i+1 are adjacent in a row: even lanes store both to the peer
                        const uint32_t mine = (uint32_t)__bfloat16_as_ushort(wb16);
                        const uint32_t next = __shfl_down_sync(0xffffffffu, mine, 1);
                        if (multi && (lane & 1) == 0) st_cluster_u32(pwb + off, mine | (next << 16));
                    }
                }
                if (multi) {
                    mbar_arrive_remote(map_to_rank(smem_u32(&s.wbar), (uint32_t)peer));   // after my stores
                    // (5) the peer's half of the operands
                    ok = mbar_wait_cluster(&s.wbar, k & 1u, ab);
                    if (named_bar_or(1, kCT, !ok)) { failed = true; break; }
                }
                fence_proxy_async_smem();                             // the operands are read by the tensor cores
                tc_fence_before();
                named_bar_sync(1, kCT);
            }
            // ---- phase 2: Z = gelu(Q Wa1^T) Wb1^T over this CTA's tiles
            for (int t = t0; t < t1 && !failed; ++t) {
                bool ok = mbar_wait(&s.full[st], ph, ab);
                if (named_bar_or(1, kCT, !ok)) { failed = true; break; }
                const uint32_t sQ = smem_u32(s.stage[st]);
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16_ss(tmem + 256u, sdesc_sw128(sQ + kk * 32, 16, 1024), sdesc_sw128(swa + kk * 32, 16, 1024),
                                    kIdH, kk > 0 ? 1u : 0u);
                }
                if (!mma_sync(ok)) { failed = true; break; }
#pragma unroll 1
                for (int c = 2 * hw; c < 2 * hw + 2; ++c) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float hv[16];
                        tmem_ld16(tmem + 256u + (uint32_t)(c * 64 + j * 16) + lane_off, hv);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; e += 8)
                            *reinterpret_cast<uint4*>(s.act[c] + sw_off(r, j * 16 + e)) =
                                make_uint4(gelu_only2(hv[e], hv[e + 1]), gelu_only2(hv[e + 2], hv[e + 3]),
                                           gelu_only2(hv[e + 4], hv[e + 5]), gelu_only2(hv[e + 6], hv[e + 7]));
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(1, kCT);
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < HID / 16; ++kk)
                        mma_bf16_ss(tmem + 384u, sdesc_sw128(sact + (kk / 4) * (TOK * 128) + (kk % 4) * 32, 16, 1024),
                                    sdesc_sw128(swb + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024), kIdY,
                                    kk > 0 ? 1u : 0u);
                    mma_commit(&s.empty[st]);
                }
                if (!mma_sync(ok)) { failed = true; break; }
                if (tid == 0 && zn > 0) bulk_wait_read<0>();          // the previous Z tile has left rz
                named_bar_sync(1, kCT);
                {
                    float zv[2][16];
#pragma unroll
                    for (int j = 0; j < 2; ++j) tmem_ld16(tmem + 384u + (uint32_t)(hw * 32 + j * 16) + lane_off, zv[j]);
                    tmem_ld_wait();
#pragma unroll
                    for (int cc = 0; cc < 32; cc += 8) {
                        const int c = hw * 32 + cc;
                        uint4 pk;
                        pk.x = pack_bf16x2(zv[cc / 16][cc % 16], zv[cc / 16][cc % 16 + 1]);
                        pk.y = pack_bf16x2(zv[cc / 16][cc % 16 + 2], zv[cc / 16][cc % 16 + 3]);
                        pk.z = pack_bf16x2(zv[cc / 16][cc % 16 + 4], zv[cc / 16][cc % 16 + 5]);
                        pk.w = pack_bf16x2(zv[cc / 16][cc % 16 + 6], zv[cc / 16][cc % 16 + 7]);
                        *reinterpret_cast<uint4*>(s.rz + sw_off(r, c)) = pk;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(1, kCT);
                if (tid == 0) {
                    tma_store_4d(&tmZ, s.rz, 0, t * TOK, h, bi);
                    bulk_commit();
                }
                ++zn;
                if (++st == STAGES) { st = 0; ph ^= 1u; }
            }
            if (tid == 0) bulk_wait<0>();                          // rz is reused by the next unit
            named_bar_sync(1, kCT);
        }
        if (tid == 0) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    // no CTA of the cluster exits while its peer may still write into its shared memory
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace mlp

size_t mlp_ws_bytes(const ttt_shape&) { return kWsHeader; }   // error word only

ttt_status launch_mlp(const Call& c) {
    using namespace mlp;
    if (c.dtype != TTT_BF16 || c.hidden != HID) return TTT_ERR_UNSUPPORTED;
    const long long units = (long long)c.batch * c.heads;
    Params p{};
    p.U = (int)units;
    p.heads = c.heads;
    p.N = c.N;
    p.tpu = (c.N + TOK - 1) / TOK;
    p.eta_scale = c.eta * (2.0f / (float)c.N);
    p.Wa = c.W0;
    p.Wb = c.W0b;
    p.Wa_out = c.W1_out;
    p.Wb_out = c.W1b_out;
    p.err = reinterpret_cast<uint32_t*>(c.ws);
    p.wait_ns = c.wait_ns;
    CUtensorMap tmK, tmV, tmQ, tmZ;
    if (!make_tmap_tokens(&tmK, c.K, c, TOK) || !make_tmap_tokens(&tmV, c.V, c, TOK) ||
        !make_tmap_tokens(&tmQ, c.Q, c, TOK) || !make_tmap_tokens(&tmZ, c.Z, c, TOK))
        return TTT_ERR_INVALID_ARG;
    const size_t smem = sizeof(Smem) + 1024;
    cudaFuncSetAttribute(mlp_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // Two CTAs per unit (a cluster; each takes half of the tokens) while that still gives every unit
    // its own pair of SMs; otherwise one CTA per unit, persistent over units.
    const int cs = (c.num_sms >= 2 && p.tpu >= 2 && 2LL * units <= c.num_sms) ? 2 : 1;
    p.CS = cs;
    const int ncl = (int)std::max<long long>(1, std::min<long long>(units, c.num_sms / cs));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(ncl * cs));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return check_launch(cudaLaunchKernelEx(&cfg, mlp_fused, tmK, tmV, tmQ, tmZ, p));
}

}  // namespace ttt
