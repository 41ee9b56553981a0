// linear.cu -- linear inner model f(x) = W x of the TTT layer (one d x d state per head; Vision-TTT
// paper notes, section 关键设计 1), one full-batch step of the L2 loss (press article "CVPR 2026
// Oral | 清華+阿里發布ViT3", Observation 2) written in Gram form:
//     G = sum_n k_n k_n^T,   C = sum_n v_n k_n^T,   W1 = W0 - eta (2/N) (W0 G - C),   z_n = W1 q_n.
//
// bf16 path: ONE persistent kernel (lin_fused_bf16), one CTA per SM, that pulls work items from an
// ordered queue in global memory (an atomic ticket):
//   items [0, U*C1)          phase 1: chunk j of unit u (TPC1 tiles of 128 tokens).  The chunk's
//                            [K | V]^T K  (128 x 64 fp32: rows 0..63 = G_j, rows 64..127 = C_j) is
//                            accumulated in tensor memory; the epilogue forms P_j = W0 G_j - C_j
//                            and writes it to partial slot (u, j).
//   items [U*C1, U*(C1+C2))  phase 2: chunk j of unit u (TPC2 Q tiles): Z = Q W1^T.
// The CTA that completes the last chunk of a unit (atomic arrival count, no waiting) sums the
// unit's slots in chunk order -- a fixed order, so results are bitwise deterministic whichever CTA
// ran which chunk -- forms W1 = W0 - eta (2/N) sum_j P_j in fp32, stores it as bf16 and raises the
// unit's ready flag.  A
// phase-2 item waits (bounded) for that flag before loading W1.  Every phase-1 item precedes every
// phase-2 item in the queue, so the CTAs a phase-2 item waits on have claimed their work already
// and are running; their MMA and epilogue warps never wait on their own producer's later items.
// Merges therefore overlap the streaming of other units and the phase boundary costs nothing.
//
// Roles (192 threads): warp 0 lane 0 claims items and issues TMA loads (128-byte swizzle); warp 1
// lane 0 issues tcgen05.mma; warps 2..5 drain tensor memory (partial slots, or bf16 Z tiles stored
// by TMA) and run merges.  Phase 1 uses one MMA stream for G and C: A = [K | V]^T (M = 128,
// MN-major straight from the token-major tiles), B = K (N = 64, MN-major), K-dim = tokens.
// Phase 2: A = Q tile (M = 128 tokens, K-major), B = W1 (bf16, K-major).
//
// fp32 path (lin_p1_f32 / lin_p2_f32): plain fp32 FMA kernels (fp32 accuracy), static partition,
// the same deterministic last-CTA merge.
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace lin {

constexpr int D = 64;
constexpr int TOK = 128;                    // tokens per tile
constexpr int TILE_BYTES = TOK * D * 2;     // one bf16 tile: 16 KB
constexpr int STAGES = 4;                   // 32 KB each: a K+V tile pair or one Q tile
constexpr int ACC = 4;                      // tensor-memory accumulators of 64 fp32 columns
constexpr int WQ = 4;                       // work-descriptor ring
constexpr int TPC1 = 8;                     // tiles per phase-1 chunk
constexpr int TPC2 = 4;                     // tiles per phase-2 chunk
constexpr int kPartialFloats = 2 * D * D;   // [G ; C] = 128 x 64
constexpr int kThreadsTc = 192;
constexpr int kW0tPitch = D + 4;           // row pitch of the transposed W0 in shared memory
constexpr uint32_t kIdescP1 = idesc_bf16_f32(128, 64, true, true);
constexpr uint32_t kIdescP2 = idesc_bf16_f32(128, 64, false, false);

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------------------------------------------
// Merge of one unit by NT threads (tid in [0, NT)): fixed-order sum of nslots consecutive partial
// slots starting at slot0, then W1 = W0 - eta_scale * (W0 G - C).
//   gc: 128 x 64 floats of shared memory, w0t: 64 x kW0tPitch floats of shared memory.
// ------------------------------------------------------------------------------------------------
struct MergeOut {
    float eta_scale;            // eta * 2 / N
    const float* W0;            // [heads][64][64]
    const float* partials;      // [slots][128][64]
    float* W1_out;              // nullable [units][64][64]
    __nv_bfloat16* W1_bf16;     // nullable [units][64][64]
    float* W1_f32;              // nullable [units][64][64]
};

template <int NT, int BAR_ID>
__device__ void merge_unit(const MergeOut& m, int u, int h, size_t slot0, int nslots, int tid, float* gc, float* w0t) {
    constexpr int PER = kPartialFloats / 4 / NT;     // float4 per thread and slot
    constexpr int SB = 2;                             // slots per batch of loads in flight
    constexpr int W4 = D * D / 4 / NT;                // float4 of W0 per thread
    {
        // W0 goes to shared memory transposed: w0t[k][i] = W0[i][k] (row pitch kW0tPitch)
        float4 wv[W4];
        const float4* W0h = reinterpret_cast<const float4*>(m.W0 + (size_t)h * D * D);
#pragma unroll
        for (int i = 0; i < W4; ++i) wv[i] = __ldg(W0h + i * NT + tid);
#pragma unroll
        for (int i = 0; i < W4; ++i) {
            const int e = (i * NT + tid) * 4;
            const int row = e / D, col = e % D;
            w0t[(col + 0) * kW0tPitch + row] = wv[i].x;
            w0t[(col + 1) * kW0tPitch + row] = wv[i].y;
            w0t[(col + 2) * kW0tPitch + row] = wv[i].z;
            w0t[(col + 3) * kW0tPitch + row] = wv[i].w;
        }
    }
    float4* g4 = reinterpret_cast<float4*>(gc);
    for (int s0 = 0; s0 < nslots; s0 += SB) {
        float4 v[SB][PER];
#pragma unroll
        for (int b = 0; b < SB; ++b) {
            if (s0 + b < nslots) {
                const float4* src = reinterpret_cast<const float4*>(m.partials + (slot0 + s0 + b) * kPartialFloats);
#pragma unroll
                for (int i = 0; i < PER; ++i) v[b][i] = __ldcg(src + i * NT + tid);
            }
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            float4 a = (s0 == 0) ? make_float4(0.f, 0.f, 0.f, 0.f) : g4[i * NT + tid];
#pragma unroll
            for (int b = 0; b < SB; ++b) {
                if (s0 + b < nslots) { a.x += v[b][i].x; a.y += v[b][i].y; a.z += v[b][i].z; a.w += v[b][i].w; }
            }
            g4[i * NT + tid] = a;
        }
    }
    named_bar_sync(BAR_ID, NT);

    // (W0 G)[i][j] for a 4 x CJ block of rows i0.. and columns j0.. per thread
    constexpr int CJ = D * D / (NT * 4);              // 8 (NT = 128) or 4 (NT = 256)
    constexpr int JG = D / CJ;                        // column groups
    const int i0 = (tid / JG) * 4, j0 = (tid % JG) * CJ;
    float acc[4][CJ];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < CJ; ++b) acc[a][b] = 0.f;
#pragma unroll 2
    for (int k = 0; k < D; ++k) {
        const float4 wk = *reinterpret_cast<const float4*>(w0t + k * kW0tPitch + i0);
        float gk[CJ];
#pragma unroll
        for (int b = 0; b < CJ; b += 4) {
            const float4 g = *reinterpret_cast<const float4*>(gc + k * D + j0 + b);
            gk[b] = g.x; gk[b + 1] = g.y; gk[b + 2] = g.z; gk[b + 3] = g.w;
        }
        const float wr[4] = {wk.x, wk.y, wk.z, wk.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < CJ; ++b) acc[a][b] = fmaf(wr[a], gk[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + a;
        float w1[CJ];
#pragma unroll
        for (int b = 0; b < CJ; ++b)
            w1[b] = w0t[(j0 + b) * kW0tPitch + i] - m.eta_scale * (acc[a][b] - gc[(D + i) * D + j0 + b]);
        const size_t row = ((size_t)u * D + i) * D + j0;
        if (m.W1_out) {
#pragma unroll
            for (int q = 0; q < CJ / 4; ++q)
                reinterpret_cast<float4*>(m.W1_out + row)[q] = make_float4(w1[4 * q], w1[4 * q + 1], w1[4 * q + 2], w1[4 * q + 3]);
        }
        if (m.W1_f32) {
#pragma unroll
            for (int q = 0; q < CJ / 4; ++q)
                reinterpret_cast<float4*>(m.W1_f32 + row)[q] = make_float4(w1[4 * q], w1[4 * q + 1], w1[4 * q + 2], w1[4 * q + 3]);
        }
        if (m.W1_bf16) {
#pragma unroll
            for (int q = 0; q < CJ / 8; ++q) {
                uint4 pk;
                pk.x = pack_bf16x2(w1[8 * q + 0], w1[8 * q + 1]);
                pk.y = pack_bf16x2(w1[8 * q + 2], w1[8 * q + 3]);
                pk.z = pack_bf16x2(w1[8 * q + 4], w1[8 * q + 5]);
                pk.w = pack_bf16x2(w1[8 * q + 6], w1[8 * q + 7]);
                reinterpret_cast<uint4*>(m.W1_bf16 + row)[q] = pk;
            }
            if (CJ % 8) {                                    // CJ == 4: half a 16-byte chunk
                uint2 pk;
                pk.x = pack_bf16x2(w1[0], w1[1]);
                pk.y = pack_bf16x2(w1[2], w1[3]);
                *reinterpret_cast<uint2*>(m.W1_bf16 + row) = pk;
            }
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Fused-path phase-1 helpers.  The epilogue of every chunk j turns its accumulator [G_j ; C_j] into
// P_j = W0 G_j - C_j (64 x 64 fp32), so that W1 = W0 - eta (2/N) sum_j P_j and the unit's merge is a
// plain ordered sum.  gc holds [G_j ; C_j] in shared memory with its 16-byte chunks XOR-swizzled by
// (row & 15); w0t holds W0 transposed.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float4* gc_chunk(float* gc, int row, int chunk) {
    return reinterpret_cast<float4*>(gc + row * D) + (chunk ^ (row & 15));
}

// W0 of head h -> w0t[k][i] = W0[i][k]  (128 threads)
__device__ __forceinline__ void load_w0t(const float* W0, int h, int tid, float* w0t) {
    float4 wv[8];
    const float4* W0h = reinterpret_cast<const float4*>(W0 + (size_t)h * D * D);
#pragma unroll
    for (int i = 0; i < 8; ++i) wv[i] = __ldg(W0h + i * 128 + tid);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = (i * 128 + tid) * 4;
        const int row = e / D, col = e % D;
        w0t[(col + 0) * kW0tPitch + row] = wv[i].x;
        w0t[(col + 1) * kW0tPitch + row] = wv[i].y;
        w0t[(col + 2) * kW0tPitch + row] = wv[i].z;
        w0t[(col + 3) * kW0tPitch + row] = wv[i].w;
    }
}

// P = W0 G - C for this thread's 4 x 8 block (rows i0.., columns j0..), written to dst (64 x 64 fp32).
__device__ __forceinline__ void chunk_product(const float* gc, const float* w0t, int tid, float* dst) {
    const int i0 = (tid >> 3) * 4, j0 = (tid & 7) * 8;
    float acc[4][8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
#pragma unroll 2
    for (int k = 0; k < D; ++k) {
        const float4 wk = *reinterpret_cast<const float4*>(w0t + k * kW0tPitch + i0);
        const float4 g0 = *gc_chunk(const_cast<float*>(gc), k, j0 / 4);
        const float4 g1 = *gc_chunk(const_cast<float*>(gc), k, j0 / 4 + 1);
        const float gk[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float wr[4] = {wk.x, wk.y, wk.z, wk.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(wr[a], gk[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + a;
        const float4 c0 = *gc_chunk(const_cast<float*>(gc), D + i, j0 / 4);
        const float4 c1 = *gc_chunk(const_cast<float*>(gc), D + i, j0 / 4 + 1);
        float4* out = reinterpret_cast<float4*>(dst + i * D + j0);
        out[0] = make_float4(acc[a][0] - c0.x, acc[a][1] - c0.y, acc[a][2] - c0.z, acc[a][3] - c0.w);
        out[1] = make_float4(acc[a][4] - c1.x, acc[a][5] - c1.y, acc[a][6] - c1.z, acc[a][7] - c1.w);
    }
}

// Merge of unit u: S = sum_j P_j over the C1 chunk slots in chunk order, W1 = W0 - eta_scale * S.
__device__ __forceinline__ void merge_chunks(const MergeOut& m, int u, int nslots, const float* slots, int tid,
                                             const float* w0t) {
    constexpr int E4 = D * D / 4 / 128;               // 8 float4 per thread
    float4 acc[E4];
#pragma unroll
    for (int i = 0; i < E4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nslots; s0 += 3) {
        float4 v[3][E4];
#pragma unroll
        for (int b = 0; b < 3; ++b)
            if (s0 + b < nslots) {
                const float4* src = reinterpret_cast<const float4*>(slots + (size_t)(s0 + b) * D * D);
#pragma unroll
                for (int i = 0; i < E4; ++i) v[b][i] = __ldcg(src + i * 128 + tid);
            }
#pragma unroll
        for (int b = 0; b < 3; ++b)
            if (s0 + b < nslots) {
#pragma unroll
                for (int i = 0; i < E4; ++i) {
                    acc[i].x += v[b][i].x; acc[i].y += v[b][i].y; acc[i].z += v[b][i].z; acc[i].w += v[b][i].w;
                }
            }
    }
#pragma unroll
    for (int i = 0; i < E4; ++i) {
        const int e = (i * 128 + tid) * 4;
        const int row = e / D, col = e % D;
        const float4 w1 = make_float4(w0t[(col + 0) * kW0tPitch + row] - m.eta_scale * acc[i].x,
                                      w0t[(col + 1) * kW0tPitch + row] - m.eta_scale * acc[i].y,
                                      w0t[(col + 2) * kW0tPitch + row] - m.eta_scale * acc[i].z,
                                      w0t[(col + 3) * kW0tPitch + row] - m.eta_scale * acc[i].w);
        const size_t off = (size_t)u * D * D + e;
        if (m.W1_out) *reinterpret_cast<float4*>(m.W1_out + off) = w1;
        uint2 pk;
        pk.x = pack_bf16x2(w1.x, w1.y);
        pk.y = pack_bf16x2(w1.z, w1.w);
        *reinterpret_cast<uint2*>(m.W1_bf16 + off) = pk;
    }
}

// ------------------------------------------------------------------------------------------------
// bf16: the fused persistent kernel
// ------------------------------------------------------------------------------------------------
enum : int { W_STOP = 0, W_P1 = 1, W_P2 = 2 };
struct Work {
    int kind, u, t0, t1;
    unsigned item;
};

struct FusedParams {
    int heads, tpu, U, C1, C2;
    unsigned total;             // U * (C1 + C2)
    MergeOut m;
    unsigned* counters;         // [U] phase-1 arrivals
    uint32_t* ready;            // [U] W1 published
    unsigned* ctrl;             // [0] next item, [1] finished CTAs
    uint32_t* err;
};

__device__ __forceinline__ Work decode_work(const FusedParams& p, unsigned item) {
    Work w;
    w.item = item;
    const unsigned n1 = (unsigned)p.U * (unsigned)p.C1;
    if (item >= p.total) {
        w.kind = W_STOP; w.u = 0; w.t0 = 0; w.t1 = 0;
    } else if (item < n1) {
        w.kind = W_P1;
        w.u = (int)(item / p.C1);
        w.t0 = (int)(item % p.C1) * TPC1;
        w.t1 = min(p.tpu, w.t0 + TPC1);
    } else {
        const unsigned k = item - n1;
        w.kind = W_P2;
        w.u = (int)(k / p.C2);
        w.t0 = (int)(k % p.C2) * TPC2;
        w.t1 = min(p.tpu, w.t0 + TPC2);
    }
    return w;
}

struct FusedSmem {
    uint8_t stage[STAGES][2 * TILE_BYTES];   // 1024-aligned
    uint8_t zbuf[2][TILE_BYTES];             // Z staging; doubles as the merge's [G ; C] buffer
    uint8_t w1[2][D * D * 2];
    float w0[D * kW0tPitch];
    uint64_t full[STAGES], empty[STAGES];
    uint64_t acc_full[ACC], acc_empty[ACC];
    uint64_t w_full[2], w_empty[2];
    uint64_t work_full[WQ], work_empty[WQ];
    Work wq[WQ];
    uint32_t tmem_base;
    int abort_flag, last_flag, done_flag;
};

__device__ __forceinline__ void producer(FusedSmem& s, const FusedParams& p, const CUtensorMap* tmK,
                                         const CUtensorMap* tmV, const CUtensorMap* tmQ, const CUtensorMap* tmW1,
                                         const Abort& ab) {
    int wqi = 0; uint32_t wqph = 0;
    int st = 0; uint32_t stph = 0;
    int p2n = 0;
    for (;;) {
        const unsigned item = atomicAdd(p.ctrl, 1u);
        const Work w = decode_work(p, item);
        if (!mbar_wait(&s.work_empty[wqi], wqph ^ 1u, ab)) return;
        s.wq[wqi] = w;
        mbar_arrive(&s.work_full[wqi]);
        if (++wqi == WQ) { wqi = 0; wqph ^= 1u; }
        if (w.kind == W_STOP) return;
        const int b = w.u / p.heads, h = w.u % p.heads;
        if (w.kind == W_P1) {
            for (int t = w.t0; t < w.t1; ++t) {
                if (!mbar_wait(&s.empty[st], stph ^ 1u, ab)) return;
                mbar_arrive_expect_tx(&s.full[st], 2 * TILE_BYTES);
                tma_load_4d(s.stage[st], tmK, &s.full[st], 0, t * TOK, h, b);
                tma_load_4d(s.stage[st] + TILE_BYTES, tmV, &s.full[st], 0, t * TOK, h, b);
                if (++st == STAGES) { st = 0; stph ^= 1u; }
            }
        } else {
            const int wsl = p2n & 1;
            for (int t = w.t0; t < w.t1; ++t) {
                if (!mbar_wait(&s.empty[st], stph ^ 1u, ab)) return;
                mbar_arrive_expect_tx(&s.full[st], TILE_BYTES);
                tma_load_4d(s.stage[st], tmQ, &s.full[st], 0, t * TOK, h, b);
                if (++st == STAGES) { st = 0; stph ^= 1u; }
                if (t == w.t0) {                               // W1 of the unit, once it is published
                    if (!mbar_wait(&s.w_empty[wsl], (((uint32_t)p2n >> 1) & 1u) ^ 1u, ab)) return;
                    if (!wait_flag(p.ready + w.u, ab)) return;
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(&s.w_full[wsl], D * D * 2);
                    tma_load_2d(s.w1[wsl], tmW1, &s.w_full[wsl], 0, w.u * D);
                }
            }
            ++p2n;
        }
    }
}

__device__ __forceinline__ void mma_issuer(FusedSmem& s, uint32_t tmem, const Abort& ab) {
    int wqi = 0; uint32_t wqph = 0;
    int st = 0; uint32_t stph = 0;
    int ai = 0; uint32_t aph = 0;
    int p2n = 0;
    for (;;) {
        if (!mbar_wait(&s.work_full[wqi], wqph, ab)) return;
        const Work w = s.wq[wqi];
        mbar_arrive(&s.work_empty[wqi]);
        if (++wqi == WQ) { wqi = 0; wqph ^= 1u; }
        if (w.kind == W_STOP) return;
        if (w.kind == W_P1) {
            if (!mbar_wait(&s.acc_empty[ai], aph ^ 1u, ab)) return;
            tc_fence_after();
            const uint32_t dacc = tmem + (uint32_t)(ai * 64);
            for (int t = w.t0; t < w.t1; ++t) {
                if (!mbar_wait(&s.full[st], stph, ab)) return;
                tc_fence_after();
                const uint32_t sK = smem_u32(s.stage[st]);
#pragma unroll
                for (int kk = 0; kk < TOK / 16; ++kk) {
                    // 16 tokens per MMA = two 8-row groups (2 x 1024 bytes); V sits TILE_BYTES after K
                    const uint64_t ad = sdesc_sw128(sK + kk * 2048, TILE_BYTES, 1024);
                    const uint64_t bd = sdesc_sw128(sK + kk * 2048, TILE_BYTES, 1024);
                    mma_bf16_ss(dacc, ad, bd, kIdescP1, (t > w.t0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&s.empty[st]);
                if (++st == STAGES) { st = 0; stph ^= 1u; }
            }
            mma_commit(&s.acc_full[ai]);
            if (++ai == ACC) { ai = 0; aph ^= 1u; }
        } else {
            const int wsl = p2n & 1;
            if (!mbar_wait(&s.w_full[wsl], ((uint32_t)p2n >> 1) & 1u, ab)) return;
            const uint32_t sW = smem_u32(s.w1[wsl]);
            for (int t = w.t0; t < w.t1; ++t) {
                if (!mbar_wait(&s.acc_empty[ai], aph ^ 1u, ab)) return;
                if (!mbar_wait(&s.full[st], stph, ab)) return;
                tc_fence_after();
                const uint32_t sQ = smem_u32(s.stage[st]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(sQ + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sW + kk * 32, 16, 1024);
                    mma_bf16_ss(tmem + (uint32_t)(ai * 64), ad, bd, kIdescP2, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s.empty[st]);
                mma_commit(&s.acc_full[ai]);
                if (++st == STAGES) { st = 0; stph ^= 1u; }
                if (++ai == ACC) { ai = 0; aph ^= 1u; }
            }
            mma_commit(&s.w_empty[wsl]);
            ++p2n;
        }
    }
}

__device__ __forceinline__ void epilogue(FusedSmem& s, const FusedParams& p, uint32_t tmem, const CUtensorMap* tmZ,
                                         const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                                   // tensor-memory lane quarter of this warp
    const int r = q * 32 + lane;                              // row of the accumulator
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int wqi = 0; uint32_t wqph = 0;
    int ai = 0; uint32_t aph = 0;
    int zn = 0;
    for (;;) {
        bool ok = mbar_wait(&s.work_full[wqi], wqph, ab);
        __syncwarp();
        const Work w = s.wq[wqi];
        if (named_bar_or(1, 128, !ok || ab.raised())) break;  // uniform decision of the 4 warps
        if (tid == 0) mbar_arrive(&s.work_empty[wqi]);
        if (++wqi == WQ) { wqi = 0; wqph ^= 1u; }
        if (w.kind == W_STOP) break;
        const int b = w.u / p.heads, h = w.u % p.heads;
        if (w.kind == W_P1) {
            load_w0t(p.m.W0, h, tid, s.w0);                  // overlaps the wait for the accumulator
            ok = mbar_wait(&s.acc_full[ai], aph, ab);
            if (tid == 0) bulk_wait_read<0>();                // gc aliases the Z staging area
            if (named_bar_or(1, 128, !ok)) break;
            __syncwarp();
            tc_fence_after();
            float* gc = reinterpret_cast<float*>(s.zbuf[0]);
#pragma unroll
            for (int j = 0; j < D; j += 16) {
                float v[16];
                tmem_ld16(tmem + (uint32_t)(ai * 64 + j) + lane_off, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; e += 4) *gc_chunk(gc, r, (j + e) / 4) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            }
            tc_fence_before();
            mbar_arrive(&s.acc_empty[ai]);
            if (++ai == ACC) { ai = 0; aph ^= 1u; }
            named_bar_sync(1, 128);
            chunk_product(gc, s.w0, tid, const_cast<float*>(p.m.partials) + (size_t)w.item * D * D);
            __threadfence();
            named_bar_sync(1, 128);
            if (tid == 0) {
                const unsigned old = atomicAdd(p.counters + w.u, 1u);
                s.last_flag = (old + 1u == (unsigned)p.C1) ? 1 : 0;
            }
            named_bar_sync(1, 128);
            if (s.last_flag) {
                __threadfence();
                merge_chunks(p.m, w.u, p.C1, p.m.partials + (size_t)w.u * p.C1 * D * D, tid, s.w0);
                fence_proxy_async_global();                   // W1 is read next by TMA (async proxy)
                __threadfence();
                named_bar_sync(1, 128);
                if (tid == 0) {
                    p.counters[w.u] = 0u;
                    st_release_gpu(p.ready + w.u, 1u);
                }
            }
            named_bar_sync(1, 128);
        } else {
            bool fail = false;
            for (int t = w.t0; t < w.t1; ++t) {
                ok = mbar_wait(&s.acc_full[ai], aph, ab);
                const int zb = zn & 1;
                if (tid == 0 && zn >= 2) bulk_wait_read<1>();  // staging buffer zb is free again
                if (named_bar_or(1, 128, !ok)) { fail = true; break; }
                __syncwarp();
                tc_fence_after();
                uint8_t* zrow = s.zbuf[zb] + r * 128;
#pragma unroll
                for (int j = 0; j < D; j += 16) {
                    float v[16];
                    tmem_ld16(tmem + (uint32_t)(ai * 64 + j) + lane_off, v);
                    tmem_ld_wait();
                    uint4 lo, hi;
                    lo.x = pack_bf16x2(v[0], v[1]);   lo.y = pack_bf16x2(v[2], v[3]);
                    lo.z = pack_bf16x2(v[4], v[5]);   lo.w = pack_bf16x2(v[6], v[7]);
                    hi.x = pack_bf16x2(v[8], v[9]);   hi.y = pack_bf16x2(v[10], v[11]);
                    hi.z = pack_bf16x2(v[12], v[13]); hi.w = pack_bf16x2(v[14], v[15]);
                    const int c0 = j / 8;                         // 16-byte chunk of columns j..j+7
                    *reinterpret_cast<uint4*>(zrow + ((c0 ^ (r & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(zrow + (((c0 + 1) ^ (r & 7)) << 4)) = hi;
                }
                tc_fence_before();
                mbar_arrive(&s.acc_empty[ai]);
                if (++ai == ACC) { ai = 0; aph ^= 1u; }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (tid == 0) {
                    tma_store_4d(tmZ, s.zbuf[zb], 0, t * TOK, h, b);
                    bulk_commit();
                }
                ++zn;
            }
            if (fail) break;
        }
    }
    if (tid == 0) bulk_wait<0>();
}

__global__ void __launch_bounds__(kThreadsTc, 1)
lin_fused_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmZ,
               const __grid_constant__ CUtensorMap tmW1, const FusedParams p) {
    extern __shared__ uint8_t smem_raw[];
    FusedSmem& s = *reinterpret_cast<FusedSmem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        for (int i = 0; i < ACC; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s.w_full[i], 1); mbar_init(&s.w_empty[i], 1); }
        for (int i = 0; i < WQ; ++i) { mbar_init(&s.work_full[i], 1); mbar_init(&s.work_empty[i], 2); }
        fence_barrier_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmQ); prefetch_tmap(&tmZ); prefetch_tmap(&tmW1);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 256); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        if (lane == 0) producer(s, p, &tmK, &tmV, &tmQ, &tmW1, ab);
    } else if (warp == 1) {
        if (lane == 0) mma_issuer(s, tmem, ab);
    } else {
        epilogue(s, p, tmem, &tmZ, ab);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
    // The last CTA to finish re-arms the queue and the ready flags for the next call.
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicAdd(p.ctrl + 1, 1u);
        s.done_flag = (old + 1u == gridDim.x) ? 1 : 0;
    }
    __syncthreads();
    if (s.done_flag) {
        __threadfence();
        for (int u = threadIdx.x; u < p.U; u += blockDim.x) p.ready[u] = 0u;
        if (threadIdx.x == 0) { p.ctrl[0] = 0u; p.ctrl[1] = 0u; }
    }
}

// ------------------------------------------------------------------------------------------------
// fp32 path (plain FMA): static partition of 128-token tiles over CTAs, the same merge.
// ------------------------------------------------------------------------------------------------
constexpr int kThreadsF32 = 256;
constexpr int F32_CHUNK = 32;   // tokens staged in shared memory at a time

struct Partition {              // CTA c owns tiles [start(c), start(c+1))
    long long T;
    int G;
    __host__ __device__ long long start(int c) const { return (long long)c * T / G; }
    __host__ __device__ int cta_of(long long t) const { return (int)(((t + 1) * G - 1) / T); }
};

struct F32Params {
    int heads, tpu, N;
    Partition part;
    MergeOut m;
    float* partials;            // [(G + units)][128][64], slot = cta + unit
    unsigned* counters;         // [units]
};

struct TokenView {              // element (b, h, n, c) of a [B][heads][N][64] view
    const float* base;
    long long bs, hs;
    __device__ __forceinline__ const float* row(int u, int heads, int n) const {
        return base + (long long)(u / heads) * bs + (long long)(u % heads) * hs + (long long)n * D;
    }
};

struct P1SmemF32 {
    float k[F32_CHUNK][D];
    float v[F32_CHUNK][D];
    float gc[kPartialFloats];
    float w0[D * kW0tPitch];
    int last_flag;
};

__global__ void __launch_bounds__(kThreadsF32)
lin_p1_f32(TokenView Kv, TokenView Vv, const F32Params p) {
    extern __shared__ uint8_t smem_raw[];
    P1SmemF32& s = *reinterpret_cast<P1SmemF32*>(align1024(smem_raw));
    const int tid = threadIdx.x;
    const int c = blockIdx.x;
    const long long t_begin = p.part.start(c), t_end = p.part.start(c + 1);
    const int r = tid >> 1, j0 = (tid & 1) * 32;
    pdl_launch_dependents();
    long long t = t_begin;
    while (t < t_end) {
        const int u = (int)(t / p.tpu);
        const long long seg_end = min(t_end, (long long)(u + 1) * p.tpu);
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
        const int n_begin = (int)(t % p.tpu) * TOK;
        const int n_end = min(p.N, (int)((seg_end - (long long)u * p.tpu) * TOK));
        for (int n0 = n_begin; n0 < n_end; n0 += F32_CHUNK) {
            for (int e = tid; e < F32_CHUNK * D; e += kThreadsF32) {
                const int tk = e / D, cc = e % D;
                const int n = n0 + tk;
                s.k[tk][cc] = (n < n_end) ? Kv.row(u, p.heads, n)[cc] : 0.f;
                s.v[tk][cc] = (n < n_end) ? Vv.row(u, p.heads, n)[cc] : 0.f;
            }
            __syncthreads();
            for (int tk = 0; tk < F32_CHUNK; ++tk) {
                const float x = (r < D) ? s.k[tk][r] : s.v[tk][r - D];
#pragma unroll
                for (int jj = 0; jj < 32; jj += 4) {
                    const float4 kv = *reinterpret_cast<const float4*>(&s.k[tk][j0 + jj]);
                    acc[jj + 0] = fmaf(x, kv.x, acc[jj + 0]);
                    acc[jj + 1] = fmaf(x, kv.y, acc[jj + 1]);
                    acc[jj + 2] = fmaf(x, kv.z, acc[jj + 2]);
                    acc[jj + 3] = fmaf(x, kv.w, acc[jj + 3]);
                }
            }
            __syncthreads();
        }
        float* dst = p.partials + (size_t)(c + u) * kPartialFloats + (size_t)r * D + j0;
#pragma unroll
        for (int jj = 0; jj < 32; jj += 4)
            *reinterpret_cast<float4*>(dst + jj) = make_float4(acc[jj], acc[jj + 1], acc[jj + 2], acc[jj + 3]);
        __threadfence();
        __syncthreads();
        const int cf = p.part.cta_of((long long)u * p.tpu), cl = p.part.cta_of((long long)(u + 1) * p.tpu - 1);
        if (tid == 0) {
            const unsigned old = atomicAdd(p.counters + u, 1u);
            s.last_flag = (old + 1u == (unsigned)(cl - cf + 1)) ? 1 : 0;
        }
        __syncthreads();
        if (s.last_flag) {
            __threadfence();
            merge_unit<kThreadsF32, 0>(p.m, u, u % p.heads, (size_t)(cf + u), cl - cf + 1, tid, s.gc, s.w0);
            if (tid == 0) p.counters[u] = 0u;
        }
        __syncthreads();
        t = seg_end;
    }
}

struct P2SmemF32 {
    float w1t[D][D];            // W1 transposed: w1t[k][o] = W1[o][k]
    float q[TOK][D + 1];
};

__global__ void __launch_bounds__(kThreadsF32)
lin_p2_f32(TokenView Qv, float* Z, long long zbs, long long zhs, const float* W1, int heads, int tpu, int N) {
    extern __shared__ uint8_t smem_raw[];
    P2SmemF32& s = *reinterpret_cast<P2SmemF32*>(align1024(smem_raw));
    const int tid = threadIdx.x;
    const long long t = blockIdx.x;                        // one tile per CTA
    const int u = (int)(t / tpu), ti = (int)(t % tpu);
    const int n0 = ti * TOK;
    for (int e = tid; e < TOK * D; e += kThreadsF32) {
        const int tk = e / D, cc = e % D;
        const int n = n0 + tk;
        s.q[tk][cc] = (n < N) ? Qv.row(u, heads, n)[cc] : 0.f;
    }
    pdl_wait_primary();
    const float* W1u = W1 + (size_t)u * D * D;
    for (int e = tid; e < D * D; e += kThreadsF32) s.w1t[e % D][e / D] = __ldcg(W1u + e);
    __syncthreads();
    const int row = tid >> 1, o0 = (tid & 1) * 32;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int k = 0; k < D; ++k) {
        const float x = s.q[row][k];
#pragma unroll
        for (int oo = 0; oo < 32; oo += 4) {
            const float4 w = *reinterpret_cast<const float4*>(&s.w1t[k][o0 + oo]);
            acc[oo + 0] = fmaf(w.x, x, acc[oo + 0]);
            acc[oo + 1] = fmaf(w.y, x, acc[oo + 1]);
            acc[oo + 2] = fmaf(w.z, x, acc[oo + 2]);
            acc[oo + 3] = fmaf(w.w, x, acc[oo + 3]);
        }
    }
    const int n = n0 + row;
    if (n < N) {
        float* dst = Z + (long long)(u / heads) * zbs + (long long)(u % heads) * zhs + (long long)n * D + o0;
#pragma unroll
        for (int oo = 0; oo < 32; oo += 4)
            *reinterpret_cast<float4*>(dst + oo) = make_float4(acc[oo], acc[oo + 1], acc[oo + 2], acc[oo + 3]);
    }
}

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
constexpr int kMaxGridF32 = 160;

struct WsLayout {
    size_t ctrl, counters, ready, w1, partials, total;
};

static WsLayout ws_layout(long long units, int tpu, int dtype) {
    WsLayout L;
    L.ctrl = kWsHeader;
    L.counters = L.ctrl + 256;
    L.ready = align_up(L.counters + (size_t)units * sizeof(unsigned), 256);
    L.w1 = align_up(L.ready + (size_t)units * sizeof(unsigned), 1024);
    const size_t w1_elem = (dtype == TTT_BF16) ? 2 : 4;
    L.partials = align_up(L.w1 + (size_t)units * D * D * w1_elem, 1024);
    const long long slots = (dtype == TTT_BF16) ? units * ((tpu + TPC1 - 1) / TPC1) : kMaxGridF32 + units;
    const size_t slot_floats = (dtype == TTT_BF16) ? (size_t)D * D : (size_t)kPartialFloats;   // P_j, or [G ; C]
    L.total = L.partials + (size_t)slots * slot_floats * sizeof(float);
    return L;
}

}  // namespace lin

size_t linear_ws_bytes(const ttt_shape& s) {
    const int tpu = (s.H * s.W + lin::TOK - 1) / lin::TOK;
    return lin::ws_layout((long long)s.batch * s.heads, tpu, s.dtype).total;
}

size_t linear_ws_control_bytes(const ttt_shape& s) {
    const int tpu = (s.H * s.W + lin::TOK - 1) / lin::TOK;
    return lin::ws_layout((long long)s.batch * s.heads, tpu, s.dtype).w1;   // error word, queue, counters, flags
}

ttt_status launch_linear(const Call& c) {
    using namespace lin;
    const long long units = (long long)c.batch * c.heads;
    const int tpu = (c.N + TOK - 1) / TOK;
    const WsLayout L = ws_layout(units, tpu, c.dtype);

    MergeOut m{};
    m.eta_scale = c.eta * (2.0f / (float)c.N);
    m.W0 = c.W0;
    m.partials = reinterpret_cast<const float*>(c.ws + L.partials);
    m.W1_out = c.W1_out;

    if (c.dtype == TTT_BF16) {
        const int C1 = (tpu + TPC1 - 1) / TPC1, C2 = (tpu + TPC2 - 1) / TPC2;
        const long long total = units * (C1 + C2);
        if (total >= (1LL << 31)) return TTT_ERR_UNSUPPORTED;
        m.W1_bf16 = reinterpret_cast<__nv_bfloat16*>(c.ws + L.w1);
        FusedParams p{};
        p.heads = c.heads;
        p.tpu = tpu;
        p.U = (int)units;
        p.C1 = C1;
        p.C2 = C2;
        p.total = (unsigned)total;
        p.m = m;
        p.counters = reinterpret_cast<unsigned*>(c.ws + L.counters);
        p.ready = reinterpret_cast<uint32_t*>(c.ws + L.ready);
        p.ctrl = reinterpret_cast<unsigned*>(c.ws + L.ctrl);
        p.err = reinterpret_cast<uint32_t*>(c.ws);
        CUtensorMap tmK, tmV, tmQ, tmZ, tmW1;
        if (!make_tmap_tokens(&tmK, c.K, c, TOK) || !make_tmap_tokens(&tmV, c.V, c, TOK) ||
            !make_tmap_tokens(&tmQ, c.Q, c, TOK) || !make_tmap_tokens(&tmZ, c.Z, c, TOK) ||
            !make_tmap_matrix(&tmW1, c.ws + L.w1, units * D, D, D))
            return TTT_ERR_INVALID_ARG;
        const size_t smem = sizeof(FusedSmem) + 1024;
        cudaFuncSetAttribute(lin_fused_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        const int G = (int)std::min<long long>(c.num_sms, total);
        lin_fused_bf16<<<G, kThreadsTc, smem, c.stream>>>(tmK, tmV, tmQ, tmZ, tmW1, p);
        return check_launch(cudaGetLastError());
    }

    // fp32
    const long long T = units * tpu;
    const int G = (int)std::min<long long>(std::min(c.num_sms, kMaxGridF32), T);
    m.W1_f32 = reinterpret_cast<float*>(c.ws + L.w1);
    F32Params p{};
    p.heads = c.heads;
    p.tpu = tpu;
    p.N = c.N;
    p.part = Partition{T, G};
    p.m = m;
    p.partials = reinterpret_cast<float*>(c.ws + L.partials);
    p.counters = reinterpret_cast<unsigned*>(c.ws + L.counters);
    const size_t sm1 = sizeof(P1SmemF32) + 1024, sm2 = sizeof(P2SmemF32) + 1024;
    cudaFuncSetAttribute(lin_p1_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    cudaFuncSetAttribute(lin_p2_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    TokenView Kv{static_cast<const float*>(c.K), c.bs, c.hs};
    TokenView Vv{static_cast<const float*>(c.V), c.bs, c.hs};
    TokenView Qv{static_cast<const float*>(c.Q), c.bs, c.hs};
    lin_p1_f32<<<G, kThreadsF32, sm1, c.stream>>>(Kv, Vv, p);
    ttt_status st = check_launch(cudaGetLastError());
    if (st != TTT_OK) return st;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)T);
    cfg.blockDim = dim3(kThreadsF32);
    cfg.dynamicSmemBytes = sm2;
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return check_launch(cudaLaunchKernelEx(&cfg, lin_p2_f32, Qv, static_cast<float*>(c.Z), c.bs, c.hs,
                                           static_cast<const float*>(m.W1_f32), c.heads, tpu, c.N));
}

}  // namespace ttt
