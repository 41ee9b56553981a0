// linear.cu -- linear inner model f(x) = W x of the TTT layer (one d x d state per head; Vision-TTT
// paper notes, section 关键设计 1), one full-batch step of the L2 loss (press article "CVPR 2026
// Oral | 清華+阿里發布ViT3", Observation 2) written in Gram form:
//     G = sum_n k_n k_n^T,   C = sum_n v_n k_n^T,   W1 = W0 - eta (2/N) (W0 G - C),   z_n = W1 q_n.
//
// bf16 path (lin_cluster_bf16): one thread-block cluster of CS <= 8 CTAs (one CTA per SM) per group
// of units; each CTA takes a 1/CS share of every unit's tokens.
//   Phase 1: each CTA streams its share of the unit's 128-token K/V tiles (TMA, 128-byte swizzle) and
//     accumulates [K | V]^T K  (128 x 64 fp32: rows 0..63 = G, rows 64..127 = C) in tensor memory with
//     tcgen05.mma: A = [K | V]^T (M = 128, MN-major straight from the token-major tiles), B = K
//     (N = 64, MN-major), K-dim = tokens.
//   Exchange: each CTA turns its own partial (G_r, C_r) into P_r = W0 G_r - C_r.  The product runs
//     on the tensor cores with both operands split into bf16 hi + lo parts (M = 128 rows
//     [W0_hi ; W0_lo], B = G_hi and then G_lo), so that it carries about 16 mantissa bits, close to
//     fp32.  Then a reduce-scatter and an all-gather over distributed shared memory: CTA j owns a
//     block of about 64 / CS rows of W1; every CTA pushes block j of its P_r into CTA j with one bulk
//     copy (completion counted on the receiver's mbarrier), CTA j sums its blocks in rank order (a
//     fixed order: bitwise deterministic), forms those rows of W1 = W0 - eta (2/N) sum_r P_r rounded
//     once to bf16, and pushes them into every peer's phase-2 B operand.  No global-memory round
//     trip, no grid-wide wait.
//   Phase 2: the CTA streams its share of 256-token Q tiles and writes Z = Q W1^T: A = Q tile
//     (M = 128 tokens, K-major), B = W1 (K-major); the epilogue drains tensor memory to bf16 and
//     stores Z with TMA.
//   Two units in flight: a cluster with several units streams K/V of unit k+1 before Q of unit k;
//     with two phase-1 accumulators and two W1 operands, the exchange of unit k runs while unit
//     k+1's keys stream in, and the exchange of unit k+1 while unit k is read out, so the exchange
//     leaves no gap in the streaming.
//   Roles (320 threads): warp 0 lane 0 TMA producer, warp 1 lane 0 MMA issuer, warps 2..5 drain the
//   phase-2 accumulators and store Z, warps 6..9 run the exchanges.  CS and the number of clusters
//   are chosen so that all clusters are co-resident (units > SMs: CS = 1 and each CTA loops over
//   units).
//
// fp32 path (lin_p1_f32 / lin_p2_f32): plain fp32 FMA kernels (fp32 accuracy), static partition,
// the same deterministic last-CTA merge.
//
// Dot-product inner loss (the ViT3 recipe of the same press article, section on the ViT3 model):
// L = -(1/N) sum <W k_n, v_n> has gradient -(1/N) C, so W1 = W0 + eta (1/N) C.  Both paths skip the
// W0 G product (bf16: the exchange carries C_r itself) and scale by -eta/N instead of eta 2/N.
#include <algorithm>
#include <mutex>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace lin {

constexpr int D = 64;
constexpr int TOK = 128;                    // tokens per tile
constexpr int TILE_BYTES = TOK * D * 2;     // one bf16 tile: 16 KB
constexpr int kPartialFloats = 2 * D * D;   // [G ; C] = 128 x 64
constexpr int kThreadsTc = 320;         // producer warp, MMA warp, 4 Z warps, 4 exchange warps
constexpr int kW0tPitch = D + 4;           // row pitch of the transposed W0 in shared memory (fp32 path)
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
    int dot;                    // dot-product loss: no W0 G term
    float eta_scale;            // eta * 2 / N  (dot-product loss: eta / N)
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
    for (int k = 0; k < (m.dot ? 0 : D); ++k) {
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
// bf16: one thread-block cluster per group of units, two units in flight per cluster
// ------------------------------------------------------------------------------------------------
constexpr int STAGES = 4;                   // 32 KB each: a K+V tile pair, or one 256-token Q tile
constexpr int ACC = 4;                      // phase-2 accumulators (64 columns each)
constexpr int Q2 = 256;                     // tokens per phase-2 stage
constexpr int kMaxCluster = 8;             // the portable limit
constexpr int kRecvBytes = 15360;
// Cost model of the cluster-size choice (host): the per-SM streaming rate, the HBM rate the SMs
// share, and one unit's exchange latency with peers and alone (measured on B200, in GB/s and us).
constexpr double kCtaGBs = 62.0, kHbmGBs = 6400.0, kExchangeUs = 4.5, kExchangeUs1 = 2.5;           // the peers' rows of my P block: (CS - 1) x ceil(64 / CS) x 256 B, CS <= 8
constexpr uint32_t kColPacc = 0;            // tensor memory: two phase-1 accumulators,
constexpr uint32_t kColAcc = 128;           //   ACC phase-2 accumulators,
constexpr uint32_t kColProd = 384;          //   the W0 G product (448 of 512 columns)
constexpr uint32_t kBarZ = 1, kBarX = 2;    // named barriers of the two epilogue warpgroups

// [G ; C] or P rows in shared memory: 16-byte chunks XOR-swizzled by (row & 15) against bank conflicts.
__device__ __forceinline__ float4* gc_chunk(float* gc, int row, int chunk) {
    return reinterpret_cast<float4*>(gc + row * D) + (chunk ^ (row & 15));
}

// Writes 8 bf16 values as 16-byte chunk `chunk` of row `row` of a 128-byte swizzled K-major operand
// (64 bf16 per row; chunk position XOR (row & 7)).
__device__ __forceinline__ void put_bf16_chunk(uint8_t* base, int row, int chunk, const float* v) {
    uint4 pk;
    pk.x = pack_bf16x2(v[0], v[1]); pk.y = pack_bf16x2(v[2], v[3]);
    pk.z = pack_bf16x2(v[4], v[5]); pk.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(base + row * 128 + ((chunk ^ (row & 7)) << 4)) = pk;
}
// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi): about 16 significant bits in two bf16 numbers.
__device__ __forceinline__ void split_bf16(const float* x, float* hi, float* lo) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        hi[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
        lo[i] = x[i] - hi[i];
    }
}

struct ClusterParams {
    int heads, U, N, CS;        // units, tokens per unit, CTAs per cluster
    int tpu1, tpu2;             // 128-token tiles and 256-token tiles per unit
    int dot;                    // dot-product loss: P_r = C_r (no W0 G product)
    float eta_scale;            // eta * 2 / N  (dot-product loss: -eta / N)
    const float* W0;            // [heads][64][64]
    float* W1_out;              // nullable [units][64][64]
    uint32_t* err;
    unsigned long long wait_ns; // bound of every device-side wait
};

struct ClusterSmem {
    uint8_t stage[STAGES][2 * TILE_BYTES];   // 1024-aligned operand buffers
    uint8_t zbuf[2][TILE_BYTES];             // Z staging of the TMA stores
    uint8_t recv[kRecvBytes];                // the peers' rows of this CTA's block of P
    uint8_t w1[2][D * D * 2];                // W1 of two units, bf16, 128-byte swizzled K-major B operand
    uint8_t a01[2 * D * D * 2];              // [W0_hi ; W0_lo] (bf16 A operand of the product)
    uint8_t gb[2 * D * D * 2];               // G_hi, G_lo (bf16 B operands); then P = W0 G - C (fp32)
    uint64_t full[STAGES], empty[STAGES];
    uint64_t pacc_full[2], pacc_empty[2];    // phase-1 accumulators
    uint64_t acc_full[ACC], acc_empty[ACC];  // phase-2 accumulators
    uint64_t w_full[2], w_empty[2];          // W1 operands
    uint64_t prod_bar;                       // the W0 G product on the tensor cores is done
    uint64_t recv_full;                      // the peers' rows of my P block have landed in recv
    uint64_t w1_full;                        // the peers' W1 rows have landed in the W1 operand
    uint64_t peer_free;                      // every peer has finished the previous exchange
    uint64_t drain_bar, pdrain_bar;          // the MMAs of the MMA lane / of the products (exit)
    uint32_t tmem_base;
    uint32_t recv_armed;                     // phases of recv_full (and of w1_full) armed so far
    int abort_flag;
};

__device__ __forceinline__ int split_lo(int n, int r, int parts) { return (int)((long long)n * r / parts); }

// Units of this cluster: u_k = cid + k * ncl for k < units_of(cid).
__device__ __forceinline__ int units_of(const ClusterParams& p, int cid, int ncl) {
    return cid < p.U ? (p.U - cid + ncl - 1) / ncl : 0;
}

// The producer streams K/V of unit k+1 before Q of unit k, so that the cluster's exchange for unit k
// runs while unit k+1's keys stream in, and unit k+1's exchange while unit k is read out.
__device__ __forceinline__ void cl_producer(ClusterSmem& s, const ClusterParams& p, const CUtensorMap* tmK,
                                            const CUtensorMap* tmV, const CUtensorMap* tmQ, int rank, int cid,
                                            int ncl, const Abort& ab) {
    int st = 0; uint32_t ph = 0;
    uint32_t issued = 0;
    bool ok = true;
    const int m = units_of(p, cid, ncl);
    auto load_kv = [&](int u) {
        const int b = u / p.heads, h = u % p.heads;
        const int t1b = split_lo(p.tpu1, rank, p.CS), t1e = split_lo(p.tpu1, rank + 1, p.CS);
        for (int t = t1b; t < t1e && ok; ++t) {
            if (!(ok = mbar_wait(&s.empty[st], ph ^ 1u, ab))) break;
            mbar_arrive_expect_tx(&s.full[st], 2 * TILE_BYTES);
            tma_load_4d(s.stage[st], tmK, &s.full[st], 0, t * TOK, h, b);
            tma_load_4d(s.stage[st] + TILE_BYTES, tmV, &s.full[st], 0, t * TOK, h, b);
            ++issued;
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
    };
    auto load_q = [&](int u) {
        const int b = u / p.heads, h = u % p.heads;
        const int t2b = split_lo(p.tpu2, rank, p.CS), t2e = split_lo(p.tpu2, rank + 1, p.CS);
        for (int t = t2b; t < t2e && ok; ++t) {
            if (!(ok = mbar_wait(&s.empty[st], ph ^ 1u, ab))) break;
            mbar_arrive_expect_tx(&s.full[st], 2 * TILE_BYTES);
            tma_load_4d(s.stage[st], tmQ, &s.full[st], 0, t * Q2, h, b);
            ++issued;
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
    };
    if (m > 0) load_kv(cid);
    for (int k = 0; k < m && ok; ++k) {
        if (k + 1 < m) load_kv(cid + (k + 1) * ncl);
        load_q(cid + k * ncl);
    }
    // Before the CTA may exit, every tile load it issued has landed (on a normal exit they were all
    // consumed already; after a wait gave up, some may still be in flight).
    for (uint32_t k = issued > (uint32_t)STAGES ? issued - STAGES : 0u; k < issued; ++k)
        mbar_drain(&s.full[k % STAGES], (k / STAGES) & 1u, ab.limit);
}

__device__ __forceinline__ void cl_mma(ClusterSmem& s, const ClusterParams& p, uint32_t tmem, int rank, int cid,
                                       int ncl, const Abort& ab) {
    int st = 0; uint32_t ph = 0;
    int ai = 0; uint32_t aph = 0;
    const int m = units_of(p, cid, ncl);
    // phase 1 of unit k: [K | V]^T K into accumulator k & 1 (A = [K | V]^T, M = 128, and B = K, N = 64,
    // both MN-major straight from the token-major tiles; 16 tokens per MMA)
    auto p1 = [&](int k) -> bool {
        const uint32_t a = (uint32_t)k & 1u, n = (uint32_t)k >> 1;
        if (!mbar_wait(&s.pacc_empty[a], (n & 1u) ^ 1u, ab)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kColPacc + a * 64u;
        const int t1b = split_lo(p.tpu1, rank, p.CS), t1e = split_lo(p.tpu1, rank + 1, p.CS);
        for (int t = t1b; t < t1e; ++t) {
            if (!mbar_wait(&s.full[st], ph, ab)) return false;
            tc_fence_after();
            const uint32_t sK = smem_u32(s.stage[st]);
#pragma unroll
            for (int kk = 0; kk < TOK / 16; ++kk) {
                // 16 tokens per MMA = two 8-row groups (2 x 1024 bytes); V sits TILE_BYTES after K
                const uint64_t ad = sdesc_sw128(sK + kk * 2048, TILE_BYTES, 1024);
                const uint64_t bd = sdesc_sw128(sK + kk * 2048, TILE_BYTES, 1024);
                mma_bf16_ss(d, ad, bd, kIdescP1, (t > t1b || kk > 0) ? 1u : 0u);
            }
            mma_commit(&s.empty[st]);
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
        mma_commit(&s.pacc_full[a]);
        return true;
    };
    // phase 2 of unit k: Z = Q W1^T per 128-token half tile (A = Q, M = 128, K-major; B = W1, K-major)
    auto p2 = [&](int k) -> bool {
        const uint32_t wb = (uint32_t)k & 1u, n = (uint32_t)k >> 1;
        if (!mbar_wait(&s.w_full[wb], n & 1u, ab)) return false;
        tc_fence_after();
        const uint32_t sW = smem_u32(s.w1[wb]);
        const int t2b = split_lo(p.tpu2, rank, p.CS), t2e = split_lo(p.tpu2, rank + 1, p.CS);
        for (int t = t2b; t < t2e; ++t) {
            if (!mbar_wait(&s.full[st], ph, ab)) return false;
            tc_fence_after();
            for (int hf = 0; hf < 2; ++hf) {
                if (!mbar_wait(&s.acc_empty[ai], aph ^ 1u, ab)) return false;
                tc_fence_after();
                const uint32_t sQ = smem_u32(s.stage[st]) + hf * TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(sQ + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sW + kk * 32, 16, 1024);
                    mma_bf16_ss(tmem + kColAcc + (uint32_t)(ai * 64), ad, bd, kIdescP2, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s.acc_full[ai]);
                if (++ai == ACC) { ai = 0; aph ^= 1u; }
            }
            mma_commit(&s.empty[st]);
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
        mma_commit(&s.w_empty[wb]);
        return true;
    };
    if (m > 0 && !p1(0)) return;
    for (int k = 0; k < m; ++k) {
        if (k + 1 < m && !p1(k + 1)) return;
        if (!p2(k)) return;
    }
}

// Warps 2..5: drain the phase-2 accumulators of every unit in turn and store Z with TMA.
__device__ __forceinline__ void cl_zepi(ClusterSmem& s, const ClusterParams& p, uint32_t tmem, const CUtensorMap* tmZ,
                                        int rank, int cid, int ncl, const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                                   // tensor-memory lane quarter of this warp
    const int r = q * 32 + lane;                              // accumulator row
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int ai = 0; uint32_t aph = 0;
    int zn = 0;
    const int m = units_of(p, cid, ncl);
    for (int k = 0; k < m; ++k) {
        const int u = cid + k * ncl;
        const int b = u / p.heads, h = u % p.heads;
        const int t2b = split_lo(p.tpu2, rank, p.CS), t2e = split_lo(p.tpu2, rank + 1, p.CS);
        for (int t = t2b; t < t2e; ++t) {
            for (int hf = 0; hf < 2; ++hf) {
                const bool ok = mbar_wait(&s.acc_full[ai], aph, ab);
                const int zb = zn & 1;
                if (tid == 0 && zn >= 2) bulk_wait_read<1>();  // staging buffer zb is free again
                if (named_bar_or(kBarZ, 128, !ok)) { if (tid == 0) bulk_wait<0>(); return; }
                __syncwarp();
                tc_fence_after();
                uint8_t* zrow = s.zbuf[zb] + r * 128;
                float va[4][16];
#pragma unroll
                for (int j = 0; j < 4; ++j) tmem_ld16(tmem + kColAcc + (uint32_t)(ai * 64 + j * 16) + lane_off, va[j]);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&s.acc_empty[ai]);
                if (++ai == ACC) { ai = 0; aph ^= 1u; }
#pragma unroll
                for (int j = 0; j < D; j += 16) {
                    const float* v = va[j / 16];
                    uint4 lo, hi;
                    lo.x = pack_bf16x2(v[0], v[1]);   lo.y = pack_bf16x2(v[2], v[3]);
                    lo.z = pack_bf16x2(v[4], v[5]);   lo.w = pack_bf16x2(v[6], v[7]);
                    hi.x = pack_bf16x2(v[8], v[9]);   hi.y = pack_bf16x2(v[10], v[11]);
                    hi.z = pack_bf16x2(v[12], v[13]); hi.w = pack_bf16x2(v[14], v[15]);
                    const int c0 = j / 8;                          // 16-byte chunk of columns j..j+7
                    *reinterpret_cast<uint4*>(zrow + ((c0 ^ (r & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(zrow + (((c0 + 1) ^ (r & 7)) << 4)) = hi;
                }
                fence_proxy_async_smem();
                named_bar_sync(kBarZ, 128);
                const int row0 = t * Q2 + hf * TOK;
                if (tid == 0 && row0 < p.N) {
                    tma_store_4d(tmZ, s.zbuf[zb], 0, row0, h, b);
                    bulk_commit();
                }
                ++zn;
            }
        }
    }
    if (tid == 0) bulk_wait<0>();
}

// The product's A operand [bf16(W0) ; bf16(W0 - bf16(W0))] (rows 0..63, 64..127): each exchange
// thread fetches row wrow, columns c0w .. c0w + 31 of W0 into registers, and later writes its share.
__device__ __forceinline__ void load_w0_share(const ClusterParams& p, int h, int wrow, int c0w, float4 (&wa)[8]) {
    const float4* src = reinterpret_cast<const float4*>(p.W0 + ((size_t)h * D + wrow) * D + c0w);
#pragma unroll
    for (int c = 0; c < 8; ++c) wa[c] = __ldg(src + c);
}
__device__ __forceinline__ void put_w0_share(ClusterSmem& s, int wrow, int c0w, const float4 (&wa)[8]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float x[8] = {wa[2 * c].x, wa[2 * c].y, wa[2 * c].z, wa[2 * c].w,
                            wa[2 * c + 1].x, wa[2 * c + 1].y, wa[2 * c + 1].z, wa[2 * c + 1].w};
        float hi[8], lo[8];
        split_bf16(x, hi, lo);
        put_bf16_chunk(s.a01, wrow, c0w / 8 + c, hi);
        put_bf16_chunk(s.a01, D + wrow, c0w / 8 + c, lo);
    }
}

// Where row i of P goes: this CTA's pb (own = true), or the owner's receive slot for this rank (same
// chunk swizzle as pb), counted on the owner's recv_full.
struct PRowDst {
    bool own;
    uint32_t row, bar;                       // shared::cluster addresses of the row and of the barrier
};
__device__ __forceinline__ PRowDst p_row_dst(ClusterSmem& s, const ClusterParams& p, int rank, int i) {
    int o = 0;
    while (o + 1 < p.CS && split_lo(D, o + 1, p.CS) <= i) ++o;
    PRowDst d;
    d.own = o == rank;
    const int slot_rows = (D + p.CS - 1) / p.CS;
    const int slot = (rank < o) ? rank : rank - 1;
    d.row = d.own ? 0u
                  : map_to_rank(smem_u32(s.recv) + (uint32_t)((slot * slot_rows + i - split_lo(D, o, p.CS)) * D * 4),
                                (uint32_t)o);
    d.bar = d.own ? 0u : map_to_rank(smem_u32(&s.recv_full), (uint32_t)o);
    return d;
}
// Chunk c (columns 4c .. 4c+3) of row i of P to its destination.
__device__ __forceinline__ void put_p_chunk(const PRowDst& d, float* pb, int i, int c, float4 v) {
    if (d.own) *gc_chunk(pb, i, c) = v;
    else st_async_f4(d.row + (uint32_t)((c ^ (i & 15)) << 4), v, d.bar);
}

// Warps 6..9: the cluster exchange of every unit in turn.  Each CTA turns its partial (G_r, C_r) into
// P_r = W0 G_r - C_r on the tensor cores (both operands split into bf16 hi + lo: about 16 mantissa
// bits).  Rows of W1 are then formed in blocks, one per CTA (rank j owns rows [64 j / CS, 64 (j+1) / CS)):
// the thread holding row i of P stores it straight into the receive slot of the row's owner
// (reduce-scatter), the owner sums the rows it receives in rank order (a fixed order: bitwise
// deterministic), forms its rows of W1 = W0 - eta (2/N) sum_r P_r rounded once to bf16 into the unit's
// W1 operand, and stores them into the same place in every peer's operand (all-gather).  All
// transfers are st.async stores whose bytes the receiver's mbarrier counts: no bulk-copy queue (busy
// with the streaming loads) and no release fence on the way.  W0 for the next unit's product and for
// this unit's W1 rows is fetched while the peers' rows are in flight.
__device__ __forceinline__ void cl_xepi(ClusterSmem& s, const ClusterParams& p, uint32_t tmem, int rank, int cid,
                                        int ncl, const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int tid = threadIdx.x - 192;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool multi = p.CS > 1;
    const int m = units_of(p, cid, ncl);
    float* pb = reinterpret_cast<float*>(s.gb);               // my rows of P (fp32, swizzled chunks)
    uint8_t* bhi = s.gb;
    uint8_t* blo = s.gb + D * D * 2;
    const bool has_p1 = split_lo(p.tpu1, rank + 1, p.CS) > split_lo(p.tpu1, rank, p.CS);
    const int rb0 = split_lo(D, rank, p.CS), rb1 = split_lo(D, rank + 1, p.CS);   // my block of rows
    const int slot_rows = (D + p.CS - 1) / p.CS;                                  // rows per receive slot
    // this thread's share of the product's A operand: row wrow of W0, columns c0w .. c0w + 31
    const int wrow = tid >> 1, c0w = (tid & 1) * 32;
    float4 wa[8];
    if (!p.dot && m > 0) {
        load_w0_share(p, cid % p.heads, wrow, c0w, wa);
        put_w0_share(s, wrow, c0w, wa);
    }
    int k = 0;
    bool failed = false;
    for (; k < m; ++k) {
        const int u = cid + k * ncl;
        const int h = u % p.heads;
        const uint32_t a = (uint32_t)k & 1u, n = (uint32_t)k >> 1;
        // (0) my W1 buffer a is free once the MMAs of unit k - 2 have read it; then arm the receive
        //     barriers and tell the peers they may store into recv and into W1 buffer a
        bool ok = mbar_wait(&s.w_empty[a], (n & 1u) ^ 1u, ab);
        if (named_bar_or(kBarX, 128, !ok)) { failed = true; break; }
        if (multi && tid == 0) {
            ++s.recv_armed;
            mbar_arrive_expect_tx(&s.recv_full, (uint32_t)((p.CS - 1) * (rb1 - rb0) * D * 4));
            mbar_arrive_expect_tx(&s.w1_full, (uint32_t)((D - (rb1 - rb0)) * 128));
            for (int pr = 0; pr < p.CS; ++pr)
                if (pr != rank) mbar_arrive_remote_relaxed(map_to_rank(smem_u32(&s.peer_free), (uint32_t)pr));
        }
        // (1) my phase-1 accumulator, and every peer ready for this exchange
        ok = mbar_wait(&s.pacc_full[a], n & 1u, ab);
        if (multi) ok = ok && mbar_wait_cluster(&s.peer_free, (uint32_t)k & 1u, ab);
        if (named_bar_or(kBarX, 128, !ok)) { failed = true; break; }
        __syncwarp();
        tc_fence_after();
        // (2) accumulator rows 0..63 (G, warps 8 and 9) as bf16 hi / lo B operands; rows 64..127 (C)
        //     stay in tensor memory until P is formed
        const uint32_t pacc = tmem + kColPacc + a * 64u + lane_off;
        if (!p.dot) {
            if (r < D) {                                      // G is symmetric: row r of G = column r
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float g[16];
                    tmem_ld16(pacc + (uint32_t)(j * 16), g);
                    tmem_ld_wait();
                    if (!has_p1)
#pragma unroll
                        for (int e = 0; e < 16; ++e) g[e] = 0.f;
                    float hi[8], lo[8];
                    split_bf16(g, hi, lo);
                    put_bf16_chunk(bhi, r, 2 * j, hi);
                    put_bf16_chunk(blo, r, 2 * j, lo);
                    split_bf16(g + 8, hi, lo);
                    put_bf16_chunk(bhi, r, 2 * j + 1, hi);
                    put_bf16_chunk(blo, r, 2 * j + 1, lo);
                }
                tc_fence_before();
                mbar_arrive(&s.pacc_empty[a]);
            }
            fence_proxy_async_smem();                         // the operands are read by the tensor cores
            named_bar_sync(kBarX, 128);
            // (3) D = [W0_hi ; W0_lo] (G_hi + G_lo) (M = 128, N = 64, K = 64 twice)
            if (tid == 0) {
                tc_fence_after();
                const uint32_t sa = smem_u32(s.a01), sh = smem_u32(bhi), sl = smem_u32(blo);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16_ss(tmem + kColProd, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sh + kk * 32, 16, 1024),
                                kIdescP2, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16_ss(tmem + kColProd, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sl + kk * 32, 16, 1024),
                                kIdescP2, 1u);
                mma_commit(&s.prod_bar);
            }
            ok = mbar_wait(&s.prod_bar, (uint32_t)k & 1u, ab);
            if (named_bar_or(kBarX, 128, !ok)) { failed = true; break; }
            __syncwarp();
            tc_fence_after();
            // (4) P = D[0:64] + D[64:128] - C: warps 6, 7 (rows 64..127: the lo half, and C from the
            //     phase-1 accumulator) put D_lo - C into pb, then warps 8, 9 (rows 0..63) complete
            //     their rows in registers and send them (the G operands in gb are consumed); 16
            //     columns at a time
            if (r >= D) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float dd[16], c16[16];
                    tmem_ld16(tmem + kColProd + lane_off + (uint32_t)(j * 16), dd);
                    tmem_ld16(pacc + (uint32_t)(j * 16), c16);
                    tmem_ld_wait();
                    if (!has_p1)
#pragma unroll
                        for (int e = 0; e < 16; ++e) c16[e] = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *gc_chunk(pb, r - D, 4 * j + c) = make_float4(dd[4 * c] - c16[4 * c], dd[4 * c + 1] - c16[4 * c + 1],
                                                                      dd[4 * c + 2] - c16[4 * c + 2],
                                                                      dd[4 * c + 3] - c16[4 * c + 3]);
                }
                tc_fence_before();
                mbar_arrive(&s.pacc_empty[a]);                // the MMA lane may start unit k + 2
                named_bar_sync(kBarX, 128);
            } else {
                const PRowDst dst = p_row_dst(s, p, rank, r);
                named_bar_sync(kBarX, 128);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float x[16];
                    tmem_ld16(tmem + kColProd + lane_off + (uint32_t)(j * 16), x);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float4 l = *gc_chunk(pb, r, 4 * j + c);
                        put_p_chunk(dst, pb, r, 4 * j + c,
                                    make_float4(x[4 * c] + l.x, x[4 * c + 1] + l.y, x[4 * c + 2] + l.z, x[4 * c + 3] + l.w));
                    }
                }
                tc_fence_before();
            }
        } else {
            // dot-product loss: P = C, sent by the threads of rows 64..127
            if (r >= D) {
                const PRowDst dst = p_row_dst(s, p, rank, r - D);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float x[16];
                    tmem_ld16(pacc + (uint32_t)(j * 16), x);
                    tmem_ld_wait();
                    if (!has_p1)
#pragma unroll
                        for (int e = 0; e < 16; ++e) x[e] = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        put_p_chunk(dst, pb, r - D, 4 * j + c, make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(&s.pacc_empty[a]);
        }
        // (5) W0 for my rows of W1 (the first two passes: all of them when CS > 1), fetched while the
        //     rows travel
        float4 w0r[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = rb0 + (tid >> 3) + 16 * j;
            if (i < rb1) {
                const float4* w0 = reinterpret_cast<const float4*>(p.W0 + ((size_t)h * D + i) * D + 8 * (tid & 7));
                w0r[j][0] = __ldg(w0);
                w0r[j][1] = __ldg(w0 + 1);
            }
        }
        if (multi) ok = mbar_wait_cluster(&s.recv_full, (uint32_t)k & 1u, ab);
        if (named_bar_or(kBarX, 128, !ok)) { failed = true; break; }
        // (6) my rows of W1 = W0 - eta_scale sum_r P_r (ranks in order); thread tid: row rb0 + tid / 8
        //     (+ 16 j), columns 8 (tid % 8) .. + 8; W1_out rows from their owner
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = rb0 + (tid >> 3) + 16 * j;
            if (i >= rb1) continue;
            const int c8 = tid & 7;
            float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int pr = 0; pr < p.CS; ++pr) {
                const float* src = (pr == rank)
                    ? pb + i * D
                    : reinterpret_cast<const float*>(s.recv + ((pr < rank) ? pr : pr - 1) * slot_rows * D * 4) + (i - rb0) * D;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c = 2 * c8 + hh;                    // 16-byte chunk of columns 4c .. 4c+3
                    const float4 x = reinterpret_cast<const float4*>(src)[c ^ (i & 15)];
                    sum[4 * hh] += x.x; sum[4 * hh + 1] += x.y; sum[4 * hh + 2] += x.z; sum[4 * hh + 3] += x.w;
                }
            }
            float w1[8];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float4 w = j < 2 ? w0r[j < 2 ? j : 0][hh]
                                       : __ldg(reinterpret_cast<const float4*>(p.W0 + ((size_t)h * D + i) * D + 8 * c8) + hh);
                w1[4 * hh] = w.x - p.eta_scale * sum[4 * hh];
                w1[4 * hh + 1] = w.y - p.eta_scale * sum[4 * hh + 1];
                w1[4 * hh + 2] = w.z - p.eta_scale * sum[4 * hh + 2];
                w1[4 * hh + 3] = w.w - p.eta_scale * sum[4 * hh + 3];
            }
            if (p.W1_out) {
                float4* o = reinterpret_cast<float4*>(p.W1_out + ((size_t)u * D + i) * D + 8 * c8);
                o[0] = make_float4(w1[0], w1[1], w1[2], w1[3]);
                o[1] = make_float4(w1[4], w1[5], w1[6], w1[7]);
            }
            uint4 pk;
            pk.x = pack_bf16x2(w1[0], w1[1]); pk.y = pack_bf16x2(w1[2], w1[3]);
            pk.z = pack_bf16x2(w1[4], w1[5]); pk.w = pack_bf16x2(w1[6], w1[7]);
            const uint32_t off = (uint32_t)(i * 128 + ((c8 ^ (i & 7)) << 4));   // 128-byte swizzled K-major
            *reinterpret_cast<uint4*>(s.w1[a] + off) = pk;
            for (int pr = 0; pr < p.CS; ++pr)
                if (pr != rank)
                    st_async_u4(map_to_rank(smem_u32(s.w1[a]) + off, (uint32_t)pr), pk,
                                map_to_rank(smem_u32(&s.w1_full), (uint32_t)pr));
        }
        // (7) the next unit's product operand when its head differs (the product of this unit has read
        //     a01); then my W1 rows and the peers' rows, once landed, go to the tensor cores
        if (!p.dot && k + 1 < m && (cid + (k + 1) * ncl) % p.heads != h) {
            load_w0_share(p, (cid + (k + 1) * ncl) % p.heads, wrow, c0w, wa);
            put_w0_share(s, wrow, c0w, wa);
        }
        fence_proxy_async_smem();
        if (multi) {
            ok = mbar_wait_cluster(&s.w1_full, (uint32_t)k & 1u, ab);
            fence_proxy_async_smem();                         // rows stored by the peers, now observed here
        }
        if (named_bar_or(kBarX, 128, !ok)) { failed = true; break; }
        if (tid == 0) mbar_arrive(&s.w_full[a]);
    }
    // Final handshake: once every peer has finished its last exchange, nobody stores into this CTA
    // again (each CTA's own stores are then known to have landed: every receiver waited for them).
    if (multi && !failed) {
        named_bar_sync(kBarX, 128);
        if (tid == 0)
            for (int pr = 0; pr < p.CS; ++pr)
                if (pr != rank) mbar_arrive_remote_relaxed(map_to_rank(smem_u32(&s.peer_free), (uint32_t)pr));
        mbar_wait_cluster(&s.peer_free, (uint32_t)k & 1u, ab);
    }
    if (tid == 0 && !p.dot && k > 0) {                       // the product MMAs this thread issued
        mma_commit(&s.pdrain_bar);
        mbar_drain(&s.pdrain_bar, 0u, ab.limit);
    }
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kThreadsTc, 1)
lin_cluster_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmZ,
                 const ClusterParams p) {
    extern __shared__ uint8_t smem_raw[];
    ClusterSmem& s = *reinterpret_cast<ClusterSmem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank(), cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        s.recv_armed = 0;
        for (int i = 0; i < STAGES; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.pacc_full[i], 1); mbar_init(&s.pacc_empty[i], 128);
            mbar_init(&s.w_full[i], 1); mbar_init(&s.w_empty[i], 1);
        }
        for (int i = 0; i < ACC; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
        mbar_init(&s.prod_bar, 1);
        mbar_init(&s.recv_full, 1);
        mbar_init(&s.w1_full, 1);
        mbar_init(&s.peer_free, (uint32_t)(p.CS > 1 ? p.CS - 1 : 1));
        mbar_init(&s.drain_bar, 1); mbar_init(&s.pdrain_bar, 1);
        fence_barrier_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmQ); prefetch_tmap(&tmZ);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();                  // every CTA's barriers exist before any peer arrives on them
    // Launched as a programmatic dependent of the preceding kernel in the stream: the prologue above
    // overlaps that kernel's tail, and nothing is read from global memory before it has completed
    // (with its memory visible).  Only then may a kernel queued behind this one as a programmatic
    // dependent (the conv heads of the same layer) start: it takes the SMs this grid leaves free.
    pdl_wait_primary();
    pdl_launch_dependents();
    const uint32_t tmem = s.tmem_base;

    // Lane 0 of warps 0 and 1 carries the producer and MMA roles; the rest of each warp waits for it
    // here, so that every warp reaches the block barrier below converged.
    if (warp == 0) {
        if (lane == 0) cl_producer(s, p, &tmK, &tmV, &tmQ, rank, cid, ncl, ab);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            cl_mma(s, p, tmem, rank, cid, ncl, ab);
            // every MMA this thread issued has completed before tensor memory is freed
            mma_commit(&s.drain_bar);
            mbar_drain(&s.drain_bar, 0u, ab.limit);
        }
        __syncwarp();
    } else if (warp < 6) {
        cl_zepi(s, p, tmem, &tmZ, rank, cid, ncl, ab);
    } else {
        cl_xepi(s, p, tmem, rank, cid, ncl, ab);
    }

    tc_fence_before();
    __syncthreads();
    if (p.CS > 1) {
        // No CTA leaves while a peer may still push into it: every CTA of the cluster gets here after
        // issuing its last push, and then each waits (bounded) for the pushes it was promised to land.
        cluster_sync_all();
        if (threadIdx.x == 0 && s.recv_armed > 0) {
            mbar_drain(&s.recv_full, (s.recv_armed - 1) & 1u, ab.limit);
            mbar_drain(&s.w1_full, (s.recv_armed - 1) & 1u, ab.limit);
        }
        __syncthreads();
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    // As a programmatic dependent of a preceding kernel: complete only after it has completed.
    pdl_wait_primary();
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
        // the chunk's K and V rows as 16-byte loads into registers, all issued before any is used;
        // the next chunk's loads are in flight while the current chunk is accumulated
        constexpr int F4 = F32_CHUNK * D / 4 / kThreadsF32;   // float4 of K (and of V) per thread
        float4 fk[F4], fv[F4];
        auto fetch = [&](int n0) {
#pragma unroll
            for (int q = 0; q < F4; ++q) {
                const int e4 = q * kThreadsF32 + tid, tk = e4 / (D / 4), c4 = e4 % (D / 4);
                const int n = n0 + tk;
                fk[q] = n < n_end ? __ldg(reinterpret_cast<const float4*>(Kv.row(u, p.heads, n)) + c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                fv[q] = n < n_end ? __ldg(reinterpret_cast<const float4*>(Vv.row(u, p.heads, n)) + c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        fetch(n_begin);
        for (int n0 = n_begin; n0 < n_end; n0 += F32_CHUNK) {
#pragma unroll
            for (int q = 0; q < F4; ++q) {
                const int e4 = q * kThreadsF32 + tid, tk = e4 / (D / 4), c4 = e4 % (D / 4);
                *reinterpret_cast<float4*>(&s.k[tk][4 * c4]) = fk[q];
                *reinterpret_cast<float4*>(&s.v[tk][4 * c4]) = fv[q];
            }
            __syncthreads();
            if (n0 + F32_CHUNK < n_end) fetch(n0 + F32_CHUNK);
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
    float q[TOK][D + 4];        // row pitch 272 B: 16-byte aligned rows for the vector stores
};

__global__ void __launch_bounds__(kThreadsF32)
lin_p2_f32(TokenView Qv, float* Z, long long zbs, long long zhs, const float* W1, int heads, int tpu, int N) {
    extern __shared__ uint8_t smem_raw[];
    P2SmemF32& s = *reinterpret_cast<P2SmemF32*>(align1024(smem_raw));
    const int tid = threadIdx.x;
    const long long t = blockIdx.x;                        // one tile per CTA
    const int u = (int)(t / tpu), ti = (int)(t % tpu);
    const int n0 = ti * TOK;
    {
        // the Q tile as 16-byte loads, all issued before any is stored
        constexpr int F4 = TOK * D / 4 / kThreadsF32;
        float4 fq[F4];
#pragma unroll
        for (int q = 0; q < F4; ++q) {
            const int e4 = q * kThreadsF32 + tid, tk = e4 / (D / 4), c4 = e4 % (D / 4);
            const int n = n0 + tk;
            fq[q] = n < N ? __ldg(reinterpret_cast<const float4*>(Qv.row(u, heads, n)) + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < F4; ++q) {
            const int e4 = q * kThreadsF32 + tid, tk = e4 / (D / 4), c4 = e4 % (D / 4);
            *reinterpret_cast<float4*>(&s.q[tk][4 * c4]) = fq[q];
        }
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
// ------------------------------------------------------------------------------------------------
// lin_small_f32: fp32 units of at most kSmallN tokens (the 1e-5 case of a few hundred tokens, where
// the tile kernels above are pure latency).  One cluster of kSmallCS CTAs per unit (a persistent loop
// when there are more units than clusters).  Each CTA holds the unit's keys in shared memory and forms
// kSmallRows rows of G = sum k k^T and C = sum v k^T; its G rows go to every CTA of the cluster
// (distributed shared memory), each CTA forms its rows of W1 = W0 - eta_scale (W0 G - C) and sends
// them likewise, then reads out its share of the tokens, z = W1 q.  Two cluster barriers per unit,
// no workspace, every sum in a fixed order (bitwise reproducible).
// ------------------------------------------------------------------------------------------------
constexpr int kSmallCS = 8;
constexpr int kSmallN = 384;
constexpr int kSmallThreads = 512;
constexpr int kSmallRows = D / kSmallCS;            // 8 rows of G, C, W1 per CTA
constexpr int kSmallQ = kSmallN / kSmallCS + 1;     // tokens read out per CTA, at most

struct SmallSmem {
    float k[kSmallN][D];                 // the unit's keys
    float v[kSmallN][kSmallRows];        // this CTA's columns of V
    float q[kSmallQ][D];                 // this CTA's query tokens
    float g[D][D];                       // G, gathered from the cluster
    float w1t[D][D];                     // W1 transposed (w1t[m][j] = W1[j][m]), gathered
    float w0[kSmallRows][D];             // this CTA's rows of W0
    float part[kSmallRows][2][kSmallRows][D];   // the token groups' rows of G and C
    float c[kSmallRows][D];              // this CTA's rows of C
    uint64_t bar;                        // the bulk copies of a unit's rows
    int abort_flag;
};

struct SmallParams {
    TokenView Kv, Vv, Qv;
    float* Z;
    long long zbs, zhs;
    const float* W0;
    float* W1_out;
    int heads, N, units, dot;
    float eta_scale;                     // W1 = W0 - eta_scale (W0 G - C); dot loss: no W0 G term
    uint32_t* err;
    unsigned long long wait_ns;
};

__global__ void __launch_bounds__(kSmallThreads, 1)
lin_small_f32(const SmallParams p) {
    extern __shared__ uint8_t smem_raw[];
    SmallSmem& s = *reinterpret_cast<SmallSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, lane = tid & 31;
    const int rank = (int)cluster_ctarank();
    const int N = p.N;
    const int n0 = rank * N / kSmallCS, n1 = (rank + 1) * N / kSmallCS;    // this CTA's query tokens
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};
    if (tid == 0) {
        s.abort_flag = 0;
        mbar_init(&s.bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();
    uint32_t it = 0;
    for (int u = (int)cluster_id_x(); u < p.units; u += (int)cluster_count_x(), ++it) {
        const int h = u % p.heads;
        // ---- the unit's keys, its query tokens and this CTA's rows of W0 by bulk copies (the rows
        //      are contiguous), this CTA's columns of V by loads
        if (tid == 0) {
            const uint32_t nq = (uint32_t)(n1 - n0) * D * 4;
            mbar_arrive_expect_tx(&s.bar, (uint32_t)N * D * 4 + nq + kSmallRows * D * 4);
            bulk_g2s(&s.k[0][0], p.Kv.row(u, p.heads, 0), (uint32_t)N * D * 4, &s.bar);
            if (nq) bulk_g2s(&s.q[0][0], p.Qv.row(u, p.heads, n0), nq, &s.bar);
            bulk_g2s(&s.w0[0][0], p.W0 + ((size_t)h * D + rank * kSmallRows) * D, kSmallRows * D * 4, &s.bar);
        }
        {
            float4 v4[(2 * kSmallN + kSmallThreads - 1) / kSmallThreads];
#pragma unroll
            for (int k = 0; k < (2 * kSmallN + kSmallThreads - 1) / kSmallThreads; ++k) {
                const int e = tid + k * kSmallThreads;
                if (e < 2 * N)
                    v4[k] = __ldg(reinterpret_cast<const float4*>(p.Vv.row(u, p.heads, e >> 1) + rank * kSmallRows) + (e & 1));
            }
#pragma unroll
            for (int k = 0; k < (2 * kSmallN + kSmallThreads - 1) / kSmallThreads; ++k) {
                const int e = tid + k * kSmallThreads;
                if (e < 2 * N) reinterpret_cast<float4*>(&s.v[e >> 1][0])[e & 1] = v4[k];
            }
        }
        // every CTA of the cluster runs before any peer writes into it (first unit); peers are done
        // reading what this unit's gathers overwrite (later units)
        if (it == 0) cluster_sync_all();
        mbar_wait(&s.bar, it & 1u, ab);  // on a timeout the error word says so; the cluster stays in step
        __syncthreads();
        // ---- rows of G and C: warp tg (< 8) sums tokens [tg N / 8, (tg + 1) N / 8) for all of this
        //      CTA's rows and the lane's columns 2 lane, 2 lane + 1: per token one pair of key columns
        //      and the CTA's eight key and value entries feed 32 FMAs
        {
            const int tg = tid >> 5;
            if (tg < kSmallRows) {
                float ag[kSmallRows][2], ac[kSmallRows][2];
#pragma unroll
                for (int a = 0; a < kSmallRows; ++a) { ag[a][0] = ag[a][1] = 0.f; ac[a][0] = ac[a][1] = 0.f; }
                const int na = tg * N / kSmallRows, nb = (tg + 1) * N / kSmallRows;
                for (int n = na; n < nb; ++n) {
                    const float2 kj = *reinterpret_cast<const float2*>(&s.k[n][2 * lane]);
                    const float4 k0 = *reinterpret_cast<const float4*>(&s.k[n][rank * kSmallRows]);
                    const float4 k1 = *reinterpret_cast<const float4*>(&s.k[n][rank * kSmallRows + 4]);
                    const float4 v0 = *reinterpret_cast<const float4*>(&s.v[n][0]);
                    const float4 v1 = *reinterpret_cast<const float4*>(&s.v[n][4]);
                    const float kr[kSmallRows] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                    const float vr[kSmallRows] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                    for (int a = 0; a < kSmallRows; ++a) {
                        ag[a][0] = fmaf(kr[a], kj.x, ag[a][0]); ag[a][1] = fmaf(kr[a], kj.y, ag[a][1]);
                        ac[a][0] = fmaf(vr[a], kj.x, ac[a][0]); ac[a][1] = fmaf(vr[a], kj.y, ac[a][1]);
                    }
                }
#pragma unroll
                for (int a = 0; a < kSmallRows; ++a) {
                    *reinterpret_cast<float2*>(&s.part[tg][0][a][2 * lane]) = make_float2(ag[a][0], ag[a][1]);
                    *reinterpret_cast<float2*>(&s.part[tg][1][a][2 * lane]) = make_float2(ac[a][0], ac[a][1]);
                }
            }
        }
        __syncthreads();
        // the token groups added in order: this CTA's rows of G (into the gathered G) and of C
        for (int e = tid; e < 2 * kSmallRows * D; e += kSmallThreads) {
            const int x = e / (kSmallRows * D), a = (e / D) % kSmallRows, j = e % D;
            float acc = s.part[0][x][a][j];
#pragma unroll
            for (int t = 1; t < kSmallRows; ++t) acc += s.part[t][x][a][j];
            if (x == 0) s.g[rank * kSmallRows + a][j] = acc;
            else s.c[a][j] = acc;
        }
        __syncthreads();
        // ---- this CTA's rows of G into every other CTA of the cluster, 16 bytes a store
        for (int e = tid; e < (kSmallCS - 1) * kSmallRows * (D / 4); e += kSmallThreads) {
            const int r = (rank + 1 + e / (kSmallRows * (D / 4))) % kSmallCS, f = e % (kSmallRows * (D / 4));
            const uint32_t la = smem_u32(&s.g[rank * kSmallRows][0]) + (uint32_t)f * 16;
            st_cluster_v4(map_to_rank(la, (uint32_t)r), *reinterpret_cast<const uint4*>(&s.g[rank * kSmallRows][4 * f]));
        }
        cluster_sync_all();
        // ---- W1[i][j] = W0[i][j] - eta_scale ((W0 G)[i][j] - C[i][j]): thread (row a, column j)
        {
            const int a = tid >> 6, j = tid & (D - 1), i = rank * kSmallRows + a;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (!p.dot) {
#pragma unroll 4
                for (int m = 0; m < D; m += 4)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[q] = fmaf(s.w0[a][m + q], s.g[m + q][j], acc[q]);
            }
            const float w1 = s.w0[a][j] - p.eta_scale * (((acc[0] + acc[1]) + (acc[2] + acc[3])) - s.c[a][j]);
            if (p.W1_out) p.W1_out[((size_t)u * D + i) * D + j] = w1;
            s.w1t[j][i] = w1;
        }
        __syncthreads();
        // ---- this CTA's rows of W1 are columns 8 rank .. 8 rank + 7 of w1t: two 16-byte pieces of each
        //      of its 64 rows, into every other CTA of the cluster
        for (int e = tid; e < (kSmallCS - 1) * D * 2; e += kSmallThreads) {
            const int r = (rank + 1 + e / (D * 2)) % kSmallCS, m = (e / 2) % D, half = e & 1;
            float* src = &s.w1t[m][rank * kSmallRows + 4 * half];
            st_cluster_v4(map_to_rank(smem_u32(src), (uint32_t)r), *reinterpret_cast<const uint4*>(src));
        }
        cluster_sync_all();
        // ---- z = W1 q for this CTA's tokens: thread (token group tg, output channel j) holds row j of
        //      W1 in registers; the token's q comes as broadcast float4
        {
            const int j = tid & (D - 1), tg = tid >> 6;
            float wr[D];
#pragma unroll
            for (int m = 0; m < D; ++m) wr[m] = s.w1t[m][j];
            float* zb = p.Z + (long long)(u / p.heads) * p.zbs + (long long)h * p.zhs;
            for (int t = tg; t < n1 - n0; t += kSmallThreads / D) {
                float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < D; m += 4) {
                    const float4 q4 = *reinterpret_cast<const float4*>(&s.q[t][m]);
                    z[0] = fmaf(wr[m], q4.x, z[0]); z[1] = fmaf(wr[m + 1], q4.y, z[1]);
                    z[2] = fmaf(wr[m + 2], q4.z, z[2]); z[3] = fmaf(wr[m + 3], q4.w, z[3]);
                }
                zb[(long long)(n0 + t) * D + j] = (z[0] + z[1]) + (z[2] + z[3]);
            }
        }
        // s.k, s.v, s.q, s.w0 are reloaded for the next unit, and the peers' gathers of the next
        // unit overwrite s.g and s.w1t: every CTA of the cluster is done with this unit first
        cluster_sync_all();
    }
    // after a wait that gave up, the last unit's copies may still be landing
    if (tid == 0 && it > 0) mbar_drain(&s.bar, (it - 1) & 1u, ab.limit);
}

constexpr int kMaxGridF32 = 160;

struct WsLayout {
    size_t counters, w1, partials, total;
};

// bf16: the cluster kernel keeps all intermediates on chip; its workspace is the error word only.
// fp32: counters, W1 and the per-CTA [G ; C] partial slots of the two-kernel path.
static WsLayout ws_layout(long long units, int dtype) {
    WsLayout L;
    if (dtype == TTT_BF16) {
        L.counters = L.w1 = L.partials = L.total = kWsHeader;
        return L;
    }
    L.counters = kWsHeader;
    L.w1 = align_up(L.counters + (size_t)units * sizeof(unsigned), 1024);
    L.partials = align_up(L.w1 + (size_t)units * D * D * sizeof(float), 1024);
    L.total = L.partials + (size_t)(kMaxGridF32 + units) * kPartialFloats * sizeof(float);
    return L;
}

// Largest number of co-resident clusters of `cs` CTAs of the cluster kernel (cached per device).
static int max_active_clusters(int cs, size_t smem) {
    static std::mutex mu;
    static int cache[64][kMaxCluster + 1];
    static bool init = false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) { cudaGetLastError(); return 0; }
    std::lock_guard<std::mutex> lock(mu);
    if (!init) {
        for (auto& row : cache)
            for (int& v : row) v = -1;
        init = true;
    }
    if (cache[dev][cs] < 0) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(cs * 64);
        cfg.blockDim = dim3(kThreadsTc);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cs; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, (void*)lin_cluster_bf16, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][cs] = n;
    }
    return cache[dev][cs];
}

}  // namespace lin

size_t linear_ws_bytes(const ttt_shape& s) {
    return lin::ws_layout((long long)s.batch * s.heads, s.dtype).total;
}

size_t linear_ws_control_bytes(const ttt_shape& s) {
    return lin::ws_layout((long long)s.batch * s.heads, s.dtype).w1;   // error word (and fp32 counters)
}

// fp32 units of at most kSmallN tokens: one kSmallCS-CTA cluster per unit (lin_small_f32).
static ttt_status launch_small_f32(const Call& c, long long units) {
    using namespace lin;
    const size_t smem = sizeof(SmallSmem) + 128;
    cudaFuncSetAttribute(lin_small_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kSmallThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kSmallCS; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    // every cluster co-resident: a persistent loop takes the units beyond them
    long long ncl = std::min<long long>(units, c.num_sms / kSmallCS);
    cfg.gridDim = dim3((unsigned)(ncl * kSmallCS));
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, lin_small_f32, &cfg) == cudaSuccess && active > 0)
        ncl = std::min<long long>(ncl, active);
    cudaGetLastError();
    cfg.gridDim = dim3((unsigned)(ncl * kSmallCS));
    if (c.grid_out) *c.grid_out = (int)(ncl * kSmallCS);
    SmallParams p{};
    p.Kv = TokenView{static_cast<const float*>(c.K), c.bs, c.hs};
    p.Vv = TokenView{static_cast<const float*>(c.V), c.bs, c.hs};
    p.Qv = TokenView{static_cast<const float*>(c.Q), c.bs, c.hs};
    p.Z = static_cast<float*>(c.Z);
    p.zbs = c.bs;
    p.zhs = c.hs;
    p.W0 = c.W0;
    p.W1_out = c.W1_out;
    p.heads = c.heads;
    p.N = c.N;
    p.units = (int)units;
    p.dot = c.loss == TTT_LOSS_DOT;
    p.eta_scale = p.dot ? c.eta / (float)c.N : c.eta * (2.0f / (float)c.N);
    p.err = reinterpret_cast<uint32_t*>(c.err_ws ? c.err_ws : c.ws);
    p.wait_ns = c.wait_ns;
    return check_launch(cudaLaunchKernelEx(&cfg, lin_small_f32, p));
}

ttt_status launch_linear(const Call& c) {
    using namespace lin;
    const long long units = (long long)c.batch * c.heads;
    const int tpu = (c.N + TOK - 1) / TOK;
    const WsLayout L = ws_layout(units, c.dtype);

    if (c.dtype == TTT_BF16) {
        const size_t smem = sizeof(ClusterSmem) + 1024;
        cudaFuncSetAttribute(lin_cluster_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        // CTAs per cluster (cs) and clusters (ncl): every cluster co-resident (a second wave would
        // double the time), and the least estimated time.  A CTA streams its 1/cs share of each of its
        // cluster's units (32 KB stages at the per-SM rate, or at its share of HBM when the SMs
        // together would exceed it), and each unit's exchange takes a latency of its own; with two
        // units in flight a unit costs the larger of the two, and the first unit's streaming and the
        // last unit's exchange are not overlapped.  Large units are streaming-bound (fewer units per
        // cluster over more CTAs wins); small ones are exchange-bound (fewest units per cluster wins).
        int cs = 1, ncl = (int)std::min<long long>(units, std::max(1, c.num_sms));
        double best = 1e30;
        const int tpu2 = (c.N + Q2 - 1) / Q2;
        for (int k = 1; k <= kMaxCluster; ++k) {
            const long long n = std::min<long long>(units, c.num_sms / k);
            if (n < 1) break;
            const long long upc = (units + n - 1) / n;
            const long long need = (units + upc - 1) / upc;
            if (k > 1 && max_active_clusters(k, smem) < need) continue;
            const double ctas = (double)need * k;
            const double gbs = std::min(kCtaGBs, kHbmGBs / ctas);                 // per-CTA rate
            const double t_stage = 32768.0 / (gbs * 1e3);                         // us per 32 KB stage
            const double ts = ((tpu + k - 1) / k + (tpu2 + k - 1) / k) * t_stage;  // one unit's share
            const double tx = k > 1 ? kExchangeUs : kExchangeUs1;
            const double cost = (double)upc * std::max(ts, tx) + std::min(ts, tx);
            if (cost <= best * 1.001) { best = std::min(best, cost); cs = k; ncl = (int)need; }   // ties: larger
        }
        ClusterParams p{};
        p.heads = c.heads;
        p.U = (int)units;
        p.N = c.N;
        p.CS = cs;
        p.tpu1 = tpu;
        p.tpu2 = (c.N + Q2 - 1) / Q2;
        p.dot = c.loss == TTT_LOSS_DOT;
        p.eta_scale = p.dot ? -c.eta / (float)c.N : c.eta * (2.0f / (float)c.N);
        p.W0 = c.W0;
        p.W1_out = c.W1_out;
        p.err = reinterpret_cast<uint32_t*>(c.ws);
        p.wait_ns = c.wait_ns;
        CUtensorMap tmK, tmV, tmQ, tmZ;
        if (!make_tmap_tokens(&tmK, c.K, c, TOK) || !make_tmap_tokens(&tmV, c.V, c, TOK) ||
            !make_tmap_tokens(&tmQ, c.Q, c, Q2) || !make_tmap_tokens(&tmZ, c.Z, c, TOK))
            return TTT_ERR_INVALID_ARG;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(ncl * cs));
        if (c.grid_out) *c.grid_out = ncl * cs;
        cfg.blockDim = dim3(kThreadsTc);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = c.stream;
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cs; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
        at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see the kernel's prologue
        at[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 2;
        return check_launch(cudaLaunchKernelEx(&cfg, lin_cluster_bf16, tmK, tmV, tmQ, tmZ, p));
    }

    MergeOut m{};
    m.dot = c.loss == TTT_LOSS_DOT;
    m.eta_scale = m.dot ? c.eta / (float)c.N : c.eta * (2.0f / (float)c.N);
    m.W0 = c.W0;
    m.partials = reinterpret_cast<const float*>(c.ws + L.partials);
    m.W1_out = c.W1_out;

    // fp32
    if (c.N <= kSmallN && c.num_sms >= kSmallCS) return launch_small_f32(c, units);
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
