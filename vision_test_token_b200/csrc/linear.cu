// linear.cu -- linear inner model f(x) = W x of the TTT layer (one d x d state per head; Vision-TTT
// paper notes, section 关键设计 1), one full-batch step of the L2 loss (press article "CVPR 2026
// Oral | 清華+阿里發布ViT3", Observation 2) written in Gram form:
//     G = sum_n k_n k_n^T,   C = sum_n v_n k_n^T,   W1 = W0 - eta (2/N) (W0 G - C),   z_n = W1 q_n.
//
// Phase 1 (lin_p1_*): every CTA owns a contiguous range of 128-token tiles of the flattened
//   (unit, tile) index space.  For each unit it touches it accumulates the stacked product
//   [K | V]^T K  (a 128 x 64 fp32 block: rows 0..63 = G, rows 64..127 = C) and writes it to a
//   partial slot.  The last CTA to finish a unit (atomic arrival count, no waiting) sums that
//   unit's partial slots in CTA order -- a fixed order, so the result is deterministic -- and forms
//   W1 in fp32.
// Phase 2 (lin_p2_*): streams Q tiles and writes Z = Q W1^T; launched with programmatic dependent
//   launch so its prologue and first Q loads overlap the end of phase 1.
//
// bf16 path: TMA (128-byte swizzle) stages K/V/Q tiles, tcgen05.mma accumulates in tensor memory.
//   Phase 1 uses one MMA stream for both G and C: A = [K | V]^T (M = 128, MN-major straight from
//   the token-major tiles), B = K (N = 64, MN-major), K-dim = tokens.
//   Phase 2: A = Q tile (M = 128 tokens, K-major), B = W1 (bf16, K-major), D = 128 x 64 fp32.
// fp32 path: plain fp32 FMA (keeps fp32 accuracy; used for fp32 inputs).
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace lin {

constexpr int D = 64;
constexpr int TOK = 128;                    // tokens per tile
constexpr int TILE_BYTES = TOK * D * 2;     // one bf16 tile: 16 KB
constexpr int P1_STAGES = 4;
constexpr int P2_STAGES = 4;
constexpr int kMaxGrid = 160;               // CTAs per phase at most (>= SM count of a B200)
constexpr int kPartialFloats = 2 * D * D;   // [G ; C] = 128 x 64
constexpr int kThreadsTc = 192;             // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr uint32_t kIdescP1 = idesc_bf16_f32(128, 64, true, true);
constexpr uint32_t kIdescP2 = idesc_bf16_f32(128, 64, false, false);

// Flat static partition of T tiles over G CTAs: CTA c owns tiles [start(c), start(c+1)).
struct Partition {
    long long T;
    int G;
    __host__ __device__ long long start(int c) const { return (long long)c * T / G; }
    __host__ __device__ int cta_of(long long t) const { return (int)(((t + 1) * G - 1) / T); }
};

struct P1Params {
    int heads, tpu;             // tiles per unit
    Partition part;
    float eta_scale;            // eta * 2 / N
    const float* W0;            // [heads][64][64]
    float* W1_out;              // nullable [units][64][64]
    __nv_bfloat16* W1_bf16;     // workspace (bf16 path)
    float* W1_f32;              // workspace (fp32 path)
    float* partials;            // workspace [(kMaxGrid + units)][128][64]
    unsigned* counters;         // workspace [units]
    uint32_t* err;
};

struct P2Params {
    int heads, tpu, N;
    Partition part;
    uint32_t* err;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------------------------------------------
// Merge of one unit by NT threads (tid in [0, NT)): fixed-order sum of the partial slots of CTAs
// cf..cl, then W1 = W0 - eta_scale * (W0 G - C).  gc: 128 x 64 floats, w0: 64 x 65 floats (smem).
// ------------------------------------------------------------------------------------------------
template <int NT, int BAR_ID>
__device__ void merge_unit(const P1Params& p, int u, int cf, int cl, int tid, float* gc, float* w0) {
    constexpr int V4 = kPartialFloats / 4;      // float4 per partial
    constexpr int PER = V4 / NT;
    float4 acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int cc = cf; cc <= cl; ++cc) {
        const float4* src = reinterpret_cast<const float4*>(p.partials + (size_t)(cc + u) * kPartialFloats);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const float4 v = __ldcg(src + i * NT + tid);
            acc[i].x += v.x; acc[i].y += v.y; acc[i].z += v.z; acc[i].w += v.w;
        }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) reinterpret_cast<float4*>(gc)[i * NT + tid] = acc[i];
    const int h = u % p.heads;
    const float* W0h = p.W0 + (size_t)h * D * D;
    for (int e = tid; e < D * D; e += NT) w0[(e / D) * 65 + (e % D)] = __ldg(W0h + e);
    named_bar_sync(BAR_ID, NT);

    constexpr int OUT = D * D / NT;             // outputs per thread, one row segment
    constexpr int SEGS = D / OUT;
    const int i = tid / SEGS;
    const int j0 = (tid % SEGS) * OUT;
    float m[OUT];
#pragma unroll
    for (int jj = 0; jj < OUT; ++jj) m[jj] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
        const float w = w0[i * 65 + k];
        const float4* g4 = reinterpret_cast<const float4*>(gc + k * D + j0);
#pragma unroll
        for (int q = 0; q < OUT / 4; ++q) {
            const float4 g = g4[q];
            m[4 * q + 0] = fmaf(w, g.x, m[4 * q + 0]);
            m[4 * q + 1] = fmaf(w, g.y, m[4 * q + 1]);
            m[4 * q + 2] = fmaf(w, g.z, m[4 * q + 2]);
            m[4 * q + 3] = fmaf(w, g.w, m[4 * q + 3]);
        }
    }
    float w1[OUT];
#pragma unroll
    for (int jj = 0; jj < OUT; ++jj)
        w1[jj] = w0[i * 65 + j0 + jj] - p.eta_scale * (m[jj] - gc[(D + i) * D + j0 + jj]);
    const size_t row = ((size_t)u * D + i) * D + j0;
    if (p.W1_out) {
#pragma unroll
        for (int q = 0; q < OUT / 4; ++q)
            reinterpret_cast<float4*>(p.W1_out + row)[q] = make_float4(w1[4 * q], w1[4 * q + 1], w1[4 * q + 2], w1[4 * q + 3]);
    }
    if (p.W1_bf16) {
#pragma unroll
        for (int q = 0; q < OUT / 8; ++q) {
            uint4 pk;
            pk.x = pack_bf16x2(w1[8 * q + 0], w1[8 * q + 1]);
            pk.y = pack_bf16x2(w1[8 * q + 2], w1[8 * q + 3]);
            pk.z = pack_bf16x2(w1[8 * q + 4], w1[8 * q + 5]);
            pk.w = pack_bf16x2(w1[8 * q + 6], w1[8 * q + 7]);
            reinterpret_cast<uint4*>(p.W1_bf16 + row)[q] = pk;
        }
    }
    if (p.W1_f32) {
#pragma unroll
        for (int q = 0; q < OUT / 4; ++q)
            reinterpret_cast<float4*>(p.W1_f32 + row)[q] = make_float4(w1[4 * q], w1[4 * q + 1], w1[4 * q + 2], w1[4 * q + 3]);
    }
}

// Arrival on unit u after this CTA's partial slot is written (called by NT threads after a
// __threadfence and a barrier).  Returns true in every thread if this CTA is the unit's last.
template <int NT, int BAR_ID>
__device__ bool arrive_unit(const P1Params& p, int c, int u, int tid, int* flag_smem, int& cf, int& cl) {
    cf = p.part.cta_of((long long)u * p.tpu);
    cl = p.part.cta_of((long long)(u + 1) * p.tpu - 1);
    if (tid == 0) {
        const unsigned expected = (unsigned)(cl - cf + 1);
        const unsigned old = atomicAdd(p.counters + u, 1u);
        *flag_smem = (old + 1u == expected) ? 1 : 0;
    }
    named_bar_sync(BAR_ID, NT);
    const bool last = *reinterpret_cast<volatile int*>(flag_smem) != 0;
    if (last) __threadfence();
    return last;
}

// ------------------------------------------------------------------------------------------------
// Phase 1, bf16, tcgen05
// ------------------------------------------------------------------------------------------------
struct P1Smem {
    uint8_t kv[P1_STAGES][2][TILE_BYTES];   // K tile then V tile per stage (1024-aligned)
    float gc[kPartialFloats];
    float w0[D * 65];
    uint64_t full[P1_STAGES], empty[P1_STAGES];
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
    int last_flag;
};

__global__ void __launch_bounds__(kThreadsTc, 1)
lin_p1_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const P1Params p) {
    extern __shared__ uint8_t smem_raw[];
    P1Smem& s = *reinterpret_cast<P1Smem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const long long t_begin = p.part.start(c), t_end = p.part.start(c + 1);
    const Abort ab{&s.abort_flag, p.err};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < P1_STAGES; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
        fence_barrier_init();
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 128); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    pdl_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {                                    // TMA producer
            int stage = 0; uint32_t phase = 0;
            for (long long t = t_begin; t < t_end; ++t) {
                if (!mbar_wait(&s.empty[stage], phase ^ 1u, ab)) break;
                const int u = (int)(t / p.tpu), ti = (int)(t % p.tpu);
                const int b = u / p.heads, h = u % p.heads;
                mbar_arrive_expect_tx(&s.full[stage], 2 * TILE_BYTES);
                tma_load_4d(s.kv[stage][0], &tmK, &s.full[stage], 0, ti * TOK, h, b);
                tma_load_4d(s.kv[stage][1], &tmV, &s.full[stage], 0, ti * TOK, h, b);
                if (++stage == P1_STAGES) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {                                    // MMA issuer
            int stage = 0; uint32_t phase = 0; int seg = 0;
            long long t = t_begin;
            bool ok = true;
            while (ok && t < t_end) {
                const int u = (int)(t / p.tpu);
                const long long seg_end = min(t_end, (long long)(u + 1) * p.tpu);
                const int ai = seg & 1;
                if (!mbar_wait(&s.acc_empty[ai], (((uint32_t)seg >> 1) & 1u) ^ 1u, ab)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + (uint32_t)(ai * 64);
                bool first = true;
                for (; t < seg_end; ++t) {
                    if (!mbar_wait(&s.full[stage], phase, ab)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sK = smem_u32(s.kv[stage][0]);
#pragma unroll
                    for (int kk = 0; kk < TOK / 16; ++kk) {
                        // 16 tokens per MMA = two 8-row groups (2 x 1024 bytes)
                        const uint64_t ad = sdesc_sw128(sK + kk * 2048, TILE_BYTES, 1024);
                        const uint64_t bd = sdesc_sw128(sK + kk * 2048, TILE_BYTES, 1024);
                        mma_bf16_ss(dacc, ad, bd, kIdescP1, (first && kk == 0) ? 0u : 1u);
                    }
                    first = false;
                    mma_commit(&s.empty[stage]);
                    if (++stage == P1_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(&s.acc_full[ai]);
                ++seg;
            }
        }
    } else {                                                // epilogue warps 2..5
        const int q = warp & 3;                             // TMEM lane quarter of this warp
        const int r = q * 32 + lane;                        // row of [G ; C]
        const int tid = threadIdx.x - 64;
        int seg = 0;
        long long t = t_begin;
        while (t < t_end) {
            const int u = (int)(t / p.tpu);
            t = min(t_end, (long long)(u + 1) * p.tpu);
            const int ai = seg & 1;
            if (!mbar_wait(&s.acc_full[ai], ((uint32_t)seg >> 1) & 1u, ab)) break;
            __syncwarp();
            tc_fence_after();
            float* dst = p.partials + (size_t)(c + u) * kPartialFloats + (size_t)r * D;
#pragma unroll
            for (int j = 0; j < D; j += 16) {
                float v[16];
                tmem_ld16(tmem + (uint32_t)(ai * 64 + j) + ((uint32_t)(q * 32) << 16), v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4*>(dst + j + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            }
            tc_fence_before();
            mbar_arrive(&s.acc_empty[ai]);
            __threadfence();
            named_bar_sync(1, 128);
            int cf, cl;
            if (arrive_unit<128, 1>(p, c, u, tid, &s.last_flag, cf, cl)) {
                merge_unit<128, 1>(p, u, cf, cl, tid, s.gc, s.w0);
                if (tid == 0) p.counters[u] = 0u;
            }
            named_bar_sync(1, 128);
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ------------------------------------------------------------------------------------------------
// Phase 2, bf16, tcgen05
// ------------------------------------------------------------------------------------------------
struct P2Smem {
    uint8_t q[P2_STAGES][TILE_BYTES];
    uint8_t z[2][TILE_BYTES];
    uint8_t w1[2][D * D * 2];
    uint64_t full[P2_STAGES], empty[P2_STAGES];
    uint64_t w_full[2], w_empty[2];
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(kThreadsTc, 1)
lin_p2_bf16(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmZ,
            const __grid_constant__ CUtensorMap tmW1, const P2Params p) {
    extern __shared__ uint8_t smem_raw[];
    P2Smem& s = *reinterpret_cast<P2Smem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const long long t_begin = p.part.start(c), t_end = p.part.start(c + 1);
    const Abort ab{&s.abort_flag, p.err};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < P2_STAGES; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.w_full[i], 1); mbar_init(&s.w_empty[i], 1);
            mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128);
        }
        fence_barrier_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmZ);
        prefetch_tmap(&tmW1);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 128); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        if (lane == 0) {                                    // TMA producer
            // Q does not depend on phase 1: the first stages are loaded before waiting for it.
            const int npro = (int)min((long long)P2_STAGES, t_end - t_begin);
            for (int i = 0; i < npro; ++i) {
                const long long t = t_begin + i;
                const int u = (int)(t / p.tpu), ti = (int)(t % p.tpu);
                mbar_arrive_expect_tx(&s.full[i], TILE_BYTES);
                tma_load_4d(s.q[i], &tmQ, &s.full[i], 0, ti * TOK, u % p.heads, u / p.heads);
            }
            pdl_wait_primary();
            int stage = npro % P2_STAGES;
            uint32_t phase = (npro == P2_STAGES) ? 1u : 0u;
            int useg = -1, prev_u = -1;
            for (long long t = t_begin; t < t_end; ++t) {
                const int u = (int)(t / p.tpu), ti = (int)(t % p.tpu);
                if (u != prev_u) {
                    ++useg;
                    const int wb = useg & 1;
                    if (!mbar_wait(&s.w_empty[wb], (((uint32_t)useg >> 1) & 1u) ^ 1u, ab)) break;
                    mbar_arrive_expect_tx(&s.w_full[wb], D * D * 2);
                    tma_load_2d(s.w1[wb], &tmW1, &s.w_full[wb], 0, u * D);
                    prev_u = u;
                }
                if (t - t_begin >= npro) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1u, ab)) break;
                    mbar_arrive_expect_tx(&s.full[stage], TILE_BYTES);
                    tma_load_4d(s.q[stage], &tmQ, &s.full[stage], 0, ti * TOK, u % p.heads, u / p.heads);
                    if (++stage == P2_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {                                    // MMA issuer
            int stage = 0; uint32_t phase = 0;
            int useg = -1, prev_u = -1, ti_local = 0;
            for (long long t = t_begin; t < t_end; ++t, ++ti_local) {
                const int u = (int)(t / p.tpu);
                if (u != prev_u) {
                    if (useg >= 0) mma_commit(&s.w_empty[useg & 1]);
                    ++useg;
                    if (!mbar_wait(&s.w_full[useg & 1], ((uint32_t)useg >> 1) & 1u, ab)) break;
                    prev_u = u;
                }
                const int ai = ti_local & 1;
                if (!mbar_wait(&s.acc_empty[ai], (((uint32_t)ti_local >> 1) & 1u) ^ 1u, ab)) break;
                if (!mbar_wait(&s.full[stage], phase, ab)) break;
                tc_fence_after();
                const uint32_t sQ = smem_u32(s.q[stage]);
                const uint32_t sW = smem_u32(s.w1[useg & 1]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(sQ + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sW + kk * 32, 16, 1024);
                    mma_bf16_ss(tmem + (uint32_t)(ai * 64), ad, bd, kIdescP2, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s.empty[stage]);
                mma_commit(&s.acc_full[ai]);
                if (++stage == P2_STAGES) { stage = 0; phase ^= 1u; }
            }
        }
    } else {                                                // epilogue warps 2..5
        const int q = warp & 3;
        const int r = q * 32 + lane;                        // token row within the tile
        const int tid = threadIdx.x - 64;
        int ti_local = 0;
        for (long long t = t_begin; t < t_end; ++t, ++ti_local) {
            const int u = (int)(t / p.tpu), ti = (int)(t % p.tpu);
            const int ai = ti_local & 1;
            if (!mbar_wait(&s.acc_full[ai], ((uint32_t)ti_local >> 1) & 1u, ab)) break;
            __syncwarp();
            tc_fence_after();
            const int zb = ti_local & 1;
            if (ti_local >= 2) {
                if (tid == 0) bulk_wait_read<1>();
                named_bar_sync(1, 128);
            }
            uint8_t* zrow = s.z[zb] + r * 128;
#pragma unroll
            for (int j = 0; j < D; j += 16) {
                float v[16];
                tmem_ld16(tmem + (uint32_t)(ai * 64 + j) + ((uint32_t)(q * 32) << 16), v);
                tmem_ld_wait();
                uint4 lo, hi;
                lo.x = pack_bf16x2(v[0], v[1]);   lo.y = pack_bf16x2(v[2], v[3]);
                lo.z = pack_bf16x2(v[4], v[5]);   lo.w = pack_bf16x2(v[6], v[7]);
                hi.x = pack_bf16x2(v[8], v[9]);   hi.y = pack_bf16x2(v[10], v[11]);
                hi.z = pack_bf16x2(v[12], v[13]); hi.w = pack_bf16x2(v[14], v[15]);
                const int c0 = j / 8;                       // 16-byte chunk index of columns j..j+7
                *reinterpret_cast<uint4*>(zrow + (((c0) ^ (r & 7)) << 4)) = lo;
                *reinterpret_cast<uint4*>(zrow + (((c0 + 1) ^ (r & 7)) << 4)) = hi;
            }
            tc_fence_before();
            mbar_arrive(&s.acc_empty[ai]);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (tid == 0) {
                tma_store_4d(&tmZ, s.z[zb], 0, ti * TOK, u % p.heads, u / p.heads);
                bulk_commit();
            }
        }
        if (tid == 0) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ------------------------------------------------------------------------------------------------
// fp32 path (plain FMA): same partition, partial slots and merge as the bf16 path.
// ------------------------------------------------------------------------------------------------
constexpr int kThreadsF32 = 256;
constexpr int F32_CHUNK = 32;   // tokens staged in shared memory at a time

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
    float w0[D * 65];
    int last_flag;
};

__global__ void __launch_bounds__(kThreadsF32)
lin_p1_f32(TokenView Kv, TokenView Vv, int N, const P1Params p) {
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
        const int n_end = min(N, (int)((seg_end - (long long)u * p.tpu) * TOK));
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
        int cf, cl;
        if (arrive_unit<kThreadsF32, 0>(p, c, u, tid, &s.last_flag, cf, cl)) {
            merge_unit<kThreadsF32, 0>(p, u, cf, cl, tid, s.gc, s.w0);
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
lin_p2_f32(TokenView Qv, float* Z, long long zbs, long long zhs, const float* W1, const P2Params p) {
    extern __shared__ uint8_t smem_raw[];
    P2SmemF32& s = *reinterpret_cast<P2SmemF32*>(align1024(smem_raw));
    const int tid = threadIdx.x;
    const long long t = blockIdx.x;                        // one tile per CTA
    const int u = (int)(t / p.tpu), ti = (int)(t % p.tpu);
    const int n0 = ti * TOK;
    for (int e = tid; e < TOK * D; e += kThreadsF32) {
        const int tk = e / D, cc = e % D;
        const int n = n0 + tk;
        s.q[tk][cc] = (n < p.N) ? Qv.row(u, p.heads, n)[cc] : 0.f;
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
    if (n < p.N) {
        float* dst = Z + (long long)(u / p.heads) * zbs + (long long)(u % p.heads) * zhs + (long long)n * D + o0;
#pragma unroll
        for (int oo = 0; oo < 32; oo += 4)
            *reinterpret_cast<float4*>(dst + oo) = make_float4(acc[oo], acc[oo + 1], acc[oo + 2], acc[oo + 3]);
    }
}

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
struct WsLayout {
    size_t counters, w1, partials, total;
};

static WsLayout ws_layout(long long units, int dtype) {
    WsLayout L;
    L.counters = kWsHeader;
    L.w1 = align_up(L.counters + (size_t)units * sizeof(unsigned), 1024);
    const size_t w1_elem = (dtype == TTT_BF16) ? 2 : 4;
    L.partials = align_up(L.w1 + (size_t)units * D * D * w1_elem, 1024);
    L.total = L.partials + (size_t)(kMaxGrid + units) * kPartialFloats * sizeof(float);
    return L;
}

template <typename T>
static size_t smem_bytes() { return sizeof(T) + 1024; }

}  // namespace lin

size_t linear_ws_bytes(const ttt_shape& s) {
    return lin::ws_layout((long long)s.batch * s.heads, s.dtype).total;
}

ttt_status launch_linear(const Call& c) {
    using namespace lin;
    const long long units = (long long)c.batch * c.heads;
    const int tpu = (c.N + TOK - 1) / TOK;
    const long long T = units * tpu;
    const WsLayout L = ws_layout(units, c.dtype);
    const int G = (int)std::min<long long>(std::min(c.num_sms, kMaxGrid), T);

    P1Params p1{};
    p1.heads = c.heads;
    p1.tpu = tpu;
    p1.part = Partition{T, G};
    p1.eta_scale = c.eta * (2.0f / (float)c.N);
    p1.W0 = c.W0;
    p1.W1_out = c.W1_out;
    p1.W1_bf16 = (c.dtype == TTT_BF16) ? reinterpret_cast<__nv_bfloat16*>(c.ws + L.w1) : nullptr;
    p1.W1_f32 = (c.dtype == TTT_FP32) ? reinterpret_cast<float*>(c.ws + L.w1) : nullptr;
    p1.partials = reinterpret_cast<float*>(c.ws + L.partials);
    p1.counters = reinterpret_cast<unsigned*>(c.ws + L.counters);
    p1.err = reinterpret_cast<uint32_t*>(c.ws);

    P2Params p2{};
    p2.heads = c.heads;
    p2.tpu = tpu;
    p2.N = c.N;
    p2.err = p1.err;

    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;

    if (c.dtype == TTT_BF16) {
        CUtensorMap tmK, tmV, tmQ, tmZ, tmW1;
        if (!make_tmap_tokens(&tmK, c.K, c, TOK) || !make_tmap_tokens(&tmV, c.V, c, TOK) ||
            !make_tmap_tokens(&tmQ, c.Q, c, TOK) || !make_tmap_tokens(&tmZ, c.Z, c, TOK) ||
            !make_tmap_matrix(&tmW1, c.ws + L.w1, units * D, D, D))
            return TTT_ERR_INVALID_ARG;
        const size_t sm1 = smem_bytes<P1Smem>(), sm2 = smem_bytes<P2Smem>();
        cudaFuncSetAttribute(lin_p1_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
        cudaFuncSetAttribute(lin_p2_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
        lin_p1_bf16<<<G, kThreadsTc, sm1, c.stream>>>(tmK, tmV, p1);
        ttt_status st = check_launch(cudaGetLastError());
        if (st != TTT_OK) return st;
        const int G2 = G;
        p2.part = Partition{T, G2};
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(G2);
        cfg.blockDim = dim3(kThreadsTc);
        cfg.dynamicSmemBytes = sm2;
        cfg.stream = c.stream;
        cfg.attrs = pdl;
        cfg.numAttrs = 1;
        return check_launch(cudaLaunchKernelEx(&cfg, lin_p2_bf16, tmQ, tmZ, tmW1, p2));
    }

    // fp32
    const size_t sm1 = smem_bytes<P1SmemF32>(), sm2 = smem_bytes<P2SmemF32>();
    cudaFuncSetAttribute(lin_p1_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    cudaFuncSetAttribute(lin_p2_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    TokenView Kv{static_cast<const float*>(c.K), c.bs, c.hs};
    TokenView Vv{static_cast<const float*>(c.V), c.bs, c.hs};
    TokenView Qv{static_cast<const float*>(c.Q), c.bs, c.hs};
    lin_p1_f32<<<G, kThreadsF32, sm1, c.stream>>>(Kv, Vv, c.N, p1);
    ttt_status st = check_launch(cudaGetLastError());
    if (st != TTT_OK) return st;
    p2.part = Partition{T, (int)std::min<long long>(T, 1 << 30)};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)T);
    cfg.blockDim = dim3(kThreadsF32);
    cfg.dynamicSmemBytes = sm2;
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return check_launch(cudaLaunchKernelEx(&cfg, lin_p2_f32, Qv, static_cast<float*>(c.Z), c.bs, c.hs,
                                           static_cast<const float*>(p1.W1_f32), p2));
}

}  // namespace ttt
