// minibatch.cu -- linear inner model f(x) = W x trained by mini-batch gradient descent over
// consecutive token batches, the sequential variants of the layer's inner training:
//   prefix ("Vision-TTT" paper notes, section 关键设计 4): the raster-ordered tokens are cut into
//     consecutive mini-batches of b tokens; inside a mini-batch every gradient is taken at the
//     weights W_s the mini-batch starts from, G_t = 2 (W_s k_t - v_t) k_t^T, the weights follow the
//     causal prefix sum W_t = W_s - eta sum_{s<=t} G_s and token t reads out z_t = W_t q_t; the next
//     mini-batch starts from the last W_t.
//   epoch (press article "CVPR 2026 Oral | 清華+阿里發布ViT3", Observation 2 and Fig. 3: 2, 3 or 4
//     consecutive mini-batches, one update each): every mini-batch takes one step of its mean L2
//     loss, W <- W_s - eta (2/|batch|) sum (W_s k_t - v_t) k_t^T, and every query is read out with the
//     final weights.
//
// The loss decomposes over output features, so every row of W is an independent recurrence: row i
// needs only k_t, q_t and the i-th value feature of each token.  A CTA of 128 threads takes 8 rows of
// one unit (8 CTAs per unit), 16 lanes per row and 4 features per lane (4m..4m+3 for lane m, so that
// a row's 16 lanes read a token's 256 contiguous bytes).  Each lane keeps, for its 4 weights, W_s (the weights the mini-batch started from: the residuals are taken there) and dW,
// the update accumulated since, at its own scale (many small per-token terms added straight into W_s
// would each be rounded at the scale of W).  No CTA waits on another.
//
// Streaming: the K, Q and V tiles of a sub-block of 16 tokens (2 KB each in bf16) are brought in by
// 1-D bulk copies into a ring of kStages shared-memory stages, kStages sub-blocks ahead of the
// compute (the unit's sub-blocks are a sequential chain, so the copies must run well ahead to hide
// the memory latency).  Each sub-block is first converted to fp32 tiles.
//
// Per sub-block (sub-blocks never straddle a mini-batch):
//   - each lane forms partial dot products W_s k_t over its 4 features for the 16 tokens, and a
//     transpose-sum over the row's 16 lanes (15 shuffles) leaves lane m with the residual of token
//     m, r_t = W_s k_t - v_t, which is then broadcast to the row's lanes;
//   - token by token, dW -= scale r_t k_t (scale 2 eta, or 2 eta / |batch| in epoch mode), and in
//     prefix mode the partial readout (W_s + dW) . q_t is formed right after token t's own update,
//     so that z_t = W_t q_t; a second transpose-sum completes z;
//   - at the end of a mini-batch W_s += dW, dW = 0.
// Epoch mode then streams Q once more and reads out with the final weights.
//
// Bound: FP32 issue along a sequential chain of N/16 sub-blocks per unit (about 6 d^2 + 4 b d FLOP
// per token and head, the notes' complexity terms).  HBM traffic is that of the full-batch layer,
// 4 N d elements per unit, in both modes (epoch mode reads Q in its second pass instead of the first).
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace mb {

constexpr int D = 64;
constexpr int RB = 8;               // rows of W per CTA
constexpr int LPR = 16;             // lanes per row
constexpr int FPL = D / LPR;        // features per lane
constexpr int T = 16;               // tokens per sub-block
constexpr int THREADS = RB * LPR;   // 128
constexpr int kStages = 4;          // bulk-copy ring depth (sub-blocks in flight)
constexpr int KP = D + 4;           // padded row pitch (floats) of the fp32 K and Q tiles
constexpr int VP = RB + 1;
constexpr int ZP = RB + 1;
constexpr int kCtasPerUnit = D / RB;
constexpr int kTileChunks = T * D / 8;                  // 8-element chunks of a K or Q tile: 128
constexpr int kChunksPerThread = kTileChunks / THREADS; // 1

struct Params {
    const void* Q;
    const void* K;
    const void* V;
    void* Z;
    long long bs, hs;               // element strides of images and heads
    int heads, N, b, mode;          // mode: 0 prefix, 1 epoch
    long long items;                // units * kCtasPerUnit
    float eta;
    const float* W0;                // [heads][64][64]
    float* W1_out;                  // nullable [units][64][64]
    uint32_t* err;                  // workspace error word
    unsigned long long wait_ns;     // bound of every device-side wait
};

// Dynamic shared memory: Ctl, then Tiles, then the ring of raw stages (K, Q, V tiles as loaded).
struct Ctl {
    uint64_t full[kStages];
    int abort_flag;
};
struct Tiles {                      // fp32 tiles of the current sub-block
    float k[T][KP];
    float q[T][KP];
    float v[T][VP];                 // v[t][r]: value feature row0 + r of token t
    float z[T][ZP];                 // the sub-block's readout, [token][row]
};
constexpr size_t kCtlBytes = 128;
static_assert(sizeof(Ctl) <= kCtlBytes, "control block");

template <typename E> struct Io;
template <> struct Io<float> {
    // 8 consecutive elements of a raw tile -> fp32
    static __device__ __forceinline__ void get8(const float* src, float* dst) {
        reinterpret_cast<float4*>(dst)[0] = reinterpret_cast<const float4*>(src)[0];
        reinterpret_cast<float4*>(dst)[1] = reinterpret_cast<const float4*>(src)[1];
    }
    static __device__ __forceinline__ void store1(float* p, float x) { *p = x; }
};
template <> struct Io<__nv_bfloat16> {
    static __device__ __forceinline__ void get8(const __nv_bfloat16* src, float* dst) {
        const uint4 r = *reinterpret_cast<const uint4*>(src);
        reinterpret_cast<float4*>(dst)[0] = make_float4(bf16lo_to_f32(r.x), __uint_as_float(r.x & 0xffff0000u),
                                                        bf16lo_to_f32(r.y), __uint_as_float(r.y & 0xffff0000u));
        reinterpret_cast<float4*>(dst)[1] = make_float4(bf16lo_to_f32(r.z), __uint_as_float(r.z & 0xffff0000u),
                                                        bf16lo_to_f32(r.w), __uint_as_float(r.w & 0xffff0000u));
    }
    static __device__ __forceinline__ void store1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

// One sub-block of the schedule: tokens [t0, t0 + cnt) of phase 0 (training) or 1 (epoch readout).
struct Sub {
    int t0, cnt, phase;
    int batch_len;                  // tokens of the mini-batch the sub-block belongs to (phase 0)
    bool batch_end;                 // the sub-block closes its mini-batch
    __device__ __forceinline__ bool valid() const { return cnt > 0; }
    __device__ __forceinline__ bool reads_kv() const { return phase == 0; }
};

__device__ __forceinline__ Sub make_sub(const Params& p, int t0, int phase) {
    Sub s;
    s.phase = phase;
    s.t0 = t0;
    if (phase == 0) {
        const int bstart = (t0 / p.b) * p.b;
        const int bend = min(p.N, bstart + p.b);
        s.cnt = min(T, bend - t0);
        s.batch_len = bend - bstart;
        s.batch_end = t0 + s.cnt == bend;
    } else {
        s.cnt = min(T, p.N - t0);
        s.batch_len = 0;
        s.batch_end = false;
    }
    return s;
}

__device__ __forceinline__ Sub next_sub(const Params& p, const Sub& s) {
    const int t = s.t0 + s.cnt;
    if (t < p.N) return make_sub(p, t, s.phase);
    if (s.phase == 0 && p.mode == 1) return make_sub(p, 0, 1);
    Sub e;
    e.t0 = p.N; e.cnt = 0; e.phase = s.phase; e.batch_len = 0; e.batch_end = false;
    return e;
}

__device__ __forceinline__ bool reads_q(const Params& p, const Sub& s) { return s.phase == 1 || p.mode == 0; }

// v[0..15]: this lane's partials for tokens 0..15.  Afterwards v[0] holds, in lane m of each group
// of 16 lanes (m = lane & 15), the sum over the group's 16 lanes for token m.
__device__ __forceinline__ void transpose_sum16(float (&v)[T], int lane) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 8;
        const float send = up ? v[i] : v[i + 8];
        const float keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 4;
        const float send = up ? v[i] : v[i + 4];
        const float keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 2;
        const float send = up ? v[i] : v[i + 2];
        const float keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    {
        const bool up = lane & 1;
        const float send = up ? v[0] : v[1];
        const float keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
}

// Lane m's 4 features (4m .. 4m+3) of a 64-wide fp32 row.
__device__ __forceinline__ float dot4(const float (&w)[FPL], const float* row, int m) {
    const float4 a = *reinterpret_cast<const float4*>(row + 4 * m);
    return fmaf(w[3], a.w, fmaf(w[2], a.z, fmaf(w[1], a.y, w[0] * a.x)));
}

// Bounded wait that ignores the abort flag (draining copies that are still in flight).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_test(a, parity) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
}

template <typename E>
__global__ void __launch_bounds__(THREADS)
lin_minibatch(const Params p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Ctl& ctl = *reinterpret_cast<Ctl*>(smem_raw);
    Tiles& s = *reinterpret_cast<Tiles*>(smem_raw + kCtlBytes);
    constexpr uint32_t kTileBytes = T * D * sizeof(E);
    uint8_t* ring = smem_raw + kCtlBytes + ((sizeof(Tiles) + 127) / 128) * 128;
    const int tid = threadIdx.x, lane = tid & 31;
    const int rl = tid >> 4;                        // row of this lane within the CTA's 8 rows
    const int m = tid & 15;                         // feature group; token m after a transpose-sum
    const int gbase = lane & 16;                    // first lane of this row's group of 16
    const Abort ab{&ctl.abort_flag, p.err, p.wait_ns};
    if (tid == 0) {
        ctl.abort_flag = 0;
        for (int i = 0; i < kStages; ++i) mbar_init(&ctl.full[i], 1);
        fence_barrier_init();
    }
    __syncthreads();
    uint32_t it = 0, iss = 0;                       // sub-blocks consumed / issued (thread 0), over all items
    for (long long item = blockIdx.x; item < p.items; item += gridDim.x) {
        const int u = (int)(item / kCtasPerUnit), row0 = (int)(item % kCtasPerUnit) * RB;
        const int img = u / p.heads, h = u % p.heads;
        const size_t off = (size_t)img * p.bs + (size_t)h * p.hs;
        const E* Kb = static_cast<const E*>(p.K) + off;
        const E* Qb = static_cast<const E*>(p.Q) + off;
        const E* Vb = static_cast<const E*>(p.V) + off;
        E* Zb = static_cast<E*>(p.Z) + off;
        const int i = row0 + rl;                    // row of W

        // thread 0 keeps the copies kStages sub-blocks ahead of the compute
        Sub issue = make_sub(p, 0, 0);
        auto issue_next = [&]() {
            const int st = (int)(iss % kStages);
            uint8_t* dst = ring + (size_t)st * 3 * kTileBytes;
            const uint32_t bytes = (uint32_t)issue.cnt * D * sizeof(E);
            const bool kv = issue.reads_kv(), q = reads_q(p, issue);
            mbar_arrive_expect_tx(&ctl.full[st], (kv ? 2u : 0u) * bytes + (q ? bytes : 0u));
            const size_t n = (size_t)issue.t0 * D;
            if (kv) {
                bulk_g2s(dst, Kb + n, bytes, &ctl.full[st]);
                bulk_g2s(dst + 2 * kTileBytes, Vb + n, bytes, &ctl.full[st]);
            }
            if (q) bulk_g2s(dst + kTileBytes, Qb + n, bytes, &ctl.full[st]);
            issue = next_sub(p, issue);
            ++iss;
        };
        if (tid == 0)
            for (int j = 0; j < kStages && issue.valid(); ++j) issue_next();

        float ws[FPL], dw[FPL];
        {
            const float* src = p.W0 + ((size_t)h * D + i) * D;
            const float4 a = __ldg(reinterpret_cast<const float4*>(src + 4 * m));
            ws[0] = a.x; ws[1] = a.y; ws[2] = a.z; ws[3] = a.w;
#pragma unroll
            for (int c = 0; c < FPL; ++c) dw[c] = 0.f;
        }
        for (Sub cur = make_sub(p, 0, 0); cur.valid(); cur = next_sub(p, cur), ++it) {
            const int st = (int)(it % kStages);
            const bool ok = mbar_wait(&ctl.full[st], (it / kStages) & 1u, ab);
            if (__syncthreads_or(!ok)) {
                // a copy did not arrive in time: the error word is set; wait (bounded) for the
                // copies still in flight into this CTA's shared memory, then leave
                if (tid == 0)
                    for (uint32_t j = it; j < iss; ++j) drain_wait(&ctl.full[j % kStages], (j / kStages) & 1u);
                __syncthreads();
                return;
            }
            // raw stage -> fp32 tiles (rows past the sub-block are zero)
            {
                const E* rk = reinterpret_cast<const E*>(ring + (size_t)st * 3 * kTileBytes);
                const E* rq = rk + T * D;
                const E* rv = rq + T * D;
#pragma unroll
                for (int j = 0; j < kChunksPerThread; ++j) {
                    const int c = tid + THREADS * j, tt = c >> 3, f8 = (c & 7) * 8;
                    float* dk = &s.k[tt][f8];
                    float* dq = &s.q[tt][f8];
                    if (tt < cur.cnt) {
                        if (cur.reads_kv()) Io<E>::get8(rk + tt * D + f8, dk);
                        if (reads_q(p, cur)) Io<E>::get8(rq + tt * D + f8, dq);
                    } else {
                        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
                        reinterpret_cast<float4*>(dk)[0] = z4; reinterpret_cast<float4*>(dk)[1] = z4;
                        reinterpret_cast<float4*>(dq)[0] = z4; reinterpret_cast<float4*>(dq)[1] = z4;
                    }
                }
                if (tid < T && cur.reads_kv()) {
                    alignas(16) float tmp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (tid < cur.cnt) Io<E>::get8(rv + tid * D + row0, tmp);
#pragma unroll
                    for (int r = 0; r < RB; ++r) s.v[tid][r] = tmp[r];
                }
            }
            __syncthreads();                                 // tiles ready; the raw stage is free again
            if (tid == 0 && issue.valid()) issue_next();

            float acc[T];
            if (cur.phase == 0) {
                // residuals at the mini-batch's start weights
#pragma unroll
                for (int t = 0; t < T; ++t) acc[t] = dot4(ws, s.k[t], m);
                transpose_sum16(acc, lane);
                const float r = (m < cur.cnt) ? acc[0] - s.v[m][rl] : 0.f;
                const float scale = (p.mode == 0) ? 2.0f * p.eta : 2.0f * p.eta / (float)cur.batch_len;
                // token by token: dW -= scale r_t k_t, then (prefix mode) the partial readout
                // W_s . q_t + dW . q_t, so that z_t = W_t q_t
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float c = -scale * __shfl_sync(0xffffffffu, r, gbase + t);
                    const float4 ka = *reinterpret_cast<const float4*>(&s.k[t][4 * m]);
                    dw[0] = fmaf(c, ka.x, dw[0]); dw[1] = fmaf(c, ka.y, dw[1]);
                    dw[2] = fmaf(c, ka.z, dw[2]); dw[3] = fmaf(c, ka.w, dw[3]);
                    if (p.mode == 0) acc[t] = dot4(ws, s.q[t], m) + dot4(dw, s.q[t], m);
                }
                if (cur.batch_end) {
#pragma unroll
                    for (int c = 0; c < FPL; ++c) { ws[c] += dw[c]; dw[c] = 0.f; }
                }
            } else {
                // epoch-mode readout with the final weights
#pragma unroll
                for (int t = 0; t < T; ++t) acc[t] = dot4(ws, s.q[t], m);
            }
            const bool writes_z = reads_q(p, cur);
            if (writes_z) {
                transpose_sum16(acc, lane);
                s.z[m][rl] = acc[0];
            }
            __syncthreads();
            if (writes_z) {
#pragma unroll
                for (int j = 0; j < T * RB / THREADS; ++j) {
                    const int e = tid + THREADS * j, tt = e / RB, r = e % RB;
                    if (tt < cur.cnt) Io<E>::store1(Zb + (size_t)(cur.t0 + tt) * D + row0 + r, s.z[tt][r]);
                }
            }
        }
        if (p.W1_out) {
            float* dst = p.W1_out + ((size_t)u * D + i) * D;
            *reinterpret_cast<float4*>(dst + 4 * m) = make_float4(ws[0], ws[1], ws[2], ws[3]);
        }
    }
}

template <typename E>
static size_t smem_bytes() {
    return kCtlBytes + ((sizeof(Tiles) + 127) / 128) * 128 + (size_t)kStages * 3 * T * D * sizeof(E);
}

template <typename E>
static ttt_status launch(const Call& c, int b, int mode) {
    Params p{};
    p.Q = c.Q; p.K = c.K; p.V = c.V; p.Z = c.Z;
    p.bs = c.bs; p.hs = c.hs;
    p.heads = c.heads; p.N = c.N; p.b = b; p.mode = mode;
    p.items = (long long)c.batch * c.heads * kCtasPerUnit;
    p.eta = c.eta;
    p.W0 = c.W0;
    p.W1_out = c.W1_out;
    p.err = reinterpret_cast<uint32_t*>(c.ws);
    p.wait_ns = c.wait_ns;
    const size_t smem = smem_bytes<E>();
    cudaFuncSetAttribute(lin_minibatch<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lin_minibatch<E>, THREADS, smem) != cudaSuccess) {
        cudaGetLastError();
        per_sm = 1;
    }
    const long long grid = std::max<long long>(1, std::min<long long>(p.items, (long long)c.num_sms * std::max(1, per_sm)));
    lin_minibatch<E><<<(unsigned)grid, THREADS, smem, c.stream>>>(p);
    return check_launch(cudaGetLastError());
}

}  // namespace mb

ttt_status launch_linear_minibatch(const Call& c, int b, int mode) {
    if (c.dtype == TTT_BF16) return mb::launch<__nv_bfloat16>(c, b, mode);
    return mb::launch<float>(c, b, mode);
}

}  // namespace ttt
