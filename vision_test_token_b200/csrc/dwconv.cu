// dwconv.cu -- 3x3 depthwise-convolution inner model of the TTT layer over the H x W token grid
// (press article "CVPR 2026 Oral | 清華+阿里發布ViT3", Observation 6 and Fig. 5 part 3; ViT^3 keeps
// one such head).  One full-batch step of the L2 loss, then the readout:
//     r[c,y,x] = sum_{a,b} W0[c][a][b] K[c,y+a-1,x+b-1] - V[c,y,x]           (zero padding)
//     g[c][a][b] = (2/N) sum_{y,x} r[c,y,x] K[c,y+a-1,x+b-1],   W1 = W0 - eta g
//     Z[c,y,x] = sum_{a,b} W1[c][a][b] Q[c,y+a-1,x+b-1]
//
// Not a contraction worth a tensor core (about 7 flop per byte): packed fp32x2 FMA.
//
// One kernel, one thread-block cluster of CS CTAs per unit (one CTA per SM).  A unit's grid is cut
// into bands of R output rows of one strip of at most XT columns; each CTA of the cluster takes a
// contiguous share of the bands.
//   Phase 1: a producer lane moves each band with two TMA tile loads -- K rows y0-1 .. y0+R with a
//     one-column halo, V rows y0 .. y0+R-1 -- into a shared-memory stage; the tensor map's
//     out-of-bounds zero fill supplies the zero padding, so the inner loops carry no bounds checks.
//     16 compute warps work from shared memory: warp w owns output row w / 8 of the band and an
//     eighth of its columns, lane l owns channels 2l and 2l+1, and a 3 x 3 register window slides
//     along the columns.
//   Exchange: the warps' 64 x 9 gradients are summed in a fixed order into the CTA's partial, which
//     is pushed with one bulk copy into every other CTA of the cluster (distributed shared memory,
//     completion on the receiver's mbarrier); each CTA sums the CS partials in rank order (a fixed
//     order: bitwise deterministic) and forms W1.  Meanwhile the producer keeps loading Q bands.
//   Phase 2: the same band staging for Q; Z is written straight from registers (128 coalesced
//     bytes per token and warp).
#include <algorithm>
#include <mutex>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace dw {

constexpr int D = 64;
constexpr int TAPS = 9;
constexpr int R = 2;                        // output rows per band
constexpr int CW = 16;                      // compute warps
constexpr int WPR = CW / R;                 // compute warps per output row
constexpr int THREADS = (CW + 1) * 32;      // + one producer warp
constexpr int kPart = D * TAPS;             // 576 floats: a 64 x 9 gradient or kernel, tap-major
constexpr int kMaxCluster = 16;
constexpr int STAGES = 2;

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {                 // two bf16 channels in one 32-bit word
    using Raw = uint32_t;
    static constexpr int kTokenBytes = D * 2;
    static constexpr int kXtMax = 80;
    static __device__ __forceinline__ float2 unpack(Raw w) { return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w)); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float2 v) {
        *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v.x, v.y);
    }
};
template <>
struct Elem<float> {
    using Raw = float2;
    static constexpr int kTokenBytes = D * 4;
    static constexpr int kXtMax = 40;
    static __device__ __forceinline__ float2 unpack(Raw w) { return w; }
    static __device__ __forceinline__ void store(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
};

struct Geom {
    int heads, H, W;
    int Sx, XT, Hb;                  // strips, strip width, bands per strip
    int bands_per_unit;              // Sx * Hb
    long long bs, hs;                // element strides of Q/K/V/Z
    int k_pitch;                     // tokens per staged K/Q row (XT + 2)
    uint32_t k_bytes, v_bytes;       // bytes of the staged K/Q rows and V rows of a band
    uint32_t stage_bytes;
};

struct Params {
    Geom g;
    int U, CS;
    float eta_scale;                 // eta * 2 / N
    const float* W0;                 // [heads][64][9]
    float* W1_out;                   // nullable [units][64][9]
    uint32_t* err;
};

struct Band {
    int s, y0, xs, xe;               // strip, first output row, output columns [xs, xe)
};

__device__ __forceinline__ Band decode_band(const Geom& g, int b) {
    Band r;
    r.s = b / g.Hb;
    r.y0 = (b % g.Hb) * R;
    r.xs = r.s * g.XT;
    r.xe = min(g.W, r.xs + g.XT);
    return r;
}

struct SmemTail {                            // follows the stages
    float red[CW][kPart];                    // per-warp gradients (phase 1)
    float recv[kMaxCluster - 1][kPart];      // the peers' partials
    float mine[kPart];                       // this CTA's partial (sent to the peers)
    float w1[kPart];                         // W1 of the unit, tap-major
    uint64_t full[STAGES], empty[STAGES];
    uint64_t recv_full, peer_free;
    int abort_flag;
};

__device__ __forceinline__ int split_lo(int n, int r, int parts) { return (int)((long long)n * r / parts); }

// Channel pair `lane` of staged row `row`, column `col` (no bounds checks: the halo is staged).
template <typename T>
__device__ __forceinline__ float2 staged(const uint8_t* base, int pitch, int row, int col, int lane) {
    return Elem<T>::unpack(reinterpret_cast<const typename Elem<T>::Raw*>(
        base + ((size_t)row * pitch + col) * Elem<T>::kTokenBytes)[lane]);
}

template <typename T>
__global__ void __launch_bounds__(THREADS, 1)
dw_cluster(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
           const __grid_constant__ CUtensorMap tmQ, T* __restrict__ Z, const Params p) {
    using E = Elem<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const Geom& g = p.g;
    uint8_t* stages = base;
    SmemTail& s = *reinterpret_cast<SmemTail*>(base + (size_t)STAGES * g.stage_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank(), cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
    const bool multi = p.CS > 1;
    const Abort ab{&s.abort_flag, p.err};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], CW); }
        mbar_init(&s.recv_full, 1);
        mbar_init(&s.peer_free, (uint32_t)(multi ? p.CS - 1 : 1));
        fence_barrier_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmQ);
    }
    __syncthreads();
    // every CTA's barriers exist before any peer arrives on them
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");

    const int b_lo = split_lo(g.bands_per_unit, rank, p.CS), b_hi = split_lo(g.bands_per_unit, rank + 1, p.CS);

    if (warp == CW) {                                                // producer
        if (lane == 0) {
            int st = 0; uint32_t ph = 0;
            for (int u = cid; u < p.U; u += ncl) {
                const int bi = u / g.heads, h = u % g.heads;
                for (int b = b_lo; b < b_hi; ++b) {
                    const Band bd = decode_band(g, b);
                    if (!mbar_wait(&s.empty[st], ph ^ 1u, ab)) return;
                    uint8_t* sp = stages + (size_t)st * g.stage_bytes;
                    mbar_arrive_expect_tx(&s.full[st], g.k_bytes + g.v_bytes);
                    tma_load_5d(sp, &tmK, &s.full[st], 0, bd.xs - 1, bd.y0 - 1, h, bi);
                    tma_load_5d(sp + g.k_bytes, &tmV, &s.full[st], 0, bd.xs, bd.y0, h, bi);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
                // Q does not depend on W1: it streams in while the cluster exchanges its partials.
                for (int b = b_lo; b < b_hi; ++b) {
                    const Band bd = decode_band(g, b);
                    if (!mbar_wait(&s.empty[st], ph ^ 1u, ab)) return;
                    uint8_t* sp = stages + (size_t)st * g.stage_bytes;
                    mbar_arrive_expect_tx(&s.full[st], g.k_bytes);
                    tma_load_5d(sp, &tmQ, &s.full[st], 0, bd.xs - 1, bd.y0 - 1, h, bi);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
            }
        }
        return;
    }

    // compute warps
    const int tid = threadIdx.x;                                     // 0 .. CW*32-1
    const int orow = warp / WPR, oseg = warp % WPR;
    int st = 0; uint32_t ph = 0;
    uint32_t k = 0;
    bool failed = false;
    for (int u = cid; u < p.U && !failed; u += ncl, ++k) {
        const int bi = u / g.heads, h = u % g.heads;
        if (multi && tid == 0) {                                     // my receive slots are free: arm, then tell the peers
            mbar_arrive_expect_tx(&s.recv_full, (uint32_t)((p.CS - 1) * kPart * 4));
            for (int pr = 0; pr < p.CS; ++pr)
                if (pr != rank) mbar_arrive_remote(map_to_rank(smem_u32(&s.peer_free), (uint32_t)pr));
        }
        float2 w[TAPS], gacc[TAPS];
#pragma unroll
        for (int t = 0; t < TAPS; ++t) {
            w[t] = make_float2(__ldg(p.W0 + ((size_t)h * D + 2 * lane) * TAPS + t),
                               __ldg(p.W0 + ((size_t)h * D + 2 * lane + 1) * TAPS + t));
            gacc[t] = make_float2(0.f, 0.f);
        }
        // ---- phase 1
        for (int b = b_lo; b < b_hi; ++b) {
            const Band bd = decode_band(g, b);
            const bool okb = mbar_wait(&s.full[st], ph, ab);
            __syncwarp();
            const uint8_t* sp = stages + (size_t)st * g.stage_bytes;
            const int y = bd.y0 + orow;
            const int cols = bd.xe - bd.xs, segw = (cols + WPR - 1) / WPR;
            const int xa = oseg * segw, xb = min(cols, xa + segw);      // strip-relative output columns
            if (okb && y < g.H && xa < xb) {
                const uint8_t* vrow = sp + g.k_bytes + (size_t)orow * g.XT * E::kTokenBytes;
                float2 win[3][3];
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    win[a][0] = staged<T>(sp, g.k_pitch, orow + a, xa, lane);
                    win[a][1] = staged<T>(sp, g.k_pitch, orow + a, xa + 1, lane);
                }
                for (int x = xa; x < xb; ++x) {
#pragma unroll
                    for (int a = 0; a < 3; ++a) win[a][2] = staged<T>(sp, g.k_pitch, orow + a, x + 2, lane);
                    const float2 v =
                        E::unpack(reinterpret_cast<const typename E::Raw*>(vrow + (size_t)x * E::kTokenBytes)[lane]);
                    float2 r = make_float2(-v.x, -v.y);
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int c = 0; c < 3; ++c) r = ffma2(w[a * 3 + c], win[a][c], r);
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int c = 0; c < 3; ++c) gacc[a * 3 + c] = ffma2(r, win[a][c], gacc[a * 3 + c]);
#pragma unroll
                    for (int a = 0; a < 3; ++a) { win[a][0] = win[a][1]; win[a][1] = win[a][2]; }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty[st]);
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
        // ---- the CTA's partial, in a fixed order over the warps
        bool ok = true;
        if (multi) ok = mbar_wait_cluster(&s.peer_free, k & 1u, ab);  // my last pushes have landed
#pragma unroll
        for (int t = 0; t < TAPS; ++t) *reinterpret_cast<float2*>(&s.red[warp][t * D + 2 * lane]) = gacc[t];
        if (named_bar_or(1, CW * 32, !ok)) { failed = true; break; }
        for (int e = tid; e < kPart; e += CW * 32) {
            float acc = 0.f;
#pragma unroll
            for (int ww = 0; ww < CW; ++ww) acc += s.red[ww][e];
            s.mine[e] = acc;
        }
        // ---- exchange with the cluster, then W1 = W0 - eta (2/N) sum_r partial_r (rank order)
        if (multi) {
            fence_proxy_async_smem();                                // `mine` is read by the bulk-copy engine
            named_bar_sync(1, CW * 32);
            if (tid == 0)
                for (int pr = 0; pr < p.CS; ++pr) {
                    if (pr == rank) continue;
                    const int slot = (rank < pr) ? rank : rank - 1;
                    bulk_s2cluster(map_to_rank(smem_u32(s.recv[slot]), (uint32_t)pr), s.mine, kPart * 4,
                                   map_to_rank(smem_u32(&s.recv_full), (uint32_t)pr));
                }
            ok = mbar_wait_cluster(&s.recv_full, k & 1u, ab);
        }
        if (named_bar_or(1, CW * 32, !ok)) { failed = true; break; }
        for (int e = tid; e < kPart; e += CW * 32) {
            float acc = 0.f;
            for (int pr = 0; pr < p.CS; ++pr) acc += (pr == rank) ? s.mine[e] : s.recv[(pr < rank) ? pr : pr - 1][e];
            const int t = e / D, ch = e % D;                        // tap-major index
            const float w1 = __ldg(p.W0 + ((size_t)h * D + ch) * TAPS + t) - p.eta_scale * acc;
            s.w1[e] = w1;
            if (p.W1_out && rank == 0) p.W1_out[((size_t)u * D + ch) * TAPS + t] = w1;
        }
        named_bar_sync(1, CW * 32);
#pragma unroll
        for (int t = 0; t < TAPS; ++t) w[t] = *reinterpret_cast<const float2*>(&s.w1[t * D + 2 * lane]);
        // ---- phase 2
        const long long off = (long long)bi * g.bs + (long long)h * g.hs;
        for (int b = b_lo; b < b_hi; ++b) {
            const Band bd = decode_band(g, b);
            if (!mbar_wait(&s.full[st], ph, ab)) { failed = true; break; }   // no CTA barrier follows
            __syncwarp();
            const uint8_t* sp = stages + (size_t)st * g.stage_bytes;
            const int y = bd.y0 + orow;
            const int cols = bd.xe - bd.xs, segw = (cols + WPR - 1) / WPR;
            const int xa = oseg * segw, xb = min(cols, xa + segw);
            if (y < g.H && xa < xb) {
                T* zrow = Z + off + ((long long)y * g.W + bd.xs) * D + 2 * lane;
                float2 win[3][3];
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    win[a][0] = staged<T>(sp, g.k_pitch, orow + a, xa, lane);
                    win[a][1] = staged<T>(sp, g.k_pitch, orow + a, xa + 1, lane);
                }
                for (int x = xa; x < xb; ++x) {
#pragma unroll
                    for (int a = 0; a < 3; ++a) win[a][2] = staged<T>(sp, g.k_pitch, orow + a, x + 2, lane);
                    float2 z = make_float2(0.f, 0.f);
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int c = 0; c < 3; ++c) z = ffma2(w[a * 3 + c], win[a][c], z);
                    E::store(zrow + (long long)x * D, z);
#pragma unroll
                    for (int a = 0; a < 3; ++a) { win[a][0] = win[a][1]; win[a][1] = win[a][2]; }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty[st]);
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
    }
    // Final handshake: once every peer has finished its last unit, all of this CTA's pushes have
    // landed and nobody will push into it again; only then may it exit.
    if (multi && !failed) {
        named_bar_sync(1, CW * 32);
        if (tid == 0)
            for (int pr = 0; pr < p.CS; ++pr)
                if (pr != rank) mbar_arrive_remote(map_to_rank(smem_u32(&s.peer_free), (uint32_t)pr));
        mbar_wait_cluster(&s.peer_free, k & 1u, ab);
    }
}

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
template <typename T>
static Geom make_geom(const Call& c) {
    constexpr int TB = Elem<T>::kTokenBytes;
    Geom g;
    g.heads = c.heads;
    g.H = c.H;
    g.W = c.W;
    g.Sx = (c.W + Elem<T>::kXtMax - 1) / Elem<T>::kXtMax;
    g.XT = (c.W + g.Sx - 1) / g.Sx;
    g.Hb = (c.H + R - 1) / R;
    g.bands_per_unit = g.Sx * g.Hb;
    g.bs = c.bs;
    g.hs = c.hs;
    g.k_pitch = g.XT + 2;
    g.k_bytes = (uint32_t)((R + 2) * g.k_pitch * TB);
    g.v_bytes = (uint32_t)(R * g.XT * TB);
    g.stage_bytes = (g.k_bytes + g.v_bytes + 127u) & ~127u;
    return g;
}

template <typename T>
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
        cfg.gridDim = dim3(cs * 16);
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cs; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, (void*)dw_cluster<T>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][cs] = n;
    }
    return cache[dev][cs];
}

template <typename T>
static ttt_status launch(const Call& c) {
    const long long units = (long long)c.batch * c.heads;
    const Geom g = make_geom<T>(c);
    const size_t smem = 128 + (size_t)STAGES * g.stage_bytes + sizeof(SmemTail);
    if (smem > 227 * 1024) return TTT_ERR_UNSUPPORTED;
    cudaFuncSetAttribute(dw_cluster<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(dw_cluster<T>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    // CTAs per cluster: spread each unit over up to 16 SMs while every cluster stays co-resident.
    int cs = (int)std::max<long long>(1, std::min<long long>(kMaxCluster, c.num_sms / std::max<long long>(1, units)));
    cs = std::min(cs, g.bands_per_unit);
    while (cs > 1 && max_active_clusters<T>(cs, smem) < (int)std::min<long long>(units, c.num_sms / cs)) --cs;
    const int ncl = (int)std::min<long long>(units, cs == 1 ? c.num_sms : c.num_sms / cs);

    CUtensorMap tmK, tmV, tmQ;
    if (!make_tmap_grid(&tmK, c.K, c, g.XT + 2, R + 2) || !make_tmap_grid(&tmV, c.V, c, g.XT, R) ||
        !make_tmap_grid(&tmQ, c.Q, c, g.XT + 2, R + 2))
        return TTT_ERR_INVALID_ARG;
    Params p;
    p.g = g;
    p.U = (int)units;
    p.CS = cs;
    p.eta_scale = c.eta * (2.0f / (float)c.N);
    p.W0 = c.W0;
    p.W1_out = c.W1_out;
    p.err = reinterpret_cast<uint32_t*>(c.ws);
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
    return check_launch(cudaLaunchKernelEx(&cfg, dw_cluster<T>, tmK, tmV, tmQ, static_cast<T*>(c.Z), p));
}

}  // namespace dw

// The cluster kernel keeps every intermediate on chip: the workspace is the error word only.
size_t dwconv_ws_bytes(const ttt_shape&) { return kWsHeader; }

ttt_status launch_dwconv(const Call& c) {
    if (c.dtype == TTT_BF16) return dw::launch<__nv_bfloat16>(c);
    return dw::launch<float>(c);
}

}  // namespace ttt
