// dwconv.cu -- 3x3 depthwise-convolution inner model of the TTT layer over the H x W token grid
// (press article "CVPR 2026 Oral | 清華+阿里發布ViT3", Observation 6 and Fig. 5 part 3; ViT^3 keeps
// one such head).  One full-batch step of the L2 loss, then the readout:
//     r[c,y,x] = sum_{a,b} W0[c][a][b] K[c,y+a-1,x+b-1] - V[c,y,x]           (zero padding)
//     g[c][a][b] = (2/N) sum_{y,x} r[c,y,x] K[c,y+a-1,x+b-1],   W1 = W0 - eta g
//     Z[c,y,x] = sum_{a,b} W1[c][a][b] Q[c,y+a-1,x+b-1]
//
// Not a contraction worth a tensor core (about 7 flop per byte): packed fp32x2 FMA, HBM bound.
//
// Work is cut into bands: one unit, one strip of at most XT_MAX columns, R consecutive output rows.
// A band needs R+2 rows of K (or Q) with a one-column halo and R rows of V.  One producer lane moves
// each of those row pieces with a 1-D bulk copy (cp.async.bulk) into a shared-memory stage; the
// 16 compute warps then work from shared memory: warp w owns output row w / 8 of the band and one
// eighth of its columns, lane l owns feature channels 2l and 2l+1, and a 3 x 3 register window slides
// along the columns.  Bands are dealt to the CTAs as contiguous ranges of the flattened
// (unit, strip, band) index space.
//
// Phase 1 (dw_p1): per unit, the warps' 64 x 9 gradients are reduced in a fixed order into one
//   partial slot per (CTA, unit); the last CTA to finish a unit (atomic arrival count, no waiting)
//   sums the unit's slots in CTA order and writes W1.  Deterministic.
// Phase 2 (dw_p2): same staging for Q, reads W1 once the programmatic-launch dependency on phase 1
//   has resolved, writes Z in the input dtype straight from registers (128 coalesced bytes per
//   token and warp).
#include <algorithm>

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
constexpr int kPartialFloats = D * TAPS;    // 576
constexpr int kMaxGrid = 160;
constexpr int kMaxStages = 3;
constexpr size_t kSmemBudget = 220 * 1024;

// fp32x2 helpers: (x, y) = channels 2l and 2l+1 of a lane.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(c.x), "+f"(c.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return c;
}

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {                 // two bf16 channels in one 32-bit word
    using Raw = uint32_t;
    static constexpr int kTokenBytes = D * 2;
    static constexpr int kXtMax = 120;
    static __device__ __forceinline__ Raw zero() { return 0u; }
    static __device__ __forceinline__ float2 unpack(Raw w) { return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w)); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float2 v) {
        *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v.x, v.y);
    }
};
template <>
struct Elem<float> {
    using Raw = float2;
    static constexpr int kTokenBytes = D * 4;
    static constexpr int kXtMax = 56;
    static __device__ __forceinline__ Raw zero() { return make_float2(0.f, 0.f); }
    static __device__ __forceinline__ float2 unpack(Raw w) { return w; }
    static __device__ __forceinline__ void store(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
};

struct Geom {
    int heads, H, W;
    int Sx, XT, Hb;                  // strips, strip width, bands per strip
    int bands_per_unit;              // Sx * Hb
    long long bs, hs;                // element strides of Q/K/V/Z
    int stages;
    int k_pitch;                     // tokens per K row in smem (XT + 2)
    uint32_t stage_bytes, k_bytes;   // bytes per stage, bytes of its K rows
    __host__ __device__ long long unit_off(int u) const {
        return (long long)(u / heads) * bs + (long long)(u % heads) * hs;
    }
};

struct Band {
    int u, s, y0, xs, xe;            // unit, strip, first output row, output columns [xs, xe)
};

__device__ __forceinline__ Band decode_band(const Geom& g, long long b) {
    Band r;
    r.u = (int)(b / g.bands_per_unit);
    const int rem = (int)(b % g.bands_per_unit);
    r.s = rem / g.Hb;
    r.y0 = (rem % g.Hb) * R;
    r.xs = r.s * g.XT;
    r.xe = min(g.W, r.xs + g.XT);
    return r;
}

struct Partition {
    long long T;
    int G;
    __host__ __device__ long long start(int c) const { return (long long)c * T / G; }
    __host__ __device__ int cta_of(long long t) const { return (int)(((t + 1) * G - 1) / T); }
};

struct P1Params {
    Geom g;
    Partition part;
    float eta_scale;             // eta * 2 / N
    const float* W0;             // [heads][64][9]
    float* W1;                   // workspace [units][9][64] (tap-major)
    float* W1_out;               // nullable [units][64][9]
    float* partials;             // workspace [(kMaxGrid + units)][576]
    unsigned* counters;          // workspace [units]
    uint32_t* err;
};

struct P2Params {
    Geom g;
    Partition part;
    const float* W1;             // workspace [units][9][64]
    uint32_t* err;
};

__device__ __forceinline__ uint8_t* align128(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 127) & ~uintptr_t(127));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Producer: stages the K (or Q) rows y0-1 .. y0+R with their column halo and, in phase 1, the V rows.
template <typename T, bool WITH_V>
__device__ __forceinline__ void stage_band(const Geom& g, const Band& bd, const T* X, const T* V, uint8_t* stage,
                                           uint64_t* full) {
    constexpr int TB = Elem<T>::kTokenBytes;
    const long long off = g.unit_off(bd.u);
    const int lc0 = max(0, bd.xs - 1), lc1 = min(g.W, bd.xe + 1);
    const int yk0 = max(0, bd.y0 - 1), yk1 = min(g.H, bd.y0 + R + 1);
    const int yv1 = min(g.H, bd.y0 + R);
    uint32_t bytes = (uint32_t)((yk1 - yk0) * (lc1 - lc0) * TB);
    if (WITH_V) bytes += (uint32_t)((yv1 - bd.y0) * (bd.xe - bd.xs) * TB);
    mbar_arrive_expect_tx(full, bytes);
    for (int yy = yk0; yy < yk1; ++yy) {
        uint8_t* dst = stage + ((size_t)(yy - (bd.y0 - 1)) * g.k_pitch + (lc0 - (bd.xs - 1))) * TB;
        bulk_g2s(dst, X + off + ((long long)yy * g.W + lc0) * D, (uint32_t)((lc1 - lc0) * TB), full);
    }
    if (WITH_V) {
        for (int y = bd.y0; y < yv1; ++y) {
            uint8_t* dst = stage + g.k_bytes + (size_t)(y - bd.y0) * (bd.xe - bd.xs) * TB;
            bulk_g2s(dst, V + off + ((long long)y * g.W + bd.xs) * D, (uint32_t)((bd.xe - bd.xs) * TB), full);
        }
    }
}

// The window value at grid row yy, column xx (0 outside the grid) from a staged band.
template <typename T>
__device__ __forceinline__ typename Elem<T>::Raw kval(const Geom& g, const Band& bd, const uint8_t* stage, int yy,
                                                      int xx, int lane) {
    using Raw = typename Elem<T>::Raw;
    if (yy < 0 || yy >= g.H || xx < 0 || xx >= g.W) return Elem<T>::zero();
    const Raw* p = reinterpret_cast<const Raw*>(
        stage + ((size_t)(yy - (bd.y0 - 1)) * g.k_pitch + (xx - (bd.xs - 1))) * Elem<T>::kTokenBytes);
    return p[lane];
}

// ------------------------------------------------------------------------------------------------
// Phase 1
// ------------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(THREADS, 1)
dw_p1(const T* __restrict__ K, const T* __restrict__ V, const P1Params p) {
    using E = Elem<T>;
    using Raw = typename E::Raw;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align128(smem_raw);
    const Geom& g = p.g;
    uint8_t* stages = base;
    float* red = reinterpret_cast<float*>(base + (size_t)g.stages * g.stage_bytes);     // [CW][576]
    uint64_t* full = reinterpret_cast<uint64_t*>(red + CW * kPartialFloats);
    uint64_t* empty = full + kMaxStages;
    volatile int* flags = reinterpret_cast<volatile int*>(empty + kMaxStages);          // [0] abort, [1] last
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const long long b_begin = p.part.start(c), b_end = p.part.start(c + 1);
    const Abort ab{flags, p.err};

    if (threadIdx.x == 0) {
        flags[0] = 0;
        for (int i = 0; i < g.stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], CW); }
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == CW) {                                                // producer warp
        if (lane == 0) {
            int st = 0; uint32_t ph = 0;
            for (long long b = b_begin; b < b_end; ++b) {
                if (!mbar_wait(&empty[st], ph ^ 1u, ab)) break;
                stage_band<T, true>(g, decode_band(g, b), K, V, stages + (size_t)st * g.stage_bytes, &full[st]);
                if (++st == g.stages) { st = 0; ph ^= 1u; }
            }
        }
        return;
    }

    // compute warps
    const int orow = warp / WPR, oseg = warp % WPR;
    const int tid = threadIdx.x;                                     // 0 .. CW*32-1
    float2 w[TAPS], gacc[TAPS];
    int cur_u = -1;
    int st = 0; uint32_t ph = 0;
    for (long long b = b_begin; b <= b_end; ++b) {
        const Band bd = (b < b_end) ? decode_band(g, b) : Band{-1, 0, 0, 0, 0};
        if (bd.u != cur_u) {
            if (cur_u >= 0) {                                        // flush the finished unit
#pragma unroll
                for (int k = 0; k < TAPS; ++k) {
                    red[warp * kPartialFloats + k * D + 2 * lane] = gacc[k].x;
                    red[warp * kPartialFloats + k * D + 2 * lane + 1] = gacc[k].y;
                }
                named_bar_sync(1, CW * 32);
                float* slot = p.partials + (size_t)(c + cur_u) * kPartialFloats;
                for (int e = tid; e < kPartialFloats; e += CW * 32) {
                    float s = 0.f;
#pragma unroll
                    for (int ww = 0; ww < CW; ++ww) s += red[ww * kPartialFloats + e];
                    slot[e] = s;
                }
                __threadfence();
                named_bar_sync(1, CW * 32);
                const long long per = g.bands_per_unit;
                const int cf = p.part.cta_of((long long)cur_u * per), cl = p.part.cta_of((long long)(cur_u + 1) * per - 1);
                if (tid == 0) {
                    const unsigned old = atomicAdd(p.counters + cur_u, 1u);
                    flags[1] = (old + 1u == (unsigned)(cl - cf + 1)) ? 1 : 0;
                }
                named_bar_sync(1, CW * 32);
                if (flags[1]) {                                      // last CTA of the unit: merge
                    __threadfence();
                    const int h = cur_u % g.heads;
                    for (int e = tid; e < kPartialFloats; e += CW * 32) {
                        float s = 0.f;
                        for (int cc = cf; cc <= cl; ++cc) s += __ldcg(p.partials + (size_t)(cc + cur_u) * kPartialFloats + e);
                        const int k = e / D, ch = e % D;                 // e = tap-major index
                        const float w1 = __ldg(p.W0 + ((size_t)h * D + ch) * TAPS + k) - p.eta_scale * s;
                        p.W1[(size_t)cur_u * kPartialFloats + e] = w1;
                        if (p.W1_out) p.W1_out[((size_t)cur_u * D + ch) * TAPS + k] = w1;
                    }
                    if (tid == 0) p.counters[cur_u] = 0u;
                }
                named_bar_sync(1, CW * 32);
            }
            if (b == b_end) break;
            cur_u = bd.u;
            const int h = cur_u % g.heads;
#pragma unroll
            for (int k = 0; k < TAPS; ++k) {
                w[k] = make_float2(__ldg(p.W0 + ((size_t)h * D + 2 * lane) * TAPS + k),
                                   __ldg(p.W0 + ((size_t)h * D + 2 * lane + 1) * TAPS + k));
                gacc[k] = make_float2(0.f, 0.f);
            }
        }
        // A failed (timed-out) wait skips the band but keeps this warp in step with the CTA's
        // barriers; the error word records the failure.
        const bool ok = mbar_wait(&full[st], ph, ab);
        __syncwarp();
        const uint8_t* stage = stages + (size_t)st * g.stage_bytes;
        const int y = bd.y0 + orow;
        if (ok && y < g.H) {
            const int cols = bd.xe - bd.xs;
            const int segw = (cols + WPR - 1) / WPR;
            const int xa = bd.xs + oseg * segw, xb = min(bd.xe, xa + segw);
            if (xa < xb) {
                const Raw* vrow = reinterpret_cast<const Raw*>(stage + g.k_bytes + (size_t)orow * cols * E::kTokenBytes);
                float2 win[3][3];
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    win[a][0] = E::unpack(kval<T>(g, bd, stage, y + a - 1, xa - 1, lane));
                    win[a][1] = E::unpack(kval<T>(g, bd, stage, y + a - 1, xa, lane));
                }
                for (int x = xa; x < xb; ++x) {
#pragma unroll
                    for (int a = 0; a < 3; ++a) win[a][2] = E::unpack(kval<T>(g, bd, stage, y + a - 1, x + 1, lane));
                    const float2 v = E::unpack(reinterpret_cast<const Raw*>(
                        reinterpret_cast<const uint8_t*>(vrow) + (size_t)(x - bd.xs) * E::kTokenBytes)[lane]);
                    float2 r = make_float2(-v.x, -v.y);
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int bb = 0; bb < 3; ++bb) r = fma2(w[a * 3 + bb], win[a][bb], r);
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int bb = 0; bb < 3; ++bb) gacc[a * 3 + bb] = fma2(r, win[a][bb], gacc[a * 3 + bb]);
#pragma unroll
                    for (int a = 0; a < 3; ++a) { win[a][0] = win[a][1]; win[a][1] = win[a][2]; }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (++st == g.stages) { st = 0; ph ^= 1u; }
    }
}

// ------------------------------------------------------------------------------------------------
// Phase 2
// ------------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(THREADS, 1)
dw_p2(const T* __restrict__ Q, T* __restrict__ Z, const P2Params p) {
    using E = Elem<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align128(smem_raw);
    const Geom& g = p.g;
    uint8_t* stages = base;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + (size_t)g.stages * g.stage_bytes);
    uint64_t* empty = full + kMaxStages;
    volatile int* flags = reinterpret_cast<volatile int*>(empty + kMaxStages);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const long long b_begin = p.part.start(c), b_end = p.part.start(c + 1);
    const Abort ab{flags, p.err};

    if (threadIdx.x == 0) {
        flags[0] = 0;
        for (int i = 0; i < g.stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], CW); }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == CW) {                                                // producer: Q does not depend on phase 1
        if (lane == 0) {
            int st = 0; uint32_t ph = 0;
            for (long long b = b_begin; b < b_end; ++b) {
                if (!mbar_wait(&empty[st], ph ^ 1u, ab)) break;
                stage_band<T, false>(g, decode_band(g, b), Q, nullptr, stages + (size_t)st * g.stage_bytes, &full[st]);
                if (++st == g.stages) { st = 0; ph ^= 1u; }
            }
        }
        return;
    }

    pdl_wait_primary();                                              // W1 comes from phase 1
    const int orow = warp / WPR, oseg = warp % WPR;
    float2 w[TAPS];
    int cur_u = -1;
    int st = 0; uint32_t ph = 0;
    for (long long b = b_begin; b < b_end; ++b) {
        const Band bd = decode_band(g, b);
        if (bd.u != cur_u) {
            cur_u = bd.u;
            const float2* W1u = reinterpret_cast<const float2*>(p.W1 + (size_t)cur_u * kPartialFloats);
#pragma unroll
            for (int k = 0; k < TAPS; ++k) w[k] = __ldcg(W1u + k * (D / 2) + lane);
        }
        if (!mbar_wait(&full[st], ph, ab)) break;                  // no CTA barrier follows in phase 2
        __syncwarp();
        const uint8_t* stage = stages + (size_t)st * g.stage_bytes;
        const int y = bd.y0 + orow;
        if (y < g.H) {
            const int cols = bd.xe - bd.xs;
            const int segw = (cols + WPR - 1) / WPR;
            const int xa = bd.xs + oseg * segw, xb = min(bd.xe, xa + segw);
            if (xa < xb) {
                T* zrow = Z + g.unit_off(bd.u) + (long long)y * g.W * D + 2 * lane;
                float2 win[3][3];
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    win[a][0] = E::unpack(kval<T>(g, bd, stage, y + a - 1, xa - 1, lane));
                    win[a][1] = E::unpack(kval<T>(g, bd, stage, y + a - 1, xa, lane));
                }
                for (int x = xa; x < xb; ++x) {
#pragma unroll
                    for (int a = 0; a < 3; ++a) win[a][2] = E::unpack(kval<T>(g, bd, stage, y + a - 1, x + 1, lane));
                    float2 z = make_float2(0.f, 0.f);
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int bb = 0; bb < 3; ++bb) z = fma2(w[a * 3 + bb], win[a][bb], z);
                    E::store(zrow + (long long)x * D, z);
#pragma unroll
                    for (int a = 0; a < 3; ++a) { win[a][0] = win[a][1]; win[a][1] = win[a][2]; }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (++st == g.stages) { st = 0; ph ^= 1u; }
    }
}

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
struct WsLayout {
    size_t counters, w1, partials, total;
};

static WsLayout ws_layout(long long units) {
    WsLayout L;
    L.counters = kWsHeader;
    L.w1 = align_up(L.counters + (size_t)units * sizeof(unsigned), 256);
    L.partials = align_up(L.w1 + (size_t)units * kPartialFloats * sizeof(float), 256);
    L.total = L.partials + (size_t)(kMaxGrid + units) * kPartialFloats * sizeof(float);
    return L;
}

template <typename T>
static Geom make_geom(const Call& c, bool with_v) {
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
    g.stage_bytes = g.k_bytes + (with_v ? (uint32_t)(R * g.XT * TB) : 0u);
    g.stage_bytes = (g.stage_bytes + 127u) & ~127u;
    const size_t fixed = (with_v ? CW * kPartialFloats * sizeof(float) : 0) + 2 * kMaxStages * 8 + 64 + 128;
    g.stages = (int)std::min<size_t>(kMaxStages, (kSmemBudget - fixed) / g.stage_bytes);
    return g;
}

template <typename T>
static size_t smem_bytes(const Geom& g, bool with_v) {
    return 128 + (size_t)g.stages * g.stage_bytes + (with_v ? CW * kPartialFloats * sizeof(float) : 0) +
           2 * kMaxStages * 8 + 64;
}

template <typename T>
static ttt_status launch(const Call& c) {
    const long long units = (long long)c.batch * c.heads;
    const WsLayout L = ws_layout(units);
    const Geom g1 = make_geom<T>(c, true), g2 = make_geom<T>(c, false);
    if (g1.stages < 2 || g2.stages < 2) return TTT_ERR_UNSUPPORTED;
    const long long bands = units * g1.bands_per_unit;
    const int G = (int)std::min<long long>(std::min(c.num_sms, kMaxGrid), bands);

    P1Params p1;
    p1.g = g1;
    p1.part = Partition{bands, G};
    p1.eta_scale = c.eta * (2.0f / (float)c.N);
    p1.W0 = c.W0;
    p1.W1 = reinterpret_cast<float*>(c.ws + L.w1);
    p1.W1_out = c.W1_out;
    p1.partials = reinterpret_cast<float*>(c.ws + L.partials);
    p1.counters = reinterpret_cast<unsigned*>(c.ws + L.counters);
    p1.err = reinterpret_cast<uint32_t*>(c.ws);
    const size_t sm1 = smem_bytes<T>(g1, true), sm2 = smem_bytes<T>(g2, false);
    cudaFuncSetAttribute(dw_p1<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    cudaFuncSetAttribute(dw_p2<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    dw_p1<T><<<G, THREADS, sm1, c.stream>>>(static_cast<const T*>(c.K), static_cast<const T*>(c.V), p1);
    ttt_status st = check_launch(cudaGetLastError());
    if (st != TTT_OK) return st;

    P2Params p2;
    p2.g = g2;
    p2.part = Partition{bands, G};
    p2.W1 = p1.W1;
    p2.err = p1.err;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = sm2;
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return check_launch(cudaLaunchKernelEx(&cfg, dw_p2<T>, static_cast<const T*>(c.Q), static_cast<T*>(c.Z), p2));
}

}  // namespace dw

size_t dwconv_ws_bytes(const ttt_shape& s) { return dw::ws_layout((long long)s.batch * s.heads).total; }

ttt_status launch_dwconv(const Call& c) {
    if (c.dtype == TTT_BF16) return dw::launch<__nv_bfloat16>(c);
    return dw::launch<float>(c);
}

}  // namespace ttt
