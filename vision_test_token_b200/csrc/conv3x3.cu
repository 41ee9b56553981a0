// conv3x3.cu -- full 3x3 convolution inner model of the TTT layer over the H x W token grid (press
// article "CVPR 2026 Oral | 清華+阿里發布ViT3", Observation 6 and Fig. 5 part 3: the inner model
// implemented as a 3x3 convolution, beside the depthwise one).  Every output channel reads every
// input channel:
//     f(X;W)[c,y,x] = sum_{c'} sum_{a,b} W[c][c'][a][b] X[c', y+a-1, x+b-1]      (zero padding)
//     r = f(K;W0) - V,   g[c][c'][a][b] = (2/N) sum_{y,x} r[c,y,x] K[c', y+a-1, x+b-1],
//     W1 = W0 - eta g,   Z = f(Q;W1).
// With the 576 features of a position's 3 x 3 neighbourhood (im2col, K~ = [K_0 | ... | K_8], K_t the
// grid shifted by tap t), f is the linear map W~ (64 x 576) and the step is three dense contractions,
// which go to the tensor cores (tcgen05, bf16 operands, fp32 accumulation in tensor memory):
//     R = K~ W0~^T - V          (positions x 64,   K = 576: nine taps of 64 channels)
//     G = sum_pos K~^T R        (576 x 64: the gradient, transposed)
//     Z = Q~ W1~^T              (positions x 64)
// The tap shifts are never materialised.  Tiles are 8 rows x 16 columns of the grid (128 positions,
// the MMA's M); a tile's K (or Q) comes as three TMA boxes of its rows -1 .. 8, one per x shift, and
// tap (a, b) is the 128 rows of box b that start at row 16a (tap_box below).  The boxes' out-of-bounds
// zero fill is the zero padding.
//
// Four kernels on one stream, each a programmatic dependent of the one before:
//   conv3_wprep   W0 rounded to bf16 and laid out as nine swizzled tap operand images per head (row
//                 c, K = c'), once per call, so that each gradient CTA loads its head's weights with
//                 one bulk copy instead of gathering them from the [c][c'][a][b] layout.
//   conv3_grad    (a fixed number of CTAs per unit, each a contiguous share of one unit's tiles;
//                 per tile) the three K halo boxes by TMA, two tiles' halos resident; R = K~ W0~^T
//                 accumulates over the taps (A = the tap's rows of a halo box, K-major; B = W0 tap
//                 image, rows c, K = c'); the epilogue reads V straight from global memory, forms
//                 r = R - V, zeroes positions outside the grid and splits r into bf16 hi + lo (about
//                 16 significant bits); G^T += [K_a | K_b]^T (r_hi + r_lo) accumulates in five
//                 tap-pair accumulators (A MN-major, M = 128 = two taps' channels; B = r, MN-major).
//                 The MMAs run R(n+1) before G(n).  At the end of its tiles the CTA writes the
//                 accumulators to its workspace slot as G[tap][c][c'], so that the 32 lanes of a
//                 warp (32 consecutive c') store one 128-byte line per instruction.
//   conv3_merge   per (unit, tap): the unit's slots summed in CTA order (a fixed order: bitwise
//                 reproducible for a given grid), W1 = W0 - eta (2/N) g in fp32 (W1_out), and W1
//                 rounded once to bf16 as the tap's operand image for the readout.
//   conv3_readout (per CTA, a contiguous range of tiles) Z = sum_t Q_t W1_t^T over the tile's three
//                 Q halo boxes, drained to bf16 and stored with TMA (the store clips positions
//                 outside the grid).
// The weights are read in bf16 for R (their rounding changes r by about 2^-9 of |f(K;W0)|) and r is
// carried as hi + lo, so the update keeps close to fp32 accuracy relative to the gradient's terms.
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace c3 {

constexpr int D = 64;
constexpr int TAPS = 9;
constexpr int TR = 8, TC = 16;              // a tile: 8 grid rows x 16 grid columns
constexpr int TILE = TR * TC;               // 128 positions (the MMA's M)
constexpr int BOX = TILE * D * 2;           // one tap box: 16 KB (128 bytes per position)
constexpr int HALO = (TR + 2) * TC * 128;   // a tile's rows -1 .. 8 at one x shift: 20 KB
constexpr int NPAIR = 5;                    // gradient accumulators: two taps each (the last one tap)
constexpr int kWImg = D * D * 2;            // one tap's weights as a bf16 operand image: 8 KB
constexpr int kThreads = 192;
constexpr int kMaxGrid = 160;               // slots of the workspace: (kMaxGrid + units)
constexpr int kSlotFloats = TAPS * D * D;   // one gradient partial, G [tap][c][c']
constexpr uint32_t kIdescRow = idesc_bf16_f32(128, 64, false, false);  // D[pos][c] = sum_k A[pos][k] B[c][k]
constexpr uint32_t kIdescCol = idesc_bf16_f32(128, 64, true, true);    // D[m][c] = sum_pos A[pos][m] B[pos][c]
constexpr uint32_t kColR = 0;               // tensor memory: two R accumulators,
constexpr uint32_t kColG = 128;             //   five tap-pair gradient accumulators (448 columns)

// A tile's operands are three halo buffers: buffer b holds grid rows y0-1 .. y0+8 at columns
// x0+b-1 .. x0+b+14 (a 10 x 16 TMA box, 128-byte swizzled rows of 64 channels).  Tap t = 3a + b
// (shift (a-1, b-1)) is the 128 rows of buffer b starting at row 16a: 1024-byte aligned, so every
// tap is an ordinary operand box and the nine taps cost three loads.
__device__ __forceinline__ uint32_t tap_box(uint32_t halo0, int t9) {
    return halo0 + (uint32_t)((t9 % 3) * HALO + (t9 / 3) * TC * 128);
}
// The gradient's tap pairs: the two taps of pair k are one M = 128 operand whose second half lies
// kPairLbo[k] bytes after the first (the same x shift one grid row further, or the next buffer);
// the last accumulator's second half reads rows nothing uses.
__constant__ int kPairTap[NPAIR][2] = {{0, 3}, {1, 4}, {2, 5}, {6, 7}, {8, 8}};
__constant__ uint32_t kPairLbo[NPAIR] = {TC * 128, TC * 128, TC * 128, (uint32_t)HALO, TC * 128};

struct Geo {
    int heads, H, W;
    int tiles_x, tpu;                        // tiles along x, tiles per unit
    long long T;                             // tiles of the call
    float eta_scale;                         // eta * 2 / N
};

// CTA c of G owns tiles [start(c), start(c + 1)); the CTA that owns tile t.
__host__ __device__ __forceinline__ long long part_start(long long T, int G, int c) { return (long long)c * T / G; }
__host__ __device__ __forceinline__ int part_cta(long long T, int G, long long t) { return (int)(((t + 1) * G - 1) / T); }

// The gradient kernel's tiles: with cpu > 0, cpu CTAs per unit, CTA c taking a contiguous share of
// unit c / cpu's tiles only (no CTA drains two units' gradients); with cpu = 0 (more units than CTAs),
// the contiguous split above.
struct GradPart {
    long long T;
    int G, cpu, tpu;
    __host__ __device__ __forceinline__ long long start(int c) const {
        if (cpu == 0) return part_start(T, G, c);
        const int u = c / cpu, k = c % cpu;
        return (long long)u * tpu + (long long)k * tpu / cpu;
    }
    __host__ __device__ __forceinline__ int first_cta(int u) const {
        return cpu ? u * cpu : part_cta(T, G, (long long)u * tpu);
    }
    __host__ __device__ __forceinline__ int last_cta(int u) const {
        return cpu ? (u + 1) * cpu - 1 : part_cta(T, G, (long long)(u + 1) * tpu - 1);
    }
};

struct TileXY {
    int u, b, h, x0, y0;
};
__device__ __forceinline__ TileXY tile_xy(const Geo& g, long long t) {
    TileXY r;
    r.u = (int)(t / g.tpu);
    const int i = (int)(t % g.tpu);
    r.b = r.u / g.heads;
    r.h = r.u % g.heads;
    r.x0 = (i % g.tiles_x) * TC;
    r.y0 = (i / g.tiles_x) * TR;
    return r;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 16-byte chunk j (channels 8j .. 8j+7) of position row `row` of a 128-byte swizzled operand image.
__device__ __forceinline__ uint32_t sw_off(int row, int j) { return (uint32_t)(row * 128 + ((j ^ (row & 7)) << 4)); }

__device__ __forceinline__ uint4 pack8(const float* v) {
    uint4 pk;
    pk.x = pack_bf16x2(v[0], v[1]); pk.y = pack_bf16x2(v[2], v[3]);
    pk.z = pack_bf16x2(v[4], v[5]); pk.w = pack_bf16x2(v[6], v[7]);
    return pk;
}

// ------------------------------------------------------------------------------------------------
// conv3_grad
// ------------------------------------------------------------------------------------------------
// ------------------------------------------------------------------------------------------------
// conv3_wprep: one CTA per (head, output channel c), one thread per input channel c'
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(D)
conv3_wprep(const float* __restrict__ W0, uint8_t* __restrict__ w0img) {
    const int h = blockIdx.x / D, c = blockIdx.x % D, cp = threadIdx.x;
    pdl_wait_primary();                                      // the previous call's kernels are done with the images
    pdl_launch_dependents();
    const float* w = W0 + (((size_t)h * D + c) * D + cp) * TAPS;
    float v[TAPS];
#pragma unroll
    for (int t9 = 0; t9 < TAPS; ++t9) v[t9] = __ldg(w + t9);
#pragma unroll
    for (int t9 = 0; t9 < TAPS; ++t9)
        *reinterpret_cast<__nv_bfloat16*>(w0img + ((size_t)h * TAPS + t9) * kWImg + sw_off(c, cp / 8) + (cp % 8) * 2) =
            __float2bfloat16_rn(v[t9]);
}

struct GradParams {
    Geo g;
    GradPart part;                           // the CTAs' tile ranges
    const uint8_t* w0img;                    // [heads][9][kWImg], written by conv3_wprep
    const __nv_bfloat16* V;                  // V, read directly by the epilogue
    long long bs, hs;                        // V's element strides of an image and of a head
    float* slots;                            // [(kMaxGrid + U)][9][64][64]: G of a (CTA, unit) part
    uint32_t* err;
    unsigned long long wait_ns;
};

struct GradSmem {
    uint8_t kh[2][3][HALO];                  // two tiles' K halo buffers (x shift b = 0, 1, 2)
    uint8_t w0img[TAPS][kWImg];              // W0 of the part's head, bf16 (row c, K = c')
    uint8_t rhi[BOX], rlo[BOX];              // r = R - V as bf16 hi and lo (position-major)
    uint64_t kfull[2], kempty[2];
    uint64_t dr_full[2], dr_empty[2];        // R accumulators
    uint64_t r_full, r_empty;                // r operands written / read by every MMA of the tile
    uint64_t w_full, w_empty;                // W0 images written / no longer read
    uint64_t g_full, g_empty;                // a part's gradient accumulators complete / drained
    uint64_t drain_bar;
    uint32_t tmem_base;
    int abort_flag;
};

// The CTA's tiles n = 0 .. N-1 go through the tensor pipe in the order R(0), R(1), G(0), R(2), G(1),
// ..., R(N-1), G(N-2), G(N-1): while the epilogue turns R(n) into the residual operand of G(n), the
// MMAs of R(n+1) run.  Tile n's K halo (three boxes) sits in buffer n & 1 from R(n) to G(n).
__host__ __device__ __forceinline__ bool first_of_part(const Geo& g, long long t0, long long t) {
    return t == t0 || t % g.tpu == 0;
}
__host__ __device__ __forceinline__ bool last_of_part(const Geo& g, long long t1, long long t) {
    return t + 1 == t1 || (t + 1) % g.tpu == 0;
}

__device__ __forceinline__ void grad_producer(GradSmem& s, const GradParams& p, const CUtensorMap* tmH,
                                              const Abort& ab) {
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    uint32_t parts = 0, n = 0;
    for (long long t = t0; t < t1; ++t, ++n) {
        const TileXY x = tile_xy(p.g, t);
        if (first_of_part(p.g, t0, t)) {
            // the head's W0 tap images, once the previous part's R MMAs are done with them
            if (t == t0) pdl_wait_primary();                 // conv3_wprep has written the images
            if (!mbar_wait(&s.w_empty, (parts & 1u) ^ 1u, ab)) break;
            fence_proxy_async_global();
            mbar_arrive_expect_tx(&s.w_full, TAPS * kWImg);
            bulk_g2s(s.w0img, p.w0img + (size_t)x.h * TAPS * kWImg, TAPS * kWImg, &s.w_full);
            ++parts;
        }
        const uint32_t kb = n & 1u;
        if (!mbar_wait(&s.kempty[kb], ((n >> 1) & 1u) ^ 1u, ab)) break;
        mbar_arrive_expect_tx(&s.kfull[kb], 3 * HALO);
        for (int b = 0; b < 3; ++b)
            tma_load_5d(s.kh[kb][b], tmH, &s.kfull[kb], 0, x.x0 + b - 1, x.y0 - 1, x.h, x.b);
    }
    // every copy issued has landed before the CTA may exit
    for (uint32_t k = n > 2u ? n - 2u : 0u; k < n; ++k) mbar_drain(&s.kfull[k & 1u], (k >> 1) & 1u, ab.limit);
    if (parts > 0) mbar_drain(&s.w_full, (parts - 1) & 1u, ab.limit);
}

// R(t) = sum_t9 K_t9 W0_t9^T into R accumulator n & 1 (A: the tap's rows of the K halo, K-major;
// B: W0 tap image).
__device__ __forceinline__ bool mma_R(GradSmem& s, const GradParams& p, uint32_t tmem, long long t0, long long t1,
                                      long long t, uint32_t n, uint32_t& wparts, const Abort& ab) {
    if (first_of_part(p.g, t0, t)) {
        if (!mbar_wait(&s.w_full, wparts & 1u, ab)) return false;
        ++wparts;
    }
    const uint32_t dr = n & 1u, kb = n & 1u;
    if (!mbar_wait(&s.dr_empty[dr], ((n >> 1) & 1u) ^ 1u, ab)) return false;
    if (!mbar_wait(&s.kfull[kb], (n >> 1) & 1u, ab)) return false;
    tc_fence_after();
    for (int t9 = 0; t9 < TAPS; ++t9) {
        const uint32_t sa = tap_box(smem_u32(s.kh[kb][0]), t9), sb = smem_u32(s.w0img[t9]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + kColR + dr * 64u, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024),
                        kIdescRow, (t9 | kk) ? 1u : 0u);
    }
    mma_commit(&s.dr_full[dr]);
    if (last_of_part(p.g, t1, t)) mma_commit(&s.w_empty);    // the part's last reads of the W0 images
    return true;
}

// G^T[pair k] += [K_a | K_b]^T (r_hi + r_lo) for tile t, the pair's two taps as one M = 128 operand
// (MN-major: the second tap's rows lie kPairLbo[k] bytes after the first's); frees the K halo.
__device__ __forceinline__ bool mma_G(GradSmem& s, const GradParams& p, uint32_t tmem, long long t0, long long t1,
                                      long long t, uint32_t n, uint32_t& gparts, const Abort& ab) {
    if (!mbar_wait(&s.r_full, n & 1u, ab)) return false;
    const bool first = first_of_part(p.g, t0, t);
    if (first && !mbar_wait(&s.g_empty, (gparts & 1u) ^ 1u, ab)) return false;
    tc_fence_after();
    const uint32_t shi = smem_u32(s.rhi), slo = smem_u32(s.rlo), kh = smem_u32(s.kh[n & 1u][0]);
    for (int k = 0; k < NPAIR; ++k) {
        const uint32_t sa = tap_box(kh, kPairTap[k][0]), lbo = kPairLbo[k];
        const uint32_t dg = tmem + kColG + (uint32_t)k * 64u;
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sa + kk * 2048, lbo, 1024);
            mma_bf16_ss(dg, ad, sdesc_sw128(shi + kk * 2048, BOX, 1024), kIdescCol, (first && kk == 0) ? 0u : 1u);
            mma_bf16_ss(dg, ad, sdesc_sw128(slo + kk * 2048, BOX, 1024), kIdescCol, 1u);
        }
    }
    mma_commit(&s.kempty[n & 1u]);
    mma_commit(&s.r_empty);
    if (last_of_part(p.g, t1, t)) {
        mma_commit(&s.g_full);
        ++gparts;
    }
    return true;
}

__device__ __forceinline__ void grad_mma(GradSmem& s, const GradParams& p, uint32_t tmem, const Abort& ab) {
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    uint32_t wparts = 0, gparts = 0;
    for (long long t = t0; t <= t1; ++t) {
        const uint32_t n = (uint32_t)(t - t0);
        if (t < t1 && !mma_R(s, p, tmem, t0, t1, t, n, wparts, ab)) return;
        if (t > t0 && !mma_G(s, p, tmem, t0, t1, t - 1, n - 1, gparts, ab)) return;
    }
}

__device__ __forceinline__ void grad_epilogue(GradSmem& s, const GradParams& p, uint32_t tmem, const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int r = q * 32 + lane;                              // accumulator row = tile position
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const long long t0 = p.part.start(blockIdx.x), t1 = p.part.start(blockIdx.x + 1);
    uint32_t n = 0, part = 0;
    bool failed = false;
    for (long long t = t0; t < t1 && !failed;) {
        const int u = (int)(t / p.g.tpu);
        const long long pe = (t1 < (long long)(u + 1) * p.g.tpu) ? t1 : (long long)(u + 1) * p.g.tpu;
        bool ok = true;
        for (long long tt = t; tt < pe; ++tt, ++n) {
            const TileXY x = tile_xy(p.g, tt);
            // this position's V row (positions outside the grid contribute nothing), loaded before the
            // wait for R
            const int y = x.y0 + r / TC, xx = x.x0 + r % TC;
            const bool inside = y < p.g.H && xx < p.g.W;
            uint4 vw[8];
            const uint4* vrow = reinterpret_cast<const uint4*>(
                p.V + (size_t)x.b * p.bs + (size_t)x.h * p.hs + ((size_t)y * p.g.W + xx) * D);
#pragma unroll
            for (int j = 0; j < 8; ++j) vw[j] = inside ? __ldg(vrow + j) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t dr = n & 1u;
            ok = mbar_wait(&s.dr_full[dr], (n >> 1) & 1u, ab);
            if (named_bar_or(1, 128, !ok)) { failed = true; break; }
            __syncwarp();
            tc_fence_after();
            float v[4][16];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(tmem + kColR + dr * 64u + (uint32_t)(j * 16) + lane_off, v[j]);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&s.dr_empty[dr]);
            // r = R - V
            float res[64];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t ww[4] = {vw[j].x, vw[j].y, vw[j].z, vw[j].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 8 * j + 2 * e;
                    res[c] = inside ? v[c / 16][c % 16] - bf16lo_to_f32(ww[e]) : 0.f;
                    res[c + 1] = inside ? v[(c + 1) / 16][(c + 1) % 16] - bf16hi_to_f32(ww[e]) : 0.f;
                }
            }
            ok = mbar_wait(&s.r_empty, (n & 1u) ^ 1u, ab);   // the previous tile's MMAs read r
            if (named_bar_or(1, 128, !ok)) { failed = true; break; }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float hi[8], lo[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    hi[e] = __bfloat162float(__float2bfloat16_rn(res[8 * j + e]));
                    lo[e] = res[8 * j + e] - hi[e];
                }
                *reinterpret_cast<uint4*>(s.rhi + sw_off(r, j)) = pack8(hi);
                *reinterpret_cast<uint4*>(s.rlo + sw_off(r, j)) = pack8(lo);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (tid == 0) mbar_arrive(&s.r_full);
        }
        if (failed) break;
        // the part's gradient: accumulator k, row r is channel c' = r % 64 of tap kPairTap[k][r / 64]
        ok = mbar_wait(&s.g_full, part & 1u, ab);
        if (named_bar_or(1, 128, !ok)) break;
        __syncwarp();
        tc_fence_after();
        float* slot = p.slots + (size_t)(blockIdx.x + u) * kSlotFloats;
        for (int k = 0; k < NPAIR; ++k) {
            float g[4][16];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(tmem + kColG + (uint32_t)(k * 64 + j * 16) + lane_off, g[j]);
            tmem_ld_wait();
            if (k < NPAIR - 1 || r < D) {
                const int t9 = kPairTap[k][r / D];
                float* dst = slot + (size_t)t9 * D * D + (r % D);    // G[t9][c][c' = r % 64]
#pragma unroll
                for (int c = 0; c < D; ++c) __stcg(dst + (size_t)c * D, g[c / 16][c % 16]);
            }
        }
        tc_fence_before();
        mbar_arrive(&s.g_empty);
        ++part;
        t = pe;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
conv3_grad(const __grid_constant__ CUtensorMap tmH, const GradParams p) {
    extern __shared__ uint8_t smem_raw[];
    GradSmem& s = *reinterpret_cast<GradSmem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};
    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < 2; ++i) { mbar_init(&s.kfull[i], 1); mbar_init(&s.kempty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s.dr_full[i], 1); mbar_init(&s.dr_empty[i], 128); }
        mbar_init(&s.r_full, 1); mbar_init(&s.r_empty, 1);
        mbar_init(&s.w_full, 1); mbar_init(&s.w_empty, 1);
        mbar_init(&s.g_full, 1); mbar_init(&s.g_empty, 128);
        mbar_init(&s.drain_bar, 1);
        fence_barrier_init();
        prefetch_tmap(&tmH);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();                                 // the merge kernel may be scheduled
    const uint32_t tmem = s.tmem_base;
    if (warp == 0) {
        if (lane == 0) grad_producer(s, p, &tmH, ab);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            grad_mma(s, p, tmem, ab);
            mma_commit(&s.drain_bar);                        // every MMA issued has completed
            mbar_drain(&s.drain_bar, 0u, ab.limit);
        }
        __syncwarp();
    } else {
        grad_epilogue(s, p, tmem, ab);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------------
// conv3_merge: four CTAs per (unit, tap), each a quarter of the tap's 64 x 64 matrix: one float4
// of it per thread, summed over the unit's slots in slot order with 16 loads in flight at a time
// ------------------------------------------------------------------------------------------------
struct MergeParams {
    Geo g;
    GradPart part;                           // the tile ranges of conv3_grad's CTAs
    float eta;
    const float* W0;                         // [heads][64][64][9]
    const float* slots;
    float* W1_out;                           // nullable [units][64][64][9]
    uint8_t* w1img;                          // [units][9][kWImg]
};

__global__ void __launch_bounds__(256)
conv3_merge(const MergeParams p) {
    const int q4 = blockIdx.x & 3, ut = blockIdx.x >> 2;
    const int u = ut / TAPS, t9 = ut % TAPS, h = u % p.g.heads;
    pdl_launch_dependents();
    pdl_wait_primary();                                      // every gradient slot is written
    const int cf = p.part.first_cta(u), cl = p.part.last_cta(u);
    uint8_t* img = p.w1img + ((size_t)u * TAPS + t9) * kWImg;
    const int e4 = q4 * 256 + (int)threadIdx.x;              // float4 of the tap's matrix: elements 4 e4 ..
    const float4* src = reinterpret_cast<const float4*>(p.slots + (size_t)t9 * D * D) + e4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = cf; c0 <= cl; c0 += 16) {
        float4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            v[i] = (c0 + i <= cl) ? __ldcg(src + (size_t)(c0 + i + u) * (kSlotFloats / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (c0 + i <= cl) { acc.x += v[i].x; acc.y += v[i].y; acc.z += v[i].z; acc.w += v[i].w; }
    }
    const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = 4 * e4 + i, c = e / D, cp = e % D;     // slot element G[t9][c][cp]
        const size_t wi = (((size_t)h * D + c) * D + cp) * TAPS + t9;
        const float w1 = __ldg(p.W0 + wi) - p.g.eta_scale * a4[i];
        if (p.W1_out) p.W1_out[(((size_t)u * D + c) * D + cp) * TAPS + t9] = w1;
        *reinterpret_cast<__nv_bfloat16*>(img + sw_off(c, cp / 8) + (cp % 8) * 2) = __float2bfloat16_rn(w1);
    }
}

// ------------------------------------------------------------------------------------------------
// conv3_readout
// ------------------------------------------------------------------------------------------------
struct ReadParams {
    Geo g;
    int G;                                   // CTAs of this kernel
    const uint8_t* w1img;                    // [units][9][kWImg]
    uint32_t* err;
    unsigned long long wait_ns;
};

struct ReadSmem {
    uint8_t qh[2][3][HALO];                  // two tiles' Q halo buffers (x shift b = 0, 1, 2)
    uint8_t w1img[TAPS][kWImg];
    uint8_t zbuf[2][BOX];
    uint64_t qfull[2], qempty[2];
    uint64_t w_full, w_empty;
    uint64_t dz_full[2], dz_empty[2];
    uint64_t drain_bar;
    uint32_t tmem_base;
    int abort_flag;
};

// W1 of unit u (written by the merge kernel): one bulk copy of its nine tap images, once the
// previous part's MMAs are done with the images.
__device__ __forceinline__ bool load_w1(ReadSmem& s, const ReadParams& p, int u, uint32_t& parts, const Abort& ab) {
    if (parts == 0) pdl_wait_primary();
    if (!mbar_wait(&s.w_empty, (parts & 1u) ^ 1u, ab)) return false;
    fence_proxy_async_global();
    mbar_arrive_expect_tx(&s.w_full, TAPS * kWImg);
    bulk_g2s(s.w1img, p.w1img + (size_t)u * TAPS * kWImg, TAPS * kWImg, &s.w_full);
    ++parts;
    return true;
}

__device__ __forceinline__ void read_producer(ReadSmem& s, const ReadParams& p, const CUtensorMap* tmH,
                                              const Abort& ab) {
    const long long t0 = part_start(p.g.T, p.G, blockIdx.x), t1 = part_start(p.g.T, p.G, blockIdx.x + 1);
    uint32_t parts = 0, n = 0;
    int pending = -1;                                        // unit whose W1 images are not requested yet
    bool ok = true;
    for (long long t = t0; t < t1 && ok; ++t, ++n) {
        const TileXY x = tile_xy(p.g, t);
        if (t == t0) {
            pending = x.u;          // the first Q halos (an input) load while the merge kernel still writes W1
        } else if (t % p.g.tpu == 0) {
            if (pending >= 0 && !(ok = load_w1(s, p, pending, parts, ab))) break;
            pending = -1;
            if (!(ok = load_w1(s, p, x.u, parts, ab))) break;
        }
        if (pending >= 0 && n == 2u) {                       // the next buffer is freed by the MMAs
            if (!(ok = load_w1(s, p, pending, parts, ab))) break;
            pending = -1;
        }
        const uint32_t qb = n & 1u;
        if (!(ok = mbar_wait(&s.qempty[qb], ((n >> 1) & 1u) ^ 1u, ab))) break;
        mbar_arrive_expect_tx(&s.qfull[qb], 3 * HALO);
        for (int b = 0; b < 3; ++b)
            tma_load_5d(s.qh[qb][b], tmH, &s.qfull[qb], 0, x.x0 + b - 1, x.y0 - 1, x.h, x.b);
    }
    if (ok && pending >= 0) load_w1(s, p, pending, parts, ab);
    for (uint32_t k = n > 2u ? n - 2u : 0u; k < n; ++k) mbar_drain(&s.qfull[k & 1u], (k >> 1) & 1u, ab.limit);
    if (parts > 0) mbar_drain(&s.w_full, (parts - 1) & 1u, ab.limit);
}

__device__ __forceinline__ void read_mma(ReadSmem& s, const ReadParams& p, uint32_t tmem, const Abort& ab) {
    const long long t0 = part_start(p.g.T, p.G, blockIdx.x), t1 = part_start(p.g.T, p.G, blockIdx.x + 1);
    uint32_t n = 0, parts = 0;
    for (long long t = t0; t < t1; ++t, ++n) {
        if (first_of_part(p.g, t0, t)) {
            if (!mbar_wait(&s.w_full, parts & 1u, ab)) return;
            ++parts;
        }
        const uint32_t dz = n & 1u, qb = n & 1u;
        if (!mbar_wait(&s.dz_empty[dz], ((n >> 1) & 1u) ^ 1u, ab)) return;
        if (!mbar_wait(&s.qfull[qb], (n >> 1) & 1u, ab)) return;
        tc_fence_after();
        for (int t9 = 0; t9 < TAPS; ++t9) {
            const uint32_t sa = tap_box(smem_u32(s.qh[qb][0]), t9), sb = smem_u32(s.w1img[t9]);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16_ss(tmem + dz * 64u, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024),
                            kIdescRow, (t9 | kk) ? 1u : 0u);
        }
        mma_commit(&s.qempty[qb]);
        mma_commit(&s.dz_full[dz]);
        if (last_of_part(p.g, t1, t)) mma_commit(&s.w_empty);
    }
}

__device__ __forceinline__ void read_epilogue(ReadSmem& s, const ReadParams& p, uint32_t tmem, const CUtensorMap* tmZ,
                                              const Abort& ab) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const long long t0 = part_start(p.g.T, p.G, blockIdx.x), t1 = part_start(p.g.T, p.G, blockIdx.x + 1);
    uint32_t n = 0;
    for (long long t = t0; t < t1; ++t, ++n) {
        const TileXY x = tile_xy(p.g, t);
        const uint32_t dz = n & 1u;
        const bool ok = mbar_wait(&s.dz_full[dz], (n >> 1) & 1u, ab);
        if (tid == 0 && n >= 2) bulk_wait_read<1>();          // staging buffer dz is free again
        if (named_bar_or(1, 128, !ok)) break;
        __syncwarp();
        tc_fence_after();
        float v[4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld16(tmem + dz * 64u + (uint32_t)(j * 16) + lane_off, v[j]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s.dz_empty[dz]);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(s.zbuf[dz] + sw_off(r, j)) = pack8(&v[j / 2][(j % 2) * 8]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (tid == 0) {
            asm volatile("cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(tmZ),
                         "r"(smem_u32(s.zbuf[dz])), "r"(0), "r"(x.x0), "r"(x.y0), "r"(x.h), "r"(x.b)
                         : "memory");
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait<0>();
}

__global__ void __launch_bounds__(kThreads, 1)
conv3_readout(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmZ, const ReadParams p) {
    extern __shared__ uint8_t smem_raw[];
    ReadSmem& s = *reinterpret_cast<ReadSmem*>(align1024(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};
    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < 2; ++i) { mbar_init(&s.qfull[i], 1); mbar_init(&s.qempty[i], 1); }
        mbar_init(&s.w_full, 1); mbar_init(&s.w_empty, 1);
        for (int i = 0; i < 2; ++i) { mbar_init(&s.dz_full[i], 1); mbar_init(&s.dz_empty[i], 128); }
        mbar_init(&s.drain_bar, 1);
        fence_barrier_init();
        prefetch_tmap(&tmH); prefetch_tmap(&tmZ);
    }
    if (warp == 1) { tmem_alloc(&s.tmem_base, 128); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;
    if (warp == 0) {
        if (lane == 0) read_producer(s, p, &tmH, ab);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            read_mma(s, p, tmem, ab);
            mma_commit(&s.drain_bar);
            mbar_drain(&s.drain_bar, 0u, ab.limit);
        }
        __syncwarp();
    } else {
        read_epilogue(s, p, tmem, &tmZ, ab);
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
// Host side
// ------------------------------------------------------------------------------------------------
struct WsLayout {
    size_t slots, w1img, w0img, total;
};
static WsLayout ws_layout(long long units, int heads) {
    WsLayout L;
    L.slots = kWsHeader;
    L.w1img = align_up(L.slots + (size_t)(kMaxGrid + units) * kSlotFloats * sizeof(float), 1024);
    L.w0img = L.w1img + (size_t)units * TAPS * kWImg;
    L.total = L.w0img + (size_t)heads * TAPS * kWImg;
    return L;
}

static Geo make_geo(const Call& c) {
    Geo g;
    g.heads = c.heads;
    g.H = c.H;
    g.W = c.W;
    g.tiles_x = (c.W + TC - 1) / TC;
    g.tpu = g.tiles_x * ((c.H + TR - 1) / TR);
    g.T = (long long)c.batch * c.heads * g.tpu;
    g.eta_scale = c.eta * (2.0f / (float)c.N);
    return g;
}

}  // namespace c3

size_t conv3x3_ws_bytes(const ttt_shape& s) { return c3::ws_layout((long long)s.batch * s.heads, s.heads).total; }

ttt_status launch_conv3x3(const Call& c) {
    using namespace c3;
    if (c.dtype != TTT_BF16 || c.loss != TTT_LOSS_L2) return TTT_ERR_UNSUPPORTED;
    const long long units = (long long)c.batch * c.heads;
    const WsLayout L = ws_layout(units, c.heads);
    if (c.ws_bytes < L.total) return TTT_ERR_WORKSPACE;
    const Geo g = make_geo(c);
    if (g.T > (1LL << 40)) return TTT_ERR_UNSUPPORTED;
    CUtensorMap tmKH, tmQH, tmZ;
    if (!make_tmap_grid_sw128(&tmKH, c.K, c, TC, TR + 2) || !make_tmap_grid_sw128(&tmQH, c.Q, c, TC, TR + 2) ||
        !make_tmap_grid_sw128(&tmZ, c.Z, c, TC, TR))
        return TTT_ERR_INVALID_ARG;
    // gradient CTAs: as many per unit as fit, each within one unit, when there are fewer units than SMs
    const int S = std::min(c.num_sms, kMaxGrid);
    GradPart gpart{g.T, 0, 0, g.tpu};
    if (units <= S) {
        gpart.cpu = std::max(1, std::min(S / (int)units, g.tpu));
        gpart.G = (int)units * gpart.cpu;
    } else {
        gpart.G = (int)std::max<long long>(1, std::min<long long>(S, g.T));
    }
    const int G1 = gpart.G;
    const int G3 = (int)std::max<long long>(1, std::min<long long>(c.num_sms, g.T));
    uint32_t* err = reinterpret_cast<uint32_t*>(c.ws);

    GradParams gp{};
    gp.g = g;
    gp.part = gpart;
    gp.w0img = c.ws + L.w0img;
    gp.V = static_cast<const __nv_bfloat16*>(c.V);
    gp.bs = c.bs;
    gp.hs = c.hs;
    gp.slots = reinterpret_cast<float*>(c.ws + L.slots);
    gp.err = err;
    gp.wait_ns = c.wait_ns;
    const size_t sm1 = sizeof(GradSmem) + 1024, sm3 = sizeof(ReadSmem) + 1024;
    if (sm1 > 227 * 1024 || sm3 > 227 * 1024) return TTT_ERR_UNSUPPORTED;
    cudaFuncSetAttribute(conv3_grad, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    cudaFuncSetAttribute(conv3_readout, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3);
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(c.heads * D));
    cfg.blockDim = dim3(D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = c.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = c.overlap_previous ? 1 : 0;
    ttt_status st = check_launch(cudaLaunchKernelEx(&cfg, conv3_wprep, c.W0, c.ws + L.w0img));
    if (st != TTT_OK) return st;

    cfg.gridDim = dim3((unsigned)G1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sm1;
    cfg.numAttrs = 1;
    st = check_launch(cudaLaunchKernelEx(&cfg, conv3_grad, tmKH, gp));
    if (st != TTT_OK) return st;

    MergeParams mp{};
    mp.g = g;
    mp.part = gpart;
    mp.eta = c.eta;
    mp.W0 = c.W0;
    mp.slots = gp.slots;
    mp.W1_out = c.W1_out;
    mp.w1img = c.ws + L.w1img;
    cfg.gridDim = dim3((unsigned)(units * TAPS * 4));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.numAttrs = 1;
    st = check_launch(cudaLaunchKernelEx(&cfg, conv3_merge, mp));
    if (st != TTT_OK) return st;

    ReadParams rp{};
    rp.g = g;
    rp.G = G3;
    rp.w1img = mp.w1img;
    rp.err = err;
    rp.wait_ns = c.wait_ns;
    cfg.gridDim = dim3((unsigned)G3);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sm3;
    return check_launch(cudaLaunchKernelEx(&cfg, conv3_readout, tmQH, tmZ, rp));
}

}  // namespace ttt
