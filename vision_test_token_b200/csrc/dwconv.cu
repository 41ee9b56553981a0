// dwconv.cu -- 3x3 depthwise-convolution inner model of the TTT layer over the H x W token grid
// (press article "CVPR 2026 Oral | 清華+阿里發布ViT3", Observation 6 and Fig. 5 part 3; ViT^3 keeps
// one such head).  One full-batch step of the L2 loss, then the readout:
//     r[c,y,x] = sum_{a,b} W0[c][a][b] K[c,y+a-1,x+b-1] - V[c,y,x]           (zero padding)
//     g[c][a][b] = (2/N) sum_{y,x} r[c,y,x] K[c,y+a-1,x+b-1],   W1 = W0 - eta g
//     Z[c,y,x] = sum_{a,b} W1[c][a][b] Q[c,y+a-1,x+b-1]
// With the dot-product inner loss of the ViT^3 recipe (same article, section on the ViT3 model),
// L = -(1/N) sum <f(K;W), V>, the gradient has no residual: g[c][a][b] = -(1/N) sum V K[shifted]
// (the kernel's DOT instantiation, half the phase-1 FMAs).
//
// Not a contraction worth a tensor core (about 7 flop per byte, and no sharing across channels): fp32
// FMA in registers.
//
// One kernel (dw_band) of independent CTAs -- no clusters, so it fits whatever SMs are free, e.g. next
// to the linear-head kernel of the same layer.  A unit's grid is cut into tasks: a band of row pairs
// of one strip of at most XT columns; a launch makes about one task per CTA.  CTA c takes tasks c,
// c + grid, ...: first the gradient (phase 1) of each of its tasks, then the readout (phase 2) of
// each, so a CTA only waits for other CTAs after all of its own phase-1 work is done.
//   Streaming: the producer lane loads the task's rows as 2-row groups into two shared-memory rings:
//     K groups with a one-column halo on both sides, and V groups; then, without waiting for W1, the
//     Q groups of the readout into the K ring (so Q streams in while the unit's gradients are merged).
//     Output row pair j reads K groups j (rows 2j-1, 2j) and j+1 (rows 2j+1, 2j+2) and V group j.  The
//     tensor map's out-of-bounds zero fill supplies the zero padding, so the inner loops carry no
//     bounds checks.
//   Compute: three groups of 5 warps; group g takes the row pairs j = g (mod 3) of every task.  In a
//     group, warp w owns a column segment of both rows of a pair, lane l owns channels 2l and 2l+1,
//     and a 4 x 3 register window slides along the columns (unrolled by 3, so the window never moves
//     between registers), fed by explicit shared-memory loads.  The residual is carried negated
//     (s = V - W0 (*) K, from the negated taps), which saves a negation per token.
//   Merge: each group folds its warps' 64 x 9 sums in a fixed order, the CTA adds the three groups'
//     sums in group order into the task's partial, written to the workspace slot of (unit, task).
//     The CTA that writes a unit's last partial sums all of the unit's partials with all its compute
//     threads (three slices of tasks, each summed in task order with its loads in flight at once, then
//     the slices in order: a fixed order, so W1 is bitwise reproducible whichever CTA ran which task,
//     for a given grid), writes W1 and raises the unit's ready flag; the readout of the unit's tasks
//     waits for that flag (bounded).  Z is written straight from registers (128 coalesced bytes per
//     token and warp).
//   The last CTA to finish returns the workspace's counters and flags to zero for the next call.
//   When launched as a programmatic dependent of the preceding kernel (the linear heads of the same
//   layer), the kernel starts while that kernel runs and, at its very end, waits for it, so the
//   stream sees both complete when this one does.
#include <algorithm>

#include "sm100.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace dw {

constexpr int D = 64;
constexpr int TAPS = 9;
constexpr int GW = 5;                       // warps of a compute group (column segments of a row pair)
constexpr int CG = 3;                       // compute groups (row pairs j = g mod CG)
constexpr int CW = GW * CG;                 // compute warps
constexpr int THREADS = (CW + 1) * 32;      // + one producer warp (16 warps: 128 registers a thread)
constexpr int NK = 6;                       // K / Q ring slots (2-row groups)
constexpr int NV = 4;                       // V ring slots (2-row groups)
constexpr int kPart = D * TAPS;             // 576 floats: a 64 x 9 gradient or kernel, tap-major
constexpr int kRed = (GW + 1) / 2;          // a group's per-warp gradients are folded pairwise into kRed slots
constexpr int kTasksPerCta = 1;             // tasks a launch aims for per CTA
constexpr uint32_t kComputeBar = 4;         // named barrier of all compute warps (groups use 1..3)

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {                 // two bf16 channels in one 32-bit word
    static constexpr int kTokenBytes = D * 2;
    static constexpr int kXtMax = 80;
    static __device__ __forceinline__ float2 lds(uint32_t addr) {
        const uint32_t w = lds_u32(addr);
        return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float2 v) {
        *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v.x, v.y);
    }
};
template <>
struct Elem<float> {
    static constexpr int kTokenBytes = D * 4;
    static constexpr int kXtMax = 38;
    static __device__ __forceinline__ float2 lds(uint32_t addr) { return lds_f2(addr); }
    static __device__ __forceinline__ void store(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
};

struct Geom {
    int heads, H, W;
    int Sx, XT;                      // strips, strip width
    int Hp;                          // row pairs per strip: ceil(H / 2)
    int tps, tpu;                    // tasks per strip (each a contiguous band of row pairs), per unit
    long long bs, hs;                // element strides of Q/K/V/Z
    int k_pitch;                     // tokens per staged K/Q row (XT + 2)
    uint32_t kg_bytes, vg_bytes;     // one staged K/Q group (2 x k_pitch tokens), one V group (2 x XT)
};

struct Params {
    Geom g;
    int U;                           // units
    int T;                           // tasks (each: its gradient, then its readout)
    float eta_scale;                 // eta * 2 / N  (dot-product loss: eta / N)
    const float* W0;                 // [heads][64][9]
    float* W1_out;                   // nullable [units][64][9]
    uint32_t* err;                   // workspace error word
    uint32_t* done;                  // CTAs finished
    uint32_t* unit_count;            // [U] gradient partials written per unit
    uint32_t* ready;                 // [U] 1 once the unit's W1 is formed
    float* partials;                 // [U][mtpu][576] negated gradient sums per task, tap-major
    int mtpu;                        // partial slots per unit (one task per row pair, the most a call uses)
    float* w1g;                      // [U][576] W1 per unit, tap-major
    unsigned long long wait_ns;      // bound of every device-side wait
};

// Workspace layout: the 256-byte header (word 0: error word), the control words (done,
// unit_count[U], ready[U]) padded to 256 bytes, the partials, W1.
struct WsLayout {
    size_t ctl, partials, w1g, total;
};
static WsLayout ws_layout(long long U, int tpu) {
    WsLayout l;
    l.ctl = kWsHeader;
    l.partials = l.ctl + align_up((size_t)(1 + 2 * U) * 4, 256);
    l.w1g = l.partials + align_up((size_t)U * tpu * kPart * 4, 256);
    l.total = l.w1g + (size_t)U * kPart * 4;
    return l;
}

struct SmemTail {                            // follows the rings
    float red[CG][kRed][kPart];              // per-warp gradients of each group, folded pairwise
    uint64_t kfull[NK], kempty[NK], vfull[NV], vempty[NV];
    int last;
    int abort_flag;
};

__host__ __device__ __forceinline__ int split_lo(int n, int r, int parts) { return (int)((long long)n * r / parts); }

struct Task {
    int u, r, sx, pa, n;                     // unit, task index in the unit, strip, first pair, pairs
};

__device__ __forceinline__ Task decode(const Params& p, int t) {
    Task k;
    k.u = t / p.g.tpu;
    k.r = t % p.g.tpu;
    k.sx = k.r / p.g.tps;
    const int c = k.r % p.g.tps;
    k.pa = split_lo(p.g.Hp, c, p.g.tps);
    k.n = split_lo(p.g.Hp, c + 1, p.g.tps) - k.pa;
    return k;
}

__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}

// Waits for fill number q of a ring slot (q = sequence number / slots).  A group reads only some of
// the fills, so the fill before q -- another group's -- may still be in flight, and a parity wait on
// `full` alone would then pass one phase early.  Waiting first for that fill's release on `empty`
// (which needs this reader's own arrival before it can move past fill q) leaves the `full` wait
// unambiguous.
__device__ __forceinline__ bool ring_wait(uint64_t* full, uint64_t* empty, uint32_t q, const Abort& ab) {
    return mbar_wait(empty, (q & 1u) ^ 1u, ab) && mbar_wait(full, q & 1u, ab);
}

// The 4 staged rows around an output row pair: rows 0, 1 from one group, rows 2, 3 from the next
// (32-bit shared addresses of the lane's channel pair in column 0 of each group).
struct Rows {
    uint32_t a;                      // rows y0-1, y0
    uint32_t b;                      // rows y0+1, y0+2
    uint32_t row_bytes;              // bytes of one staged row (k_pitch tokens)
};

template <typename T, int C>
__device__ __forceinline__ void load_col(float2 (&win)[4][3], const Rows& rw, int col) {
    const uint32_t o = (uint32_t)col * Elem<T>::kTokenBytes;
    win[0][C] = Elem<T>::lds(rw.a + o);
    win[1][C] = Elem<T>::lds(rw.a + rw.row_bytes + o);
    win[2][C] = Elem<T>::lds(rw.b + o);
    win[3][C] = Elem<T>::lds(rw.b + rw.row_bytes + o);
}

// s = v + sum over the 3 x 3 taps of nw * K at window rows r0 .. r0+2, as three independent
// 3-term chains (one per tap row) added at the end: a dependency depth of 5 instead of 9.
template <int L, int M, int R>
__device__ __forceinline__ float2 neg_residual(const float2 (&win)[4][3], const float2 (&nw)[TAPS], int r0, float2 v) {
    constexpr int cidx[3] = {L, M, R};
    const float2 zero = make_float2(0.f, 0.f);
    float2 t0 = v, t1 = zero, t2 = zero;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        t0 = ffma2(nw[c], win[r0][cidx[c]], t0);
        t1 = ffma2(nw[3 + c], win[r0 + 1][cidx[c]], t1);
        t2 = ffma2(nw[6 + c], win[r0 + 2][cidx[c]], t2);
    }
    return make_float2(t0.x + t1.x + t2.x, t0.y + t1.y + t2.y);
}

// Both rows of a pair: s0 from window rows 0..2, s1 from rows 1..3, with their six chains interleaved.
template <int L, int M, int R>
__device__ __forceinline__ void neg_residual2(const float2 (&win)[4][3], const float2 (&nw)[TAPS], float2 v0,
                                              float2 v1, float2& s0, float2& s1) {
    constexpr int cidx[3] = {L, M, R};
    const float2 zero = make_float2(0.f, 0.f);
    float2 a0 = v0, a1 = zero, a2 = zero, b0 = v1, b1 = zero, b2 = zero;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        a0 = ffma2(nw[c], win[0][cidx[c]], a0);
        b0 = ffma2(nw[c], win[1][cidx[c]], b0);
        a1 = ffma2(nw[3 + c], win[1][cidx[c]], a1);
        b1 = ffma2(nw[3 + c], win[2][cidx[c]], b1);
        a2 = ffma2(nw[6 + c], win[2][cidx[c]], a2);
        b2 = ffma2(nw[6 + c], win[3][cidx[c]], b2);
    }
    s0 = make_float2(a0.x + a1.x + a2.x, a0.y + a1.y + a2.y);
    s1 = make_float2(b0.x + b1.x + b2.x, b0.y + b1.y + b2.y);
}

// Phase-1 work of output column x (strip-relative) of the row pair: window columns L, M, R hold
// staged columns x, x+1, x+2 (image columns x-1, x, x+1); R is loaded here.  nw = -W0 taps;
// gacc accumulates sum s * K with s = V - W0 (*) K = -r (L2 loss) or s = V (dot-product loss, whose
// gradient has no residual: nw is unused).  vg: shared address of the lane's channels in V column 0
// of the group's first row; vrow: bytes of one staged V row.
template <typename T, bool DOT, bool ROW1, int L, int M, int R>
__device__ __forceinline__ void p1_col(float2 (&win)[4][3], const float2 (&nw)[TAPS], float2 (&gacc)[TAPS],
                                       const Rows& rw, uint32_t vg, uint32_t vrow, int x) {
    using E = Elem<T>;
    load_col<T, R>(win, rw, x + 2);
    const uint32_t vo = vg + (uint32_t)x * E::kTokenBytes;
    constexpr int cidx[3] = {L, M, R};
    if (ROW1) {                                            // the second row of the pair lies inside the grid
        // both rows' residual chains side by side (six independent 3-term chains), then the nine
        // row-0 updates before the nine row-1 updates, so that no update waits on the one before it
        float2 s0, s1;
        if (DOT) {
            s0 = E::lds(vo);
            s1 = E::lds(vo + vrow);
        } else {
            neg_residual2<L, M, R>(win, nw, E::lds(vo), E::lds(vo + vrow), s0, s1);
        }
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int c = 0; c < 3; ++c) gacc[a * 3 + c] = ffma2(s0, win[a][cidx[c]], gacc[a * 3 + c]);
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int c = 0; c < 3; ++c) gacc[a * 3 + c] = ffma2(s1, win[a + 1][cidx[c]], gacc[a * 3 + c]);
    } else {
        const float2 v0 = E::lds(vo);
        const float2 s0 = DOT ? v0 : neg_residual<L, M, R>(win, nw, 0, v0);
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int c = 0; c < 3; ++c) gacc[a * 3 + c] = ffma2(s0, win[a][cidx[c]], gacc[a * 3 + c]);
    }
}

template <typename T, bool DOT, bool ROW1>
__device__ __forceinline__ void p1_pair(const float2 (&nw)[TAPS], float2 (&gacc)[TAPS], const Rows& rw,
                                        uint32_t vg, uint32_t vrow, int xa, int xb) {
    float2 win[4][3];
    load_col<T, 0>(win, rw, xa);
    load_col<T, 1>(win, rw, xa + 1);
    int x = xa;
    for (; x + 3 <= xb; x += 3) {
        p1_col<T, DOT, ROW1, 0, 1, 2>(win, nw, gacc, rw, vg, vrow, x);
        p1_col<T, DOT, ROW1, 1, 2, 0>(win, nw, gacc, rw, vg, vrow, x + 1);
        p1_col<T, DOT, ROW1, 2, 0, 1>(win, nw, gacc, rw, vg, vrow, x + 2);
    }
    if (x < xb) {
        p1_col<T, DOT, ROW1, 0, 1, 2>(win, nw, gacc, rw, vg, vrow, x);
        if (x + 1 < xb) p1_col<T, DOT, ROW1, 1, 2, 0>(win, nw, gacc, rw, vg, vrow, x + 1);
    }
}

// Phase-2 work of output column x: z = W1 (*) Q for the rows of the pair.
template <typename T, bool ROW1, int L, int M, int R>
__device__ __forceinline__ void p2_col(float2 (&win)[4][3], const float2 (&w)[TAPS], const Rows& rw, T* z0, T* z1,
                                       int x) {
    load_col<T, R>(win, rw, x + 2);
    constexpr int cidx[3] = {L, M, R};
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            a0 = ffma2(w[a * 3 + c], win[a][cidx[c]], a0);
            if (ROW1) a1 = ffma2(w[a * 3 + c], win[a + 1][cidx[c]], a1);
        }
    Elem<T>::store(z0 + (size_t)x * D, a0);
    if (ROW1) Elem<T>::store(z1 + (size_t)x * D, a1);
}

template <typename T, bool ROW1>
__device__ __forceinline__ void p2_pair(const float2 (&w)[TAPS], const Rows& rw, T* z0, T* z1, int xa, int xb) {
    float2 win[4][3];
    load_col<T, 0>(win, rw, xa);
    load_col<T, 1>(win, rw, xa + 1);
    int x = xa;
    for (; x + 3 <= xb; x += 3) {
        p2_col<T, ROW1, 0, 1, 2>(win, w, rw, z0, z1, x);
        p2_col<T, ROW1, 1, 2, 0>(win, w, rw, z0, z1, x + 1);
        p2_col<T, ROW1, 2, 0, 1>(win, w, rw, z0, z1, x + 2);
    }
    if (x < xb) {
        p2_col<T, ROW1, 0, 1, 2>(win, w, rw, z0, z1, x);
        if (x + 1 < xb) p2_col<T, ROW1, 1, 2, 0>(win, w, rw, z0, z1, x + 1);
    }
}

template <typename T, bool DOT>
__global__ void __launch_bounds__(THREADS, 1)
dw_band(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
        const __grid_constant__ CUtensorMap tmQ, T* __restrict__ Z, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 128-byte aligned start, derived from the shared array by pointer arithmetic only
    uint8_t* base = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const Geom& g = p.g;
    uint8_t* kring = base;
    uint8_t* vring = kring + (size_t)NK * g.kg_bytes;
    SmemTail& s = *reinterpret_cast<SmemTail*>(vring + (size_t)NV * g.vg_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&s.abort_flag, p.err, p.wait_ns};

    if (threadIdx.x == 0) {
        s.abort_flag = 0;
        // a K group is read by two row pairs, each by GW warps; a V group by one row pair
        for (int i = 0; i < NK; ++i) { mbar_init(&s.kfull[i], 1); mbar_init(&s.kempty[i], 2 * GW); }
        for (int i = 0; i < NV; ++i) { mbar_init(&s.vfull[i], 1); mbar_init(&s.vempty[i], GW); }
        fence_barrier_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmQ);
    }
    __syncthreads();
    // A kernel queued behind this one as a programmatic dependent (the next call's linear heads) may
    // be scheduled as SMs free up; it waits for this grid to complete before it reads anything.
    pdl_launch_dependents();

    if (warp == CW) {                                                // producer
        if (lane == 0) {
            uint32_t kq = 0, vq = 0;                                 // loads issued into each ring
            auto load_k = [&](const CUtensorMap* tm, int xs, int y, int h, int bi) -> bool {
                const uint32_t sl = kq % NK, ph = (kq / NK) & 1u;
                if (!mbar_wait(&s.kempty[sl], ph ^ 1u, ab)) return false;
                mbar_arrive_expect_tx(&s.kfull[sl], g.kg_bytes);
                tma_load_5d(kring + (size_t)sl * g.kg_bytes, tm, &s.kfull[sl], 0, xs - 1, y, h, bi);
                ++kq;
                return true;
            };
            auto load_v = [&](int xs, int y, int h, int bi) -> bool {
                const uint32_t sl = vq % NV, ph = (vq / NV) & 1u;
                if (!mbar_wait(&s.vempty[sl], ph ^ 1u, ab)) return false;
                mbar_arrive_expect_tx(&s.vfull[sl], g.vg_bytes);
                tma_load_5d(vring + (size_t)sl * g.vg_bytes, &tmV, &s.vfull[sl], 0, xs, y, h, bi);
                ++vq;
                return true;
            };
            bool ok = true;
            // phase 1 of every task of this CTA (K(0), then K(j+1), V(j)), then the readout rows of
            // every task: Q streams in while the gradients are merged
            for (int t = blockIdx.x; t < p.T && ok; t += gridDim.x) {
                const Task tk = decode(p, t);
                const int bi = tk.u / g.heads, h = tk.u % g.heads, xs = tk.sx * g.XT, y0 = 2 * tk.pa;
                ok = load_k(&tmK, xs, y0 - 1, h, bi);
                for (int j = 0; j < tk.n && ok; ++j)
                    ok = load_k(&tmK, xs, y0 + 2 * j + 1, h, bi) && load_v(xs, y0 + 2 * j, h, bi);
            }
            for (int t = blockIdx.x; t < p.T && ok; t += gridDim.x) {
                const Task tk = decode(p, t);
                const int bi = tk.u / g.heads, h = tk.u % g.heads, xs = tk.sx * g.XT, y0 = 2 * tk.pa;
                for (int j = 0; j <= tk.n && ok; ++j) ok = load_k(&tmQ, xs, y0 + 2 * j - 1, h, bi);
            }
            // Before the CTA may exit, every load issued into the rings has landed (on a normal exit
            // they were all consumed already; after a wait gave up, some may still be in flight).
            for (uint32_t q = kq > (uint32_t)NK ? kq - NK : 0u; q < kq; ++q)
                mbar_drain(&s.kfull[q % NK], (q / NK) & 1u, ab.limit);
            for (uint32_t q = vq > (uint32_t)NV ? vq - NV : 0u; q < vq; ++q)
                mbar_drain(&s.vfull[q % NV], (q / NV) & 1u, ab.limit);
        }
        __syncwarp();                                                // the warp reaches the block barrier converged
    } else {
        // compute warps: CG groups of GW warps; group g takes the row pairs j = g (mod CG) of every task
        // (a fixed split, so each partial holds the same sums whichever CTA runs the task) and publishes
        // its own partial, so the groups never wait for one another
        const int tid = threadIdx.x;                                 // 0 .. CW*32-1
        const int grp = warp / GW, seg = warp % GW, gtid = tid - grp * GW * 32;
        const uint32_t gbar = 1u + (uint32_t)grp;                    // the group's named barrier
        const uint32_t kring_s = smem_u32(kring), vring_s = smem_u32(vring);
        const uint32_t krow = (uint32_t)g.k_pitch * Elem<T>::kTokenBytes;
        const uint32_t vrow = (uint32_t)g.XT * Elem<T>::kTokenBytes;
        const uint32_t lane_b = (uint32_t)lane * (Elem<T>::kTokenBytes / 32);
        uint32_t kq = 0, vq = 0;                                     // ring sequence numbers
        bool failed = false;
        // ---- phase 1 of every task of this CTA
        for (int t = blockIdx.x; t < p.T && !failed; t += gridDim.x) {
            const Task tk = decode(p, t);
            const int h = tk.u % g.heads, xs = tk.sx * g.XT;
            const int cols = min(g.W - xs, g.XT), segw = (cols + GW - 1) / GW;
            const int xa = seg * segw, xb = min(cols, xa + segw);    // strip-relative output columns
            const int n = tk.n;
            // negated gradient sums over this group's row pairs of the task
            float2 nw[TAPS], gacc[TAPS];
#pragma unroll
            for (int t9 = 0; t9 < TAPS; ++t9) {
                nw[t9] = DOT ? make_float2(0.f, 0.f)
                             : make_float2(-__ldg(p.W0 + ((size_t)h * D + 2 * lane) * TAPS + t9),
                                           -__ldg(p.W0 + ((size_t)h * D + 2 * lane + 1) * TAPS + t9));
                gacc[t9] = make_float2(0.f, 0.f);
            }
            for (int j = 0; j < n; ++j) {
                if (j % CG != grp || failed) continue;
                const uint32_t k0 = kq + j, k1 = kq + j + 1, v0 = vq + j;
                bool okb = ring_wait(&s.kfull[k0 % NK], &s.kempty[k0 % NK], k0 / NK, ab);
                okb = okb && ring_wait(&s.kfull[k1 % NK], &s.kempty[k1 % NK], k1 / NK, ab);
                okb = okb && ring_wait(&s.vfull[v0 % NV], &s.vempty[v0 % NV], v0 / NV, ab);
                if (!okb) { failed = true; continue; }
                __syncwarp();
                if (xa < xb) {
                    const Rows rw{kring_s + (k0 % NK) * g.kg_bytes + lane_b, kring_s + (k1 % NK) * g.kg_bytes + lane_b,
                                  krow};
                    const uint32_t vg = vring_s + (v0 % NV) * g.vg_bytes + lane_b;
                    if (2 * (tk.pa + j) + 1 < g.H) p1_pair<T, DOT, true>(nw, gacc, rw, vg, vrow, xa, xb);
                    else p1_pair<T, DOT, false>(nw, gacc, rw, vg, vrow, xa, xb);
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_n(&s.kempty[k0 % NK], j == 0 ? 2u : 1u);          // group 0 has one reader pair
                    mbar_arrive_n(&s.kempty[k1 % NK], j == n - 1 ? 2u : 1u);      // so has the last group
                    mbar_arrive(&s.vempty[v0 % NV]);
                }
            }
            kq += (uint32_t)n + 1; vq += (uint32_t)n;
            // every compute warp stops on a failure anywhere in the CTA (a uniform decision: the
            // groups meet at CTA-wide barriers below)
            if (named_bar_or(kComputeBar, CW * 32, failed)) { failed = true; break; }
            // ---- the group's partial, summed over its warps in a fixed order, into red[grp][0]
            float(*red)[kPart] = s.red[grp];
            if (seg >= kRed) {                                       // warps kRed.. store, warps 0.. add
#pragma unroll
                for (int t9 = 0; t9 < TAPS; ++t9)
                    *reinterpret_cast<float2*>(&red[seg - kRed][t9 * D + 2 * lane]) = gacc[t9];
            }
            named_bar_sync(gbar, GW * 32);
            if (seg < kRed) {
                const bool pair = seg + kRed < GW;                   // a partner warp stored into this slot
#pragma unroll
                for (int t9 = 0; t9 < TAPS; ++t9) {
                    float2* q = reinterpret_cast<float2*>(&red[seg][t9 * D + 2 * lane]);
                    const float2 o = pair ? *q : make_float2(0.f, 0.f);
                    *q = make_float2(gacc[t9].x + o.x, gacc[t9].y + o.y);
                }
            }
            named_bar_sync(gbar, GW * 32);
            for (int e = gtid; e < kPart; e += GW * 32) {
                float acc = 0.f;
#pragma unroll
                for (int ww = 0; ww < kRed; ++ww) acc += red[ww][e];
                red[0][e] = acc;                                     // this thread's own element only
            }
            // ---- the task's partial: the three groups' partials in group order (all compute warps
            //      of the CTA take the same tasks in the same order, so they meet here once per task)
            named_bar_sync(kComputeBar, CW * 32);
            float* part = p.partials + ((size_t)tk.u * p.mtpu + tk.r) * kPart;
            for (int e = tid; e < kPart; e += CW * 32)
                part[e] = (s.red[0][0][e] + s.red[1][0][e]) + s.red[2][0][e];
            __threadfence();
            named_bar_sync(kComputeBar, CW * 32);
            if (tid == 0) s.last = (atomicAdd(p.unit_count + tk.u, 1u) == (uint32_t)(g.tpu - 1)) ? 1 : 0;
            named_bar_sync(kComputeBar, CW * 32);
            if (s.last) {
                // ---- the unit's last partial: W1 = W0 - eta (2/N) g = W0 + eta_scale * (sum of the
                //      unit's task partials in task order).  Thread (e4, sl) sums slice sl of the tasks
                //      (about a third, all loads in flight), then the slices are added in order.
                __threadfence();
                const float* pu = p.partials + (size_t)tk.u * p.mtpu * kPart;
                const int R = g.tpu;
                constexpr int kE4 = kPart / 4;                       // 144 float4 per partial
                float4* sl_sum = reinterpret_cast<float4*>(&s.red[1][0][0]);   // [3][144] (red[1], red[2] free)
                const int e4 = tid % kE4, sl = tid / kE4;
                if (sl < 3) {
                    const int r0 = split_lo(R, sl, 3), r1 = split_lo(R, sl + 1, 3);
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int rb = r0; rb < r1; rb += 8) {            // 8 loads in flight, added in order
                        float4 v[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            v[q] = (rb + q < r1) ? __ldcg(reinterpret_cast<const float4*>(pu + (size_t)(rb + q) * kPart) + e4)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            if (rb + q < r1) { acc.x += v[q].x; acc.y += v[q].y; acc.z += v[q].z; acc.w += v[q].w; }
                    }
                    sl_sum[sl * kE4 + e4] = acc;
                }
                named_bar_sync(kComputeBar, CW * 32);
                if (tid < kE4) {
                    const float4 x0 = sl_sum[tid], x1 = sl_sum[kE4 + tid], x2 = sl_sum[2 * kE4 + tid];
                    const float a4[4] = {(x0.x + x1.x) + x2.x, (x0.y + x1.y) + x2.y, (x0.z + x1.z) + x2.z,
                                         (x0.w + x1.w) + x2.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int e = 4 * tid + i, t9 = e / D, ch = e % D;   // tap-major index
                        const float w1 = __ldg(p.W0 + ((size_t)h * D + ch) * TAPS + t9) + p.eta_scale * a4[i];
                        p.w1g[(size_t)tk.u * kPart + e] = w1;
                        if (p.W1_out) p.W1_out[((size_t)tk.u * D + ch) * TAPS + t9] = w1;
                    }
                }
                __threadfence();
                named_bar_sync(kComputeBar, CW * 32);
                if (tid == 0) st_release_gpu(p.ready + tk.u, 1u);
            }
            named_bar_sync(kComputeBar, CW * 32);                    // s.last and red are reused by the next task
        }
        // ---- phase 2 of every task of this CTA: Z = W1 (*) Q over this group's row pairs
        for (int t = blockIdx.x; t < p.T && !failed; t += gridDim.x) {
            const Task tk = decode(p, t);
            const int bi = tk.u / g.heads, h = tk.u % g.heads, xs = tk.sx * g.XT;
            const int cols = min(g.W - xs, g.XT), segw = (cols + GW - 1) / GW;
            const int xa = seg * segw, xb = min(cols, xa + segw);
            const int n = tk.n;
            // the unit's W1 (lane 0 waits, bounded; the warp follows its decision)
            int okw = 1;
            if (lane == 0) okw = wait_flag(p.ready + tk.u, ab) ? 1 : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) failed = true;
            float2 w[TAPS];
#pragma unroll
            for (int t9 = 0; t9 < TAPS; ++t9)
                w[t9] = __ldcg(reinterpret_cast<const float2*>(p.w1g + (size_t)tk.u * kPart + t9 * D) + lane);
            const long long off = (long long)bi * g.bs + (long long)h * g.hs;
            for (int j = 0; j < n; ++j) {
                if (j % CG != grp || failed) continue;
                const uint32_t k0 = kq + j, k1 = kq + j + 1;
                bool okb = ring_wait(&s.kfull[k0 % NK], &s.kempty[k0 % NK], k0 / NK, ab);
                okb = okb && ring_wait(&s.kfull[k1 % NK], &s.kempty[k1 % NK], k1 / NK, ab);
                if (!okb) { failed = true; continue; }
                __syncwarp();
                const int y0 = 2 * (tk.pa + j);
                if (xa < xb) {
                    const Rows rw{kring_s + (k0 % NK) * g.kg_bytes + lane_b, kring_s + (k1 % NK) * g.kg_bytes + lane_b,
                                  krow};
                    T* z0 = Z + off + ((long long)y0 * g.W + xs) * D + 2 * lane;
                    T* z1 = z0 + (long long)g.W * D;
                    if (y0 + 1 < g.H) p2_pair<T, true>(w, rw, z0, z1, xa, xb);
                    else p2_pair<T, false>(w, rw, z0, z1, xa, xb);
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_n(&s.kempty[k0 % NK], j == 0 ? 2u : 1u);
                    mbar_arrive_n(&s.kempty[k1 % NK], j == n - 1 ? 2u : 1u);
                }
            }
            kq += (uint32_t)n + 1;
        }
    }
    // The last CTA to finish puts the control words back to zero for the next call.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s.last = (atomicAdd(p.done, 1u) == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (s.last) {
        __threadfence();
        for (int i = threadIdx.x; i < p.U; i += blockDim.x) { p.unit_count[i] = 0u; p.ready[i] = 0u; }
        if (threadIdx.x == 0) *p.done = 0u;
    }
    // As a programmatic dependent of the preceding kernel: complete only after it has completed.
    pdl_wait_primary();
}

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
// Tasks per strip: about kTasksPerCta tasks per CTA (at most one task per row pair).
template <typename T>
static Geom make_geom(long long units, int grid, int heads, int H, int W, long long bs, long long hs) {
    constexpr int TB = Elem<T>::kTokenBytes;
    Geom g;
    g.heads = heads;
    g.H = H;
    g.W = W;
    g.Sx = (W + Elem<T>::kXtMax - 1) / Elem<T>::kXtMax;
    g.XT = (W + g.Sx - 1) / g.Sx;
    g.Hp = (H + 1) / 2;
    g.tps = (int)std::min<long long>(g.Hp, std::max<long long>(1, kTasksPerCta * grid / std::max<long long>(1, units * g.Sx)));
    g.tpu = g.Sx * g.tps;
    g.bs = bs;
    g.hs = hs;
    g.k_pitch = g.XT + 2;
    g.kg_bytes = (uint32_t)(2 * g.k_pitch * TB);
    g.vg_bytes = (uint32_t)(2 * g.XT * TB);
    return g;
}

template <typename T>
static size_t smem_bytes(const Geom& g) {
    return 128 + (size_t)NK * g.kg_bytes + (size_t)NV * g.vg_bytes + sizeof(SmemTail);
}

// Partial slots a unit may need: one task per row pair of every strip (the workspace is sized for
// that, so that its size does not depend on the grid).
static int max_tasks_per_unit(const ttt_shape& s) {
    const int xt = (s.dtype == TTT_BF16) ? Elem<__nv_bfloat16>::kXtMax : Elem<float>::kXtMax;
    return ((s.W + xt - 1) / xt) * ((s.H + 1) / 2);
}

template <typename T, bool DOT>
static ttt_status launch(const Call& c) {
    const long long units = (long long)c.batch * c.heads;
    const int grid_max = std::max(1, c.num_sms);
    const Geom g = make_geom<T>(units, grid_max, c.heads, c.H, c.W, c.bs, c.hs);
    const size_t smem = smem_bytes<T>(g);
    if (smem > 227 * 1024) return TTT_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(units, g.Sx * g.Hp);
    if (c.ws_bytes < L.total) return TTT_ERR_WORKSPACE;
    cudaFuncSetAttribute(dw_band<T, DOT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const long long T_all = units * g.tpu;
    if (T_all > (1LL << 30)) return TTT_ERR_UNSUPPORTED;
    const int grid = (int)std::max<long long>(1, std::min<long long>(grid_max, T_all));

    CUtensorMap tmK, tmV, tmQ;
    if (!make_tmap_grid(&tmK, c.K, c, g.k_pitch, 2) || !make_tmap_grid(&tmV, c.V, c, g.XT, 2) ||
        !make_tmap_grid(&tmQ, c.Q, c, g.k_pitch, 2))
        return TTT_ERR_INVALID_ARG;
    Params p;
    p.g = g;
    p.U = (int)units;
    p.T = (int)T_all;
    // W1 = W0 + eta_scale * sum s K:  L2 loss s = -r, gradient (2/N) sum r K;  dot-product loss
    // s = V, gradient -(1/N) sum V K
    p.eta_scale = c.eta * ((DOT ? 1.0f : 2.0f) / (float)c.N);
    p.W0 = c.W0;
    p.W1_out = c.W1_out;
    p.err = reinterpret_cast<uint32_t*>(c.err_ws ? c.err_ws : c.ws);
    uint32_t* ctl = reinterpret_cast<uint32_t*>(c.ws + L.ctl);
    p.done = ctl;
    p.unit_count = ctl + 1;
    p.ready = ctl + 1 + units;
    p.partials = reinterpret_cast<float*>(c.ws + L.partials);
    p.mtpu = g.Sx * g.Hp;
    p.w1g = reinterpret_cast<float*>(c.ws + L.w1g);
    p.wait_ns = c.wait_ns;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = c.overlap_previous ? 1 : 0;
    return check_launch(cudaLaunchKernelEx(&cfg, dw_band<T, DOT>, tmK, tmV, tmQ, static_cast<T*>(c.Z), p));
}

}  // namespace dw

size_t dwconv_ws_bytes(const ttt_shape& s) {
    const long long units = (long long)s.batch * s.heads;
    return dw::ws_layout(units, dw::max_tasks_per_unit(s)).total;
}

size_t dwconv_ws_control_bytes(const ttt_shape& s) {
    const long long units = (long long)s.batch * s.heads;
    return dw::ws_layout(units, dw::max_tasks_per_unit(s)).partials;
}

ttt_status launch_dwconv(const Call& c) {
    const bool dot = c.loss == TTT_LOSS_DOT;
    if (c.dtype == TTT_BF16) return dot ? dw::launch<__nv_bfloat16, true>(c) : dw::launch<__nv_bfloat16, false>(c);
    return dot ? dw::launch<float, true>(c) : dw::launch<float, false>(c);
}

}  // namespace ttt
