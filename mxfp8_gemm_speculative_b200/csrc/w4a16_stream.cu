// INT4 W4A16 weight-streaming GEMM for small M (decode / MTP verify chunks).
//
// At M <= 32 the layer reads each weight byte once and does 2*M flops per
// weight: it is bound by HBM bytes of W, and the whole design is about
// keeping enough weight bytes in flight on every SM while the decode and the
// MMAs run behind them.
//
//  * Columns are taken eight n32 tiles (256 columns) at a time, a "column
//    group".  The weight stream of a group row is cut into units of
//    max(KS, G) rows of K (KS = rows per pipeline stage), and every CTA of a
//    one-CTA-per-SM grid takes one contiguous run of units (stream-K), so all
//    SMs stream the same number of bytes.
//  * One producer warp fills a CTA-wide ring of stages with 2-D tensor-map
//    copies (TMA): per stage the codes of the eight tiles for KS rows of K
//    (one box), their scales (one box) and the activations X for the same
//    rows (64-wide boxes with 128-byte swizzle; rows past M are zero-filled by
//    the copy).  Completion is an mbarrier per stage; the consumers release a
//    stage through a second mbarrier.  Weights are marked evict-first in L2,
//    the activations evict-last (every CTA re-reads them).
//  * Eight consumer warps, warp w owning tile w of the group for the whole
//    K range of the CTA's segment: no reduction between warps.  Each warp
//    decodes a pair of nibbles to the bf16 pair (128 + q) with one
//    mask-and-or (plus a shift) and multiplies on the tensor cores with
//    m16n8k16 MMAs where the weights are the 16-row operand and the tokens
//    the 8-column operand ("swap AB"); one more MMA with an all-ones weight
//    tile gives the per-token activation sum that turns (128 + q) into
//    (q - 8).  A zero-initialised partial sum per scale group is folded in
//    as acc += (part - 136 * activation sum) * scale in fp32, so weights are
//    never rounded (every product is exact in fp32).
//  * A group row cut between CTAs is finished by the CTA holding its first
//    unit, which reaches it last in its run; the other contributors (for
//    whom it is the first segment of their run) publish their fragments
//    early, so the finisher adds them in CTA order (deterministic) and
//    writes bf16 Y.  A group row inside one run is written directly.
//  * The footprint (9 warps, <= 112 registers for M <= 16, ~100 KB of shared
//    memory) lets two CTAs share an SM: the next GEMM on the stream (launched
//    with programmatic dependent launch) becomes resident while this one
//    streams, issues its first weight copies and warms L2 with the next part
//    of its run, and only then waits for this grid before reading X.
//
// The same kernel runs INT8 W8A16 weights (the vocabulary head): their
// re-pack splits each 8-bit code q = 16 hi + lo into a plane of low and a
// plane of high nibbles in the INT4 layout, the kernel decodes both planes
// with the same mask-and-or, runs one MMA per plane and forms
// 16 * P_hi + P_lo - 2304 * (activation sum) per group.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

#ifndef MXG_STREAM_KS
#define MXG_STREAM_KS 64
#endif
#ifndef MXG_STREAM_RING_KB
#define MXG_STREAM_RING_KB 104
#endif
#ifndef MXG_STREAM_RING2_KB
#define MXG_STREAM_RING2_KB 192
#endif
#ifndef MXG_STREAM_WPT2_MAX_TT
#define MXG_STREAM_WPT2_MAX_TT 0
#endif
#ifndef MXG_STREAM_PF_STAGES
#define MXG_STREAM_PF_STAGES 12
#endif

constexpr int kWarps = 8;                     // n32 tiles of a column group

// Consumer warps per tile: two for narrow token tiles (each takes every
// other stage of the run, so a warp has two stages' time for the latency
// chain of one), one for wide ones (whose registers allow no more warps).
template <int TT>
struct Wpt {
    static constexpr int value = TT <= MXG_STREAM_WPT2_MAX_TT ? 2 : 1;
};

// Group modes: 0 -> G = 128, 1 -> G = 64, 2 -> G = 32.  P code planes: 1 for
// INT4; 2 for INT8 (low and high nibbles, each in the INT4 layout).
template <int TT, int GM, int P>
struct Cfg {
    static constexpr int kWPT = Wpt<TT>::value;
    static constexpr int kConsumers = kWarps * kWPT;
    static constexpr int kThreads = (kConsumers + 1) * 32;         // + the producer warp
    static constexpr int kProducer = kConsumers;                   // its warp index
    // one CTA per SM with two consumer warps per tile; with one, the ring
    // leaves room for a second CTA (the next GEMM on the stream)
    static constexpr int kRingBytes = (kWPT == 2 ? MXG_STREAM_RING2_KB : MXG_STREAM_RING_KB) * 1024;
    static constexpr int kG = GM == 0 ? 128 : (GM == 1 ? 64 : 32);
    static constexpr int kKS = P == 2 ? 64 : MXG_STREAM_KS;       // rows of K per stage
    static constexpr int kChunks = kKS / 64;                       // k64 chunks per stage
    static constexpr int kSteps = kKS / 16;                        // k16 MMA steps per stage
    static constexpr int kStepsPerGroup = kG / 16;
    // steps between scale epilogues: a group, or a stage when a group spans
    // stages that different warps take
    static constexpr int kEpi = (kWPT == 2 && kStepsPerGroup > kSteps) ? kSteps : kStepsPerGroup;
    static constexpr int kUS = kG > kKS ? kG / kKS : 1;            // stages per stream-K unit
    static constexpr int kUnitK = kUS * kKS;                       // rows of K per unit
    static constexpr int kScaleGroups = kKS >= kG ? kKS / kG : 1;  // groups in a stage's scale box
    static constexpr int kCodeTile = kChunks * 1024 * P;           // code bytes of a tile per stage
    static constexpr int kCode = kWarps * kCodeTile;
    static constexpr int kXBox = 128 * 8 * TT;                     // 64 k x 8TT rows of bf16
    static constexpr int kX = kChunks * kXBox;
    static constexpr int kScaleTile = 64 * kScaleGroups;
    static constexpr int kScale = kWarps * kScaleTile;
    static constexpr int kTx = kX + kCode + kScale;                // bytes landing per stage
    static constexpr int kStage = (kTx + 1023) / 1024 * 1024;      // X boxes stay 1024-aligned
    static constexpr int kStages = kRingBytes / kStage > 3 ? kRingBytes / kStage : 3;
    static constexpr int kF = 2 * TT;                              // float4 per lane fragment
    // fragments the second warp of a tile hands to the first at a segment end
    static constexpr int kXchgOff = kStages * kStage;
    static constexpr int kXchg = kWPT == 2 ? kWarps * kF * 32 * 16 : 0;
    static constexpr int kBarOff = kXchgOff + kXchg;
    static constexpr size_t kSmem = (size_t)kBarOff + 2 * kStages * 8 + 1024;  // + alignment
};

struct Params {
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [column groups * 8]
    float4 *partial;         // [ctas][8 warps][2*TT][32]: a CTA's fragments of its first, cut group row
    int M, N;
    int ntiles;              // N / 32
    int upr;                 // units per group row
    int q, r;                // units = q * ctas + r: CTAs below r run q + 1 units, the rest q
    int early;               // load the first weights before waiting for the previous kernel
    int pf_stages;           // stages after the ring warmed in L2 at entry
};

__device__ __forceinline__ int run_start(const Params &p, int c)
{
    return c * p.q + min(c, p.r);
}

// The CTA whose run contains unit u.
__device__ __forceinline__ int cta_of_unit(const Params &p, int u)
{
    const int big = p.r * (p.q + 1);   // units covered by the longer runs
    return u < big ? u / (p.q + 1) : p.r + (u - big) / p.q;
}

// Writes the four outputs of fragment float4 j (= h * TT + tt) of `lane`.
template <int TT>
__device__ __forceinline__ void store_y4(const Params &p, int tile, int j, int lane, float4 v)
{
    const int h = j / TT, tt = j % TT;
    const int g = lane >> 2, t = lane & 3;
    const int m0 = tt * 8 + 2 * t;
    const int n0 = tile * 32 + h * 16 + g;
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + (i & 1);
        const int n = n0 + ((i & 2) ? 8 : 0);
        if (m < p.M)
            p.Y[(size_t)m * p.N + n] = f32_to_bf16_bits(e[i]);
    }
}

// ------------------------------------------------------------------ producer
template <int TT, int GM, int P>
__device__ __forceinline__ void produce(const Params &p, const CUtensorMap *cmap,
                                        const CUtensorMap *smap, const CUtensorMap *xmap,
                                        uint8_t *ring, uint64_t *full, uint64_t *empty, int S0,
                                        int ns)
{
    using C = Cfg<TT, GM, P>;
    constexpr int R = C::kStages;
    const int spr = p.upr * C::kUS;   // stages per group row
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    prefetch_tensormap(cmap);
    prefetch_tensormap(smap);
    prefetch_tensormap(xmap);
    // box coordinates of run stage s: codes x (u64), group row y (tiles), first k
    auto coords = [&](int s, int &cx, int &sx, int &ty, int &k0) {
        const int a = S0 + s;
        const int gr = a / spr, ks = a - gr * spr;
        k0 = ks * C::kKS;
        cx = ks * (C::kCodeTile / 8);
        sx = (k0 / C::kG) * 8;
        ty = gr * kWarps;
    };
    auto issue_w = [&](int s) {
        int cx, sx, ty, k0;
        coords(s, cx, sx, ty, k0);
        uint8_t *st = ring + (size_t)(s % R) * C::kStage;
        uint64_t *bar = &full[s % R];
        mbar_arrive_expect_tx(bar, C::kTx);
        tma_load_2d(st + C::kX, cmap, cx, ty, bar, pol_w);
        tma_load_2d(st + C::kX + C::kCode, smap, sx, ty, bar, pol_w);
    };
    auto issue_x = [&](int s) {
        int cx, sx, ty, k0;
        coords(s, cx, sx, ty, k0);
        uint8_t *st = ring + (size_t)(s % R) * C::kStage;
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_2d(st + ch * C::kXBox, xmap, k0 + 64 * ch, 0, &full[s % R], pol_x);
    };
    const int first = min(R, ns);
    // Weights are not written by the previous kernel on the stream (the
    // caller's contract, unless early loads are off): the first stages fill,
    // and the stages after them are pulled into L2, while that kernel drains.
    if (p.early)
        for (int s = 0; s < first; ++s)
            issue_w(s);
    const int pf_end = min(ns, R + p.pf_stages);
    for (int s = R; s < pf_end; ++s) {
        int cx, sx, ty, k0;
        coords(s, cx, sx, ty, k0);
        prefetch_tensor_l2(cmap, cx, ty);
        prefetch_tensor_l2(smap, sx, ty);
    }
    pdl_wait();
    if (!p.early)
        for (int s = 0; s < first; ++s)
            issue_w(s);
    for (int s = 0; s < first; ++s)
        issue_x(s);
    int issued = first;
    for (int s = first; s < ns; ++s) {
        // stage s reuses the slot of stage s - R: its release is phase
        // (s / R - 1) of that slot's empty barrier
        if (!mbar_wait(&empty[s % R], (uint32_t)((s / R - 1) & 1), kWaitLimitNs)) {
            record_error(p.hdr, MXG_ERR_TIMEOUT, 140 + GM);
            break;
        }
        issue_w(s);
        issue_x(s);
        issued = s + 1;
    }
    // every copy this CTA issued has landed before it exits (the consumers
    // wait for them too; this only matters after a timeout)
    for (int s = max(0, issued - R); s < issued; ++s)
        if (!mbar_wait(&full[s % R], (uint32_t)((s / R) & 1), kWaitLimitNs))
            record_error(p.hdr, MXG_ERR_TIMEOUT, 150 + GM);
}

// ----------------------------------------------------------------- finisher
// Run by warp `warp` of a CTA whose segment of group row `gr` is cut (the
// row goes on in other CTAs' runs), with the warp's fragment in `sum`.  The
// CTA whose run holds the row's first unit finishes that segment last in its
// run: it adds the other contributors' fragments (in CTA order) to its own
// and writes bf16 Y.  Every other contributor (its segment is the first one
// of its run) publishes its fragment and bumps the tile's counter without
// waiting for anybody.
template <int TT>
__device__ __forceinline__ void finish_cut(const Params &p, float4 (&sum)[2 * TT], int c, int gr,
                                        int warp, int lane)
{
    constexpr int F = 2 * TT;
    const int tile = gr * kWarps + warp;
    const int c_first = cta_of_unit(p, gr * p.upr);
    float4 *mine = p.partial + ((size_t)c * kWarps + warp) * F * 32;
    if (c != c_first) {
#pragma unroll
        for (int j = 0; j < F; ++j)
            __stcg(mine + j * 32 + lane, sum[j]);
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            atomicAdd(&p.counters[tile], 1);
        }
        return;
    }
    const int c_last = cta_of_unit(p, (gr + 1) * p.upr - 1);
    if (lane == 0) {
        const unsigned long long t0 = global_ns();
        while (ld_acquire_gpu(&p.counters[tile]) < c_last - c_first) {
            if (global_ns() - t0 > kWaitLimitNs) {
                record_error(p.hdr, MXG_ERR_TIMEOUT, 120);
                break;
            }
            __nanosleep(64);
        }
    }
    __syncwarp();
    for (int cc = c_first + 1; cc <= c_last; ++cc) {
        const float4 *src = p.partial + ((size_t)cc * kWarps + warp) * F * 32;
#pragma unroll
        for (int j = 0; j < F; ++j) {
            const float4 f = __ldcg(src + j * 32 + lane);
            sum[j].x += f.x;
            sum[j].y += f.y;
            sum[j].z += f.z;
            sum[j].w += f.w;
        }
    }
#pragma unroll
    for (int j = 0; j < F; ++j)
        store_y4<TT>(p, tile, j, lane, sum[j]);
    __syncwarp();
    if (lane == 0)
        p.counters[tile] = 0;  // leave the counter zero for the next call
}

// ------------------------------------------------------------------- kernel
template <int TT, int GM, int P>
__global__ void __launch_bounds__(Cfg<TT, GM, P>::kThreads,
                                  Cfg<TT, GM, P>::kWPT == 1 && TT <= 2 ? 2 : 1)
    w4a16_stream_kernel(const __grid_constant__ CUtensorMap cmap,
                        const __grid_constant__ CUtensorMap smap,
                        const __grid_constant__ CUtensorMap xmap, const Params p)
{
    using C = Cfg<TT, GM, P>;
    constexpr int R = C::kStages;
    constexpr int F = C::kF;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled activation boxes
    uint8_t *ring = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + C::kBarOff);
    uint64_t *empty = full + R;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    const int c = blockIdx.x;
    const int U0 = run_start(p, c), U1 = run_start(p, c + 1);
    const int S0 = U0 * C::kUS;
    const int ns = (U1 - U0) * C::kUS;
    if (threadIdx.x == 0) {
        for (int s = 0; s < R; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);   // one warp of each tile takes a stage
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == C::kProducer) {
        if (lane == 0)
            produce<TT, GM, P>(p, &cmap, &smap, &xmap, ring, full, empty, S0, ns);
        return;
    }

    // ------------------------------------------------------------ consumers
    pdl_wait();   // Y, the counters and the partials may be in use before it
    const int g = lane >> 2, t = lane & 3;
    const int wt = warp % kWarps;        // this warp's tile in the column group
    const int parity = warp / kWarps;    // which stages of the run it takes
    // swizzled offsets of this lane's activations inside a 64-k box: row
    // 8 tt + g, bytes 32 j + 8 t of the row; the 16-byte chunk index is
    // XORed with the row modulo 8 by the 128-byte swizzle
    uint32_t xoff[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        xoff[j] = g * 128 + (((2 * j + (t >> 1)) ^ g) << 4) + 8 * (t & 1);

    constexpr uint32_t kOnes = 0x3F803F80u;  // bf16 pair (1, 1)
    float acc[2][TT][4], part[2][TT][4], xsum[TT][4];
    float parthi[P == 2 ? 2 : 1][TT][4];  // INT8: sums over the high-nibble plane
    bool ok = true;
    int s = 0;   // run stage
    for (int u = U0; u < U1;) {
        const int gr = u / p.upr;
        const int seg_begin = u;
        const int seg_end = min(U1, (gr + 1) * p.upr);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[h][tt][e] = 0.f;
        for (; u < seg_end; ++u) {
#pragma unroll
            for (int su = 0; su < C::kUS; ++su, ++s) {
                if (C::kWPT == 2 && (s & 1) != parity)
                    continue;   // the other warp of the tile takes this stage
                const int slot = s % R;
                if (!mbar_wait(&full[slot], (uint32_t)((s / R) & 1), ok ? kWaitLimitNs : 0)) {
                    if (ok && lane == 0)
                        record_error(p.hdr, MXG_ERR_TIMEOUT, 100 + GM);
                    ok = false;
                }
                const uint8_t *st = ring + (size_t)slot * C::kStage;
                const uint8_t *cs = st + C::kX + wt * C::kCodeTile;
                const uint8_t *ss = st + C::kX + C::kCode + wt * C::kScaleTile;
#pragma unroll
                for (int ch = 0; ch < C::kChunks; ++ch) {
                    // INT4: [half][lane][16 B]; INT8: [half][plane][lane][16 B]
                    const uint8_t *cp = cs + ch * 1024 * P + lane * 16;
                    const uint4 wl = lds128(cp);
                    const uint4 wh = lds128(cp + 512 * P);
                    const uint32_t w[2][4] = {{wl.x, wl.y, wl.z, wl.w}, {wh.x, wh.y, wh.z, wh.w}};
                    uint32_t whi[2][4] = {};
                    if constexpr (P == 2) {
                        const uint4 ul = lds128(cp + 512);
                        const uint4 uh = lds128(cp + 1536);
                        whi[0][0] = ul.x; whi[0][1] = ul.y; whi[0][2] = ul.z; whi[0][3] = ul.w;
                        whi[1][0] = uh.x; whi[1][1] = uh.y; whi[1][2] = uh.z; whi[1][3] = uh.w;
                    }
                    const uint8_t *xb = st + ch * C::kXBox;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // k16 step inside the unit (one warp) or the stage (two)
                        const int gstep = (C::kWPT == 1 ? su * C::kSteps : 0) + ch * 4 + j;
                        const bool first = (gstep % C::kEpi) == 0;
                        const bool last = ((gstep + 1) % C::kEpi) == 0;
                        uint2 xf[TT];
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt)
                            xf[tt] = lds64(xb + tt * 1024 + xoff[j]);
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt) {
                            // per token: the sum of the step's activations (an
                            // MMA with an all-ones weight tile)
                            if (first)
                                mma_bf16_16816_zero(xsum[tt], kOnes, kOnes, kOnes, kOnes, xf[tt].x,
                                                    xf[tt].y);
                            else
                                mma_bf16_16816(xsum[tt], kOnes, kOnes, kOnes, kOnes, xf[tt].x,
                                               xf[tt].y);
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t a0 = int4_pair_plus128<0>(w[h][j]);
                            const uint32_t a1 = int4_pair_plus128<4>(w[h][j]);
                            const uint32_t a2 = int4_pair_plus128<8>(w[h][j]);
                            const uint32_t a3 = int4_pair_plus128<12>(w[h][j]);
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt) {
                                if (first)
                                    mma_bf16_16816_zero(part[h][tt], a0, a1, a2, a3, xf[tt].x,
                                                        xf[tt].y);
                                else
                                    mma_bf16_16816(part[h][tt], a0, a1, a2, a3, xf[tt].x,
                                                   xf[tt].y);
                            }
                            if constexpr (P == 2) {
                                const uint32_t b0 = int4_pair_plus128<0>(whi[h][j]);
                                const uint32_t b1 = int4_pair_plus128<4>(whi[h][j]);
                                const uint32_t b2 = int4_pair_plus128<8>(whi[h][j]);
                                const uint32_t b3 = int4_pair_plus128<12>(whi[h][j]);
#pragma unroll
                                for (int tt = 0; tt < TT; ++tt) {
                                    if (first)
                                        mma_bf16_16816_zero(parthi[h][tt], b0, b1, b2, b3,
                                                            xf[tt].x, xf[tt].y);
                                    else
                                        mma_bf16_16816(parthi[h][tt], b0, b1, b2, b3, xf[tt].x,
                                                       xf[tt].y);
                                }
                            }
                        }
                        if (last) {
                            // end of a scale group: the MMAs summed (128 + q) * x,
                            // so acc += (part - 136 * sum(x)) * scale, in fp32
                            const int gi = C::kScaleGroups > 1 ? (ch * 4 + j) / C::kStepsPerGroup
                                                               : 0;
                            const uint2 sv = lds64(ss + gi * 64 + g * 8);
                            const float2 s01 =
                                __half22float2(*reinterpret_cast<const __half2 *>(&sv.x));
                            const float2 s23 =
                                __half22float2(*reinterpret_cast<const __half2 *>(&sv.y));
                            const float sc[2][2] = {{s01.x, s01.y}, {s23.x, s23.y}};
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        // outputs e and e ^ 2 are rows g, g + 8 of
                                        // token 2t + (e & 1)
                                        float v;
                                        if constexpr (P == 2) {
                                            // INT8 q = 16 hi + lo: the planes summed
                                            // (128 + hi) x and (128 + lo) x, so
                                            // sum (q - 128) x = 16 Phi + Plo - 2304 sum(x)
                                            v = fmaf(16.f, parthi[h][tt][e], part[h][tt][e]);
                                            v = fmaf(-2304.f, xsum[tt][e & 1], v);
                                        } else {
                                            v = fmaf(-136.f, xsum[tt][e & 1], part[h][tt][e]);
                                        }
                                        acc[h][tt][e] = fmaf(v, sc[h][e >> 1], acc[h][tt][e]);
                                    }
                        }
                    }
                }
                // every lane's reads of the stage have returned (their values
                // are consumed above): release it to the producer
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[slot]);
            }
        }

        // ---- end of the segment: this warp's tile of group row gr
        float4 sum[F];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
                sum[h * TT + tt] =
                    make_float4(acc[h][tt][0], acc[h][tt][1], acc[h][tt][2], acc[h][tt][3]);
        if constexpr (C::kWPT == 2) {
            // the tile's second warp hands its fragment to the first (a named
            // barrier per tile: ids 1..8, the tile's two warps)
            float4 *xch = reinterpret_cast<float4 *>(ring + C::kXchgOff) + wt * F * 32;
            if (parity == 1)
#pragma unroll
                for (int j = 0; j < F; ++j)
                    xch[j * 32 + lane] = sum[j];
            named_bar_sync(1 + wt, 64);
            if (parity == 0)
#pragma unroll
                for (int j = 0; j < F; ++j) {
                    const float4 v = xch[j * 32 + lane];
                    sum[j].x += v.x;
                    sum[j].y += v.y;
                    sum[j].z += v.z;
                    sum[j].w += v.w;
                }
            named_bar_sync(1 + wt, 64);   // read before the next segment's write
            if (parity == 1)
                continue;
        }
        const int tile = gr * kWarps + wt;
        if (tile < p.ntiles) {
            const bool whole = seg_begin == gr * p.upr && seg_end == (gr + 1) * p.upr;
            if (whole) {
#pragma unroll
                for (int j = 0; j < F; ++j)
                    store_y4<TT>(p, tile, j, lane, sum[j]);
            } else {
                finish_cut<TT>(p, sum, c, gr, wt, lane);
            }
        }
    }
}

template <int TT, int GM, int P>
const void *kernel_ptr()
{
    return reinterpret_cast<const void *>(&w4a16_stream_kernel<TT, GM, P>);
}

// variant = group mode (INT4) or 3 + group mode (INT8)
const void *select_kernel(int tt, int variant)
{
#define MXG_CASE(T, V) \
    if (tt == T && variant == V) return kernel_ptr<T, V % 3, V / 3 + 1>();
    MXG_CASE(1, 0) MXG_CASE(1, 1) MXG_CASE(1, 2) MXG_CASE(1, 3) MXG_CASE(1, 4) MXG_CASE(1, 5)
    MXG_CASE(2, 0) MXG_CASE(2, 1) MXG_CASE(2, 2) MXG_CASE(2, 3) MXG_CASE(2, 4) MXG_CASE(2, 5)
    MXG_CASE(3, 0) MXG_CASE(3, 1) MXG_CASE(3, 2) MXG_CASE(3, 3) MXG_CASE(3, 4) MXG_CASE(3, 5)
    MXG_CASE(4, 0) MXG_CASE(4, 1) MXG_CASE(4, 2) MXG_CASE(4, 3) MXG_CASE(4, 4) MXG_CASE(4, 5)
#undef MXG_CASE
    return nullptr;
}

template <int TT>
void cfg_of(int variant, size_t *smem, int *us, int *ks, int *code_tile, int *g, int *threads)
{
#define MXG_CFG(V)                                         \
    if (variant == V) {                                    \
        using C = Cfg<TT, V % 3, V / 3 + 1>;               \
        *smem = C::kSmem;                                  \
        *us = C::kUS;                                      \
        *ks = C::kKS;                                      \
        *code_tile = C::kCodeTile;                         \
        *g = C::kG;                                        \
        *threads = C::kThreads;                            \
        return;                                            \
    }
    MXG_CFG(0) MXG_CFG(1) MXG_CFG(2) MXG_CFG(3) MXG_CFG(4) MXG_CFG(5)
#undef MXG_CFG
}

struct VariantCfg {
    size_t smem;
    int us, ks, code_tile, g, threads;
};

VariantCfg variant_cfg(int tt, int variant)
{
    VariantCfg v{};
    switch (tt) {
    case 1: cfg_of<1>(variant, &v.smem, &v.us, &v.ks, &v.code_tile, &v.g, &v.threads); break;
    case 2: cfg_of<2>(variant, &v.smem, &v.us, &v.ks, &v.code_tile, &v.g, &v.threads); break;
    case 3: cfg_of<3>(variant, &v.smem, &v.us, &v.ks, &v.code_tile, &v.g, &v.threads); break;
    default: cfg_of<4>(variant, &v.smem, &v.us, &v.ks, &v.code_tile, &v.g, &v.threads); break;
    }
    return v;
}

int group_mode(int G)
{
    return G == 128 ? 0 : (G == 64 ? 1 : 2);
}

// bits: 4 (INT4) or 8 (INT8, two code planes)
bool plan_stream(int device, int M, int N, int K, int G, int bits, StreamPlan *plan)
{
    if (M < 1 || M > 32 || N % 64 != 0 || K % 64 != 0 || K % G != 0)
        return false;
    if (device < 0 || device >= kMaxDeviceCache)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    pl.variant = (bits == 8 ? 3 : 0) + group_mode(G);
    const VariantCfg vc = variant_cfg(pl.tt, pl.variant);
    pl.warps_per_cta = vc.threads / 32;
    pl.smem = vc.smem;
    if ((int)pl.smem > di.smem_optin)
        return false;
    const int unit_k = vc.us * vc.ks;
    if (K % unit_k != 0)
        return false;
    pl.upt = K / unit_k;                      // units per group row
    const int ngroups = (N / 32 + kWarps - 1) / kWarps;
    pl.ntiles = ngroups * kWarps;             // arrival counters (one per tile slot)
    if ((size_t)pl.ntiles > kMaxCounters)
        return false;
    pl.units = (long long)ngroups * pl.upt;
    if (pl.units > (1LL << 30))
        return false;
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return false;
    // every CTA of the grid must be resident at once (a cut row's finishing
    // CTA waits for the others); function attributes and occupancy are per
    // device: cached per device
    static std::atomic<int> occ_cache[kMaxDeviceCache][4][6];
    std::atomic<int> &occ_slot = occ_cache[device][pl.tt - 1][pl.variant];
    int occ = occ_slot.load(std::memory_order_acquire);
    if (occ == 0) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) !=
            cudaSuccess)
            return false;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, vc.threads, pl.smem) !=
                cudaSuccess ||
            o < 1)
            return false;
        occ = o;
        occ_slot.store(occ, std::memory_order_release);
    }
    // one CTA per SM (a second resident CTA, where it fits, is left to the
    // next GEMM on the stream), no run shorter than one unit
    pl.Wt = (int)std::max<long long>(1, std::min<long long>(di.sms, pl.units));
    pl.grid = pl.Wt;
    pl.partial_bytes = (size_t)pl.Wt * kWarps * (2 * pl.tt * 32) * sizeof(float4);
    *plan = pl;
    return true;
}

}  // namespace

bool plan_w4a16_stream(int device, int M, int N, int K, int G, StreamPlan *plan)
{
    return plan_stream(device, M, N, K, G, 4, plan);
}

bool plan_w8a16_stream(int device, int M, int N, int K, int G, StreamPlan *plan)
{
    return plan_stream(device, M, N, K, G, 8, plan);
}

cudaError_t launch_w4a16_stream(const StreamPlan &pl, const void *X, const void *packed, int M,
                                int N, int K, int G, void *Y, void *workspace, bool early,
                                cudaStream_t stream)
{
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return cudaErrorInvalidValue;
    const VariantCfg vc = variant_cfg(pl.tt, pl.variant);
    const int planes = pl.variant >= 3 ? 2 : 1;
    const uint8_t *codes = static_cast<const uint8_t *>(packed);
    // codes take half a byte per weight (INT4) or one byte in two planes (INT8)
    const uint8_t *scales = codes + (size_t)N * K / 2 * planes;
    const uint64_t tiles = (uint64_t)N / 32;
    alignas(64) CUtensorMap cmap, smap, xmap;
    // codes: one row of 16 * K * planes bytes per n32 tile, in 8-byte elements
    // scales: one row of 64 * K / G bytes per tile
    // X: bf16 [M][K], boxes of 64 k x 8 TT rows with 128-byte swizzle
    if (!encode_tensor_map_2d(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT64, codes,
                              (uint64_t)K * 2 * planes, tiles, (uint64_t)K * 16 * planes,
                              (uint32_t)(vc.code_tile / 8), kWarps, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tensor_map_2d(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT64, scales,
                              (uint64_t)(K / G) * 8, tiles, (uint64_t)(K / G) * 64,
                              (uint32_t)(vc.ks >= G ? vc.ks / G : 1) * 8, kWarps,
                              CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K,
                              (uint64_t)M, (uint64_t)K * 2, 64, (uint32_t)(8 * pl.tt),
                              CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const WorkspaceMap wm = make_workspace_map(pl.ntiles, pl.partial_bytes);
    Params p{};
    p.Y = static_cast<uint16_t *>(Y);
    p.early = early ? 1 : 0;
    p.pf_stages = MXG_STREAM_PF_STAGES;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wm.counters_off);
    p.partial = reinterpret_cast<float4 *>(static_cast<uint8_t *>(workspace) + wm.partial_off);
    p.M = M;
    p.N = N;
    p.ntiles = N / 32;
    p.upr = pl.upt;
    p.q = (int)(pl.units / pl.Wt);
    p.r = (int)(pl.units % pl.Wt);
    void *args[] = {&cmap, &smap, &xmap, &p};
    return launch_pdl(fn, dim3(pl.grid), dim3(vc.threads), pl.smem, stream, args);
}

}  // namespace mxg
