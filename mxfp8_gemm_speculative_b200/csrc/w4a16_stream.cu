// INT4 W4A16 weight-streaming GEMM for small M (decode / MTP verify chunks).
//
// At M <= 32 the layer reads each weight byte once and does 2*M flops per
// weight: it is bound by HBM bytes of W, and the design is about keeping
// enough weight bytes in flight on every SM while the decode and the MMAs
// run behind them, with few, large copies.
//
//  * Columns are taken eight n32 tiles (256 columns) at a time, a "column
//    group" of the re-packed layout (common.cuh), in which the codes of a
//    group for 128 rows of K are one contiguous 16 KB range and their scales
//    one contiguous range.  The stream of a group row is cut into units of
//    128 rows (one pipeline stage).  With fewer group rows than SMs (the
//    decode layers), every row is split into S equal pieces, one CTA each,
//    so every CTA has one segment and the pieces of a row end together;
//    with more rows, every CTA of a one-CTA-per-SM grid takes one contiguous
//    run of units across rows (stream-K).  Either way all SMs stream about
//    the same number of bytes.
//  * One producer thread fills a CTA-wide ring of stages with two 1-D bulk
//    copies per stage (codes, scales), completion on an mbarrier per stage;
//    the consumers release a stage through a second mbarrier.  Weights are
//    marked evict-first in L2.
//  * The activations X of the CTA's run (the k ranges of its at most two
//    group-row segments, or all of K when the run spans more rows) are
//    copied into shared memory once by the consumer warps' own loads (after
//    an L2 prefetch issued at entry), as fp16 values scaled per (scale
//    group, token) by a power of two 2^-e, with a table of the sums of the
//    stored values and 2^e.  When they do not fit beside the ring (wide
//    token tiles, long runs) every stage carries its bf16 activations (2-D
//    tensor-map boxes with 128-byte swizzle) and every warp forms the sums
//    with all-ones MMAs.
//  * Consumer warps own tiles: warp w (and, for M <= 16, warp w + 8, the two
//    taking alternate stages) owns tile w of the group for the whole K range
//    of the CTA's segment, so no warp reduces against another except the
//    pair at a segment end.  The tensor cores run m16n8k16 MMAs where the
//    weights are the 16-row operand and the tokens the 8-column operand
//    ("swap AB").  The decode is integer logic only, and that logic is the
//    loop's busiest pipe: on fp16 windows four mask-and-ors and one shift
//    turn a 32-bit word of codes into the pairs 1024 + q (rows g of the
//    fragment) and 1024 + 16 q (rows g + 8); on bf16 stages four
//    mask-and-ors and three shifts give 128 + q.  A zero-initialised partial
//    sum per scale group is folded in fp32 as acc += (part - c * activation
//    sum) * scale, with c and a factor 1/16 per fragment row, so weights
//    are never rounded (every product is exact in fp32).
//  * A group row cut between CTAs: every contributor publishes its fragment
//    and counts itself in the tile's counter; the last one to arrive adds
//    all fragments in CTA order (deterministic) and writes bf16 Y, so no CTA
//    waits for another.  A group row inside one run is written directly.
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

#ifndef MXG_STREAM_PF_STAGES
#define MXG_STREAM_PF_STAGES 8
#endif
#ifndef MXG_STREAM_MAX_RING_KB
#define MXG_STREAM_MAX_RING_KB 200
#endif
#ifndef MXG_STREAM_X_PREFETCH
#define MXG_STREAM_X_PREFETCH 1
#endif
#ifndef MXG_STREAM_EARLY_MAX
#define MXG_STREAM_EARLY_MAX 64
#endif
#ifndef MXG_STREAM_WPT2_MAX_TT
#define MXG_STREAM_WPT2_MAX_TT 2
#endif

constexpr int kWarps = 8;          // n32 tiles of a column group
constexpr int kKS = 128;           // rows of K per stage (= per stream-K unit)
constexpr int kChunks = kKS / 64;  // k64 chunks per stage
constexpr int kXPad = 16;          // bf16 columns of padding per resident activation row
constexpr int kMaxSmem = 227 * 1024;

// Consumer warps per tile: two for narrow token tiles (each takes every
// other stage of the run, so a warp has two stages' time for the latency
// chain of one), one for wide ones (whose registers allow no more warps).
template <int TT>
struct Wpt {
    static constexpr int value = TT <= MXG_STREAM_WPT2_MAX_TT ? 2 : 1;
};

// Group modes: 0 -> G = 128, 1 -> G = 64, 2 -> G = 32.  P code planes: 1 for
// INT4; 2 for INT8 (low and high nibbles, each in the INT4 layout).  XR: the
// activations are resident for the whole run (1) or carried by every stage (0).
template <int TT, int GM, int P, int XR>
struct Cfg {
    static constexpr int kWPT = Wpt<TT>::value;
    static constexpr int kConsumers = kWarps * kWPT;
    static constexpr int kThreads = (kConsumers + 1) * 32;         // + the producer warp
    static constexpr int kProducer = kConsumers;                   // its warp index
    static constexpr int kG = GM == 0 ? 128 : (GM == 1 ? 64 : 32);
    static constexpr int kStepsPerGroup = kG / 16;
    static constexpr int kGroupsPerStage = kKS / kG;
    static constexpr int kXBox = 128 * 8 * TT;                     // 64 k x 8TT rows of bf16
    static constexpr int kX = XR ? 0 : kChunks * kXBox;           // staged activations
    static constexpr int kCodeMax = kChunks * kWarps * 1024 * P;   // codes of a full group
    static constexpr int kScaleMax = kGroupsPerStage * kWarps * 64;
    static constexpr int kStage = XR ? (kX + kCodeMax + kScaleMax + 127) / 128 * 128
                                     : (kX + kCodeMax + kScaleMax + 1023) / 1024 * 1024;
    static constexpr int kF = 2 * TT;                              // float4 per lane fragment
    static constexpr int kXchg = kWPT == 2 ? kWarps * kF * 32 * 16 : 0;
};

struct Params {
    const uint16_t *X;       // bf16 [M][K]
    const uint8_t *codes;    // re-packed codes (column-group layout)
    const uint8_t *scales;   // re-packed scales
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [column groups * 8]
    float4 *partial;         // [ctas][2 slots][8 tiles][2*TT][32]: a CTA's fragments of its cut rows
    int frag;                // float4 per fragment: 2 * TT * 32
    int M, N, K;
    int ntiles;              // N / 32
    int upr;                 // units (stages) per group row: ceil(K / 128)
    int q, r;                // stream-K: units = q * ctas + r: CTAs below r run q + 1 units
    int S;                   // pieces per group row (row split), or 0 (stream-K)
    int R;                   // ring stages
    int x_off, xs_off, xchg_off, bar_off;   // shared-memory regions (bytes from the base)
    int early;               // load the first weights before waiting for the previous kernel
    int pf_stages;           // stages after the ring warmed in L2 at entry
};

// First unit of CTA c's run: piece c % S of row c / S (row split), or
// stream-K's c-th run (CTAs below r run q + 1 units, the rest q).  c may be
// the CTA count (the end of the last run).
__host__ __device__ __forceinline__ int run_start(int q, int r, int S, int upr, int c)
{
    if (S > 0)
        return (c / S) * upr + (c % S) * upr / S;
    return c * q + (c < r ? c : r);
}

// The CTA whose run contains unit u.
__device__ __forceinline__ int cta_of_unit(const Params &p, int u)
{
    if (p.S > 0) {
        const int row = u / p.upr, o = u - row * p.upr;
        int i = (o * p.S) / p.upr;   // piece i covers [i * upr / S, (i + 1) * upr / S)
        while (i + 1 < p.S && (i + 1) * p.upr / p.S <= o)
            ++i;
        while (i > 0 && i * p.upr / p.S > o)
            --i;
        return row * p.S + i;
    }
    const int big = p.r * (p.q + 1);   // units covered by the longer runs
    return u < big ? u / (p.q + 1) : p.r + (u - big) / p.q;
}

// The resident activation windows of the run [U0, U1): one per segment
// (group row) when the run touches at most two rows and the two ranges are
// shorter than K together, else one window [0, K) for every segment.
struct XWindows {
    int n;                   // windows
    int klo[2], cols[2];     // k range of each window
    bool fullk;
};

__host__ __device__ inline XWindows x_windows(int U0, int U1, int upr, int K)
{
    XWindows w{};
    const int row0 = U0 / upr, row1 = (U1 - 1) / upr;
    int cols = 0;
    if (row1 - row0 <= 1) {
        for (int rr = row0, i = 0; rr <= row1; ++rr, ++i) {
            const int a = (U0 > rr * upr ? U0 : rr * upr) - rr * upr;
            const int b = (U1 < (rr + 1) * upr ? U1 : (rr + 1) * upr) - rr * upr;
            w.klo[i] = a * kKS;
            w.cols[i] = (b * kKS < K ? b * kKS : K) - a * kKS;
            cols += w.cols[i];
        }
        w.n = row1 - row0 + 1;
    }
    if (row1 - row0 > 1 || cols >= K) {
        w.n = 1;
        w.klo[0] = 0;
        w.cols[0] = K;
        w.fullk = true;
    }
    return w;
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
template <int TT, int GM, int P, int XR>
__device__ __forceinline__ void produce(const Params &p, const CUtensorMap *xmap, uint8_t *smem,
                                        uint64_t *full, uint64_t *empty, int U0,
                                        int ns)
{
    using C = Cfg<TT, GM, P, XR>;
    const int R = p.R;
    const int K = p.K;
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    if (!XR)
        prefetch_tensormap(xmap);
    // source ranges of run stage s
    struct Src {
        const uint8_t *codes, *scales;
        uint32_t code_bytes, scale_bytes;
        int k0;
    };
    auto source = [&](int s) {
        const int a = U0 + s;
        const int gr = a / p.upr, ks = a - gr * p.upr;
        const int nt = group_tiles(gr, p.ntiles);
        Src src;
        src.k0 = ks * kKS;
        const int nch = K - src.k0 >= kKS ? kChunks : (K - src.k0) / 64;
        const int ngs = (nch * 64 + C::kG - 1) / C::kG;
        src.codes = p.codes + (size_t)gr * kWarps * 16 * K * P + (size_t)ks * kChunks * nt * 1024 * P;
        src.scales = p.scales + (size_t)gr * kWarps * (K / C::kG) * 64 +
                     (size_t)(src.k0 / C::kG) * nt * 64;
        src.code_bytes = (uint32_t)(nch * nt * 1024 * P);
        src.scale_bytes = (uint32_t)(ngs * nt * 64);
        return src;
    };
    auto issue_w = [&](int s) {
        const Src src = source(s);
        uint8_t *st = smem + (size_t)(s % R) * C::kStage;
        uint64_t *bar = &full[s % R];
        mbar_arrive_expect_tx(bar, src.code_bytes + src.scale_bytes + (XR ? 0 : C::kX));
        bulk_g2s(st + C::kX, src.codes, src.code_bytes, bar, pol_w);
        bulk_g2s(st + C::kX + C::kCodeMax, src.scales, src.scale_bytes, bar, pol_w);
    };
    auto issue_x = [&](int s) {   // staged activations of stage s
        const Src src = source(s);
        uint8_t *st = smem + (size_t)(s % R) * C::kStage;
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch)
            tma_load_2d(st + ch * C::kXBox, xmap, src.k0 + 64 * ch, 0, &full[s % R], pol_x);
    };
    const int first = min(R, ns);
    if (XR && MXG_STREAM_X_PREFETCH) {
        // the run's activations are pulled into L2 ahead of the weights, so
        // the consumers' loads of them after the wait do not queue behind
        // the ring (a hint: L2 is coherent, data written later is not hidden)
        const XWindows xw = x_windows(U0, U0 + ns, p.upr, K);
        const int rows = min(p.M, 8 * TT);
        for (int w = 0; w < xw.n; ++w)
            for (int m = 0; m < rows; ++m)
                prefetch_l2(p.X + (size_t)m * K + xw.klo[w], (uint32_t)xw.cols[w] * 2);
    }
    // Weights are not written by the previous kernel on the stream (the
    // caller's contract, unless early loads are off): the first stages fill,
    // and the stages after them are pulled into L2, while that kernel drains.
    const int early_n = p.early ? min(first, MXG_STREAM_EARLY_MAX) : 0;
    for (int s = 0; s < early_n; ++s)
        issue_w(s);
    const int pf_end = min(ns, R + p.pf_stages);
    for (int s = R; s < pf_end; ++s) {
        const Src src = source(s);
        prefetch_l2(src.codes, src.code_bytes);
    }
    pdl_wait();
    for (int s = early_n; s < first; ++s)
        issue_w(s);
    if (!XR)
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
        if (!XR)
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
// Fragment slot of CTA cc for group row gr: 0 when gr is the first row of its
// run, else 1 (a cut row can only be the first or the last segment of a run).
__device__ __forceinline__ float4 *partial_of(const Params &p, int cc, int gr, int wt)
{
    const int row0 = run_start(p.q, p.r, p.S, p.upr, cc) / p.upr;
    return p.partial + ((size_t)(cc * 2 + (row0 == gr ? 0 : 1)) * kWarps + wt) * (size_t)p.frag;
}

// Run by the warp owning tile slot `wt` of a CTA whose segment of group row
// `gr` is cut (the row goes on in other CTAs' runs), with the warp's fragment
// in `sum`.  Every contributor publishes its fragment in its own slot and
// counts itself in the tile's counter; the one that arrives last adds all the
// row's fragments in CTA order (so the sum does not depend on which CTA ends
// last) and writes bf16 Y.  No CTA waits for another.
template <int TT>
__device__ __forceinline__ void finish_cut(const Params &p, float4 (&sum)[2 * TT], int c, int gr,
                                           int wt, int lane)
{
    constexpr int F = 2 * TT;
    constexpr int kB = F >= 8 ? 1 : 8 / F;   // contributors whose fragments load together
    const int tile = gr * kWarps + wt;
    const int c_first = cta_of_unit(p, gr * p.upr);
    const int c_last = cta_of_unit(p, (gr + 1) * p.upr - 1);
    float4 *mine = partial_of(p, c, gr, wt);
#pragma unroll
    for (int j = 0; j < F; ++j)
        __stcg(mine + j * 32 + lane, sum[j]);
    // every lane's stores are performed at GPU scope before the warp counts
    // itself (a release by one lane orders only that lane's own accesses)
    __threadfence();
    __syncwarp();
    int old = 0;
    if (lane == 0)
        old = atomic_add_acq_rel(&p.counters[tile], 1);
    old = __shfl_sync(0xFFFFFFFFu, old, 0);
    if (old != c_last - c_first)
        return;
    // the last contributor: its count saw every other contributor's; every
    // lane fences before reading their fragments
    __threadfence();
    float4 tot[F];
#pragma unroll
    for (int j = 0; j < F; ++j)
        tot[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = c_first; c0 <= c_last; c0 += kB) {
        float4 f[kB][F];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int cc = c0 + u;
            if (cc <= c_last && cc != c) {
                const float4 *src = partial_of(p, cc, gr, wt);
#pragma unroll
                for (int j = 0; j < F; ++j)
                    f[u][j] = __ldcg(src + j * 32 + lane);
            } else {
#pragma unroll
                for (int j = 0; j < F; ++j)
                    f[u][j] = sum[j];
            }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u)
            if (c0 + u <= c_last)
#pragma unroll
                for (int j = 0; j < F; ++j) {
                    tot[j].x += f[u][j].x;
                    tot[j].y += f[u][j].y;
                    tot[j].z += f[u][j].z;
                    tot[j].w += f[u][j].w;
                }
    }
#pragma unroll
    for (int j = 0; j < F; ++j)
        store_y4<TT>(p, tile, j, lane, tot[j]);
    if (lane == 0)
        p.counters[tile] = 0;  // leave the counter zero for the next call
}

// ------------------------------------------------------------------- kernel
template <int TT, int GM, int P, int XR, int MX>
__global__ void __launch_bounds__(Cfg<TT, GM, P, XR>::kThreads, 1)
    w4a16_stream_kernel(const __grid_constant__ CUtensorMap xmap, const Params p)
{
    using C = Cfg<TT, GM, P, XR>;
    constexpr int F = C::kF;
    constexpr uint32_t kOnes = 0x3F803F80u;  // bf16 pair (1, 1)
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled activation boxes
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int R = p.R;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    uint64_t *empty = full + R;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    const int c = blockIdx.x;
    const int U0 = run_start(p.q, p.r, p.S, p.upr, c), U1 = run_start(p.q, p.r, p.S, p.upr, c + 1);
    const int ns = U1 - U0;
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
            produce<TT, GM, P, XR>(p, &xmap, smem, full, empty, U0, ns);
        return;
    }

    // ------------------------------------------------------------ consumers
    pdl_wait();   // Y, the counters and the partials may be in use before it
    const int g = lane >> 2, t = lane & 3;
    const int wt = warp % kWarps;        // this warp's tile in the column group
    const int parity = warp / kWarps;    // which stages of the run it takes
    const uint32_t sb = smem_u32(smem);  // shared-window address of the base
    bool ok = true;

    // resident activations: windows of fp16 values, and per (group of the
    // windows, token) the sum of the stored values and their power-of-two
    // factor (table [group][8 TT tokens] of float2)
    XWindows xw{};
    if constexpr (XR != 0) {
        xw = x_windows(U0, U1, p.upr, p.K);
        // One pass: every (group, token) segment of G activations is read by
        // a team of G / 8 lanes, 16 bytes each (the consumers' own loads: a
        // bulk copy would queue behind the ring's weight copies, which the
        // producer issued before the wait and which may take microseconds to
        // drain on a CTA that started late).  The team scales the segment by
        // the power of two 2^-e that brings its largest magnitude into
        // [2^14, 2^15), so every bf16 value becomes an fp16 value exactly
        // (unless it is 2^28 times smaller than the largest one), stores it,
        // and enters the sum of the stored values and 2^e in the table.
        constexpr int L = C::kG / 8;   // lanes per segment
        constexpr int kTeams = C::kConsumers * (32 / L);
        const int rows = min(p.M, 8 * TT);
        const int ngr0 = xw.cols[0] / C::kG;
        const int ngr1 = xw.n > 1 ? xw.cols[1] / C::kG : 0;
        const int nseg0 = ngr0 * rows, nseg = (ngr0 + ngr1) * rows;
        const uint32_t stride0 = (xw.cols[0] + kXPad) * 2;
        const uint32_t stride1 = (xw.n > 1 ? xw.cols[1] + kXPad : 0) * 2;
        const int team = warp * (32 / L) + lane / L, piece = lane % L;
        for (int i0 = 0; i0 < nseg; i0 += 4 * kTeams) {   // the same trip count in every lane
            uint4 v[4];
            uint32_t dst[4];
            int ent[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int sgi = i0 + u * kTeams + team;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                dst[u] = 0;
                ent[u] = -1;
                if (sgi < nseg) {
                    const int w = sgi < nseg0 ? 0 : 1;
                    const int loc = sgi - (w ? nseg0 : 0);
                    const int gl = loc / rows, m = loc - gl * rows;
                    const int k = (w ? xw.klo[1] : xw.klo[0]) + gl * C::kG + piece * 8;
                    v[u] = __ldcg(reinterpret_cast<const uint4 *>(p.X + (size_t)m * p.K + k));
                    dst[u] = p.x_off + (w ? 8 * TT * stride0 : 0) + m * (w ? stride1 : stride0) +
                             (gl * C::kG + piece * 8) * 2;
                    ent[u] = ((w ? ngr0 : 0) + gl) * 8 * TT + m;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t b[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                float f[8];
                float mx = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    f[2 * i] = __uint_as_float(b[i] << 16);
                    f[2 * i + 1] = __uint_as_float(b[i] & 0xFFFF0000u);
                    mx = fmaxf(mx, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
                }
#pragma unroll
                for (int o = L / 2; o >= 1; o >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                // e = exponent(mx) - 14, within [-126, 126]; zeros and
                // non-finite segments are stored unscaled
                const int E = (int)((__float_as_uint(mx) >> 23) & 0xFF);
                int e = 0;
                if (mx > 0.f && E != 0xFF)
                    e = max(-126, min(126, E - 127 - 14));
                const float down = __uint_as_float((uint32_t)(127 - e) << 23);
                uint32_t h[4];
                float sum = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 hv = __floats2half2_rn(f[2 * i] * down, f[2 * i + 1] * down);
                    h[i] = *reinterpret_cast<const uint32_t *>(&hv);
                    const float2 back = __half22float2(hv);
                    sum += back.x + back.y;
                }
#pragma unroll
                for (int o = L / 2; o >= 1; o >>= 1)
                    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
                if (ent[u] >= 0) {
                    *reinterpret_cast<uint4 *>(smem + dst[u]) = make_uint4(h[0], h[1], h[2], h[3]);
                    if (piece == 0)
                        *reinterpret_cast<float2 *>(smem + p.xs_off + ent[u] * 8) =
                            make_float2(sum, __uint_as_float((uint32_t)(127 + e) << 23));
                }
            }
        }
        named_bar_sync(9, C::kConsumers * 32);   // the windows and the table are complete
    }
    // swizzled offsets of this lane's activations inside a staged 64-k box:
    // row 8 tt + g, bytes 32 j + 8 t of the row; the 16-byte chunk index is
    // XORed with the row modulo 8 by the 128-byte swizzle
    uint32_t xoff[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        xoff[j] = g * 128 + (((2 * j + (t >> 1)) ^ g) << 4) + 8 * (t & 1);

    float acc[2][TT][4], part[2][TT][4], xsum[TT][4];
    float parthi[P == 2 ? 2 : 1][TT][4];  // INT8: sums over the high-nibble plane
    // this warp's stages of the run: s = parity, parity + WPT, ...; the ring
    // slot and phase of stage s follow it incrementally
    int s = parity;
    int slot = parity;
    uint32_t phase = 0;
    int seg = 0;
    for (int seg_begin = U0; seg_begin < U1; ++seg) {
        const int gr = seg_begin / p.upr;
        const int seg_end = min(U1, (gr + 1) * p.upr);
        const int nt = group_tiles(gr, p.ntiles);
        const bool live = wt < nt;           // a last group may hold fewer tiles
        // resident window of this segment: the shared-memory address of this
        // lane's token row at k = 0 of the row and the stride between token
        // rows; the table row of the segment's k = 0
        uint32_t xrow = 0, xstride = 0;
        int xg0 = 0;
        if constexpr (XR != 0) {
            const int w = xw.fullk ? 0 : seg;
            const int xklo = w ? xw.klo[1] : xw.klo[0];
            const uint32_t stride0 = (xw.cols[0] + kXPad) * 2;
            xstride = ((w ? xw.cols[1] : xw.cols[0]) + kXPad) * 2;
            xrow = sb + p.x_off + (w ? 8 * TT * stride0 : 0) + g * xstride + 8 * t - xklo * 2;
            xg0 = (w ? xw.cols[0] / C::kG : 0) - xklo / C::kG;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[h][tt][e] = 0.f;
        for (; U0 + s < seg_end; s += C::kWPT) {
            const int k0 = (U0 + s - gr * p.upr) * kKS;   // first row of K of the stage
            if (!mbar_wait(&full[slot], phase, ok ? kWaitLimitNs : 0)) {
                if (ok && lane == 0)
                    record_error(p.hdr, MXG_ERR_TIMEOUT, 100 + GM);
                ok = false;
            }
            const uint32_t st = sb + slot * C::kStage;
            const uint32_t cs = st + C::kX + wt * 1024 * P + lane * 16;
            const uint32_t ss = st + C::kX + C::kCodeMax + wt * 64 + g * 8;
            if (MX && live) {
                // MXFP8: per k64 chunk and tile, [half][pair of steps][lane][16 B];
                // step j of the lane holds (row na, nb) x k0 .. k0 + 3 as
                // E4M3 pairs (na k0 k0+1 | nb k0 k0+1), (na k0+2 k0+3 | nb ...),
                // which the hardware converts to f16 pairs exactly; a partial
                // per 32-k block is scaled by 2^(E - 127) and the window factor
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) {
                    if (ch > 0 && k0 + 64 * ch >= p.K)
                        break;   // the last stage of a row may hold one chunk
                    const uint32_t cp = cs + ch * nt * 2048;
                    uint4 wq[2][2];
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int q = 0; q < 2; ++q)
                            wq[h][q] = lds128a(cp + h * 1024 + q * 512);
                    const uint32_t xk = xrow + (k0 + 64 * ch) * 2;
                    // window factors of the chunk (table group = chunk)
                    float2 fx[TT];
                    {
                        const uint32_t xa =
                            sb + p.xs_off + ((xg0 + k0 / C::kG + ch) * 8 * TT + 2 * t) * 8;
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt) {
                            const uint4 tv = lds128a(xa + tt * 64);
                            fx[tt] = make_float2(__uint_as_float(tv.y), __uint_as_float(tv.w));
                        }
                    }
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        // E8M0 of rows na, nb (half 0) and na, nb (half 1)
                        const uint32_t s4 = lds32a(st + C::kX + C::kCodeMax + (ch * nt + wt) * 64 +
                                                   b * 32 + g * 4);
                        const float sc[2][2] = {{e8m0_to_f32(s4 & 0xFF), e8m0_to_f32((s4 >> 8) & 0xFF)},
                                                {e8m0_to_f32((s4 >> 16) & 0xFF), e8m0_to_f32(s4 >> 24)}};
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int j = 2 * b + jj;
                            uint2 xf[TT];
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt)
                                xf[tt] = lds64a(xk + tt * 8 * xstride + 32 * j);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t w0 = jj ? wq[h][b].z : wq[h][b].x;
                                const uint32_t w1 = jj ? wq[h][b].w : wq[h][b].y;
                                uint32_t a0, a1, a2, a3;
                                e4m3x2_f16x2(w0, a0, a1);
                                e4m3x2_f16x2(w1, a2, a3);
#pragma unroll
                                for (int tt = 0; tt < TT; ++tt) {
                                    if (jj == 0)
                                        mma_f16_16816_zero(part[h][tt], a0, a1, a2, a3, xf[tt].x,
                                                           xf[tt].y);
                                    else
                                        mma_f16_16816(part[h][tt], a0, a1, a2, a3, xf[tt].x,
                                                      xf[tt].y);
                                }
                            }
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    // outputs e and e ^ 2 are rows g, g + 8 of
                                    // token 2t + (e & 1)
                                    const float f = (e & 1) ? fx[tt].y : fx[tt].x;
                                    acc[h][tt][e] =
                                        fmaf(part[h][tt][e], sc[h][e >> 1] * f, acc[h][tt][e]);
                                }
                    }
                }
            } else if (live) {
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) {
                    if (ch > 0 && k0 + 64 * ch >= p.K)
                        break;   // the last stage of a row may hold one chunk
                    // INT4: [half][lane][16 B]; INT8: [half][plane][lane][16 B]
                    const uint32_t cp = cs + ch * nt * 1024 * P;
                    const uint4 wl = lds128a(cp);
                    const uint4 wh = lds128a(cp + 512 * P);
                    const uint32_t wv[2][4] = {{wl.x, wl.y, wl.z, wl.w}, {wh.x, wh.y, wh.z, wh.w}};
                    uint32_t whi[2][4] = {};
                    if constexpr (P == 2) {
                        const uint4 ul = lds128a(cp + 512);
                        const uint4 uh = lds128a(cp + 1536);
                        whi[0][0] = ul.x; whi[0][1] = ul.y; whi[0][2] = ul.z; whi[0][3] = ul.w;
                        whi[1][0] = uh.x; whi[1][1] = uh.y; whi[1][2] = uh.z; whi[1][3] = uh.w;
                    }
                    const uint32_t xk = xrow + (k0 + 64 * ch) * 2;   // resident: k of the chunk
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int step = ch * 4 + j;   // k16 step inside the stage
                        const bool first = (step % C::kStepsPerGroup) == 0;
                        const bool last = ((step + 1) % C::kStepsPerGroup) == 0;
                        uint2 xf[TT];
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt) {
                            if constexpr (XR != 0)
                                xf[tt] = lds64a(xk + tt * 8 * xstride + 32 * j);
                            else
                                xf[tt] = lds64a(st + ch * C::kXBox + tt * 1024 + xoff[j]);
                        }
                        if constexpr (XR == 0) {
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt) {
                                // per token: the sum of the step's activations
                                // (an MMA with an all-ones weight tile)
                                if (first)
                                    mma_bf16_16816_zero(xsum[tt], kOnes, kOnes, kOnes, kOnes,
                                                        xf[tt].x, xf[tt].y);
                                else
                                    mma_bf16_16816(xsum[tt], kOnes, kOnes, kOnes, kOnes,
                                                   xf[tt].x, xf[tt].y);
                            }
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if constexpr (XR != 0) {
                                // fp16: registers a0, a2 (rows g) hold 1024 + q,
                                // a1, a3 (rows g + 8) hold 1024 + 16 q
                                const uint32_t w = wv[h][j], w8 = w >> 8;
                                const uint32_t a0 = int4_pair_f16<0>(w);
                                const uint32_t a1 = int4_pair_f16<1>(w);
                                const uint32_t a2 = int4_pair_f16<0>(w8);
                                const uint32_t a3 = int4_pair_f16<1>(w8);
#pragma unroll
                                for (int tt = 0; tt < TT; ++tt) {
                                    if (first)
                                        mma_f16_16816_zero(part[h][tt], a0, a1, a2, a3, xf[tt].x,
                                                           xf[tt].y);
                                    else
                                        mma_f16_16816(part[h][tt], a0, a1, a2, a3, xf[tt].x,
                                                      xf[tt].y);
                                }
                                if constexpr (P == 2) {
                                    const uint32_t u = whi[h][j], u8 = u >> 8;
                                    const uint32_t b0 = int4_pair_f16<0>(u);
                                    const uint32_t b1 = int4_pair_f16<1>(u);
                                    const uint32_t b2 = int4_pair_f16<0>(u8);
                                    const uint32_t b3 = int4_pair_f16<1>(u8);
#pragma unroll
                                    for (int tt = 0; tt < TT; ++tt) {
                                        if (first)
                                            mma_f16_16816_zero(parthi[h][tt], b0, b1, b2, b3,
                                                               xf[tt].x, xf[tt].y);
                                        else
                                            mma_f16_16816(parthi[h][tt], b0, b1, b2, b3,
                                                          xf[tt].x, xf[tt].y);
                                    }
                                }
                            } else {
                                const uint32_t a0 = int4_pair_plus128<0>(wv[h][j]);
                                const uint32_t a1 = int4_pair_plus128<4>(wv[h][j]);
                                const uint32_t a2 = int4_pair_plus128<8>(wv[h][j]);
                                const uint32_t a3 = int4_pair_plus128<12>(wv[h][j]);
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
                                            mma_bf16_16816(parthi[h][tt], b0, b1, b2, b3,
                                                           xf[tt].x, xf[tt].y);
                                    }
                                }
                            }
                        }
                        if (last) {
                            const int gi = step / C::kStepsPerGroup;   // group in the stage
                            const uint2 sv = lds64a(ss + gi * nt * 64);
                            const float2 s01 =
                                __half22float2(*reinterpret_cast<const __half2 *>(&sv.x));
                            const float2 s23 =
                                __half22float2(*reinterpret_cast<const __half2 *>(&sv.y));
                            const float sc[2][2] = {{s01.x, s01.y}, {s23.x, s23.y}};
                            if constexpr (XR != 0) {
                                // end of a scale group, fp16 windows: per token the
                                // table holds the sum S of the stored values x' and
                                // their factor f (x = f x').  Rows g summed
                                // (1024 + q) x', rows g + 8 (1024 + 16 q) x', so
                                // sum (q - 8) x = f (part - 1032 S) for rows g and
                                // f / 16 (part - 1152 S) for rows g + 8; INT8 (q =
                                // 16 hi + lo over two planes): f (16 Phi + Plo -
                                // 17536 S) and f / 16 (16 Phi + Plo - 19456 S).
                                const uint32_t xa = sb + p.xs_off +
                                                    ((xg0 + k0 / C::kG + gi) * 8 * TT + 2 * t) * 8;
#pragma unroll
                                for (int tt = 0; tt < TT; ++tt) {
                                    const uint4 tv = lds128a(xa + tt * 64);
                                    const float xs[2] = {__uint_as_float(tv.x), __uint_as_float(tv.z)};
                                    const float fx[2] = {__uint_as_float(tv.y), __uint_as_float(tv.w)};
#pragma unroll
                                    for (int h = 0; h < 2; ++h)
#pragma unroll
                                        for (int e = 0; e < 4; ++e) {
                                            // outputs e and e ^ 2 are rows g, g + 8
                                            // of token 2t + (e & 1)
                                            const int rh = e >> 1, tp = e & 1;
                                            float v;
                                            if constexpr (P == 2) {
                                                v = fmaf(16.f, parthi[h][tt][e], part[h][tt][e]);
                                                v = fmaf(rh ? -19456.f : -17536.f, xs[tp], v);
                                            } else {
                                                v = fmaf(rh ? -1152.f : -1032.f, xs[tp], part[h][tt][e]);
                                            }
                                            const float w = sc[h][rh] * (rh ? 0.0625f : 1.f) * fx[tp];
                                            acc[h][tt][e] = fmaf(v, w, acc[h][tt][e]);
                                        }
                                }
                            } else {
                                // end of a scale group: the MMAs summed (128 + q) * x,
                                // so acc += (part - 136 * sum(x)) * scale, in fp32
                                float2 xsv[TT];
#pragma unroll
                                for (int tt = 0; tt < TT; ++tt)
                                    xsv[tt] = make_float2(xsum[tt][0], xsum[tt][1]);
#pragma unroll
                                for (int h = 0; h < 2; ++h)
#pragma unroll
                                    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                                        for (int e = 0; e < 4; ++e) {
                                            // outputs e and e ^ 2 are rows g, g + 8 of
                                            // token 2t + (e & 1)
                                            const float xe = (e & 1) ? xsv[tt].y : xsv[tt].x;
                                            float v;
                                            if constexpr (P == 2) {
                                                // INT8 q = 16 hi + lo: the planes summed
                                                // (128 + hi) x and (128 + lo) x, so
                                                // sum (q - 128) x = 16 Phi + Plo - 2304 sum(x)
                                                v = fmaf(16.f, parthi[h][tt][e], part[h][tt][e]);
                                                v = fmaf(-2304.f, xe, v);
                                            } else {
                                                v = fmaf(-136.f, xe, part[h][tt][e]);
                                            }
                                            acc[h][tt][e] = fmaf(v, sc[h][e >> 1], acc[h][tt][e]);
                                        }
                            }
                        }
                    }
                }
            }
            // every lane's reads of the stage have returned (their values
            // are consumed above): release it to the producer
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[slot]);
            slot += C::kWPT;
            if (slot >= R) {
                slot -= R;
                phase ^= 1;
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
        const int seg_first = seg_begin;
        seg_begin = seg_end;
        if constexpr (C::kWPT == 2) {
            // the tile's second warp hands its fragment to the first (a named
            // barrier per tile: ids 1..8, the tile's two warps)
            float4 *xch = reinterpret_cast<float4 *>(smem + p.xchg_off) + wt * F * 32;
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
        if (live) {
            const bool whole = seg_first == gr * p.upr && seg_end == (gr + 1) * p.upr;
            if (whole) {
#pragma unroll
                for (int j = 0; j < F; ++j)
                    store_y4<TT>(p, gr * kWarps + wt, j, lane, sum[j]);
            } else {
                finish_cut<TT>(p, sum, c, gr, wt, lane);
            }
        }
    }
}

// variant = group mode + 3 * (INT8) + 6 * (resident activations), or 12:
// MXFP8 (64-k scale chunks, two bytes per tile lane and step, resident
// activations)
template <int V>
struct VariantOf {
    static constexpr int kGM = V == 12 ? 1 : V % 3;
    static constexpr int kP = V == 12 ? 2 : (V / 3) % 2 + 1;
    static constexpr int kXR = V == 12 ? 1 : V / 6;
    static constexpr int kMX = V == 12 ? 1 : 0;
};

template <int TT, int V>
const void *kernel_ptr()
{
    using W = VariantOf<V>;
    return reinterpret_cast<const void *>(
        &w4a16_stream_kernel<TT, W::kGM, W::kP, W::kXR, W::kMX>);
}

const void *select_kernel(int tt, int variant)
{
#define MXG_CASE(T, V) \
    if (tt == T && variant == V) return kernel_ptr<T, V>();
    MXG_CASE(1, 0) MXG_CASE(1, 1) MXG_CASE(1, 2) MXG_CASE(1, 3) MXG_CASE(1, 4) MXG_CASE(1, 5)
    MXG_CASE(1, 6) MXG_CASE(1, 7) MXG_CASE(1, 8) MXG_CASE(1, 9) MXG_CASE(1, 10) MXG_CASE(1, 11)
    MXG_CASE(2, 0) MXG_CASE(2, 1) MXG_CASE(2, 2) MXG_CASE(2, 3) MXG_CASE(2, 4) MXG_CASE(2, 5)
    MXG_CASE(2, 6) MXG_CASE(2, 7) MXG_CASE(2, 8) MXG_CASE(2, 9) MXG_CASE(2, 10) MXG_CASE(2, 11)
    MXG_CASE(1, 12) MXG_CASE(2, 12)
    MXG_CASE(3, 0) MXG_CASE(3, 1) MXG_CASE(3, 2) MXG_CASE(3, 3) MXG_CASE(3, 4) MXG_CASE(3, 5)
    MXG_CASE(4, 0) MXG_CASE(4, 1) MXG_CASE(4, 2) MXG_CASE(4, 3) MXG_CASE(4, 4) MXG_CASE(4, 5)
#undef MXG_CASE
    return nullptr;
}

struct VariantCfg {
    int stage, xchg, threads, consumers, g, xbox;
};

template <int TT, int V>
VariantCfg cfg_one()
{
    using W = VariantOf<V>;
    using C = Cfg<TT, W::kGM, W::kP, W::kXR>;
    return {C::kStage, C::kXchg, C::kThreads, C::kConsumers, C::kG, C::kXBox};
}

VariantCfg variant_cfg(int tt, int v)
{
#define MXG_CFG(T, V) \
    if (tt == T && v == V) return cfg_one<T, V>();
    MXG_CFG(1, 0) MXG_CFG(1, 1) MXG_CFG(1, 2) MXG_CFG(1, 3) MXG_CFG(1, 4) MXG_CFG(1, 5)
    MXG_CFG(1, 6) MXG_CFG(1, 7) MXG_CFG(1, 8) MXG_CFG(1, 9) MXG_CFG(1, 10) MXG_CFG(1, 11)
    MXG_CFG(2, 0) MXG_CFG(2, 1) MXG_CFG(2, 2) MXG_CFG(2, 3) MXG_CFG(2, 4) MXG_CFG(2, 5)
    MXG_CFG(2, 6) MXG_CFG(2, 7) MXG_CFG(2, 8) MXG_CFG(2, 9) MXG_CFG(2, 10) MXG_CFG(2, 11)
    MXG_CFG(1, 12) MXG_CFG(2, 12)
    MXG_CFG(3, 0) MXG_CFG(3, 1) MXG_CFG(3, 2) MXG_CFG(3, 3) MXG_CFG(3, 4) MXG_CFG(3, 5)
    MXG_CFG(4, 0) MXG_CFG(4, 1) MXG_CFG(4, 2) MXG_CFG(4, 3) MXG_CFG(4, 4) MXG_CFG(4, 5)
#undef MXG_CFG
    return {};
}

int group_mode(int G)
{
    return G == 128 ? 0 : (G == 64 ? 1 : 2);
}

// Shared-memory regions of a launch: ring, then resident activations and
// their sums, then the pair exchange, then the barriers.
struct SmemPlan {
    int R, x_off, xs_off, xchg_off, bar_off;
    size_t total;
};

SmemPlan smem_plan(const VariantCfg &vc, int R, int xbytes, int xsbytes)
{
    SmemPlan s{};
    s.R = R;
    s.x_off = R * vc.stage;
    s.xs_off = s.x_off + (xbytes + 127) / 128 * 128;
    s.xchg_off = s.xs_off + (xsbytes + 127) / 128 * 128;
    s.bar_off = s.xchg_off + vc.xchg;
    s.total = (size_t)s.bar_off + 2 * R * 8 + 1024;   // + alignment
    return s;
}

// bits: 4 (INT4), 8 (INT8, two code planes) or 0 (re-packed MXFP8: G = 64
// chunks, resident activations only, so M <= 16)
bool plan_stream(int device, int M, int N, int K, int G, int bits, StreamPlan *plan)
{
    if (M < 1 || M > 32 || N % 64 != 0 || K % 64 != 0 || K % G != 0)
        return false;
    if (bits == 0 && (G != 64 || M > 16))
        return false;
    if (device < 0 || device >= kMaxDeviceCache)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    const int ntiles = N / 32;
    const int ngroups = (ntiles + kWarps - 1) / kWarps;
    pl.upt = (K + kKS - 1) / kKS;                  // units (stages) per group row
    pl.ntiles = ngroups * kWarps;                  // arrival counters (one per tile slot)
    if ((size_t)pl.ntiles > kMaxCounters)
        return false;
    pl.units = (long long)ngroups * pl.upt;
    if (pl.units > (1LL << 30))
        return false;
    // fewer group rows than SMs: S pieces per row (at most one unit each);
    // else stream-K with one CTA per SM, no run shorter than one unit
    int S = 0;
    if (ngroups < di.sms) {
        S = std::min(di.sms / ngroups, pl.upt);
        pl.Wt = ngroups * S;
    } else {
        pl.Wt = (int)std::max<long long>(1, std::min<long long>(di.sms, pl.units));
    }
    pl.grid = pl.Wt;
    pl.split = S;
    const int q = (int)(pl.units / pl.Wt), r = (int)(pl.units % pl.Wt);
    const int base = bits == 0 ? 6 : (bits == 8 ? 3 : 0) + group_mode(G);
    const int budget = std::min(di.smem_optin, kMaxSmem);
    // resident activations for narrow token tiles, when they fit beside a
    // deep enough ring: the largest windows over all runs
    bool xr = false;
    int xbytes = 0, xsbytes = 0;
    if (pl.tt <= 2) {
        int xcols = 0, xgroups = 0;
        for (int cc = 0; cc < pl.Wt; ++cc) {
            const int U0 = run_start(q, r, S, pl.upt, cc), U1 = run_start(q, r, S, pl.upt, cc + 1);
            const XWindows w = x_windows(U0, U1, pl.upt, K);
            int cols = 0, groups = 0;
            for (int i = 0; i < w.n; ++i) {
                cols += w.cols[i] + kXPad;
                groups += w.cols[i] / G;
            }
            xcols = std::max(xcols, cols);
            xgroups = std::max(xgroups, groups);
        }
        xbytes = xcols * 2 * 8 * pl.tt;
        xsbytes = xgroups * 8 * pl.tt * 8;   // (sum, factor) per group and token
        // at least six stages (96 KB of INT4 codes), four for MXFP8's
        // twice larger stages
        const VariantCfg vr = variant_cfg(pl.tt, base + 6);
        if ((int)smem_plan(vr, bits == 0 ? 4 : 6, xbytes, xsbytes).total <= budget)
            xr = true;
    }
    if (bits == 0 && !xr)
        return false;
    pl.variant = base + (xr ? 6 : 0);
    const VariantCfg vc = variant_cfg(pl.tt, pl.variant);
    if (!xr)
        xbytes = xsbytes = 0;
    // the deepest ring that fits, up to MXG_STREAM_MAX_RING_KB of stages
    int R = (MXG_STREAM_MAX_RING_KB * 1024) / vc.stage;
    while (R > 2 && (int)smem_plan(vc, R, xbytes, xsbytes).total > budget)
        --R;
    if (R < 3)
        return false;
    const SmemPlan sp = smem_plan(vc, R, xbytes, xsbytes);
    pl.smem = sp.total;
    pl.ring = R;
    pl.x_off = sp.x_off;
    pl.xs_off = sp.xs_off;
    pl.xchg_off = sp.xchg_off;
    pl.bar_off = sp.bar_off;
    pl.warps_per_cta = vc.threads / 32;
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return false;
    // the attribute is set per device and variant to the largest shared
    // memory a launch may ask for
    static std::atomic<int> occ_cache[kMaxDeviceCache][4][13];
    std::atomic<int> &occ_slot = occ_cache[device][pl.tt - 1][pl.variant];
    if (occ_slot.load(std::memory_order_acquire) == 0) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, budget) !=
            cudaSuccess)
            return false;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, vc.threads, budget) !=
                cudaSuccess ||
            o < 1)
            return false;
        occ_slot.store(o, std::memory_order_release);
    }
    pl.partial_bytes = (size_t)pl.Wt * 2 * kWarps * (2 * pl.tt * 32) * sizeof(float4);
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

bool plan_mxfp8_packed_stream(int device, int M, int N, int K, StreamPlan *plan)
{
    return plan_stream(device, M, N, K, 64, 0, plan);
}

cudaError_t launch_w4a16_stream(const StreamPlan &pl, const void *X, const void *packed, int M,
                                int N, int K, int G, void *Y, void *workspace, bool early,
                                cudaStream_t stream)
{
    (void)G;
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return cudaErrorInvalidValue;
    const VariantCfg vc = variant_cfg(pl.tt, pl.variant);
    const int planes = pl.variant == 12 ? 2 : (pl.variant / 3) % 2 + 1;
    const uint8_t *codes = static_cast<const uint8_t *>(packed);
    alignas(64) CUtensorMap xmap;
    // X: bf16 [M][K], boxes of 64 k x 8 TT rows with 128-byte swizzle (used
    // by the variants whose stages carry their activations)
    if (!encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K,
                              (uint64_t)M, (uint64_t)K * 2, 64, (uint32_t)(8 * pl.tt),
                              CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const WorkspaceMap wm = make_workspace_map(pl.ntiles, pl.partial_bytes);
    Params p{};
    p.X = static_cast<const uint16_t *>(X);
    p.codes = codes;
    // codes take half a byte per weight (INT4) or one byte in two planes (INT8)
    p.scales = codes + (size_t)N * K / 2 * planes;
    p.Y = static_cast<uint16_t *>(Y);
    p.early = early ? 1 : 0;
    p.pf_stages = MXG_STREAM_PF_STAGES;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wm.counters_off);
    p.partial = reinterpret_cast<float4 *>(static_cast<uint8_t *>(workspace) + wm.partial_off);
    p.frag = 2 * pl.tt * 32;
    p.M = M;
    p.N = N;
    p.K = K;
    p.ntiles = N / 32;
    p.upr = pl.upt;
    p.q = (int)(pl.units / pl.Wt);
    p.r = (int)(pl.units % pl.Wt);
    p.S = pl.split;
    p.R = pl.ring;
    p.x_off = pl.x_off;
    p.xs_off = pl.xs_off;
    p.xchg_off = pl.xchg_off;
    p.bar_off = pl.bar_off;
    void *args[] = {&xmap, &p};
    return launch_pdl(fn, dim3(pl.grid), dim3(vc.threads), pl.smem, stream, args);
}

}  // namespace mxg
