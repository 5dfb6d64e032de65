// INT4 W4A16 weight-streaming GEMM for small M (decode / MTP verify chunks).
//
// At M <= 32 the layer reads each weight byte once and does 2*M flops per
// weight: it is bound by HBM bytes of W.  The kernel therefore
//  * cuts the re-packed weight stream into equal units (one n32 tile x one
//    or two spans of max(G, 64) rows of K) and gives every CTA of a
//    persistent grid (one per SM) one contiguous run of units (stream-K at
//    CTA granularity), so all SMs stream the same number of bytes;
//  * the CTA's warps take the run's units in turn (unit i goes to warp
//    i mod C), so every warp works on the same n32 tile at once and a warp
//    the scheduler serves less only delays its own units;
//  * each warp moves its units through its own ring of shared-memory slots
//    with 1-D bulk copies (cp.async.bulk, completion on an mbarrier; codes
//    and scales of a unit), several units ahead, weights marked evict-first
//    in L2;
//  * each warp decodes a pair of nibbles to the bf16 pair (128 + q) with one
//    mask-and-or (plus a shift) and multiplies on the tensor cores with
//    m16n8k16 MMAs where the weights are the 16-row operand and the tokens
//    the 8-column operand ("swap AB"); the two n16 halves of a unit share
//    each activation fragment, and one more MMA with an all-ones weight tile
//    gives the per-token activation sum that turns (128 + q) into (q - 8);
//  * starts a zero-initialised partial sum per scale group (every MMA step
//    lies inside one group for G = 32, 64, 128) and adds
//    (partial - 136 * activation sum) * scale in fp32 once per group, so
//    weights are never rounded (every product is exact in fp32);
//  * at the end of each tile every warp leaves its fragment in shared memory
//    and goes on; the last warp to arrive adds the fragments.  A tile inside
//    the CTA's run is written to Y at once.  A tile cut between CTAs is
//    finished by the CTA holding its first unit, at the end of that CTA's
//    run: the other contributors (for whom it is the first tile of the run)
//    published their fragments early, so it adds them in CTA order
//    (deterministic) and writes bf16 Y.
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

#ifndef MXG_STREAM_CONSUMERS
#define MXG_STREAM_CONSUMERS 12
#endif
#ifndef MXG_STREAM_CTAS_PER_SM
#define MXG_STREAM_CTAS_PER_SM 1
#endif
#ifndef MXG_STREAM_STAGES_BIG
#define MXG_STREAM_STAGES_BIG 2
#endif
constexpr int kConsumers = MXG_STREAM_CONSUMERS;  // warps per CTA
constexpr int kThreads = kConsumers * 32;
constexpr int kCtasPerSm = MXG_STREAM_CTAS_PER_SM;   // resident CTAs per SM (grid size / SMs)
constexpr int kMinUnitsPerCta = 2 * kConsumers;  // shortest run

// Group modes: 0 -> G = 128, 1 -> G = 64, 2 -> G = 32.  A unit (what one
// ring slot holds) spans SU times max(G, 64) rows of K of one n32 tile.
// P code planes: 1 for INT4; 2 for INT8, whose codes are stored as a plane
// of low nibbles and a plane of high nibbles, each in the INT4 layout.
template <int GM, int SU, int P = 1>
struct Mode {
    static constexpr int kG = GM == 0 ? 128 : (GM == 1 ? 64 : 32);
    static constexpr int kChunks = (GM == 0 ? 2 : 1) * SU;    // k64 chunks per unit
    static constexpr int kGroups = (GM == 2 ? 2 : 1) * SU;    // scale groups per unit
    static constexpr int kStepsPerGroup = kG / 16;            // MMA k16 steps per group
    static constexpr int kCode = kChunks * 1024 * P;          // code bytes per unit
    static constexpr int kScale = kGroups * 64;               // scale bytes per unit
    // slots per warp: shallow rings (12 warps x 2-3 slots keep enough bytes in
    // flight) leave most of the SM's shared-memory/L1 split to L1, where the
    // re-read activations hit
    static constexpr int kStages = kCode >= 4096 ? MXG_STREAM_STAGES_BIG : 3;
};

// Shared memory: every warp's ring of kStages slots (a slot holds one
// unit's codes, then its scales), kRed reduction buffers of kConsumers
// fragments (segment s of the run uses buffer s mod kRed), one mbarrier per
// slot, then per reduction buffer an arrival count and a use count.
template <int TT, int GM, int SU, int P = 1>
struct Smem {
    using MD = Mode<GM, SU, P>;
    static constexpr int kFrag4 = 2 * TT * 32;                // float4 per warp fragment
    static constexpr int kSlot = (MD::kCode + MD::kScale + 127) / 128 * 128;
    // One reduction buffer: a warp that ends a segment before the previous
    // segment's reduction is done waits for it (rarely), and the smaller
    // shared-memory footprint leaves a larger L1 for the activation loads
    // (every CTA re-reads X for each of its tiles).
    static constexpr int kRed = 1;
    static constexpr size_t kRingBytes = (size_t)kConsumers * MD::kStages * kSlot;
    static constexpr size_t kRedBytes = (size_t)kRed * kConsumers * kFrag4 * 16;
    static constexpr size_t kBarBytes = (size_t)kConsumers * MD::kStages * 8;
    static constexpr size_t kRedOff = kRingBytes;
    static constexpr size_t kBarOff = kRedOff + kRedBytes;
    static constexpr size_t kSyncOff = kBarOff + kBarBytes;
    static constexpr size_t kTotal = kSyncOff + 2 * kRed * sizeof(int);
};

struct Params {
    const uint16_t *X;       // bf16 [M][K]
    const uint8_t *codes;    // re-packed codes  [N/32][K/64][2][32][16 B]
    const uint8_t *scales;   // re-packed scales [N/32][K/G][8][4 halves]
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [N/32]
    float4 *partial;         // [ctas][2*TT][32]: a CTA's fragment of its first, cut tile
    int M, N, K;
    int upt;                 // units per n32 tile
    int units;
    int ctas;
    int q, r;                // units = q * ctas + r: CTAs below r run q + 1 units, the rest q
    int early;               // load the first weights before waiting for the previous kernel
};

// First unit of CTA c's run.
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

// Run by warp 0 of a CTA whose segment of `tile` is cut (the tile goes on
// in other CTAs' runs), with the CTA's warp fragments in `frags`.  The CTA
// whose run holds the tile's first unit finishes that segment last in its
// run: it adds the other contributors' fragments (in CTA order) to its own
// and writes bf16 Y.  Every other contributor (its segment is the first one
// of its run) publishes its fragment and bumps the tile's counter without
// waiting for anybody.
template <int TT>
__device__ __noinline__ void finish_cut_tile(const Params &p, const float4 *frags, int c, int tile,
                                             int lane)
{
    constexpr int F = 2 * TT;
    constexpr int kFrag4 = F * 32;
    float4 sum[F];
#pragma unroll
    for (int j = 0; j < F; ++j) {
        sum[j] = frags[j * 32 + lane];
        for (int w = 1; w < kConsumers; ++w) {
            const float4 v = frags[w * kFrag4 + j * 32 + lane];
            sum[j].x += v.x;
            sum[j].y += v.y;
            sum[j].z += v.z;
            sum[j].w += v.w;
        }
    }
    const int tile_begin = tile * p.upt;
    const int c_first = cta_of_unit(p, tile_begin);
    if (c != c_first) {
#pragma unroll
        for (int j = 0; j < F; ++j)
            __stcg(p.partial + ((size_t)c * F + j) * 32 + lane, sum[j]);
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            atomicAdd(&p.counters[tile], 1);
        }
        return;
    }
    const int c_last = cta_of_unit(p, tile_begin + p.upt - 1);
    if (lane == 0) {
        // the other contributors published early in their runs (or at their
        // ends, for runs inside the tile); the wait is bounded
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
#pragma unroll
        for (int j = 0; j < F; ++j) {
            const float4 f = __ldcg(p.partial + ((size_t)cc * F + j) * 32 + lane);
            sum[j].x += f.x;
            sum[j].y += f.y;
            sum[j].z += f.z;
            sum[j].w += f.w;
        }
    }
#pragma unroll
    for (int j = 0; j < F; ++j)
        store_y4<TT>(p, tile, j, lane, sum[j]);
    if (lane == 0)
        p.counters[tile] = 0;  // leave the counter zero for the next call
}

template <int TT>
__device__ __forceinline__ void zero_acc(float (&a)[2][TT][4])
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                a[h][tt][e] = 0.f;
}

// Copies unit u (codes, then scales) into a ring slot; completion on `bar`.
template <int GM, int SU, int P>
__device__ __forceinline__ void fetch_unit(const Params &p, uint8_t *slot, uint64_t *bar, int u,
                                           uint64_t policy)
{
    using MD = Mode<GM, SU, P>;
    mbar_arrive_expect_tx(bar, MD::kCode + MD::kScale);
    bulk_g2s(slot, p.codes + (size_t)u * MD::kCode, MD::kCode, bar, policy);
    bulk_g2s(slot + MD::kCode, p.scales + (size_t)u * MD::kScale, MD::kScale, bar, policy);
}

template <int TT, int GM, int SU, int P>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) w4a16_stream_kernel(const Params p)
{
    using MD = Mode<GM, SU, P>;
    using SL = Smem<TT, GM, SU, P>;
    constexpr int kStages = MD::kStages;
    constexpr int F = 2 * TT;  // float4 per lane fragment
    extern __shared__ __align__(128) uint8_t smem[];
    float4 *red = reinterpret_cast<float4 *>(smem + SL::kRedOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    const int c = blockIdx.x;
    const int U0 = run_start(p, c), U1 = run_start(p, c + 1);
    const int n = U1 - U0;
    uint8_t *ring = smem + (size_t)warp * kStages * SL::kSlot;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SL::kBarOff) + warp * kStages;
    uint64_t policy = 0;
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s)
            mbar_init(&full[s], 1);
        fence_barrier_init();
        policy = l2_policy_evict_first();
    }
    int *red_count = reinterpret_cast<int *>(smem + SL::kSyncOff);  // arrivals per buffer
    int *red_done = red_count + SL::kRed;                           // reductions per buffer
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2 * SL::kRed; ++b)
            red_count[b] = 0;
        // while the previous kernel drains: pull the first units into L2
        const int nu = min(kConsumers * kStages, n);
        prefetch_l2(p.codes + (size_t)U0 * MD::kCode, nu * MD::kCode);
        prefetch_l2(p.scales + (size_t)U0 * MD::kScale, nu * MD::kScale);
    }
    __syncthreads();
    // this warp takes units warp, warp + C, ... of the run; its k-th unit
    // goes to slot k mod kStages.  The weights are not written by the
    // previous kernel on the stream (the caller's contract, unless it turned
    // early weight loads off): the first slots fill while that kernel drains.
    auto fill_ring = [&]() {
        if (lane == 0)
            for (int k = 0; k < kStages && warp + k * kConsumers < n; ++k)
                fetch_unit<GM, SU, P>(p, ring + k * SL::kSlot, &full[k], U0 + warp + k * kConsumers,
                                   policy);
    };
    if (p.early)
        fill_ring();
    pdl_wait();
    if (!p.early)
        fill_ring();

    // ------------------------------------------------------------ consumers
    const int g = lane >> 2, t = lane & 3;
    // activation rows of this lane: m = g + 8 tt; the lane reads k = 4t .. 4t+3
    // of every k16 step
    // (rows m >= M read row 0 instead: their outputs are never stored)
    const uint16_t *xrow[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
        const int m = tt * 8 + g;
        xrow[tt] = p.X + (size_t)(m < p.M ? m : 0) * p.K + 4 * t;
    }
    const int upt = p.upt;

    // Activation fragments of one unit, requested one unit ahead for narrow
    // token tiles (a whole unit of work hides their L2 latency).
    constexpr bool kPipeX = MD::kChunks * TT <= 4;
    uint2 xs[MD::kChunks][TT][4], xn[MD::kChunks][TT][4];
    // ku: the unit's place in its tile
    auto load_x = [&](uint2 (&dst)[MD::kChunks][TT][4], int ku) {
        const int kc = ku * MD::kChunks;  // first k64 chunk of the unit
#pragma unroll
        for (int ch = 0; ch < MD::kChunks; ++ch)
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    dst[ch][tt][j] = __ldg(
                        reinterpret_cast<const uint2 *>(xrow[tt] + (kc + ch) * 64 + 16 * j));
    };
    // place in its tile of the unit kConsumers further on
    auto next_ku = [&](int ku) {
        ku += kConsumers;
        while (ku >= upt)
            ku -= upt;
        return ku;
    };

    constexpr uint32_t kOnes = 0x3F803F80u;  // bf16 pair (1, 1)
    float acc[2][TT][4], part[2][TT][4], xsum[TT][4];
    float parthi[P == 2 ? 2 : 1][TT][4];  // INT8: sums over the high-nibble plane
    bool ok = true;
    int i = warp;          // run index of this warp's next unit
    int slot = 0;          // ring slot of unit i
    uint32_t phase = 0;    // parity of the phase of unit i
    int ku = (U0 + i) % upt;  // place of unit i in its tile
    if (kPipeX && i < n)
        load_x(xs, ku);
    int sidx = 0;          // segment of the run
    int tile = U0 / upt;
    for (int seg = U0; seg < U1; ++tile) {
        const int tile_begin = tile * upt;
        const int seg_end = min(U1, tile_begin + upt);
        zero_acc<TT>(acc);
        for (; U0 + i < seg_end; i += kConsumers) {
            const int u = U0 + i;
            const int ku_next = next_ku(ku);
            if (kPipeX) {
                if (i + kConsumers < n)
                    load_x(xn, ku_next);
            } else {
                load_x(xs, ku);
            }
            ku = ku_next;
            if (!mbar_wait(&full[slot], phase, ok ? kWaitLimitNs : 0)) {
                if (ok && lane == 0)
                    record_error(p.hdr, MXG_ERR_TIMEOUT, 100 + GM);
                ok = false;
            }
            const uint8_t *st = ring + slot * SL::kSlot;
            const uint8_t *ss = st + MD::kCode;
#pragma unroll
            for (int ch = 0; ch < MD::kChunks; ++ch) {
                // INT4: [half][lane][16 B]; INT8: [half][plane][lane][16 B]
                const uint8_t *cp = st + ch * 1024 * P + lane * 16;
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
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int step = ch * 4 + j;  // k16 step inside the unit
                    const bool first = (step % MD::kStepsPerGroup) == 0;
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt) {
                        // per token: the sum of the step's activations (an MMA
                        // with an all-ones weight tile)
                        if (first)
                            mma_bf16_16816_zero(xsum[tt], kOnes, kOnes, kOnes, kOnes,
                                                xs[ch][tt][j].x, xs[ch][tt][j].y);
                        else
                            mma_bf16_16816(xsum[tt], kOnes, kOnes, kOnes, kOnes,
                                           xs[ch][tt][j].x, xs[ch][tt][j].y);
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
                                mma_bf16_16816_zero(part[h][tt], a0, a1, a2, a3,
                                                    xs[ch][tt][j].x, xs[ch][tt][j].y);
                            else
                                mma_bf16_16816(part[h][tt], a0, a1, a2, a3, xs[ch][tt][j].x,
                                               xs[ch][tt][j].y);
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
                                                        xs[ch][tt][j].x, xs[ch][tt][j].y);
                                else
                                    mma_bf16_16816(parthi[h][tt], b0, b1, b2, b3,
                                                   xs[ch][tt][j].x, xs[ch][tt][j].y);
                            }
                        }
                    }
                    if ((step + 1) % MD::kStepsPerGroup == 0) {
                        // end of a scale group: the MMAs summed (128 + q) * x, so
                        // acc += (part - 136 * sum(x)) * scale, in fp32
                        const int gi = step / MD::kStepsPerGroup;  // group inside the unit
                        const uint2 sv = lds64(ss + gi * 64 + g * 8);
                        const float2 s01 = __half22float2(*reinterpret_cast<const __half2 *>(&sv.x));
                        const float2 s23 = __half22float2(*reinterpret_cast<const __half2 *>(&sv.y));
                        const float sc[2][2] = {{s01.x, s01.y}, {s23.x, s23.y}};
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    // outputs e and e ^ 2 are rows g, g + 8 of token 2t + (e & 1)
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
            // every lane's reads of the slot have returned (their values are
            // consumed above): refill it with this warp's unit kStages ahead
            __syncwarp();
            if (lane == 0 && i + kStages * kConsumers < n)
                fetch_unit<GM, SU, P>(p, ring + slot * SL::kSlot, &full[slot],
                               u + kStages * kConsumers, policy);
            if (kPipeX) {
#pragma unroll
                for (int ch = 0; ch < MD::kChunks; ++ch)
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            xs[ch][tt][j] = xn[ch][tt][j];
            }
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1;
            }
        }

        // ---- end of the tile segment.  Every warp leaves its fragment in the
        // segment's reduction buffer and goes on; the last warp to arrive adds
        // the fragments.  A buffer is reused kRed segments later, once the
        // reduction of its previous segment is done.
        const int rb = sidx % SL::kRed;
        const int uses = sidx / SL::kRed;  // earlier segments that used buffer rb
        if (uses > 0) {
            if (lane == 0) {
                const unsigned long long t0 = global_ns();
                while (*reinterpret_cast<volatile int *>(&red_done[rb]) < uses) {
                    if (global_ns() - t0 > kWaitLimitNs) {
                        record_error(p.hdr, MXG_ERR_TIMEOUT, 130);
                        break;
                    }
                    __nanosleep(32);
                }
                __threadfence_block();
            }
            __syncwarp();
        }
        float4 *frags = red + (size_t)rb * kConsumers * SL::kFrag4;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
                frags[(size_t)warp * SL::kFrag4 + (h * TT + tt) * 32 + lane] =
                    make_float4(acc[h][tt][0], acc[h][tt][1], acc[h][tt][2], acc[h][tt][3]);
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            __threadfence_block();
            last = atomicAdd(&red_count[rb], 1) == kConsumers - 1;
            __threadfence_block();
        }
        if (__shfl_sync(0xffffffffu, last, 0)) {
            if (lane == 0)
                red_count[rb] = 0;
            const bool whole = seg == tile_begin && seg_end == tile_begin + upt;
            if (whole) {
#pragma unroll
                for (int j = 0; j < F; ++j) {
                    float4 s = frags[j * 32 + lane];
#pragma unroll
                    for (int w = 1; w < kConsumers; ++w) {
                        const float4 v = frags[(size_t)w * SL::kFrag4 + j * 32 + lane];
                        s.x += v.x;
                        s.y += v.y;
                        s.z += v.z;
                        s.w += v.w;
                    }
                    store_y4<TT>(p, tile, j, lane, s);
                }
            } else {
                finish_cut_tile<TT>(p, frags, c, tile, lane);
            }
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                atomicAdd(&red_done[rb], 1);
            }
        }
        ++sidx;
        seg = seg_end;
    }
}

template <int TT, int GM, int SU, int P = 1>
const void *kernel_ptr()
{
    return reinterpret_cast<const void *>(&w4a16_stream_kernel<TT, GM, SU, P>);
}

// SU = 2 (two scale-group spans per unit) for up to two token tiles,
// SU = 1 otherwise; variant = gm + 3 * (SU - 1).
const void *select_kernel(int tt, int variant)
{
#define MXG_CASE(T, G_, S_) \
    if (tt == T && variant == G_ + 3 * (S_ - 1)) return kernel_ptr<T, G_, S_>();
    MXG_CASE(1, 0, 1) MXG_CASE(1, 1, 1) MXG_CASE(1, 2, 1)
    MXG_CASE(2, 0, 1) MXG_CASE(2, 1, 1) MXG_CASE(2, 2, 1)
    MXG_CASE(3, 0, 1) MXG_CASE(3, 1, 1) MXG_CASE(3, 2, 1)
    MXG_CASE(4, 0, 1) MXG_CASE(4, 1, 1) MXG_CASE(4, 2, 1)
    MXG_CASE(1, 0, 2) MXG_CASE(1, 1, 2) MXG_CASE(1, 2, 2)
    MXG_CASE(2, 0, 2) MXG_CASE(2, 1, 2) MXG_CASE(2, 2, 2)
#undef MXG_CASE
    // INT8 (two code planes), SU = 1: variant = 6 + gm
#define MXG_CASE8(T, G_) \
    if (tt == T && variant == 6 + G_) return kernel_ptr<T, G_, 1, 2>();
    MXG_CASE8(1, 0) MXG_CASE8(1, 1) MXG_CASE8(1, 2)
    MXG_CASE8(2, 0) MXG_CASE8(2, 1) MXG_CASE8(2, 2)
    MXG_CASE8(3, 0) MXG_CASE8(3, 1) MXG_CASE8(3, 2)
    MXG_CASE8(4, 0) MXG_CASE8(4, 1) MXG_CASE8(4, 2)
#undef MXG_CASE8
    return nullptr;
}

template <int GM, int SU, int P = 1>
size_t smem_bytes_gs(int tt)
{
    switch (tt) {
    case 1: return Smem<1, GM, SU, P>::kTotal;
    case 2: return Smem<2, GM, SU, P>::kTotal;
    case 3: return Smem<3, GM, 1, P>::kTotal;
    default: return Smem<4, GM, 1, P>::kTotal;
    }
}

size_t smem_bytes(int tt, int variant)
{
    switch (variant) {
    case 0: return smem_bytes_gs<0, 1>(tt);
    case 1: return smem_bytes_gs<1, 1>(tt);
    case 2: return smem_bytes_gs<2, 1>(tt);
    case 3: return smem_bytes_gs<0, 2>(tt);
    case 4: return smem_bytes_gs<1, 2>(tt);
    case 5: return smem_bytes_gs<2, 2>(tt);
    case 6: return smem_bytes_gs<0, 1, 2>(tt);
    case 7: return smem_bytes_gs<1, 1, 2>(tt);
    default: return smem_bytes_gs<2, 1, 2>(tt);
    }
}

int group_mode(int G)
{
    return G == 128 ? 0 : (G == 64 ? 1 : 2);
}

}  // namespace

namespace {

// bits: 4 (INT4) or 8 (INT8, two code planes, one scale-group span per unit)
bool plan_stream(int device, int M, int N, int K, int G, int bits, StreamPlan *plan)
{
    if (M < 1 || M > 32 || N % 32 != 0)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    const int unit_k = std::max(G, 64);
    const int su = (bits == 4 && pl.tt <= 2 && (K / unit_k) % 2 == 0) ? 2 : 1;
    pl.variant = bits == 8 ? 6 + group_mode(G) : group_mode(G) + 3 * (su - 1);
    pl.warps_per_cta = kConsumers;
    pl.smem = smem_bytes(pl.tt, pl.variant);
    if ((int)pl.smem > di.smem_optin)
        return false;
    pl.upt = K / (unit_k * su);
    pl.ntiles = N / 32;
    if ((size_t)pl.ntiles > kMaxCounters)
        return false;
    pl.units = (long long)pl.ntiles * pl.upt;
    if (pl.units > (1LL << 30))
        return false;
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return false;
    // resident CTAs per SM for this variant: every CTA of the grid must be
    // resident at once (a cut tile's finishing CTA waits for the others)
    // (function attributes and occupancy are per device: cached per device)
    if (device < 0 || device >= kMaxDeviceCache)
        return false;
    static std::atomic<int> occ_cache[kMaxDeviceCache][4][9];
    std::atomic<int> &occ_slot = occ_cache[device][pl.tt - 1][pl.variant];
    int occ = occ_slot.load(std::memory_order_acquire);
    if (occ == 0) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) !=
            cudaSuccess)
            return false;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, kThreads, pl.smem) !=
                cudaSuccess ||
            o < 1)
            return false;
        occ = std::min(o, kCtasPerSm);
        occ_slot.store(occ, std::memory_order_release);
    }
    // kCtasPerSm CTAs per SM, but no run shorter than kMinUnitsPerCta units;
    // a layer too small for 32 such runs gets at least one CTA per n32 tile
    // instead (one CTA streaming many short tiles would serialise their
    // reductions)
    long long wt = std::min<long long>((long long)di.sms * occ, pl.units / kMinUnitsPerCta);
    if (wt < 32)
        wt = std::min<long long>((long long)di.sms * occ, std::max<long long>(wt, pl.ntiles));
    pl.Wt = (int)std::max<long long>(1, wt);
    pl.grid = pl.Wt;
    pl.partial_bytes = (size_t)pl.Wt * (2 * pl.tt * 32) * sizeof(float4);
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
                                int N, int K, int G, void *Y, void *workspace, cudaStream_t stream)
{
    (void)G;
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return cudaErrorInvalidValue;
    const WorkspaceMap wm = make_workspace_map(pl.ntiles, pl.partial_bytes);
    Params p{};
    p.X = static_cast<const uint16_t *>(X);
    p.codes = static_cast<const uint8_t *>(packed);
    // codes take half a byte per weight (INT4) or one byte in two planes (INT8)
    p.scales = p.codes + (pl.variant >= 6 ? (size_t)N * K : (size_t)N * K / 2);
    p.Y = static_cast<uint16_t *>(Y);
    p.early = early_weight_loads() ? 1 : 0;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wm.counters_off);
    p.partial = reinterpret_cast<float4 *>(static_cast<uint8_t *>(workspace) + wm.partial_off);
    p.M = M;
    p.N = N;
    p.K = K;
    p.upt = pl.upt;
    p.units = (int)pl.units;
    p.ctas = pl.Wt;
    p.q = (int)(pl.units / pl.Wt);
    p.r = (int)(pl.units % pl.Wt);
    void *args[] = {&p};
    return launch_pdl(fn, dim3(pl.grid), dim3(kThreads), pl.smem, stream, args);
}

}  // namespace mxg
