// INT4 W4A16 weight-streaming GEMM for small M (decode / MTP verify chunks).
//
// At M <= 32 the layer reads each weight byte once and does 2*M flops per
// weight: it is bound by HBM bytes of W.  The kernel therefore
//  * cuts the re-packed weight stream into equal units (one n32 tile x one
//    scale-group span of max(G, 64) rows of K) and gives every warp of a
//    persistent grid one contiguous run of units (stream-K), so all SMs
//    stream the same number of bytes; a run is one contiguous byte range of
//    the re-packed buffer, and never shorter than a few stages;
//  * moves each warp's run through its own ring of shared-memory stages
//    with 1-D bulk copies (cp.async.bulk, completion on an mbarrier), four
//    2 KB stages in flight per warp, weights marked evict-first in L2;
//  * decodes nibbles to exact bf16 (q - 8) in registers (shift + lop3 and
//    one bf16x2 add per two weights) and multiplies on the tensor cores
//    with m16n8k16 MMAs where the weights are the 16-row operand and the
//    tokens the 8-column operand ("swap AB"); the two n16 halves of a unit
//    share each activation fragment;
//  * starts a zero-initialised partial sum per scale group (every MMA step
//    lies inside one group for G = 32, 64, 128) and adds partial * scale
//    in fp32 once per group, so weights are never rounded;
//  * n32 tiles covered whole by one warp are written directly; a tile cut
//    between warps is reduced through the workspace: at the end of its run
//    each contributor stores its fragment and bumps the tile's arrival
//    counter (acquire-release), and the last one adds all fragments in warp
//    order (deterministic) and writes bf16 Y.  Nobody waits on anybody.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

constexpr int kWarps = 8;         // warps per CTA
#ifndef MXG_STREAM_RING
#define MXG_STREAM_RING 4
#endif
#ifndef MXG_STREAM_MIN_STAGES
#define MXG_STREAM_MIN_STAGES 6
#endif
constexpr int kRing = MXG_STREAM_RING;          // stages per warp
constexpr int kMinStages = MXG_STREAM_MIN_STAGES;  // shortest run, in stages
constexpr int kStageCode = 2048;  // code bytes per stage (two k64 chunks of an n32 tile)
constexpr int kStageScale = 256;  // scale bytes reserved per stage
constexpr int kStageBytes = kStageCode + kStageScale;
// per-warp ring: stages, then one mbarrier per stage; rounded so every
// warp's ring (and every stage) starts 128-byte aligned
constexpr int kWarpSmem = (kRing * kStageBytes + kRing * 8 + 127) / 128 * 128;
static_assert(kStageBytes % 128 == 0, "stages must stay 128-byte aligned");

// Group modes: 0 -> G = 128, 1 -> G = 64, 2 -> G = 32.
template <int GM>
struct Mode {
    static constexpr int kG = GM == 0 ? 128 : (GM == 1 ? 64 : 32);
    static constexpr int kChunks = GM == 0 ? 2 : 1;          // k64 chunks per unit
    static constexpr int kGroups = GM == 2 ? 2 : 1;          // scale groups per unit
    static constexpr int kUnitsPerStage = 2 / kChunks;
    static constexpr int kStepsPerGroup = kG / 16;            // MMA k16 steps per group
};

struct Params {
    const uint16_t *X;       // bf16 [M][K]
    const uint8_t *codes;    // re-packed codes  [N/32][K/64][2][32][16 B]
    const uint8_t *scales;   // re-packed scales [N/32][K/G][8][4 halves]
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [N/32]
    float *partial;          // [Wt][2][32][2*4*TT]
    int M, N, K;
    int upt;                 // units per n32 tile
    int units;
    int Wt;
    int q, r;                // units = q * Wt + r: warps below r run q + 1 units, the rest q
};

// First unit of warp w's run.
__device__ __forceinline__ int run_start(const Params &p, int w)
{
    return w * p.q + min(w, p.r);
}

// The warp whose run contains unit u.
__device__ __forceinline__ int warp_of_unit(const Params &p, int u)
{
    const int big = p.r * (p.q + 1);   // units covered by the longer runs
    return u < big ? u / (p.q + 1) : p.r + (u - big) / p.q;
}

template <int TT>
__device__ __forceinline__ void store_tile_y(const Params &p, int tile,
                                             const float (&v)[2][TT][4], int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = tt * 8 + 2 * t + (e & 1);
                const int n = tile * 32 + h * 16 + g + ((e & 2) ? 8 : 0);
                if (m < p.M)
                    p.Y[(size_t)m * p.N + n] = f32_to_bf16_bits(v[h][tt][e]);
            }
}

template <int TT>
__device__ __forceinline__ void store_partial(const Params &p, int gw, int slot, int lane,
                                              const float (&v)[2][TT][4])
{
    float *dst = p.partial + ((size_t)(gw * 2 + slot) * 32 + lane) * (8 * TT);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
            __stcg(reinterpret_cast<float4 *>(dst + (h * TT + tt) * 4),
                   make_float4(v[h][tt][0], v[h][tt][1], v[h][tt][2], v[h][tt][3]));
}

// Run by the last contributor of a cut tile: add every fragment of the tile
// in warp order and write bf16 Y.
template <int TT>
__device__ __noinline__ void reduce_tile(const Params &p, int tile, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    const int tile_begin = tile * p.upt, tile_end = tile_begin + p.upt;
    const int w_first = warp_of_unit(p, tile_begin);
    const int w_last = warp_of_unit(p, tile_end - 1);
    float sum[2][TT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                sum[h][tt][e] = 0.f;
#pragma unroll 4
    for (int w = w_first; w <= w_last; ++w) {
        const int s = (run_start(p, w) >= tile_begin) ? 0 : 1;
        const float *src = p.partial + ((size_t)(w * 2 + s) * 32 + lane) * (8 * TT);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int tt = 0; tt < TT; ++tt) {
                const float4 f = ldcg_f4(src + (h * TT + tt) * 4);
                sum[h][tt][0] += f.x;
                sum[h][tt][1] += f.y;
                sum[h][tt][2] += f.z;
                sum[h][tt][3] += f.w;
            }
    }
    store_tile_y<TT>(p, tile, sum, g, t);
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

template <int TT, int GM>
__global__ void __launch_bounds__(kWarps * 32, 2) w4a16_stream_kernel(const Params p)
{
    using MD = Mode<GM>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    pdl_launch_dependents();
    if (gw >= p.Wt)
        return;  // the kernel has no CTA-wide barrier
    const int g = lane >> 2, t = lane & 3;

    uint8_t *ring = smem + (size_t)warp * kWarpSmem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + kRing * kStageBytes);

    const int u0 = run_start(p, gw);
    const int u1 = run_start(p, gw + 1);
    const int nstages = (u1 - u0 + MD::kUnitsPerStage - 1) / MD::kUnitsPerStage;

    // lane 0 owns the ring: source pointers advance by one stage per issue
    const uint8_t *csrc = p.codes + (size_t)u0 * (MD::kChunks * 1024);
    const uint8_t *ssrc = p.scales + (size_t)u0 * (MD::kGroups * 64);
    int left = u1 - u0;  // units not yet requested
    uint64_t policy = 0;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kRing; ++s)
            mbar_init(&bars[s], 1);
        fence_barrier_init();
        policy = l2_policy_evict_first();
        // while the previous kernel drains: pull the first stages into L2
        {
            const int nu = min(kRing * MD::kUnitsPerStage, left);
            prefetch_l2(csrc, nu * MD::kChunks * 1024);
            prefetch_l2(ssrc, nu * MD::kGroups * 64);
        }
    }
    pdl_wait();
    if (lane == 0) {
        for (int s = 0; s < min(kRing, nstages); ++s) {
            const int nu = min(MD::kUnitsPerStage, left);
            const uint32_t cb = nu * MD::kChunks * 1024, sb = nu * MD::kGroups * 64;
            uint8_t *dst = ring + s * kStageBytes;
            mbar_arrive_expect_tx(&bars[s], cb + sb);
            bulk_g2s(dst, csrc, cb, &bars[s], policy);
            bulk_g2s(dst + kStageCode, ssrc, sb, &bars[s], policy);
            csrc += cb;
            ssrc += sb;
            left -= nu;
        }
    }
    __syncwarp();

    // activation rows of this lane: m = g + 8 tt; the lane reads k = 4t .. 4t+3
    // of every k16 step
    const uint16_t *xrow[TT];
    bool xvalid[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
        const int m = tt * 8 + g;
        xvalid[tt] = m < p.M;
        xrow[tt] = p.X + (size_t)(xvalid[tt] ? m : 0) * p.K + 4 * t;
    }

    float acc[2][TT][4], part[2][TT][4];
    zero_acc<TT>(acc);
    bool first_cut = false;  // the run's first segment ended inside the run, cut
    int first_tile = 0;

    int tile = u0 / p.upt;
    int lu = u0 - tile * p.upt;            // unit inside the tile
    const int kchunks = p.K / 64;
    int kc = lu * MD::kChunks;             // chunk inside the tile
    int seg_begin = u0;

    // Activation fragments of the stage's two chunks.  For narrow token tiles
    // they are requested one stage ahead (a whole stage of work hides their
    // L2 latency); wide token tiles load them per chunk.
    constexpr bool kPipeX = TT <= 2;
    auto inc = [&](int k) { return (k + 1 == kchunks) ? 0 : k + 1; };
    uint2 xs[2][TT][4], xn[2][TT][4];
    auto load_x = [&](uint2 (&dst)[2][TT][4], int slot_x, int chunk) {
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint2 v = make_uint2(0, 0);
                if (xvalid[tt])
                    v = __ldg(reinterpret_cast<const uint2 *>(xrow[tt] + chunk * 64 + 16 * j));
                dst[slot_x][tt][j] = v;
            }
    };
    if (kPipeX) {
        load_x(xs, 0, kc);
        load_x(xs, 1, inc(kc));
    }

    for (int s = 0; s < nstages; ++s) {
        const int slot = s % kRing;
        const uint8_t *stage = ring + slot * kStageBytes;
        const int kc1 = inc(kc);
        if (kPipeX) {
            if (s + 1 < nstages) {
                const int kn0 = inc(kc1);
                load_x(xn, 0, kn0);
                load_x(xn, 1, inc(kn0));
            }
        } else {
            load_x(xs, 0, kc);
        }
        if (!mbar_wait(&bars[slot], (s / kRing) & 1, kWaitLimitNs)) {
            if (lane == 0)
                record_error(p.hdr, MXG_ERR_TIMEOUT, 100 + GM);
            for (int r = s + 1; r < min(s + kRing, nstages); ++r)
                mbar_wait(&bars[r % kRing], (r / kRing) & 1, kWaitLimitNs / 16);
            return;
        }
#pragma unroll
        for (int iu = 0; iu < MD::kUnitsPerStage; ++iu) {
            const int u = u0 + s * MD::kUnitsPerStage + iu;
            if (iu > 0 && u >= u1)
                break;
#pragma unroll
            for (int ch = 0; ch < MD::kChunks; ++ch) {
                const int c2 = iu * MD::kChunks + ch;  // chunk inside the stage
                const int xi = kPipeX ? c2 : 0;
                if (!kPipeX && c2 == 1)
                    load_x(xs, 0, kc1);
                const uint8_t *cp = stage + c2 * 1024 + lane * 16;
                const uint4 wl = lds128(cp);
                const uint4 wh = lds128(cp + 512);
                const uint32_t w[2][4] = {{wl.x, wl.y, wl.z, wl.w}, {wh.x, wh.y, wh.z, wh.w}};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int step = ch * 4 + j;  // k16 step inside the unit
                    const bool first = (step % MD::kStepsPerGroup) == 0;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t a0 = int4_pair_minus8<0>(w[h][j]);
                        const uint32_t a1 = int4_pair_minus8<4>(w[h][j]);
                        const uint32_t a2 = int4_pair_minus8<8>(w[h][j]);
                        const uint32_t a3 = int4_pair_minus8<12>(w[h][j]);
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt) {
                            if (first)
                                mma_bf16_16816_zero(part[h][tt], a0, a1, a2, a3,
                                                    xs[xi][tt][j].x, xs[xi][tt][j].y);
                            else
                                mma_bf16_16816(part[h][tt], a0, a1, a2, a3, xs[xi][tt][j].x,
                                               xs[xi][tt][j].y);
                        }
                    }
                    if ((step + 1) % MD::kStepsPerGroup == 0) {
                        // end of a scale group: acc += part * scale (fp32)
                        const int gi = step / MD::kStepsPerGroup;  // group inside the unit
                        const uint2 sv =
                            lds64(stage + kStageCode + (iu * MD::kGroups + gi) * 64 + g * 8);
                        const float2 s01 = __half22float2(*reinterpret_cast<const __half2 *>(&sv.x));
                        const float2 s23 = __half22float2(*reinterpret_cast<const __half2 *>(&sv.y));
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt) {
                            acc[0][tt][0] = fmaf(part[0][tt][0], s01.x, acc[0][tt][0]);
                            acc[0][tt][1] = fmaf(part[0][tt][1], s01.x, acc[0][tt][1]);
                            acc[0][tt][2] = fmaf(part[0][tt][2], s01.y, acc[0][tt][2]);
                            acc[0][tt][3] = fmaf(part[0][tt][3], s01.y, acc[0][tt][3]);
                            acc[1][tt][0] = fmaf(part[1][tt][0], s23.x, acc[1][tt][0]);
                            acc[1][tt][1] = fmaf(part[1][tt][1], s23.x, acc[1][tt][1]);
                            acc[1][tt][2] = fmaf(part[1][tt][2], s23.y, acc[1][tt][2]);
                            acc[1][tt][3] = fmaf(part[1][tt][3], s23.y, acc[1][tt][3]);
                        }
                    }
                }
                kc = (kc + 1 == kchunks) ? 0 : kc + 1;
            }
            if (++lu == p.upt) {
                // a tile ends inside the run
                if (seg_begin == tile * p.upt) {
                    store_tile_y<TT>(p, tile, acc, g, t);   // whole tile: write it now
                } else {
                    // the run's first segment, cut: park it in slot 0 now, announce it
                    // at the end of the run
                    store_partial<TT>(p, gw, 0, lane, acc);
                    first_cut = true;
                    first_tile = tile;
                }
                zero_acc<TT>(acc);
                ++tile;
                lu = 0;
                seg_begin = u + 1;
            }
        }
        if (kPipeX) {
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
                for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        xs[c2][tt][j] = xn[c2][tt][j];
        }
        // every lane's reads of this slot have returned (their values are
        // consumed above), so the slot can be refilled
        __syncwarp();
        if (lane == 0 && left > 0) {
            const int nu = min(MD::kUnitsPerStage, left);
            const uint32_t cb = nu * MD::kChunks * 1024, sb = nu * MD::kGroups * 64;
            uint8_t *dst = ring + slot * kStageBytes;
            mbar_arrive_expect_tx(&bars[slot], cb + sb);
            bulk_g2s(dst, csrc, cb, &bars[slot], policy);
            bulk_g2s(dst + kStageCode, ssrc, sb, &bars[slot], policy);
            csrc += cb;
            ssrc += sb;
            left -= nu;
        }
    }

    // publish the cut segments: the first one (slot 0) and the last one
    // (slot 0 if it is also the first segment of the run, else slot 1)
    const bool last_cut = seg_begin < u1;
    if (last_cut)
        store_partial<TT>(p, gw, seg_begin == u0 ? 0 : 1, lane, acc);
    if (!first_cut && !last_cut)
        return;
    __syncwarp();
    int arrivals[2] = {0, 0};
    if (lane == 0) {
        if (first_cut)
            arrivals[0] = atomic_add_acq_rel(&p.counters[first_tile], 1);
        if (last_cut)
            arrivals[1] = atomic_add_acq_rel(&p.counters[tile], 1);
    }
    arrivals[0] = __shfl_sync(0xffffffffu, arrivals[0], 0);
    arrivals[1] = __shfl_sync(0xffffffffu, arrivals[1], 0);
    if (first_cut) {
        const int wf = warp_of_unit(p, first_tile * p.upt);
        const int wl = warp_of_unit(p, first_tile * p.upt + p.upt - 1);
        if (arrivals[0] == wl - wf)
            reduce_tile<TT>(p, first_tile, lane);
    }
    if (last_cut) {
        const int wf = warp_of_unit(p, tile * p.upt);
        const int wl = warp_of_unit(p, tile * p.upt + p.upt - 1);
        if (arrivals[1] == wl - wf)
            reduce_tile<TT>(p, tile, lane);
    }
}

template <int TT, int GM>
const void *kernel_ptr()
{
    return reinterpret_cast<const void *>(&w4a16_stream_kernel<TT, GM>);
}

const void *select_kernel(int tt, int gm)
{
#define MXG_CASE(T, G_) \
    if (tt == T && gm == G_) return kernel_ptr<T, G_>();
    MXG_CASE(1, 0) MXG_CASE(1, 1) MXG_CASE(1, 2)
    MXG_CASE(2, 0) MXG_CASE(2, 1) MXG_CASE(2, 2)
    MXG_CASE(3, 0) MXG_CASE(3, 1) MXG_CASE(3, 2)
    MXG_CASE(4, 0) MXG_CASE(4, 1) MXG_CASE(4, 2)
#undef MXG_CASE
    return nullptr;
}

int group_mode(int G)
{
    return G == 128 ? 0 : (G == 64 ? 1 : 2);
}

}  // namespace

bool plan_w4a16_stream(int device, int M, int N, int K, int G, StreamPlan *plan)
{
    if (M < 1 || M > 32 || N % 32 != 0)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    pl.variant = group_mode(G);
    pl.warps_per_cta = kWarps;
    pl.smem = (size_t)kWarps * kWarpSmem;
    const int unit_k = std::max(G, 64);
    pl.upt = K / unit_k;
    pl.ntiles = N / 32;
    if ((size_t)pl.ntiles > kMaxCounters)
        return false;
    pl.units = (long long)pl.ntiles * pl.upt;
    if (pl.units > (1LL << 30))
        return false;
    const void *fn = select_kernel(pl.tt, pl.variant);
    if (!fn)
        return false;
    static int occ_cache[4][3] = {};
    int &occ = occ_cache[pl.tt - 1][pl.variant];
    if (occ == 0) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) !=
            cudaSuccess)
            return false;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, kWarps * 32, pl.smem) !=
                cudaSuccess ||
            o < 1)
            return false;
        occ = o;
    }
    // enough warps to fill the GPU, but no run shorter than kMinStages stages
    const int units_per_stage = 2 / (unit_k / 64);
    const long long min_units = (long long)kMinStages * units_per_stage;
    const long long max_warps = (long long)di.sms * occ * kWarps;
    pl.Wt = (int)std::max<long long>(1, std::min<long long>(max_warps, pl.units / min_units));
    pl.grid = (pl.Wt + kWarps - 1) / kWarps;
    pl.partial_bytes = (size_t)pl.Wt * 2 * 32 * 2 * 4 * pl.tt * sizeof(float);
    *plan = pl;
    return true;
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
    p.scales = p.codes + (size_t)N * K / 2;
    p.Y = static_cast<uint16_t *>(Y);
    p.hdr = static_cast<WsHeader *>(workspace);
    p.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wm.counters_off);
    p.partial = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + wm.partial_off);
    p.M = M;
    p.N = N;
    p.K = K;
    p.upt = pl.upt;
    p.units = (int)pl.units;
    p.Wt = pl.Wt;
    p.q = (int)(pl.units / pl.Wt);
    p.r = (int)(pl.units % pl.Wt);
    void *args[] = {&p};
    return launch_pdl(fn, dim3(pl.grid), dim3(kWarps * 32), pl.smem, stream, args);
}

}  // namespace mxg
