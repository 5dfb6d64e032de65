// INT4 W4A16 weight-streaming GEMM for small M (decode / MTP verify chunks).
//
// At M <= 32 the layer reads each weight byte once and does 2*M flops per
// weight: it is bound by HBM bytes of W.  The kernel therefore
//  * cuts the re-packed weight stream into equal units (one n16 tile x one
//    scale group) and gives every warp of a persistent grid one contiguous
//    run of units (stream-K), so all SMs stream the same number of bytes;
//  * moves each warp's run through its own ring of shared-memory stages with
//    1-D bulk copies (cp.async.bulk, completion on an mbarrier), several
//    stages in flight per warp, weights marked evict-first in L2;
//  * decodes nibbles to exact bf16 (q - 8) in registers (mask/or + one
//    bf16x2 fma per two weights) and multiplies on the tensor cores with
//    m16n8k16 MMAs where the weights are the 16-row operand and the tokens
//    the 8-column operand ("swap AB"), so M = 1..8 costs one MMA per 256
//    weights;
//  * applies the fp16 group scale once per group to the fp32 partial sum
//    (G = 64, 128), or folds it into the bf16 weight with one rounding
//    (G = 32, whose groups are narrower than one MMA's k span);
//  * reduces the partial sums of n16 tiles shared by several warps through
//    the workspace: each contributor stores its fragment, bumps the tile's
//    arrival counter, and the last one adds all fragments in warp order
//    (deterministic) and writes bf16 Y.  Nobody waits on anybody.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

constexpr int kWarps = 8;        // warps per CTA
constexpr int kRing = 4;         // stages per warp
constexpr int kStageCode = 2048; // code bytes per stage
constexpr int kStageScale = 256; // scale bytes reserved per stage
constexpr int kStageBytes = kStageCode + kStageScale;
constexpr int kWarpSmem = kRing * kStageBytes + kRing * 8;

// Group modes: 0 -> G = 128 (unit = 2 chunks, 1 scale row), 1 -> G = 64
// (unit = 1 chunk, 1 scale row), 2 -> G = 32 (unit = 1 chunk, 2 scale rows).
template <int GM>
struct Mode {
    static constexpr int kChunks = (GM == 0) ? 2 : 1;       // k64 chunks per unit
    static constexpr int kScaleRows = (GM == 2) ? 2 : 1;    // 32-byte scale rows per unit
    static constexpr int kUnitsPerStage = kStageCode / (kChunks * 512);
    static constexpr bool kPostScale = (GM != 2);
};

struct Params {
    const uint16_t *X;       // bf16 [M][K]
    const uint8_t *codes;    // re-packed codes
    const uint8_t *scales;   // re-packed scales
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [N/16]
    float *partial;          // [Wt][2][32][4*TT]
    int M, N, K;
    int upt;                 // units per n16 tile
    long long units;
    int Wt;
};

__device__ __forceinline__ long long run_start(long long w, long long units, int Wt)
{
    return w * units / Wt;
}

// The warp whose run contains unit u.
__device__ __forceinline__ int warp_of_unit(long long u, long long units, int Wt)
{
    return (int)(((u + 1) * (long long)Wt - 1) / units);
}

template <int TT>
__device__ __forceinline__ void store_tile_y(const Params &p, int nt, const float (&v)[TT][4], int g,
                                             int t)
{
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = tt * 8 + 2 * t + (e & 1);
            const int n = nt * 16 + g + ((e & 2) ? 8 : 0);
            if (m < p.M)
                p.Y[(size_t)m * p.N + n] = f32_to_bf16_bits(v[tt][e]);
        }
}

// Finish the segment [seg_begin, seg_end) of n16 tile nt held in acc.
template <int TT>
__device__ __forceinline__ void flush_segment(const Params &p, int gw, int lane, long long nt,
                                              long long seg_begin, long long seg_end,
                                              long long run_begin, float (&acc)[TT][4])
{
    const int g = lane >> 2, t = lane & 3;
    const long long tile_begin = nt * p.upt, tile_end = tile_begin + p.upt;
    if (seg_begin == tile_begin && seg_end == tile_end) {
        store_tile_y<TT>(p, (int)nt, acc, g, t);
        return;
    }
    const int slot = (seg_begin == run_begin) ? 0 : 1;
    float *dst = p.partial + ((size_t)(gw * 2 + slot) * 32 + lane) * (4 * TT);
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
        __stcg(reinterpret_cast<float4 *>(dst + 4 * tt),
               make_float4(acc[tt][0], acc[tt][1], acc[tt][2], acc[tt][3]));
    __threadfence();
    __syncwarp();
    int old = 0;
    if (lane == 0)
        old = atomicAdd(&p.counters[nt], 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    const int w_first = warp_of_unit(tile_begin, p.units, p.Wt);
    const int w_last = warp_of_unit(tile_end - 1, p.units, p.Wt);
    if (old != w_last - w_first)
        return;
    // last contributor: add every fragment of this tile in warp order
    __threadfence();
    float sum[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            sum[tt][e] = 0.f;
    for (int w = w_first; w <= w_last; ++w) {
        const int s = (run_start(w, p.units, p.Wt) >= tile_begin) ? 0 : 1;
        const float *src = p.partial + ((size_t)(w * 2 + s) * 32 + lane) * (4 * TT);
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            const float4 f = ldcg_f4(src + 4 * tt);
            sum[tt][0] += f.x;
            sum[tt][1] += f.y;
            sum[tt][2] += f.z;
            sum[tt][3] += f.w;
        }
    }
    store_tile_y<TT>(p, (int)nt, sum, g, t);
    if (lane == 0)
        p.counters[nt] = 0;  // leave the workspace zeroed for the next call
}

template <int TT, int GM>
__global__ void __launch_bounds__(kWarps * 32) w4a16_stream_kernel(const Params p)
{
    using MD = Mode<GM>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    if (gw >= p.Wt)
        return;  // the kernel has no CTA-wide barrier
    const int g = lane >> 2, t = lane & 3;

    uint8_t *ring = smem + (size_t)warp * kWarpSmem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + kRing * kStageBytes);

    const long long u0 = run_start(gw, p.units, p.Wt);
    const long long u1 = run_start(gw + 1, p.units, p.Wt);
    const int nstages = (int)((u1 - u0 + MD::kUnitsPerStage - 1) / MD::kUnitsPerStage);

    uint64_t policy = 0;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kRing; ++s)
            mbar_init(&bars[s], 1);
        fence_barrier_init();
        policy = l2_policy_evict_first();
    }
    __syncwarp();

    auto issue = [&](int s) {
        const int slot = s % kRing;
        const long long ub = u0 + (long long)s * MD::kUnitsPerStage;
        const int nu = (int)min((long long)MD::kUnitsPerStage, u1 - ub);
        const uint32_t cbytes = nu * MD::kChunks * 512;
        const uint32_t sbytes = nu * MD::kScaleRows * 32;
        uint8_t *dst = ring + slot * kStageBytes;
        mbar_arrive_expect_tx(&bars[slot], cbytes + sbytes);
        bulk_g2s(dst, p.codes + ub * (MD::kChunks * 512), cbytes, &bars[slot], policy);
        bulk_g2s(dst + kStageCode, p.scales + ub * (MD::kScaleRows * 32), sbytes, &bars[slot],
                 policy);
    };

    if (lane == 0)
        for (int s = 0; s < min(kRing, nstages); ++s)
            issue(s);

    float acc[TT][4];
    float part[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            acc[tt][e] = part[tt][e] = 0.f;

    long long cur_nt = u0 / p.upt;
    long long seg_begin = u0;
    const uint16_t *xrow[TT];
    bool xvalid[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
        const int m = tt * 8 + g;
        xvalid[tt] = m < p.M;
        xrow[tt] = p.X + (size_t)(xvalid[tt] ? m : 0) * p.K;
    }

    for (int s = 0; s < nstages; ++s) {
        const int slot = s % kRing;
        if (!mbar_wait(&bars[slot], (s / kRing) & 1, kWaitLimitNs)) {
            if (lane == 0)
                record_error(p.hdr, MXG_ERR_TIMEOUT, 100 + GM);
            // give the copies still in flight a bounded chance to land
            for (int r = s + 1; r < min(s + kRing, nstages); ++r)
                mbar_wait(&bars[r % kRing], (r / kRing) & 1, kWaitLimitNs / 16);
            return;
        }
        const uint8_t *stage = ring + slot * kStageBytes;
        const long long ub = u0 + (long long)s * MD::kUnitsPerStage;
#pragma unroll
        for (int iu = 0; iu < MD::kUnitsPerStage; ++iu) {
            const long long u = ub + iu;
            if (u >= u1)
                break;
            const long long nt = u / p.upt;
            if (nt != cur_nt) {
                flush_segment<TT>(p, gw, lane, cur_nt, seg_begin, u, u0, acc);
#pragma unroll
                for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[tt][e] = 0.f;
                cur_nt = nt;
                seg_begin = u;
            }
            const int lu = (int)(u - nt * p.upt);
            const uint8_t *sc = stage + kStageCode + iu * (MD::kScaleRows * 32);
#pragma unroll
            for (int ch = 0; ch < MD::kChunks; ++ch) {
                const int kc = lu * MD::kChunks + ch;          // chunk inside the tile
                const int kl = kc * 64 + t * 16;               // lane's first k
                uint32_t xb[TT][8];
#pragma unroll
                for (int tt = 0; tt < TT; ++tt) {
                    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
                    if (xvalid[tt]) {
                        x0 = ldg128(xrow[tt] + kl);
                        x1 = ldg128(xrow[tt] + kl + 8);
                    }
                    xb[tt][0] = x0.x; xb[tt][1] = x0.y; xb[tt][2] = x0.z; xb[tt][3] = x0.w;
                    xb[tt][4] = x1.x; xb[tt][5] = x1.y; xb[tt][6] = x1.z; xb[tt][7] = x1.w;
                }
                const uint4 wv = lds128(stage + (iu * MD::kChunks + ch) * 512 + lane * 16);
                const uint32_t wj[4] = {wv.x, wv.y, wv.z, wv.w};
                if constexpr (MD::kPostScale) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t a0 = int4_pair_minus8<0>(wj[j]);
                        const uint32_t a1 = int4_pair_minus8<4>(wj[j]);
                        const uint32_t a2 = int4_pair_minus8<8>(wj[j]);
                        const uint32_t a3 = int4_pair_minus8<12>(wj[j]);
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt)
                            mma_bf16_16816(part[tt], a0, a1, a2, a3, xb[tt][2 * j], xb[tt][2 * j + 1]);
                    }
                } else {
                    // G = 32: this lane's 16 rows are in scale row t / 2 of the unit
                    const uint32_t sw = lds32(sc + (t >> 1) * 32 + g * 4);
                    const ScaleSplit sa = split_scale((uint16_t)(sw & 0xFFFF));
                    const ScaleSplit sb = split_scale((uint16_t)(sw >> 16));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t a0 = scale_pair_rn(int4_pair_minus8<0>(wj[j]), sa);
                        const uint32_t a1 = scale_pair_rn(int4_pair_minus8<4>(wj[j]), sb);
                        const uint32_t a2 = scale_pair_rn(int4_pair_minus8<8>(wj[j]), sa);
                        const uint32_t a3 = scale_pair_rn(int4_pair_minus8<12>(wj[j]), sb);
#pragma unroll
                        for (int tt = 0; tt < TT; ++tt)
                            mma_bf16_16816(acc[tt], a0, a1, a2, a3, xb[tt][2 * j], xb[tt][2 * j + 1]);
                    }
                }
            }
            if constexpr (MD::kPostScale) {
                const uint32_t sw = lds32(sc + g * 4);
                const float sa = __half2float(__ushort_as_half((uint16_t)(sw & 0xFFFF)));
                const float sb = __half2float(__ushort_as_half((uint16_t)(sw >> 16)));
#pragma unroll
                for (int tt = 0; tt < TT; ++tt) {
                    acc[tt][0] = fmaf(part[tt][0], sa, acc[tt][0]);
                    acc[tt][1] = fmaf(part[tt][1], sa, acc[tt][1]);
                    acc[tt][2] = fmaf(part[tt][2], sb, acc[tt][2]);
                    acc[tt][3] = fmaf(part[tt][3], sb, acc[tt][3]);
                    part[tt][0] = part[tt][1] = part[tt][2] = part[tt][3] = 0.f;
                }
            }
        }
        __syncwarp();
        if (lane == 0 && s + kRing < nstages) {
            fence_proxy_async_smem();  // our reads of this slot precede the next copy into it
            issue(s + kRing);
        }
    }
    flush_segment<TT>(p, gw, lane, cur_nt, seg_begin, u1, u0, acc);
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
    if (M < 1 || M > 32)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    pl.variant = group_mode(G);
    pl.warps_per_cta = kWarps;
    pl.smem = (size_t)kWarps * kWarpSmem;
    const int unit_k = std::max(G, 64);
    pl.upt = K / unit_k;
    pl.ntiles = N / 16;
    pl.units = (long long)pl.ntiles * pl.upt;
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
    const long long max_warps = (long long)di.sms * occ * kWarps;
    pl.Wt = (int)std::min<long long>(max_warps, pl.units);
    pl.grid = (pl.Wt + kWarps - 1) / kWarps;
    pl.partial_bytes = (size_t)pl.Wt * 2 * 32 * 4 * pl.tt * sizeof(float);
    *plan = pl;
    return true;
}

cudaError_t launch_w4a16_stream(const StreamPlan &pl, const void *X, const void *packed, int M,
                                int N, int K, int G, void *Y, void *workspace, cudaStream_t stream)
{
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
    p.units = pl.units;
    p.Wt = pl.Wt;
    void *args[] = {&p};
    return cudaLaunchKernel(fn, dim3(pl.grid), dim3(kWarps * 32), args, pl.smem, stream);
}

}  // namespace mxg
