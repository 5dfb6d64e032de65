// MXFP8 weight-streaming GEMM for small M.
//
// Same structure as the INT4 streaming kernel: stream-K over units, one
// shared-memory ring per warp, swap-AB m16n8k16 MMAs, last-arriver reduction
// of shared tiles.  Differences:
//  * the weights are consumed in their stored layout, Wq[N][K] (no re-pack):
//    a unit is one n16 tile x 128 k, fetched as a 2-D tensor-map box of
//    16 rows x 128 bytes with the 128-byte swizzle (conflict-free 16-byte
//    shared loads by lane g of row g and row g + 8); rows past N and columns
//    past K are zero-filled by the copy engine;
//  * lane t of a unit owns k = 32t .. 32t + 31 of rows g and g + 8, which is
//    exactly one E8M0 block, so each lane needs two scales per unit, loaded
//    one stage ahead into registers;
//  * E4M3 -> bf16 with the block scale folded in (exact for normal bf16
//    results): hardware e4m3x2 -> f16x2, f16 -> f32, times 2^(E-127), one
//    rounding to bf16.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

constexpr int kWarps = 8;
constexpr int kRing = 6;                  // stages per warp
constexpr int kStage = 2048;              // one 16 x 128-byte box
constexpr int kWarpSmem = kRing * kStage;
constexpr int kMinUnits = 6;              // shortest run per warp

struct Params {
    const uint16_t *X;       // bf16 [M][K]
    const uint8_t *Ws;       // E8M0 [N][K/32]
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [ceil(N/16)]
    float *partial;          // [Wt][2][32][4*TT]
    int M, N, K;
    int upt;                 // units per n16 tile = ceil(K / 128)
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
    const int big = p.r * (p.q + 1);
    return u < big ? u / (p.q + 1) : p.r + (u - big) / p.q;
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
            if (m < p.M && n < p.N)
                p.Y[(size_t)m * p.N + n] = f32_to_bf16_bits(v[tt][e]);
        }
}

template <int TT>
__device__ __forceinline__ void store_partial(const Params &p, int gw, int slot, int lane,
                                              const float (&v)[TT][4])
{
    float *dst = p.partial + ((size_t)(gw * 2 + slot) * 32 + lane) * (4 * TT);
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
        __stcg(reinterpret_cast<float4 *>(dst + 4 * tt),
               make_float4(v[tt][0], v[tt][1], v[tt][2], v[tt][3]));
}

// Run by the last contributor of a cut tile: add every fragment of the tile
// in warp order and write bf16 Y.
template <int TT>
__device__ __noinline__ void reduce_tile(const Params &p, int nt, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    const int tile_begin = nt * p.upt, tile_end = tile_begin + p.upt;
    const int w_first = warp_of_unit(p, tile_begin);
    const int w_last = warp_of_unit(p, tile_end - 1);
    float sum[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            sum[tt][e] = 0.f;
#pragma unroll 4
    for (int w = w_first; w <= w_last; ++w) {
        const int s = (run_start(p, w) >= tile_begin) ? 0 : 1;
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
    store_tile_y<TT>(p, nt, sum, g, t);
    if (lane == 0)
        p.counters[nt] = 0;
}

// The E8M0 scales of one unit for lane (g, t): rows g and g + 8, block t.
struct UnitScales {
    float a, b;
};

__device__ __forceinline__ UnitScales load_unit_scales(const Params &p, int tile, int kb, int g,
                                                       int t)
{
    const int blocks = p.K / 32;
    const int blk = kb * 4 + t;
    const int ra = tile * 16 + g, rb = ra + 8;
    uint32_t ea = 127, eb = 127;  // any finite scale for zero-filled weights
    if (blk < blocks) {
        if (ra < p.N)
            ea = __ldg(p.Ws + (size_t)ra * blocks + blk);
        if (rb < p.N)
            eb = __ldg(p.Ws + (size_t)rb * blocks + blk);
    }
    return UnitScales{e8m0_to_f32(ea), e8m0_to_f32(eb)};
}

template <int TT>
__global__ void __launch_bounds__(kWarps * 32)
    mxfp8_stream_kernel(const __grid_constant__ CUtensorMap wq_map, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    // the 128-byte swizzle pattern needs 1024-byte aligned boxes
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    pdl_launch_dependents();
    if (gw >= p.Wt)
        return;
    const int g = lane >> 2, t = lane & 3;
    uint8_t *ring = smem + (size_t)warp * kWarpSmem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kWarps * kWarpSmem) + warp * kRing;

    const int u0 = run_start(p, gw);
    const int u1 = run_start(p, gw + 1);
    const int nstages = u1 - u0;
    int tile = u0 / p.upt;
    int kb = u0 - tile * p.upt;

    // lane 0 owns the ring; (itile, ikb) is the next unit to fetch
    int itile = tile, ikb = kb;
    uint64_t policy = 0;
    if (lane == 0) {
        prefetch_tensormap(&wq_map);
#pragma unroll
        for (int s = 0; s < kRing; ++s)
            mbar_init(&bars[s], 1);
        fence_barrier_init();
        policy = l2_policy_evict_first();
        // while the previous kernel drains: pull the first units into L2
        {
            int pt = tile, pk = kb;
            for (int s = 0; s < min(kRing, nstages); ++s) {
                prefetch_tensor_l2(&wq_map, pk * 128, pt * 16);
                if (++pk == p.upt) {
                    pk = 0;
                    ++pt;
                }
            }
        }
    }
    pdl_wait();
    if (lane == 0) {
        for (int s = 0; s < min(kRing, nstages); ++s) {
            mbar_arrive_expect_tx(&bars[s], kStage);
            tma_load_2d(ring + s * kStage, &wq_map, ikb * 128, itile * 16, &bars[s], policy);
            if (++ikb == p.upt) {
                ikb = 0;
                ++itile;
            }
        }
    }
    __syncwarp();

    float acc[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            acc[tt][e] = 0.f;
    bool first_cut = false;
    int first_tile = 0;
    int seg_begin = u0;

    const uint16_t *xrow[TT];
    bool xvalid[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
        const int m = tt * 8 + g;
        xvalid[tt] = m < p.M;
        xrow[tt] = p.X + (size_t)(xvalid[tt] ? m : 0) * p.K;
    }
    UnitScales sc_next = load_unit_scales(p, tile, kb, g, t);
    // activation fragment of unit column kb: lane (g, t) takes k = 128 kb + 32t .. +31
    constexpr bool kPipeX = TT <= 2;
    auto load_x = [&](uint32_t (&dst)[TT][16], int kbx) {
        const int kl = kbx * 128 + t * 32;
        const bool kvalid = kl < p.K;
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (xvalid[tt] && kvalid)
                    v = ldg128(xrow[tt] + kl + 8 * q);
                dst[tt][4 * q + 0] = v.x;
                dst[tt][4 * q + 1] = v.y;
                dst[tt][4 * q + 2] = v.z;
                dst[tt][4 * q + 3] = v.w;
            }
        }
    };
    uint32_t xn[TT][16];
    if (kPipeX)
        load_x(xn, kb);
    const int c_lo = ((2 * t) ^ g) * 16, c_hi = ((2 * t + 1) ^ g) * 16;

    for (int s = 0; s < nstages; ++s) {
        const int u = u0 + s;
        const UnitScales sc = sc_next;
        if (s + 1 < nstages) {
            // scales of the next unit, one unit ahead
            const bool wrap = kb + 1 == p.upt;
            sc_next = load_unit_scales(p, wrap ? tile + 1 : tile, wrap ? 0 : kb + 1, g, t);
        }
        // activations of this unit (requested one unit ahead for narrow token tiles)
        uint32_t xb[TT][16];
        if (kPipeX) {
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    xb[tt][i] = xn[tt][i];
            if (s + 1 < nstages)
                load_x(xn, kb + 1 == p.upt ? 0 : kb + 1);
        } else {
            load_x(xb, kb);
        }
        const int slot = s % kRing;
        if (!mbar_wait(&bars[slot], (s / kRing) & 1, kWaitLimitNs)) {
            if (lane == 0)
                record_error(p.hdr, MXG_ERR_TIMEOUT, 200);
            for (int r = s + 1; r < min(s + kRing, nstages); ++r)
                mbar_wait(&bars[r % kRing], (r / kRing) & 1, kWaitLimitNs / 16);
            return;
        }
        const uint8_t *stage = ring + slot * kStage;
        const uint4 ra0 = lds128(stage + g * 128 + c_lo);
        const uint4 ra1 = lds128(stage + g * 128 + c_hi);
        const uint4 rb0 = lds128(stage + (g + 8) * 128 + c_lo);
        const uint4 rb1 = lds128(stage + (g + 8) * 128 + c_hi);
        const uint32_t wa[8] = {ra0.x, ra0.y, ra0.z, ra0.w, ra1.x, ra1.y, ra1.z, ra1.w};
        const uint32_t wb[8] = {rb0.x, rb0.y, rb0.z, rb0.w, rb1.x, rb1.y, rb1.z, rb1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t a0, a1, a2, a3;
            e4m3x4_scaled(wa[j], sc.a, a0, a2);
            e4m3x4_scaled(wb[j], sc.b, a1, a3);
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
                mma_bf16_16816(acc[tt], a0, a1, a2, a3, xb[tt][2 * j], xb[tt][2 * j + 1]);
        }
        // every lane's reads of this slot have returned, so it can be refilled
        __syncwarp();
        if (lane == 0 && s + kRing < nstages) {
            mbar_arrive_expect_tx(&bars[slot], kStage);
            tma_load_2d(ring + slot * kStage, &wq_map, ikb * 128, itile * 16, &bars[slot], policy);
            if (++ikb == p.upt) {
                ikb = 0;
                ++itile;
            }
        }
        if (++kb == p.upt) {
            // a tile ends inside the run
            if (seg_begin == tile * p.upt) {
                store_tile_y<TT>(p, tile, acc, g, t);
            } else {
                store_partial<TT>(p, gw, 0, lane, acc);
                first_cut = true;
                first_tile = tile;
            }
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[tt][e] = 0.f;
            ++tile;
            kb = 0;
            seg_begin = u + 1;
        }
    }

    // publish the cut segments (see the INT4 streaming kernel)
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

const void *select_kernel(int tt)
{
    switch (tt) {
    case 1: return reinterpret_cast<const void *>(&mxfp8_stream_kernel<1>);
    case 2: return reinterpret_cast<const void *>(&mxfp8_stream_kernel<2>);
    case 3: return reinterpret_cast<const void *>(&mxfp8_stream_kernel<3>);
    case 4: return reinterpret_cast<const void *>(&mxfp8_stream_kernel<4>);
    default: return nullptr;
    }
}

constexpr size_t kSmemBytes = 1024 + (size_t)kWarps * kWarpSmem + (size_t)kWarps * kRing * 8;

}  // namespace

bool plan_mxfp8_stream(int device, int M, int N, int K, StreamPlan *plan)
{
    if (M < 1 || M > 32)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    pl.variant = 0;
    pl.warps_per_cta = kWarps;
    pl.smem = kSmemBytes;
    pl.upt = (K + 127) / 128;
    pl.ntiles = (N + 15) / 16;
    if ((size_t)pl.ntiles > kMaxCounters)
        return false;
    pl.units = (long long)pl.ntiles * pl.upt;
    if (pl.units > (1LL << 30))
        return false;
    const void *fn = select_kernel(pl.tt);
    static int occ_cache[4] = {};
    int &occ = occ_cache[pl.tt - 1];
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
    // no run shorter than kMinUnits units (2 KB each)
    pl.Wt = (int)std::max<long long>(1, std::min<long long>(max_warps, pl.units / kMinUnits));
    pl.grid = (pl.Wt + kWarps - 1) / kWarps;
    pl.partial_bytes = (size_t)pl.Wt * 2 * 32 * 4 * pl.tt * sizeof(float);
    *plan = pl;
    return true;
}

cudaError_t launch_mxfp8_stream(const StreamPlan &pl, const void *X, const uint8_t *Wq,
                                const uint8_t *Ws, int M, int N, int K, void *Y, void *workspace,
                                cudaStream_t stream)
{
    const void *fn = select_kernel(pl.tt);
    if (!fn)
        return cudaErrorInvalidValue;
    alignas(64) CUtensorMap map;
    if (!encode_tensor_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                              (uint64_t)K, 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const WorkspaceMap wm = make_workspace_map(pl.ntiles, pl.partial_bytes);
    Params p{};
    p.X = static_cast<const uint16_t *>(X);
    p.Ws = Ws;
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
    void *args[] = {&map, &p};
    return launch_pdl(fn, dim3(pl.grid), dim3(kWarps * 32), pl.smem, stream, args);
}

}  // namespace mxg
