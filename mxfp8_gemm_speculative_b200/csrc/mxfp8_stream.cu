// MXFP8 weight-streaming GEMM for small M.
//
// Same structure as the INT4 streaming kernel (one contiguous stream-K run
// of units per CTA, units dealt to the CTA's warps in turn, one ring of
// bulk-copied slots per warp, swap-AB m16n8k16 MMAs, non-blocking tile
// reductions through shared memory, cut tiles finished by the CTA holding
// their first unit).  Differences:
//  * the weights are consumed in their stored layout, Wq[N][K] (no re-pack):
//    a unit is one n16 tile x SU * 128 k, fetched as SU 2-D tensor-map boxes
//    of 16 rows x 128 bytes with the 128-byte swizzle (conflict-free 16-byte
//    shared loads by lane g of row g and row g + 8); rows past N and columns
//    past K are zero-filled by the copy engine;
//  * lane t of a box owns k = 32t .. 32t + 31 of rows g and g + 8, which is
//    exactly one E8M0 block, so each lane needs two scales per box, loaded
//    one unit ahead into registers;
//  * E4M3 -> bf16 with the block scale folded in (exact for normal bf16
//    results): hardware e4m3x2 -> f16x2, f16 -> f32, times 2^(E-127), one
//    rounding to bf16.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

#ifndef MXG_MX_SU2_TT
#define MXG_MX_SU2_TT 2
#endif
constexpr int kConsumers = 12;                  // warps per CTA
constexpr int kThreads = kConsumers * 32;
constexpr int kBox = 2048;                      // one 16 x 128-byte box
constexpr int kMinUnitsPerCta = 2 * kConsumers; // shortest run

// A unit (what one ring slot holds) is SU boxes along K of one n16 tile.
template <int SU>
struct Unit {
    static constexpr int kBytes = SU * kBox;
    // ring slots per warp: shallow rings leave most of the SM's
    // shared-memory/L1 split to L1, where the re-read activations hit
    static constexpr int kStages = SU == 2 ? 2 : 3;
};

// Shared memory (1024-byte aligned for the swizzle): every warp's ring,
// kRed reduction buffers of kConsumers fragments, one mbarrier per slot,
// then per reduction buffer an arrival count and a use count.
template <int TT, int SU>
struct Smem {
    static constexpr int kFrag4 = TT * 32;       // float4 per warp fragment
    // one reduction buffer: the smaller footprint leaves a larger L1 for the
    // activation loads (every CTA re-reads X for each of its tiles)
    static constexpr int kRed = 1;
    static constexpr size_t kRingBytes = (size_t)kConsumers * Unit<SU>::kStages * Unit<SU>::kBytes;
    static constexpr size_t kRedOff = kRingBytes;
    static constexpr size_t kBarOff = kRedOff + (size_t)kRed * kConsumers * kFrag4 * 16;
    static constexpr size_t kSyncOff = kBarOff + (size_t)kConsumers * Unit<SU>::kStages * 8;
    static constexpr size_t kTotal = kSyncOff + 2 * kRed * sizeof(int) + 1024;  // + alignment
};

struct Params {
    const uint16_t *X;       // bf16 [M][K]
    const uint8_t *Ws;       // E8M0 [N][K/32]
    uint16_t *Y;             // bf16 [M][N]
    WsHeader *hdr;
    int *counters;           // [ceil(N/16)]
    float4 *partial;         // [ctas][TT][32]: a CTA's fragment of its first, cut tile
    int M, N, K;
    int upt;                 // units per n16 tile
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
    const int big = p.r * (p.q + 1);
    return u < big ? u / (p.q + 1) : p.r + (u - big) / p.q;
}

// Writes the four outputs of fragment float4 tt of `lane` for n16 tile nt.
__device__ __forceinline__ void store_y4(const Params &p, int nt, int tt, int lane, float4 v)
{
    const int g = lane >> 2, t = lane & 3;
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = tt * 8 + 2 * t + (i & 1);
        const int n = nt * 16 + g + ((i & 2) ? 8 : 0);
        if (m < p.M && n < p.N)
            p.Y[(size_t)m * p.N + n] = f32_to_bf16_bits(e[i]);
    }
}

// Sum of the kConsumers warp fragments (warp order) for this lane.
template <int TT>
__device__ __forceinline__ void sum_fragments(const float4 *frags, int lane, float4 (&sum)[TT])
{
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
        sum[tt] = frags[tt * 32 + lane];
        for (int w = 1; w < kConsumers; ++w) {
            const float4 v = frags[w * TT * 32 + tt * 32 + lane];
            sum[tt].x += v.x;
            sum[tt].y += v.y;
            sum[tt].z += v.z;
            sum[tt].w += v.w;
        }
    }
}

// Run by one warp of a CTA whose segment of tile `nt` is cut (see the INT4
// streaming kernel): the CTA holding the tile's first unit finishes it last
// in its run and adds the other contributors' fragments in CTA order; every
// other contributor publishes its fragment early without waiting.
template <int TT>
__device__ __noinline__ void finish_cut_tile(const Params &p, const float4 *frags, int c, int nt,
                                             int lane)
{
    float4 sum[TT];
    sum_fragments<TT>(frags, lane, sum);
    const int tile_begin = nt * p.upt;
    const int c_first = cta_of_unit(p, tile_begin);
    if (c != c_first) {
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
            __stcg(p.partial + ((size_t)c * TT + tt) * 32 + lane, sum[tt]);
        __threadfence();   // every lane's stores, before the warp counts itself
        __syncwarp();
        if (lane == 0)
            atomicAdd(&p.counters[nt], 1);
        return;
    }
    const int c_last = cta_of_unit(p, tile_begin + p.upt - 1);
    if (lane == 0) {
        const unsigned long long t0 = global_ns();
        while (ld_acquire_gpu(&p.counters[nt]) < c_last - c_first) {
            if (global_ns() - t0 > kWaitLimitNs) {
                record_error(p.hdr, MXG_ERR_TIMEOUT, 220);
                break;
            }
            __nanosleep(64);
        }
    }
    __syncwarp();
    __threadfence();
    for (int cc = c_first + 1; cc <= c_last; ++cc) {
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            const float4 f = __ldcg(p.partial + ((size_t)cc * TT + tt) * 32 + lane);
            sum[tt].x += f.x;
            sum[tt].y += f.y;
            sum[tt].z += f.z;
            sum[tt].w += f.w;
        }
    }
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
        store_y4(p, nt, tt, lane, sum[tt]);
    if (lane == 0)
        p.counters[nt] = 0;  // leave the counter zero for the next call
}

// The E8M0 scales of box column kbox (128 k) for lane (g, t): rows g, g + 8,
// block t of the box.
__device__ __forceinline__ float2 box_scales(const Params &p, int nt, int kbox, int g, int t)
{
    const int blocks = p.K / 32;
    const int blk = kbox * 4 + t;
    const int ra = nt * 16 + g, rb = ra + 8;
    uint32_t ea = 127, eb = 127;  // any finite scale for zero-filled weights
    if (blk < blocks) {
        if (ra < p.N)
            ea = __ldg(p.Ws + (size_t)ra * blocks + blk);
        if (rb < p.N)
            eb = __ldg(p.Ws + (size_t)rb * blocks + blk);
    }
    return make_float2(e8m0_to_f32(ea), e8m0_to_f32(eb));
}

// Copies unit u (SU boxes of one n16 tile) into a ring slot.
template <int SU>
__device__ __forceinline__ void fetch_unit(const Params &p, const CUtensorMap *map, uint8_t *slot,
                                           uint64_t *bar, int u, uint64_t policy)
{
    const int nt = u / p.upt, ku = u - nt * p.upt;
    mbar_arrive_expect_tx(bar, Unit<SU>::kBytes);
#pragma unroll
    for (int b = 0; b < SU; ++b)
        tma_load_2d(slot + b * kBox, map, (ku * SU + b) * 128, nt * 16, bar, policy);
}

template <int TT, int SU>
__global__ void __launch_bounds__(kThreads, 1)
    mxfp8_stream_kernel(const __grid_constant__ CUtensorMap wq_map, const Params p)
{
    using SL = Smem<TT, SU>;
    constexpr int kStages = Unit<SU>::kStages;
    extern __shared__ uint8_t smem_raw[];
    // the 128-byte swizzle pattern needs 1024-byte aligned boxes
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float4 *red = reinterpret_cast<float4 *>(smem + SL::kRedOff);
    int *red_count = reinterpret_cast<int *>(smem + SL::kSyncOff);  // arrivals per buffer
    int *red_done = red_count + SL::kRed;                           // reductions per buffer

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    const int c = blockIdx.x;
    const int U0 = run_start(p, c), U1 = run_start(p, c + 1);
    const int n = U1 - U0;
    uint8_t *ring = smem + (size_t)warp * kStages * Unit<SU>::kBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SL::kBarOff) + warp * kStages;
    uint64_t policy = 0;
    if (lane == 0) {
        prefetch_tensormap(&wq_map);
        for (int s = 0; s < kStages; ++s)
            mbar_init(&full[s], 1);
        fence_barrier_init();
        policy = l2_policy_evict_first();
    }
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2 * SL::kRed; ++b)
            red_count[b] = 0;
        // while the previous kernel drains: pull the first units into L2
        for (int k = 0; k < min(kConsumers * kStages, n); ++k) {
            const int u = U0 + k, nt = u / p.upt, ku = u - nt * p.upt;
#pragma unroll
            for (int b = 0; b < SU; ++b)
                prefetch_tensor_l2(&wq_map, (ku * SU + b) * 128, nt * 16);
        }
    }
    __syncthreads();
    // this warp takes units warp, warp + C, ... of the run; its k-th unit
    // goes to slot k mod kStages.  The weights are not written by the
    // previous kernel on the stream (the caller's contract, unless it turned
    // early weight loads off): the first slots fill while that kernel drains.
    auto fill_ring = [&]() {
        if (lane == 0)
            for (int k = 0; k < kStages && warp + k * kConsumers < n; ++k)
                fetch_unit<SU>(p, &wq_map, ring + k * Unit<SU>::kBytes, &full[k],
                               U0 + warp + k * kConsumers, policy);
    };
    if (p.early)
        fill_ring();
    pdl_wait();
    if (!p.early)
        fill_ring();

    const int g = lane >> 2, t = lane & 3;
    const uint16_t *xrow[TT];
    bool xvalid[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
        const int m = tt * 8 + g;
        xvalid[tt] = m < p.M;
        xrow[tt] = p.X + (size_t)(xvalid[tt] ? m : 0) * p.K;
    }
    const int upt = p.upt;
    // activation fragments of one unit: for box b, lane (g, t) takes
    // k = 128 (SU ku + b) + 32t .. +31; requested one unit ahead for narrow
    // token tiles
    constexpr bool kPipeX = SU * TT <= 2;
    uint32_t xs[SU][TT][16], xn[SU][TT][16];
    auto load_x = [&](uint32_t (&dst)[SU][TT][16], int u) {
        const int ku = u % upt;
#pragma unroll
        for (int b = 0; b < SU; ++b) {
            const int kl = (ku * SU + b) * 128 + t * 32;
            const bool kvalid = kl < p.K;
#pragma unroll
            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (xvalid[tt] && kvalid)
                        v = ldg128(xrow[tt] + kl + 8 * q);
                    dst[b][tt][4 * q + 0] = v.x;
                    dst[b][tt][4 * q + 1] = v.y;
                    dst[b][tt][4 * q + 2] = v.z;
                    dst[b][tt][4 * q + 3] = v.w;
                }
        }
    };
    auto load_scales = [&](float2 (&dst)[SU], int u) {
        const int nt = u / upt, ku = u - nt * upt;
#pragma unroll
        for (int b = 0; b < SU; ++b)
            dst[b] = box_scales(p, nt, ku * SU + b, g, t);
    };
    const int c_lo = ((2 * t) ^ g) * 16, c_hi = ((2 * t + 1) ^ g) * 16;

    float acc[TT][4];
    bool ok = true;
    int i = warp;          // run index of this warp's next unit
    int slot = 0;          // ring slot of unit i
    uint32_t phase = 0;    // parity of the phase of unit i
    float2 sc[SU], scn[SU];
    if (i < n) {
        load_scales(scn, U0 + i);
        if (kPipeX)
            load_x(xn, U0 + i);
    }
    int sidx = 0;          // segment of the run
    int tile = U0 / upt;
    for (int seg = U0; seg < U1; ++tile) {
        const int tile_begin = tile * upt;
        const int seg_end = min(U1, tile_begin + upt);
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[tt][e] = 0.f;
        for (; U0 + i < seg_end; i += kConsumers) {
            const int u = U0 + i;
#pragma unroll
            for (int b = 0; b < SU; ++b)
                sc[b] = scn[b];
            if (kPipeX) {
#pragma unroll
                for (int b = 0; b < SU; ++b)
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            xs[b][tt][k] = xn[b][tt][k];
                if (i + kConsumers < n)
                    load_x(xn, u + kConsumers);
            } else {
                load_x(xs, u);
            }
            if (i + kConsumers < n)
                load_scales(scn, u + kConsumers);
            if (!mbar_wait(&full[slot], phase, ok ? kWaitLimitNs : 0)) {
                if (ok && lane == 0)
                    record_error(p.hdr, MXG_ERR_TIMEOUT, 200);
                ok = false;
            }
            const uint8_t *st = ring + slot * Unit<SU>::kBytes;
#pragma unroll
            for (int b = 0; b < SU; ++b) {
                const uint8_t *box = st + b * kBox;
                const uint4 ra0 = lds128(box + g * 128 + c_lo);
                const uint4 ra1 = lds128(box + g * 128 + c_hi);
                const uint4 rb0 = lds128(box + (g + 8) * 128 + c_lo);
                const uint4 rb1 = lds128(box + (g + 8) * 128 + c_hi);
                const uint32_t wa[8] = {ra0.x, ra0.y, ra0.z, ra0.w, ra1.x, ra1.y, ra1.z, ra1.w};
                const uint32_t wb[8] = {rb0.x, rb0.y, rb0.z, rb0.w, rb1.x, rb1.y, rb1.z, rb1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t a0, a1, a2, a3;
                    e4m3x4_scaled(wa[j], sc[b].x, a0, a2);
                    e4m3x4_scaled(wb[j], sc[b].y, a1, a3);
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt)
                        mma_bf16_16816(acc[tt], a0, a1, a2, a3, xs[b][tt][2 * j],
                                       xs[b][tt][2 * j + 1]);
                }
            }
            // every lane's reads of the slot have returned: refill it with
            // this warp's unit kStages ahead
            __syncwarp();
            if (lane == 0 && i + kStages * kConsumers < n)
                fetch_unit<SU>(p, &wq_map, ring + slot * Unit<SU>::kBytes, &full[slot],
                               u + kStages * kConsumers, policy);
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1;
            }
        }

        // ---- end of the tile segment: every warp leaves its fragment in the
        // segment's reduction buffer and goes on; the last to arrive adds them
        const int rb = sidx % SL::kRed;
        const int uses = sidx / SL::kRed;  // earlier segments that used buffer rb
        if (uses > 0) {
            if (lane == 0) {
                const unsigned long long t0 = global_ns();
                while (*reinterpret_cast<volatile int *>(&red_done[rb]) < uses) {
                    if (global_ns() - t0 > kWaitLimitNs) {
                        record_error(p.hdr, MXG_ERR_TIMEOUT, 230);
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
        for (int tt = 0; tt < TT; ++tt)
            frags[(size_t)warp * SL::kFrag4 + tt * 32 + lane] =
                make_float4(acc[tt][0], acc[tt][1], acc[tt][2], acc[tt][3]);
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
                float4 sum[TT];
                sum_fragments<TT>(frags, lane, sum);
#pragma unroll
                for (int tt = 0; tt < TT; ++tt)
                    store_y4(p, tile, tt, lane, sum[tt]);
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

template <int TT, int SU>
const void *kernel_ptr()
{
    return reinterpret_cast<const void *>(&mxfp8_stream_kernel<TT, SU>);
}

// SU = 2 for narrow token tiles (MXG_MX_SU2_TT tiles of 8 at most), SU = 1 otherwise.
const void *select_kernel(int tt, int su)
{
    if (su == 2)
        return tt == 1 ? kernel_ptr<1, 2>() : tt == 2 ? kernel_ptr<2, 2>() : nullptr;
    switch (tt) {
    case 1: return kernel_ptr<1, 1>();
    case 2: return kernel_ptr<2, 1>();
    case 3: return kernel_ptr<3, 1>();
    case 4: return kernel_ptr<4, 1>();
    default: return nullptr;
    }
}

size_t smem_bytes(int tt, int su)
{
    if (su == 2)
        return tt == 1 ? Smem<1, 2>::kTotal : Smem<2, 2>::kTotal;
    switch (tt) {
    case 1: return Smem<1, 1>::kTotal;
    case 2: return Smem<2, 1>::kTotal;
    case 3: return Smem<3, 1>::kTotal;
    default: return Smem<4, 1>::kTotal;
    }
}

}  // namespace

bool plan_mxfp8_stream(int device, int M, int N, int K, StreamPlan *plan)
{
    if (M < 1 || M > 32)
        return false;
    const DeviceInfo &di = device_info(device);
    StreamPlan pl{};
    pl.tt = (M + 7) / 8;
    const int boxes = (K + 127) / 128;             // 128-k boxes per row
    const int su = pl.tt <= MXG_MX_SU2_TT && boxes % 2 == 0 ? 2 : 1;
    pl.variant = su;
    pl.warps_per_cta = kConsumers;
    pl.smem = smem_bytes(pl.tt, su);
    if ((int)pl.smem > di.smem_optin)
        return false;
    pl.upt = boxes / su;
    pl.ntiles = (N + 15) / 16;
    if ((size_t)pl.ntiles > kMaxCounters)
        return false;
    pl.units = (long long)pl.ntiles * pl.upt;
    if (pl.units > (1LL << 30))
        return false;
    const void *fn = select_kernel(pl.tt, su);
    if (!fn)
        return false;
    // every CTA of the grid must be resident at once (a cut tile's finishing
    // CTA waits for the others)
    // (function attributes and occupancy are per device: cached per device)
    if (device < 0 || device >= kMaxDeviceCache)
        return false;
    static std::atomic<int> occ_cache[kMaxDeviceCache][4][3];
    std::atomic<int> &occ_slot = occ_cache[device][pl.tt - 1][su];
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
        occ = std::min(o, 1);
        occ_slot.store(occ, std::memory_order_release);
    }
    // no run shorter than kMinUnitsPerCta units; a layer too small for 32
    // such runs gets at least one CTA per n16 tile instead (one CTA streaming
    // many short tiles would serialise their reductions)
    long long wt = std::min<long long>((long long)di.sms * occ, pl.units / kMinUnitsPerCta);
    if (wt < 32)
        wt = std::min<long long>((long long)di.sms * occ, std::max<long long>(wt, pl.ntiles));
    pl.Wt = (int)std::max<long long>(1, wt);
    pl.grid = pl.Wt;
    pl.partial_bytes = (size_t)pl.Wt * pl.tt * 32 * sizeof(float4);
    *plan = pl;
    return true;
}

cudaError_t launch_mxfp8_stream(const StreamPlan &pl, const void *X, const uint8_t *Wq,
                                const uint8_t *Ws, int M, int N, int K, void *Y, void *workspace,
                                bool early, cudaStream_t stream)
{
    const void *fn = select_kernel(pl.tt, pl.variant);
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
    p.early = early ? 1 : 0;
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
    void *args[] = {&map, &p};
    return launch_pdl(fn, dim3(pl.grid), dim3(kThreads), pl.smem, stream, args);
}

}  // namespace mxg
