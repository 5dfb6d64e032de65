// Tensor-core GEMM for larger M (MTP verify batches, prefill chunks).
//
// Y[M][N] = X[M][K] * dequant(W)^T on the 5th-generation tensor cores.
// Persistent, warp-specialised CTA (one per SM), output tile 128 x 256,
// k-block 64:
//   warp 0        producer: tensor-map copies of the X tile (128-byte
//                 swizzle, the MMA's A operand as is) and of the packed
//                 weight tile (codes + scales) into two shared-memory rings;
//   warp 1        allocates 512 TMEM columns (two 128 x 256 fp32
//                 accumulators) and issues tcgen05.mma (kind::f16, bf16 x
//                 bf16 -> fp32) from one thread; tcgen05.commit releases
//                 the operand slots and publishes finished accumulators;
//   warps 2..5    epilogue: tcgen05.ld of their 32 TMEM lanes, fp32 -> bf16,
//                 stores to Y; overlaps the next tile's main loop;
//   warps 6..13   dequantisers: packed weight slot -> bf16 B operand in the
//                 128-byte-swizzled K-major layout the MMA reads, one
//                 rounding per weight (INT4: (q - 8) * scale; MXFP8:
//                 e4m3 * 2^(E - 127)), then a proxy fence so the tensor
//                 core sees the generic-proxy stores.
// Every wait is an mbarrier phase wait with a time limit; a timeout sets
// a CTA-wide abort flag, records MXG_ERR_TIMEOUT and every role drains to
// the final barrier, where TMEM is released.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kSX = 4;   // X ring depth
constexpr int kSW = 4;   // packed-weight ring depth
constexpr int kSB = 3;   // bf16-weight ring depth
constexpr int kXBytes = BM * BK * 2;                 // 16 KB
constexpr int kWbBytes = BN * BK * 2;                // 32 KB
constexpr int kWpBytes = 9 * 1024;                   // codes (8 KB or 16 KB MXFP8: see below)
constexpr int kWpBytesMx = BN * BK;                  // 16 KB of E4M3 codes
constexpr int kProducerWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2, kNumEpiWarps = 4;
constexpr int kDqWarp0 = 6, kNumDqWarps = 8;
constexpr int kThreads = (kDqWarp0 + kNumDqWarps) * 32;
constexpr uint32_t kTmemCols = 512;

enum Fmt { kInt4 = 0, kMxfp8 = 1 };

template <int F>
struct Layout {
    static constexpr int wp_bytes = (F == kInt4) ? kWpBytes : kWpBytesMx;
    static constexpr int x_off = 0;
    static constexpr int wb_off = x_off + kSX * kXBytes;
    static constexpr int wp_off = wb_off + kSB * kWbBytes;
    static constexpr int bar_off = wp_off + kSW * wp_bytes;
    // barriers: x_full, x_empty, wp_full, wp_empty, wb_full, wb_empty, acc_full, acc_empty
    static constexpr int n_bars = 2 * kSX + 2 * kSW + 2 * kSB + 4;
    static constexpr int misc_off = bar_off + n_bars * 8;
    static constexpr int total = misc_off + 16;
    static constexpr size_t smem_bytes = (size_t)total + 1024;  // + alignment slack
};

struct TcParams {
    uint16_t *Y;
    const uint8_t *Ws;     // MXFP8 scales [N][K/32]
    WsHeader *hdr;
    int M, N, K, G;
    int mtiles, ntiles, kblocks;
    int num_tiles;
};

// ----------------------------------------------------------- tcgen05 PTX
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, kind::f16.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused (1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for this architecture
    d |= (uint64_t)2 << 61;   // 128-byte swizzle
    return d;
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool role_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          WsHeader *hdr, int where)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (*abort_flag)
            return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            record_error(hdr, MXG_ERR_TIMEOUT, where);
            return false;
        }
    }
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c)
{
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b)
{
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// INT4: one packed 16-byte chunk (n32 tile tl, half h, lane) = two columns x
// 16 k -> eight 8-byte bf16 stores into the 128-byte-swizzled B tile.
// Word j holds k = 16j + 4t .. 16j + 4t + 3 of the k-block.
__device__ __forceinline__ void dequant_int4_chunk(const uint8_t *wp_slot, uint32_t wb_slot, int tl,
                                                   int h, int lane, int G, int gpk)
{
    const int g = lane >> 2, t = lane & 3;
    const uint4 v = lds128(wp_slot + tl * 1024 + h * 512 + lane * 16);
    const uint32_t wj[4] = {v.x, v.y, v.z, v.w};
    const int ra = tl * 32 + h * 16 + g, rb = ra + 8;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int gi = (16 * j + 4 * t) / G;  // group inside the k-block
        const uint32_t sw = lds32(wp_slot + 8192 + tl * (64 * gpk) + gi * 64 + g * 8 + h * 4);
        const ScaleSplit sa = split_scale((uint16_t)(sw & 0xFFFF));
        const ScaleSplit sb = split_scale((uint16_t)(sw >> 16));
        const uint32_t w = wj[j];
        const int chunk = 2 * j + (t >> 1), half = (t & 1) * 8;
        sts64(wb_slot + sw128_off(ra, chunk) + half, scale_pair_rn(int4_pair_minus8<0>(w), sa),
              scale_pair_rn(int4_pair_minus8<8>(w), sa));
        sts64(wb_slot + sw128_off(rb, chunk) + half, scale_pair_rn(int4_pair_minus8<4>(w), sb),
              scale_pair_rn(int4_pair_minus8<12>(w), sb));
    }
}

// MXFP8: row r of the tile (64 codes, 64-byte swizzled rows) -> 128 bytes of bf16.
__device__ __forceinline__ void dequant_mx_row(const uint8_t *wp_slot, uint32_t wb_slot, int r,
                                               float s0, float s1)
{
    uint32_t out[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = lds128(wp_slot + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
        const float s = (c < 2) ? s0 : s1;
        e4m3x4_scaled(v.x, s, out[8 * c + 0], out[8 * c + 1]);
        e4m3x4_scaled(v.y, s, out[8 * c + 2], out[8 * c + 3]);
        e4m3x4_scaled(v.z, s, out[8 * c + 4], out[8 * c + 5]);
        e4m3x4_scaled(v.w, s, out[8 * c + 6], out[8 * c + 7]);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
        sts128(wb_slot + sw128_off(r, c), out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
}

template <int F>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap x_map,
                   const __grid_constant__ CUtensorMap w_map,
                   const __grid_constant__ CUtensorMap s_map, const TcParams p)
{
    using L = Layout<F>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::bar_off);
    uint64_t *x_full = bars, *x_empty = bars + kSX;
    uint64_t *wp_full = bars + 2 * kSX, *wp_empty = wp_full + kSW;
    uint64_t *wb_full = wp_empty + kSW, *wb_empty = wb_full + kSB;
    uint64_t *acc_full = wb_empty + kSB, *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::misc_off + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSX; ++i) {
            mbar_init(&x_full[i], 1);
            mbar_init(&x_empty[i], 1);
        }
        for (int i = 0; i < kSW; ++i) {
            mbar_init(&wp_full[i], 1);
            mbar_init(&wp_empty[i], kNumDqWarps);
        }
        for (int i = 0; i < kSB; ++i) {
            mbar_init(&wb_full[i], kNumDqWarps);
            mbar_init(&wb_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kNumEpiWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp)
        tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int gpk = (F == kInt4) ? max(1, BK / p.G) : 1;  // scale groups per k-block

    if (warp == kProducerWarp) {
        if (lane == 0) {
            prefetch_tensormap(&x_map);
            prefetch_tensormap(&w_map);
            if (F == kInt4)
                prefetch_tensormap(&s_map);
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                const int nb = tile / p.mtiles, mt = tile % p.mtiles;
                for (int kb = 0; kb < p.kblocks && ok; ++kb, ++it) {
                    const int sw = it % kSW, sx = it % kSX;
                    ok = role_wait(&wp_empty[sw], ((it / kSW) & 1) ^ 1, abort_flag, p.hdr, 301);
                    if (!ok)
                        break;
                    uint8_t *wdst = smem + L::wp_off + sw * L::wp_bytes;
                    if (F == kInt4) {
                        const uint32_t sbytes = 512u * gpk;
                        mbar_arrive_expect_tx(&wp_full[sw], 8192u + sbytes);
                        tma_load_2d(wdst, &w_map, kb * 128, nb * 8, &wp_full[sw], pol_w);
                        tma_load_2d(wdst + 8192, &s_map, (kb * 64 / p.G) * 8, nb * 8, &wp_full[sw],
                                    pol_w);
                    } else {
                        mbar_arrive_expect_tx(&wp_full[sw], (uint32_t)kWpBytesMx);
                        tma_load_2d(wdst, &w_map, kb * 64, nb * BN, &wp_full[sw], pol_w);
                    }
                    ok = role_wait(&x_empty[sx], ((it / kSX) & 1) ^ 1, abort_flag, p.hdr, 302);
                    if (!ok)
                        break;
                    mbar_arrive_expect_tx(&x_full[sx], (uint32_t)kXBytes);
                    tma_load_2d(smem + L::x_off + sx * kXBytes, &x_map, kb * 64, mt * BM, &x_full[sx],
                                pol_x);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
                const int acc = tcount & 1;
                ok = role_wait(&acc_empty[acc], ((tcount >> 1) & 1) ^ 1, abort_flag, p.hdr, 311);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                    const int sx = it % kSX, sb = it % kSB;
                    ok = role_wait(&x_full[sx], (it / kSX) & 1, abort_flag, p.hdr, 312) &&
                         role_wait(&wb_full[sb], (it / kSB) & 1, abort_flag, p.hdr, 313);
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t xa = smem_u32(smem + L::x_off + sx * kXBytes);
                    const uint32_t wa = smem_u32(smem + L::wb_off + sb * kWbBytes);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_f16(d, sw128_desc(xa + 32 * k), sw128_desc(wa + 32 * k), kIdesc,
                                   (kb > 0 || k > 0) ? 1u : 0u);
                    tc_commit(&x_empty[sx]);
                    tc_commit(&wb_empty[sb]);
                }
                if (ok)
                    tc_commit(&acc_full[acc]);
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
            const int acc = tcount & 1;
            if (!role_wait(&acc_full[acc], (tcount >> 1) & 1, abort_flag, p.hdr, 321))
                break;
            tc_fence_after();
            const int nb = tile / p.mtiles, mt = tile % p.mtiles;
            const int row = mt * BM + q * 32 + lane;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tbase + c * 32, r);
                const int n0 = nb * BN + c * 32;
                if (row < p.M && n0 < p.N) {
                    uint32_t o[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[2 * i]),
                                                                 __uint_as_float(r[2 * i + 1]));
                        o[i] = *reinterpret_cast<uint32_t *>(&b);
                    }
                    uint16_t *yrow = p.Y + (size_t)row * p.N;
                    if (n0 + 32 <= p.N && (p.N & 7) == 0) {
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + n0);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                    } else {
                        for (int i = 0; i < 32 && n0 + i < p.N; ++i)
                            yrow[n0 + i] = (uint16_t)(o[i >> 1] >> ((i & 1) * 16));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[acc]);
        }
    } else {
        // dequantisers
        const int dw = warp - kDqWarp0;
        const int dt = dw * 32 + lane;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
            const int nb = tile / p.mtiles;
            for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                const int sw = it % kSW, sb = it % kSB;
                float s0 = 0.f, s1 = 0.f;
                if (F == kMxfp8) {
                    // the row's two E8M0 scales of this k-block (from L2)
                    const int n = nb * BN + dt;
                    const int blocks = p.K / 32;
                    const int b0 = kb * 2;
                    uint32_t e0 = 127, e1 = 127;
                    if (n < p.N) {
                        e0 = __ldg(p.Ws + (size_t)n * blocks + b0);
                        if (b0 + 1 < blocks)
                            e1 = __ldg(p.Ws + (size_t)n * blocks + b0 + 1);
                    }
                    s0 = e8m0_to_f32(e0);
                    s1 = e8m0_to_f32(e1);
                }
                ok = role_wait(&wp_full[sw], (it / kSW) & 1, abort_flag, p.hdr, 331) &&
                     role_wait(&wb_empty[sb], ((it / kSB) & 1) ^ 1, abort_flag, p.hdr, 332);
                if (!ok)
                    break;
                const uint8_t *wp_slot = smem + L::wp_off + sw * L::wp_bytes;
                const uint32_t wb_slot = smem_u32(smem + L::wb_off + sb * kWbBytes);
                if (F == kInt4) {
                    dequant_int4_chunk(wp_slot, wb_slot, dw, 0, lane, p.G, gpk);
                    dequant_int4_chunk(wp_slot, wb_slot, dw, 1, lane, p.G, gpk);
                } else {
                    dequant_mx_row(wp_slot, wb_slot, dt, s0, s1);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&wb_full[sb]);
                    mbar_arrive(&wp_empty[sw]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp)
        tmem_dealloc(tmem_base, kTmemCols);
}

template <int F>
bool tc_plan(int device, int M, int N, int K, TcPlan *plan)
{
    const DeviceInfo &di = device_info(device);
    if ((size_t)di.smem_optin < Layout<F>::smem_bytes)
        return false;
    TcPlan pl{};
    pl.bm = BM;
    pl.bn = BN;
    pl.bk = BK;
    pl.mtiles = (M + BM - 1) / BM;
    pl.ntiles = (N + BN - 1) / BN;
    pl.splits = 1;
    const int tiles = pl.mtiles * pl.ntiles;
    pl.grid = std::min(tiles, di.sms);
    pl.smem = Layout<F>::smem_bytes;
    pl.partial_bytes = 0;
    pl.counters = 0;
    *plan = pl;
    return true;
}

template <int F>
cudaError_t tc_launch(const TcPlan &pl, const CUtensorMap &xm, const CUtensorMap &wm,
                      const CUtensorMap &sm, TcParams p, cudaStream_t stream)
{
    const void *fn = reinterpret_cast<const void *>(&tc_gemm_kernel<F>);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e =
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
        if (e != cudaSuccess)
            return e;
        attr_set = true;
    }
    void *args[] = {const_cast<CUtensorMap *>(&xm), const_cast<CUtensorMap *>(&wm),
                    const_cast<CUtensorMap *>(&sm), &p};
    return cudaLaunchKernel(fn, dim3(pl.grid), dim3(kThreads), args, pl.smem, stream);
}

bool x_map(CUtensorMap *m, const void *X, int M, int K)
{
    return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M,
                                (uint64_t)K * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool plan_w4a16_tc(int device, int M, int N, int K, int G, TcPlan *plan)
{
    (void)G;
    return tc_plan<kInt4>(device, M, N, K, plan);
}

cudaError_t launch_w4a16_tc(const TcPlan &pl, const void *X, const void *packed, int M, int N,
                            int K, int G, void *Y, void *workspace, cudaStream_t stream)
{
    alignas(64) CUtensorMap xm, wm, sm;
    const uint8_t *codes = static_cast<const uint8_t *>(packed);
    const uint8_t *scales = codes + (size_t)N * K / 2;
    const int gpk = std::max(1, BK / G);
    if (!x_map(&xm, X, M, K) ||
        // codes: rows = n32 tiles of 2K u64 words (K/64 chunks of 1 KB); box = one chunk x 8 tiles
        !encode_tensor_map_2d(&wm, CU_TENSOR_MAP_DATA_TYPE_UINT64, codes, (uint64_t)K * 2,
                              (uint64_t)(N / 32), (uint64_t)K * 16, 128, 8,
                              CU_TENSOR_MAP_SWIZZLE_NONE) ||
        // scales: rows = n32 tiles, K/G groups of 8 u64 words (64 bytes) per row
        !encode_tensor_map_2d(&sm, CU_TENSOR_MAP_DATA_TYPE_UINT64, scales, (uint64_t)(K / G) * 8,
                              (uint64_t)(N / 32), (uint64_t)(K / G) * 64, 8 * gpk, 8,
                              CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    TcParams p{};
    p.Y = static_cast<uint16_t *>(Y);
    p.Ws = nullptr;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = G;
    p.mtiles = pl.mtiles;
    p.ntiles = pl.ntiles;
    p.kblocks = K / BK;
    p.num_tiles = pl.mtiles * pl.ntiles;
    return tc_launch<kInt4>(pl, xm, wm, sm, p, stream);
}

bool plan_mxfp8_tc(int device, int M, int N, int K, TcPlan *plan)
{
    return tc_plan<kMxfp8>(device, M, N, K, plan);
}

cudaError_t launch_mxfp8_tc(const TcPlan &pl, const void *X, const uint8_t *Wq,
                            const uint8_t *Ws, int M, int N, int K, void *Y, void *workspace,
                            cudaStream_t stream)
{
    alignas(64) CUtensorMap xm, wm;
    if (!x_map(&xm, X, M, K) ||
        !encode_tensor_map_2d(&wm, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                              (uint64_t)K, BK, BN, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    TcParams p{};
    p.Y = static_cast<uint16_t *>(Y);
    p.Ws = Ws;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 32;
    p.mtiles = pl.mtiles;
    p.ntiles = pl.ntiles;
    p.kblocks = (K + BK - 1) / BK;
    p.num_tiles = pl.mtiles * pl.ntiles;
    return tc_launch<kMxfp8>(pl, xm, wm, wm, p, stream);
}

}  // namespace mxg
