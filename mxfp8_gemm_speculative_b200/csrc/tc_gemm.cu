// Tensor-core GEMM for larger M (MTP verify batches, prefill chunks).
//
// Y[M][N] = X[M][K] * dequant(W)^T on the 5th-generation tensor cores, with
// the roles of the operands swapped so that the dequantized weights never
// touch shared memory:
//   * a CTA pair (cluster of 2, tcgen05 cta_group::2) owns 256 weight
//     columns (128 per CTA) x BT tokens; the MMA is D[n][m] += W[n][k] X[m][k]
//     with M_mma = 256 weight columns, N_mma = BT tokens, K = 16 per step;
//   * A = the weights, decoded by eight dequantiser warps per CTA straight
//     from the packed bytes into tensor memory (tcgen05.st, 16 lanes x 256
//     bits per store): the packed INT4 layout places one lane's 16 bytes
//     exactly on one thread's share of such a store;
//   * B = the activations, fetched by the tensor-map engine with the 128-byte
//     swizzle (each CTA its BT/2 tokens; the pair's MMA reads both halves);
//   * D = fp32 accumulators in tensor memory; four epilogue warps per CTA
//     read them back (tcgen05.ld) and store bf16 Y.
// Shared memory then only holds packed weights (0.5 or 1 byte per weight)
// and activations, which keeps the pair inside the SM's shared-memory
// bandwidth at full tensor rate.
//
// Warp roles per CTA (480 threads):
//   warp 0        producer of the activation copies;
//   warp 1        tensor-memory allocation; in the even CTA also the single
//                 thread that issues tcgen05.mma and tcgen05.commit;
//   warps 2..5    epilogue;
//   warps 6..13   dequantisers (warp w writes lanes 32*(w%4) + 16*h .. +15,
//                 h = (w - 6) / 4);
//   warp 14       producer of the packed-weight copies, on a ring of its own
//                 so the weights run ahead of the activations.
// Every wait is an mbarrier phase wait with a time limit; a timeout sets a
// CTA-wide abort flag, records MXG_ERR_TIMEOUT and every role drains to the
// end, where tensor memory is released.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

constexpr int BW = 128;  // weight columns per CTA
constexpr int BK = 64;   // k per block
constexpr int kProducerWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2, kNumEpiWarps = 4;
constexpr int kDqWarp0 = 6, kNumDqWarps = 8;
constexpr int kWProducerWarp = kDqWarp0 + kNumDqWarps;   // packed-weight loads
constexpr int kThreads = (kWProducerWarp + 1) * 32;
constexpr uint32_t kTmemCols = 512;

enum Fmt { kInt4 = 0, kMxfp8 = 1 };

// Ring depths: with 128 tokens per tile the activation and weight slots are
// small and a k-block's MMA is short, so the rings are deeper to cover the
// load latency; the A ring takes the tensor memory the accumulator leaves.
template <int F, int BT>
struct Layout {
    static constexpr int kSX = BT == 128 ? 8 : 5;    // activation ring
    static constexpr int kSW = BT == 128 ? (F == kInt4 ? 24 : 16) : (F == kInt4 ? 16 : 12);   // packed-weight ring
    static constexpr int kSA = BT == 128 ? 12 : 8;    // tensor-memory A ring (32 columns each)
    static constexpr int x_slot = (BT / 2) * BK * 2;                // bf16 activations
    static constexpr int wp_slot = (F == kInt4) ? 5120 : BW * BK;   // packed weights
    static constexpr int x_off = 0;
    static constexpr int wp_off = x_off + kSX * x_slot;
    static constexpr int bar_off = wp_off + kSW * wp_slot;
    static constexpr int n_bars = 2 * kSX + 2 * kSW + 2 * kSA + 2;
    static constexpr int misc_off = bar_off + n_bars * 8;
    static constexpr int total = misc_off + 16;
    static constexpr size_t smem_bytes = (size_t)total + 1024;  // + alignment slack
    static constexpr uint32_t acc_col = 0;                     // D: columns [0, BT)
    static constexpr uint32_t a_col = BT;                      // A ring after D
    static_assert(BT + 32 * kSA <= (int)kTmemCols, "tensor memory budget");
};

struct TcParams {
    uint16_t *Y;
    const uint8_t *Ws;     // MXFP8 scales [N][K/32]
    WsHeader *hdr;
    float *partial;        // split-K partial sums [num_items][BT][2 * BW] (splits > 1)
    int *counters;         // split-K arrivals per (tile, CTA of the pair, quadrant)
    int M, N, K, G;
    int mtiles, ntiles, kblocks;
    int num_tiles;
    int splits;            // K splits per output tile
    int num_items;         // num_tiles * splits work items
    int early;             // load the first weights before waiting for the previous kernel
};

// Output tile -> weight block nb (256 columns) and token tile mt.  With
// several token tiles the tiles run token-tile-major: the pairs working at
// the same time share one activation tile and sweep all weight blocks, which
// stay in L2 (marked evict-last) from one token tile to the next, so each
// weight and activation byte is read from DRAM a few times at most.
__device__ __forceinline__ int tile_nb(const TcParams &p, int tile)
{
    return p.mtiles > 1 ? tile % p.ntiles : tile / p.mtiles;
}
__device__ __forceinline__ int tile_mt(const TcParams &p, int tile)
{
    return p.mtiles > 1 ? tile / p.ntiles : tile % p.mtiles;
}

// Work item -> output tile and its k-block range [kb0, kb1).
__device__ __forceinline__ void item_range(const TcParams &p, int item, int &tile, int &kb0,
                                           int &kb1)
{
    tile = item / p.splits;
    const int s = item - tile * p.splits;
    kb0 = (int)((long long)s * p.kblocks / p.splits);
    kb1 = (int)((long long)(s + 1) * p.kblocks / p.splits);
}

// ----------------------------------------------------------- cluster PTX
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive on a barrier of either CTA of the pair.  What the waiter needs to
// see is ordered by the tcgen05 fences around the hand-off, so the arrive
// itself carries no cluster-scope release.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Tensor copy into this CTA's shared memory that completes on an mbarrier of
// the even CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, int c0, int c1,
                                                 uint32_t leader_bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(leader_bar), "l"(policy)
        : "memory");
}

// ----------------------------------------------------------- tcgen05 PTX
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *slot, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
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

// Arrive on the barrier at this offset in both CTAs of the pair once every
// tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"((uint16_t)0x3)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T over the CTA pair, kind::f16.
__device__ __forceinline__ void tc_mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 lanes x 256 bits, four times along the columns: thread (g, t) writes
// lanes g and g + 8 of the 16-lane slab, columns 8r + 2t and 8r + 2t + 1 of
// repetition r, from registers v[4r .. 4r + 3] (lane g: two columns, then
// lane g + 8: two columns).
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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

// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 256 (pair), N = BT.
template <int BT>
__host__ __device__ constexpr uint32_t idesc_pair()
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BT >> 3) << 17) |
           ((uint32_t)(256 >> 4) << 24);
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool role_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          WsHeader *hdr, int where)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    while (true) {
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

// INT4: the dequantiser thread's 16 packed bytes (n32 tile q of the CTA,
// half h, lane) -> 16 registers of bf16 pairs for a 16x256b x4 store.
__device__ __forceinline__ void dequant_int4(const uint8_t *wp_slot, int q, int h, int lane, int G,
                                             int gpk, uint32_t (&v)[16])
{
    const int g = lane >> 2;
    const uint4 c = lds128(wp_slot + q * 1024 + h * 512 + lane * 16);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    // words 0-1 and 2-3 lie in one scale group each (the same one for G >= 64)
    (void)gpk;
    const uint8_t *sbase = wp_slot + 4096 + q * 64 + g * 8 + h * 4;
    const uint32_t sw0 = lds32(sbase);
    const uint32_t sw1 = G == 32 ? lds32(sbase + 256) : sw0;
    const ScaleSplit sa0 = split_scale((uint16_t)(sw0 & 0xFFFF));
    const ScaleSplit sb0 = split_scale((uint16_t)(sw0 >> 16));
    ScaleSplit sa1 = sa0, sb1 = sb0;
    if (G == 32) {
        sa1 = split_scale((uint16_t)(sw1 & 0xFFFF));
        sb1 = split_scale((uint16_t)(sw1 >> 16));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const ScaleSplit &sa = j < 2 ? sa0 : sa1;
        const ScaleSplit &sb = j < 2 ? sb0 : sb1;
        v[4 * j + 0] = scale_pair_rn(int4_pair_minus8<0>(w[j]), sa);
        v[4 * j + 1] = scale_pair_rn(int4_pair_minus8<8>(w[j]), sa);
        v[4 * j + 2] = scale_pair_rn(int4_pair_minus8<4>(w[j]), sb);
        v[4 * j + 3] = scale_pair_rn(int4_pair_minus8<12>(w[j]), sb);
    }
}

// MXFP8: rows ra = 32q + 16h + g and ra + 8 of the CTA's [128][64 B] code
// tile (64-byte swizzle); for repetition j the thread needs k = 16j + 4t ..
// 16j + 4t + 3 of both rows (one 32-bit word each).
__device__ __forceinline__ void dequant_mx(const uint8_t *wp_slot, int q, int h, int lane,
                                           const float (&sa)[2], const float (&sb)[2],
                                           uint32_t (&v)[16])
{
    const int g = lane >> 2, t = lane & 3;
    const int ra = q * 32 + h * 16 + g, rb = ra + 8;
    const int swa = (ra >> 1) & 3, swb = (rb >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t wa = lds32(wp_slot + ra * 64 + ((j ^ swa) << 4) + 4 * t);
        const uint32_t wb = lds32(wp_slot + rb * 64 + ((j ^ swb) << 4) + 4 * t);
        e4m3x4_scaled(wa, sa[j >> 1], v[4 * j + 0], v[4 * j + 1]);
        e4m3x4_scaled(wb, sb[j >> 1], v[4 * j + 2], v[4 * j + 3]);
    }
}

template <int F, int BT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap x_map,
                   const __grid_constant__ CUtensorMap w_map,
                   const __grid_constant__ CUtensorMap s_map, const TcParams p)
{
    using L = Layout<F, BT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::bar_off);
    uint64_t *x_full = bars, *x_empty = bars + L::kSX;
    uint64_t *wp_full = bars + 2 * L::kSX, *wp_empty = wp_full + L::kSW;
    uint64_t *a_full = wp_empty + L::kSW, *a_empty = a_full + L::kSA;
    uint64_t *acc_full = a_empty + L::kSA, *acc_empty = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::misc_off + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();   // 0: issues the MMAs; 1: its pair
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::kSX; ++i) {
            mbar_init(&x_full[i], 1);            // leader: producer arrive + both copies
            mbar_init(&x_empty[i], 1);           // commit from the MMA
        }
        for (int i = 0; i < L::kSW; ++i) {
            mbar_init(&wp_full[i], 1);
            mbar_init(&wp_empty[i], kNumDqWarps);
        }
        for (int i = 0; i < L::kSA; ++i) {
            mbar_init(&a_full[i], 2 * kNumDqWarps);   // leader: dequantisers of both CTAs
            mbar_init(&a_empty[i], 1);                 // commit from the MMA
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * kNumEpiWarps);        // leader: epilogues of both CTAs
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp)
        tmem_alloc_pair(tmem_slot, kTmemCols);
    if (threadIdx.x == 32 * kProducerWarp && pair < p.num_items) {
        // while the previous kernel drains: pull the first k-blocks into L2
        int tile0, kb0, kb1;
        item_range(p, pair, tile0, kb0, kb1);
        const int nb = tile_nb(p, tile0), mt = tile_mt(p, tile0);
        const int n32 = (nb * 2 * BW + (int)rank * BW) / 32;
        for (int kb = kb0; kb < min(kb0 + L::kSW, kb1); ++kb) {
            prefetch_tensor_l2(&x_map, kb * BK, mt * BT + (int)rank * (BT / 2));
            if (F == kInt4)
                prefetch_tensor_l2(&w_map, 0, (int)(code_offset(n32, kb, p.K, p.N / 32, 1) >> 10));
            else
                prefetch_tensor_l2(&w_map, kb * BK, n32 * 32);
        }
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int gpk = (F == kInt4) ? max(1, BK / p.G) : 1;  // scale groups per k-block

    // Packed weights of this CTA's 128 columns (lane 0 of the weight
    // producer), on their own deeper ring, not held back by the activation
    // ring.  w_issue(n) issues the loads of the CTA's k-blocks in order until
    // n of them have been issued.
    int w_item = pair, w_tile = 0, w_kb = 0, w_kb1 = 0;
    uint32_t w_it = 0;
    if (w_item < p.num_items)
        item_range(p, w_item, w_tile, w_kb, w_kb1);
    auto w_issue = [&](uint32_t until) -> bool {
        // weights stream once when there is one token tile, else every token
        // tile reads them again
        const uint64_t pol_w = p.mtiles > 1 ? l2_policy_evict_last() : l2_policy_evict_first();
        while (w_item < p.num_items && w_it < until) {
            if (w_kb >= w_kb1) {
                w_item += npairs;
                if (w_item < p.num_items)
                    item_range(p, w_item, w_tile, w_kb, w_kb1);
                continue;
            }
            const int sw = w_it % L::kSW;
            if (!role_wait(&wp_empty[sw], ((w_it / L::kSW) & 1) ^ 1, abort_flag, p.hdr, 402))
                return false;
            const int nb = tile_nb(p, w_tile);
            const int n32 = (nb * 2 * BW + (int)rank * BW) / 32;
            uint8_t *wdst = smem + L::wp_off + sw * L::wp_slot;
            if (F == kInt4) {
                // the CTA's four tiles of the column group for this k-block:
                // one 4-row box of codes (a row = one tile's 1 KB of a k64
                // chunk, rows in memory order) and one 4-row box of scales
                // per scale group (a row = one tile's 64 B).  In a last group
                // of fewer than eight tiles the rows past the group belong to
                // the next chunk or lie past the end (zero-filled): their
                // columns are past N and never stored.
                mbar_arrive_expect_tx(&wp_full[sw], 4096u + 256u * gpk);
                tma_load_2d(wdst, &w_map, 0, (int)(code_offset(n32, w_kb, p.K, p.N / 32, 1) >> 10),
                            &wp_full[sw], pol_w);
                for (int gi = 0; gi < gpk; ++gi)
                    tma_load_2d(wdst + 4096 + gi * 256, &s_map, 0,
                                (int)(scale_offset(n32, w_kb * BK / p.G + gi, p.K, p.G, p.N / 32) >> 6),
                                &wp_full[sw], pol_w);
            } else {
                mbar_arrive_expect_tx(&wp_full[sw], (uint32_t)(BW * BK));
                tma_load_2d(wdst, &w_map, w_kb * BK, n32 * 32, &wp_full[sw], pol_w);
            }
            ++w_kb;
            ++w_it;
        }
        return true;
    };
    if (warp == kWProducerWarp && lane == 0) {
        prefetch_tensormap(&w_map);
        if (F == kInt4)
            prefetch_tensormap(&s_map);
        // The weights are not written by the previous kernel on the stream
        // (the caller's contract, unless it turned early weight loads off):
        // the first ring of them fills while that kernel drains.  Everything
        // else waits for it.
        if (p.early)
            w_issue(L::kSW);
    }
    pdl_wait();

    if (warp == kProducerWarp) {
        // activations: this CTA's BT/2 tokens of every k-block, completing on
        // the leader's barrier
        if (lane == 0) {
            prefetch_tensormap(&x_map);
            // one token tile: read by every weight block; several: each is
            // read by the pairs of one sweep and then not again
            const uint64_t pol_x = p.mtiles > 1 ? l2_policy_evict_first() : l2_policy_evict_last();
            uint32_t it = 0;
            bool ok = true;
            for (int item = pair; item < p.num_items && ok; item += npairs) {
                int tile, kb0, kb1;
                item_range(p, item, tile, kb0, kb1);
                const int mt = tile_mt(p, tile);
                for (int kb = kb0; kb < kb1 && ok; ++kb, ++it) {
                    const int sx = it % L::kSX;
                    ok = role_wait(&x_empty[sx], ((it / L::kSX) & 1) ^ 1, abort_flag, p.hdr, 401);
                    if (!ok)
                        break;
                    if (rank == 0)
                        mbar_arrive_expect_tx(&x_full[sx], 2u * L::x_slot);
                    tma_load_2d_pair(smem + L::x_off + sx * L::x_slot, &x_map, kb * BK,
                                     mt * BT + (int)rank * (BT / 2),
                                     mapa_shared(smem_u32(&x_full[sx]), 0), pol_x);
                }
            }
        }
    } else if (warp == kWProducerWarp) {
        if (lane == 0)
            w_issue(0xffffffffu);
    } else if (warp == kMmaWarp) {
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = idesc_pair<BT>();
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int item = pair; item < p.num_items && ok; item += npairs, ++tcount) {
                int tile, kb0, kb1;
                item_range(p, item, tile, kb0, kb1);
                ok = role_wait(acc_empty, (tcount & 1) ^ 1, abort_flag, p.hdr, 411);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + L::acc_col;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int sx = it % L::kSX, sa = it % L::kSA;
                    ok = role_wait(&x_full[sx], (it / L::kSX) & 1, abort_flag, p.hdr, 412) &&
                         role_wait(&a_full[sa], (it / L::kSA) & 1, abort_flag, p.hdr, 413);
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t xa = smem_u32(smem + L::x_off + sx * L::x_slot);
                    const uint32_t a = tmem_base + L::a_col + 32 * sa;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_ts_pair(d, a + 8 * k, sw128_desc(xa + 32 * k), idesc,
                                       (kb > kb0 || k > 0) ? 1u : 0u);
                    tc_commit_pair(&x_empty[sx]);
                    tc_commit_pair(&a_empty[sa]);
                }
                if (ok)
                    tc_commit_pair(acc_full);
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const uint32_t leader_acc_empty = mapa_shared(smem_u32(acc_empty), 0);
        uint32_t tcount = 0;
        for (int item = pair; item < p.num_items; item += npairs, ++tcount) {
            int tile, kb0, kb1;
            item_range(p, item, tile, kb0, kb1);
            if (!role_wait(acc_full, tcount & 1, abort_flag, p.hdr, 421))
                break;
            tc_fence_after();
            const int nb = tile_nb(p, tile), mt = tile_mt(p, tile);
            const int nloc = (int)rank * BW + q * 32;                    // warp's first column in the pair
            const int n = nb * 2 * BW + nloc + lane;                      // this thread's column
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + L::acc_col;
            if (p.splits == 1) {
#pragma unroll 1
                for (int c = 0; c < BT / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tbase + c * 32, r);
                    const int m0 = mt * BT + c * 32;
                    if (n < p.N) {
                        uint16_t *yc = p.Y + (size_t)m0 * p.N + n;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (m0 + i < p.M)
                                yc[(size_t)i * p.N] = f32_to_bf16_bits(__uint_as_float(r[i]));
                    }
                }
            } else {
                // split K: this item's fp32 sums of the warp's 32 columns
                float *pp = p.partial + (size_t)item * BT * (2 * BW) + nloc + lane;
#pragma unroll 1
                for (int c = 0; c < BT / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tbase + c * 32, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        __stcg(pp + (size_t)(c * 32 + i) * (2 * BW), __uint_as_float(r[i]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(leader_acc_empty);
            if (p.splits > 1) {
                // the last split of this (tile, CTA, quadrant) slab adds the splits
                // in order and writes bf16 Y
                int *cnt = p.counters + tile * 8 + (int)rank * 4 + q;
                int last = 0;
                __threadfence();   // every lane's partial sums, before the warp counts itself
                __syncwarp();
                if (lane == 0)
                    last = atomicAdd(cnt, 1) == p.splits - 1;
                if (__shfl_sync(0xffffffffu, last, 0)) {
                    __threadfence();
                    const int c4 = (lane & 7) * 4;        // 4 columns per lane
                    const int nc = nb * 2 * BW + nloc + c4;
                    const float *src0 =
                        p.partial + (size_t)tile * p.splits * BT * (2 * BW) + nloc + c4;
                    // rows r = 4 * u + lane / 8, eight rows per pass; the
                    // splits are added in order, each pass keeping its 8 loads
                    // of a split in flight together
#pragma unroll 1
                    for (int rb = 0; rb < BT / 4; rb += 8) {
                        float4 acc4[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            acc4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                        for (int sp = 0; sp < p.splits; ++sp) {
                            float4 v[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                v[u] = __ldcg(reinterpret_cast<const float4 *>(
                                    src0 + ((size_t)sp * BT + 4 * (rb + u) + (lane >> 3)) *
                                               (2 * BW)));
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                acc4[u].x += v[u].x;
                                acc4[u].y += v[u].y;
                                acc4[u].z += v[u].z;
                                acc4[u].w += v[u].w;
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int m = mt * BT + 4 * (rb + u) + (lane >> 3);
                            if (m < p.M) {
                                const float e[4] = {acc4[u].x, acc4[u].y, acc4[u].z, acc4[u].w};
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    if (nc + i < p.N)
                                        p.Y[(size_t)m * p.N + nc + i] = f32_to_bf16_bits(e[i]);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0)
                        *cnt = 0;  // leave the counter zero for the next call
                }
            }
        }
    } else if (warp >= kDqWarp0 && warp < kDqWarp0 + kNumDqWarps) {
        // dequantisers: warp -> (quadrant q, half h) of the CTA's 128 weight rows
        const int dw = warp - kDqWarp0;
        const int q = warp & 3, h = dw >> 2;
        const int g = lane >> 2;
        uint32_t it = 0;
        bool ok = true;
        for (int item = pair; item < p.num_items && ok; item += npairs) {
            int tile, kb0, kb1;
            item_range(p, item, tile, kb0, kb1);
            const int nb = tile_nb(p, tile);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int sw = it % L::kSW, sa = it % L::kSA;
                float sca[2] = {1.f, 1.f}, scb[2] = {1.f, 1.f};
                if (F == kMxfp8) {
                    // E8M0 scales of rows ra, ra + 8 for the two 32-blocks of this k-block
                    const int blocks = p.K / 32;
                    const long long ra =
                        (long long)nb * 2 * BW + (int)rank * BW + q * 32 + h * 16 + g;
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int blk = kb * 2 + b;
                        uint32_t ea = 127, eb = 127;
                        if (blk < blocks) {
                            if (ra < p.N)
                                ea = __ldg(p.Ws + ra * blocks + blk);
                            if (ra + 8 < p.N)
                                eb = __ldg(p.Ws + (ra + 8) * blocks + blk);
                        }
                        sca[b] = e8m0_to_f32(ea);
                        scb[b] = e8m0_to_f32(eb);
                    }
                }
                ok = role_wait(&wp_full[sw], (it / L::kSW) & 1, abort_flag, p.hdr, 431) &&
                     role_wait(&a_empty[sa], ((it / L::kSA) & 1) ^ 1, abort_flag, p.hdr, 432);
                if (!ok)
                    break;
                tc_fence_after();
                const uint8_t *wp_slot = smem + L::wp_off + sw * L::wp_slot;
                uint32_t v[16];
                if (F == kInt4)
                    dequant_int4(wp_slot, q, h, lane, p.G, gpk, v);
                else
                    dequant_mx(wp_slot, q, h, lane, sca, scb, v);
                tmem_st_16x256b_x4(
                    tmem_base + ((uint32_t)(q * 32 + h * 16) << 16) + L::a_col + 32 * sa, v);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&wp_empty[sw]);
                    mbar_arrive_cluster(mapa_shared(smem_u32(&a_full[sa]), 0));
                }
            }
        }
    }

    // teardown: every role of both CTAs is done with tensor memory
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == kMmaWarp)
        tmem_dealloc_pair(tmem_base, kTmemCols);
}

template <int F, int BT>
cudaError_t tc_launch(const TcPlan &pl, const CUtensorMap &xm, const CUtensorMap &wm,
                      const CUtensorMap &sm, TcParams p, cudaStream_t stream)
{
    const void *fn = reinterpret_cast<const void *>(&tc_gemm_kernel<F, BT>);
    // the attribute is per device: set once on each
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDeviceCache)
        return cudaErrorInvalidDevice;
    static std::atomic<bool> attr_set[kMaxDeviceCache];
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Layout<F, BT>::smem_bytes);
        if (e != cudaSuccess)
            return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    void *args[] = {const_cast<CUtensorMap *>(&xm), const_cast<CUtensorMap *>(&wm),
                    const_cast<CUtensorMap *>(&sm), &p};
    // the cluster shape (2, 1, 1) is part of the kernel
    return launch_pdl(fn, dim3(pl.grid), dim3(kThreads), Layout<F, BT>::smem_bytes, stream, args);
}

bool x_map(CUtensorMap *m, const void *X, int M, int K, int BT)
{
    return encode_tensor_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M,
                                (uint64_t)K * 2, BK, BT / 2, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int F>
bool tc_plan(int device, int M, int N, int K, TcPlan *plan)
{
    const DeviceInfo &di = device_info(device);
    const int BT = M <= 128 ? 128 : 256;
    const size_t smem = BT == 128 ? Layout<F, 128>::smem_bytes : Layout<F, 256>::smem_bytes;
    if ((size_t)di.smem_optin < smem || di.sms < 2)
        return false;
    TcPlan pl{};
    pl.bm = BT;
    pl.bn = 2 * BW;
    pl.bk = BK;
    pl.mtiles = (M + BT - 1) / BT;
    pl.ntiles = (N + 2 * BW - 1) / (2 * BW);
    const int tiles = pl.mtiles * pl.ntiles;
    const int pairs = di.sms / 2;
    const int kblocks = (K + BK - 1) / BK;
    // Split K when the tiles alone leave pairs idle: pick the split count
    // that minimises the k-blocks of the busiest pair plus a charge of two
    // k-blocks per split for writing and adding the fp32 partial sums.
    int best = 1;
    long long best_cost = (long long)((tiles + pairs - 1) / pairs) * kblocks;
    if (tiles < pairs) {
        for (int sp = 2; sp <= 16 && sp <= kblocks / 4; ++sp) {
            const long long items = (long long)tiles * sp;
            const long long cost =
                ((items + pairs - 1) / pairs) * ((kblocks + sp - 1) / sp) + 2 * sp;
            if (cost < best_cost) {
                best_cost = cost;
                best = sp;
            }
        }
    }
    pl.splits = best;
    const int items = tiles * best;
    if (best > 1 && (size_t)tiles * 8 > kMaxCounters)
        return false;
    pl.grid = 2 * std::min(items, pairs);
    pl.smem = smem;
    pl.partial_bytes = best > 1 ? (size_t)items * BT * 2 * BW * sizeof(float) : 0;
    pl.counters = best > 1 ? (size_t)tiles * 8 : 0;
    *plan = pl;
    return true;
}

}  // namespace

bool plan_w4a16_tc(int device, int M, int N, int K, int G, TcPlan *plan)
{
    (void)G;
    return tc_plan<kInt4>(device, M, N, K, plan);
}

cudaError_t launch_w4a16_tc(const TcPlan &pl, const void *X, const void *packed, int M, int N,
                            int K, int G, void *Y, void *workspace, bool early,
                            cudaStream_t stream)
{
    alignas(64) CUtensorMap xm, wm, sm;
    const uint8_t *codes = static_cast<const uint8_t *>(packed);
    const uint8_t *scales = codes + (size_t)N * K / 2;
    if (!x_map(&xm, X, M, K, pl.bm) ||
        // codes and scales of the column-group layout as rows of one tile's
        // 1 KB (128 u64) and 64 B (8 u64), in memory order; boxes of 4 rows
        !encode_tensor_map_2d(&wm, CU_TENSOR_MAP_DATA_TYPE_UINT64, codes, 128,
                              (uint64_t)(N / 32) * (K / 64), 1024, 128, BW / 32,
                              CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tensor_map_2d(&sm, CU_TENSOR_MAP_DATA_TYPE_UINT64, scales, 8,
                              (uint64_t)(N / 32) * (K / G), 64, 8, BW / 32,
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
    p.splits = pl.splits;
    p.num_items = p.num_tiles * pl.splits;
    p.early = early ? 1 : 0;
    {
        const WorkspaceMap wsm = make_workspace_map(pl.counters, pl.partial_bytes);
        p.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wsm.counters_off);
        p.partial = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + wsm.partial_off);
    }
    if (pl.bm == 128)
        return tc_launch<kInt4, 128>(pl, xm, wm, sm, p, stream);
    return tc_launch<kInt4, 256>(pl, xm, wm, sm, p, stream);
}

bool plan_mxfp8_tc(int device, int M, int N, int K, TcPlan *plan)
{
    return tc_plan<kMxfp8>(device, M, N, K, plan);
}

cudaError_t launch_mxfp8_tc(const TcPlan &pl, const void *X, const uint8_t *Wq,
                            const uint8_t *Ws, int M, int N, int K, void *Y, void *workspace,
                            bool early, cudaStream_t stream)
{
    alignas(64) CUtensorMap xm, wm;
    if (!x_map(&xm, X, M, K, pl.bm) ||
        !encode_tensor_map_2d(&wm, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                              (uint64_t)K, BK, BW, CU_TENSOR_MAP_SWIZZLE_64B))
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
    p.splits = pl.splits;
    p.num_items = p.num_tiles * pl.splits;
    p.early = early ? 1 : 0;
    {
        const WorkspaceMap wsm = make_workspace_map(pl.counters, pl.partial_bytes);
        p.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wsm.counters_off);
        p.partial = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + wsm.partial_off);
    }
    if (pl.bm == 128)
        return tc_launch<kMxfp8, 128>(pl, xm, wm, wm, p, stream);
    return tc_launch<kMxfp8, 256>(pl, xm, wm, wm, p, stream);
}

}  // namespace mxg
