// Device helpers shared by the mxg kernels (sm_100a only).
//
// PTX wrappers for mbarriers, bulk and tensor copies, warp-level MMA and the
// exact weight decoders of both formats.  Nothing here allocates or
// synchronizes the device.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "mxg.h"

namespace mxg {

// ---------------------------------------------------------------- workspace
// The first 256 bytes of every workspace are a header; `status` receives the
// first error a kernel records and `where` a code for the place it happened.
struct WsHeader {
    int status;
    int where;
    int reserved[62];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per pipeline wait

__device__ __forceinline__ void record_error(WsHeader *h, int status, int where)
{
    if (atomicCAS(&h->status, 0, status) == 0)
        atomicExch(&h->where, where);
}

// ------------------------------------------------ re-packed weight layout
// The re-packed INT4 (P = 1 code plane) and INT8 (P = 2: a plane of low and
// a plane of high nibbles) weights are stored by column groups of eight n32
// tiles (256 columns; when N is not a multiple of 256 the last group holds
// the remaining tiles).  Codes: group gr takes 8 * 16 * K * P bytes (less
// for the last group), as K/64 chunks of [tiles of the group][1024 * P B]; the
// 1024 * P bytes of one tile and chunk are [2 halves][P planes][32 lanes]
// [16 B].  So the codes of a group for any run of k64 chunks form one
// contiguous range, which both GEMM paths move with one bulk copy.  Scales
// follow all the codes: group gr takes 8 * (K/G) * 64 bytes (less for the
// last group), as K/G scale groups of [tiles of the group][64 B], the 64
// bytes of a tile being [8][4 halves] (see the re-pack).
__host__ __device__ __forceinline__ int group_tiles(int gr, int ntiles)
{
    return ntiles - 8 * gr < 8 ? ntiles - 8 * gr : 8;
}

// Byte offset of the codes of (n32 tile, k64 chunk) in a layer of ntiles tiles.
__host__ __device__ __forceinline__ size_t code_offset(int tile, int chunk, int K, int ntiles,
                                                       int P)
{
    const int gr = tile >> 3;
    return (size_t)gr * 8 * 16 * K * P +
           ((size_t)chunk * group_tiles(gr, ntiles) + (tile & 7)) * 1024 * P;
}

// Byte offset, inside the scale region, of the 64 scale bytes of (n32 tile,
// scale group).
__host__ __device__ __forceinline__ size_t scale_offset(int tile, int kgroup, int K, int G,
                                                        int ntiles)
{
    const int gr = tile >> 3;
    return (size_t)gr * 8 * (K / G) * 64 + ((size_t)kgroup * group_tiles(gr, ntiles) + (tile & 7)) * 64;
}

// ------------------------------------------------------------------- basics
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One bounded probe of the phase: the thread may be suspended (not issuing)
// for up to kSuspendNs while the phase is incomplete, so waiting warps leave
// the issue slots to working ones.
constexpr uint32_t kSuspendNs = 1000000;  // 1 ms

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Non-blocking probe: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after
// `limit_ns` nanoseconds without completion.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (global_ns() - t0 > limit_ns)
            return false;
    }
}

// ------------------------------------------------------------- bulk copies
__device__ __forceinline__ uint64_t l2_policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Contiguous global -> shared copy completing on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 2-D tiled tensor copy of box (c0, c1) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Warm L2 with one 2-D tensor-map box (a hint, like prefetch_l2).
__device__ __forceinline__ void prefetch_tensor_l2(const CUtensorMap *map, int c0, int c1)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map),
                 "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ------------------------------------------- programmatic dependent launch
// Let the next kernel in the stream start its prologue on SMs this grid
// frees (it still waits for this grid's results before touching them).
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Wait until the grids this one depends on have completed and their memory
// operations are visible (returns at once without such a dependency).
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Warm L2 with a global byte range (16-byte aligned, size % 16 == 0).  Only a
// hint: L2 is the point of coherence, so data written later is not hidden.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------ loads
__device__ __forceinline__ uint4 lds128(const void *p)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t lds32a(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t lds32(const void *p)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}

// Read-only 16-byte global load kept in L1 (activations are re-read by
// many warps).  Visible to the compiler, which may schedule it early.
__device__ __forceinline__ uint4 ldg128(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ uint2 lds64(const void *p)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
    return v;
}

// The same shared-memory loads from a 32-bit shared-window address (no
// generic-to-shared conversion per access).
__device__ __forceinline__ uint4 lds128a(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ uint2 lds64a(uint32_t a)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

// 16-byte load from L2 (bypassing L1), for partial sums written by other CTAs.
__device__ __forceinline__ float4 ldcg_f4(const float *p)
{
    return __ldcg(reinterpret_cast<const float4 *>(p));
}

// ----------------------------------------------------------- warp-level MMA
// D(16x8, fp32) += A(16x16, bf16, row) * B(16x8, bf16, col).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B with a zero accumulator input (starts a new partial sum).
__device__ __forceinline__ void mma_bf16_16816_zero(float (&d)[4], uint32_t a0, uint32_t a1,
                                                    uint32_t a2, uint32_t a3, uint32_t b0,
                                                    uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// The same MMAs on fp16 operands.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816_zero(float (&d)[4], uint32_t a0, uint32_t a1,
                                                   uint32_t a2, uint32_t a3, uint32_t b0,
                                                   uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// Arrival counter increment with acquire-release semantics at GPU scope:
// publishes the caller's (and, after a warp barrier, its warp's) prior
// stores and, for the last arriver, makes the other contributors' stores
// visible.
// Named barrier over `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int atomic_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// --------------------------------------------------------- INT4 decoding
// Two 4-bit codes q_lo = bits [s, s+3] and q_hi = bits [16+s, 16+s+3] of w,
// returned as the bf16 pair (q_lo - 8, q_hi - 8).  Exact: 0x4300 | q is the
// bf16 value 128 + q (one unit in the last place is 1 at exponent 7), and
// subtracting 136 leaves the small integer q - 8.
// The same pair, returned as the bf16 pair (128 + q_lo, 128 + q_hi): one
// mask-and-or, no arithmetic.  A product sum over such weights exceeds the
// sum over (q - 8) by 136 times the sum of the activations.  Written as one
// three-input logic op with both constants in registers: as a C expression
// the and and the or were issued as two ALU instructions (ncu instruction
// counts of the streaming kernel: 30 % fewer ALU instructions this way).
template <int S>
__device__ __forceinline__ uint32_t int4_pair_plus128(uint32_t w)
{
    uint32_t r;
    const uint32_t x = S ? (w >> S) : w;
    // (x & mask) | magic: truth table 0xEA for (a & b) | c
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x000F000Fu), "r"(0x43004300u));
    return r;
}

// The fp16 form: with the magic 0x6400 (1024.0, whose unit in the last
// place is 1) a nibble anywhere in the low byte of a half lands in the
// mantissa, so one mask-and-or gives the pair (1024 + q_lo, 1024 + q_hi)
// from bits 0..3 / 16..19 (HI = 0) or (1024 + 16 q_lo, 1024 + 16 q_hi) from
// bits 4..7 / 20..23 (HI = 1); a shift by 8 reaches the other two nibble
// positions.  Four registers of a 32-bit word then take four mask-and-ors
// and one shift, not four and three.
template <int HI>
__device__ __forceinline__ uint32_t int4_pair_f16(uint32_t x)
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;"
        : "=r"(r)
        : "r"(x), "r"(HI ? 0x00F000F0u : 0x000F000Fu), "r"(0x64006400u));
    return r;
}

template <int S>
__device__ __forceinline__ uint32_t int4_pair_minus8(uint32_t w)
{
    const uint32_t t = int4_pair_plus128<S>(w);
    // written with intrinsics so the compiler can fold the constant operand
    const __nv_bfloat162 v = __hadd2(*reinterpret_cast<const __nv_bfloat162 *>(&t),
                                     __halves2bfloat162(__ushort_as_bfloat16(0xC308),
                                                        __ushort_as_bfloat16(0xC308)));
    return *reinterpret_cast<const uint32_t *>(&v);
}

// An fp16 scale s split as s = hi + lo with hi, lo both bf16: hi keeps the
// top 8 significant bits of s, lo the remaining (at most 3) bits.  Both are
// broadcast to the two halves of a bf16x2 register.
struct ScaleSplit {
    uint32_t hi2;
    uint32_t lo2;
};

__device__ __forceinline__ ScaleSplit split_scale(uint16_t s_bits)
{
    const float f = __half2float(__ushort_as_half(s_bits));
    const uint32_t fb = __float_as_uint(f);
    const uint32_t hi = fb & 0xFFFF0000u;                 // truncated to bf16
    const float lo = f - __uint_as_float(hi);              // exact remainder
    const uint32_t lob = __float_as_uint(lo) >> 16;        // exact in bf16
    ScaleSplit r;
    r.hi2 = hi | (hi >> 16);
    r.lo2 = lob | (lob << 16);
    return r;
}

// bf16 nearest to (q - 8) * s for a pair of exact (q - 8) values, with one
// rounding: (q-8)*lo is exact in bf16 (<= 4 x 3 significant bits), and the
// fused multiply-add (q-8)*hi + (q-8)*lo rounds the exact product once.
__device__ __forceinline__ uint32_t scale_pair_rn(uint32_t qm8, const ScaleSplit &s)
{
    uint32_t t, r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(qm8), "r"(s.lo2));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(qm8), "r"(s.hi2), "r"(t));
    return r;
}

// -------------------------------------------------------- MXFP8 decoding
// fp32 value of an E8M0 exponent: 2^(E - 127) (E = 0 is the fp32 subnormal
// 2^-127; E = 255, NaN in the format, is not checked).
__device__ __forceinline__ float e8m0_to_f32(uint32_t e)
{
    return e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);
}

// Four E4M3 codes (the bytes of w, byte 0 first) as two f16 pairs: r01 =
// (w0, w1), r23 = (w2, w3); exact (every E4M3 value is an f16 value).
__device__ __forceinline__ void e4m3x2_f16x2(uint32_t w, uint32_t &r01, uint32_t &r23)
{
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(r01), "=r"(r23)
        : "r"(w));
}

// Four E4M3 codes (the bytes of w, byte 0 first) times `scale`, as two bf16
// pairs: r01 = (w0, w1), r23 = (w2, w3).  E4M3 -> f16 is exact in hardware,
// f16 -> f32 is exact, the product with a power of two is exact in fp32, and
// the only rounding is the final fp32 -> bf16 (nearest, ties to even).
__device__ __forceinline__ void e4m3x4_scaled(uint32_t w, float scale, uint32_t &r01, uint32_t &r23)
{
    uint32_t h01, h23;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(h01), "=r"(h23)
        : "r"(w));
    float2 f01 = __half22float2(*reinterpret_cast<__half2 *>(&h01));
    float2 f23 = __half22float2(*reinterpret_cast<__half2 *>(&h23));
    // packed fp32 multiplies (two lanes per instruction)
    asm("{\n\t.reg .b64 a, b, s;\n\t"
        "mov.b64 s, {%4, %4};\n\t"
        "mov.b64 a, {%0, %1};\n\t"
        "mov.b64 b, {%2, %3};\n\t"
        "mul.rn.f32x2 a, a, s;\n\t"
        "mul.rn.f32x2 b, b, s;\n\t"
        "mov.b64 {%0, %1}, a;\n\t"
        "mov.b64 {%2, %3}, b;\n\t}"
        : "+f"(f01.x), "+f"(f01.y), "+f"(f23.x), "+f"(f23.y)
        : "f"(scale));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r01) : "f"(f01.y), "f"(f01.x));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r23) : "f"(f23.y), "f"(f23.x));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

}  // namespace mxg
