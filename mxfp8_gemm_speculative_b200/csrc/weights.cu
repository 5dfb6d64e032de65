// Offline weight re-pack for INT4 W4A16 and the decode kernels the tests use.
//
// Re-packed INT4 layout (one buffer, codes then scales), by column groups of
// eight n32 tiles (code_offset / scale_offset in common.cuh):
//   codes  [N/256 groups][K/64 chunks][tiles of the group][2 halves][32 lanes][4 words]
//   scales [N/256 groups][K/G][tiles of the group][8][4 halves]
// For n32 tile T, k64 chunk c, half h and lane = 4*g + t (g = 0..7,
// t = 0..3), the lane's 16 bytes hold columns na = 32T + 16h + g and
// nb = na + 8.  Word j covers the four rows k0 = 64c + 16j + 4t .. k0 + 3:
//   bits [ 0, 4) q(na, k0)    [16,20) q(na, k0+1)
//   bits [ 4, 8) q(nb, k0)    [20,24) q(nb, k0+1)
//   bits [ 8,12) q(na, k0+2)  [24,28) q(na, k0+3)
//   bits [12,16) q(nb, k0+2)  [28,32) q(nb, k0+3)
// so that (w >> 4r) & 0x000F000F puts a pair of codes in the two halves of
// one bf16x2 register.  For the weight-streaming path, word j of the 32
// lanes is exactly the A operand of one m16n8k16 MMA step over
// k = 64c + 16j .. 64c + 16j + 15 (rows na, nb; lane t holds k positions
// 4t .. 4t+3 of the step, and the activations are loaded in the same
// order), so every step lies inside one group of 32.  For the tensor-core
// path the same 16 bytes, decoded in register order (pair 0, pair 2) for
// column na and (pair 1, pair 3) for nb, are exactly one thread's share of
// a 16-lane x 256-bit tensor-memory store per word (lanes na, nb; columns
// 2t, 2t+1 of the k16 block j).  Scales: entry (T, group, g) is the four
// halves s[32T+g], s[32T+g+8], s[32T+16+g], s[32T+16+g+8].
#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

__device__ __forceinline__ int chunk_k0(int c, int t, int j)
{
    return c * 64 + 16 * j + 4 * t;
}

// Input words: word (i, n) (codes of rows 8i .. 8i+7 of column n, LSB
// first) sits at qweight[i * wk + n * wn]: wk = N, wn = 1 for GPTQ
// qweight[K/8][N]; wk = 1, wn = K/8 for compressed-tensors
// weight_packed[N][K/8].
// Tiles [tile0, tile0 + N/32) of a layer of ntiles tiles (a fused part
// starts at a later tile).
__global__ void repack_codes_kernel(const int32_t *__restrict__ qweight, int K, int N,
                                    size_t wk, size_t wn, int tile0, int ntiles,
                                    uint8_t *__restrict__ out)
{
    const long long total = (long long)(N / 32) * (K / 64) * 64;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int lane = (int)(idx & 31);
    const int h = (int)((idx >> 5) & 1);
    const long long rest = idx >> 6;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int T = (int)(rest / kc_count);
    const int g = lane >> 2, t = lane & 3;
    const int na = T * 32 + h * 16 + g, nb = na + 8;
    uint32_t words[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k0 = chunk_k0(c, t, j);
        const int shift = 4 * (k0 & 7);
        const uint32_t qa = ((uint32_t)qweight[(size_t)(k0 >> 3) * wk + na * wn]) >> shift;
        const uint32_t qb = ((uint32_t)qweight[(size_t)(k0 >> 3) * wk + nb * wn]) >> shift;
        uint32_t w = 0;
        w |= (qa & 0xFu);
        w |= ((qa >> 4) & 0xFu) << 16;
        w |= (qb & 0xFu) << 4;
        w |= ((qb >> 4) & 0xFu) << 20;
        w |= ((qa >> 8) & 0xFu) << 8;
        w |= ((qa >> 12) & 0xFu) << 24;
        w |= ((qb >> 8) & 0xFu) << 12;
        w |= ((qb >> 12) & 0xFu) << 28;
        words[j] = w;
    }
    *reinterpret_cast<uint4 *>(out + code_offset(tile0 + T, c, K, ntiles, 1) + h * 512 +
                               lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
}

// INT8 codes (4 per int32 word along K, byte j = row 4i + j, zero point
// 128) into two planes in the INT4 layout: one output pair per (tile, k64
// chunk, half, lane), the low-nibble plane's 16 bytes then, 512 bytes on,
// the high-nibble plane's.  Word (i, n) sits at qweight[i * wk + n * wn]:
// wk = N, wn = 1 for GPTQ-style [K/4][N]; wk = 1, wn = K/4 for the
// compressed-tensors [N][K/4] export.
__global__ void repack8_codes_kernel(const int32_t *__restrict__ qweight, int K, int N, size_t wk,
                                     size_t wn, int ntiles, uint8_t *__restrict__ out)
{
    const long long total = (long long)(N / 32) * (K / 64) * 64;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int lane = (int)(idx & 31);
    const int h = (int)((idx >> 5) & 1);
    const long long rest = idx >> 6;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int T = (int)(rest / kc_count);
    const int g = lane >> 2, t = lane & 3;
    const int na = T * 32 + h * 16 + g, nb = na + 8;
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k0 = chunk_k0(c, t, j);  // a multiple of 4: one word holds k0 .. k0 + 3
        const uint32_t qa = (uint32_t)qweight[(size_t)(k0 >> 2) * wk + na * wn];
        const uint32_t qb = (uint32_t)qweight[(size_t)(k0 >> 2) * wk + nb * wn];
        // nibble plane p of code r (r = 0..3) of column a / b
        auto nib = [](uint32_t q, int r, int p) { return (q >> (8 * r + 4 * p)) & 0xFu; };
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            uint32_t w = 0;
            w |= nib(qa, 0, p);
            w |= nib(qa, 1, p) << 16;
            w |= nib(qb, 0, p) << 4;
            w |= nib(qb, 1, p) << 20;
            w |= nib(qa, 2, p) << 8;
            w |= nib(qa, 3, p) << 24;
            w |= nib(qb, 2, p) << 12;
            w |= nib(qb, 3, p) << 28;
            (p ? hi : lo)[j] = w;
        }
    }
    // (T, c): [h][plane][lane][16 B]
    uint4 *base = reinterpret_cast<uint4 *>(out + code_offset(T, c, K, ntiles, 2)) + h * 2 * 32;
    base[lane] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    base[32 + lane] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
}

// Scale (group, n) sits at scales[group * sg + n * sn]: sg = N, sn = 1 for
// GPTQ scales[K/G][N]; sg = 1, sn = K/G for compressed-tensors
// weight_scale[N][K/G].
__global__ void repack_scales_kernel(const uint16_t *__restrict__ scales, int K, int N, int G,
                                     size_t sg, size_t sn, int tile0, int ntiles,
                                     uint8_t *__restrict__ out)
{
    const int groups = K / G;
    const long long total = (long long)(N / 32) * groups * 32;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int i4 = (int)(idx & 3);
    const int g = (int)((idx >> 2) & 7);
    const long long rest = idx >> 5;
    const int grp = (int)(rest % groups);
    const int T = (int)(rest / groups);
    const int n = T * 32 + g + 8 * (i4 & 1) + 16 * (i4 >> 1);
    reinterpret_cast<uint16_t *>(out + scale_offset(tile0 + T, grp, K, G, ntiles))[g * 4 + i4] =
        scales[(size_t)grp * sg + n * sn];
}

// One thread per 16-byte code chunk: writes 16 codes of two columns, and
// optionally their fp32 and bf16 dequantized values, using the decoders of
// the GEMM paths.
__global__ void unpack_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ sc,
                              int K, int N, int G, uint8_t *__restrict__ out_codes,
                              float *__restrict__ w_fp32, uint16_t *__restrict__ w_bf16)
{
    const long long total = (long long)(N / 32) * (K / 64) * 64;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int lane = (int)(idx & 31);
    const int h = (int)((idx >> 5) & 1);
    const long long rest = idx >> 6;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int T = (int)(rest / kc_count);
    const int g = lane >> 2, t = lane & 3;
    const int ntiles = N / 32;
    const uint4 v =
        *reinterpret_cast<const uint4 *>(codes + code_offset(T, c, K, ntiles, 1) + h * 512 + lane * 16);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    const int na = T * 32 + h * 16 + g, nb = na + 8;

#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k0 = chunk_k0(c, t, j);
        const uint16_t *e =
            reinterpret_cast<const uint16_t *>(sc + scale_offset(T, k0 / G, K, G, ntiles)) + g * 4 +
            2 * h;
        const uint16_t s_a = e[0], s_b = e[1];
        const ScaleSplit sp_a = split_scale(s_a), sp_b = split_scale(s_b);
        const float fa = __half2float(__ushort_as_half(s_a));
        const float fb = __half2float(__ushort_as_half(s_b));
        const uint32_t w = wv[j];
        const uint32_t ba0 = scale_pair_rn(int4_pair_minus8<0>(w), sp_a);
        const uint32_t ba1 = scale_pair_rn(int4_pair_minus8<8>(w), sp_a);
        const uint32_t bb0 = scale_pair_rn(int4_pair_minus8<4>(w), sp_b);
        const uint32_t bb1 = scale_pair_rn(int4_pair_minus8<12>(w), sp_b);
        const int qa[4] = {(int)(w & 0xF), (int)((w >> 16) & 0xF), (int)((w >> 8) & 0xF),
                           (int)((w >> 24) & 0xF)};
        const int qb[4] = {(int)((w >> 4) & 0xF), (int)((w >> 20) & 0xF), (int)((w >> 12) & 0xF),
                           (int)((w >> 28) & 0xF)};
        const size_t oa = (size_t)na * K + k0, ob = (size_t)nb * K + k0;
        if (out_codes) {
            *reinterpret_cast<uint32_t *>(out_codes + oa) =
                qa[0] | (qa[1] << 8) | (qa[2] << 16) | ((uint32_t)qa[3] << 24);
            *reinterpret_cast<uint32_t *>(out_codes + ob) =
                qb[0] | (qb[1] << 8) | (qb[2] << 16) | ((uint32_t)qb[3] << 24);
        }
        if (w_fp32) {
            *reinterpret_cast<float4 *>(w_fp32 + oa) =
                make_float4((float)(qa[0] - 8) * fa, (float)(qa[1] - 8) * fa,
                            (float)(qa[2] - 8) * fa, (float)(qa[3] - 8) * fa);
            *reinterpret_cast<float4 *>(w_fp32 + ob) =
                make_float4((float)(qb[0] - 8) * fb, (float)(qb[1] - 8) * fb,
                            (float)(qb[2] - 8) * fb, (float)(qb[3] - 8) * fb);
        }
        if (w_bf16) {
            *reinterpret_cast<uint2 *>(w_bf16 + oa) = make_uint2(ba0, ba1);
            *reinterpret_cast<uint2 *>(w_bf16 + ob) = make_uint2(bb0, bb1);
        }
    }
}

// One thread per 4 codes.
__global__ void mxfp8_dequant_kernel(const uint32_t *__restrict__ Wq, const uint8_t *__restrict__ Ws,
                                     int N, int K, uint2 *__restrict__ out)
{
    const long long total = (long long)N * (K / 4);
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const long long n = idx / (K / 4);
    const int k = (int)(idx - n * (K / 4)) * 4;
    const float s = e8m0_to_f32(Ws[n * (K / 32) + k / 32]);
    uint32_t r01, r23;
    e4m3x4_scaled(Wq[idx], s, r01, r23);
    out[idx] = make_uint2(r01, r23);
}

// MXFP8 re-pack for the weight-streaming kernel, by column groups of eight
// n32 tiles like the INT4 layout:
//   codes  [N/256 groups][K/64 chunks][tiles of the group][2 halves][2 pairs of steps][32 lanes][16 B]
//   scales [N/256 groups][K/64 chunks][tiles of the group][2 blocks][8][4 B]
// Lane 4g + t of half h holds columns na = 32T + 16h + g and nb = na + 8;
// for step j (k0 = 64c + 16j + 4t) its 8 bytes are the E4M3 codes
// (na, k0) (na, k0+1) (nb, k0) (nb, k0+1) (na, k0+2) (na, k0+3) (nb, k0+2)
// (nb, k0+3): the f16 pairs of one m16n8k16 A operand after the hardware
// conversion, in the INT4 layout's k order.  Scale entry (T, c, b, g) holds
// the E8M0 of block 2c + b for columns 32T + g, +8, +16, +24.
__global__ void mxfp8_repack_codes_kernel(const uint32_t *__restrict__ Wq, int N, int K,
                                          int ntiles, uint8_t *__restrict__ out)
{
    const long long total = (long long)(N / 32) * (K / 64) * 2 * 2 * 32;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int lane = (int)(idx & 31);
    const int q = (int)((idx >> 5) & 1);      // pair of steps 2q, 2q + 1
    const int h = (int)((idx >> 6) & 1);
    const long long rest = idx >> 7;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int T = (int)(rest / kc_count);
    const int g = lane >> 2, t = lane & 3;
    const size_t na = (size_t)T * 32 + h * 16 + g, nb = na + 8;
    uint32_t w[4];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int k0 = chunk_k0(c, t, 2 * q + s);   // 4 codes of each column
        const uint32_t qa = Wq[(na * K + k0) >> 2];
        const uint32_t qb = Wq[(nb * K + k0) >> 2];
        w[2 * s] = (qa & 0xFFFFu) | (qb << 16);
        w[2 * s + 1] = (qa >> 16) | (qb & 0xFFFF0000u);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out + code_offset(T, c, K, ntiles, 2)) + (h * 2 + q) * 32;
    dst[lane] = make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void mxfp8_repack_scales_kernel(const uint8_t *__restrict__ Ws, int N, int K,
                                           int ntiles, uint8_t *__restrict__ out)
{
    const long long total = (long long)(N / 32) * (K / 64) * 2 * 8;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int g = (int)(idx & 7);
    const int b = (int)((idx >> 3) & 1);
    const long long rest = idx >> 4;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int T = (int)(rest / kc_count);
    const size_t blocks = (size_t)K / 32, blk = (size_t)c * 2 + b, n0 = (size_t)T * 32 + g;
    const uint32_t v = (uint32_t)Ws[n0 * blocks + blk] | ((uint32_t)Ws[(n0 + 8) * blocks + blk] << 8) |
                       ((uint32_t)Ws[(n0 + 16) * blocks + blk] << 16) |
                       ((uint32_t)Ws[(n0 + 24) * blocks + blk] << 24);
    // scale_offset with G = 64: 64 bytes per tile and chunk
    *reinterpret_cast<uint32_t *>(out + scale_offset(T, c, K, 64, ntiles) + b * 32 + g * 4) = v;
}

__global__ void wait_timeout_kernel(WsHeader *hdr, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // nothing ever arrives on `bar`: the wait must give up after limit_ns
    if (!mbar_wait(&bar, 0, limit_ns)) {
        if (threadIdx.x == 0)
            record_error(hdr, MXG_ERR_TIMEOUT, 1);
    }
}

// Launched after the re-pack kernels: a GEMM right after w4a16_repack on the
// stream may load weights before it waits for the kernel before it, which is
// then this one (it starts only once the re-pack kernels have completed).
__global__ void repack_done_kernel() {}

inline unsigned blocks_for(long long total, int threads)
{
    return (unsigned)((total + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_w4a16_repack_part(const int32_t *qweight, const uint16_t *scales, int K, int Np,
                                     int G, int n0, int N, void *packed, cudaStream_t stream)
{
    // part columns [n0, n0 + Np) of a fused layer with N columns: its n32
    // tiles are tiles n0 / 32 onwards of the fused layer
    const long long nchunks = (long long)(Np / 32) * (K / 64) * 64;
    uint8_t *out = static_cast<uint8_t *>(packed);
    repack_codes_kernel<<<blocks_for(nchunks, 256), 256, 0, stream>>>(
        qweight, K, Np, (size_t)Np, 1, n0 / 32, N / 32, out);
    const long long nsc = (long long)(Np / 32) * (K / G) * 32;
    repack_scales_kernel<<<blocks_for(nsc, 256), 256, 0, stream>>>(
        scales, K, Np, G, (size_t)Np, 1, n0 / 32, N / 32, out + (size_t)N * K / 2);
    return cudaGetLastError();
}

cudaError_t launch_repack_done(cudaStream_t stream)
{
    repack_done_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

cudaError_t launch_w4a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int G,
                                bool n_major, void *packed, cudaStream_t stream)
{
    // GPTQ inputs are K-major ([K/8][N] words, [K/G][N] scales), compressed-
    // tensors inputs N-major ([N][K/8], [N][K/G]); the output is the same
    const size_t wk = n_major ? 1 : (size_t)N, wn = n_major ? (size_t)K / 8 : 1;
    const size_t sg = n_major ? 1 : (size_t)N, sn = n_major ? (size_t)(K / G) : 1;
    const long long nchunks = (long long)(N / 32) * (K / 64) * 64;
    uint8_t *out = static_cast<uint8_t *>(packed);
    repack_codes_kernel<<<blocks_for(nchunks, 256), 256, 0, stream>>>(qweight, K, N, wk, wn, 0,
                                                                       N / 32, out);
    const long long nsc = (long long)(N / 32) * (K / G) * 32;
    repack_scales_kernel<<<blocks_for(nsc, 256), 256, 0, stream>>>(scales, K, N, G, sg, sn, 0,
                                                                   N / 32, out + (size_t)N * K / 2);
    repack_done_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

cudaError_t launch_w8a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int G,
                                bool n_major, void *packed, cudaStream_t stream)
{
    const size_t wk = n_major ? 1 : (size_t)N, wn = n_major ? (size_t)K / 4 : 1;
    const size_t sg = n_major ? 1 : (size_t)N, sn = n_major ? (size_t)(K / G) : 1;
    const long long npairs = (long long)(N / 32) * (K / 64) * 64;
    repack8_codes_kernel<<<blocks_for(npairs, 256), 256, 0, stream>>>(
        qweight, K, N, wk, wn, N / 32, static_cast<uint8_t *>(packed));
    const long long nsc = (long long)(N / 32) * (K / G) * 32;
    repack_scales_kernel<<<blocks_for(nsc, 256), 256, 0, stream>>>(
        scales, K, N, G, sg, sn, 0, N / 32, static_cast<uint8_t *>(packed) + (size_t)N * K);
    repack_done_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

cudaError_t launch_w4a16_unpack(const void *packed, int K, int N, int G, uint8_t *codes,
                                float *w_fp32, uint16_t *w_bf16, cudaStream_t stream)
{
    const long long nchunks = (long long)(N / 32) * (K / 64) * 64;
    const uint8_t *pk = static_cast<const uint8_t *>(packed);
    unpack_kernel<<<blocks_for(nchunks, 256), 256, 0, stream>>>(pk, pk + (size_t)N * K / 2, K, N, G,
                                                                codes, w_fp32, w_bf16);
    return cudaGetLastError();
}

cudaError_t launch_mxfp8_repack(const uint8_t *Wq, const uint8_t *Ws, int N, int K, void *packed,
                               cudaStream_t stream)
{
    uint8_t *out = static_cast<uint8_t *>(packed);
    const long long nc = (long long)(N / 32) * (K / 64) * 128;
    mxfp8_repack_codes_kernel<<<blocks_for(nc, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(Wq), N, K, N / 32, out);
    const long long ns = (long long)(N / 32) * (K / 64) * 16;
    mxfp8_repack_scales_kernel<<<blocks_for(ns, 256), 256, 0, stream>>>(Ws, N, K, N / 32,
                                                                        out + (size_t)N * K);
    repack_done_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

cudaError_t launch_mxfp8_dequant(const uint8_t *Wq, const uint8_t *Ws, int N, int K,
                                 uint16_t *w_bf16, cudaStream_t stream)
{
    const long long total = (long long)N * (K / 4);
    mxfp8_dequant_kernel<<<blocks_for(total, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(Wq), Ws, N, K, reinterpret_cast<uint2 *>(w_bf16));
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(void *workspace, int limit_us, cudaStream_t stream)
{
    wait_timeout_kernel<<<1, 32, 0, stream>>>(reinterpret_cast<WsHeader *>(workspace),
                                              (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace mxg
