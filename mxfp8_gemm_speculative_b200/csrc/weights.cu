// Offline weight re-pack for INT4 W4A16 and the decode kernels the tests use.
//
// Re-packed INT4 layout (one buffer, codes then scales):
//   codes  [N/16][K/64][32 lanes][4 words]
//   scales [N/16][K/G][16 halves]
// For n16 tile `nt`, k64 chunk `c` and lane = 4*g + t (g = 0..7, t = 0..3),
// the lane's 16 bytes hold columns n = 16nt + g and n + 8 for the sixteen
// rows k = 64c + 16t .. 64c + 16t + 15.  Word j covers k0 = 64c + 16t + 4j:
//   bits [ 0, 4) q(n,   k0)    [16,20) q(n,   k0+1)
//   bits [ 4, 8) q(n+8, k0)    [20,24) q(n+8, k0+1)
//   bits [ 8,12) q(n,   k0+2)  [24,28) q(n,   k0+3)
//   bits [12,16) q(n+8, k0+2)  [28,32) q(n+8, k0+3)
// so that masking (w >> 4r) & 0x000F000F yields a pair of codes that lands in
// the two halves of one bf16x2 register: r = 0..3 give exactly the four A
// registers of an m16n8k16 MMA step whose 16 k positions are the
// k0 .. k0+3 of the four lanes t (the k order inside a step is permuted
// consistently with the activations, which the sum does not see), and they
// also give four consecutive k of one column for the tensor-core path.
// Scales: the 16 halves of (nt, group) are ordered s[n0], s[n0+8], s[n0+1],
// s[n0+9], ... so that lane g reads its two columns as one 32-bit word.
#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

__global__ void repack_codes_kernel(const int32_t *__restrict__ qweight, int K, int N,
                                    uint4 *__restrict__ out)
{
    const long long total = (long long)(N / 16) * (K / 64) * 32;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int lane = (int)(idx & 31);
    const long long rest = idx >> 5;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int nt = (int)(rest / kc_count);
    const int g = lane >> 2, t = lane & 3;
    const int na = nt * 16 + g, nb = na + 8;
    uint32_t words[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k0 = c * 64 + t * 16 + j * 4;
        const int shift = 4 * (k0 & 7);
        const uint32_t qa = ((uint32_t)qweight[(size_t)(k0 >> 3) * N + na]) >> shift;
        const uint32_t qb = ((uint32_t)qweight[(size_t)(k0 >> 3) * N + nb]) >> shift;
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
    out[idx] = make_uint4(words[0], words[1], words[2], words[3]);
}

__global__ void repack_scales_kernel(const uint16_t *__restrict__ scales, int K, int N, int G,
                                     uint16_t *__restrict__ out)
{
    const int groups = K / G;
    const long long total = (long long)(N / 16) * groups * 16;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int i = (int)(idx & 15);
    const long long rest = idx >> 4;
    const int grp = (int)(rest % groups);
    const int nt = (int)(rest / groups);
    const int n = nt * 16 + (i >> 1) + ((i & 1) ? 8 : 0);
    out[idx] = scales[(size_t)grp * N + n];
}

// One thread per 16-byte code chunk: writes 16 codes of two columns, and
// optionally their fp32 and bf16 dequantized values, using the decoders of
// the GEMM paths.
__global__ void unpack_kernel(const uint4 *__restrict__ codes, const uint32_t *__restrict__ sc,
                              int K, int N, int G, uint8_t *__restrict__ out_codes,
                              float *__restrict__ w_fp32, uint16_t *__restrict__ w_bf16)
{
    const long long total = (long long)(N / 16) * (K / 64) * 32;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    const int lane = (int)(idx & 31);
    const long long rest = idx >> 5;
    const int kc_count = K / 64;
    const int c = (int)(rest % kc_count);
    const int nt = (int)(rest / kc_count);
    const int g = lane >> 2, t = lane & 3;
    const int groups = K / G;
    const int kbase = c * 64 + t * 16;
    // the lane's 16 rows lie in one group for G >= 32
    const uint32_t sword = sc[((size_t)nt * groups + kbase / G) * 8 + g];
    const uint16_t s_a = (uint16_t)(sword & 0xFFFF), s_b = (uint16_t)(sword >> 16);
    const ScaleSplit sp_a = split_scale(s_a), sp_b = split_scale(s_b);
    const float fa = __half2float(__ushort_as_half(s_a)), fb = __half2float(__ushort_as_half(s_b));
    const uint4 v = codes[idx];
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};

    uint8_t qa[16], qb[16];
    uint32_t ba[8], bb[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = wv[j];
        // decoded exactly as the MMA operands: pairs (k0, k0+1) and (k0+2, k0+3)
        const uint32_t a01 = int4_pair_minus8<0>(w), b01 = int4_pair_minus8<4>(w);
        const uint32_t a23 = int4_pair_minus8<8>(w), b23 = int4_pair_minus8<12>(w);
        ba[2 * j] = scale_pair_rn(a01, sp_a);
        ba[2 * j + 1] = scale_pair_rn(a23, sp_a);
        bb[2 * j] = scale_pair_rn(b01, sp_b);
        bb[2 * j + 1] = scale_pair_rn(b23, sp_b);
        qa[4 * j + 0] = (w >> 0) & 0xF;
        qa[4 * j + 1] = (w >> 16) & 0xF;
        qa[4 * j + 2] = (w >> 8) & 0xF;
        qa[4 * j + 3] = (w >> 24) & 0xF;
        qb[4 * j + 0] = (w >> 4) & 0xF;
        qb[4 * j + 1] = (w >> 20) & 0xF;
        qb[4 * j + 2] = (w >> 12) & 0xF;
        qb[4 * j + 3] = (w >> 28) & 0xF;
    }
    const int na = nt * 16 + g, nb = na + 8;
    const size_t oa = (size_t)na * K + kbase, ob = (size_t)nb * K + kbase;
    if (out_codes) {
        uint32_t pa[4], pb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            pa[i] = qa[4 * i] | (qa[4 * i + 1] << 8) | (qa[4 * i + 2] << 16) | ((uint32_t)qa[4 * i + 3] << 24);
            pb[i] = qb[4 * i] | (qb[4 * i + 1] << 8) | (qb[4 * i + 2] << 16) | ((uint32_t)qb[4 * i + 3] << 24);
        }
        *reinterpret_cast<uint4 *>(out_codes + oa) = make_uint4(pa[0], pa[1], pa[2], pa[3]);
        *reinterpret_cast<uint4 *>(out_codes + ob) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
    }
    if (w_fp32) {
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
            float4 a, b;
            a.x = (float)((int)qa[i] - 8) * fa;
            a.y = (float)((int)qa[i + 1] - 8) * fa;
            a.z = (float)((int)qa[i + 2] - 8) * fa;
            a.w = (float)((int)qa[i + 3] - 8) * fa;
            b.x = (float)((int)qb[i] - 8) * fb;
            b.y = (float)((int)qb[i + 1] - 8) * fb;
            b.z = (float)((int)qb[i + 2] - 8) * fb;
            b.w = (float)((int)qb[i + 3] - 8) * fb;
            *reinterpret_cast<float4 *>(w_fp32 + oa + i) = a;
            *reinterpret_cast<float4 *>(w_fp32 + ob + i) = b;
        }
    }
    if (w_bf16) {
        *reinterpret_cast<uint4 *>(w_bf16 + oa) = make_uint4(ba[0], ba[1], ba[2], ba[3]);
        *reinterpret_cast<uint4 *>(w_bf16 + oa + 8) = make_uint4(ba[4], ba[5], ba[6], ba[7]);
        *reinterpret_cast<uint4 *>(w_bf16 + ob) = make_uint4(bb[0], bb[1], bb[2], bb[3]);
        *reinterpret_cast<uint4 *>(w_bf16 + ob + 8) = make_uint4(bb[4], bb[5], bb[6], bb[7]);
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

inline unsigned blocks_for(long long total, int threads)
{
    return (unsigned)((total + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_w4a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int G,
                                void *packed, cudaStream_t stream)
{
    const long long nchunks = (long long)(N / 16) * (K / 64) * 32;
    repack_codes_kernel<<<blocks_for(nchunks, 256), 256, 0, stream>>>(
        qweight, K, N, reinterpret_cast<uint4 *>(packed));
    const long long nsc = (long long)(N / 16) * (K / G) * 16;
    uint16_t *sc_out = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(packed) + (size_t)N * K / 2);
    repack_scales_kernel<<<blocks_for(nsc, 256), 256, 0, stream>>>(scales, K, N, G, sc_out);
    return cudaGetLastError();
}

cudaError_t launch_w4a16_unpack(const void *packed, int K, int N, int G, uint8_t *codes,
                                float *w_fp32, uint16_t *w_bf16, cudaStream_t stream)
{
    const long long nchunks = (long long)(N / 16) * (K / 64) * 32;
    const uint32_t *sc = reinterpret_cast<const uint32_t *>(static_cast<const uint8_t *>(packed) +
                                                            (size_t)N * K / 2);
    unpack_kernel<<<blocks_for(nchunks, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(packed), sc, K, N, G, codes, w_fp32, w_bf16);
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
