// Dense bf16 projection with few output columns at decode token counts:
// Y[M][N] = X[M][K] * W[N][K]^T, M <= 8, N <= 256.  The case it is built for
// is the paired GDN A/B projection of the "Qwen3.8-27B and native MTP
// speculative decoding" recipe (section "Pack inference projections": two
// dense bf16 projections of 48 x 5120 computed together for single-token
// decoding and four-token verification), i.e. N = 96, K = 5120, M = 1 or 4.
//
// The layer is ~1 MB of weights, so it is bound by latency, not bandwidth:
// every global round trip after the wait for the previous kernel counts.
// One CTA per 8 rows of W and 16 warps that split K: each warp loads its
// share of the weights straight into MMA fragments (before that wait, like
// the other weight-streaming kernels; the m16 MMA's rows 8..15 are zero),
// then all of its activations at once, runs its MMAs, and the CTA adds the
// warps' fragments in shared memory in warp order (bitwise reproducible).
// No cross-CTA reduction, no atomics.
//
// k order inside a 64-wide chunk: lane t of a warp covers the 16 consecutive
// k 64q + 16t .. 64q + 16t + 15 (two 16-byte loads per row); MMA step j
// takes k = 64q + 16t + 4j .. + 3 into the lane's k slots (2t, 2t+1, 2t+8,
// 2t+9), for the weights and the activations alike, so every k of the chunk
// meets its activation exactly once.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace mxg {
namespace {

constexpr int kChunkK = 64;
constexpr int kRows = 8;          // rows of W per CTA
constexpr int kWarps = 16;        // warps per CTA, splitting K
constexpr int kHold = 5;          // chunks per warp held in registers at once

struct SmallParams {
    const uint16_t *X;   // bf16 [M][K]
    const uint16_t *W;   // bf16 [N][K]
    uint16_t *Y;         // bf16 [M][N]
    int M, N, K;
    int chunks;          // K / 64
    int early;           // load the weights before waiting for the previous kernel
};

__global__ void __launch_bounds__(kWarps * 32, 1) bf16_small_kernel(const SmallParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    __shared__ float2 red[kWarps][32];
    pdl_launch_dependents();
    const int row0 = blockIdx.x * kRows;
    // this warp's chunks [q0, q1), taken kHold at a time
    const int q0 = (int)((long long)warp * p.chunks / kWarps);
    const int q1 = (int)((long long)(warp + 1) * p.chunks / kWarps);
    const uint16_t *wr = p.W + (size_t)(row0 + g) * p.K + 16 * t;  // row g of the CTA's rows
    // activations of token g (rows >= M read row 0; their outputs are not stored)
    const uint16_t *xr = p.X + (size_t)(g < p.M ? g : 0) * p.K + 16 * t;
    uint4 A[kHold][2];
    auto load_w = [&](int q, int nq) {
#pragma unroll
        for (int i = 0; i < kHold; ++i)
            if (i < nq) {
                A[i][0] = ldg128(wr + (size_t)(q + i) * kChunkK);
                A[i][1] = ldg128(wr + (size_t)(q + i) * kChunkK + 8);
            }
    };
    // The weights are not written by the previous kernel on the stream (the
    // caller's contract, unless it turned early weight loads off).
    int nq = min(kHold, q1 - q0);
    if (p.early)
        load_w(q0, nq);
    pdl_wait();
    if (!p.early)
        load_w(q0, nq);

    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int q = q0; q < q1;) {
        uint4 x[kHold][2];
#pragma unroll
        for (int i = 0; i < kHold; ++i)
            if (i < nq) {
                x[i][0] = ldg128(xr + (size_t)(q + i) * kChunkK);
                x[i][1] = ldg128(xr + (size_t)(q + i) * kChunkK + 8);
            }
#pragma unroll
        for (int i = 0; i < kHold; ++i)
            if (i < nq) {
                const uint4 a0 = A[i][0], a1 = A[i][1];
                // step j: slots (2t, 2t+1) <- k 4j, 4j+1 and (2t+8, 2t+9) <- k 4j+2, 4j+3;
                // rows 8..15 of the MMA are zero
                mma_bf16_16816(d, a0.x, 0u, a0.y, 0u, x[i][0].x, x[i][0].y);
                mma_bf16_16816(d, a0.z, 0u, a0.w, 0u, x[i][0].z, x[i][0].w);
                mma_bf16_16816(d, a1.x, 0u, a1.y, 0u, x[i][1].x, x[i][1].y);
                mma_bf16_16816(d, a1.z, 0u, a1.w, 0u, x[i][1].z, x[i][1].w);
            }
        q += nq;
        nq = min(kHold, q1 - q);
        if (nq > 0)
            load_w(q, nq);
    }

    // the warps' fragments (row g, tokens 2t and 2t + 1), added in warp order
    red[warp][lane] = make_float2(d[0], d[1]);
    __syncthreads();
    if (warp != 0)
        return;
    float2 s = red[0][lane];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        const float2 v = red[w][lane];
        s.x += v.x;
        s.y += v.y;
    }
    const int n = row0 + g;
    if (2 * t < p.M)
        p.Y[(size_t)(2 * t) * p.N + n] = f32_to_bf16_bits(s.x);
    if (2 * t + 1 < p.M)
        p.Y[(size_t)(2 * t + 1) * p.N + n] = f32_to_bf16_bits(s.y);
}

}  // namespace

bool plan_bf16_small(int M, int N, int K, SmallPlan *plan)
{
    if (M < 1 || M > 8 || N < 16 || N > 2048 || N % 16 != 0 || K < kChunkK || K % kChunkK != 0)
        return false;
    SmallPlan pl{};
    pl.chunks = K / kChunkK;
    pl.ctas = N / kRows;
    pl.threads = kWarps * 32;
    pl.partial_bytes = 0;
    *plan = pl;
    return true;
}

cudaError_t launch_bf16_small(const SmallPlan &pl, const void *X, const void *W, int M, int N, int K,
                              void *Y, void *workspace, bool early, cudaStream_t stream)
{
    (void)workspace;
    SmallParams p{};
    p.X = static_cast<const uint16_t *>(X);
    p.W = static_cast<const uint16_t *>(W);
    p.Y = static_cast<uint16_t *>(Y);
    p.M = M;
    p.N = N;
    p.K = K;
    p.chunks = pl.chunks;
    p.early = early ? 1 : 0;
    void *args[] = {&p};
    return launch_pdl(reinterpret_cast<const void *>(&bf16_small_kernel), dim3(pl.ctas),
                      dim3(pl.threads), 0, stream, args);
}

}  // namespace mxg
