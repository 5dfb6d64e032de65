// INT4 weight-streaming GEMM whose scratch is a fixed array in device
// global memory, for callers that cannot hand the library a workspace: a
// plain C host that links only this library and owns no device allocator,
// or a serving process whose device memory has been reserved up front (by
// a cache manager that sizes its pools from the free memory at start-up),
// where a later cudaMalloc can fail or take memory the pools count on.
// This call allocates nothing: the array below is part of this file's
// module and is loaded with it.
//
// Shared-state contract (the array is one per device and per process):
//   - the 256-byte header and the arrival counters must be zero when a call
//     starts.  The first call on a device zeroes them (stream-ordered on
//     that call's stream); every call that completes leaves them zero.
//   - the partial-sum scratch keeps whatever the last call left; nothing
//     reads it before writing it.
//   - two calls on one device that are not ordered with respect to each
//     other (different streams without an event between them, or different
//     host threads) race on the counters and the scratch.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "mxg.h"

namespace mxg {
namespace {

// Header + counters (256 KiB) + partial sums.  The streaming plan keeps one
// fragment of 1 KiB per CTA and 8-row token tile; with one CTA per SM on
// 148 SMs and M <= 32 (4 token tiles) that is 592 KiB, so 2 MiB holds every
// M <= 32 shape on a B200.
constexpr size_t kStaticScratchBytes = size_t(2) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDev = 64;
std::once_flag g_setup_once[kMaxDev];
void *g_scratch[kMaxDev] = {};
cudaError_t g_setup_err[kMaxDev] = {};

bool aligned16(const void *p)
{
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Once per device, with that device current: look the array up and zero
// what must start at zero, ordered before this first call's launch.
void *scratch_for(int dev, cudaStream_t stream, cudaError_t *err)
{
    std::call_once(g_setup_once[dev], [dev, stream]() {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(p, 0, sizeof(WsHeader) + kMaxCounters * sizeof(int), stream);
        g_setup_err[dev] = e;
        g_scratch[dev] = e == cudaSuccess ? p : nullptr;
    });
    *err = g_setup_err[dev];
    return g_scratch[dev];
}

}  // namespace
}  // namespace mxg

using namespace mxg;

extern "C" int w4a16_gemm_static_scratch(const void *X, const void *packed, int M, int N, int K,
                                         int group_size, void *Y, cudaStream_t stream)
{
    if (!aligned16(X) || !aligned16(packed) || !aligned16(Y) || M < 1)
        return MXG_ERR_INVALID_ARG;
    if (K <= 0 || N <= 0 || (group_size != 32 && group_size != 64 && group_size != 128) ||
        K % 64 != 0 || K % group_size != 0 || N % 64 != 0 || M > 32)
        return MXG_ERR_UNSUPPORTED_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return MXG_ERR_CUDA;
    StreamPlan sp;
    if (!plan_w4a16_stream(dev, M, N, K, group_size, &sp))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    if (make_workspace_map(sp.ntiles, sp.partial_bytes).total > kStaticScratchBytes)
        return MXG_ERR_WORKSPACE;
    cudaError_t e = cudaSuccess;
    void *scratch = scratch_for(dev, stream, &e);
    if (!scratch)
        return MXG_ERR_CUDA;
    return launch_w4a16_stream(sp, X, packed, M, N, K, group_size, Y, scratch, stream) ==
                   cudaSuccess
               ? MXG_OK
               : MXG_ERR_CUDA;
}
