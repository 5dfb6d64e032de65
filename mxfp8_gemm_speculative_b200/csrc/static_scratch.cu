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
//     that call's stream); every call that completes without an error
//     leaves them zero.
//   - a kernel that gives up a bounded wait records MXG_ERR_TIMEOUT in the
//     header and may leave counters non-zero; w4a16_static_scratch_status
//     reads the header and, on request, zeroes the header and the counters.
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

// Header + counters (256 KiB) + partial sums.  The streaming plan keeps, per
// CTA, two fragment slots of 512 bytes per consumer warp (8) and 8-row token
// tile; with one CTA per SM on 148 SMs and M <= 32 (4 token tiles) that is
// 9.3 MiB, so 16 MiB holds every M <= 32 shape on a B200.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_setup_mutex[kMaxDev];
void *g_scratch[kMaxDev] = {};   // set once the set-up of that device succeeded

constexpr size_t kZeroedBytes = sizeof(WsHeader) + kMaxCounters * sizeof(int);

bool aligned16(const void *p)
{
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

}  // namespace

// With `dev` current: the device address of its static array, looked up and
// its header and counters zeroed on `stream` by the first successful call.
// A failed set-up is not remembered (a later call tries again); a set-up
// asked for while `stream` is being captured is refused with
// MXG_ERR_CAPTURE, since the symbol lookup may load the module.
void *static_scratch(int dev, cudaStream_t stream, int *status)
{
    *status = MXG_OK;
    if (dev < 0 || dev >= kMaxDev) {
        *status = MXG_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex[dev]);
    if (g_scratch[dev])
        return g_scratch[dev];
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        *status = MXG_ERR_CUDA;
        return nullptr;
    }
    if (cs != cudaStreamCaptureStatusNone) {
        *status = MXG_ERR_CAPTURE;
        return nullptr;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess ||
        cudaMemsetAsync(p, 0, kZeroedBytes, stream) != cudaSuccess) {
        *status = MXG_ERR_CUDA;
        return nullptr;
    }
    g_scratch[dev] = p;
    return p;
}

size_t static_scratch_bytes()
{
    return kStaticScratchBytes;
}

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
    // the one-time set-up first: inside a capture it is refused before the
    // plan touches any kernel attribute
    int st = MXG_OK;
    void *scratch = static_scratch(dev, stream, &st);
    if (!scratch)
        return st;
    StreamPlan sp;
    if (!plan_w4a16_stream(dev, M, N, K, group_size, &sp))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    if (make_workspace_map(sp.ntiles, sp.partial_bytes).total > kStaticScratchBytes)
        return MXG_ERR_WORKSPACE;
    return launch_w4a16_stream(sp, X, packed, M, N, K, group_size, Y, scratch, true, stream) ==
                   cudaSuccess
               ? MXG_OK
               : MXG_ERR_CUDA;
}

extern "C" int w4a16_static_scratch_status(int *status, int reset, cudaStream_t stream)
{
    if (!status || (reset != 0 && reset != 1))
        return MXG_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return MXG_ERR_CUDA;
    int st = MXG_OK;
    void *scratch = static_scratch(dev, stream, &st);
    if (!scratch)
        return st;
    int v = 0;
    if (cudaMemcpyAsync(&v, scratch, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MXG_ERR_CUDA;
    if (reset && cudaMemsetAsync(scratch, 0, kZeroedBytes, stream) != cudaSuccess)
        return MXG_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return MXG_ERR_CUDA;
    *status = v;
    return MXG_OK;
}
