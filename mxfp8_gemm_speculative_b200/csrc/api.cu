// C ABI of libmxg.so: argument validation, path selection, workspace layout
// and launches.  Every check happens before any launch; nothing here
// allocates device memory or synchronizes (except mxg_workspace_status,
// which is documented to).
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "mxg.h"

namespace mxg {

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_info_once[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

size_t round_up(size_t v, size_t a)
{
    return (v + a - 1) / a * a;
}

bool aligned16(const void *p)
{
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

int current_device()
{
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess)
        return -1;
    return d;
}

int to_status(cudaError_t e)
{
    return e == cudaSuccess ? MXG_OK : MXG_ERR_CUDA;
}

bool w4a16_shape_ok(int K, int N, int G)
{
    if (K <= 0 || N <= 0)
        return false;
    if (G != 32 && G != 64 && G != 128)
        return false;
    return K % 64 == 0 && K % G == 0 && N % 64 == 0;
}

bool mxfp8_shape_ok(int K, int N)
{
    return K > 0 && N >= 128 && K % 32 == 0;
}
}  // namespace

const DeviceInfo &device_info(int device)
{
    if (device < 0 || device >= kMaxDevices)
        device = 0;
    std::call_once(g_info_once[device], [device]() {
        DeviceInfo di{};
        cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, device);
        cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
        if (di.sms < 1)
            di.sms = 1;
        g_info[device] = di;
    });
    return g_info[device];
}

WorkspaceMap make_workspace_map(size_t counters, size_t partial_bytes)
{
    WorkspaceMap m{};
    m.counters_off = sizeof(WsHeader);
    m.counters = counters;
    m.partial_off = m.counters_off + kMaxCounters * sizeof(int);
    m.partial_bytes = partial_bytes;
    m.total = m.partial_off + round_up(partial_bytes, 256);
    return m;
}

bool encode_tensor_map_2d(void *map, int dtype_cu, const void *base, uint64_t inner, uint64_t outer,
                          uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                          int swizzle_cu)
{
    std::call_once(g_encode_once, []() {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode)
        return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t elem[2] = {1, 1};
    CUresult r = g_encode(reinterpret_cast<CUtensorMap *>(map),
                          static_cast<CUtensorMapDataType>(dtype_cu), 2, const_cast<void *>(base),
                          dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          static_cast<CUtensorMapSwizzle>(swizzle_cu),
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_pdl(const void *fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       void **args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// Workspace needs of the two paths for one shape (0 when the path cannot run it).
static size_t w4a16_stream_ws(int dev, int M, int N, int K, int G)
{
    StreamPlan sp;
    if (!plan_w4a16_stream(dev, M, N, K, G, &sp))
        return 0;
    return make_workspace_map(sp.ntiles, sp.partial_bytes).total;
}

static size_t w4a16_tc_ws(int dev, int M, int N, int K, int G)
{
    TcPlan tp;
    if (!plan_w4a16_tc(dev, M, N, K, G, &tp))
        return 0;
    return make_workspace_map(tp.counters, tp.partial_bytes).total;
}

static size_t mxfp8_stream_ws(int dev, int M, int N, int K)
{
    StreamPlan sp;
    if (!plan_mxfp8_stream(dev, M, N, K, &sp))
        return 0;
    return make_workspace_map(sp.ntiles, sp.partial_bytes).total;
}

static size_t mxfp8_tc_ws(int dev, int M, int N, int K)
{
    TcPlan tp;
    if (!plan_mxfp8_tc(dev, M, N, K, &tp))
        return 0;
    return make_workspace_map(tp.counters, tp.partial_bytes).total;
}

// The call's options with the defaults filled in; false for values outside
// their documented range.
static bool resolve_options(const mxg_gemm_options *o, int *path, bool *early)
{
    *path = MXG_PATH_AUTO;
    *early = true;
    if (!o)
        return true;
    if (o->path < MXG_PATH_AUTO || o->path > MXG_PATH_TENSOR)
        return false;
    if (o->late_weights != 0 && o->late_weights != 1)
        return false;
    *path = o->path;
    *early = o->late_weights == 0;
    return true;
}

// 1 = streaming, 2 = tensor cores, 0 = no path.
static int choose_path(int forced, int M, bool stream_ok, bool tc_ok)
{
    if (forced == MXG_PATH_STREAM)
        return stream_ok ? 1 : 0;
    if (forced == MXG_PATH_TENSOR)
        return tc_ok ? 2 : 0;
    if (M <= 32 && stream_ok)
        return 1;
    if (tc_ok)
        return 2;
    return stream_ok ? 1 : 0;
}

}  // namespace mxg

using namespace mxg;

extern "C" {

const char *mxg_status_string(int status)
{
    switch (status) {
    case MXG_OK: return "ok";
    case MXG_ERR_INVALID_ARG: return "invalid argument (NULL or misaligned pointer, or bad size)";
    case MXG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or group size";
    case MXG_ERR_WORKSPACE: return "workspace too small";
    case MXG_ERR_CUDA: return "CUDA runtime or launch error";
    case MXG_ERR_TIMEOUT: return "a bounded in-kernel wait timed out";
    case MXG_ERR_CAPTURE:
        return "a call that needs its one-time device set-up was made during stream capture";
    default: return "unknown status";
    }
}

size_t w4a16_packed_bytes(int K, int N, int group_size)
{
    if (!w4a16_shape_ok(K, N, group_size))
        return 0;
    return (size_t)N * K / 2 + (size_t)N * (K / group_size) * 2;
}

int w4a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int group_size,
                 void *packed, cudaStream_t stream)
{
    if (!aligned16(qweight) || !aligned16(scales) || !aligned16(packed))
        return MXG_ERR_INVALID_ARG;
    if (!w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(launch_w4a16_repack(qweight, scales, K, N, group_size, false, packed, stream));
}

int w4a16_repack_fused(int count, const int32_t *const *qweights, const uint16_t *const *scales,
                       const int *Ns, int K, int group_size, void *packed, cudaStream_t stream)
{
    if (count < 1 || count > 64 || !qweights || !scales || !Ns || !aligned16(packed))
        return MXG_ERR_INVALID_ARG;
    long long N = 0;
    for (int i = 0; i < count; ++i) {
        if (!aligned16(qweights[i]) || !aligned16(scales[i]))
            return MXG_ERR_INVALID_ARG;
        if (!w4a16_shape_ok(K, Ns[i], group_size))
            return MXG_ERR_UNSUPPORTED_SHAPE;
        N += Ns[i];
    }
    if (N > (1LL << 30))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    int n0 = 0;
    for (int i = 0; i < count; ++i) {
        const cudaError_t e = launch_w4a16_repack_part(qweights[i], scales[i], K, Ns[i], group_size,
                                                       n0, (int)N, packed, stream);
        if (e != cudaSuccess)
            return to_status(e);
        n0 += Ns[i];
    }
    return to_status(launch_repack_done(stream));
}

int w4a16_repack_ct(const int32_t *weight_packed, const uint16_t *weight_scale, int K, int N,
                    int group_size, void *packed, cudaStream_t stream)
{
    if (!aligned16(weight_packed) || !aligned16(weight_scale) || !aligned16(packed))
        return MXG_ERR_INVALID_ARG;
    if (!w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(
        launch_w4a16_repack(weight_packed, weight_scale, K, N, group_size, true, packed, stream));
}

size_t w4a16_workspace_bytes(int M, int N, int K, int group_size)
{
    if (M < 1 || !w4a16_shape_ok(K, N, group_size))
        return 0;
    const int dev = current_device();
    if (dev < 0)
        return 0;
    size_t a = w4a16_stream_ws(dev, M, N, K, group_size);
    size_t b = w4a16_tc_ws(dev, M, N, K, group_size);
    size_t r = a > b ? a : b;
    return r ? r : sizeof(WsHeader);
}

int w4a16_gemm_ex(const void *X, const void *packed, int M, int N, int K, int group_size, void *Y,
                  void *workspace, size_t workspace_bytes, const mxg_gemm_options *opts,
                  cudaStream_t stream)
{
    int forced = 0;
    bool early = true;
    if (!resolve_options(opts, &forced, &early))
        return MXG_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(Y) || !aligned16(workspace) || M < 1)
        return MXG_ERR_INVALID_ARG;
    if (!w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    const int dev = current_device();
    if (dev < 0)
        return MXG_ERR_CUDA;
    StreamPlan sp;
    TcPlan tp;
    const bool s_ok = plan_w4a16_stream(dev, M, N, K, group_size, &sp);
    // the tensor-core plan only matters when the streaming path is not taken
    const bool t_ok = (M <= 32 && s_ok && forced != MXG_PATH_TENSOR)
                          ? false
                          : plan_w4a16_tc(dev, M, N, K, group_size, &tp);
    const int path = choose_path(forced, M, s_ok, t_ok);
    if (path == 1) {
        if (workspace_bytes < make_workspace_map(sp.ntiles, sp.partial_bytes).total)
            return MXG_ERR_WORKSPACE;
        return to_status(
            launch_w4a16_stream(sp, X, packed, M, N, K, group_size, Y, workspace, early, stream));
    }
    if (path == 2) {
        if (workspace_bytes < make_workspace_map(tp.counters, tp.partial_bytes).total)
            return MXG_ERR_WORKSPACE;
        return to_status(
            launch_w4a16_tc(tp, X, packed, M, N, K, group_size, Y, workspace, early, stream));
    }
    return MXG_ERR_UNSUPPORTED_SHAPE;
}

int w4a16_gemm(const void *X, const void *packed, int M, int N, int K, int group_size, void *Y,
               void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    return w4a16_gemm_ex(X, packed, M, N, K, group_size, Y, workspace, workspace_bytes, nullptr,
                         stream);
}

size_t w8a16_packed_bytes(int K, int N, int group_size)
{
    if (!w4a16_shape_ok(K, N, group_size))
        return 0;
    return (size_t)N * K + (size_t)N * (K / group_size) * 2;
}

int w8a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int group_size,
                 void *packed, cudaStream_t stream)
{
    if (!aligned16(qweight) || !aligned16(scales) || !aligned16(packed))
        return MXG_ERR_INVALID_ARG;
    if (!w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(launch_w8a16_repack(qweight, scales, K, N, group_size, false, packed, stream));
}

int w8a16_repack_ct(const int32_t *weight_packed, const uint16_t *weight_scale, int K, int N,
                    int group_size, void *packed, cudaStream_t stream)
{
    if (!aligned16(weight_packed) || !aligned16(weight_scale) || !aligned16(packed))
        return MXG_ERR_INVALID_ARG;
    if (!w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(
        launch_w8a16_repack(weight_packed, weight_scale, K, N, group_size, true, packed, stream));
}

size_t w8a16_workspace_bytes(int M, int N, int K, int group_size)
{
    if (M < 1 || M > 32 || !w4a16_shape_ok(K, N, group_size))
        return 0;
    const int dev = current_device();
    if (dev < 0)
        return 0;
    StreamPlan sp;
    if (!plan_w8a16_stream(dev, M, N, K, group_size, &sp))
        return 0;
    return make_workspace_map(sp.ntiles, sp.partial_bytes).total;
}

int w8a16_gemm_ex(const void *X, const void *packed, int M, int N, int K, int group_size, void *Y,
                  void *workspace, size_t workspace_bytes, const mxg_gemm_options *opts,
                  cudaStream_t stream)
{
    int forced = 0;
    bool early = true;
    if (!resolve_options(opts, &forced, &early) || forced == MXG_PATH_TENSOR)
        return MXG_ERR_INVALID_ARG;   // INT8 has the weight-streaming path only
    if (!aligned16(X) || !aligned16(packed) || !aligned16(Y) || !aligned16(workspace) || M < 1)
        return MXG_ERR_INVALID_ARG;
    if (M > 32 || !w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    const int dev = current_device();
    if (dev < 0)
        return MXG_ERR_CUDA;
    StreamPlan sp;
    if (!plan_w8a16_stream(dev, M, N, K, group_size, &sp))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    if (workspace_bytes < make_workspace_map(sp.ntiles, sp.partial_bytes).total)
        return MXG_ERR_WORKSPACE;
    return to_status(
        launch_w4a16_stream(sp, X, packed, M, N, K, group_size, Y, workspace, early, stream));
}

int w8a16_gemm(const void *X, const void *packed, int M, int N, int K, int group_size, void *Y,
               void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    return w8a16_gemm_ex(X, packed, M, N, K, group_size, Y, workspace, workspace_bytes, nullptr,
                         stream);
}

size_t mxfp8_workspace_bytes(int M, int N, int K)
{
    if (M < 1 || !mxfp8_shape_ok(K, N))
        return 0;
    const int dev = current_device();
    if (dev < 0)
        return 0;
    size_t a = mxfp8_stream_ws(dev, M, N, K);
    size_t b = mxfp8_tc_ws(dev, M, N, K);
    size_t r = a > b ? a : b;
    return r ? r : sizeof(WsHeader);
}

int mxfp8_gemm_ex(const void *X, const uint8_t *Wq, const uint8_t *Ws, int M, int N, int K,
                  void *Y, void *workspace, size_t workspace_bytes, const mxg_gemm_options *opts,
                  cudaStream_t stream)
{
    int forced = 0;
    bool early = true;
    if (!resolve_options(opts, &forced, &early))
        return MXG_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(Y) ||
        !aligned16(workspace) || M < 1)
        return MXG_ERR_INVALID_ARG;
    if (!mxfp8_shape_ok(K, N))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    const int dev = current_device();
    if (dev < 0)
        return MXG_ERR_CUDA;
    StreamPlan sp;
    TcPlan tp;
    const bool s_ok = plan_mxfp8_stream(dev, M, N, K, &sp);
    const bool t_ok = (M <= 32 && s_ok && forced != MXG_PATH_TENSOR)
                          ? false
                          : plan_mxfp8_tc(dev, M, N, K, &tp);
    const int path = choose_path(forced, M, s_ok, t_ok);
    if (path == 1) {
        if (workspace_bytes < make_workspace_map(sp.ntiles, sp.partial_bytes).total)
            return MXG_ERR_WORKSPACE;
        return to_status(
            launch_mxfp8_stream(sp, X, Wq, Ws, M, N, K, Y, workspace, early, stream));
    }
    if (path == 2) {
        if (workspace_bytes < make_workspace_map(tp.counters, tp.partial_bytes).total)
            return MXG_ERR_WORKSPACE;
        return to_status(launch_mxfp8_tc(tp, X, Wq, Ws, M, N, K, Y, workspace, early, stream));
    }
    return MXG_ERR_UNSUPPORTED_SHAPE;
}

int mxfp8_gemm(const void *X, const uint8_t *Wq, const uint8_t *Ws, int M, int N, int K, void *Y,
               void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    return mxfp8_gemm_ex(X, Wq, Ws, M, N, K, Y, workspace, workspace_bytes, nullptr, stream);
}

namespace {
bool mxfp8_packed_shape_ok(int K, int N)
{
    return K > 0 && N > 0 && K % 64 == 0 && N % 64 == 0;
}
}  // namespace

size_t mxfp8_packed_bytes(int N, int K)
{
    if (!mxfp8_packed_shape_ok(K, N))
        return 0;
    return (size_t)N * K + (size_t)N * (K / 32);
}

int mxfp8_repack(const uint8_t *Wq, const uint8_t *Ws, int N, int K, void *packed,
                 cudaStream_t stream)
{
    if (!aligned16(Wq) || !aligned16(Ws) || !aligned16(packed))
        return MXG_ERR_INVALID_ARG;
    if (!mxfp8_packed_shape_ok(K, N))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(launch_mxfp8_repack(Wq, Ws, N, K, packed, stream));
}

size_t mxfp8_packed_workspace_bytes(int M, int N, int K)
{
    if (M < 1 || M > 16 || !mxfp8_packed_shape_ok(K, N))
        return 0;
    const int dev = current_device();
    if (dev < 0)
        return 0;
    StreamPlan sp;
    if (!plan_mxfp8_packed_stream(dev, M, N, K, &sp))
        return 0;
    return make_workspace_map(sp.ntiles, sp.partial_bytes).total;
}

int mxfp8_gemm_packed_ex(const void *X, const void *packed, int M, int N, int K, void *Y,
                         void *workspace, size_t workspace_bytes, const mxg_gemm_options *opts,
                         cudaStream_t stream)
{
    int forced = 0;
    bool early = true;
    if (!resolve_options(opts, &forced, &early) || forced == MXG_PATH_TENSOR)
        return MXG_ERR_INVALID_ARG;   // the re-packed layout has the weight-streaming path only
    if (!aligned16(X) || !aligned16(packed) || !aligned16(Y) || !aligned16(workspace) || M < 1)
        return MXG_ERR_INVALID_ARG;
    if (M > 16 || !mxfp8_packed_shape_ok(K, N))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    const int dev = current_device();
    if (dev < 0)
        return MXG_ERR_CUDA;
    StreamPlan sp;
    if (!plan_mxfp8_packed_stream(dev, M, N, K, &sp))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    if (workspace_bytes < make_workspace_map(sp.ntiles, sp.partial_bytes).total)
        return MXG_ERR_WORKSPACE;
    return to_status(launch_w4a16_stream(sp, X, packed, M, N, K, 64, Y, workspace, early, stream));
}

int mxfp8_gemm_packed(const void *X, const void *packed, int M, int N, int K, void *Y,
                      void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    return mxfp8_gemm_packed_ex(X, packed, M, N, K, Y, workspace, workspace_bytes, nullptr, stream);
}

int w4a16_unpack(const void *packed, int K, int N, int group_size, uint8_t *codes, float *w_fp32,
                 uint16_t *w_bf16, cudaStream_t stream)
{
    if (!aligned16(packed) || !aligned16(codes))
        return MXG_ERR_INVALID_ARG;
    if ((w_fp32 && !aligned16(w_fp32)) || (w_bf16 && !aligned16(w_bf16)))
        return MXG_ERR_INVALID_ARG;
    if (!w4a16_shape_ok(K, N, group_size))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(launch_w4a16_unpack(packed, K, N, group_size, codes, w_fp32, w_bf16, stream));
}

int mxfp8_dequant(const uint8_t *Wq, const uint8_t *Ws, int N, int K, uint16_t *w_bf16,
                  cudaStream_t stream)
{
    if (!aligned16(Wq) || !aligned16(Ws) || !aligned16(w_bf16))
        return MXG_ERR_INVALID_ARG;
    if (!mxfp8_shape_ok(K, N))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    return to_status(launch_mxfp8_dequant(Wq, Ws, N, K, w_bf16, stream));
}

int mxg_workspace_status(const void *workspace, int *status, cudaStream_t stream)
{
    if (!aligned16(workspace) || !status)
        return MXG_ERR_INVALID_ARG;
    int v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MXG_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return MXG_ERR_CUDA;
    *status = v;
    return MXG_OK;
}

int mxg_selftest_wait_timeout(void *workspace, int limit_us, cudaStream_t stream)
{
    if ((workspace && !aligned16(workspace)) || limit_us < 1 || limit_us > 10000000)
        return MXG_ERR_INVALID_ARG;
    if (!workspace) {
        // the static scratch array of w4a16_gemm_static_scratch on this device
        const int dev = current_device();
        if (dev < 0)
            return MXG_ERR_CUDA;
        int st = MXG_OK;
        workspace = static_scratch(dev, stream, &st);
        if (!workspace)
            return st;
    }
    return to_status(launch_wait_timeout_selftest(workspace, limit_us, stream));
}

size_t bf16_gemm_small_workspace_bytes(int M, int N, int K)
{
    SmallPlan sp;
    if (!plan_bf16_small(M, N, K, &sp))
        return 0;
    return make_workspace_map(1, sp.partial_bytes).total;
}

int bf16_gemm_small_ex(const void *X, const void *W, int M, int N, int K, void *Y, void *workspace,
                       size_t workspace_bytes, const mxg_gemm_options *opts, cudaStream_t stream)
{
    int forced = 0;
    bool early = true;
    if (!resolve_options(opts, &forced, &early) || forced != MXG_PATH_AUTO)
        return MXG_ERR_INVALID_ARG;   // one kernel: no path to choose
    if (!aligned16(X) || !aligned16(W) || !aligned16(Y) || !aligned16(workspace) || M < 1)
        return MXG_ERR_INVALID_ARG;
    SmallPlan sp;
    if (!plan_bf16_small(M, N, K, &sp))
        return MXG_ERR_UNSUPPORTED_SHAPE;
    if (workspace_bytes < make_workspace_map(1, sp.partial_bytes).total)
        return MXG_ERR_WORKSPACE;
    return to_status(launch_bf16_small(sp, X, W, M, N, K, Y, workspace, early, stream));
}

int bf16_gemm_small(const void *X, const void *W, int M, int N, int K, void *Y, void *workspace,
                    size_t workspace_bytes, cudaStream_t stream)
{
    return bf16_gemm_small_ex(X, W, M, N, K, Y, workspace, workspace_bytes, nullptr, stream);
}

}  // extern "C"
