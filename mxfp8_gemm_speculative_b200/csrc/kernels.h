// Internal launch interface of the mxg kernels (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace mxg {

// ------------------------------------------------------------ device facts
struct DeviceInfo {
    int sms;              // streaming multiprocessors
    int smem_optin;       // max dynamic shared memory per block (bytes)
};
const DeviceInfo &device_info(int device);

// ------------------------------------------------------------ workspace map
// [0, 256)                   header (status word)
// [256, 256 + 4*kMaxCounters) arrival counters, at the same place for every
//                            shape, so one zero-initialised workspace serves
//                            calls of any shape (each call leaves them zero)
// [then ...)                 fp32 partial sums (scratch)
constexpr size_t kMaxCounters = 65536;
// Devices for which per-device launch state (function attributes, occupancy)
// is cached.
constexpr int kMaxDeviceCache = 64;

struct WorkspaceMap {
    size_t counters_off;
    size_t counters;      // number of int counters
    size_t partial_off;
    size_t partial_bytes;
    size_t total;
};
WorkspaceMap make_workspace_map(size_t counters, size_t partial_bytes);

// ------------------------------------------------------ weight-streaming path
// Stream-K plan: the layer's weight bytes are cut into equal "units" (one
// 256-column group x 128 rows of K for INT4 and INT8, one n16 tile x 128 k
// for MXFP8) and every CTA (INT4) or warp (MXFP8) of a persistent grid takes
// one contiguous run of units.
struct StreamPlan {
    int tt;               // token tiles of 8 rows (ceil(M / 8)), 1..4
    int variant;          // kernel variant
    int warps_per_cta;
    int grid;             // CTAs
    int Wt;               // runs: CTAs (INT4) or warps (MXFP8), <= units
    long long units;      // total units
    int upt;              // units per output tile (INT4: per group row)
    size_t smem;          // dynamic shared memory per CTA
    size_t partial_bytes; // workspace for partial sums
    int ntiles;           // arrival counters
    // INT4 / INT8: pieces per group row (0: stream-K runs across rows);
    // shared-memory plan: ring stages and region offsets
    int split;
    int ring;
    int x_off, xs_off, xchg_off, bar_off;
};

bool plan_w4a16_stream(int device, int M, int N, int K, int G, StreamPlan *plan);
// INT8 W8A16 (two code planes) on the same kernel; launch_w4a16_stream runs
// either plan.
bool plan_w8a16_stream(int device, int M, int N, int K, int G, StreamPlan *plan);
// Re-packed MXFP8 (mxfp8_repack) on the same kernel, M <= 16; launch with
// launch_w4a16_stream and G = 64.
bool plan_mxfp8_packed_stream(int device, int M, int N, int K, StreamPlan *plan);
// early: load the first weights before waiting for the previous kernel on
// the stream (every launch function below takes it per call).
cudaError_t launch_w4a16_stream(const StreamPlan &plan, const void *X, const void *packed, int M,
                                int N, int K, int G, void *Y, void *workspace, bool early,
                                cudaStream_t stream);

bool plan_mxfp8_stream(int device, int M, int N, int K, StreamPlan *plan);
cudaError_t launch_mxfp8_stream(const StreamPlan &plan, const void *X, const uint8_t *Wq,
                                const uint8_t *Ws, int M, int N, int K, void *Y, void *workspace,
                                bool early, cudaStream_t stream);

// ----------------------------------------------------- tensor-core path
struct TcPlan {
    int bm, bn, bk;       // CTA tile
    int mtiles, ntiles;   // output tiles
    int splits;           // K splits (1 = none)
    int grid;             // CTAs (persistent)
    size_t smem;
    size_t partial_bytes; // split-K partial sums
    size_t counters;      // split-K arrival counters
};
bool plan_w4a16_tc(int device, int M, int N, int K, int G, TcPlan *plan);
cudaError_t launch_w4a16_tc(const TcPlan &plan, const void *X, const void *packed, int M, int N,
                            int K, int G, void *Y, void *workspace, bool early,
                            cudaStream_t stream);
bool plan_mxfp8_tc(int device, int M, int N, int K, TcPlan *plan);
cudaError_t launch_mxfp8_tc(const TcPlan &plan, const void *X, const uint8_t *Wq,
                            const uint8_t *Ws, int M, int N, int K, void *Y, void *workspace,
                            bool early, cudaStream_t stream);

// ------------------------------------------ dense bf16, few output columns
// Split-K plan: K in 64-wide chunks over `ctas` CTAs of N/16 warps each.
struct SmallPlan {
    int chunks;
    int ctas;
    int threads;
    size_t partial_bytes;
};
bool plan_bf16_small(int M, int N, int K, SmallPlan *plan);
cudaError_t launch_bf16_small(const SmallPlan &plan, const void *X, const void *W, int M, int N,
                              int K, void *Y, void *workspace, bool early, cudaStream_t stream);

// ------------------------------------------------------------ weight tools
// n_major: compressed-tensors inputs ([N][K/8] words, [N][K/G] scales)
// instead of GPTQ's ([K/8][N], [K/G][N]).
cudaError_t launch_w4a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int G,
                                bool n_major, void *packed, cudaStream_t stream);
// Columns [n0, n0 + Np) of a fused buffer of N columns from GPTQ inputs of
// Np columns (no completion kernel; launch_repack_done ends the re-pack).
cudaError_t launch_w4a16_repack_part(const int32_t *qweight, const uint16_t *scales, int K, int Np,
                                     int G, int n0, int N, void *packed, cudaStream_t stream);
cudaError_t launch_repack_done(cudaStream_t stream);
// INT8 W8A16: GPTQ-style words [K/4][N] with 8-bit codes into two INT4-layout
// code planes ([N/32][K/64][2][2 planes][32][16 B], N*K bytes), then scales.
// n_major: compressed-tensors inputs ([N][K/4] words, [N][K/G] scales).
cudaError_t launch_w8a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N, int G,
                                bool n_major, void *packed, cudaStream_t stream);
cudaError_t launch_w4a16_unpack(const void *packed, int K, int N, int G, uint8_t *codes,
                                float *w_fp32, uint16_t *w_bf16, cudaStream_t stream);
cudaError_t launch_mxfp8_repack(const uint8_t *Wq, const uint8_t *Ws, int N, int K, void *packed,
                               cudaStream_t stream);
cudaError_t launch_mxfp8_dequant(const uint8_t *Wq, const uint8_t *Ws, int N, int K,
                                 uint16_t *w_bf16, cudaStream_t stream);
cudaError_t launch_wait_timeout_selftest(void *workspace, int limit_us, cudaStream_t stream);

// The static scratch array of w4a16_gemm_static_scratch on device `dev`
// (current), set up on `stream` by the first successful call; NULL with
// *status set (MXG_ERR_CAPTURE while `stream` is captured before that
// set-up, MXG_ERR_CUDA otherwise).
void *static_scratch(int dev, cudaStream_t stream, int *status);
size_t static_scratch_bytes();

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream drains (it calls griddepcontrol.wait
// before touching anything that kernel could have written).
cudaError_t launch_pdl(const void *fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       void **args);

// Encodes tensor maps through the driver entry point (no libcuda link).
bool encode_tensor_map_2d(void *map, int dtype_cu, const void *base, uint64_t inner,
                          uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                          uint32_t box_outer, int swizzle_cu);

}  // namespace mxg
