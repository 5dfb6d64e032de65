/*
 * mxg — weight-quantized linear layer for speculative-decoding verify chunks,
 * B200 (sm_100a).  C ABI of libmxg.so.
 *
 *     Y[M][N] = X[M][K] * dequant(W)^T      bf16 in, fp32 accumulate, bf16 out
 *
 * Two weight formats:
 *
 *  INT4 W4A16 (GPTQ, symmetric, group G along K).  Defined by the
 *  "Qwen3.8-27B GPTQ-Int4-sym-G128" model card, section "Quantization
 *  contract" (GPTQ INT4, symmetric, group size 128, desc_act=false, packed
 *  int32) and the Eole Qwen3.8 recipe, section "Compressed-tensors INT4
 *  layout" (symmetric grouped W4A16; group size 32, 64 or 128; asymmetric,
 *  act-order and sparse exports rejected) and "INT4 tensor parallelism"
 *  (packed weights are partitioned, then re-packed once for the kernel).
 *  Codes q in 0..15, eight per int32 word along K: the code of row k = 8i + j
 *  is bits [4j, 4j+3] of word (i, n) of qweight[K/8][N].  Weight
 *  w[n][k] = (q - 8) * scale[k / G][n], scales fp16.
 *
 *  MXFP8 (OCP Microscaling).  Defined by the "Qwen3.8-27B-MXFP8 AutoRound"
 *  model card: header (8-bit block FP with E8M0 group scales), section 2
 *  (kernel constraints N >= 128 and K % 32 == 0) and section 8 (OCP MX
 *  specification, one E8M0 shared scale per 32-element block).  Codes are
 *  OCP E4M3 ("fn": bias 7, no infinities, S.1111.111 is NaN) in Wq[N][K]
 *  (K contiguous), exponents E8M0 in Ws[N][K/32]; w = e4m3 * 2^(E - 127).
 *
 * Conventions for every entry point:
 *  - All buffers are owned and allocated by the caller, in device memory of
 *    the current CUDA device unless stated.  The library never allocates,
 *    frees or synchronizes; every call is asynchronous and stream-ordered
 *    on `stream` (0 = legacy default stream).
 *  - Pointers must be non-NULL and 16-byte aligned.  Y must not alias any
 *    input or the workspace.
 *  - Errors are reported before any launch as a negative mxg_status; a
 *    launch failure maps to MXG_ERR_CUDA.  A pipeline wait inside a kernel
 *    that exceeds its time limit records MXG_ERR_TIMEOUT in the workspace
 *    status word (read it with mxg_workspace_status) and the kernel returns.
 *  - The GPU path does not scan inputs: NaN E4M3 codes (0x7F / 0xFF), E8M0
 *    0xFF and non-finite scales give unspecified output.
 *  - GEMM kernels are launched with programmatic dependent launch: they may
 *    start while the previous kernel on `stream` drains, and wait for it
 *    before they read X or touch Y and the workspace.  By default they also
 *    start loading WEIGHTS (packed, Wq, Ws, W) before that wait: the weight
 *    buffers must then not be written by the kernel immediately before the
 *    GEMM on `stream`.  w4a16_repack ends with a kernel that writes nothing,
 *    so a GEMM may follow it directly; any other writer of weights needs
 *    another launch, or a synchronization, between it and the GEMM (in
 *    serving, weights are written once at load time), or the call's
 *    late_weights option (the *_ex entry points).
 *  - No entry point keeps settings between calls: every choice a caller can
 *    make is an argument of the call (mxg_gemm_options).  The only global
 *    state is a per-device cache of device attributes and kernel launch
 *    attributes, and the scratch array of w4a16_gemm_static_scratch.
 */
#ifndef MXG_H
#define MXG_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MXG_API __attribute__((visibility("default")))
#else
#define MXG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXG_OK = 0,
    MXG_ERR_INVALID_ARG = -1,        /* NULL or misaligned pointer, M < 1, ... */
    MXG_ERR_UNSUPPORTED_SHAPE = -2,  /* a size the format or the kernels reject */
    MXG_ERR_WORKSPACE = -3,          /* workspace smaller than the size query */
    MXG_ERR_CUDA = -4,               /* a CUDA runtime or launch error */
    MXG_ERR_TIMEOUT = -5,            /* a bounded in-kernel wait ran out */
    MXG_ERR_CAPTURE = -6             /* a one-time device set-up was asked for inside a
                                        stream capture (make that first call outside it) */
} mxg_status;

/* Per-call options of the *_ex GEMM entry points.  NULL, or a struct whose
 * fields are all zero, gives the behaviour of the plain entry points.
 *   path          MXG_PATH_AUTO: M <= 32 streams the weights, larger M runs on
 *                 the tensor cores; MXG_PATH_STREAM / MXG_PATH_TENSOR force
 *                 one path (the streaming path takes M <= 32 only; a shape
 *                 the forced path cannot run returns
 *                 MXG_ERR_UNSUPPORTED_SHAPE).
 *   late_weights  0: the kernels may load weights before waiting for the
 *                 previous kernel on the stream (see the conventions above);
 *                 1: only after that wait, for a caller whose previous kernel
 *                 on the stream writes these weights.
 * A value outside these returns MXG_ERR_INVALID_ARG before any launch. */
enum { MXG_PATH_AUTO = 0, MXG_PATH_STREAM = 1, MXG_PATH_TENSOR = 2 };
typedef struct mxg_gemm_options {
    int path;
    int late_weights;
} mxg_gemm_options;

/* Short English text for a status code (static storage, never NULL). */
MXG_API const char *mxg_status_string(int status);

/* ------------------------------------------------------------------ INT4 */

/* Bytes of the re-packed weight buffer for a K x N layer with group size G:
 * N*K/2 code bytes followed by 2*N*K/G scale bytes (no padding).  Returns 0
 * for a shape w4a16_repack rejects. */
MXG_API size_t w4a16_packed_bytes(int K, int N, int group_size);

/* Offline re-pack (once per weight, after any fusion or sharding).
 *   qweight  device, int32 [K/8][N], GPTQ words as described above.
 *   scales   device, fp16 bits [K/G][N].
 *   packed   device, caller-allocated, w4a16_packed_bytes(K, N, G) bytes.
 * Layout written (private to this library, stable for a given K, N, G), by
 * column groups of 256 columns (eight n32 tiles; the last group holds the
 * remaining tiles when N % 256 != 0): codes as [N/256 groups][K/64][tiles of
 * the group][2 halves][32 lanes][16 B] (one 16-byte load is one lane's MMA
 * fragment for four k16 steps of two weight columns; the codes of a group
 * for any run of k64 chunks are contiguous), then scales as [N/256 groups]
 * [K/G][tiles of the group][8][4].
 * Requirements: G in {32, 64, 128}; K % 64 == 0; K % G == 0; N % 64 == 0.
 * Otherwise MXG_ERR_UNSUPPORTED_SHAPE. */
MXG_API int w4a16_repack(const int32_t *qweight, const uint16_t *scales,
                 int K, int N, int group_size, void *packed, cudaStream_t stream);

/* The same re-pack from the compressed-tensors export of the same weights
 * (the Eole recipe, section "Compressed-tensors INT4 layout": symmetric
 * grouped W4A16 "pack-quantized" weights, which its converter only
 * transposes into the GPTQ layout, without re-quantizing).
 *   weight_packed  device, int32 [N][K/8]: word (n, i) holds the codes of
 *                  rows k = 8i + j, j = 0..7, in bits [4j, 4j+3] (LSB first),
 *                  the same code values as GPTQ (w = (q - 8) * scale).
 *   weight_scale   device, fp16 bits [N][K/G].
 *   packed         as for w4a16_repack; the bytes written are identical to
 *                  w4a16_repack of the transposed words and scales.
 * Requirements and errors as for w4a16_repack. */
MXG_API int w4a16_repack_ct(const int32_t *weight_packed, const uint16_t *weight_scale,
                 int K, int N, int group_size, void *packed, cudaStream_t stream);

/* Fused projections (the Eole recipe, section "Pack inference projections":
 * K/V/Q and gate/up projections that share their input are packed into one
 * projection before the kernel re-pack, to cut launches per step).  Re-packs
 * `count` GPTQ weights with the same K and group size, part i having Ns[i]
 * columns, into ONE buffer for a layer of N = sum Ns[i] columns: part i is
 * columns [Ns[0] + ... + Ns[i-1], ... + Ns[i]) of that layer (the bytes equal
 * w4a16_repack of the parts' words and scales concatenated along N).  A
 * w4a16_gemm with N = sum Ns[i] then computes every part in one launch, Y
 * holding the parts' outputs side by side.
 *   count            1..64;
 *   qweights, scales host arrays of `count` device pointers (GPTQ layout,
 *                    int32 [K/8][Ns[i]] and fp16 bits [K/G][Ns[i]]);
 *   Ns               host array of `count` column counts;
 *   packed           device, w4a16_packed_bytes(K, sum Ns[i], G) bytes.
 * Requirements: every part as for w4a16_repack (so each Ns[i] % 64 == 0).
 * Errors as for w4a16_repack; MXG_ERR_INVALID_ARG for a NULL array or a
 * count outside 1..64. */
MXG_API int w4a16_repack_fused(int count, const int32_t *const *qweights,
                 const uint16_t *const *scales, const int *Ns, int K, int group_size,
                 void *packed, cudaStream_t stream);

/* Workspace bytes w4a16_gemm needs for this shape on the current device
 * (split-K partial sums, arrival counters and the status word). */
MXG_API size_t w4a16_workspace_bytes(int M, int N, int K, int group_size);

/* Y = X * dequant(W)^T.
 *   X         device, bf16 [M][K] row-major.
 *   packed    device, output of w4a16_repack for (K, N, G).
 *   Y         device, bf16 [M][N] row-major.
 *   workspace device, >= w4a16_workspace_bytes(M, N, K, G) bytes, zero-filled
 *             once before its first use.  Its first 256 bytes hold the status
 *             word, then come arrival counters, then scratch for partial
 *             sums; every call leaves the status word and the counters zero
 *             again (except after an error, when the caller must zero it
 *             before reuse), while the scratch keeps whatever it held.  Calls
 *             that share a workspace must be ordered on one stream.
 * M >= 1.  M <= 32 runs the weight-streaming path (the layer is bound by HBM
 * bytes of W); larger M runs the tensor-core path.  Shape rules as for
 * w4a16_repack. */
MXG_API int w4a16_gemm(const void *X, const void *packed, int M, int N, int K, int group_size,
               void *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* w4a16_gemm with per-call options (NULL = the defaults of w4a16_gemm). */
MXG_API int w4a16_gemm_ex(const void *X, const void *packed, int M, int N, int K,
               int group_size, void *Y, void *workspace, size_t workspace_bytes,
               const mxg_gemm_options *opts, cudaStream_t stream);

/* w4a16_gemm on the weight-streaming path without a caller workspace.  The
 * source pages have no counterpart to this call: it exists for callers that
 * cannot allocate a workspace (a plain C host with no device allocator of its
 * own; a serving process whose device memory is reserved up front).  It
 * allocates nothing: its scratch is one fixed 2 MiB array in device global
 * memory, one per device and process, shared by every call of this entry
 * point.
 *   X, packed, Y, shape rules: as for w4a16_gemm, with 1 <= M <= 32 (else
 *   MXG_ERR_UNSUPPORTED_SHAPE).  A shape whose partial sums and counters do
 *   not fit the array returns MXG_ERR_WORKSPACE before any launch (on a
 *   148-SM B200 every M <= 32 shape fits).
 * The first call on a device does a one-time set-up with that device
 * current: it looks the array up and zeroes its status word and counters on
 * `stream`; make that first call before any stream capture (inside one it
 * returns MXG_ERR_CAPTURE, and a later call outside a capture sets up).
 * Every call that completes without an error leaves the counters zero; the
 * partial-sum scratch keeps the last call's contents.  Calls that are not
 * ordered with respect to each other race on the array.  The array is 16 MiB
 * per device (every M <= 32 shape fits on a 148-SM B200).
 * A kernel that gives up a bounded wait records MXG_ERR_TIMEOUT in the
 * array's status word and returns MXG_OK to nobody: callers check the status
 * word with w4a16_static_scratch_status (for instance after each step of a
 * serving loop, outside any capture) and clear it before further calls. */
MXG_API int w4a16_gemm_static_scratch(const void *X, const void *packed, int M, int N, int K,
               int group_size, void *Y, cudaStream_t stream);

/* Status word of this device's w4a16_gemm_static_scratch array (no
 * counterpart on the source pages).  Copies it to *status (MXG_OK or the
 * first error a kernel recorded, e.g. MXG_ERR_TIMEOUT); with reset = 1 also
 * zeroes the status word and the arrival counters, which a timed-out call
 * may have left non-zero, so later calls start clean.  Stream-ordered on
 * `stream` (behind the calls queued there) and synchronizes it.  Does the
 * array's one-time set-up if no call did yet (so not inside a capture).
 * reset other than 0 or 1, or a NULL status: MXG_ERR_INVALID_ARG. */
MXG_API int w4a16_static_scratch_status(int *status, int reset, cudaStream_t stream);

/* ------------------------------------------------------------------ INT8 */

/* INT8 W8A16 for the vocabulary head (the Eole recipe, section "Optional
 * vocabulary-head quantization": symmetric group-wise round-to-nearest int8,
 * group size 32, 64 or 128; the W4A16 LowLatency model card: INT8 lm_head,
 * RTN g128).  Codes q in 0..255, four per int32 word along K: the code of
 * row k = 4i + j is bits [8j, 8j+7] of word (i, n) of qweight[K/4][N];
 * w[n][k] = (q - 128) * scale[k / G][n], scales fp16 [K/G][N].  Only the
 * weight-streaming path exists for INT8 (M <= 32: decode and verify chunks
 * against a vocabulary-sized N).
 *
 * Re-packed bytes: N*K code bytes (the codes split into a low-nibble and a
 * high-nibble plane, each in the INT4 layout) then 2*N*K/G scale bytes;
 * 0 for a shape w8a16_repack rejects. */
MXG_API size_t w8a16_packed_bytes(int K, int N, int group_size);

/* Offline re-pack: qweight device int32 [K/4][N]; scales device fp16 bits
 * [K/G][N]; packed device, w8a16_packed_bytes(K, N, G) bytes.
 * Requirements as for w4a16_repack (G in {32, 64, 128}; K % 64 == 0;
 * K % G == 0; N % 64 == 0), else MXG_ERR_UNSUPPORTED_SHAPE. */
MXG_API int w8a16_repack(const int32_t *qweight, const uint16_t *scales, int K, int N,
                 int group_size, void *packed, cudaStream_t stream);

/* The same re-pack from the compressed-tensors export of the head (the W4A16
 * LowLatency model card: the INT8 lm_head is written in compressed-tensors
 * form): weight_packed device int32 [N][K/4] (word (n, i) holds rows
 * 4i .. 4i+3 of column n, least significant byte first, same code values),
 * weight_scale device fp16 bits [N][K/G].  The bytes written equal
 * w8a16_repack of the transposed words and scales. */
MXG_API int w8a16_repack_ct(const int32_t *weight_packed, const uint16_t *weight_scale, int K,
                 int N, int group_size, void *packed, cudaStream_t stream);

/* Workspace bytes w8a16_gemm needs (0 for a rejected shape or M > 32). */
MXG_API size_t w8a16_workspace_bytes(int M, int N, int K, int group_size);

/* Y = X * dequant(W)^T for INT8 weights re-packed by w8a16_repack.
 * Arguments, workspace and errors as for w4a16_gemm; 1 <= M <= 32, else
 * MXG_ERR_UNSUPPORTED_SHAPE. */
MXG_API int w8a16_gemm(const void *X, const void *packed, int M, int N, int K, int group_size,
               void *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* w8a16_gemm with per-call options (NULL = defaults; path MXG_PATH_TENSOR is
 * MXG_ERR_INVALID_ARG: INT8 has the weight-streaming path only). */
MXG_API int w8a16_gemm_ex(const void *X, const void *packed, int M, int N, int K,
               int group_size, void *Y, void *workspace, size_t workspace_bytes,
               const mxg_gemm_options *opts, cudaStream_t stream);

/* ----------------------------------------------------------------- MXFP8 */

/* Workspace bytes mxfp8_gemm needs for this shape on the current device. */
MXG_API size_t mxfp8_workspace_bytes(int M, int N, int K);

/* Y = X * dequant(W)^T with MXFP8 weights.
 *   X   device, bf16 [M][K];  Wq device, E4M3 [N][K];  Ws device, E8M0 [N][K/32];
 *   Y   device, bf16 [M][N];  workspace as for w4a16_gemm.
 * Requirements (the format's kernel constraints): N >= 128 and K % 32 == 0,
 * else MXG_ERR_UNSUPPORTED_SHAPE.  N need not be a multiple of 16 and K need
 * not be a multiple of 128: ragged tiles are predicated.  Activations stay
 * bf16 (weight-only quantization). */
MXG_API int mxfp8_gemm(const void *X, const uint8_t *Wq, const uint8_t *Ws, int M, int N, int K,
               void *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* mxfp8_gemm with per-call options (NULL = the defaults of mxfp8_gemm). */
MXG_API int mxfp8_gemm_ex(const void *X, const uint8_t *Wq, const uint8_t *Ws, int M, int N,
               int K, void *Y, void *workspace, size_t workspace_bytes,
               const mxg_gemm_options *opts, cudaStream_t stream);

/* Re-packed MXFP8 for the decode shapes: this library's arrangement of the
 * format's codes and scales (the format fixes the values, not the layout).
 * The codes and E8M0 scales are laid out by column groups of 256 so that a
 * group's 128 rows of K are one contiguous range, like the INT4 layout;
 * mxfp8_gemm_packed streams them with one bulk copy per stage, converts
 * E4M3 pairs to f16 pairs in hardware (exact), multiplies on fp16 tensor
 * cores against the activations converted to fp16 with a power-of-two
 * factor per 64 rows of K and token (exact unless a value is 2^28 times
 * smaller than the largest of its 64), and applies 2^(E - 127) per 32-k
 * block in fp32.
 * Packed bytes: N*K codes then N*K/32 scales; 0 for a rejected shape
 * (N % 64 == 0 and K % 64 == 0 are required). */
MXG_API size_t mxfp8_packed_bytes(int N, int K);

/* Offline re-pack: Wq device E4M3 [N][K], Ws device E8M0 [N][K/32], packed
 * device, mxfp8_packed_bytes(N, K) bytes (all 16-byte aligned, else
 * MXG_ERR_INVALID_ARG).  MXG_ERR_UNSUPPORTED_SHAPE unless N % 64 == 0 and
 * K % 64 == 0.  Asynchronous on `stream`; Wq and Ws may be freed once the
 * stream has passed the call. */
MXG_API int mxfp8_repack(const uint8_t *Wq, const uint8_t *Ws, int N, int K, void *packed,
                 cudaStream_t stream);

/* Workspace bytes mxfp8_gemm_packed needs (0 for a rejected shape, M > 16,
 * or activations too wide to stay resident). */
MXG_API size_t mxfp8_packed_workspace_bytes(int M, int N, int K);

/* Y = X * dequant(W)^T from mxfp8_repack's buffer: the same result as
 * mxfp8_gemm on the original Wq, Ws up to fp32 summation order.
 *   X device bf16 [M][K]; packed as above; Y device bf16 [M][N];
 *   workspace as for w4a16_gemm, sized by mxfp8_packed_workspace_bytes.
 * 1 <= M <= 16 (the weight-streaming path only; larger M goes to mxfp8_gemm
 * with the original layout), N % 64 == 0, K % 64 == 0, and the CTA's
 * activations must fit in shared memory beside the ring; else
 * MXG_ERR_UNSUPPORTED_SHAPE. */
MXG_API int mxfp8_gemm_packed(const void *X, const void *packed, int M, int N, int K, void *Y,
               void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* mxfp8_gemm_packed with per-call options (NULL = defaults; path
 * MXG_PATH_TENSOR is MXG_ERR_INVALID_ARG). */
MXG_API int mxfp8_gemm_packed_ex(const void *X, const void *packed, int M, int N, int K,
               void *Y, void *workspace, size_t workspace_bytes,
               const mxg_gemm_options *opts, cudaStream_t stream);

/* ------------------------------------- dense bf16, few output columns */

/* Y = X * W^T with dense bf16 weights, for the paired GDN A/B projection of
 * the Eole recipe (section "Pack inference projections": two dense bf16
 * projections of 48 x 5120 computed together, N = 96, for single-token
 * decoding and four-token verification; below the N >= 128 of the MXFP8
 * path).  Latency-bound: one CTA per 8 rows of W, whose warps split K and
 * add their fp32 partials in a fixed order (bitwise reproducible).
 *   X  device, bf16 [M][K];  W device, bf16 [N][K] (K contiguous);
 *   Y  device, bf16 [M][N];  workspace as for w4a16_gemm, sized by
 *   bf16_gemm_small_workspace_bytes.
 * Requirements: 1 <= M <= 8; 16 <= N <= 2048 with N % 16 == 0; K >= 64 and
 * K % 64 == 0; else MXG_ERR_UNSUPPORTED_SHAPE.  Weights are read before the
 * wait for the previous kernel (see the conventions above). */
MXG_API size_t bf16_gemm_small_workspace_bytes(int M, int N, int K);
MXG_API int bf16_gemm_small(const void *X, const void *W, int M, int N, int K, void *Y,
               void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* bf16_gemm_small with per-call options (NULL = defaults; only
 * late_weights applies, a path other than MXG_PATH_AUTO is
 * MXG_ERR_INVALID_ARG). */
MXG_API int bf16_gemm_small_ex(const void *X, const void *W, int M, int N, int K, void *Y,
               void *workspace, size_t workspace_bytes, const mxg_gemm_options *opts,
               cudaStream_t stream);

/* --------------------------------------------------- test and diagnostics */

/* Decode a re-packed INT4 buffer with the device routines of the GEMM paths.
 *   codes  device, uint8 [N][K]: the 4-bit codes;
 *   w_fp32 device, float [N][K] or NULL: (q - 8) * scale, exact in fp32;
 *   w_bf16 device, bf16 bits [N][K] or NULL: the bf16 nearest (q - 8) * scale
 *          (ties to even), the operand of the tensor-core path. */
MXG_API int w4a16_unpack(const void *packed, int K, int N, int group_size,
                 uint8_t *codes, float *w_fp32, uint16_t *w_bf16, cudaStream_t stream);

/* Decode MXFP8 weights with the device routine of the GEMM paths:
 * w_bf16[N][K] = bf16 nearest e4m3(Wq) * 2^(Ws - 127) (exact whenever that
 * value is a normal bf16). */
MXG_API int mxfp8_dequant(const uint8_t *Wq, const uint8_t *Ws, int N, int K,
                  uint16_t *w_bf16, cudaStream_t stream);

/* Copy the workspace status word to the host (synchronizes `stream`).
 * *status receives MXG_OK or the first error a kernel recorded. */
MXG_API int mxg_workspace_status(const void *workspace, int *status, cudaStream_t stream);

/* Runs one CTA whose pipeline wait can never complete (nothing arrives on
 * its barrier) with a time limit of `limit_us` microseconds, to exercise the
 * timeout path.  The kernel records MXG_ERR_TIMEOUT in the workspace status
 * word and returns; the context stays usable.  workspace: >= 256 bytes, or
 * NULL for the static scratch array of w4a16_gemm_static_scratch on the
 * current device (read and clear it with w4a16_static_scratch_status). */
MXG_API int mxg_selftest_wait_timeout(void *workspace, int limit_us, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXG_H */
