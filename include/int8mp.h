/*
 * int8mp.h -- C ABI of libint8mp, the LLM.int8() forward linear layer
 * (bitsandbytes Linear8bitLt with has_fp16_weights=False) for NVIDIA B200
 * (sm_100a).
 *
 * The operation (Hugging Face integration page for LLM.int8(), "Core idea of
 * LLM.int8()", steps 1-3, and "Quantization mechanics"):
 *   1. outlier columns: k is an outlier if |X[t,k]| > threshold for some token t
 *      (bitsandbytes Linear8bitLt docstring, `threshold`; issue #1609: the
 *      threshold acts on activations; state.idx lists the outlier columns);
 *   2. the non-outlier part of X is quantised row-wise to int8 with scale
 *      127/absmax (absmax over the row's non-outlier columns), the weight
 *      row-wise per output feature (CB int8, SCB = absmax fp32, so that W is
 *      recovered as CB*SCB/127, "Integration into transformers"); the two are
 *      multiplied in int8 with int32 accumulation, while the outlier columns
 *      are multiplied in 16-bit floating point;
 *   3. the int8 result is dequantised with (row scale) x (column scale) / 127^2,
 *      summed with the 16-bit result and the bias, and returned in fp16.
 *
 * Conventions for every entry point:
 *   - Matrices are row-major.  X fp16 [T,K] (K = in_features contiguous),
 *     W fp16 [N,K] (the nn.Linear weight layout, N = out_features),
 *     Y fp16 [T,N].
 *   - Pointers documented as "device" must be CUDA device memory of the
 *     current device; the caller owns every buffer.  The library allocates
 *     nothing and keeps no per-call state outside the caller's workspace.
 *     Per device and process it caches device properties and what the first
 *     launch of a kernel learns (whether its 2-CTA or T-CTA clusters can be
 *     scheduled; a shared-memory carveout hint set on the kernel).
 *   - Calls are asynchronous on `stream` unless stated otherwise.  Argument
 *     errors are reported synchronously before any work is enqueued; launch
 *     failures are reported as I8_ERR_CUDA.  A device-side wait that gives up
 *     (I8_ERR_TIMEOUT) is recorded in the workspace and read back by
 *     int8_check_status().
 *   - Shape rules: K and N are positive multiples of 16 with K <= 131072
 *     (so that |acc| <= K*127^2 fits int32); T >= 0.  X, CB, Y and the
 *     workspace must be 16-byte aligned, SCB 4-byte aligned, bias and idx
 *     naturally aligned.
 *   - Results are deterministic: idx is ascending, and the integer stages
 *     (idx, n_out, CB, SCB, the int8 codes of X, the row scales and the int32
 *     accumulators) are identical from run to run.
 */
#ifndef INT8MP_H_
#define INT8MP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

typedef enum i8_status {
  I8_OK = 0,
  I8_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad shape */
  I8_ERR_WORKSPACE = 2,   /* workspace too small or misaligned */
  I8_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  I8_ERR_TIMEOUT = 4,     /* a device-side wait gave up; the kernel returned early */
  I8_ERR_UNSUPPORTED = 5  /* no sm_100 device, or the driver lacks TMA map encoding */
} i8_status;

/* 16-bit element types of the *_ex calls (see "16-bit element type" below). */
enum { I8_DTYPE_F16 = 0, I8_DTYPE_BF16 = 1 };

/* Human-readable name of a status code (static string, never NULL). */
const char* int8_status_string(int status);

/* Library ABI version (major*100 + minor). */
int int8_version(void);

/*
 * Weight quantisation, done once per layer (the `.to(device)` step of
 * Linear8bitLt with has_fp16_weights=False; Hugging Face integration page,
 * "Integration into transformers": CB in [-127, 127], W ~ CB*SCB/127).
 *   W   device fp16 [N,K]   input weight, read only
 *   CB  device int8 [N,K]   output codes: clamp(roundf(W*(127/SCB[j])), -127, 127),
 *                           ties away from zero; all zero when SCB[j] == 0
 *   SCB device fp32 [N]     output per-row absmax max_k |W[j,k]|
 * Asynchronous on `stream`.
 */
i8_status int8_quantize_weight(const void* W, int64_t N, int64_t K, int8_t* CB, float* SCB,
                               cudaStream_t stream);

/* Bytes of device workspace int8_linear_forward needs for a T x K -> N
 * forward (worst case: every column an outlier).  Host-only; never fails. */
size_t int8_linear_workspace_bytes(int64_t T, int64_t K, int64_t N);

/*
 * The forward (steps 1-3 above).
 *   X         device fp16 [T,K]   activations, read only
 *   CB, SCB   device              output of int8_quantize_weight for [N,K]
 *   bias      device fp16 [N] or NULL (no bias)
 *   threshold outlier threshold; a column is an outlier iff some |X[t,k]| >
 *             threshold (strict).  threshold <= 0 or NaN switches the
 *             decomposition off (no outlier columns, pure int8 product).
 *             NaN entries of X never flag a column.
 *   Y         device fp16 [T,N]   output
 *   idx       device int32 [K]    capacity K; receives the ascending outlier
 *                                 column indices (Linear8bitLt state.idx)
 *   n_out     device int32 [1]    receives the number of outlier columns
 *   workspace device, >= int8_linear_workspace_bytes(T,K,N) bytes, 256-byte
 *             aligned; its contents need no initialisation and are
 *             overwritten.  One workspace must not be shared by forwards
 *             that can run concurrently.
 * T <= 16 takes the weight-streaming decode kernel, larger T a tensor-core
 * GEMM (see int8_linear_forward_path); all give the same integer stages.  Asynchronous on `stream`; n_out
 * stays on the device (no host synchronisation).
 */
i8_status int8_linear_forward(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                              const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                              int32_t* n_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* As int8_linear_forward, with the product kernel chosen explicitly:
 * path 0 = automatic: the decode GEMV for T <= 16, else the tensor-core GEMM
 * as path 1; 1 = tensor-core GEMM (any T; SM pairs with 256x512 tiles when
 * 2-CTA clusters can be launched, else single SMs);
 * 2 = decode GEMV (T <= 16, else I8_ERR_INVALID_ARG); 3 = tensor-core GEMM
 * on single SMs (128x256 tiles). */
i8_status int8_linear_forward_path(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                   const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                   int32_t* n_out, void* workspace, size_t workspace_bytes, int path,
                                   cudaStream_t stream);

/*
 * The forward of a layer with has_fp16_weights=True (bitsandbytes
 * Linear8bitLt docstring: the weights remain fp16 and are quantised on the fly
 * during each forward pass).  Each call quantises W exactly as
 * int8_quantize_weight does (into the workspace) and runs the forward; the
 * outlier columns are multiplied with W's own fp16 columns W[:, idx] rather
 * than the dequantised CB.
 *   W         device fp16 [N,K]
 *   workspace device, >= int8_linear_fp16w_workspace_bytes(T,K,N), 256-byte
 *             aligned (the forward's workspace followed by CB [N,K], SCB [N]).
 * Other arguments, results and errors as int8_linear_forward.
 */
size_t int8_linear_fp16w_workspace_bytes(int64_t T, int64_t K, int64_t N);
i8_status int8_linear_forward_fp16w(const void* X, int64_t T, int64_t K, const void* W, const void* bias, int64_t N,
                                    float threshold, void* Y, int32_t* idx, int32_t* n_out, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of
 * `workspace`: I8_OK, or I8_ERR_TIMEOUT if a kernel of the most recent
 * forward using this workspace gave up a wait.  *where (may be NULL)
 * receives the tag of the wait that gave up; 0xffffffff when the
 * synchronisation itself failed (I8_ERR_CUDA, see int8_last_cuda_error), and
 * 0xbad00000 | value when the status word holds a value no kernel writes.
 */
i8_status int8_check_status(void* workspace, uint32_t* where, cudaStream_t stream);

/* Text of the last CUDA error this thread's calls into the library met
 * ("no error" if none).  Host-only. */
const char* int8_last_cuda_error(void);

/*
 * The forward with HOST activations and output: copies X host->device,
 * runs int8_linear_forward, copies Y (and idx, n_out when non-NULL) back,
 * and synchronises `stream` before returning (blocking).  CB, SCB, bias stay
 * device pointers (the quantised layer is resident).  X_host and Y_host
 * should be page-locked for full copy bandwidth.
 *   idx_host  host int32 [K] or NULL;  n_out_host host int32 [1] or NULL.
 *   workspace device, >= int8_linear_forward_host_workspace_bytes(T,K,N).
 * Returns I8_ERR_TIMEOUT if a kernel gave up a wait.
 */
size_t int8_linear_forward_host_workspace_bytes(int64_t T, int64_t K, int64_t N);
i8_status int8_linear_forward_host(const void* X_host, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                   const void* bias, int64_t N, float threshold, void* Y_host,
                                   int32_t* idx_host, int32_t* n_out_host, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/* As int8_linear_forward_host for element type `dtype` (I8_DTYPE_F16 or
 * I8_DTYPE_BF16 below), but non-blocking: the copies and kernels are enqueued
 * on `stream` and the call returns at once.  X_host, Y_host, idx_host and
 * n_out_host must stay valid (and Y_host unread) until `stream` has been
 * synchronised; then int8_check_status(workspace, ...) reads the status word.
 * X_host and Y_host must be page-locked: pageable memory makes the copies
 * synchronous.  Two calls on two streams with two workspaces overlap one
 * forward's Y download with the next one's X upload and kernels. */
i8_status int8_linear_forward_host_async(const void* X_host, int dtype, int64_t T, int64_t K, const int8_t* CB,
                                         const float* SCB, const void* bias, int64_t N, float threshold,
                                         void* Y_host, int32_t* idx_host, int32_t* n_out_host, void* workspace,
                                         size_t workspace_bytes, cudaStream_t stream);

/* As int8_linear_forward_path, and records caller-created CUDA events
 * (cudaEvent_t, passed as void*) on `stream` around the stages:
 * events[0] before the first stage, events[1] after the outlier pass,
 * events[2] after the row quantisation, events[3] after the product kernel.
 * On the decode path (the weight-streaming product, T <= 16) the outlier pass
 * and the row quantisation are one kernel: events[1] and events[2] both
 * follow it.  For measurement: event deltas time each kernel on its launching
 * stream (the events between kernels stop them from overlapping). */
i8_status int8_linear_forward_timed(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                    const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                    int32_t* n_out, void* workspace, size_t workspace_bytes, int path,
                                    void* const* events, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Persistence of a quantised layer (host memory only; no CUDA call).
 *
 * The Hugging Face integration page lists, under "Future work and
 * limitations", that INT8 checkpoints omitted the quantisation statistics
 * CB/SCB, so a quantised layer could not be loaded directly.  These calls
 * store CB, SCB and (optionally) the bias in one byte image and read them
 * back, so a layer is loaded without its fp16 weight and without quantising
 * again.  Image (little-endian): "I8MPLYR1", int64 N, int64 K, uint32 flags
 * (bit 0 = bias present, bit 1 = the bias is bf16 rather than fp16), uint32 0,
 * then fp32 SCB[N], the 16-bit bias[N] if present, int8 CB[N*K] row-major.
 * Shapes follow the forward's rules.
 * ------------------------------------------------------------------------- */

/* Image size in bytes (0 for an unsupported shape). */
size_t int8_layer_packed_bytes(int64_t N, int64_t K, int has_bias);
/* Writes the image of host CB [N,K], SCB [N], bias [N] (or NULL) into `out`
 * (>= int8_layer_packed_bytes bytes, else I8_ERR_WORKSPACE). */
i8_status int8_layer_pack(const int8_t* CB, const float* SCB, const void* bias, int64_t N, int64_t K, void* out,
                          size_t out_bytes);
/* Validates an image (magic, shape rules, flags, length) and reads N, K and
 * whether it holds a bias.  I8_ERR_INVALID_ARG for anything malformed. */
i8_status int8_layer_unpack_header(const void* buf, size_t bytes, int64_t* N, int64_t* K, int* has_bias);
/* Copies an image's SCB, bias (when present and `bias` is not NULL) and CB
 * into host buffers sized from int8_layer_unpack_header. */
i8_status int8_layer_unpack(const void* buf, size_t bytes, int8_t* CB, float* SCB, void* bias);
/* int8_layer_pack with the bias's element type (I8_DTYPE_F16 or I8_DTYPE_BF16,
 * ignored without a bias) recorded in the image. */
i8_status int8_layer_pack_ex(const int8_t* CB, const float* SCB, const void* bias, int bias_dtype, int64_t N,
                             int64_t K, void* out, size_t out_bytes);
/* int8_layer_unpack_header that also reads the bias's element type into
 * *bias_dtype (may be NULL; I8_DTYPE_F16 when the image has no bias). */
i8_status int8_layer_unpack_header_ex(const void* buf, size_t bytes, int64_t* N, int64_t* K, int* has_bias,
                                      int* bias_dtype);

/* ---------------------------------------------------------------------------
 * Inspection entry points (used by the parity tests; not needed for inference)
 * ------------------------------------------------------------------------- */

/* Byte offsets of the forward's intermediate buffers inside the workspace, so
 * a caller can read the stage results of the most recent forward:
 *   mask  uint32 [ceil(K/32)]  outlier column bitmask (bit k%32 of word k/32),
 *                              followed by uint32 [ceil(K/32)] prefix counts
 *                              (outlier columns in the words before each word)
 *   sA    fp32 [T]             row absmax over non-outlier columns
 *   Xq    int8 [T,K]           row codes (outlier columns 0)
 *   Xo    fp16 [T,ldo]         X[:, idx[o]] for o < n_out, zero up to a multiple of 64
 *   Wo    fp16 [N,ldo]         fp16((CB[j,idx[o]]*SCB[j])/127), same padding
 *                              (written by the tensor-core path only)
 * ldo (elements) = K rounded up to a multiple of 64.  Host-only. */
typedef struct int8_ws_layout {
  uint64_t status, mask, sA, Xq, Xo, Wo, total;
  int64_t ldo;
} int8_ws_layout;
i8_status int8_linear_workspace_layout(int64_t T, int64_t K, int64_t N, int8_ws_layout* out);

/*
 * Int8 product alone: acc[t,j] = sum_k Xq[t,k]*CB[j,k] (exact int32), with the
 * same kernels as the forward (path 1 = tensor-core GEMM on SM pairs, 2 =
 * decode GEMV for T <= 16, 3 = tensor-core GEMM on single SMs, 0 = automatic).
 *   Xq device int8 [T,K], CB device int8 [N,K], acc device int32 [T,N].
 *   workspace as for int8_linear_forward (only its status word is used).
 */
i8_status int8_gemm_i32(const int8_t* Xq, int64_t T, int64_t K, const int8_t* CB, int64_t N, int32_t* acc,
                        int path, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Self-test of failure detection: launches one thread that waits, with a
 * limit of `limit_us` microseconds (1 .. 2000000), on an mbarrier that nothing
 * arrives on -- the same bounded wait the tensor-core GEMM uses for every
 * pipeline barrier.  The wait gives up, records I8_ERR_TIMEOUT (tag 0x5e1f) in
 * the workspace status word and returns; int8_check_status() then reports it,
 * and the CUDA context stays usable.  Nothing faults, traps or hangs. */
i8_status int8_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                     cudaStream_t stream);

/* The largest fp16 magnitude bit pattern (0..0x7bff) whose value is <= threshold;
 * the outlier test |x| > threshold is (bits(x) & 0x7fff) > this value for
 * non-NaN x.  Host-only; 0xffffffff when threshold <= 0 or NaN (no outliers). */
uint32_t int8_outlier_threshold_bits(float threshold);

/* ---------------------------------------------------------------------------
 * 16-bit element type.
 *
 * The bitsandbytes Linear8bitLt docstring describes the module for fp16 or
 * bf16 weights; the calls above take fp16.  The calls below take the element
 * type of every 16-bit operand -- X, W, bias, Y and the internal outlier
 * operands -- as `dtype`: I8_DTYPE_F16 (the calls above) or I8_DTYPE_BF16.
 * With bf16 the outlier test compares bf16 magnitudes, the outlier product
 * multiplies bf16 operands (the dequantised outlier weights are rounded to
 * bf16) with fp32 accumulation, and Y is rounded to bf16 (round to nearest
 * even).  The int8 stages and the fp32 arithmetic are those of the fp16 path.
 * Any other dtype value is I8_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------- */

/* int8_quantize_weight with W of element type `dtype`. */
i8_status int8_quantize_weight_ex(const void* W, int dtype, int64_t N, int64_t K, int8_t* CB, float* SCB,
                                  cudaStream_t stream);

/* The forward with X, bias and Y of element type `dtype`, the product kernel
 * chosen by `path` (as int8_linear_forward_path) and, when `events` is not
 * NULL, the four stage events of int8_linear_forward_timed.  Workspace size,
 * arguments, results and errors as int8_linear_forward. */
i8_status int8_linear_forward_ex(const void* X, int dtype, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                 const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                 int32_t* n_out, void* workspace, size_t workspace_bytes, int path,
                                 void* const* events, cudaStream_t stream);

/* int8_linear_forward_fp16w (has_fp16_weights=True) with X, W, bias and Y of
 * element type `dtype`. */
i8_status int8_linear_forward_fp16w_ex(const void* X, int dtype, int64_t T, int64_t K, const void* W,
                                       const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                       int32_t* n_out, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * N-sharded forward (one shard of the output features per GPU).
 *
 * The Hugging Face integration page ("Speed trade-offs", the table of
 * BLOOM-176B runs) serves the INT8 model over several GPUs.  The forward
 * splits along N with no exchange in the compute: every GPU holds the rows
 * [col_offset, col_offset + N) of CB, SCB and bias, sees the whole X, finds
 * the same outlier columns and row scales, and produces the matching column
 * block of Y.  This call computes that block and stores it straight into up
 * to 8 copies of the full output -- the caller's own and, for the gather, the
 * same buffer of every other GPU mapped into this device's address space --
 * so that the all-gather of Y happens inside the product kernel's epilogue.
 *   X, dtype, T, K, threshold, idx, n_out, workspace, path: as
 *             int8_linear_forward_ex (workspace sized for T, K, N).
 *   CB, SCB, bias  this GPU's shard: [N,K], [N], [N] (bias may be NULL).
 *   Y_dst     HOST array of n_dst (1..8) device pointers, each the start
 *             (column 0) of a row-major [T, ldY] output of element type
 *             `dtype`, 16-byte aligned; Y_dst[0] is this GPU's own.
 *   ldY       row stride of every Y_dst in elements: a multiple of 8, >= N.
 *   col_offset first column of this shard in Y: a multiple of 8, with
 *             col_offset + N <= ldY.
 * Columns outside [col_offset, col_offset + N) are not touched.  The stores to
 * other GPUs' memory are complete when the kernel is; before any GPU reads
 * its full Y, every GPU's forward must have completed (for example a
 * stream-ordered barrier across the GPUs after this call).  Errors as
 * int8_linear_forward_ex; a bad Y_dst, ldY or col_offset is
 * I8_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------- */
i8_status int8_linear_forward_sharded(const void* X, int dtype, int64_t T, int64_t K, const int8_t* CB,
                                      const float* SCB, const void* bias, int64_t N, float threshold,
                                      void* const* Y_dst, int n_dst, int64_t ldY, int64_t col_offset,
                                      int32_t* idx, int32_t* n_out, void* workspace, size_t workspace_bytes,
                                      int path, cudaStream_t stream);

/* Which product kernel a forward of T x K -> N on `path` (as
 * int8_linear_forward_path) runs on the current device: 1 = tensor-core GEMM
 * on SM pairs, 2 = decode GEMV, 3 = tensor-core GEMM on single SMs; -1 for
 * arguments the forward would reject or no sm_100 device.  Host-only
 * apart from reading device attributes. */
int int8_linear_product_kernel(int64_t T, int64_t K, int64_t N, int path);

/* int8_outlier_threshold_bits for element type `dtype`: the largest magnitude
 * pattern of that type (bf16: 0..0x7f80) whose value is <= threshold.
 * 0xffffffff when threshold <= 0 or NaN, 0xfffffffe for an unknown dtype. */
uint32_t int8_outlier_threshold_bits_ex(float threshold, int dtype);

/* ---------------------------------------------------------------------------
 * Forward without any caller-provided or allocated scratch memory.
 *
 * The pages have no counterpart to this call: it exists for callers that
 * cannot allocate device memory and cannot pass a workspace -- for example a
 * plugin inside an inference runtime that owns all device memory and forbids
 * allocation during its execute call (cudaMalloc may synchronise the device
 * and escapes the host's memory accounting), or an application with a fixed
 * device-memory budget.
 *
 * Same arguments and results as int8_linear_forward for the decode case
 * (1 <= T <= 16, same kernels, same integer stages), minus the workspace:
 * the intermediate buffers live in a 4 MiB array compiled into the library
 * (a file-scope __device__ array, held by every GPU that loads the library
 * until the process exits).  It allocates nothing (no cudaMalloc, cudaFree or
 * allocating library call).
 *   - Size limit: the scratch holds 256 B + 8*ceil(K/32) + 4*T + T*K +
 *     2*T*ceil(K/64)*64 bytes (each part rounded up to 256 B); a T x K that
 *     needs more than 4 MiB (for T = 16: K above about 87000) is rejected
 *     with I8_ERR_WORKSPACE before any work is enqueued.  T outside
 *     [1, 16] is I8_ERR_INVALID_ARG.
 *   - The first call on each device does all of this call's per-device
 *     set-up, with that device current: it resolves the array's device
 *     address (cudaGetSymbolAddress) and, for every T in 1..16, asks whether
 *     the decode prep kernel's T-CTA cluster can be scheduled, and sets the
 *     decode GEMV's shared-memory carveout hint.  One first call with any T
 *     is enough; make it before any stream capture.  Later calls make no CUDA
 *     call other than cudaGetDevice, the two kernel launches and the launch
 *     error query.  A failing CUDA call is reported as I8_ERR_CUDA and its
 *     text by int8_last_cuda_error().
 *   - Every call on a device shares the one array, and the array keeps the
 *     previous call's contents (each call clears what must start at zero).
 *     Calls that can overlap on the GPU (other streams, other host threads)
 *     race on it: serialise them.
 *   - These kernels contain no device-side waits, so there is no status word
 *     to read back.
 */
i8_status int8_linear_forward_decode_static(const void* X, int64_t T, int64_t K, const int8_t* CB,
                                            const float* SCB, const void* bias, int64_t N, float threshold,
                                            void* Y, int32_t* idx, int32_t* n_out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* INT8MP_H_ */
