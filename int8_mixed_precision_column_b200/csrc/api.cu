// C ABI of libint8mp: argument validation, workspace layout and dispatch of
// the LLM.int8() forward linear layer kernels.  See include/int8mp.h for the
// contract of every entry point.
#include <cmath>
#include <cstring>

#include "int8mp.h"
#include "kernels.h"

using namespace i8mp;

namespace {

constexpr int64_t kMaxK = 131072;      // K*127^2 < 2^31
constexpr int64_t kMaxRows = int64_t(1) << 30;
constexpr int kMaxDevices = 64;

struct DevInfo {
  bool probed = false;
  bool sm100 = false;
  int num_sms = 0;
};
DevInfo g_dev[kMaxDevices];

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Maps a CUDA result to a status, remembering the error for int8_last_cuda_error().
inline i8_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return I8_OK;
  g_last_cuda_error = e;
  return I8_ERR_CUDA;
}

i8_status device_info(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return I8_ERR_UNSUPPORTED;
  DevInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_status(e);
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return cuda_status(e);
    d.sm100 = (major == 10);
    d.num_sms = sms;
    d.probed = true;
  }
  if (!d.sm100) return I8_ERR_UNSUPPORTED;
  *num_sms = d.num_sms;
  return I8_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline uint64_t align_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

bool shape_ok(int64_t T, int64_t K, int64_t N) {
  return T >= 0 && T <= kMaxRows && K >= 16 && K % 16 == 0 && K <= kMaxK && N >= 16 && N % 16 == 0 &&
         N <= kMaxRows;
}

int8_ws_layout make_layout(int64_t T, int64_t K, int64_t N) {
  int8_ws_layout L;
  L.ldo = ((K + 63) / 64) * 64;
  L.status = 0;
  L.mask = 256;
  // mask words, then the per-word prefix counts of the outlier columns
  const uint64_t mask_bytes = static_cast<uint64_t>((K + 31) / 32) * 4;
  L.sA = align_up(L.mask + 2 * mask_bytes, 256);
  L.Xq = align_up(L.sA + static_cast<uint64_t>(T) * 4, 256);
  L.Xo = align_up(L.Xq + static_cast<uint64_t>(T) * K, 256);
  L.Wo = align_up(L.Xo + static_cast<uint64_t>(T) * L.ldo * 2, 256);
  L.total = align_up(L.Wo + static_cast<uint64_t>(N) * L.ldo * 2, 256);
  return L;
}

struct HostExtra {
  uint64_t x, y, idx, n_out, total;
};
HostExtra make_host_extra(int64_t T, int64_t K, int64_t N) {
  const int8_ws_layout L = make_layout(T, K, N);
  HostExtra h;
  h.x = L.total;
  h.y = align_up(h.x + static_cast<uint64_t>(T) * K * 2, 256);
  h.idx = align_up(h.y + static_cast<uint64_t>(T) * N * 2, 256);
  h.n_out = align_up(h.idx + static_cast<uint64_t>(K) * 4, 256);
  h.total = align_up(h.n_out + 4, 256);
  return h;
}

float half_bits_value(uint32_t h) {
  const uint32_t e = (h >> 10) & 0x1fu;
  const uint32_t m = h & 0x3ffu;
  if (e == 0) return std::ldexp(static_cast<float>(m), -24);
  if (e == 31) return m == 0 ? INFINITY : NAN;
  return std::ldexp(static_cast<float>(m | 0x400u), static_cast<int>(e) - 25);
}

// bf16 is the upper half of an fp32 pattern.
float bf16_bits_value(uint32_t h) {
  const uint32_t u = h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint32_t threshold_bits(float thr, int dtype = kF16) {
  if (!(thr > 0.0f)) return 0xffffffffu;
  // largest pattern p in [0, inf pattern] with value(p) <= thr; value is monotone in p.
  const bool bf = dtype == kBF16;
  uint32_t lo = 0, hi = bf ? 0x7f80u : 0x7c00u;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) / 2;
    if ((bf ? bf16_bits_value(mid) : half_bits_value(mid)) <= thr)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

inline bool dtype_ok(int dtype) { return dtype == kF16 || dtype == kBF16; }


// The product kernel: decode GEMV, or the tensor-core GEMM on SM pairs (the
// single-SM GEMM when pairs are not launchable or when asked for explicitly).
// Which product kernel a forward of T x K -> N on `path` runs.  Automatic: the
// decode GEMV for T <= 16, else the SM-pair GEMM (256 x 512 tiles; measured
// at least as fast as the single-SM GEMM from under one wave of tiles up, to
// within 1 %), or the single-SM GEMM wherever 2-CTA clusters cannot be
// launched.
int product_kernel(int64_t T, int64_t N, int path) {
  (void)N;
  if (path == kPathDecode || (path == kPathAuto && T <= kDecodeMaxT)) return kPathDecode;
  if (path == kPathTensorCoreSingleSM) return kPathTensorCoreSingleSM;
  if (pair_kernel_max_clusters() <= 0) return kPathTensorCoreSingleSM;
  return kPathTensorCore;
}

cudaError_t launch_product(const GemmArgs& a, int path, bool gemv, int num_sms, cudaStream_t stream) {
  if (gemv) return launch_gemv_decode(a, num_sms, stream);
  if (product_kernel(a.T, a.N, path) == kPathTensorCore) return launch_gemm_tc2(a, stream);
  return launch_gemm_tc(a, num_sms, stream);
}

i8_status forward_impl(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB, const void* bias,
                       int64_t N, float threshold, void* Y, int32_t* idx, int32_t* n_out, void* ws, size_t ws_bytes,
                       int path, void* const* events, cudaStream_t stream, int dtype = kF16,
                       const void* Wf = nullptr, int64_t ldY = 0, void* const* ydst = nullptr, int n_ydst = 0) {
  if (!shape_ok(T, K, N) || !dtype_ok(dtype)) return I8_ERR_INVALID_ARG;
  if (path < kPathAuto || path > kPathTensorCoreSingleSM) return I8_ERR_INVALID_ARG;
  if (path == kPathDecode && T > kDecodeMaxT) return I8_ERR_INVALID_ARG;
  if (idx == nullptr || n_out == nullptr || !aligned(idx, 4) || !aligned(n_out, 4)) return I8_ERR_INVALID_ARG;
  if (T > 0) {
    if (X == nullptr || CB == nullptr || SCB == nullptr || Y == nullptr) return I8_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(CB, 16) || !aligned(Y, 16) || !aligned(SCB, 4) ||
        (bias != nullptr && !aligned(bias, 2)))
      return I8_ERR_INVALID_ARG;
  }
  const int8_ws_layout L = make_layout(T, K, N);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < L.total) return I8_ERR_WORKSPACE;
  int num_sms = 0;
  i8_status st = device_info(&num_sms);
  if (st != I8_OK) return st;

  auto mark = [&](int i) -> bool {
    return events == nullptr || cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream)) == I8_OK;
  };
  if (!mark(0)) return I8_ERR_CUDA;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const uint64_t mask_bytes = static_cast<uint64_t>((K + 31) / 32) * 4;
  const bool gemv = (path == kPathDecode) || (path == kPathAuto && T <= kDecodeMaxT);
  // the decode prep kernel clears the status word itself and keeps the mask
  // in shared memory; otherwise status word + mask start at zero
  const bool small_prep = gemv && T >= 1;
  cudaError_t e = small_prep ? cudaSuccess : cudaMemsetAsync(w, 0, L.mask + mask_bytes, stream);
  if (e != cudaSuccess) return cuda_status(e);
  if (T == 0) {
    e = cudaMemsetAsync(n_out, 0, sizeof(int32_t), stream);
    if (e != cudaSuccess) return cuda_status(e);
    return (mark(1) && mark(2) && mark(3)) ? I8_OK : I8_ERR_CUDA;
  }

  DevStatus* dst = reinterpret_cast<DevStatus*>(w + L.status);
  uint32_t* mask = reinterpret_cast<uint32_t*>(w + L.mask);
  uint32_t* prefix = mask + (K + 31) / 32;
  float* sA = reinterpret_cast<float*>(w + L.sA);
  int8_t* Xq = reinterpret_cast<int8_t*>(w + L.Xq);
  void* Xo = w + L.Xo;
  void* Wo = w + L.Wo;

  const uint32_t hb = threshold_bits(threshold, dtype);
  if (small_prep) {
    // one kernel for the outlier pass and the row quantisation
    e = launch_prep_small(X, dtype, T, K, hb, mask, prefix, idx, n_out, Xq, sA, Xo, L.ldo, dst, stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (!mark(1) || !mark(2)) return I8_ERR_CUDA;
  } else {
    if (hb == 0xffffffffu)
      e = cudaMemsetAsync(n_out, 0, sizeof(int32_t), stream);
    else
      e = launch_outliers(X, dtype, T, K, hb, mask, prefix, idx, n_out, dst, stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (!mark(1)) return I8_ERR_CUDA;
    // programmatic launches only directly after one of our kernels
    const bool after_outliers = (hb != 0xffffffffu);
    e = launch_rowquant(X, dtype, T, K, mask, prefix, idx, n_out, Xq, sA, Xo, L.ldo, CB, SCB, N, Wo, !gemv, Wf,
                        num_sms, dst, after_outliers, stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (!mark(2)) return I8_ERR_CUDA;
  }

  GemmArgs a;
  a.Xq = Xq;
  a.CB = CB;
  a.Xo = Xo;
  a.Wo = Wo;
  a.ldo = L.ldo;
  a.sA = sA;
  a.SCB = SCB;
  a.bias = bias;
  a.Y = Y;
  a.acc_out = nullptr;
  a.n_out = n_out;
  a.idx = idx;
  a.st = dst;
  a.T = T;
  a.N = N;
  a.K = K;
  a.mode = 0;
  a.pdl = true;  // follows the row quantisation kernel
  a.Wf = Wf;
  a.dtype = dtype;
  a.ldY = ldY;
  a.n_ydst = n_ydst;
  for (int d = 0; d < n_ydst; ++d) a.ydst[d] = ydst[d];
  e = launch_product(a, path, gemv, num_sms, stream);
  if (e != cudaSuccess) return cuda_status(e);
  return mark(3) ? I8_OK : I8_ERR_CUDA;
}

}  // namespace

namespace i8mp {
cudaError_t note_cuda_error(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error = e;
  return e;
}
}  // namespace i8mp

extern "C" {

const char* int8_status_string(int status) {
  switch (status) {
    case I8_OK: return "I8_OK";
    case I8_ERR_INVALID_ARG: return "I8_ERR_INVALID_ARG";
    case I8_ERR_WORKSPACE: return "I8_ERR_WORKSPACE";
    case I8_ERR_CUDA: return "I8_ERR_CUDA";
    case I8_ERR_TIMEOUT: return "I8_ERR_TIMEOUT";
    case I8_ERR_UNSUPPORTED: return "I8_ERR_UNSUPPORTED";
    default: return "I8_ERR_UNKNOWN";
  }
}

int int8_version(void) { return 100; }

uint32_t int8_outlier_threshold_bits(float threshold) { return threshold_bits(threshold, kF16); }

int int8_linear_product_kernel(int64_t T, int64_t K, int64_t N, int path) {
  if (!shape_ok(T, K, N) || path < kPathAuto || path > kPathTensorCoreSingleSM) return -1;
  if (path == kPathDecode && T > kDecodeMaxT) return -1;
  int num_sms = 0;
  if (device_info(&num_sms) != I8_OK) return -1;
  return product_kernel(T, N, path);
}

uint32_t int8_outlier_threshold_bits_ex(float threshold, int dtype) {
  if (!dtype_ok(dtype)) return 0xfffffffeu;
  return threshold_bits(threshold, dtype);
}

i8_status int8_quantize_weight_ex(const void* W, int dtype, int64_t N, int64_t K, int8_t* CB, float* SCB,
                                  cudaStream_t stream) {
  if (!dtype_ok(dtype)) return I8_ERR_INVALID_ARG;
  if (N < 0 || N > kMaxRows || K < 16 || K % 16 != 0 || K > kMaxK) return I8_ERR_INVALID_ARG;
  if (N == 0) return I8_OK;
  if (W == nullptr || CB == nullptr || SCB == nullptr) return I8_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(CB, 8) || !aligned(SCB, 4)) return I8_ERR_INVALID_ARG;
  int num_sms = 0;
  i8_status st = device_info(&num_sms);
  if (st != I8_OK) return st;
  return cuda_status(launch_quantize_weight(W, dtype, N, K, CB, SCB, stream));
}

i8_status int8_quantize_weight(const void* W, int64_t N, int64_t K, int8_t* CB, float* SCB, cudaStream_t stream) {
  return int8_quantize_weight_ex(W, kF16, N, K, CB, SCB, stream);
}

size_t int8_linear_workspace_bytes(int64_t T, int64_t K, int64_t N) {
  if (!shape_ok(T, K, N)) return 0;
  return static_cast<size_t>(make_layout(T, K, N).total);
}

i8_status int8_linear_workspace_layout(int64_t T, int64_t K, int64_t N, int8_ws_layout* out) {
  if (out == nullptr || !shape_ok(T, K, N)) return I8_ERR_INVALID_ARG;
  *out = make_layout(T, K, N);
  return I8_OK;
}

i8_status int8_linear_forward(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                              const void* bias, int64_t N, float threshold, void* Y, int32_t* idx, int32_t* n_out,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, Y, idx, n_out, workspace, workspace_bytes, 0, nullptr,
                      stream);
}

i8_status int8_linear_forward_path(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                   const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                   int32_t* n_out, void* workspace, size_t workspace_bytes, int path,
                                   cudaStream_t stream) {
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, Y, idx, n_out, workspace, workspace_bytes, path,
                      nullptr, stream);
}

i8_status int8_linear_forward_timed(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                    const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                    int32_t* n_out, void* workspace, size_t workspace_bytes, int path,
                                    void* const* events, cudaStream_t stream) {
  if (events == nullptr) return I8_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (events[i] == nullptr) return I8_ERR_INVALID_ARG;
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, Y, idx, n_out, workspace, workspace_bytes, path, events,
                      stream);
}

i8_status int8_linear_forward_ex(const void* X, int dtype, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                 const void* bias, int64_t N, float threshold, void* Y, int32_t* idx, int32_t* n_out,
                                 void* workspace, size_t workspace_bytes, int path, void* const* events,
                                 cudaStream_t stream) {
  if (events != nullptr)
    for (int i = 0; i < 4; ++i)
      if (events[i] == nullptr) return I8_ERR_INVALID_ARG;
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, Y, idx, n_out, workspace, workspace_bytes, path, events,
                      stream, dtype);
}

i8_status int8_linear_forward_sharded(const void* X, int dtype, int64_t T, int64_t K, const int8_t* CB,
                                      const float* SCB, const void* bias, int64_t N, float threshold,
                                      void* const* Y_dst, int n_dst, int64_t ldY, int64_t col_offset, int32_t* idx,
                                      int32_t* n_out, void* workspace, size_t workspace_bytes, int path,
                                      cudaStream_t stream) {
  if (Y_dst == nullptr || n_dst < 1 || n_dst > kMaxYDst + 1) return I8_ERR_INVALID_ARG;
  if (ldY < N || ldY % 8 != 0 || col_offset < 0 || col_offset % 8 != 0 || col_offset + N > ldY)
    return I8_ERR_INVALID_ARG;
  void* dst[kMaxYDst + 1];
  for (int d = 0; d < n_dst; ++d) {
    if (Y_dst[d] == nullptr || !aligned(Y_dst[d], 16)) return I8_ERR_INVALID_ARG;
    dst[d] = static_cast<uint8_t*>(Y_dst[d]) + col_offset * 2;
  }
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, dst[0], idx, n_out, workspace, workspace_bytes, path,
                      nullptr, stream, dtype, nullptr, ldY, dst + 1, n_dst - 1);
}

i8_status int8_check_status(void* workspace, uint32_t* where, cudaStream_t stream) {
  if (workspace == nullptr || !aligned(workspace, 256)) return I8_ERR_WORKSPACE;
  if (where != nullptr) *where = 0xffffffffu;  // "the synchronisation itself failed"
  i8_status st = cuda_status(cudaStreamSynchronize(stream));
  if (st != I8_OK) return st;
  DevStatus h;
  st = cuda_status(cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost));
  if (st != I8_OK) return st;
  if (where != nullptr) *where = h.where;
  if (h.error == 0) return I8_OK;
  st = cuda_status(cudaMemset(workspace, 0, 2 * sizeof(uint32_t)));
  if (st != I8_OK) return st;
  if (h.error == kErrTimeout) return I8_ERR_TIMEOUT;
  if (where != nullptr) *where = 0xbad00000u | (h.error & 0xfffffu);  // not a code the kernels write
  return I8_ERR_CUDA;
}

const char* int8_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

// has_fp16_weights=True: the forward's workspace, then CB [N,K] and SCB [N].
size_t int8_linear_fp16w_workspace_bytes(int64_t T, int64_t K, int64_t N) {
  if (!shape_ok(T, K, N)) return 0;
  const int8_ws_layout L = make_layout(T, K, N);
  return static_cast<size_t>(align_up(align_up(L.total + static_cast<uint64_t>(N) * K, 256) + N * 4, 256));
}

i8_status int8_linear_forward_fp16w_ex(const void* X, int dtype, int64_t T, int64_t K, const void* W,
                                       const void* bias, int64_t N, float threshold, void* Y, int32_t* idx,
                                       int32_t* n_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!shape_ok(T, K, N) || !dtype_ok(dtype)) return I8_ERR_INVALID_ARG;
  if (W == nullptr || !aligned(W, 16)) return I8_ERR_INVALID_ARG;
  const int8_ws_layout L = make_layout(T, K, N);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < int8_linear_fp16w_workspace_bytes(T, K, N))
    return I8_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int8_t* CB = reinterpret_cast<int8_t*>(w + L.total);
  float* SCB = reinterpret_cast<float*>(w + align_up(L.total + static_cast<uint64_t>(N) * K, 256));
  int num_sms = 0;
  i8_status st = device_info(&num_sms);
  if (st != I8_OK) return st;
  // the weight is quantised anew in every forward (Linear8bitLt, has_fp16_weights=True)
  const cudaError_t e = launch_quantize_weight(W, dtype, N, K, CB, SCB, stream);
  if (e != cudaSuccess) return cuda_status(e);
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, Y, idx, n_out, workspace, L.total, 0, nullptr, stream,
                      dtype, W);
}

i8_status int8_linear_forward_fp16w(const void* X, int64_t T, int64_t K, const void* W, const void* bias, int64_t N,
                                    float threshold, void* Y, int32_t* idx, int32_t* n_out, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
  return int8_linear_forward_fp16w_ex(X, kF16, T, K, W, bias, N, threshold, Y, idx, n_out, workspace,
                                      workspace_bytes, stream);
}

size_t int8_linear_forward_host_workspace_bytes(int64_t T, int64_t K, int64_t N) {
  if (!shape_ok(T, K, N)) return 0;
  return static_cast<size_t>(make_host_extra(T, K, N).total);
}

// The forward on host buffers: X in, forward, Y (and idx, n_out) out, all
// enqueued on `stream`; `sync` waits and reads the status word.
static i8_status host_forward(const void* X_host, int dtype, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                       const void* bias, int64_t N, float threshold, void* Y_host, int32_t* idx_host,
                       int32_t* n_out_host, void* workspace, size_t workspace_bytes, cudaStream_t stream, bool sync) {
  if (!shape_ok(T, K, N) || !dtype_ok(dtype)) return I8_ERR_INVALID_ARG;
  if (T > 0 && (X_host == nullptr || Y_host == nullptr)) return I8_ERR_INVALID_ARG;
  const HostExtra H = make_host_extra(T, K, N);
  const int8_ws_layout L = make_layout(T, K, N);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < H.total) return I8_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void* Xd = w + H.x;
  void* Yd = w + H.y;
  int32_t* idxd = reinterpret_cast<int32_t*>(w + H.idx);
  int32_t* nd = reinterpret_cast<int32_t*>(w + H.n_out);
  const size_t xbytes = static_cast<size_t>(T) * K * 2;
  const size_t ybytes = static_cast<size_t>(T) * N * 2;
  if (xbytes && cuda_status(cudaMemcpyAsync(Xd, X_host, xbytes, cudaMemcpyHostToDevice, stream)) != I8_OK)
    return I8_ERR_CUDA;
  i8_status st = forward_impl(Xd, T, K, CB, SCB, bias, N, threshold, Yd, idxd, nd, workspace, L.total, 0, nullptr,
                              stream, dtype);
  if (st != I8_OK) return st;
  if (ybytes && cuda_status(cudaMemcpyAsync(Y_host, Yd, ybytes, cudaMemcpyDeviceToHost, stream)) != I8_OK)
    return I8_ERR_CUDA;
  if (idx_host && cuda_status(cudaMemcpyAsync(idx_host, idxd, static_cast<size_t>(K) * 4, cudaMemcpyDeviceToHost,
                                              stream)) != I8_OK)
    return I8_ERR_CUDA;
  if (n_out_host && cuda_status(cudaMemcpyAsync(n_out_host, nd, 4, cudaMemcpyDeviceToHost, stream)) != I8_OK)
    return I8_ERR_CUDA;
  return sync ? int8_check_status(workspace, nullptr, stream) : I8_OK;
}

i8_status int8_linear_forward_host(const void* X_host, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                                   const void* bias, int64_t N, float threshold, void* Y_host, int32_t* idx_host,
                                   int32_t* n_out_host, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
  return host_forward(X_host, kF16, T, K, CB, SCB, bias, N, threshold, Y_host, idx_host, n_out_host, workspace,
                      workspace_bytes, stream, true);
}

i8_status int8_linear_forward_host_async(const void* X_host, int dtype, int64_t T, int64_t K, const int8_t* CB,
                                         const float* SCB, const void* bias, int64_t N, float threshold,
                                         void* Y_host, int32_t* idx_host, int32_t* n_out_host, void* workspace,
                                         size_t workspace_bytes, cudaStream_t stream) {
  return host_forward(X_host, dtype, T, K, CB, SCB, bias, N, threshold, Y_host, idx_host, n_out_host, workspace,
                      workspace_bytes, stream, false);
}

i8_status int8_gemm_i32(const int8_t* Xq, int64_t T, int64_t K, const int8_t* CB, int64_t N, int32_t* acc, int path,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!shape_ok(T, K, N) || path < kPathAuto || path > kPathTensorCoreSingleSM) return I8_ERR_INVALID_ARG;
  if (path == kPathDecode && T > kDecodeMaxT) return I8_ERR_INVALID_ARG;
  if (T > 0 && (Xq == nullptr || CB == nullptr || acc == nullptr)) return I8_ERR_INVALID_ARG;
  if (T > 0 && (!aligned(Xq, 16) || !aligned(CB, 16) || !aligned(acc, 16))) return I8_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < sizeof(DevStatus)) return I8_ERR_WORKSPACE;
  int num_sms = 0;
  i8_status st = device_info(&num_sms);
  if (st != I8_OK) return st;
  if (cuda_status(cudaMemsetAsync(workspace, 0, sizeof(DevStatus), stream)) != I8_OK) return I8_ERR_CUDA;
  if (T == 0) return I8_OK;
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.Xq = Xq;
  a.CB = CB;
  a.acc_out = acc;
  a.st = static_cast<DevStatus*>(workspace);
  a.T = T;
  a.N = N;
  a.K = K;
  a.mode = 1;
  const bool gemv = (path == kPathDecode) || (path == kPathAuto && T <= kDecodeMaxT);
  return cuda_status(launch_product(a, path, gemv, num_sms, stream));
}

}  // extern "C"
