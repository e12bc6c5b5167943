// Decode-path forward whose scratch memory is a fixed array compiled into the
// library, for callers that cannot allocate device memory.
//
// Who needs it: a host runtime that owns all device memory and forbids
// allocation inside its execute/enqueue call (a plugin of an inference server
// or engine), or an application running under a fixed device-memory budget.
// For them cudaMalloc is not an option -- it may synchronise the device and it
// bypasses the host's memory accounting -- and they may not be able to hand us
// a workspace either.  This entry point needs nothing but its inputs and
// outputs: the intermediate buffers of the forward (status word, outlier
// bitmask, row scales, int8 row codes, fp16 outlier columns) live in
// `g_scratch` below, a file-scope device array of kScratchBytes (4 MiB) that
// every GPU which loads this library keeps until the process exits.
//
// It runs the same kernels as int8_linear_forward's decode path (T <= 16).
#include <mutex>

#include "int8mp.h"
#include "kernels.h"

using namespace i8mp;

namespace {

constexpr uint64_t kScratchBytes = 4ull << 20;
static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};

inline uint64_t up256(uint64_t v) { return (v + 255) / 256 * 256; }

struct StaticLayout {
  uint64_t status, mask, sA, Xq, Xo, total;
  int64_t ldo;
};

StaticLayout static_layout(int64_t T, int64_t K) {
  StaticLayout L;
  L.ldo = ((K + 63) / 64) * 64;
  L.status = 0;
  L.mask = 256;
  L.sA = up256(L.mask + static_cast<uint64_t>((K + 31) / 32) * 8);  // mask words + prefix counts
  L.Xq = up256(L.sA + static_cast<uint64_t>(T) * 4);
  L.Xo = up256(L.Xq + static_cast<uint64_t>(T) * K);
  L.total = up256(L.Xo + static_cast<uint64_t>(T) * L.ldo * 2);
  return L;
}

// Device address of g_scratch on the current device, resolved once per device
// with that device current.  Host code must not use `g_scratch` itself: on the
// host it names a stand-in object, not device memory.  The same first call
// also does the decode kernels' own once-per-device set-up for every T in
// 1..16, so that no later call makes a CUDA call other than the launches.
i8_status scratch_for_current_device(void** addr, int* num_sms) {
  int dev = 0;
  if (note_cuda_error(cudaGetDevice(&dev)) != cudaSuccess) return I8_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return I8_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    int major = 0, sms = 0;
    if (note_cuda_error(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return I8_ERR_CUDA;
    if (major != 10) return I8_ERR_UNSUPPORTED;
    if (note_cuda_error(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return I8_ERR_CUDA;
    void* p = nullptr;
    if (note_cuda_error(cudaGetSymbolAddress(&p, g_scratch)) != cudaSuccess || p == nullptr) return I8_ERR_CUDA;
    if (note_cuda_error(prepare_prep_small(kF16)) != cudaSuccess) return I8_ERR_CUDA;
    prepare_gemv_decode();
    g_num_sms[dev] = sms;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
  return I8_OK;
}

}  // namespace

extern "C" i8_status int8_linear_forward_decode_static(const void* X, int64_t T, int64_t K, const int8_t* CB,
                                                       const float* SCB, const void* bias, int64_t N,
                                                       float threshold, void* Y, int32_t* idx, int32_t* n_out,
                                                       cudaStream_t stream) {
  if (T < 1 || T > kDecodeMaxT || K < 16 || K % 16 != 0 || K > 131072 || N < 16 || N % 16 != 0 ||
      N > (int64_t(1) << 30))
    return I8_ERR_INVALID_ARG;
  if (X == nullptr || CB == nullptr || SCB == nullptr || Y == nullptr || idx == nullptr || n_out == nullptr)
    return I8_ERR_INVALID_ARG;
  auto al = [](const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; };
  if (!al(X, 16) || !al(CB, 16) || !al(Y, 16) || !al(SCB, 4) || !al(idx, 4) || !al(n_out, 4) ||
      (bias != nullptr && !al(bias, 2)))
    return I8_ERR_INVALID_ARG;
  const StaticLayout L = static_layout(T, K);
  if (L.total > kScratchBytes) return I8_ERR_WORKSPACE;  // this T x K needs more than the fixed scratch

  void* base = nullptr;
  int num_sms = 0;
  i8_status st = scratch_for_current_device(&base, &num_sms);
  if (st != I8_OK) return st;
  uint8_t* w = static_cast<uint8_t*>(base);

  // The scratch keeps whatever the previous call left; the prep kernel
  // rebuilds the outlier bitmask from scratch and clears the status word.
  DevStatus* dst = reinterpret_cast<DevStatus*>(w + L.status);
  uint32_t* mask = reinterpret_cast<uint32_t*>(w + L.mask);
  float* sA = reinterpret_cast<float*>(w + L.sA);
  int8_t* Xq = reinterpret_cast<int8_t*>(w + L.Xq);
  void* Xo = w + L.Xo;

  const uint32_t hb = int8_outlier_threshold_bits(threshold);
  const cudaError_t e = launch_prep_small(X, kF16, T, K, hb, mask, mask + (K + 31) / 32, idx, n_out, Xq, sA, Xo,
                                          L.ldo, dst, stream);
  if (note_cuda_error(e) != cudaSuccess) return I8_ERR_CUDA;

  GemmArgs a;
  a.Xq = Xq;
  a.CB = CB;
  a.Xo = Xo;
  a.Wo = nullptr;
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
  a.pdl = true;  // follows the prep kernel
  return note_cuda_error(launch_gemv_decode(a, num_sms, stream)) == cudaSuccess ? I8_OK : I8_ERR_CUDA;
}
