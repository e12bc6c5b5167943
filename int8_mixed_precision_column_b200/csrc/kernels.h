// Internal launcher declarations of libint8mp (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace i8mp {

// Element type of the 16-bit operands (X, Xo, Wo, bias, Y, Wf): `dtype` is a
// DType (kF16 or kBF16) throughout.

// Weight quantisation: W [N,K] (16-bit) -> CB int8 [N,K], SCB fp32 [N].
cudaError_t launch_quantize_weight(const void* W, int dtype, int64_t N, int64_t K, int8_t* CB, float* SCB,
                                   cudaStream_t s);

// Column outlier mask (atomicOr into a zeroed mask) followed, in the last CTA
// to finish, by compaction into the ascending idx list and n_out.
// `hbits` is the largest magnitude bit pattern of the element type whose value
// is <= threshold.  Also writes prefix[w] = number of outlier columns in mask
// words 0..w-1.
cudaError_t launch_outliers(const void* X, int dtype, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                            uint32_t* prefix, int32_t* idx, int32_t* n_out, DevStatus* st, cudaStream_t s);

// Row-wise absmax int8 quantisation over non-outlier columns, 16-bit gather of
// the outlier activation columns into Xo, and (when `with_wo`) the gather and
// dequantisation of the matching weight columns into Wo -- or, when `Wf` (the
// 16-bit weight of a has_fp16_weights=True layer) is given, its own columns.
// `pdl`: launch with programmatic stream serialisation (only when the previous
// operation in the stream is the outlier-pass kernel).
cudaError_t launch_rowquant(const void* X, int dtype, int64_t T, int64_t K, const uint32_t* mask,
                            const uint32_t* prefix, const int32_t* idx, const int32_t* n_out, int8_t* Xq, float* sA,
                            void* Xo, int64_t ldo, const int8_t* CB, const float* SCB, int64_t N, void* Wo,
                            bool with_wo, const void* Wf, int num_sms, DevStatus* st, bool pdl, cudaStream_t s);

// Extra destinations of Y besides `Y` itself: the same [T, ldY] buffer on the
// other GPUs of an N-sharded layer (peer-mapped), so that one kernel computes
// its column block and stores it everywhere.
constexpr int kMaxYDst = 7;

// Kernel-side view of the output layout: row stride and extra destinations.
struct YDst {
  int64_t ld;          // row stride of Y in elements
  int n;               // number of extra destinations (0..kMaxYDst)
  void* p[kMaxYDst];
};

// Store one 16-byte vector at element offset `off` of every extra destination
// (the loop is unrolled so every index is a constant).
template <typename TE>
__device__ __forceinline__ void store_extra_u4(const YDst& y, int64_t off, const uint4& v) {
  #pragma unroll
  for (int d = 0; d < kMaxYDst; ++d)
    if (d < y.n) *reinterpret_cast<uint4*>(static_cast<TE*>(y.p[d]) + off) = v;
}
template <typename TE>
__device__ __forceinline__ void store_extra(const YDst& y, int64_t off, TE v) {
  #pragma unroll
  for (int d = 0; d < kMaxYDst; ++d)
    if (d < y.n) static_cast<TE*>(y.p[d])[off] = v;
}

// Decode prep (1 <= T <= kDecodeMaxT, product by the decode GEMV): outlier
// mask, idx, n_out and row quantisation in one kernel, one CTA per row; also
// clears the status word.  hbits == 0xffffffff: no outliers.  No Wo.
cudaError_t launch_prep_small(const void* X, int dtype, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                              uint32_t* prefix, int32_t* idx, int32_t* n_out, int8_t* Xq, float* sA, void* Xo,
                              int64_t ldo, DevStatus* st, cudaStream_t s);

struct GemmArgs {
  const int8_t* Xq;      // [T,K]
  const int8_t* CB;      // [N,K]
  const void* Xo;        // [T,ldo] 16-bit (may be null when no outliers are possible)
  const void* Wo;        // [N,ldo] 16-bit
  int64_t ldo;
  const float* sA;       // [T]
  const float* SCB;      // [N]
  const void* bias;      // [N] 16-bit, or null
  void* Y;               // [T,N] 16-bit output (mode 0)
  int32_t* acc_out;      // [T,N] raw int32 accumulators (mode 1)
  const int32_t* n_out;  // device count of outlier columns, or null (= 0)
  const int32_t* idx;    // ascending outlier columns (decode path)
  DevStatus* st;
  int64_t T, N, K;
  int mode;              // 0: fused 16-bit Y, 1: int32 accumulators only
  bool pdl = false;      // launch with programmatic stream serialisation (previous op is our kernel)
  const void* Wf = nullptr;  // 16-bit weight [N,K] (has_fp16_weights=True): outlier weights come from it
  int dtype = kF16;          // element type of Xo, Wo, bias, Y, Wf
  int64_t ldY = 0;           // row stride of Y (and of every ydst) in elements; 0 means N
  int n_ydst = 0;            // number of extra destinations in ydst (0..kMaxYDst)
  void* ydst[kMaxYDst] = {};  // extra copies of Y (mode 0 only), same layout and column offset
};

inline YDst make_ydst(const GemmArgs& a) {
  YDst y;
  y.ld = a.ldY > 0 ? a.ldY : a.N;
  y.n = a.n_ydst;
  for (int d = 0; d < kMaxYDst; ++d) y.p[d] = d < a.n_ydst ? a.ydst[d] : nullptr;
  return y;
}

// Prefill: persistent tcgen05 kind::i8 GEMM with TMEM accumulators, fused
// kind::f16 outlier product and dequant/bias epilogue.
cudaError_t launch_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t s);

// Prefill, pair-of-SMs version: 2-CTA clusters, two tcgen05.mma.cta_group::2
// of 256 x 256 per K-step for a 256 x 512 tile.  Returns
// cudaErrorNotSupported if such clusters cannot be launched on the current
// device.
cudaError_t launch_gemm_tc2(const GemmArgs& a, cudaStream_t s);
int pair_kernel_max_clusters();

// Decode (T <= 16): weight-streaming int8 GEMV on mma.sync with the outlier
// columns dequantised from CB in the epilogue.
cudaError_t launch_gemv_decode(const GemmArgs& a, int num_sms, cudaStream_t s);

constexpr int kDecodeMaxT = 16;

// The per-device, per-process set-up the decode kernels otherwise do at their
// first launch with a given T: whether the prep kernel's T-CTA cluster can be
// scheduled (T = 2..kDecodeMaxT, element type `dtype`) and the GEMV's
// shared-memory carveout hint.  Afterwards their launchers make no CUDA call
// besides cudaGetDevice and the launch itself.
cudaError_t prepare_prep_small(int dtype);
void prepare_gemv_decode();

// Remembers a failed CUDA result for int8_last_cuda_error() (this host
// thread) and returns it unchanged.
cudaError_t note_cuda_error(cudaError_t e);

// Product-kernel choice (the `path` argument of the C ABI).
enum Path : int { kPathAuto = 0, kPathTensorCore = 1, kPathDecode = 2, kPathTensorCoreSingleSM = 3 };

}  // namespace i8mp
