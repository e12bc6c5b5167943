// Internal launcher declarations of libint8mp (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace i8mp {

// Weight quantisation: W fp16 [N,K] -> CB int8 [N,K], SCB fp32 [N].
cudaError_t launch_quantize_weight(const __half* W, int64_t N, int64_t K, int8_t* CB, float* SCB,
                                   cudaStream_t s);

// Column outlier mask (atomicOr into a zeroed mask) followed, in the last CTA
// to finish, by compaction into the ascending idx list and n_out.
// `hbits` is the largest fp16 magnitude bit pattern whose value is <= threshold.
// Also writes prefix[w] = number of outlier columns in mask words 0..w-1.
cudaError_t launch_outliers(const __half* X, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                            uint32_t* prefix, int32_t* idx, int32_t* n_out, DevStatus* st, cudaStream_t s);

// Row-wise absmax int8 quantisation over non-outlier columns, fp16 gather of
// the outlier activation columns into Xo, and (when `with_wo`) the gather and
// dequantisation of the matching weight columns into Wo -- or, when `Wf` (the
// fp16 weight of a has_fp16_weights=True layer) is given, its own columns.
// `pdl`: launch with programmatic stream serialisation (only when the previous
// operation in the stream is the outlier-pass kernel).
cudaError_t launch_rowquant(const __half* X, int64_t T, int64_t K, const uint32_t* mask, const uint32_t* prefix,
                            const int32_t* idx, const int32_t* n_out, int8_t* Xq, float* sA, __half* Xo,
                            int64_t ldo, const int8_t* CB, const float* SCB, int64_t N, __half* Wo, bool with_wo,
                            const __half* Wf, int num_sms, DevStatus* st, bool pdl, cudaStream_t s);

struct GemmArgs {
  const int8_t* Xq;      // [T,K]
  const int8_t* CB;      // [N,K]
  const __half* Xo;      // [T,ldo] (may be null when no outliers are possible)
  const __half* Wo;      // [N,ldo]
  int64_t ldo;
  const float* sA;       // [T]
  const float* SCB;      // [N]
  const __half* bias;    // [N] or null
  __half* Y;             // [T,N] fp16 output (mode 0)
  int32_t* acc_out;      // [T,N] raw int32 accumulators (mode 1)
  const int32_t* n_out;  // device count of outlier columns, or null (= 0)
  const int32_t* idx;    // ascending outlier columns (decode path)
  DevStatus* st;
  int64_t T, N, K;
  int mode;              // 0: fused fp16 Y, 1: int32 accumulators only
  bool pdl = false;      // launch with programmatic stream serialisation (previous op is our kernel)
  const __half* Wf = nullptr;  // fp16 weight [N,K] (has_fp16_weights=True): outlier weights come from it
};

// Prefill: persistent tcgen05 kind::i8 GEMM with TMEM accumulators, fused
// kind::f16 outlier product and dequant/bias epilogue.
cudaError_t launch_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t s);

// Prefill, pair-of-SMs version: 2-CTA clusters, tcgen05.mma.cta_group::2 with
// 256 x 256 tiles.  Returns cudaErrorNotSupported if such clusters cannot be
// launched on the current device.
cudaError_t launch_gemm_tc2(const GemmArgs& a, cudaStream_t s);
int pair_kernel_max_clusters();

// Decode (T <= 16): weight-streaming int8 GEMV on mma.sync with the outlier
// columns dequantised from CB in the epilogue.
cudaError_t launch_gemv_decode(const GemmArgs& a, int num_sms, cudaStream_t s);

constexpr int kDecodeMaxT = 16;

// Product-kernel choice (the `path` argument of the C ABI).
enum Path : int { kPathAuto = 0, kPathTensorCore = 1, kPathDecode = 2, kPathTensorCoreSingleSM = 3 };

}  // namespace i8mp
