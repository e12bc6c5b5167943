// Persistence of a quantised layer: CB, SCB (and the bias) in one byte image,
// so that an int8 layer can be stored and loaded without the fp16 weight and
// without quantising again.  The Hugging Face integration page lists the
// missing quantisation statistics (CB, SCB) in INT8 checkpoints under "Future
// work and limitations".  Host-only code: no CUDA call is made here.
//
// Image layout (little-endian, as written by an x86-64 or arm64 host):
//   offset  0  char[8]   magic "I8MPLYR1"
//   offset  8  int64     N (output features)
//   offset 16  int64     K (input features)
//   offset 24  uint32    flags (bit 0: a bias follows SCB; bit 1: the bias is
//                        bf16, else fp16)
//   offset 28  uint32    reserved (0)
//   offset 32  float32   SCB[N]
//   then       16-bit    bias[N]            (only when flags bit 0 is set)
//   then       int8      CB[N*K], row-major
#include <cstring>

#include "int8mp.h"

namespace {

constexpr char kMagic[8] = {'I', '8', 'M', 'P', 'L', 'Y', 'R', '1'};
constexpr size_t kHeader = 32;

bool shape_ok(int64_t N, int64_t K) {
  return N >= 16 && N % 16 == 0 && N <= (int64_t(1) << 30) && K >= 16 && K % 16 == 0 && K <= 131072;
}

size_t packed_bytes(int64_t N, int64_t K, bool bias) {
  return kHeader + static_cast<size_t>(N) * 4 + (bias ? static_cast<size_t>(N) * 2 : 0) +
         static_cast<size_t>(N) * static_cast<size_t>(K);
}

}  // namespace

extern "C" {

size_t int8_layer_packed_bytes(int64_t N, int64_t K, int has_bias) {
  if (!shape_ok(N, K)) return 0;
  return packed_bytes(N, K, has_bias != 0);
}

i8_status int8_layer_pack_ex(const int8_t* CB, const float* SCB, const void* bias, int bias_dtype, int64_t N,
                             int64_t K, void* out, size_t out_bytes) {
  if (!shape_ok(N, K) || CB == nullptr || SCB == nullptr || out == nullptr) return I8_ERR_INVALID_ARG;
  if (bias_dtype != I8_DTYPE_F16 && bias_dtype != I8_DTYPE_BF16) return I8_ERR_INVALID_ARG;
  const bool has_bias = bias != nullptr;
  if (out_bytes < packed_bytes(N, K, has_bias)) return I8_ERR_WORKSPACE;
  uint8_t* o = static_cast<uint8_t*>(out);
  std::memcpy(o, kMagic, 8);
  std::memcpy(o + 8, &N, 8);
  std::memcpy(o + 16, &K, 8);
  const uint32_t flags = has_bias ? (1u | (bias_dtype == I8_DTYPE_BF16 ? 2u : 0u)) : 0u, reserved = 0;
  std::memcpy(o + 24, &flags, 4);
  std::memcpy(o + 28, &reserved, 4);
  size_t off = kHeader;
  std::memcpy(o + off, SCB, static_cast<size_t>(N) * 4);
  off += static_cast<size_t>(N) * 4;
  if (has_bias) {
    std::memcpy(o + off, bias, static_cast<size_t>(N) * 2);
    off += static_cast<size_t>(N) * 2;
  }
  std::memcpy(o + off, CB, static_cast<size_t>(N) * static_cast<size_t>(K));
  return I8_OK;
}

i8_status int8_layer_pack(const int8_t* CB, const float* SCB, const void* bias, int64_t N, int64_t K, void* out,
                          size_t out_bytes) {
  return int8_layer_pack_ex(CB, SCB, bias, I8_DTYPE_F16, N, K, out, out_bytes);
}

i8_status int8_layer_unpack_header_ex(const void* buf, size_t bytes, int64_t* N, int64_t* K, int* has_bias,
                                      int* bias_dtype) {
  if (buf == nullptr || bytes < kHeader || N == nullptr || K == nullptr || has_bias == nullptr)
    return I8_ERR_INVALID_ARG;
  const uint8_t* b = static_cast<const uint8_t*>(buf);
  if (std::memcmp(b, kMagic, 8) != 0) return I8_ERR_INVALID_ARG;
  int64_t n, k;
  uint32_t flags, reserved;
  std::memcpy(&n, b + 8, 8);
  std::memcpy(&k, b + 16, 8);
  std::memcpy(&flags, b + 24, 4);
  std::memcpy(&reserved, b + 28, 4);
  if (!shape_ok(n, k) || (flags & ~3u) != 0 || flags == 2u || reserved != 0) return I8_ERR_INVALID_ARG;
  if (bytes < packed_bytes(n, k, (flags & 1u) != 0)) return I8_ERR_INVALID_ARG;
  *N = n;
  *K = k;
  *has_bias = static_cast<int>(flags & 1u);
  if (bias_dtype != nullptr) *bias_dtype = (flags & 2u) ? I8_DTYPE_BF16 : I8_DTYPE_F16;
  return I8_OK;
}

i8_status int8_layer_unpack_header(const void* buf, size_t bytes, int64_t* N, int64_t* K, int* has_bias) {
  return int8_layer_unpack_header_ex(buf, bytes, N, K, has_bias, nullptr);
}

i8_status int8_layer_unpack(const void* buf, size_t bytes, int8_t* CB, float* SCB, void* bias) {
  int64_t N = 0, K = 0;
  int has_bias = 0;
  const i8_status st = int8_layer_unpack_header(buf, bytes, &N, &K, &has_bias);
  if (st != I8_OK) return st;
  if (CB == nullptr || SCB == nullptr) return I8_ERR_INVALID_ARG;
  const uint8_t* b = static_cast<const uint8_t*>(buf);
  size_t off = kHeader;
  std::memcpy(SCB, b + off, static_cast<size_t>(N) * 4);
  off += static_cast<size_t>(N) * 4;
  if (has_bias) {
    if (bias != nullptr) std::memcpy(bias, b + off, static_cast<size_t>(N) * 2);
    off += static_cast<size_t>(N) * 2;
  }
  std::memcpy(CB, b + off, static_cast<size_t>(N) * static_cast<size_t>(K));
  return I8_OK;
}

}  // extern "C"
