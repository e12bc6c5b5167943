// Plain C++17 CPU oracle of the LLM.int8() forward linear layer -- TEST
// INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
// baseline of bench.py load it (through oracle/cpp.py); it shares no code,
// header or table with the CUDA library, and includes nothing of it.
//
// Each function restates one step of the method as the pages describe it,
// with plain loops: no intrinsics, no fast-math, no FMA contraction (built
// with -ffp-contract=off), so every fp32 and fp64 operation is one IEEE
// operation in source order.
//
//  * "Hugging Face integrates LLM.int8() ... into Transformers and
//    Accelerate", "Core idea of LLM.int8()": (1) the outlier columns of the
//    hidden state, (2) vector-wise int8 product of the rest (row-wise for the
//    activations, one constant per output feature for the weights) and a 16-bit
//    product of the outlier columns, (3) dequantise and add up.
//  * same page, "Quantization mechanics": absmax scaling by 127/absmax to codes
//    in [-127, 127]; "Integration into transformers": W is recovered as
//    CB * SCB / 127.
//  * bitsandbytes Linear8bitLt docstring, `threshold`: activation columns in
//    which some value exceeds the threshold go through the 16-bit product.
//  * bitsandbytes issue #1609: state.idx is the ascending list of those columns.
//
// Readings where the pages are silent (the same ones the numpy oracle takes):
// threshold <= 0 or NaN switches the decomposition off; "exceeds" is strict;
// one token is enough to flag a column for all tokens; the row absmax runs
// over the non-outlier columns; codes are roundf(x * fp32(127/absmax)) with
// ties away from zero, clamped to +-127; a zero absmax gives zero codes; SCB
// holds the fp32 absmax; the outlier weights are the 16-bit rounding (nearest,
// ties to even) of the fp32 value (CB * SCB) / 127; Y is computed in fp64.
//
// 16-bit values travel as bit patterns (uint16_t) with an element-type
// argument: 0 = IEEE binary16 (fp16), 1 = bfloat16 (the upper half of a
// binary32 pattern).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// 16-bit formats, from their definitions
// ---------------------------------------------------------------------------

// fp16: 1 sign bit, 5 exponent bits (bias 15), 10 stored mantissa bits.
float fp16_value(uint16_t h) {
  const int e = (h >> 10) & 0x1f;
  const int m = h & 0x3ff;
  float v;
  if (e == 0)
    v = std::ldexp(static_cast<float>(m), -24);  // subnormal: m * 2^-24
  else if (e == 31)
    v = m == 0 ? INFINITY : NAN;
  else
    v = std::ldexp(static_cast<float>(m + 1024), e - 25);  // (1024 + m) * 2^(e - 15 - 10)
  return (h & 0x8000) ? -v : v;
}

// bf16: the upper 16 bits of the binary32 pattern.
float bf16_value(uint16_t h) {
  const uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

float value16(uint16_t h, int elem) { return elem == 1 ? bf16_value(h) : fp16_value(h); }

// The nearest value of a binary format with `mb` stored mantissa bits and `eb`
// exponent bits, ties to the even significand; magnitudes that round past the
// largest finite value become infinity.  Works on the exact fp64 widening.
uint16_t narrow16(float f, int mb, int eb) {
  const int bias = (1 << (eb - 1)) - 1;
  const uint16_t sign = std::signbit(f) ? 0x8000 : 0;
  const uint16_t exp_all = static_cast<uint16_t>(((1 << eb) - 1) << mb);
  if (std::isnan(f)) return static_cast<uint16_t>(exp_all | (1 << (mb - 1)));  // quiet NaN
  const double a = std::fabs(static_cast<double>(f));
  if (std::isinf(a)) return sign | exp_all;
  if (a == 0.0) return sign;
  int e = 0;
  (void)std::frexp(a, &e);
  e -= 1;                                  // a in [2^e, 2^(e+1))
  const int emin = 1 - bias;               // exponent of the smallest normal value
  if (e < emin) e = emin;                  // subnormals share the smallest normal's quantum
  const double quantum = std::ldexp(1.0, e - mb);
  const double q = a / quantum;            // exact: division by a power of two
  double n = std::floor(q);
  const double r = q - n;
  if (r > 0.5 || (r == 0.5 && std::fmod(n, 2.0) != 0.0)) n += 1.0;
  int E = e;
  if (n >= std::ldexp(1.0, mb + 1)) {      // rounding carried into the next binade
    n /= 2.0;
    E += 1;
  }
  if (E > bias) return sign | exp_all;     // overflow: infinity
  const double lead = std::ldexp(1.0, mb);
  if (n < lead) return static_cast<uint16_t>(sign | static_cast<uint16_t>(n));  // subnormal (E == emin)
  const uint32_t field = static_cast<uint32_t>(E + bias);
  const uint32_t mant = static_cast<uint32_t>(n - lead);
  return static_cast<uint16_t>(sign | (field << mb) | mant);
}

uint16_t round16(float f, int elem) { return elem == 1 ? narrow16(f, 7, 8) : narrow16(f, 10, 5); }

// ---------------------------------------------------------------------------
// threads over independent rows
// ---------------------------------------------------------------------------

template <typename F>
void parallel_rows(int64_t rows, int nthreads, F body) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > rows) nthreads = static_cast<int>(rows < 1 ? 1 : rows);
  if (nthreads == 1) {
    for (int64_t r = 0; r < rows; ++r) body(r);
    return;
  }
  std::vector<std::thread> pool;
  for (int i = 0; i < nthreads; ++i)
    pool.emplace_back([=]() {
      for (int64_t r = i; r < rows; r += nthreads) body(r);
    });
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------------
// absmax quantisation ("Quantization mechanics")
// ---------------------------------------------------------------------------

// Code of x for a row whose absmax is `am`: one fp32 division 127/am, one
// fp32 multiplication, round half away from zero (std::round), clamp.
int8_t absmax_code(float x, float am) {
  if (!(am > 0.0f)) return 0;
  const float inv = 127.0f / am;
  const float y = x * inv;
  float q = std::round(y);
  if (q > 127.0f) q = 127.0f;
  if (q < -127.0f) q = -127.0f;
  return static_cast<int8_t>(q);
}

}  // namespace

extern "C" {

int oref_version(void) { return 1; }

// 16-bit patterns -> fp32 values (exact).
void oref_to_f32(const uint16_t* in, int64_t n, int elem, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = value16(in[i], elem);
}

// fp32 values -> nearest 16-bit patterns (ties to even).
void oref_from_f32(const float* in, int64_t n, int elem, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round16(in[i], elem);
}

// a0: SCB[j] = max_k |W[j,k]|; CB[j,k] = code of W[j,k] for absmax SCB[j].
void oref_quantize_weight(const uint16_t* W, int64_t N, int64_t K, int elem, int8_t* CB, float* SCB, int nthreads) {
  parallel_rows(N, nthreads, [&](int64_t j) {
    float am = 0.0f;
    for (int64_t k = 0; k < K; ++k) am = std::fmax(am, std::fabs(value16(W[j * K + k], elem)));
    SCB[j] = am;
    for (int64_t k = 0; k < K; ++k) CB[j * K + k] = absmax_code(value16(W[j * K + k], elem), am);
  });
}

// a1: mask[k] = 1 iff some |X[t,k]| > threshold (threshold > 0).
void oref_outlier_mask(const uint16_t* X, int64_t T, int64_t K, int elem, float threshold, uint8_t* mask) {
  for (int64_t k = 0; k < K; ++k) mask[k] = 0;
  if (!(threshold > 0.0f)) return;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t k = 0; k < K; ++k)
      if (std::fabs(value16(X[t * K + k], elem)) > threshold) mask[k] = 1;
}

// a2: the flagged columns in ascending order; returns their number.
int64_t oref_outlier_index(const uint8_t* mask, int64_t K, int32_t* idx) {
  int64_t n = 0;
  for (int64_t k = 0; k < K; ++k)
    if (mask[k]) idx[n++] = static_cast<int32_t>(k);
  return n;
}

// a3: sA[t] = max over non-outlier k of |X[t,k]|; Xq[t,k] = code (0 in outlier columns).
void oref_quantize_rows(const uint16_t* X, int64_t T, int64_t K, int elem, const uint8_t* mask, int8_t* Xq,
                        float* sA, int nthreads) {
  parallel_rows(T, nthreads, [&](int64_t t) {
    float am = 0.0f;
    for (int64_t k = 0; k < K; ++k)
      if (!mask[k]) am = std::fmax(am, std::fabs(value16(X[t * K + k], elem)));
    sA[t] = am;
    for (int64_t k = 0; k < K; ++k)
      Xq[t * K + k] = mask[k] ? 0 : absmax_code(value16(X[t * K + k], elem), am);
  });
}

// a4: Xo[t,o] = X[t, idx[o]] (unchanged); Wo[j,o] = 16-bit((CB[j,idx[o]] * SCB[j]) / 127).
void oref_outlier_operands(const uint16_t* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB, int64_t N,
                           const int32_t* idx, int64_t n_out, int elem, uint16_t* Xo, uint16_t* Wo) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t o = 0; o < n_out; ++o) Xo[t * n_out + o] = X[t * K + idx[o]];
  for (int64_t j = 0; j < N; ++j)
    for (int64_t o = 0; o < n_out; ++o) {
      const float p = static_cast<float>(CB[j * K + idx[o]]) * SCB[j];
      Wo[j * n_out + o] = round16(p / 127.0f, elem);
    }
}

// a5: acc[t,j] = sum_k Xq[t,k] * CB[j,k], exact (int64 sum; |acc| <= K * 127^2).
void oref_int8_matmul(const int8_t* Xq, int64_t T, int64_t K, const int8_t* CB, int64_t N, int32_t* acc,
                      int nthreads) {
  parallel_rows(T, nthreads, [&](int64_t t) {
    for (int64_t j = 0; j < N; ++j) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += static_cast<int64_t>(Xq[t * K + k]) * static_cast<int64_t>(CB[j * K + k]);
      acc[t * N + j] = static_cast<int32_t>(s);
    }
  });
}

// a7: Y[t,j] = acc * sA[t] * SCB[j] / 127^2 + sum_o Xo[t,o] * Wo[j,o] + bias[j], in fp64.
void oref_combine(const int32_t* acc, const float* sA, const float* SCB, const uint16_t* Xo, const uint16_t* Wo,
                  int64_t n_out, const uint16_t* bias, int elem, int64_t T, int64_t N, double* Y, int nthreads) {
  parallel_rows(T, nthreads, [&](int64_t t) {
    for (int64_t j = 0; j < N; ++j) {
      double y = static_cast<double>(acc[t * N + j]) * static_cast<double>(sA[t]) * static_cast<double>(SCB[j]);
      y = y / 16129.0;
      double o = 0.0;
      for (int64_t i = 0; i < n_out; ++i)
        o += static_cast<double>(value16(Xo[t * n_out + i], elem)) * static_cast<double>(value16(Wo[j * n_out + i], elem));
      y = y + o;
      if (bias != nullptr) y = y + static_cast<double>(value16(bias[j], elem));
      Y[t * N + j] = y;
    }
  });
}

}  // extern "C"
