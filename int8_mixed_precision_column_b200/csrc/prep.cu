// Memory-bound stages of the LLM.int8() forward linear layer:
//  * weight absmax quantisation (CB int8, SCB fp32), done once per layer;
//  * the column outlier mask and its compaction into the ascending index list;
//  * row-wise absmax int8 quantisation of the non-outlier activations, and the
//    gathers that feed the 16-bit outlier product.
// Every kernel is a template over the 16-bit element type (fp16 or bf16; the
// bitsandbytes Linear8bitLt docstring speaks of "fp16 / bf16 weights").
//
// Method: "Hugging Face integrates LLM.int8() 8-bit matrix multiplication into
// Transformers and Accelerate", sections "Core idea of LLM.int8()" (steps 1-2)
// and "Quantization mechanics" (absmax, 127/absmax, codes in [-127, 127]);
// bitsandbytes Linear8bitLt docstring (threshold acts on activation columns);
// bitsandbytes issue #1609 (state.idx lists the outlier columns).
#include "kernels.h"

namespace i8mp {

// ---------------------------------------------------------------------------
// Weight quantisation: one warp per output row j.
// SCB[j] = max_k |W[j,k]|; CB[j,k] = clamp(roundf(W[j,k] * (127/SCB[j])), +-127).
// ---------------------------------------------------------------------------
template <typename TE>
__global__ void __launch_bounds__(256) quantize_weight_kernel(const TE* __restrict__ W, int64_t N, int64_t K,
                                                              int8_t* __restrict__ CB, float* __restrict__ SCB) {
  using E = Elem<TE>;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int64_t nv = K / 8;
  const uint4* src = reinterpret_cast<const uint4*>(W + row * K);
  float m = 0.0f;
  for (int64_t i = lane; i < nv; i += 32) {
    uint4 v = __ldg(src + i);
    const TE* h = reinterpret_cast<const TE*>(&v);
    #pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(E::to_float(h[e])));
  }
  m = warp_max(m);
  const float inv = scale_inv(m);
  if (lane == 0) SCB[row] = m;
  uint2* dst = reinterpret_cast<uint2*>(CB + row * K);
  for (int64_t i = lane; i < nv; i += 32) {
    uint4 v = __ldg(src + i);
    const TE* h = reinterpret_cast<const TE*>(&v);
    uint32_t lo = 0, hi = 0;
    #pragma unroll
    for (int e = 0; e < 4; ++e) lo |= (static_cast<uint32_t>(quant_code(E::to_float(h[e]), inv)) & 0xffu) << (8 * e);
    #pragma unroll
    for (int e = 0; e < 4; ++e)
      hi |= (static_cast<uint32_t>(quant_code(E::to_float(h[4 + e]), inv)) & 0xffu) << (8 * e);
    dst[i] = make_uint2(lo, hi);
  }
}

cudaError_t launch_quantize_weight(const void* W, int dtype, int64_t N, int64_t K, int8_t* CB, float* SCB,
                                   cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((N + 7) / 8);
  if (dtype == kBF16)
    quantize_weight_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(W), N, K, CB, SCB);
  else
    quantize_weight_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), N, K, CB, SCB);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Column outlier mask.
//
// Each thread owns 8 consecutive columns (one 16-byte load per row) and ORs
// together, over its rows, the bits "|x| > threshold".  The comparison is done
// on 16-bit magnitude bit patterns: for non-NaN fp16 or bf16 values the
// magnitude order equals the order of the 15-bit patterns, so |x| > threshold
// <=> (bits & 0x7fff) > hbits, where hbits is the largest pattern whose value
// is <= threshold (computed on the host).  NaN patterns (above the infinity
// pattern) are excluded so that NaN never flags a column.
// CTA shape: `wc` of the 8 warps sit side by side along the columns (each warp
// 256 columns = 512 contiguous bytes of a row), the other 8/wc split the rows;
// the launcher uses wc = 1.  Four lanes' flag bytes make one mask word, ORed
// into the mask with one atomicOr.  The last CTA to finish compacts the mask
// into the ascending idx list and records, per mask word, how many outlier
// columns precede it (prefix), so that the rank of an outlier column is
// prefix[w] + popc(lower bits of word w).
// ---------------------------------------------------------------------------
constexpr int kMaskThreads = 256;

// Exclusive prefix sum of v over the NT threads of the CTA (all of them call
// it, once), by warp shuffles: inclusive scans within each warp, then one warp
// scans the warp totals.  *total receives the sum.  s_warp holds NT/32 ints.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  static_assert(NT % 32 == 0 && NT / 32 <= 32, "one warp scans the warp totals");
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  int x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = (lane < NT / 32) ? s_warp[lane] : 0;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NT / 32) s_warp[lane] = t;
  }
  __syncthreads();
  *total = s_warp[NT / 32 - 1];
  return (w > 0 ? s_warp[w - 1] : 0) + x - v;
}
constexpr int kMaskUnroll = 4;

// Largest magnitude bit pattern among the 8 elements of v (16-bit max of |x|;
// max ignores a NaN operand, so a NaN can only raise the result to a NaN
// pattern when every element is NaN -- the caller then takes the exact path).
template <typename TE>
__device__ __forceinline__ uint32_t chunk_max_mag(const uint4& v) {
  using E = Elem<TE>;
  const uint32_t m = E::max2(E::max2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu), E::max2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
  return max(m & 0xffffu, m >> 16);
}

// Exact flags of one 8-column chunk; chunks whose largest magnitude is not
// above the threshold (nearly all of them) are settled by chunk_max_mag alone.
template <typename TE>
__device__ __forceinline__ uint32_t flag_bits8(const uint4& v, uint32_t h2) {
  if (chunk_max_mag<TE>(v) <= (h2 & 0xffffu)) return 0u;
  const uint32_t inf2 = Elem<TE>::kInfBits | (Elem<TE>::kInfBits << 16);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t bits = 0;
  #pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t a = w[i] & 0x7fff7fffu;
    const uint32_t m = __vcmpgtu2(a, h2) & __vcmpleu2(a, inf2);
    bits |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * i);
  }
  return bits;
}

template <typename TE>
__global__ void __launch_bounds__(kMaskThreads) outlier_mask_kernel(const TE* __restrict__ X, int64_t T, int64_t K,
                                                                    uint32_t hbits, int wc, int64_t rows_per_cta,
                                                                    uint32_t* mask,
                                                                    uint32_t* __restrict__ prefix, int32_t* __restrict__ idx,
                                                                    int32_t* __restrict__ n_out, DevStatus* st) {
  __shared__ int s_last;
  __shared__ int s_scan[kMaskThreads / 32];
  griddep_launch_dependents();  // the row quantisation may start meanwhile
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int wcol = warp % wc;        // warp position along the columns
  const int wrow = warp / wc;        // warp position along the rows
  const int wr = (kMaskThreads / 32) / wc;
  const int64_t col8 = static_cast<int64_t>(blockIdx.x) * (256 * wc) + wcol * 256 + lane * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t r1 = min(T, r0 + rows_per_cta);
  const uint32_t h2 = hbits | (hbits << 16);

  uint32_t bits = 0;
  if (col8 < K) {
    const TE* base = X + col8;
    int64_t r = r0 + wrow;
    #pragma unroll 1
    for (; r + (kMaskUnroll - 1) * wr < r1; r += kMaskUnroll * wr) {
      uint4 v[kMaskUnroll];
      #pragma unroll
      for (int u = 0; u < kMaskUnroll; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(base + (r + u * wr) * K));
      #pragma unroll
      for (int u = 0; u < kMaskUnroll; ++u) bits |= flag_bits8<TE>(v[u], h2);
    }
    #pragma unroll 1
    for (; r < r1; r += wr) bits |= flag_bits8<TE>(__ldg(reinterpret_cast<const uint4*>(base + r * K)), h2);
  }
  // lanes 4i..4i+3 hold the 4 bytes of one mask word
  uint32_t word = bits << ((lane & 3) * 8);
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  const int64_t nwords = (K + 31) / 32;
  if ((lane & 3) == 0 && word != 0 && col8 < K) atomicOr(&mask[col8 >> 5], word);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t total = gridDim.x * gridDim.y;
    const uint32_t prev = atomicAdd(&st->counter, 1u);
    s_last = (prev == total - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Compaction: thread t owns a contiguous run of mask words, so a block-wide
  // exclusive scan of per-thread popcounts yields ascending positions.
  const int64_t per = (nwords + kMaskThreads - 1) / kMaskThreads;
  const int64_t w0 = threadIdx.x * per;
  const int64_t w1 = min(nwords, w0 + per);
  int cnt = 0;
  for (int64_t w = w0; w < w1; ++w) cnt += __popc(ld_dep_u32(&mask[w]));
  int total = 0;
  int pos = block_exclusive_scan<kMaskThreads>(cnt, s_scan, &total);
  for (int64_t w = w0; w < w1; ++w) {
    uint32_t m = ld_dep_u32(&mask[w]);
    prefix[w] = static_cast<uint32_t>(pos);
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      idx[pos++] = static_cast<int32_t>(w * 32 + b);
    }
  }
  if (threadIdx.x == kMaskThreads - 1) {
    *n_out = total;
    st->counter = 0;
  }
}

cudaError_t launch_outliers(const void* X, int dtype, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                            uint32_t* prefix, int32_t* idx, int32_t* n_out, DevStatus* st, cudaStream_t s) {
  // The 8 warps split the rows (measured faster than warps side by side along
  // the columns, which gives fewer, longer-lived CTAs).  128 rows per CTA,
  // fewer (down to 32) while the grid would hold under 4 CTAs per SM.
  const int wc = 1;
  const int64_t slabs = (K + 256 * wc - 1) / (256 * wc);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t rows_per_cta = 128;
  while (rows_per_cta > 32 && slabs * ((T + rows_per_cta - 1) / rows_per_cta) < 4 * static_cast<int64_t>(sms))
    rows_per_cta /= 2;
  const int64_t chunks = (T + rows_per_cta - 1) / rows_per_cta;
  if (slabs > 0x7fffffff || chunks > 65535) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(slabs), static_cast<unsigned>(chunks));
  if (dtype == kBF16)
    outlier_mask_kernel<__nv_bfloat16><<<grid, kMaskThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(X), T, K, hbits,
                                                                      wc, rows_per_cta, mask, prefix, idx, n_out, st);
  else
    outlier_mask_kernel<__half><<<grid, kMaskThreads, 0, s>>>(static_cast<const __half*>(X), T, K, hbits, wc,
                                                              rows_per_cta, mask, prefix, idx, n_out, st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Row quantisation + outlier gathers.
//
// Rows: one warp per token row t, two passes over the row (the second mostly
// from L1/L2), with 8 independent 16-byte loads in flight per lane.
//   pass 1: absmax over the non-outlier columns, kept as a 16-bit magnitude
//           bit pattern (integer max of (bits & 0x7fff) equals the magnitude
//           max for finite values); chunks without outlier columns use a
//           16-bit max of |x|; a warp shuffle reduces it -- no block barrier;
//   pass 2: codes clamp(round_half_away(x * fp32(127/absmax))) packed 8 per
//           8-byte store, outlier values written to Xo[t, rank] straight from
//           registers, rank = prefix[word] + popc(lower bits of the word).
// Xo is zero-padded to the next multiple of 64 (the 16-bit outlier K-block).
// Wo blocks (blockIdx >= row blocks): Wo[j, o] = TE((CB[j, idx[o]] * SCB[j]) / 127)
// with the same padding, 8 outputs per lane and 16-byte stores (only when the
// tensor-core product consumes Wo).  With a 16-bit weight Wf (the
// has_fp16_weights=True layer) Wo[j, o] = Wf[j, idx[o]] instead.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowUnroll = 8;

// The outlier pass's outputs (mask, prefix, idx, n_out) decide addresses in the
// kernels that follow it under programmatic launch.  Those kernels read them
// with the ld_dep_* loads (kept behind the programmatic wait, through L2) and
// take them through pointers without __restrict__; n_out is also clamped to
// [0, K], so that no value it could hold turns into an address outside the
// workspace.
__device__ __forceinline__ uint32_t mask_byte(const uint32_t* mask, int64_t chunk) {
  return (ld_dep_u32_l1(&mask[chunk >> 2]) >> ((chunk & 3) * 8)) & 0xffu;
}

__device__ __forceinline__ int load_n_out(const int32_t* n_out_p, int64_t K) {
  const int32_t n = ld_dep_i32(n_out_p);
  return static_cast<int>(n < 0 ? 0 : (n > K ? K : n));
}

// Largest magnitude pattern among the non-outlier elements of a chunk.
template <typename TE>
__device__ __forceinline__ uint32_t chunk_max_mag_kept(const uint4& v, uint32_t mb) {
  if (mb == 0) return chunk_max_mag<TE>(v);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
  #pragma unroll
  for (int e = 0; e < 8; ++e)
    if (!((mb >> e) & 1u)) m = max(m, (w[e >> 1] >> ((e & 1) * 16)) & 0x7fffu);
  return m;
}

// Round half away from zero for y = x * fp32(127/absmax) with |x| <= absmax.
// y + copysign(0.5, y) equals sign(y) * (|y| + 0.5) as fp32 computes it; for
// |y| >= 0.5 that sum is exact or rounds within the same integer interval, so
// truncating toward zero gives the nearest integer with ties away from zero.
// For |y| < 0.5 the code is 0 (tested explicitly: just below 0.5, |y| + 0.5
// rounds up to 1.0 in fp32).  |y| <= 127 * (1 + 2^-24)^2 < 127.5 keeps the
// result within +-127 without a clamp.
// Round half away from zero for |y| <= 127.5 (the codes' range): with
// n = floor(|y| + 0.5), an integer and so exactly representable, the fp32 sum
// |y| + 0.5 rounded toward zero lies in [n, n + 1), and truncating it gives n.
// (Rounded to nearest, the sum fails below 0.5: 0.49999997 + 0.5 -> 1.0.)
__device__ __forceinline__ int round_away_code(float y) {
  return __float2int_rz(copysignf(__fadd_rz(fabsf(y), 0.5f), y));
}

template <typename TE>
__device__ __forceinline__ uint2 row_codes_fast(const uint4& v, uint32_t mb, float inv) {
  const uint32_t pairs[4] = {v.x, v.y, v.z, v.w};
  int q[8];
  #pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = Elem<TE>::to_float2(pairs[p]);
    q[2 * p] = round_away_code(__fmul_rn(f.x, inv));
    q[2 * p + 1] = round_away_code(__fmul_rn(f.y, inv));
  }
  // low bytes of the codes, 4 to a word
  uint32_t w0 = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
  uint32_t w1 = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
  if (mb) {  // outlier columns get code 0 (rare: a byte mask from the 8 flag bits)
    uint32_t k0 = 0, k1 = 0;
    #pragma unroll
    for (int e = 0; e < 4; ++e) {
      k0 |= ((mb >> e) & 1u) ? (0xffu << (8 * e)) : 0u;
      k1 |= ((mb >> (4 + e)) & 1u) ? (0xffu << (8 * e)) : 0u;
    }
    w0 &= ~k0;
    w1 &= ~k1;
  }
  return make_uint2(w0, w1);
}

// Scatter the outlier entries of one 8-column chunk into the Xo row.  mask and
// prefix are in global memory (read-only path) or, with kShared, in shared
// memory.
template <typename TE, bool kShared = false>
__device__ __forceinline__ void scatter_outliers(const uint4& v, uint32_t mb, int64_t chunk, const uint32_t* mask,
                                                 const uint32_t* prefix, TE* xo_row) {
  const TE* h = reinterpret_cast<const TE*>(&v);
  const uint32_t mw = kShared ? mask[chunk >> 2] : ld_dep_u32_l1(&mask[chunk >> 2]);
  const uint32_t base = kShared ? prefix[chunk >> 2] : ld_dep_u32_l1(&prefix[chunk >> 2]);
  const int sh = static_cast<int>(chunk & 3) * 8;
  const uint32_t first = base + __popc(mw & ((1u << sh) - 1u));
  if (mb == 0xffu && (first & 7u) == 0) {
    // all 8 columns are outliers and their ranks start on a 16-byte boundary
    // of the row (ldo is a multiple of 64): one vector store
    *reinterpret_cast<uint4*>(xo_row + first) = v;
    return;
  }
  #pragma unroll
  for (int e = 0; e < 8; ++e)
    if ((mb >> e) & 1u) xo_row[base + __popc(mw & ((1u << (sh + e)) - 1u))] = h[e];
}

// Wo[j, o] for the outlier columns, by the `wo_blocks` CTAs of NT threads
// that follow the row CTAs.  A warp covers whole rows j: its lanes split into
// groups of L = min(32, npad/8 rounded up to a power of two) lanes per row,
// each lane builds 8 consecutive outputs and writes them with one 16-byte
// store (npad is a multiple of 64, ldo of 64: rows stay 16-byte aligned).
// idx entries a Wo-gather CTA keeps in shared memory: every warp of the
// gather reads the same few idx words, which through L2 alone would put all
// of the grid's requests on one or two L2 lines.
constexpr int kWoIdx = 2048;

template <typename TE, int NT>
__device__ __forceinline__ void wo_gather(int64_t wblk, int64_t wo_blocks, int n_out, int64_t npad,
                                          const int32_t* idx, const int8_t* __restrict__ CB,
                                          const float* __restrict__ SCB, int64_t N, int64_t K, TE* __restrict__ Wo,
                                          int64_t ldo, const TE* __restrict__ Wf) {
  using E = Elem<TE>;
  __shared__ int32_t s_idx[kWoIdx];
  if (n_out == 0) return;  // n_out is the same for every thread of the grid
  const int n_staged = n_out < kWoIdx ? n_out : kWoIdx;
  for (int o = threadIdx.x; o < n_staged; o += NT) s_idx[o] = ld_dep_i32(&idx[o]);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int chunks = static_cast<int>(npad / 8);
  int lpr_log = 0;  // log2 of lanes per row
  while ((1 << lpr_log) < chunks && lpr_log < 5) ++lpr_log;
  const int lpr = 1 << lpr_log;
  const int sub = lane >> lpr_log;   // row within the warp's group
  const int l = lane & (lpr - 1);
  const int64_t rows_per_warp = 32 >> lpr_log;
  const int64_t warps = wo_blocks * (NT / 32);
  const int64_t warp = wblk * (NT / 32) + (threadIdx.x >> 5);
  for (int64_t j = warp * rows_per_warp + sub; j < N; j += warps * rows_per_warp) {
    const float scb = Wf == nullptr ? __ldg(&SCB[j]) : 0.0f;
    const int8_t* cbrow = CB + j * K;
    const TE* wfrow = Wf == nullptr ? nullptr : Wf + j * K;
    TE* worow = Wo + j * ldo;
    for (int c = l; c < chunks; c += lpr) {
      const int o0 = c * 8;
      uint32_t packed[4];
      #pragma unroll
      for (int i = 0; i < 8; i += 2) {
        float f[2];
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int o = o0 + i + h;
          f[h] = 0.0f;
          if (o < n_out) {
            const int col = o < kWoIdx ? s_idx[o] : static_cast<int>(ld_dep_u32_l1(&idx[o]));
            f[h] = wfrow != nullptr ? E::to_float(wfrow[col])
                                    : __fdiv_rn(__fmul_rn(static_cast<float>(__ldg(&cbrow[col])), scb), 127.0f);
          }
        }
        packed[i >> 1] = E::pack2(f[0], f[1]);
      }
      *reinterpret_cast<uint4*>(worow + o0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
}

template <typename TE>
__global__ void __launch_bounds__(kRowThreads) rowquant_kernel(
    const TE* __restrict__ X, int64_t T, int64_t K, const uint32_t* mask, const uint32_t* prefix,
    const int32_t* idx, const int32_t* n_out_p,
    int8_t* __restrict__ Xq, float* __restrict__ sA, TE* __restrict__ Xo, int64_t ldo,
    const int8_t* __restrict__ CB, const float* __restrict__ SCB, int64_t N, TE* __restrict__ Wo,
    const TE* __restrict__ Wf, int64_t row_blocks, int64_t wo_blocks) {
  using E = Elem<TE>;
  const int lane = threadIdx.x & 31;
  griddep_launch_dependents();
  griddep_wait();  // mask, prefix, idx, n_out come from the outlier pass
  const int n_out = load_n_out(n_out_p, K);
  const int64_t npad = ((static_cast<int64_t>(n_out) + 63) / 64) * 64;

  if (static_cast<int64_t>(blockIdx.x) >= row_blocks) {
    wo_gather<TE, kRowThreads>(static_cast<int64_t>(blockIdx.x) - row_blocks, wo_blocks, n_out, npad, idx, CB, SCB,
                               N, K, Wo, ldo, Wf);
    return;
  }

  // ---- one warp per token row ----
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int64_t nv = K / 8;
  const uint4* src = reinterpret_cast<const uint4*>(X + t * K);
  uint32_t mmax = 0;
  for (int64_t c0 = lane; c0 < nv; c0 += 32 * kRowUnroll) {
    uint4 v[kRowUnroll];
    #pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int64_t c = c0 + 32 * u;
      v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
    #pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int64_t c = c0 + 32 * u;
      if (c < nv) mmax = max(mmax, chunk_max_mag_kept<TE>(v[u], mask_byte(mask, c)));
    }
  }
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) mmax = max(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  const float absmax = E::mag_to_float(mmax);
  const float inv = scale_inv(absmax);
  if (lane == 0) sA[t] = absmax;

  uint2* dst = reinterpret_cast<uint2*>(Xq + t * K);
  TE* xo_row = Xo + t * ldo;
  for (int64_t c0 = lane; c0 < nv; c0 += 32 * kRowUnroll) {
    uint4 v[kRowUnroll];
    #pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int64_t c = c0 + 32 * u;
      v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
    #pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int64_t c = c0 + 32 * u;
      if (c < nv) {
        const uint32_t mb = mask_byte(mask, c);
        dst[c] = row_codes_fast<TE>(v[u], mb, inv);
        if (mb) scatter_outliers<TE>(v[u], mb, c, mask, prefix, xo_row);
      }
    }
  }
  for (int64_t o = n_out + lane; o < npad; o += 32) xo_row[o] = E::from_float(0.0f);
}

// One 256-thread CTA per row: a pass over the row needs about one round of
// loads, and the absmax is reduced across the CTA.  kResident (rows of at
// most 256 x 8 chunks, K <= 16384): the row is loaded once and stays in
// registers between the absmax and the codes, so X is read once.  (Measured
// against 512 x 4 and 128 x 16: equal at K = 14336, 15 % faster at K = 4096.)
constexpr int kRowCtaThreads = 256;
constexpr int kRowCtaUnroll = 8;
constexpr int64_t kResidentMaxK = static_cast<int64_t>(kRowCtaThreads) * kRowCtaUnroll * 8;

// A CTA takes R = 2^rpc_log rows (1, 2, 4 or 8), S = 256 / R threads per row:
// short rows share a CTA, so that every thread still has up to 8 loads in
// flight (R > 1 only when the row fits the S threads x 8 chunks).
template <typename TE, bool kResident>
__global__ void __launch_bounds__(kRowCtaThreads) rowquant_cta_kernel(
    const TE* __restrict__ X, int64_t T, int64_t K, const uint32_t* mask, const uint32_t* prefix,
    const int32_t* idx, const int32_t* n_out_p,
    int8_t* __restrict__ Xq, float* __restrict__ sA, TE* __restrict__ Xo, int64_t ldo,
    const int8_t* __restrict__ CB, const float* __restrict__ SCB, int64_t N, TE* __restrict__ Wo,
    const TE* __restrict__ Wf, int64_t row_blocks, int64_t wo_blocks, int rpc_log) {
  using E = Elem<TE>;
  __shared__ uint32_t s_max[kRowCtaThreads / 32];
  griddep_launch_dependents();
  griddep_wait();  // mask, prefix, idx, n_out come from the outlier pass
  const int n_out = load_n_out(n_out_p, K);
  const int64_t npad = ((static_cast<int64_t>(n_out) + 63) / 64) * 64;
  if (static_cast<int64_t>(blockIdx.x) >= row_blocks) {
    wo_gather<TE, kRowCtaThreads>(static_cast<int64_t>(blockIdx.x) - row_blocks, wo_blocks, n_out, npad, idx, CB,
                                  SCB, N, K, Wo, ldo, Wf);
    return;
  }
  const int S = kRowCtaThreads >> rpc_log;  // threads per row, a multiple of 32
  const int sub = static_cast<int>(threadIdx.x) / S;
  const int tid = static_cast<int>(threadIdx.x) - sub * S;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) << rpc_log) + sub;
  const bool live = t < T;   // whole warps share a row, so `live` is warp-uniform
  const int64_t nv = K / 8;
  const uint4* src = reinterpret_cast<const uint4*>(X + t * K);
  const int64_t step = static_cast<int64_t>(S) * kRowCtaUnroll;
  uint32_t mmax = 0;
  uint4 v[kRowCtaUnroll];   // with kResident: the whole row share of this thread
  uint32_t mbs[kRowCtaUnroll];
  if (live) {
    for (int64_t c0 = tid; c0 < nv; c0 += step) {
      #pragma unroll
      for (int u = 0; u < kRowCtaUnroll; ++u) {
        const int64_t c = c0 + static_cast<int64_t>(S) * u;
        v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        mbs[u] = (c < nv) ? mask_byte(mask, c) : 0u;
      }
      #pragma unroll
      for (int u = 0; u < kRowCtaUnroll; ++u) {
        const int64_t c = c0 + static_cast<int64_t>(S) * u;
        if (c < nv) mmax = max(mmax, chunk_max_mag_kept<TE>(v[u], mbs[u]));
      }
      if constexpr (kResident) break;
    }
  }
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) mmax = max(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = mmax;
  __syncthreads();
  if (!live) return;
  mmax = 0;
  const int w0 = sub * (S / 32);
  for (int w = w0; w < w0 + S / 32; ++w) mmax = max(mmax, s_max[w]);
  const float absmax = E::mag_to_float(mmax);
  const float inv = scale_inv(absmax);
  if (tid == 0) sA[t] = absmax;

  uint2* dst = reinterpret_cast<uint2*>(Xq + t * K);
  TE* xo_row = Xo + t * ldo;
  for (int64_t c0 = tid; c0 < nv; c0 += step) {
    if constexpr (!kResident) {
      #pragma unroll
      for (int u = 0; u < kRowCtaUnroll; ++u) {
        const int64_t c = c0 + static_cast<int64_t>(S) * u;
        v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        mbs[u] = (c < nv) ? mask_byte(mask, c) : 0u;
      }
    }
    #pragma unroll
    for (int u = 0; u < kRowCtaUnroll; ++u) {
      const int64_t c = c0 + static_cast<int64_t>(S) * u;
      if (c < nv) {
        dst[c] = row_codes_fast<TE>(v[u], mbs[u], inv);
        if (mbs[u]) scatter_outliers<TE>(v[u], mbs[u], c, mask, prefix, xo_row);
      }
    }
    if constexpr (kResident) break;
  }
  for (int64_t o = n_out + tid; o < npad; o += S) xo_row[o] = E::from_float(0.0f);
}

// ---------------------------------------------------------------------------
// Decode prep (T <= 16, weight-streaming product): the outlier pass and the
// row quantisation in one kernel, one 512-thread CTA per token row.  Every
// CTA rebuilds the column mask from all T rows (at most 16 x K x 2 bytes, read
// through L2) into shared memory, with the per-word prefix counts, and then
// quantises its row.  CTA 0 also publishes mask, prefix, idx and n_out and
// clears the status word, so the forward needs no memset and no separate
// outlier launch.  hbits == 0xffffffff means "no outliers".
// ---------------------------------------------------------------------------
constexpr int kSmallMaxK = 131072;
constexpr int kSmallThreads = 512;
constexpr int kSmallUnroll = 4;
constexpr int64_t kSmallResidentK = static_cast<int64_t>(kSmallThreads) * kSmallUnroll * 8;

// 32-bit load from the shared memory of CTA `rank` of this cluster, at the
// offset `local` has in this CTA.
__device__ __forceinline__ uint32_t ld_dsmem_u32(const uint32_t* local, uint32_t rank) {
  uint32_t v;
  asm volatile(
      "{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %1, %2;\n\tld.shared::cluster.u32 %0, [ra];\n\t}"
      : "=r"(v)
      : "r"(smem_u32(local)), "r"(rank)
      : "memory");
  return v;
}

// kResident (K <= 512 x 4 x 8): each thread keeps its 4 chunks of the CTA's own
// row in registers from the first load to the codes; other rows are read for
// the mask only.
// kCluster (with kResident; the T CTAs form one thread-block cluster): each
// CTA flags only its own row, into its own shared memory, and the column mask
// is the OR of the T CTAs' flags read through distributed shared memory,
// instead of every CTA testing all T rows.
template <typename TE, bool kResident, bool kCluster>
__global__ void __launch_bounds__(kSmallThreads) prep_small_kernel(
    const TE* __restrict__ X, int64_t T, int64_t K, uint32_t hbits, uint32_t* __restrict__ mask,
    uint32_t* __restrict__ prefix, int32_t* __restrict__ idx, int32_t* __restrict__ n_out_p, int8_t* __restrict__ Xq,
    float* __restrict__ sA, TE* __restrict__ Xo, int64_t ldo, DevStatus* st) {
  using E = Elem<TE>;
  __shared__ uint32_t s_mask[kSmallMaxK / 32];
  __shared__ uint32_t s_prefix[kSmallMaxK / 32];
  __shared__ int s_scan[kSmallThreads / 32];
  __shared__ uint32_t s_max[kSmallThreads / 32];
  __shared__ uint32_t s_own[kCluster ? kSmallResidentK / 32 : 1];  // this row's flags
  static_assert(!kCluster || kResident, "the cluster form keeps the row in registers");
  griddep_launch_dependents();  // the product kernel may start its prologue
  const int64_t nv = K / 8;
  const int64_t nw = (K + 31) / 32;
  const bool on = hbits != 0xffffffffu;
  const uint32_t h2 = hbits | (hbits << 16);
  const int64_t t = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(X + t * K);
  uint4 v[kSmallUnroll];  // with kResident: this thread's chunks of row t
  if constexpr (kResident) {
    #pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u) {
      const int64_t c = threadIdx.x + static_cast<int64_t>(kSmallThreads) * u;
      v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
  }
  if constexpr (kCluster) {
    for (int64_t w = threadIdx.x; w < nw; w += kSmallThreads) s_own[w] = 0;
    __syncthreads();
    if (on) {
      #pragma unroll
      for (int u = 0; u < kSmallUnroll; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(kSmallThreads) * u;
        if (c >= nv) continue;
        const uint32_t bits = flag_bits8<TE>(v[u], h2);
        if (bits) atomicOr(&s_own[c >> 2], bits << ((c & 3) * 8));
      }
    }
    cluster_sync();  // every CTA's flags are complete (release / acquire, cluster scope)
    for (int64_t w = threadIdx.x; w < nw; w += kSmallThreads) {
      uint32_t m = 0;
      for (int64_t r = 0; r < T; ++r) m |= ld_dsmem_u32(&s_own[w], static_cast<uint32_t>(r));
      s_mask[w] = m;
    }
    cluster_sync();  // no CTA reads another's flags after this; s_mask is complete
  } else {
  for (int64_t w = threadIdx.x; w < nw; w += kSmallThreads) s_mask[w] = 0;
  __syncthreads();
  // mask: column chunk c is flagged from all T rows
  if (on && kResident) {
    #pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u) {
      const int64_t c = threadIdx.x + static_cast<int64_t>(kSmallThreads) * u;
      if (c >= nv) continue;
      uint32_t bits = flag_bits8<TE>(v[u], h2);
      for (int64_t r = 0; r < T; r += 4) {
        uint4 o[4];
        #pragma unroll
        for (int q = 0; q < 4; ++q)
          o[q] = (r + q < T && r + q != t) ? __ldg(reinterpret_cast<const uint4*>(X + (r + q) * K) + c)
                                           : make_uint4(0, 0, 0, 0);
        #pragma unroll
        for (int q = 0; q < 4; ++q) bits |= flag_bits8<TE>(o[q], h2);
      }
      if (bits) atomicOr(&s_mask[c >> 2], bits << ((c & 3) * 8));
    }
  } else if (on) {
    for (int64_t c = threadIdx.x; c < nv; c += kSmallThreads) {
      uint32_t bits = 0;
      int64_t r = 0;
      for (; r + 4 <= T; r += 4) {
        uint4 v[4];
        #pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(X + (r + u) * K) + c);
        #pragma unroll
        for (int u = 0; u < 4; ++u) bits |= flag_bits8<TE>(v[u], h2);
      }
      for (; r < T; ++r) bits |= flag_bits8<TE>(__ldg(reinterpret_cast<const uint4*>(X + r * K) + c), h2);
      if (bits) atomicOr(&s_mask[c >> 2], bits << ((c & 3) * 8));
    }
  }
  __syncthreads();
  }
  // prefix counts: thread i owns a contiguous run of mask words
  const int64_t per = (nw + kSmallThreads - 1) / kSmallThreads;
  const int64_t w0 = threadIdx.x * per;
  const int64_t w1 = min(nw, w0 + per);
  int cnt = 0;
  for (int64_t w = w0; w < w1; ++w) cnt += __popc(s_mask[w]);
  int n_out = 0;
  int pos = block_exclusive_scan<kSmallThreads>(cnt, s_scan, &n_out);
  for (int64_t w = w0; w < w1; ++w) {
    s_prefix[w] = static_cast<uint32_t>(pos);
    if (blockIdx.x == 0) {
      uint32_t m = s_mask[w];
      mask[w] = m;
      prefix[w] = static_cast<uint32_t>(pos);
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1;
        idx[pos++] = static_cast<int32_t>(w * 32 + b);
      }
    } else {
      pos += __popc(s_mask[w]);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *n_out_p = n_out;
    st->error = 0;
    st->where = 0;
  }
  __syncthreads();

  // this CTA's row, as rowquant_cta_kernel with the mask from shared memory
  const int64_t npad = ((static_cast<int64_t>(n_out) + 63) / 64) * 64;
  const uint8_t* mb8 = reinterpret_cast<const uint8_t*>(s_mask);
  constexpr int64_t kStep = static_cast<int64_t>(kSmallThreads) * kSmallUnroll;
  uint32_t mmax = 0;
  for (int64_t c0 = threadIdx.x; c0 < nv; c0 += kStep) {
    if constexpr (!kResident) {
      #pragma unroll
      for (int u = 0; u < kSmallUnroll; ++u) {
        const int64_t c = c0 + static_cast<int64_t>(kSmallThreads) * u;
        v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      }
    }
    #pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u) {
      const int64_t c = c0 + static_cast<int64_t>(kSmallThreads) * u;
      if (c < nv) mmax = max(mmax, chunk_max_mag_kept<TE>(v[u], mb8[c]));
    }
    if constexpr (kResident) break;
  }
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) mmax = max(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = mmax;
  __syncthreads();
  mmax = 0;
  #pragma unroll
  for (int w = 0; w < kSmallThreads / 32; ++w) mmax = max(mmax, s_max[w]);
  const float absmax = E::mag_to_float(mmax);
  const float inv = scale_inv(absmax);
  if (threadIdx.x == 0) sA[t] = absmax;
  uint2* dst = reinterpret_cast<uint2*>(Xq + t * K);
  TE* xo_row = Xo + t * ldo;
  for (int64_t c0 = threadIdx.x; c0 < nv; c0 += kStep) {
    if constexpr (!kResident) {
      #pragma unroll
      for (int u = 0; u < kSmallUnroll; ++u) {
        const int64_t c = c0 + static_cast<int64_t>(kSmallThreads) * u;
        v[u] = (c < nv) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      }
    }
    #pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u) {
      const int64_t c = c0 + static_cast<int64_t>(kSmallThreads) * u;
      if (c < nv) {
        const uint32_t mb = mb8[c];
        dst[c] = row_codes_fast<TE>(v[u], mb, inv);
        if (mb) scatter_outliers<TE, true>(v[u], mb, c, s_mask, s_prefix, xo_row);
      }
    }
    if constexpr (kResident) break;
  }
  for (int64_t o = n_out + threadIdx.x; o < npad; o += kSmallThreads) xo_row[o] = E::from_float(0.0f);
}

// Whether the T CTAs of the cluster form can be co-scheduled as one cluster
// (per device, element type and T; 1 yes, -1 no, 0 not yet asked).  Clusters
// of more than 8 CTAs need the non-portable size opt-in.  Written without a
// lock: concurrent first calls ask the same question and store the same answer.
int8_t g_cluster_ok[64][2][kDecodeMaxT + 1];

template <typename TE>
bool cluster_form_ok(int64_t T, int et) {
  int dev = 0;
  if (T < 2 || T > kDecodeMaxT || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  int8_t& c = g_cluster_ok[dev][et][T];
  if (c != 0) return c > 0;
  auto* k = prep_small_kernel<TE, true, true>;
  bool ok = T <= 8 || cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  int n = 0;
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(T);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(T), 1, 1);
    cfg.blockDim = dim3(kSmallThreads, 1, 1);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ok = cudaOccupancyMaxActiveClusters(&n, k, &cfg) == cudaSuccess && n > 0;
  }
  if (!ok) (void)cudaGetLastError();  // a refused opt-in or query only means: no cluster form
  c = ok ? 1 : -1;
  return ok;
}

cudaError_t prepare_prep_small(int dtype) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  for (int64_t T = 2; T <= kDecodeMaxT; ++T) {
    if (dtype == kBF16)
      (void)cluster_form_ok<__nv_bfloat16>(T, 1);
    else
      (void)cluster_form_ok<__half>(T, 0);
  }
  return cudaSuccess;
}

template <typename TE>
cudaError_t launch_prep_small_t(const TE* X, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                                uint32_t* prefix, int32_t* idx, int32_t* n_out, int8_t* Xq, float* sA, TE* Xo,
                                int64_t ldo, DevStatus* st, int et, cudaStream_t s) {
  const bool resident = K <= kSmallResidentK;
  if (resident && cluster_form_ok<TE>(T, et)) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(T);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(T), 1, 1);
    cfg.blockDim = dim3(kSmallThreads, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prep_small_kernel<TE, true, true>, X, T, K, hbits, mask, prefix, idx, n_out, Xq,
                              sA, Xo, ldo, st);
  }
  auto* k = resident ? prep_small_kernel<TE, true, false> : prep_small_kernel<TE, false, false>;
  k<<<dim3(static_cast<unsigned>(T)), kSmallThreads, 0, s>>>(X, T, K, hbits, mask, prefix, idx, n_out, Xq, sA, Xo,
                                                              ldo, st);
  return cudaGetLastError();
}

cudaError_t launch_prep_small(const void* X, int dtype, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                              uint32_t* prefix, int32_t* idx, int32_t* n_out, int8_t* Xq, float* sA, void* Xo,
                              int64_t ldo, DevStatus* st, cudaStream_t s) {
  if (T < 1 || T > kDecodeMaxT || K > kSmallMaxK) return cudaErrorInvalidValue;
  if (dtype == kBF16)
    return launch_prep_small_t(static_cast<const __nv_bfloat16*>(X), T, K, hbits, mask, prefix, idx, n_out, Xq, sA,
                               static_cast<__nv_bfloat16*>(Xo), ldo, st, 1, s);
  return launch_prep_small_t(static_cast<const __half*>(X), T, K, hbits, mask, prefix, idx, n_out, Xq, sA,
                             static_cast<__half*>(Xo), ldo, st, 0, s);
}

template <typename TE>
static cudaError_t launch_rowquant_t(const cudaLaunchConfig_t& cfg, bool cta_rows, bool resident, int rpc_log,
                                     const void* X, int64_t T, int64_t K, const uint32_t* mask,
                                     const uint32_t* prefix, const int32_t* idx, const int32_t* n_out, int8_t* Xq,
                                     float* sA, void* Xo, int64_t ldo, const int8_t* CB, const float* SCB, int64_t N,
                                     void* Wo, const void* Wf, int64_t row_blocks, int64_t wo_blocks) {
  const TE* x = static_cast<const TE*>(X);
  TE* xo = static_cast<TE*>(Xo);
  TE* wo = static_cast<TE*>(Wo);
  const TE* wf = static_cast<const TE*>(Wf);
  if (!cta_rows)
    return cudaLaunchKernelEx(&cfg, rowquant_kernel<TE>, x, T, K, mask, prefix, idx, n_out, Xq, sA, xo, ldo, CB, SCB, N,
                              wo, wf, row_blocks, wo_blocks);
  return cudaLaunchKernelEx(&cfg, resident ? rowquant_cta_kernel<TE, true> : rowquant_cta_kernel<TE, false>, x, T, K,
                            mask, prefix, idx, n_out, Xq, sA, xo, ldo, CB, SCB, N, wo, wf, row_blocks, wo_blocks,
                            rpc_log);
}

cudaError_t launch_rowquant(const void* X, int dtype, int64_t T, int64_t K, const uint32_t* mask,
                            const uint32_t* prefix, const int32_t* idx, const int32_t* n_out, int8_t* Xq, float* sA,
                            void* Xo, int64_t ldo, const int8_t* CB, const float* SCB, int64_t N, void* Wo,
                            bool with_wo, const void* Wf, int num_sms, DevStatus* st, bool pdl, cudaStream_t s) {
  (void)st;
  // CTA rows with the row held in registers whenever it fits (X read once),
  // several short rows to a CTA; otherwise warp-per-row CTAs while they fill
  // the SMs, and one CTA per row (two passes) below that.
  const int64_t nv = K / 8;
  const bool resident = K <= kResidentMaxK;
  const bool cta_rows = resident || (T + kRowWarps - 1) / kRowWarps < num_sms;
  int rpc_log = 0;
  if (resident)
    while (rpc_log < 3 && nv * (int64_t(2) << rpc_log) <= int64_t(kRowCtaThreads) * kRowCtaUnroll) ++rpc_log;
  const int threads = cta_rows ? kRowCtaThreads : kRowThreads;
  int64_t wo_blocks = 0;
  if (with_wo) {
    wo_blocks = (N + threads / 32 - 1) / (threads / 32);  // at most one row per warp
    const int64_t cap = static_cast<int64_t>(num_sms) * 4;
    if (wo_blocks > cap) wo_blocks = cap;
    if (wo_blocks < 1) wo_blocks = 1;
  }
  const int64_t row_blocks =
      cta_rows ? (T + (int64_t(1) << rpc_log) - 1) >> rpc_log : (T + kRowWarps - 1) / kRowWarps;
  const int64_t blocks = row_blocks + wo_blocks;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (dtype == kBF16)
    return launch_rowquant_t<__nv_bfloat16>(cfg, cta_rows, resident, rpc_log, X, T, K, mask, prefix, idx, n_out, Xq,
                                            sA, Xo, ldo, CB, SCB, N, Wo, Wf, row_blocks, wo_blocks);
  return launch_rowquant_t<__half>(cfg, cta_rows, resident, rpc_log, X, T, K, mask, prefix, idx, n_out, Xq, sA, Xo,
                                   ldo, CB, SCB, N, Wo, Wf, row_blocks, wo_blocks);
}

}  // namespace i8mp
