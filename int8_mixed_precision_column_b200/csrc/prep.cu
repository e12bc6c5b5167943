// Memory-bound stages of the LLM.int8() forward linear layer:
//  * weight absmax quantisation (CB int8, SCB fp32), done once per layer;
//  * the column outlier mask and its compaction into the ascending index list;
//  * row-wise absmax int8 quantisation of the non-outlier activations, and the
//    gathers that feed the 16-bit outlier product.
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
__global__ void __launch_bounds__(256) quantize_weight_kernel(const __half* __restrict__ W, int64_t N, int64_t K,
                                                              int8_t* __restrict__ CB, float* __restrict__ SCB) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int64_t nv = K / 8;
  const uint4* src = reinterpret_cast<const uint4*>(W + row * K);
  float m = 0.0f;
  for (int64_t i = lane; i < nv; i += 32) {
    uint4 v = __ldg(src + i);
    const __half* h = reinterpret_cast<const __half*>(&v);
    #pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(__half2float(h[e])));
  }
  m = warp_max(m);
  const float inv = scale_inv(m);
  if (lane == 0) SCB[row] = m;
  uint2* dst = reinterpret_cast<uint2*>(CB + row * K);
  for (int64_t i = lane; i < nv; i += 32) {
    uint4 v = __ldg(src + i);
    const __half* h = reinterpret_cast<const __half*>(&v);
    uint32_t lo = 0, hi = 0;
    #pragma unroll
    for (int e = 0; e < 4; ++e) lo |= (static_cast<uint32_t>(quant_code(__half2float(h[e]), inv)) & 0xffu) << (8 * e);
    #pragma unroll
    for (int e = 0; e < 4; ++e) hi |= (static_cast<uint32_t>(quant_code(__half2float(h[4 + e]), inv)) & 0xffu) << (8 * e);
    dst[i] = make_uint2(lo, hi);
  }
}

cudaError_t launch_quantize_weight(const __half* W, int64_t N, int64_t K, int8_t* CB, float* SCB, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int64_t blocks = (N + 7) / 8;
  quantize_weight_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(W, N, K, CB, SCB);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Column outlier mask.
//
// Each thread owns 8 consecutive columns (one 16-byte load per row) and ORs
// together, over its rows, the bits "|x| > threshold".  The comparison is done
// on fp16 magnitude bit patterns: for non-NaN fp16 values the magnitude order
// equals the order of the 15-bit patterns, so |x| > threshold  <=>
// (bits & 0x7fff) > hbits, where hbits is the largest pattern whose value is
// <= threshold (computed on the host).  NaN patterns (> 0x7c00) are excluded so
// that NaN never flags a column.
// CTA shape: `wc` of the 8 warps sit side by side along the columns (each warp
// 256 columns = 512 contiguous bytes of a row), the other 8/wc split the rows.
// Large T uses wc = 8 (a CTA reads 4 KB contiguous of each of its rows, 8 rows
// of loads in flight per thread); small T uses wc = 1 so that enough CTAs
// exist.  Four lanes' flag bytes make one mask word, ORed into the mask with
// one atomicOr.  The last CTA to finish compacts the mask into the ascending
// idx list and records, per mask word, how many outlier columns precede it
// (prefix), so that the rank of an outlier column is prefix[w] + popc(lower
// bits of word w).
// ---------------------------------------------------------------------------
constexpr int kMaskThreads = 256;
constexpr int kMaskUnroll = 8;

__device__ __forceinline__ uint32_t flag_bits8(const uint4& v, uint32_t h2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t bits = 0;
  #pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t a = w[i] & 0x7fff7fffu;
    const uint32_t m = __vcmpgtu2(a, h2) & __vcmpleu2(a, 0x7c007c00u);
    bits |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * i);
  }
  return bits;
}

__global__ void __launch_bounds__(kMaskThreads) outlier_mask_kernel(const __half* __restrict__ X, int64_t T, int64_t K,
                                                                    uint32_t hbits, int wc, int64_t rows_per_cta,
                                                                    uint32_t* __restrict__ mask,
                                                                    uint32_t* __restrict__ prefix, int32_t* __restrict__ idx,
                                                                    int32_t* __restrict__ n_out, DevStatus* st) {
  __shared__ int s_last;
  __shared__ int s_scan[kMaskThreads];
  griddep_launch_dependents();  // the row quantisation may start loading X meanwhile
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
    const __half* base = X + col8;
    int64_t r = r0 + wrow;
    #pragma unroll 1
    for (; r + (kMaskUnroll - 1) * wr < r1; r += kMaskUnroll * wr) {
      uint4 v[kMaskUnroll];
      #pragma unroll
      for (int u = 0; u < kMaskUnroll; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(base + (r + u * wr) * K));
      #pragma unroll
      for (int u = 0; u < kMaskUnroll; ++u) bits |= flag_bits8(v[u], h2);
    }
    #pragma unroll 1
    for (; r < r1; r += wr) bits |= flag_bits8(__ldg(reinterpret_cast<const uint4*>(base + r * K)), h2);
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
  for (int64_t w = w0; w < w1; ++w) cnt += __popc(__ldcg(&mask[w]));
  s_scan[threadIdx.x] = cnt;
  __syncthreads();
  for (int off = 1; off < kMaskThreads; off <<= 1) {
    int v = (threadIdx.x >= off) ? s_scan[threadIdx.x - off] : 0;
    __syncthreads();
    s_scan[threadIdx.x] += v;
    __syncthreads();
  }
  int pos = s_scan[threadIdx.x] - cnt;
  for (int64_t w = w0; w < w1; ++w) {
    uint32_t m = __ldcg(&mask[w]);
    prefix[w] = static_cast<uint32_t>(pos);
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      idx[pos++] = static_cast<int32_t>(w * 32 + b);
    }
  }
  if (threadIdx.x == kMaskThreads - 1) {
    *n_out = s_scan[kMaskThreads - 1];
    st->counter = 0;
  }
}

cudaError_t launch_outliers(const __half* X, int64_t T, int64_t K, uint32_t hbits, uint32_t* mask,
                            uint32_t* prefix, int32_t* idx, int32_t* n_out, DevStatus* st, cudaStream_t s) {
  // Large T: 8 warps along the columns, 64-row chunks.  Small T: warps split the rows.
  const int wc = (T >= 512) ? 8 : 1;
  const int64_t rows_per_cta = (wc == 8) ? 64 : 128;
  const int64_t slabs = (K + 256 * wc - 1) / (256 * wc);
  const int64_t chunks = (T + rows_per_cta - 1) / rows_per_cta;
  if (slabs > 0x7fffffff || chunks > 65535) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(slabs), static_cast<unsigned>(chunks));
  outlier_mask_kernel<<<grid, kMaskThreads, 0, s>>>(X, T, K, hbits, wc, rows_per_cta, mask, prefix, idx, n_out, st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Row quantisation + outlier gathers.
//
// Blocks [0, T): one CTA per token row t.  The row is read once into registers
// (8 columns per 16-byte chunk), the absmax over non-outlier columns is
// reduced across the CTA, and the codes are written as 8-byte packets.  Each
// outlier value goes from registers straight to Xo[t, rank], its rank among
// the outlier columns being prefix[word] + popc(lower bits of the word); Xo is
// zero-padded to the next multiple of 64 (the K-block of the fp16 outlier MMA).
// Blocks [T, ...): Wo[j, o] = fp16((CB[j, idx[o]] * SCB[j]) / 127) with the
// same padding (only when the tensor-core path consumes Wo), four independent
// gathers per thread in flight.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 256;
constexpr int kRowChunks = 8;   // registers hold rows up to 256*8*8 = 16384 columns
constexpr int kWoUnroll = 4;

__device__ __forceinline__ uint32_t mask_byte(const uint32_t* mask, int64_t chunk) {
  return (__ldg(&mask[chunk >> 2]) >> ((chunk & 3) * 8)) & 0xffu;
}

__device__ __forceinline__ float row_absmax_part(const uint4& v, uint32_t mb) {
  const __half* h = reinterpret_cast<const __half*>(&v);
  float m = 0.0f;
  #pragma unroll
  for (int e = 0; e < 8; ++e)
    if (!((mb >> e) & 1u)) m = fmaxf(m, fabsf(__half2float(h[e])));
  return m;
}

__device__ __forceinline__ uint2 row_codes(const uint4& v, uint32_t mb, float inv) {
  const __half* h = reinterpret_cast<const __half*>(&v);
  uint32_t w[2] = {0u, 0u};
  #pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int q = ((mb >> e) & 1u) ? 0 : quant_code(__half2float(h[e]), inv);
    w[e >> 2] |= (static_cast<uint32_t>(q) & 0xffu) << (8 * (e & 3));
  }
  return make_uint2(w[0], w[1]);
}

// Scatter the outlier entries of one 8-column chunk into the Xo row.
__device__ __forceinline__ void scatter_outliers(const uint4& v, uint32_t mb, int64_t chunk, const uint32_t* mask,
                                                 const uint32_t* prefix, __half* xo_row) {
  const __half* h = reinterpret_cast<const __half*>(&v);
  const uint32_t mw = __ldg(&mask[chunk >> 2]);
  const uint32_t base = __ldg(&prefix[chunk >> 2]);
  const int sh = static_cast<int>(chunk & 3) * 8;
  #pragma unroll
  for (int e = 0; e < 8; ++e)
    if ((mb >> e) & 1u) xo_row[base + __popc(mw & ((1u << (sh + e)) - 1u))] = h[e];
}

__global__ void __launch_bounds__(kRowThreads, 3) rowquant_regs_kernel(
    const __half* __restrict__ X, int64_t T, int64_t K, const uint32_t* __restrict__ mask,
    const uint32_t* __restrict__ prefix, const int32_t* __restrict__ idx, const int32_t* __restrict__ n_out_p,
    int8_t* __restrict__ Xq, float* __restrict__ sA, __half* __restrict__ Xo, int64_t ldo,
    const int8_t* __restrict__ CB, const float* __restrict__ SCB, int64_t N, __half* __restrict__ Wo,
    int64_t wo_blocks) {
  __shared__ float s_red[kRowThreads / 32];
  const int tid = threadIdx.x;
  griddep_launch_dependents();
  griddep_wait();  // mask, prefix, idx, n_out come from the outlier pass
  const int n_out = *n_out_p;
  const int64_t npad = ((static_cast<int64_t>(n_out) + 63) / 64) * 64;

  if (static_cast<int64_t>(blockIdx.x) >= T) {
    // ---- Wo rows ----
    if (n_out == 0) return;
    const int64_t total = N * npad;
    const int64_t stride = wo_blocks * kRowThreads * kWoUnroll;
    for (int64_t e0 = (static_cast<int64_t>(blockIdx.x) - T) * kRowThreads * kWoUnroll + tid; e0 < total;
         e0 += stride) {
      int8_t cbv[kWoUnroll];
      int64_t jj[kWoUnroll], oo[kWoUnroll];
      #pragma unroll
      for (int u = 0; u < kWoUnroll; ++u) {
        const int64_t e = e0 + static_cast<int64_t>(u) * kRowThreads;
        jj[u] = e / npad;
        oo[u] = e - jj[u] * npad;
        cbv[u] = (e < total && oo[u] < n_out) ? __ldg(&CB[jj[u] * K + __ldg(&idx[oo[u]])]) : int8_t(0);
      }
      #pragma unroll
      for (int u = 0; u < kWoUnroll; ++u) {
        const int64_t e = e0 + static_cast<int64_t>(u) * kRowThreads;
        if (e < total) {
          __half v = __float2half_rn(0.0f);
          if (oo[u] < n_out)
            v = __float2half_rn(__fdiv_rn(__fmul_rn(static_cast<float>(cbv[u]), __ldg(&SCB[jj[u]])), 127.0f));
          Wo[jj[u] * ldo + oo[u]] = v;
        }
      }
    }
    return;
  }

  // ---- one token row ----
  const int64_t t = blockIdx.x;
  const int64_t nv = K / 8;
  const uint4* src = reinterpret_cast<const uint4*>(X + t * K);
  uint4 v[kRowChunks];
  uint32_t mb[kRowChunks];
  float m = 0.0f;
  #pragma unroll
  for (int c = 0; c < kRowChunks; ++c) {
    const int64_t i = tid + static_cast<int64_t>(c) * kRowThreads;
    if (i < nv) {
      v[c] = __ldcs(src + i);
      mb[c] = mask_byte(mask, i);
      m = fmaxf(m, row_absmax_part(v[c], mb[c]));
    }
  }
  for (int64_t i = tid + static_cast<int64_t>(kRowChunks) * kRowThreads; i < nv; i += kRowThreads)
    m = fmaxf(m, row_absmax_part(__ldg(src + i), mask_byte(mask, i)));
  m = warp_max(m);
  if ((tid & 31) == 0) s_red[tid >> 5] = m;
  __syncthreads();
  if (tid < 32) {
    float r = (tid < kRowThreads / 32) ? s_red[tid] : 0.0f;
    r = warp_max(r);
    if (tid == 0) s_red[0] = r;
  }
  __syncthreads();
  const float absmax = s_red[0];
  const float inv = scale_inv(absmax);
  if (tid == 0) sA[t] = absmax;
  uint2* dst = reinterpret_cast<uint2*>(Xq + t * K);
  __half* xo_row = Xo + t * ldo;
  #pragma unroll
  for (int c = 0; c < kRowChunks; ++c) {
    const int64_t i = tid + static_cast<int64_t>(c) * kRowThreads;
    if (i < nv) {
      dst[i] = row_codes(v[c], mb[c], inv);
      if (mb[c]) scatter_outliers(v[c], mb[c], i, mask, prefix, xo_row);
    }
  }
  for (int64_t i = tid + static_cast<int64_t>(kRowChunks) * kRowThreads; i < nv; i += kRowThreads) {
    const uint4 vv = __ldg(src + i);
    const uint32_t b = mask_byte(mask, i);
    dst[i] = row_codes(vv, b, inv);
    if (b) scatter_outliers(vv, b, i, mask, prefix, xo_row);
  }
  for (int64_t o = n_out + tid; o < npad; o += kRowThreads) xo_row[o] = __float2half_rn(0.0f);
}

// Bulk-copy variant for K <= kBulkMaxK: CTA b walks rows b, b+G, b+2G, ... with
// two shared-memory stages.  One 1-D bulk copy brings a whole fp16 row in,
// the codes are written to shared memory and leave with one bulk store, while
// the next row's copy is already in flight.  One thread waits on each load's
// mbarrier (bounded), the CTA barrier publishes it to the others.  After its
// rows, each CTA takes a 1/G share of the Wo gather (when asked for).
constexpr int64_t kBulkMaxK = 16384;
constexpr uint32_t W_ROWLOAD = 0x301;

__device__ __forceinline__ void wo_gather_share(const int8_t* __restrict__ CB, const float* __restrict__ SCB,
                                                const int32_t* __restrict__ idx, int n_out, int64_t npad, int64_t N,
                                                int64_t K, __half* __restrict__ Wo, int64_t ldo, int64_t part,
                                                int64_t parts) {
  const int64_t total = N * npad;
  const int64_t stride = parts * kRowThreads * kWoUnroll;
  for (int64_t e0 = part * kRowThreads * kWoUnroll + threadIdx.x; e0 < total; e0 += stride) {
    int8_t cbv[kWoUnroll];
    int64_t jj[kWoUnroll], oo[kWoUnroll];
    #pragma unroll
    for (int u = 0; u < kWoUnroll; ++u) {
      const int64_t e = e0 + static_cast<int64_t>(u) * kRowThreads;
      jj[u] = e / npad;
      oo[u] = e - jj[u] * npad;
      cbv[u] = (e < total && oo[u] < n_out) ? __ldg(&CB[jj[u] * K + __ldg(&idx[oo[u]])]) : int8_t(0);
    }
    #pragma unroll
    for (int u = 0; u < kWoUnroll; ++u) {
      const int64_t e = e0 + static_cast<int64_t>(u) * kRowThreads;
      if (e < total) {
        __half v = __float2half_rn(0.0f);
        if (oo[u] < n_out)
          v = __float2half_rn(__fdiv_rn(__fmul_rn(static_cast<float>(cbv[u]), __ldg(&SCB[jj[u]])), 127.0f));
        Wo[jj[u] * ldo + oo[u]] = v;
      }
    }
  }
}

__global__ void __launch_bounds__(kRowThreads) rowquant_bulk_kernel(
    const __half* __restrict__ X, int64_t T, int64_t K, const uint32_t* __restrict__ mask,
    const uint32_t* __restrict__ prefix, const int32_t* __restrict__ idx, const int32_t* __restrict__ n_out_p,
    int8_t* __restrict__ Xq, float* __restrict__ sA, __half* __restrict__ Xo, int64_t ldo,
    const int8_t* __restrict__ CB, const float* __restrict__ SCB, int64_t N, __half* __restrict__ Wo, int with_wo,
    DevStatus* st) {
  extern __shared__ __align__(128) uint8_t rq_smem[];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ float s_red[kRowThreads / 32];
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x;
  const int64_t G = gridDim.x;
  griddep_launch_dependents();

  __half* xs[2] = {reinterpret_cast<__half*>(rq_smem), reinterpret_cast<__half*>(rq_smem + 2 * K)};
  int8_t* qs[2] = {reinterpret_cast<int8_t*>(rq_smem + 4 * K), reinterpret_cast<int8_t*>(rq_smem + 5 * K)};
  const uint32_t row_bytes = static_cast<uint32_t>(2 * K);
  const int64_t nv = K / 8;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    // X is an input of the forward, not an output of the outlier pass: its
    // first two rows can stream in before that pass has finished.
    for (int b = 0; b < 2; ++b) {
      const int64_t r = blockIdx.x + b * G;
      if (r < T) {
        mbar_arrive_expect_tx(&bar[b], row_bytes);
        bulk_load(xs[b], X + r * K, row_bytes, &bar[b]);
      }
    }
  }
  griddep_wait();  // mask, prefix, idx, n_out come from the outlier pass
  const int n_out = *n_out_p;
  const int64_t npad = ((static_cast<int64_t>(n_out) + 63) / 64) * 64;
  int i = 0;
  for (int64_t t = blockIdx.x; t < T; t += G, ++i) {
    const int buf = i & 1;
    if (tid == 0) mbar_wait(&bar[buf], static_cast<uint32_t>((i >> 1) & 1), &s_abort, st, W_ROWLOAD);
    __syncthreads();
    if (s_abort) break;
    const __half* xrow = xs[buf];
    float m = 0.0f;
    for (int64_t c = tid; c < nv; c += kRowThreads)
      m = fmaxf(m, row_absmax_part(reinterpret_cast<const uint4*>(xrow)[c], mask_byte(mask, c)));
    m = warp_max(m);
    if ((tid & 31) == 0) s_red[tid >> 5] = m;
    if (tid == 0 && i >= 2) bulk_wait_read<1>();  // the store that last used qs[buf] has read it
    __syncthreads();
    float absmax = (tid < kRowThreads / 32) ? s_red[tid] : 0.0f;
    absmax = warp_max(absmax);  // warp 0 holds the block maximum in every lane
    __syncthreads();
    if (tid == 0) s_red[0] = absmax;
    __syncthreads();
    absmax = s_red[0];
    const float inv = scale_inv(absmax);
    __half* xo_row = Xo + t * ldo;
    for (int64_t c = tid; c < nv; c += kRowThreads) {
      const uint4 v = reinterpret_cast<const uint4*>(xrow)[c];
      const uint32_t mb = mask_byte(mask, c);
      reinterpret_cast<uint2*>(qs[buf])[c] = row_codes(v, mb, inv);
      if (mb) scatter_outliers(v, mb, c, mask, prefix, xo_row);
    }
    for (int64_t o = n_out + tid; o < npad; o += kRowThreads) xo_row[o] = __float2half_rn(0.0f);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      sA[t] = absmax;
      bulk_store(Xq + t * K, qs[buf], static_cast<uint32_t>(K));
      bulk_commit();
      const int64_t rn = t + 2 * G;
      if (rn < T) {
        mbar_arrive_expect_tx(&bar[buf], row_bytes);
        bulk_load(xs[buf], X + rn * K, row_bytes, &bar[buf]);
      }
    }
  }
  if (tid == 0) {
    bulk_wait<0>();
    // loads still in flight after an early exit must land before the CTA ends
    if (s_abort) {
      volatile int never = 0;
      for (int b = 0; b < 2; ++b) mbar_wait(&bar[b], static_cast<uint32_t>(((i + b) >> 1) & 1), &never, st, W_ROWLOAD);
    }
  }
  if (with_wo && n_out > 0 && !s_abort) wo_gather_share(CB, SCB, idx, n_out, npad, N, K, Wo, ldo, blockIdx.x, G);
}

cudaError_t launch_rowquant(const __half* X, int64_t T, int64_t K, const uint32_t* mask, const uint32_t* prefix,
                            const int32_t* idx, const int32_t* n_out, int8_t* Xq, float* sA, __half* Xo, int64_t ldo,
                            const int8_t* CB, const float* SCB, int64_t N, __half* Wo, bool with_wo, int num_sms,
                            DevStatus* st, bool pdl, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kRowThreads, 1, 1);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  int64_t wo_blocks = 0;
  if (with_wo) {
    wo_blocks = (N * 64 + kRowThreads * kWoUnroll - 1) / (kRowThreads * kWoUnroll);
    const int64_t cap = static_cast<int64_t>(num_sms) * 4;
    if (wo_blocks > cap) wo_blocks = cap;
    if (wo_blocks < 1) wo_blocks = 1;
  }
  if (K <= kBulkMaxK) {
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_done[dev]) {
      e = cudaFuncSetAttribute(rowquant_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(6 * kBulkMaxK));
      if (e != cudaSuccess) return e;
      attr_done[dev] = true;
    }
    // two CTAs per SM (two staged rows each); enough CTAs for the rows, and for
    // the Wo gather when the tensor-core product needs Wo
    int64_t ctas = T;
    if (with_wo && ctas < 2 * num_sms) ctas = 2 * num_sms;
    if (ctas > 2 * num_sms) ctas = 2 * num_sms;
    if (ctas == 0) return cudaSuccess;
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(6 * K);
    return cudaLaunchKernelEx(&cfg, rowquant_bulk_kernel, X, T, K, mask, prefix, idx, n_out, Xq, sA, Xo, ldo, CB, SCB,
                              N, Wo, with_wo ? 1 : 0, st);
  }
  const int64_t blocks = T + wo_blocks;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, rowquant_regs_kernel, X, T, K, mask, prefix, idx, n_out, Xq, sA, Xo, ldo, CB, SCB, N,
                            Wo, wo_blocks);
}

}  // namespace i8mp
