// Decode-regime (1..16 tokens) int8 product of the LLM.int8() forward linear
// layer: the same decomposition as the prefill GEMM (int8 vector-wise product
// over the non-outlier columns, 16-bit product over the outlier columns,
// dequantise and sum; "Core idea of LLM.int8()", Hugging Face integration
// page), shaped for streaming the int8 weight CB from HBM once.
//
// Work split: output rows are taken in groups of 8; each CTA owns a contiguous
// range of groups and walks it 4 groups (32 rows, one pass) at a time.  When
// there are at least 3 passes per CTA slot the ranges are whole passes, the
// same count (to one) per CTA: a partial last pass runs with fewer weight
// loads in flight and, measured, costs about as much as a full one.  The 8
// warps of a CTA split K; each warp multiplies its K-slice of the 16 x K token
// codes by the 32 weight rows with mma.sync m16n8k32 (s8 x s8 -> s32).
// Fragment trick: the dot product is a sum over k, so any permutation of k
// applied to both operands leaves it unchanged.  Thread (g, t) of a warp loads
// 16 contiguous bytes of weight row g at k0 + 16t and the same 16 bytes of
// token rows g and g+8; two MMAs consume them (bytes 0-7, then 8-15).  Every
// thread issues the weight loads of four K-steps for all 4 row groups before
// its first MMA, so 16 x 16 bytes per thread are in flight (measured against
// two and three K-steps: 9 % faster at one token; the few bytes the compiler
// spills at the 128-register bound cost less than the shallower pipeline).
// The warps' int32 partial sums of a pass meet in one 2 KB shared array by
// shared-memory atomic adds (exact in any order).
// Epilogue: Y = TE(acc * sA[t] * SCB[j] / 127^2 + sum_o Xo[t,o] * Wo[j,o] + b[j])
// with Wo[j,o] = TE((CB[j, idx[o]] * SCB[j]) / 127) recomputed from CB; the
// outlier operands of a 32-row chunk are staged in shared memory, DV_OB
// outlier columns at a time.
#include "kernels.h"

namespace i8mp {
namespace {

constexpr int DV_WARPS = 8;
constexpr int DV_THREADS = DV_WARPS * 32;
constexpr int DV_RG = 4;   // 8-row groups per pass (32 rows)
constexpr int DV_U = 4;    // K-steps (64 B each) loaded before computing
#ifndef I8MP_DV_OB
#define I8MP_DV_OB 16
#endif
constexpr int DV_OB = I8MP_DV_OB;  // outlier columns staged per block
constexpr int kPrefetchRows = 16;  // weight rows per CTA pulled into L2 before the wait


struct DvParams {
  const int8_t* Xq;
  const float* sA;
  const int8_t* CB;
  const float* SCB;
  const void* bias;  // TE[N] or null
  const void* Xo;    // TE[T,ldo]
  int64_t ldo;
  const int32_t* idx;
  const int32_t* n_out;
  const void* Wf;    // TE[N,K] 16-bit weight (has_fp16_weights=True) or null
  void* Y;           // TE[T,N]
  int32_t* acc_out;
  YDst yd;           // row stride of Y and its extra destinations
  int64_t T, N, K;
  int mode;
  int unit;          // 8-row groups per unit of the CTA split (1, or DV_RG)
};

__device__ __forceinline__ void mma_s8_16832(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_stream(const int8_t* p) {
  uint4 v;
  // streamed once: no L1 allocation; L2 fetches 256-byte blocks of the row
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// kExtra: Y also goes to the extra destinations of p.yd (a separate
// instantiation, so the single-destination kernel is not burdened by it).
template <typename TE, bool kExtra>
__global__ void __launch_bounds__(DV_THREADS, 2) gemv_i8_decode_kernel(const DvParams p) {
  using E = Elem<TE>;
  // int32 partial sums of the pass, added by the 8 warps with shared-memory
  // atomics (exact in any order); each entry is read and cleared by the one
  // thread that owns its output
  __shared__ int32_t red[DV_RG][32][4];
  __shared__ float wo_s[DV_RG * 8][DV_OB + 1];
  __shared__ float xo_s[kDecodeMaxT][DV_OB + 1];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t4 = lane & 3;
  const int64_t G = p.N / 8;
  const int64_t units = (G + p.unit - 1) / p.unit;
  const int64_t g_begin = min(G, p.unit * (units * blockIdx.x / gridDim.x));
  const int64_t g_end = min(G, p.unit * (units * (blockIdx.x + 1) / gridDim.x));
  const int64_t steps = (p.K + 63) / 64;
  const int64_t s_begin = steps * warp / DV_WARPS;
  const int64_t s_end = steps * (warp + 1) / DV_WARPS;
  // The weights are an input of the layer, not an output of the preceding
  // kernels: under a programmatic launch, start pulling this CTA's first rows
  // into L2 while the outlier pass and the row quantisation finish.
  if (threadIdx.x < kPrefetchRows && g_begin * 8 + threadIdx.x < g_end * 8)
    prefetch_l2(p.CB + (g_begin * 8 + threadIdx.x) * p.K, static_cast<uint32_t>(p.K));
  griddep_wait();
  // Xq, sA, Xo, idx and n_out come from the prep kernel: read with the ld_dep_*
  // loads (kept behind the wait, coherent); n_out clamped to [0, K]
  int n_out = (p.mode == 0) ? ld_dep_i32(p.n_out) : 0;
  n_out = n_out < 0 ? 0 : (n_out > p.K ? static_cast<int>(p.K) : n_out);
  const bool row_a = g < p.T;
  const bool row_b = g + 8 < p.T;
  const int8_t* xa_base = p.Xq + static_cast<int64_t>(g) * p.K + t4 * 16;
  const int8_t* xb_base = p.Xq + static_cast<int64_t>(g + 8) * p.K + t4 * 16;
  const uint4 zero4 = make_uint4(0, 0, 0, 0);
  for (int e = threadIdx.x; e < DV_RG * 32 * 4; e += DV_THREADS) (&red[0][0][0])[e] = 0;
  __syncthreads();

  for (int64_t g0 = g_begin; g0 < g_end; g0 += DV_RG) {
    int32_t c[DV_RG][4];
    #pragma unroll
    for (int r = 0; r < DV_RG; ++r) c[r][0] = c[r][1] = c[r][2] = c[r][3] = 0;
    const int8_t* wrow[DV_RG];
    bool wok[DV_RG];
    #pragma unroll
    for (int r = 0; r < DV_RG; ++r) {
      wok[r] = (g0 + r) < g_end;
      wrow[r] = p.CB + ((g0 + r) * 8 + g) * p.K + t4 * 16;
    }
    #pragma unroll 1
    for (int64_t st = s_begin; st < s_end; st += DV_U) {
      uint4 w[DV_U][DV_RG];
      uint4 xa[DV_U], xb[DV_U];
      #pragma unroll
      for (int u = 0; u < DV_U; ++u) {
        const int64_t k = (st + u) * 64;
        const bool kok = (st + u) < s_end && k + t4 * 16 < p.K;
        #pragma unroll
        for (int r = 0; r < DV_RG; ++r) w[u][r] = (wok[r] && kok) ? ld_stream(wrow[r] + k) : zero4;
      }
      #pragma unroll
      for (int u = 0; u < DV_U; ++u) {
        const int64_t k = (st + u) * 64;
        const bool kok = (st + u) < s_end && k + t4 * 16 < p.K;
        xa[u] = (row_a && kok) ? ld_dep_v4(xa_base + k) : zero4;
        xb[u] = (row_b && kok) ? ld_dep_v4(xb_base + k) : zero4;
      }
      #pragma unroll
      for (int u = 0; u < DV_U; ++u) {
        #pragma unroll
        for (int r = 0; r < DV_RG; ++r) {
          mma_s8_16832(c[r], xa[u].x, xb[u].x, xa[u].y, xb[u].y, w[u][r].x, w[u][r].y);
          mma_s8_16832(c[r], xa[u].z, xb[u].z, xa[u].w, xb[u].w, w[u][r].z, w[u][r].w);
        }
      }
    }
    #pragma unroll
    for (int r = 0; r < DV_RG; ++r) {
      #pragma unroll
      for (int i = 0; i < 4; ++i) atomicAdd(&red[r][lane][i], c[r][i]);
    }
    __syncthreads();

    // Each thread owns two (token, row) outputs of the 512 this pass produces.
    int32_t acc[2];
    float yo[2] = {0.0f, 0.0f};
    int tok[2], jr[2];
    bool live[2];
    #pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int v = threadIdx.x + h * DV_THREADS;
      const int r = v >> 7;
      const int ln = (v >> 2) & 31;
      const int i = v & 3;
      tok[h] = (ln >> 2) + ((i >> 1) << 3);
      jr[h] = r * 8 + (ln & 3) * 2 + (i & 1);
      live[h] = (g0 + r < g_end) && tok[h] < p.T;
      acc[h] = red[r][ln][i];
      red[r][ln][i] = 0;  // for the next pass (whose adds follow the pass-end barrier)
    }
    // 16-bit product over the outlier columns, DV_OB columns at a time.
    for (int ob = 0; ob < n_out; ob += DV_OB) {
      const int nb = min(DV_OB, n_out - ob);
      for (int e = threadIdx.x; e < DV_RG * 8 * nb; e += DV_THREADS) {
        const int r = e / nb;
        const int o = e - r * nb;
        const int64_t j = g0 * 8 + r;
        float wv = 0.0f;
        if (j < g_end * 8) {
          const int64_t col = static_cast<int32_t>(ld_dep_u32_l1(&p.idx[ob + o]));
          if (p.Wf != nullptr) {
            wv = E::to_float(static_cast<const TE*>(p.Wf)[j * p.K + col]);
          } else {
            const float cbv = static_cast<float>(__ldg(&p.CB[j * p.K + col]));
            wv = E::to_float(E::from_float(__fdiv_rn(__fmul_rn(cbv, __ldg(&p.SCB[j])), 127.0f)));
          }
        }
        wo_s[r][o] = wv;
      }
      for (int e = threadIdx.x; e < kDecodeMaxT * nb; e += DV_THREADS) {
        const int t = e / nb;
        const int o = e - t * nb;
        xo_s[t][o] = (t < p.T) ? E::to_float(E::from_bits(ld_dep_u16_hot(static_cast<const TE*>(p.Xo) + t * p.ldo + ob + o)))
                               : 0.0f;
      }
      __syncthreads();
      #pragma unroll
      for (int h = 0; h < 2; ++h) {
        float s = yo[h];
        for (int o = 0; o < nb; ++o) s = fmaf(xo_s[tok[h]][o], wo_s[jr[h]][o], s);
        yo[h] = s;
      }
      __syncthreads();
    }
    #pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (!live[h]) continue;
      const int64_t j = g0 * 8 + jr[h];
      if (p.mode == 1) {
        p.acc_out[tok[h] * p.N + j] = acc[h];
        continue;
      }
      const float scb = __ldg(&p.SCB[j]);
      float y = static_cast<float>(acc[h]) * (ld_dep_f32(&p.sA[tok[h]]) * (1.0f / 16129.0f) * scb) + yo[h];
      if (p.bias != nullptr) y += E::to_float(static_cast<const TE*>(p.bias)[j]);
      const int64_t off = tok[h] * p.yd.ld + j;
      const TE v = E::from_float(y);
      static_cast<TE*>(p.Y)[off] = v;
      if constexpr (kExtra) store_extra<TE>(p.yd, off, v);
    }
    __syncthreads();
  }
}

// Prefer L1 to shared memory: the kernel holds 5.3 KB of shared memory, so
// the 16 KB configuration (a 7 % carveout) still fits 2 CTAs per SM and
// leaves about 240 KB to L1 for the token codes that every pass re-reads (the
// two CTAs of an SM read the same ones).  Measured at BLOOM FFN-up width,
// product kernel in us, against the previous kernel (per-warp partial sums
// in 16 KB of shared memory, 64 outlier columns staged, 64 KB configuration):
// 142.2-142.5 against 146.5-146.9 at T = 1, 144.0-144.2 against 148.2-148.3
// at T = 4, 156.4-156.5 against 157.4-157.9 at T = 16; the same kernel with
// the 32 KB or 64 KB configuration took 143.2-144.1, 144.6-145.8 and
// 156.5-156.9.  (With the old kernel, the largest shared-memory
// configuration had doubled the time.)  A hint, set once per device; a
// failure is cleared and ignored.
#ifndef I8MP_DV_CARVE
#define I8MP_DV_CARVE 7
#endif
bool g_carveout_set[64] = {false};

void prefer_l1(int dev) {
  if (dev < 0 || dev >= 64 || g_carveout_set[dev]) return;
  const int pct = I8MP_DV_CARVE;
  bool ok = cudaFuncSetAttribute(gemv_i8_decode_kernel<__half, false>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout, pct) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemv_i8_decode_kernel<__half, true>,
                                  cudaFuncAttributePreferredSharedMemoryCarveout, pct) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemv_i8_decode_kernel<__nv_bfloat16, false>,
                                  cudaFuncAttributePreferredSharedMemoryCarveout, pct) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemv_i8_decode_kernel<__nv_bfloat16, true>,
                                  cudaFuncAttributePreferredSharedMemoryCarveout, pct) == cudaSuccess;
  if (!ok) (void)cudaGetLastError();
  g_carveout_set[dev] = true;
}

}  // namespace

void prepare_gemv_decode() {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) prefer_l1(dev);
}

cudaError_t launch_gemv_decode(const GemmArgs& a, int num_sms, cudaStream_t s) {
  if (a.T == 0 || a.N == 0) return cudaSuccess;
  if (a.T > kDecodeMaxT) return cudaErrorInvalidValue;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) prefer_l1(dev);
  DvParams p;
  p.Xq = a.Xq;
  p.sA = a.sA;
  p.CB = a.CB;
  p.SCB = a.SCB;
  p.bias = a.bias;
  p.Xo = a.Xo;
  p.ldo = a.ldo;
  p.idx = a.idx;
  p.n_out = a.n_out;
  p.Wf = a.Wf;
  p.Y = a.Y;
  p.acc_out = a.acc_out;
  p.yd = make_ydst(a);
  p.T = a.T;
  p.N = a.N;
  p.K = a.K;
  p.mode = a.mode;
  const int64_t groups = a.N / 8;
  const int64_t max_grid = static_cast<int64_t>(num_sms) * 2;
  const int64_t passes = (groups + DV_RG - 1) / DV_RG;
  int64_t grid = max_grid;
  p.unit = 1;
  if (passes > 2 * max_grid) {
    // Whole passes per CTA once there are 3 or more per CTA: e.g. 1792
    // passes -> 256 CTAs of 7 rather than 296 CTAs of 6 or 7 (the BLOOM FFN-up
    // width, 3.6 % faster at one token).  With 1 or 2 short passes per CTA the
    // product is latency-bound and the full grid measured faster.
    const int64_t per = (passes + max_grid - 1) / max_grid;
    grid = (passes + per - 1) / per;
    p.unit = DV_RG;
  }
  if (grid > groups) grid = groups;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(DV_THREADS, 1, 1);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  const bool extra = p.yd.n > 0;
  if (a.dtype == kBF16)
    return extra ? cudaLaunchKernelEx(&cfg, gemv_i8_decode_kernel<__nv_bfloat16, true>, p)
                 : cudaLaunchKernelEx(&cfg, gemv_i8_decode_kernel<__nv_bfloat16, false>, p);
  return extra ? cudaLaunchKernelEx(&cfg, gemv_i8_decode_kernel<__half, true>, p)
               : cudaLaunchKernelEx(&cfg, gemv_i8_decode_kernel<__half, false>, p);
}

}  // namespace i8mp
