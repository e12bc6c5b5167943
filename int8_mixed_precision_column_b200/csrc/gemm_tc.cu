// Prefill GEMM of the LLM.int8() forward linear layer on sm_100a tensor cores.
//
// Computes, per output tile of 128 tokens x 256 output features,
//   acc[t,j] = sum_k Xq[t,k] * CB[j,k]                 (tcgen05 kind::i8, int32 in TMEM)
//   Yo[t,j]  = sum_o Xo[t,o] * Wo[j,o]                 (tcgen05 kind::f16, fp32 in TMEM)
//   Y[t,j]   = TE(acc * sA[t] * SCB[j] / 127^2 + Yo + bias[j])   (TE: fp16 or bf16)
// i.e. steps 2 and 3 of "Core idea of LLM.int8()" on the Hugging Face
// integration page (int8 vector-wise product for the bulk, 16-bit product for
// the outlier columns, dequantise and sum), with the vector-wise constants of
// the inference-research record's "Activation scheme" (one constant per row
// of X and per row of W, i.e. per inner product).
//
// Structure (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: fills a 4-stage ring of 48 KB stages.  An int8
//               K-block is 128 bytes wide (A 128x128 B, B 256x128 B); an fp16
//               outlier K-block is 64 halves = 128 bytes wide, so both kinds
//               share the ring and the 128-byte swizzle layout.
//   warp 1      TMEM allocation (512 columns) and the single MMA-issuing thread.
//   warps 2..9  epilogue: tcgen05.ld of the accumulators, dequant + outlier
//               + bias, 16-bit stores.
// TMEM use: with no outlier columns, two int32 accumulators (columns 0 and 256)
// let the epilogue of one tile overlap the main loop of the next; with outlier
// columns, columns 0..255 hold the int32 and 256..511 the fp32 accumulator.
// No cluster multicast is used anywhere; the L2 absorbs the reuse of A and B
// panels between CTAs (grouped tile order).
#include <cuda.h>

#include "kernels.h"

namespace i8mp {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BKB = 128;  // bytes of K per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BKB;
constexpr int B_BYTES = BN * BKB;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int THREADS = 64 + NUM_EPI_WARPS * 32;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
constexpr int GROUP_M = 16;  // m-tiles per raster group
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_I8 = idesc_i8_s32(BM, BN);

// wait tags reported in DevStatus::where
constexpr uint32_t W_EMPTY = 0x101, W_FULL = 0x102, W_TEMPTY = 0x103, W_TFULL = 0x104, W_DRAIN = 0x105,
                   W_TEARDOWN = 0x106;

struct Params {
  int64_t T, N, K;
  int nkb_i8;
  const float* sA;
  const float* SCB;
  const void* bias;  // TE[N] or null
  void* Y;           // TE[T,N]
  int32_t* acc_out;
  YDst yd;           // row stride of Y and its extra destinations
  const int32_t* n_out;
  DevStatus* st;
  int mode;
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& m_blk, int& n_blk) {
  const int group_size = GROUP_M * num_n;
  const int g = tile / group_size;
  const int first_m = g * GROUP_M;
  const int gm = min(num_m - first_m, GROUP_M);
  const int local = tile - g * group_size;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

template <typename TE>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_i8_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmAo, const __grid_constant__ CUtensorMap tmBo,
                      const Params p) {
  constexpr uint32_t kIdescO = idesc_f16_f32(BM, BN, Elem<TE>::kMmaFormat);  // 16-bit outlier MMA
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int num_m = static_cast<int>((p.T + BM - 1) / BM);
  const int num_n = static_cast<int>((p.N + BN - 1) / BN);
  const int num_tiles = num_m * num_n;
  griddep_wait();  // n_out and the operands come from the preceding kernels
  int n_out = (p.n_out != nullptr) ? ld_dep_i32(p.n_out) : 0;  // clamped to [0, K] like every reader of it
  n_out = n_out < 0 ? 0 : (n_out > p.K ? static_cast<int>(p.K) : n_out);
  const int nkb_o = (p.mode == 0) ? (n_out + 63) / 64 : 0;
  const int nkb = p.nkb_i8 + nkb_o;
  const bool has_out = nkb_o > 0;
  const int nbuf = has_out ? 1 : 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], NUM_EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (has_out) {
      tma_prefetch_desc(&tmAo);
      tma_prefetch_desc(&tmBo);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued[STAGES];
      #pragma unroll
      for (int i = 0; i < STAGES; ++i) issued[i] = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(tile, num_m, num_n, m_blk, n_blk);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty_bar[s], ph ^ 1u, &abort_sh, p.st, W_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
          if (kb < p.nkb_i8) {
            tma_load_2d(sa, &tmA, &full_bar[s], kb * BKB, m_blk * BM);
            tma_load_2d(sb, &tmB, &full_bar[s], kb * BKB, n_blk * BN);
          } else {
            const int ko = kb - p.nkb_i8;
            tma_load_2d(sa, &tmAo, &full_bar[s], ko * 64, m_blk * BM);
            tma_load_2d(sb, &tmBo, &full_bar[s], ko * 64, n_blk * BN);
          }
          ++issued[s];
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // Every TMA load this thread issued must land before the CTA may exit.
      for (int i = 0; i < STAGES; ++i) {
        if (issued[i] > 0) {
          volatile int never = 0;
          mbar_wait(&full_bar[i], static_cast<uint32_t>((issued[i] - 1) & 1), &never, p.st, W_TEARDOWN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int buf = it % nbuf;
        const uint32_t aph = static_cast<uint32_t>((it / nbuf) & 1);
        if (!mbar_wait(&tempty_bar[buf], aph ^ 1u, &abort_sh, p.st, W_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d_i32 = tmem_base + static_cast<uint32_t>(buf) * 256u;
        const uint32_t d_f32 = tmem_base + 256u;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[s], ph, &abort_sh, p.st, W_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + A_BYTES);
          if (kb < p.nkb_i8) {
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(d_i32, adesc + 2u * kk, bdesc + 2u * kk, IDESC_I8, (kb | kk) != 0 ? 1u : 0u);
          } else {
            const int ko = kb - p.nkb_i8;
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(d_f32, adesc + 2u * kk, bdesc + 2u * kk, kIdescO, (ko | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty_bar[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) mma_commit(&tfull_bar[buf]);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is released.
      mma_commit(&drain_bar);
      volatile int never = 0;
      mbar_wait(&drain_bar, 0u, &never, p.st, W_DRAIN);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;    // which 128 of the 256 columns
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int buf = it % nbuf;
      const uint32_t aph = static_cast<uint32_t>((it / nbuf) & 1);
      int m_blk, n_blk;
      tile_coords(tile, num_m, num_n, m_blk, n_blk);
      const int64_t row = static_cast<int64_t>(m_blk) * BM + q * 32 + lane;
      const bool row_ok = row < p.T;
      // this warp's 128 columns: lane i holds the scale and bias of column
      // 32c + i of chunk c, loaded before the wait for the accumulators (they
      // arrive while the MMAs run)
      float sc4[4], bi4[4];
      #pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int64_t col = static_cast<int64_t>(n_blk) * BN + half * 128 + c * 32 + lane;
        const bool ok = p.mode == 0 && col < p.N;
        sc4[c] = ok ? __ldg(&p.SCB[col]) : 0.0f;
        bi4[c] = (ok && p.bias != nullptr) ? Elem<TE>::to_float(static_cast<const TE*>(p.bias)[col]) : 0.0f;
      }
      const float ra = (row_ok && p.mode == 0) ? ld_dep_f32(&p.sA[row]) * (1.0f / 16129.0f) : 0.0f;
      if (!mbar_wait(&tfull_bar[buf], aph, &abort_sh, p.st, W_TFULL)) break;
      tc_fence_after();
      #pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int col0 = half * 128 + c * 32;
        const int64_t gcol0 = static_cast<int64_t>(n_blk) * BN + col0;
        uint32_t acc[32];
        uint32_t fo[32];
        tmem_ld_32x32b_x32(tmem_base + lane_base + static_cast<uint32_t>(buf) * 256u + col0, acc);
        if (has_out) tmem_ld_32x32b_x32(tmem_base + lane_base + 256u + col0, fo);
        tmem_ld_wait();
        if (p.mode == 1) {
          if (row_ok) {
            int32_t* dst = p.acc_out + row * p.N + gcol0;
            #pragma unroll
            for (int g = 0; g < 8; ++g)
              if (gcol0 + g * 4 + 4 <= p.N)
                reinterpret_cast<int4*>(dst)[g] = make_int4(acc[4 * g], acc[4 * g + 1], acc[4 * g + 2], acc[4 * g + 3]);
          }
          continue;
        }
        const float scb_l = sc4[0], b_l = bi4[0];
        #pragma unroll
        for (int k = 0; k < 3; ++k) {  // the next chunk's values move to slot 0
          sc4[k] = sc4[k + 1];
          bi4[k] = bi4[k + 1];
        }
        uint32_t packed[16];
        #pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float s0 = __shfl_sync(0xffffffffu, scb_l, i);
          const float s1 = __shfl_sync(0xffffffffu, scb_l, i + 1);
          const float b0 = __shfl_sync(0xffffffffu, b_l, i);
          const float b1 = __shfl_sync(0xffffffffu, b_l, i + 1);
          float y0 = static_cast<float>(static_cast<int32_t>(acc[i])) * (ra * s0) + b0;
          float y1 = static_cast<float>(static_cast<int32_t>(acc[i + 1])) * (ra * s1) + b1;
          if (has_out) {
            y0 += __uint_as_float(fo[i]);
            y1 += __uint_as_float(fo[i + 1]);
          }
          packed[i >> 1] = Elem<TE>::pack2(y0, y1);
        }
        if (row_ok) {
          const int64_t off = row * p.yd.ld + gcol0;
          TE* dst = static_cast<TE*>(p.Y) + off;
          #pragma unroll
          for (int g = 0; g < 4; ++g)
            if (gcol0 + g * 8 + 8 <= p.N) {
              const uint4 v = make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
              reinterpret_cast<uint4*>(dst)[g] = v;
              if (p.yd.n > 0) store_extra_u4<TE>(p.yd, off + g * 8, v);
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode_fn() {
  static EncodeFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  }
  return fn;
}

// 2-D K-major tile map: inner dim = K (elements), outer = rows; 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
              uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  (void)elem_bytes;
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmArgs& a, int num_sms, cudaStream_t s) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_done[dev]) {
    e = cudaFuncSetAttribute(gemm_i8_tc_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_i8_tc_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  if (a.T == 0 || a.N == 0) return cudaSuccess;
  CUtensorMap tmA, tmB, tmAo, tmBo;
  if (!make_map(&tmA, a.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.T, a.K, BKB, BM)) return cudaErrorInvalidValue;
  if (!make_map(&tmB, a.CB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.K, a.N, a.K, BKB, BN)) return cudaErrorInvalidValue;
  const bool outl = a.mode == 0 && a.n_out != nullptr && a.Xo != nullptr && a.Wo != nullptr;
  const CUtensorMapDataType t16 = a.dtype == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (outl) {
    if (!make_map(&tmAo, a.Xo, t16, 2, a.ldo, a.T, a.ldo * 2, 64, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tmBo, a.Wo, t16, 2, a.ldo, a.N, a.ldo * 2, 64, BN))
      return cudaErrorInvalidValue;
  } else {
    tmAo = tmA;  // never read: the kernel runs no outlier K-blocks
    tmBo = tmB;
  }
  Params p;
  p.T = a.T;
  p.N = a.N;
  p.K = a.K;
  p.nkb_i8 = static_cast<int>((a.K + BKB - 1) / BKB);
  p.sA = a.sA;
  p.SCB = a.SCB;
  p.bias = a.bias;
  p.Y = a.Y;
  p.acc_out = a.acc_out;
  p.yd = make_ydst(a);
  p.n_out = outl ? a.n_out : nullptr;
  p.st = a.st;
  p.mode = a.mode;
  const int64_t tiles = ((a.T + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  if (tiles > 0x7fffffff) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  if (a.dtype == kBF16) return cudaLaunchKernelEx(&cfg, gemm_i8_tc_kernel<__nv_bfloat16>, tmA, tmB, tmAo, tmBo, p);
  return cudaLaunchKernelEx(&cfg, gemm_i8_tc_kernel<__half>, tmA, tmB, tmAo, tmBo, p);
}

}  // namespace i8mp
