// Prefill GEMM of the LLM.int8() forward linear layer, pair-of-SMs version.
//
// Same computation as gemm_tc.cu (int8 product over the non-outlier columns,
// fp16 product over the outlier columns, dequantise with the row and column
// absmax constants and add the bias: steps 2-3 of "Core idea of LLM.int8()" on
// the Hugging Face integration page).  A 2-CTA cluster computes a 256 x 512
// output tile with two tcgen05.mma.cta_group::2 of M=256, N=256 per K-step:
//   * CTA r of the pair holds rows [128r, 128r+128) of the A tile and, for
//     each N half h, rows [256h + 128r, 256h + 128r + 128) of the B tile, so an
//     SM streams 48 KB per 128-byte K-block for 128 x 512 outputs (a 256 x 256
//     pair tile streams 32 KB for 128 x 256: a third more bytes per MAC, and
//     operand traffic from L2 is what bounds the full grid);
//   * each CTA's TMEM (512 columns) holds its 128 output rows x 512 columns,
//     one tile at a time: the epilogue of a tile does not overlap the next
//     tile's MMAs (measured: the traffic saving outweighs that);
//   * the even CTA (leader) issues the MMAs; both CTAs' TMA loads complete on
//     the leader's "full" barrier, and the leader's commits arrive on both
//     CTAs' "empty", "TMEM full" and "outliers added" barriers;
//   * both CTAs' epilogues arrive on the leader's "TMEM empty" and "partials
//     written" barriers.
// Outlier columns (the 16-bit product), with TMEM full: after the int8
// K-blocks the epilogue rewrites each accumulator in place as the fp32 partial
// output acc * sA * SCB / 127^2 + bias (tcgen05.st), the leader then issues
// the kind::f16 MMAs over the outlier columns accumulating onto it, and a
// second epilogue pass converts to the 16-bit output.
// Epilogue: 16 warps per CTA, 4 per TMEM lane quarter, each owning 32 rows
// x 128 columns (4 chunks of 32): a warp's chunks run one after another, and
// 16 warps measured 5 % faster than 8 at the Llama width, 1-2.5 % at the
// BLOOM and density-sweep shapes.  Y leaves by TMA stores: each epilogue warp
// packs its 32 x 32 block into its 2 KB shared-memory buffer and issues one
// tiled store.  With extra destinations (the N-sharded forward) the epilogue
// stores directly.
// No TMA load uses cluster multicast: each CTA loads its own halves.
#include <cuda.h>

#include "kernels.h"

namespace i8mp {
namespace {

constexpr int BM = 128;           // rows per CTA (256 per pair)
constexpr int BN = 512;           // output columns per tile
constexpr int BN_MMA = 256;       // N of one pair MMA
constexpr int BN_BOX = 128;       // B rows per CTA per MMA
constexpr int BKB = 128;          // bytes of K per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BKB;       // 16 KB
constexpr int B_BYTES = 2 * BN_BOX * BKB;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// Epilogue warps per CTA: 4 per TMEM lane quarter with 16 (each owning 128
// columns, 4 chunks of 32) or 2 with 8 (256 columns, 8 chunks).  A warp's
// chunks run one after another, so more warps shorten the epilogue.
#ifndef I8MP_PAIR_EPI_WARPS
#define I8MP_PAIR_EPI_WARPS 16
#endif
constexpr int NUM_EPI_WARPS = I8MP_PAIR_EPI_WARPS;
static_assert(NUM_EPI_WARPS == 8 || NUM_EPI_WARPS == 16, "2 or 4 epilogue warps per TMEM lane quarter");
constexpr int EPI_COLS = BN / (NUM_EPI_WARPS / 4);  // output columns per epilogue warp
constexpr int EPI_CHUNKS = EPI_COLS / 32;
constexpr int THREADS = 64 + NUM_EPI_WARPS * 32;
constexpr int YST_BYTES = 32 * 32 * 2;  // one epilogue warp's 32 x 32 block of Y
// staging buffers per warp: with 8 warps one fills while the other is
// stored; with 16, one (shared memory holds no more beside 4 stages)
constexpr int YST_BUFS = NUM_EPI_WARPS == 8 ? 2 : 1;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NUM_EPI_WARPS * YST_BUFS * YST_BYTES + 1024;
// Pair tiles (256 rows) per raster group: a group sweeps N with GROUP_M
// m-blocks side by side, so each B panel is streamed once per group.
#ifndef I8MP_PAIR_GROUP_M
#define I8MP_PAIR_GROUP_M 16
#endif
constexpr int GROUP_M = I8MP_PAIR_GROUP_M;
// L2 eviction hints: Y is written once and never read here (evict first, so
// that it does not push the A panels a raster group re-reads out of L2);
// optionally the A panels (X codes) are marked evict-last.
#ifndef I8MP_Y_EVICT_FIRST
#define I8MP_Y_EVICT_FIRST 1
#endif
#ifndef I8MP_A_EVICT_LAST
#define I8MP_A_EVICT_LAST 0
#endif

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_I8 = idesc_i8_s32(2 * BM, BN_MMA);
constexpr uint16_t PAIR_MASK = 0x3;

constexpr uint32_t W_EMPTY = 0x201, W_FULL = 0x202, W_TEMPTY = 0x203, W_TFULL = 0x204, W_DRAIN = 0x205,
                   W_TEARDOWN = 0x206, W_MID = 0x207, W_OFULL = 0x208;

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
  int tma_y;     // Y leaves through shared memory by TMA stores (no extra destinations)
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
    gemm_i8_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmAo, const __grid_constant__ CUtensorMap tmBo,
                       const __grid_constant__ CUtensorMap tmY, const Params p) {
  constexpr uint32_t kIdescO = idesc_f16_f32(2 * BM, BN_MMA, Elem<TE>::kMmaFormat);  // 16-bit outlier MMA
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];   // used in the leader only
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar;         // int8 product in TMEM
  __shared__ __align__(8) uint64_t tempty_bar;        // TMEM free again (used in the leader only)
  __shared__ __align__(8) uint64_t mid_bar;           // fp32 partial outputs in TMEM (leader only)
  __shared__ __align__(8) uint64_t ofull_bar;         // outlier product added
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  const int num_m = static_cast<int>((p.T + 2 * BM - 1) / (2 * BM));
  const int num_n = static_cast<int>((p.N + BN - 1) / BN);
  const int num_tiles = num_m * num_n;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&tfull_bar, 1);
    mbar_init(&tempty_bar, 2 * NUM_EPI_WARPS);
    mbar_init(&mid_bar, 2 * NUM_EPI_WARPS);
    mbar_init(&ofull_bar, 1);
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmAo);
    tma_prefetch_desc(&tmBo);
    if (p.tma_y) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  // The set-up above overlaps the tail of the row quantisation (programmatic
  // launch).  Every read of what the preceding kernels wrote (A, sA, n_out,
  // the outlier operands) follows griddepcontrol.wait in the role that makes
  // it; CB, SCB and bias are not written by them.
  // Outlier K-blocks: n_out comes from the outlier pass (completed before the
  // row quantisation this kernel waits for); clamped to [0, K] like every
  // reader of it.
  auto outlier_kblocks = [&]() -> int {
    int n_out = (p.n_out != nullptr && p.mode == 0) ? ld_dep_i32(p.n_out) : 0;
    n_out = n_out < 0 ? 0 : (n_out > p.K ? static_cast<int>(p.K) : n_out);
    return (n_out + 63) / 64;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
#if I8MP_A_EVICT_LAST
      const uint64_t pol_a = l2_policy_evict_last();
#endif
      int s = 0;
      uint32_t ph = 0;
      int issued[STAGES];
      #pragma unroll
      for (int i = 0; i < STAGES; ++i) issued[i] = 0;
      // The B halves (CB) of the first tile's first K-blocks go out before the
      // wait: the stages are fresh, and CB is not an output of the preceding
      // kernels.  Their A halves follow the wait.
      int pre = 0;
      if (pair < num_tiles) {
        int m_blk, n_blk;
        tile_coords(pair, num_m, num_n, m_blk, n_blk);
        const int row_b = n_blk * BN + static_cast<int>(rank) * BN_BOX;
        pre = p.nkb_i8 < STAGES ? p.nkb_i8 : STAGES;
        for (int kb = 0; kb < pre; ++kb) {
          uint8_t* sb = smem + kb * STAGE_BYTES + A_BYTES;
          if (leader) mbar_arrive_expect_tx(&full_bar[kb], 2 * STAGE_BYTES);
          const uint32_t fb = leader_smem_addr(smem_u32(&full_bar[kb]));
          tma_load_2d_pair(sb, &tmB, fb, kb * BKB, row_b);
          tma_load_2d_pair(sb + BN_BOX * BKB, &tmB, fb, kb * BKB, row_b + BN_MMA);
        }
      }
      griddep_wait();
      int nkb_o = -1;  // read when the first outlier K-block is reached
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int m_blk, n_blk;
        tile_coords(tile, num_m, num_n, m_blk, n_blk);
        const int row_a = m_blk * 2 * BM + static_cast<int>(rank) * BM;
        const int row_b = n_blk * BN + static_cast<int>(rank) * BN_BOX;
        for (int kb = 0;; ++kb) {
          if (kb >= p.nkb_i8) {
            if (nkb_o < 0) nkb_o = outlier_kblocks();
            if (kb >= p.nkb_i8 + nkb_o) break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          const uint32_t fb = leader_smem_addr(smem_u32(&full_bar[s]));
          if (tile == pair && kb < pre) {
            // stage s == kb: armed and its B halves issued before the wait
#if I8MP_A_EVICT_LAST
            tma_load_2d_pair_hint(sa, &tmA, fb, kb * BKB, row_a, pol_a);
#else
            tma_load_2d_pair(sa, &tmA, fb, kb * BKB, row_a);
#endif
          } else {
            if (!mbar_wait(&empty_bar[s], ph ^ 1u, &abort_sh, p.st, W_EMPTY)) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * STAGE_BYTES);
            if (kb < p.nkb_i8) {
#if I8MP_A_EVICT_LAST
              tma_load_2d_pair_hint(sa, &tmA, fb, kb * BKB, row_a, pol_a);
#else
              tma_load_2d_pair(sa, &tmA, fb, kb * BKB, row_a);
#endif
              tma_load_2d_pair(sb, &tmB, fb, kb * BKB, row_b);
              tma_load_2d_pair(sb + BN_BOX * BKB, &tmB, fb, kb * BKB, row_b + BN_MMA);
            } else {
              const int ko = kb - p.nkb_i8;
              tma_load_2d_pair(sa, &tmAo, fb, ko * 64, row_a);
              tma_load_2d_pair(sb, &tmBo, fb, ko * 64, row_b);
              tma_load_2d_pair(sb + BN_BOX * BKB, &tmBo, fb, ko * 64, row_b + BN_MMA);
            }
          }
          ++issued[s];
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // The leader's full barriers count both CTAs' loads: once every armed
      // phase has completed, no load of either CTA is still in flight.
      if (leader) {
        for (int i = 0; i < STAGES; ++i) {
          if (issued[i] > 0) {
            volatile int never = 0;
            mbar_wait(&full_bar[i], static_cast<uint32_t>((issued[i] - 1) & 1), &never, p.st, W_TEARDOWN);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      griddep_wait();
      const int nkb_o = outlier_kblocks();
      const int nkb = p.nkb_i8 + nkb_o;
      const bool has_out = nkb_o > 0;  // outlier product accumulated onto the fp32 partial outputs in TMEM
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++it) {
        const uint32_t aph = static_cast<uint32_t>(it & 1);
        if (!mbar_wait_cluster(&tempty_bar, aph ^ 1u, &abort_sh, p.st, W_TEMPTY)) break;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (kb == p.nkb_i8) {
            // int8 product done; the epilogue rewrites it in place as fp32
            // partial outputs, onto which the outlier MMAs accumulate
            mma_commit_pair(&tfull_bar, PAIR_MASK);
            if (!mbar_wait_cluster(&mid_bar, aph, &abort_sh, p.st, W_MID)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait(&full_bar[s], ph, &abort_sh, p.st, W_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + A_BYTES);
          const uint64_t bdesc2 = sw128_kmajor_desc(a_addr + A_BYTES + BN_BOX * BKB);
          if (kb < p.nkb_i8) {
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
              mma_i8_pair(tmem_base, adesc + 2u * kk, bdesc + 2u * kk, IDESC_I8, accum);
              mma_i8_pair(tmem_base + 256u, adesc + 2u * kk, bdesc2 + 2u * kk, IDESC_I8, accum);
            }
          } else {
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f16_pair(tmem_base, adesc + 2u * kk, bdesc + 2u * kk, kIdescO, 1u);
              mma_f16_pair(tmem_base + 256u, adesc + 2u * kk, bdesc2 + 2u * kk, kIdescO, 1u);
            }
          }
          mma_commit_pair(&empty_bar[s], PAIR_MASK);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) mma_commit_pair(has_out ? &ofull_bar : &tfull_bar, PAIR_MASK);
      }
      mma_commit_pair(&drain_bar, 0x1);
      volatile int never = 0;
      mbar_wait(&drain_bar, 0u, &never, p.st, W_DRAIN);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    griddep_wait();
    const bool has_out = outlier_kblocks() > 0;
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // which EPI_COLS-column group of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int it = 0;
    // Column scales and bias of this warp's EPI_COLS columns of a tile: lane i holds
    // column 32c + i for chunk c.  They are loaded before the wait for the
    // accumulators, so they arrive while the MMAs run; a chunk takes its 32
    // columns' values by warp shuffles (one global round trip per tile
    // instead of one per chunk on the epilogue's critical path).
    float sc8[EPI_CHUNKS], bi8[EPI_CHUNKS];
    auto prefetch_scales = [&](int n_blk) {
      #pragma unroll
      for (int c = 0; c < EPI_CHUNKS; ++c) {
        const int64_t col = static_cast<int64_t>(n_blk) * BN + half * EPI_COLS + c * 32 + lane;
        const bool ok = col < p.N;
        sc8[c] = ok ? __ldg(&p.SCB[col]) : 0.0f;
        bi8[c] = (ok && p.bias != nullptr) ? Elem<TE>::to_float(static_cast<const TE*>(p.bias)[col]) : 0.0f;
      }
    };
    // the next chunk's values move to slot 0 (static register indices)
    auto next_chunk = [&]() {
      #pragma unroll
      for (int c = 0; c < EPI_CHUNKS - 1; ++c) {
        sc8[c] = sc8[c + 1];
        bi8[c] = bi8[c + 1];
      }
    };
    // 32 outputs of this warp's 32 rows from gcol0 (one row per lane) to Y.
    // TMA path: the block goes through one of the warp's two staging buffers;
    // rows and columns outside Y are clipped by the store.  Otherwise direct
    // stores, to Y and its extra destinations.
    uint8_t* const ystage = smem + STAGES * STAGE_BYTES + (warp - 2) * YST_BUFS * YST_BYTES;
#if I8MP_Y_EVICT_FIRST
    const uint64_t pol_y = l2_policy_evict_first();
#endif
    int ybuf = 0;
    int ystores = 0;
    auto store_y = [&](int64_t row, bool row_ok, int64_t row0, int64_t gcol0, const uint32_t (&packed)[16]) {
      if (p.tma_y) {
        uint8_t* buf = ystage + ybuf * YST_BYTES;
        if (ystores >= YST_BUFS) {
          if (lane == 0) bulk_wait_read<YST_BUFS - 1>();  // this buffer's previous store has read it
          __syncwarp();
        }
        uint4* d = reinterpret_cast<uint4*>(buf + lane * 64);
        #pragma unroll
        for (int g = 0; g < 4; ++g)
          d[g] = make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#if I8MP_Y_EVICT_FIRST
          tma_store_2d_hint(&tmY, buf, static_cast<int32_t>(gcol0), static_cast<int32_t>(row0), pol_y);
#else
          tma_store_2d(&tmY, buf, static_cast<int32_t>(gcol0), static_cast<int32_t>(row0));
#endif
          bulk_commit();
        }
        ybuf = ybuf + 1 == YST_BUFS ? 0 : ybuf + 1;  // stays within this warp's YST_BUFS buffers
        ++ystores;
        return;
      }
      if (!row_ok) return;
      const int64_t off = row * p.yd.ld + gcol0;
      TE* dst = static_cast<TE*>(p.Y) + off;
      #pragma unroll
      for (int g = 0; g < 4; ++g)
        if (gcol0 + g * 8 + 8 <= p.N) {
          const uint4 v = make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
          reinterpret_cast<uint4*>(dst)[g] = v;
          if (p.yd.n > 0) store_extra_u4<TE>(p.yd, off + g * 8, v);
        }
    };
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      const uint32_t aph = static_cast<uint32_t>(it & 1);
      int m_blk, n_blk;
      tile_coords(tile, num_m, num_n, m_blk, n_blk);
      const int64_t row = static_cast<int64_t>(m_blk) * 2 * BM + static_cast<int64_t>(rank) * BM + q * 32 + lane;
      const bool row_ok = row < p.T;
      if (p.mode == 0) prefetch_scales(n_blk);
      const float ra = (row_ok && p.mode == 0) ? ld_dep_f32(&p.sA[row]) * (1.0f / 16129.0f) : 0.0f;
      if (!mbar_wait_cluster(&tfull_bar, aph, &abort_sh, p.st, W_TFULL)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + lane_base;
      if (has_out) {
        // pass 1: acc * sA * SCB / 127^2 + bias as fp32, written back in place
        #pragma unroll 1
        for (int c = 0; c < EPI_CHUNKS; ++c) {
          const int col0 = half * EPI_COLS + c * 32;
          uint32_t acc[32];
          tmem_ld_32x32b_x32(t_row + col0, acc);
          tmem_ld_wait();
          #pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sc = __shfl_sync(0xffffffffu, sc8[0], i);
            const float bi = __shfl_sync(0xffffffffu, bi8[0], i);
            acc[i] = __float_as_uint(fmaf(static_cast<float>(static_cast<int32_t>(acc[i])), ra * sc, bi));
          }
          tmem_st_32x32b_x32(t_row + col0, acc);
          next_chunk();
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(&mid_bar, 0);
        if (!mbar_wait_cluster(&ofull_bar, aph, &abort_sh, p.st, W_OFULL)) break;
        tc_fence_after();
        // pass 2: the outlier product has been added; convert and store
        #pragma unroll 1
        for (int c = 0; c < EPI_CHUNKS; ++c) {
          const int col0 = half * EPI_COLS + c * 32;
          const int64_t gcol0 = static_cast<int64_t>(n_blk) * BN + col0;
          uint32_t yv[32];
          tmem_ld_32x32b_x32(t_row + col0, yv);
          tmem_ld_wait();
          uint32_t packed[16];
          #pragma unroll
          for (int i = 0; i < 32; i += 2)
            packed[i >> 1] = Elem<TE>::pack2(__uint_as_float(yv[i]), __uint_as_float(yv[i + 1]));
          store_y(row, row_ok, row - lane, gcol0, packed);
        }
      } else {
        #pragma unroll 1
        for (int c = 0; c < EPI_CHUNKS; ++c) {
          const int col0 = half * EPI_COLS + c * 32;
          const int64_t gcol0 = static_cast<int64_t>(n_blk) * BN + col0;
          uint32_t acc[32];
          tmem_ld_32x32b_x32(t_row + col0, acc);
          tmem_ld_wait();
          if (p.mode == 1) {
            if (row_ok) {
              int32_t* dst = p.acc_out + row * p.N + gcol0;
              #pragma unroll
              for (int g = 0; g < 8; ++g)
                if (gcol0 + g * 4 + 4 <= p.N)
                  reinterpret_cast<int4*>(dst)[g] =
                      make_int4(acc[4 * g], acc[4 * g + 1], acc[4 * g + 2], acc[4 * g + 3]);
            }
            continue;
          }
          uint32_t packed[16];
          #pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float s0 = __shfl_sync(0xffffffffu, sc8[0], i), s1 = __shfl_sync(0xffffffffu, sc8[0], i + 1);
            const float b0 = __shfl_sync(0xffffffffu, bi8[0], i), b1 = __shfl_sync(0xffffffffu, bi8[0], i + 1);
            const float y0 = fmaf(static_cast<float>(static_cast<int32_t>(acc[i])), ra * s0, b0);
            const float y1 = fmaf(static_cast<float>(static_cast<int32_t>(acc[i + 1])), ra * s1, b1);
            packed[i >> 1] = Elem<TE>::pack2(y0, y1);
          }
          next_chunk();
          store_y(row, row_ok, row - lane, gcol0, packed);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(&tempty_bar, 0);
    }
    if (p.tma_y && lane == 0) bulk_wait<0>();  // every Y store of this warp has completed
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's MMAs have drained before either CTA releases TMEM or exits
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

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

bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major 16-bit Y in 32 x 32 boxes, no swizzle (one epilogue warp's block).
bool make_map_y(CUtensorMap* m, void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                uint64_t row_stride_bytes) {
  EncodeFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int g_max_pairs[64] = {0};

}  // namespace

// Largest number of co-resident 2-CTA clusters of the pair kernel on the
// current device (0 if clusters of this kernel cannot be launched).
int pair_kernel_max_clusters() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (g_max_pairs[dev] != 0) return g_max_pairs[dev];
  if (cudaFuncSetAttribute(gemm_i8_tc2_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
          cudaSuccess ||
      cudaFuncSetAttribute(gemm_i8_tc2_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SMEM_BYTES) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_i8_tc2_kernel<__half>, &cfg) != cudaSuccess) return 0;
  g_max_pairs[dev] = n;
  return n;
}

cudaError_t launch_gemm_tc2(const GemmArgs& a, cudaStream_t s) {
  const int max_pairs = pair_kernel_max_clusters();
  if (max_pairs <= 0) return cudaErrorNotSupported;
  if (a.T == 0 || a.N == 0) return cudaSuccess;
  CUtensorMap tmA, tmB, tmAo, tmBo;
  if (!make_map(&tmA, a.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.K, a.T, a.K, BKB, BM)) return cudaErrorInvalidValue;
  if (!make_map(&tmB, a.CB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.K, a.N, a.K, BKB, BN_BOX)) return cudaErrorInvalidValue;
  const bool outl = a.mode == 0 && a.n_out != nullptr && a.Xo != nullptr && a.Wo != nullptr;
  const CUtensorMapDataType t16 = a.dtype == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (outl) {
    if (!make_map(&tmAo, a.Xo, t16, a.ldo, a.T, a.ldo * 2, 64, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tmBo, a.Wo, t16, a.ldo, a.N, a.ldo * 2, 64, BN_BOX))
      return cudaErrorInvalidValue;
  } else {
    tmAo = tmA;
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
  // Y by TMA stores when it has no extra destinations and its rows are
  // 16-byte multiples (the tensor map's stride rule)
  CUtensorMap tmY = tmA;
  p.tma_y = 0;
  if (a.mode == 0 && p.yd.n == 0 && p.yd.ld % 8 == 0 && reinterpret_cast<uintptr_t>(a.Y) % 16 == 0 &&
      a.T <= 0x7fffffff && a.N <= 0x7fffffff &&
      make_map_y(&tmY, a.Y, t16, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.T),
                 static_cast<uint64_t>(p.yd.ld) * 2))
    p.tma_y = 1;
  const int64_t tiles = ((a.T + 2 * BM - 1) / (2 * BM)) * ((a.N + BN - 1) / BN);
  if (tiles > 0x3fffffff) return cudaErrorInvalidValue;
  const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  if (a.dtype == kBF16)
    return cudaLaunchKernelEx(&cfg, gemm_i8_tc2_kernel<__nv_bfloat16>, tmA, tmB, tmAo, tmBo, tmY, p);
  return cudaLaunchKernelEx(&cfg, gemm_i8_tc2_kernel<__half>, tmA, tmB, tmAo, tmBo, tmY, p);
}

}  // namespace i8mp
