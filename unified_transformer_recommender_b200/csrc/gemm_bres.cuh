// Weight-resident persistent tensor-core GEMM for K = 256 (sm_100a):
//
//   C[(m,g), n] = epi( sum_k A[(m,g), k] * W[grp][n_lo + n][k] )
//
// With K = 256 a 128 x 256 output tile needs its A rows (64 KB) and a
// 256 x 256 weight slice (128 KB); a GEMM that streams both per tile moves
// twice as many weight bytes as activation bytes through L2 and waits on
// every stage.  Here each CTA owns one (weight group, 256-column) slice for
// the whole launch: the slice is loaded once into shared memory and only the
// A k-blocks of the CTA's row tiles stream, through a 4-slot ring of 16 KB.
// The CTAs of one slice split its row tiles into contiguous ranges.  One
// thread issues the 128 x 256 tcgen05.mma steps into one of two TMEM
// accumulators, so the MMAs of tile i+1 run while eight epilogue warps drain
// tile i (tcgen05.ld, bias / GELU / column scale, bf16) and send it out by TMA
// stores through a 32 KB staging area, half a tile at a time.  The training
// step's dz GEMM adds the GELU backward to the epilogue (ACT_GELU_BWD: u read
// per row, du out by TMA, GELU(u) stored per row), and its dX GEMMs load the
// slice from the forward's [K][N] weight as MN-major boxes (w_mn).
//
// Warp roles (320 threads): warps 0-7 epilogue (warp w and w+4 share TMEM
// lanes 32*(w%4).. and take one half of the tile's columns each), warp 8 TMA
// producer, warp 9 TMEM allocator and MMA issuer.
#pragma once
#include "gemm_tc.cuh"

namespace ot {

struct BresCfg {
  static constexpr int BM = 128, BN = 256, K = 256, KB = K / 64;
  static constexpr int A_STAGES = 4;
  static constexpr int A_BYTES = BM * 128;          // one k-block of A: 128 rows x 64 bf16
  static constexpr int B_BYTES = BN * 128;          // one k-block of the slice: 256 rows x 64 bf16
  static constexpr int W_BYTES = KB * B_BYTES;      // the resident slice: 128 KB
  static constexpr int OUT_BYTES = BM * 128 * 2;    // staging: half a tile, two boxes of 64 columns
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = W_BYTES + A_STAGES * A_BYTES + OUT_BYTES + BAR_BYTES;
  static constexpr int TMEM_COLS = 512;             // two accumulators of 256 columns
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (EPI_WARPS + 2) * 32;
};
static_assert(BresCfg::SMEM <= 232448, "shared memory of one CTA");

// 32 bf16 values (16 packed pairs) of row r into a K-major, 128-byte-swizzled
// staging tile: columns [col0, col0 + 32) of a tile whose 64-column boxes are
// 16 KB apart.
__device__ inline void st_sw128_pk32(uint8_t* tile, int r, int col0, const uint32_t* pk) {
  uint8_t* rowp = tile + (col0 >> 6) * 16384 + r * 128;
  const int ch0 = (col0 & 63) >> 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *(uint4*)(rowp + (((ch0 + i) ^ (r & 7)) << 4)) = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

__global__ void __launch_bounds__(BresCfg::THREADS, 1)
    gemm_bres_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmOut, const GemmDesc d, const int a_swap,
                     const int out_swap, const int tiles_n, const int tiles_m, const int n_slices,
                     const int ctas_per_slice) {
  using C = BresCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sW = smem;                                  // [KB][256 rows x 128 B]
  uint8_t* sA = sW + C::W_BYTES;                       // [A_STAGES][128 rows x 128 B]
  uint8_t* stage_out = sA + C::A_STAGES * C::A_BYTES;  // [2 boxes][128 rows x 128 B]
  uint64_t* bars = (uint64_t*)(stage_out + C::OUT_BYTES);
  uint64_t* w_full = bars;
  uint64_t* a_full = w_full + 1;                 // [A_STAGES]
  uint64_t* a_empty = a_full + C::A_STAGES;      // [A_STAGES]
  uint64_t* acc_full = a_empty + C::A_STAGES;    // [2]: accumulator holds a finished tile
  uint64_t* acc_empty = acc_full + 2;            // [2]: epilogue has read the accumulator
  uint32_t* tmem_slot = (uint32_t*)(acc_empty + 2);

  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  // this CTA's slice and row tiles
  const int slice = blockIdx.x / ctas_per_slice, part = blockIdx.x - slice * ctas_per_slice;
  if (slice >= n_slices) return;
  const int gi = slice / tiles_n;
  const int n0 = (slice - gi * tiles_n) * C::BN;
  const int g = d.g_lo + gi;
  const int grp = d.mode == TILE_SAMPLES ? g - d.grp_base : 0;
  const int rt0 = (int)((long long)part * tiles_m / ctas_per_slice);
  const int rt1 = (int)((long long)(part + 1) * tiles_m / ctas_per_slice);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kEpiThreads = C::EPI_WARPS * 32;

  if (threadIdx.x == 0) {
    mbar_init(w_full, 1);
    for (int s = 0; s < C::A_STAGES; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads);
    }
    fence_barrier_init();
  }
  if (warp == C::EPI_WARPS && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmOut);
  }
  if (warp == C::EPI_WARPS + 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the weight slice is not written by the previous kernel: its load starts
  // before the wait for that kernel
  if (warp == C::EPI_WARPS && lane == 0) {
    const uint64_t keep = l2_evict_last();
    mbar_expect_tx(w_full, C::W_BYTES);
    if (d.w_mn) {
      // [K][N] weight rows: per k-block four boxes of 64 columns x 64 rows (MN-major)
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
        for (int c = 0; c < C::BN / 64; ++c)
          tma_load_3d_hint(&tmB, w_full, sW + kb * C::B_BYTES + c * 8192, d.n_lo + n0 + c * 64, kb * 64, grp, keep);
    } else {
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_3d_hint(&tmB, w_full, sW + kb * C::B_BYTES, kb * 64, d.n_lo + n0, grp, keep);
    }
  }
  grid_dep_wait();
  grid_dep_launch();

  if (warp == C::EPI_WARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // A keeps the default L2 policy: the other column slices of the same
      // weight group read the same rows at about the same time
      int q = 0;  // ring position
      bool ok = true;
      for (int rt = rt0; rt < rt1 && ok; ++rt) {
        const int mt0 = d.m_lo + rt * C::BM;
        for (int kb = 0; kb < C::KB; ++kb, ++q) {
          const int s = q % C::A_STAGES;
          if (q >= C::A_STAGES && !mbar_wait(&a_empty[s], ((q / C::A_STAGES) - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = sA + s * C::A_BYTES;
          mbar_expect_tx(&a_full[s], C::A_BYTES);
          if (a_swap) tma_load_3d(&tmA, &a_full[s], sa, kb * 64, g, mt0);
          else tma_load_3d(&tmA, &a_full[s], sa, kb * 64, mt0, g);
        }
      }
    }
  } else if (warp == C::EPI_WARPS + 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = d.w_mn ? idesc_bf16(128, C::BN, false, true) : idesc_bf16(128, C::BN);
      const uint64_t da0 = sdesc_k128(smem_u32(sA));
      const uint64_t dw0 = d.w_mn ? sdesc_mn128(smem_u32(sW), 8192) : sdesc_k128(smem_u32(sW));
      const uint32_t kstep = d.w_mn ? 2048 : 32;   // 16 k: 16 rows of 128 B, or 32 bytes of a row
      bool ok = mbar_wait(w_full, 0);
      if (ok) tc_fence_after();
      int q = 0, j = 0;
      for (int rt = rt0; rt < rt1 && ok; ++rt, ++j) {
        const int acc = j & 1;
        if (j >= 2) {
          // the epilogue must have read this accumulator's previous tile
          ok = mbar_wait(&acc_empty[acc], ((j >> 1) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t tacc = tmem + (uint32_t)(acc * C::BN);
        for (int kb = 0; kb < C::KB; ++kb, ++q) {
          const int s = q % C::A_STAGES;
          ok = mbar_wait(&a_full[s], (q / C::A_STAGES) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint64_t da = desc_add(da0, s * C::A_BYTES), dw = desc_add(dw0, kb * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tacc, desc_add(da, k * 32), desc_add(dw, k * kstep), idesc, (kb | k) ? 1u : 0u);
          umma_commit(&a_empty[s]);
        }
        if (ok) umma_commit(&acc_full[acc]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3, half = warp >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t lb = (uint32_t)(q4 * 32) << 16;
    const __nv_bfloat16* bias = (const __nv_bfloat16*)d.bias;
    bool ok = true;
    int j = 0;
    for (int rt = rt0; rt < rt1; ++rt, ++j) {
      const int mt0 = d.m_lo + rt * C::BM;
      const int acc = j & 1;
      ok = ok && mbar_wait(&acc_full[acc], (j >> 1) & 1);
      tc_fence_after();
      // this thread's 128 columns of the tile (its half), as bf16 pairs
      uint32_t pk[64];
      int ob = 0, ot_ = 0;   // (b, t) of this thread's output row
      const bool row_ok = mt0 + r < d.m_lo + d.M;
      if (d.act == ACT_GELU_BWD && row_ok) row_of(d, mt0 + r, g, ob, ot_);
      const uint32_t tacc = tmem + (uint32_t)(acc * C::BN + half * (C::BN / 2)) + lb;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = n0 + half * (C::BN / 2) + c * 32;
        float v[32];
        tmem_ld32(tacc + c * 32, v);
        if (bias) {
          float bv[32];
          load_bf16x32(bias + (long long)grp * d.bias_sg + d.n_lo + n, bv);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += bv[i];
        }
        if (d.act == ACT_GELU) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_fast(v[i]);
        } else if (d.act == ACT_GELU_BWD && row_ok) {
          // v = dz; u from its rows: du = dz GELU'(u) leaves as the output, GELU(u) through act_out
          float uv[32];
          load_row32(d.act_in, rm_off(d.act_in, ob, ot_, n), uv);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float g;
            gelu_tanh_and_grad(uv[i], uv[i], g);
            v[i] *= g;
          }
          store_row32(d.act_out, rm_off(d.act_out, ob, ot_, n), uv);
        }
        if (n < d.scale_cols) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= d.col_scale;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[c * 16 + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      }
      // the accumulator is read: the MMA may start the tile after next in it
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      // the two halves leave one after the other through the staging area
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // the previous stores have finished reading the staging area
        if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (half == hh) {
#pragma unroll
          for (int c = 0; c < 4; ++c) st_sw128_pk32(stage_out, r, c * 32, pk + c * 16);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (threadIdx.x == 0 && ok) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int n = n0 + hh * (C::BN / 2) + i * 64;
            if (out_swap) tma_store_3d(&tmOut, stage_out + i * 16384, n, g, mt0);
            else tma_store_3d(&tmOut, stage_out + i * 16384, n, mt0, g);
          }
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
      }
    }
    // shared memory must stay valid until the last stores have read it
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::EPI_WARPS + 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
inline bool tc_bres_supported(const GemmDesc& d) {
  return d.K == BresCfg::K && d.out_kind == OUT_ROWS && !d.res.base && !d.rms.base && !d.out.f32 &&
         d.N % BresCfg::BN == 0 && tc_gemm_supported(d);
}

// ONETRANS_ERR_UNSUPPORTED when the output rows are not one TMA-addressable
// set, or when there are more weight slices than SMs (the caller then takes
// another kernel).
inline onetrans_status tc_bres_launch(const GemmDesc& d, int sm_count, cudaStream_t st) {
  using C = BresCfg;
  const int tiles_n = d.N / C::BN, tiles_m = (d.M + C::BM - 1) / C::BM;
  const long long n_slices = (long long)tiles_n * d.G;
  if (tiles_m <= 0 || n_slices <= 0) return ONETRANS_OK;
  if (n_slices > sm_count) return ONETRANS_ERR_UNSUPPORTED;
  const int cps = std::max(1, std::min(tiles_m, sm_count / (int)n_slices));
  CUtensorMap ta, tb, tout;
  int out_swap = 0;
  if (!make_gemm_out_tmap(&tout, d, C::BN / 2, C::OUT_BYTES, out_swap)) return ONETRANS_ERR_UNSUPPORTED;
  const uint64_t mext = (uint64_t)d.a_mext, gext = (uint64_t)d.a_gext;
  const uint64_t s_m = (uint64_t)d.a_sm, s_g = gext > 1 ? (uint64_t)d.a_sg : mext * (uint64_t)d.a_sm;
  const int a_swap = (gext > 1 && d.a_sg < d.a_sm) ? 1 : 0;
  bool ok = a_swap ? make_tmap_3d(&ta, d.A, d.K, gext, mext, s_g, s_m, 64, 1, 128)
                   : make_tmap_3d(&ta, d.A, d.K, mext, gext, s_m, s_g, 64, 128, 1);
  const uint64_t wg = (uint64_t)d.w_groups;
  const uint64_t w_sg = wg > 1 ? (uint64_t)d.w_sg : (uint64_t)d.w_rows * d.K;
  if (d.w_mn) ok = ok && make_tmap_3d(&tb, d.W, d.w_rows, d.K, wg, d.w_rows, w_sg, 64, 64, 1);
  else ok = ok && make_tmap_3d(&tb, d.W, d.K, d.w_rows, wg, d.K, w_sg, 64, C::BN, 1);
  if (!ok) return ONETRANS_ERR_CUDA;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gemm_bres_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return ONETRANS_ERR_CUDA;
    attr_set = true;
  }
  const int grid = (int)n_slices * cps;
  launch_dependent(gemm_bres_kernel, dim3(grid), dim3(C::THREADS), C::SMEM, st, ta, tb, tout, d, a_swap, out_swap,
                   tiles_n, tiles_m, (int)n_slices, cps);
  return cudaGetLastError() == cudaSuccess ? ONETRANS_OK : ONETRANS_ERR_CUDA;
}

}  // namespace ot
