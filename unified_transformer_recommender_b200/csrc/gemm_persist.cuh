// Persistent tensor-core GEMM for plain bf16 row outputs (sm_100a):
//
//   C[(m,g), n] = epi( sum_k A[(m,g), k] * W[grp][n_lo + n][k] )
//
// One CTA per SM walks the 128 x 256 output tiles of the launch (tile index
// n-fastest, so CTAs working at the same time read the same A rows and find
// them in L2).  A TMA producer warp streams the A and W k-blocks of tile
// after tile through a 3-stage ring without waiting for epilogues; one
// thread issues the 128 x 256 tcgen05.mma steps into one of two TMEM
// accumulators (256 columns each), so the MMAs of tile i+1 run while eight
// epilogue warps drain tile i: tcgen05.ld, bias / GELU / column scale, bf16
// into a shared-memory staging tile, TMA stores.  This hides the load latency
// and the epilogue that a one-tile-per-CTA kernel pays per tile.  Row-output
// GEMMs with K = 256 (the QKV projection) take the weight-resident kernel of
// gemm_bres.cuh; this one takes the others (the auto-split's K = 512 and
// 3072 among them).
//
// Warp roles (320 threads): warps 0-7 epilogue (warp w and w+4 share TMEM
// lanes 32*(w%4).. and take one half of the tile's columns each), warp 8
// TMA producer, warp 9 TMEM allocator and MMA issuer.
#pragma once
#include "gemm_tc.cuh"

namespace ot {

struct PersistCfg {
  static constexpr int BM = 128, BN = 256;
  static constexpr int STAGES = 3;
  static constexpr int A_BYTES = BM * 128;              // 128 rows x 64 bf16 of K
  static constexpr int B_BYTES = BN * 128;              // 256 rows x 64 bf16 of K
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
  static constexpr int OUT_BYTES = BM * BN * 2;          // staging: 4 boxes of 64 bf16 columns
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + OUT_BYTES + BAR_BYTES;
  static constexpr int TMEM_COLS = 512;                  // two accumulators of 256 columns
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (EPI_WARPS + 2) * 32;
};

__global__ void __launch_bounds__(PersistCfg::THREADS, 1)
    gemm_persist_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmOut, const GemmDesc d, const int a_swap,
                        const int out_swap, const int tiles_n, const int tiles_m, const int n_tiles) {
  using C = PersistCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint8_t* stage_out = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = (uint64_t*)(stage_out + C::OUT_BYTES);
  uint64_t* full = bars;                    // [STAGES]
  uint64_t* empty = full + C::STAGES;       // [STAGES]
  uint64_t* acc_full = empty + C::STAGES;   // [2]: accumulator holds a finished tile
  uint64_t* acc_empty = acc_full + 2;       // [2]: epilogue has read the accumulator
  uint32_t* tmem_slot = (uint32_t*)(acc_empty + 2);

  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = d.K / 64;
  constexpr int kEpiThreads = C::EPI_WARPS * 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
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
  grid_dep_wait();
  grid_dep_launch();

  // tile -> (first output column, first row, fixed coordinate), n fastest
  auto coords = [&](int tile, int& n0, int& mt0, int& g) {
    const int rest = tile / tiles_n;
    n0 = (tile - rest * tiles_n) * C::BN;
    const int gi = rest / tiles_m;
    mt0 = d.m_lo + (rest - gi * tiles_m) * C::BM;
    g = d.g_lo + gi;
  };

  if (warp == C::EPI_WARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t keep = l2_evict_last();
      bool ok = true;
      int q = 0;  // ring position, continuous across tiles
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        int n0, mt0, g;
        coords(tile, n0, mt0, g);
        const int grp = d.mode == TILE_SAMPLES ? g - d.grp_base : 0;
        for (int kb = 0; kb < KB; ++kb, ++q) {
          const int s = q % C::STAGES;
          if (q >= C::STAGES && !mbar_wait(&empty[s], ((q / C::STAGES) - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = ring + s * C::STAGE_BYTES;
          mbar_expect_tx(&full[s], C::STAGE_BYTES);
          if (a_swap) tma_load_3d(&tmA, &full[s], sa, kb * 64, g, mt0);
          else tma_load_3d(&tmA, &full[s], sa, kb * 64, mt0, g);
          tma_load_3d_hint(&tmB, &full[s], sa + C::A_BYTES, kb * 64, d.n_lo + n0, grp, keep);
        }
      }
    }
  } else if (warp == C::EPI_WARPS + 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, C::BN);
      const uint64_t d0 = sdesc_k128(smem_u32(ring));
      bool ok = true;
      int q = 0, j = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++j) {
        const int acc = j & 1;
        if (j >= 2) {
          // the epilogue must have read this accumulator's previous tile
          ok = mbar_wait(&acc_empty[acc], ((j >> 1) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t tacc = tmem + (uint32_t)(acc * C::BN);
        for (int kb = 0; kb < KB; ++kb, ++q) {
          const int s = q % C::STAGES;
          ok = mbar_wait(&full[s], (q / C::STAGES) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint64_t da = desc_add(d0, s * C::STAGE_BYTES);
          const uint32_t acc0 = kb ? 1u : 0u;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tacc, desc_add(da, k * 32), desc_add(da, C::A_BYTES + k * 32), idesc, k ? 1u : acc0);
          umma_commit(&empty[s]);
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
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
      int n0, mt0, g;
      coords(tile, n0, mt0, g);
      const int grp = d.mode == TILE_SAMPLES ? g - d.grp_base : 0;
      const int acc = j & 1;
      ok = ok && mbar_wait(&acc_full[acc], (j >> 1) & 1);
      tc_fence_after();
      // the previous tile's TMA stores must have finished reading the staging tile
      if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const uint32_t tacc = tmem + (uint32_t)(acc * C::BN + half * (C::BN / 2)) + lb;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int col = half * (C::BN / 2) + c * 32;  // column within the tile
        const int n = n0 + col;
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
        }
        if (n < d.scale_cols) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= d.col_scale;
        }
        st_sw128_32(stage_out, 16384, r, col, v);
      }
      // the accumulator is read: the MMA may start the tile after next in it
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (threadIdx.x == 0 && ok) {
#pragma unroll
        for (int i = 0; i < C::BN / 64; ++i) {
          if (out_swap) tma_store_3d(&tmOut, stage_out + i * 16384, n0 + i * 64, g, mt0);
          else tma_store_3d(&tmOut, stage_out + i * 16384, n0 + i * 64, mt0, g);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
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
inline bool tc_persist_supported(const GemmDesc& d) {
  return d.out_kind == OUT_ROWS && !d.res.base && !d.rms.base && !d.out.f32 && !d.w_mn && d.N % PersistCfg::BN == 0 &&
         tc_gemm_supported(d);
}

inline int device_sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || n <= 0)
      n = 1;
  }
  return n;
}

// ONETRANS_ERR_UNSUPPORTED when the output rows are not one TMA-addressable
// set (the caller then takes the one-tile-per-CTA kernel).
inline onetrans_status tc_persist_launch(const GemmDesc& d, cudaStream_t st) {
  using C = PersistCfg;
  CUtensorMap ta, tb, tout;
  int out_swap = 0;
  if (!make_gemm_out_tmap(&tout, d, C::BN, C::OUT_BYTES, out_swap)) return ONETRANS_ERR_UNSUPPORTED;
  const uint64_t mext = (uint64_t)d.a_mext, gext = (uint64_t)d.a_gext;
  const uint64_t s_m = (uint64_t)d.a_sm, s_g = gext > 1 ? (uint64_t)d.a_sg : mext * (uint64_t)d.a_sm;
  const int a_swap = (gext > 1 && d.a_sg < d.a_sm) ? 1 : 0;
  bool ok = a_swap ? make_tmap_3d(&ta, d.A, d.K, gext, mext, s_g, s_m, 64, 1, 128)
                   : make_tmap_3d(&ta, d.A, d.K, mext, gext, s_m, s_g, 64, 128, 1);
  const uint64_t wg = (uint64_t)d.w_groups;
  const uint64_t w_sg = wg > 1 ? (uint64_t)d.w_sg : (uint64_t)d.w_rows * d.K;
  ok = ok && make_tmap_3d(&tb, d.W, d.K, d.w_rows, wg, d.K, w_sg, 64, C::BN, 1);
  if (!ok) return ONETRANS_ERR_CUDA;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gemm_persist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return ONETRANS_ERR_CUDA;
    attr_set = true;
  }
  const int tiles_n = d.N / C::BN, tiles_m = (d.M + C::BM - 1) / C::BM;
  const long long n_tiles = (long long)tiles_n * tiles_m * d.G;
  if (n_tiles <= 0) return ONETRANS_OK;
  if (n_tiles > 0x7fffffff) return ONETRANS_ERR_SHAPE;
  const int grid = (int)std::min<long long>(n_tiles, device_sm_count());
  launch_dependent(gemm_persist_kernel, dim3(grid), dim3(C::THREADS), C::SMEM, st, ta, tb, tout, d, a_swap,
                   out_swap, tiles_n, tiles_m, (int)n_tiles);
  return cudaGetLastError() == cudaSuccess ? ONETRANS_OK : ONETRANS_ERR_CUDA;
}

}  // namespace ot
