// Weight-gradient GEMM on row-major operands (sm_100a).
//
//   dW[z][n][k] = sum over the row tiles i of slice z of
//                 sum over the 64 rows r of tile i of  Y[r][n] * X[r][k]
//
// Y (the output gradient rows, N_out columns) and X (the layer input rows,
// K_in columns) are read straight from their row-major buffers.  A TMA box of
// 64 rows x 64 columns with the 128-byte swizzle is, for tcgen05.mma, an
// MN-major operand tile: the rows are the reduction dimension, the columns
// the M (of Y) or N (of X) extent; 64-column boxes sit 8 KB apart (the
// descriptor's leading byte offset), 8-row groups 1 KB apart (its stride
// byte offset).  So no transposed copy of either operand is made.
//
// Row tiles come from a 3-D view (columns, r1, r2) of each operand: tile i is
// rows r1 = 64 (i mod TC) .. +63 at r2 = i / TC, TC = ceil(r1 extent / 64);
// rows past the r1 extent read as zero and add nothing.  The S weight set
// views its rows as (t, sample) and splits the tiles into slices, one partial
// gradient each (summed afterwards in slice order); each NS weight set views
// its rows as (sample, NS token) with one slice per token.
//
// One CTA computes a 128 (n) x BN (k) float32 tile of one slice and stores it
// with TMA through the idle stage buffers.  Warp roles (192 threads): warps
// 0-3 epilogue, warp 4 TMA producer, warp 5 TMEM allocator and MMA issuer.
#pragma once
#include <cudaTypedefs.h>
#include "tc_ptx.cuh"

namespace ot {

struct WgradArgs {
  int TC;      // row tiles per r2 value
  int per;     // row tiles per slice
  int total;   // row tiles of all slices
  int swap;    // the tensor maps list r2 before r1 (strides kept increasing)
};

template <int BN>
struct WgradCfg {
  static constexpr int A_BYTES = 2 * 8192;           // 128 columns of Y: two 64-column boxes
  static constexpr int B_BYTES = (BN / 64) * 8192;   // BN columns of X
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int TMEM_COLS = BN;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(128 * BN * 4 <= STAGES * STAGE_BYTES, "the output tile is staged in the stage buffers");
};

template <int BN>
__global__ void __launch_bounds__(192, 1)
    gemm_wgrad_kernel(const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmOut, const WgradArgs a) {
  using C = WgradCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint32_t* tmem_slot = (uint32_t*)(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = blockIdx.x * BN, n0 = blockIdx.y * 128, z = blockIdx.z;
  const int i0 = z * a.per;
  const int nT = max(0, min(a.per, a.total - i0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmY);
    prefetch_tmap(&tmX);
  }
  if (warp == 5) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 4) {
    if (lane == 0) {
      for (int j = 0; j < nT; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (j >= C::STAGES && !mbar_wait(&empty[s], ph ^ 1)) break;
        const int i = i0 + j, r2 = i / a.TC, r1 = (i - r2 * a.TC) * 64;
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        mbar_expect_tx(&full[s], C::STAGE_BYTES);
        const int c1 = a.swap ? r2 : r1, c2 = a.swap ? r1 : r2;
        tma_load_3d(&tmY, &full[s], sa, n0, c1, c2);
        tma_load_3d(&tmY, &full[s], sa + 8192, n0 + 64, c1, c2);
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tma_load_3d(&tmX, &full[s], sb + c * 8192, k0 + c * 64, c1, c2);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, true, true);
      const uint64_t d0 = sdesc_mn128(smem_u32(smem), 8192);   // stage 0's Y tile
      bool ok = true;
      for (int j = 0; j < nT && ok; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        ok = mbar_wait(&full[s], ph);
        if (!ok) break;
        tc_fence_after();
        const uint64_t da = desc_add(d0, s * C::STAGE_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k)   // 16 rows per MMA: 16 x 128 B further into each box
          umma_bf16(tmem, desc_add(da, k * 2048), desc_add(da, C::A_BYTES + k * 2048), idesc, (j | k) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accf);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const bool done = mbar_wait(accf, 0);
    tc_fence_after();
    const int r = warp * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < BN; c0 += 32) {
      float v[32];
      tmem_ld32(trow + c0, v);
      if (nT == 0) {
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = 0.f;
      }
      st_sw128_f32(smem, c0 >> 5, r, v);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 0 && done) {
      for (int q = 0; q < BN / 32; ++q) tma_store_3d(&tmOut, smem + q * 16384, k0 + q * 32, n0, z);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
// A 3-D view (cols, r1, r2) of bf16 rows: element (c, r1, r2) at
// base + r1 * s1 + r2 * s2 + c (elements); boxes of 64 columns x 64 rows of
// r1.  With s2 < s1 the map lists r2 first (swap = 1), so that its strides
// increase, and a box is 64 columns x 1 x 64 (the same shared-memory tile).
inline bool wgrad_rows_tmap(CUtensorMap* map, const void* base, int cols, long long e1, long long e2, long long s1,
                            long long s2, int& swap) {
  if ((uintptr_t)base % 16 || s1 % 8 || s2 % 8 || cols % 64 || e1 <= 0 || e2 <= 0) return false;
  swap = (e2 > 1 && s2 < s1) ? 1 : 0;
  if (e2 == 1) s2 = e1 * s1;
  if (swap) return make_tmap_3d(map, base, (uint64_t)cols, (uint64_t)e2, (uint64_t)e1, (uint64_t)s2, (uint64_t)s1,
                                64, 1, 64);
  return make_tmap_3d(map, base, (uint64_t)cols, (uint64_t)e1, (uint64_t)e2, (uint64_t)s1, (uint64_t)s2, 64, 64, 1);
}

// dW [Z][N_out][K_in] float32, one 16-byte-aligned slice after another.
inline bool wgrad_out_tmap(CUtensorMap* map, float* out, int N_out, int K_in, int Z) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || (uintptr_t)out % 16) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)K_in, (cuuint64_t)N_out, (cuuint64_t)Z};
  const cuuint64_t strides[2] = {(cuuint64_t)K_in * 4, (cuuint64_t)N_out * K_in * 4};
  const cuuint32_t box[3] = {32, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int wgrad_pick_bn(int K_in) { return K_in % 256 == 0 ? 256 : K_in % 128 == 0 ? 128 : 0; }

// Shapes the kernel takes: N_out a multiple of 128, K_in of 128.
inline bool wgrad_supported(int N_out, int K_in) { return N_out > 0 && N_out % 128 == 0 && wgrad_pick_bn(K_in) > 0; }

template <int BN>
inline onetrans_status wgrad_launch_bn(const CUtensorMap& tY, const CUtensorMap& tX, const CUtensorMap& tOut,
                                       int N_out, int K_in, int Z, const WgradArgs& a, cudaStream_t st) {
  using C = WgradCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gemm_wgrad_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return ONETRANS_ERR_CUDA;
    attr_set = true;
  }
  const dim3 grid((unsigned)(K_in / BN), (unsigned)(N_out / 128), (unsigned)Z);
  launch_dependent(gemm_wgrad_kernel<BN>, grid, dim3(192), C::SMEM, st, tY, tX, tOut, a);
  return cudaGetLastError() == cudaSuccess ? ONETRANS_OK : ONETRANS_ERR_CUDA;
}

inline onetrans_status wgrad_launch(const CUtensorMap& tY, const CUtensorMap& tX, const CUtensorMap& tOut, int N_out,
                                    int K_in, int Z, const WgradArgs& a, cudaStream_t st) {
  switch (wgrad_pick_bn(K_in)) {
    case 256: return wgrad_launch_bn<256>(tY, tX, tOut, N_out, K_in, Z, a, st);
    case 128: return wgrad_launch_bn<128>(tY, tX, tOut, N_out, K_in, Z, a, st);
    default: return ONETRANS_ERR_UNSUPPORTED;
  }
}

}  // namespace ot
