// Tensor-core GEMM with fused epilogues for the bf16 path (sm_100a).
//
//   C[(b,t), n] = epi( sum_k A[(m,g), k] * W[grp][n_lo + n][k] )
//
// One CTA computes a 128 x BN output tile.  A and W tiles (64 bf16 of K per
// row, 128-byte swizzle) are streamed by TMA through a STAGES-deep ring of
// shared-memory buffers guarded by mbarriers; one thread issues tcgen05.mma
// (M = 128, N = BN or BN/2, K = 16) into an fp32 accumulator in TMEM; four
// epilogue warps read the accumulator back with tcgen05.ld (one output row
// per thread) and apply bias, GELU, residual, the paged K/V store and the
// RMSNorm of the finished row (when the CTA owns the whole row, BN == N).
//
// Plain row outputs whose rows TMA can address leave through shared memory
// (the stage buffers are idle once the accumulator is complete) and TMA
// stores.  Float32 row outputs with a float32 residual and / or the
// in-epilogue RMSNorm take the staged path end to end (`rows_tma`): the
// residual comes in by TMA into the stage buffers, 16 KB boxes of 32 columns
// at a time, each thread adds its row's values and writes the sum back in
// place, the boxes leave by TMA; the RMSNorm pass then brings the stored row
// block back by TMA (from L2) and sends the normalised bf16 rows out the same
// way.  K/V pages and the remaining cases are stored per thread.
//
// Warp roles (192 threads): warps 0-3 epilogue, warp 4 TMA producer,
// warp 5 TMEM allocator and MMA issuer.
#pragma once
#include <cudaTypedefs.h>
#include "tc_ptx.cuh"

namespace ot {

template <int BN>
struct TcGemmCfg {
  static constexpr int UN = BN <= 256 ? BN : BN / 2;  // N of one tcgen05.mma
  static constexpr int NSUB = BN / UN;
  static constexpr int BOX_N = BN <= 256 ? BN : BN / 2;  // TMA box rows of W (<= 256)
  // two CTAs per SM for BN = 256 (one's epilogue overlaps the other's loads
  // and MMAs); BN = 128 takes the small grids (a handful of tiles with a long
  // K), where a deeper ring hides the load latency of the serial k-loop
  static constexpr int STAGES = BN == 128 ? 4 : BN <= 256 ? 2 : 3;
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = BN <= 128 ? 128 : (BN <= 256 ? 256 : 512);
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

// Epilogue of rows_tma: `slots` 16 KB boxes of the stage area; pass 1 adds
// the residual and stores the float32 rows, pass 2 (RMSNorm) normalises them.
template <int BN>
__device__ inline void rows_tma_epilogue(uint8_t* smem, int slots, uint64_t* ebar, const CUtensorMap* tmOut,
                                         const CUtensorMap* tmRes, const CUtensorMap* tmRms, const GemmDesc& d,
                                         uint32_t trow, int r, bool done, int n0, int mt0, int g, int grp,
                                         int out_swap) {
  const __nv_bfloat16* bias = (const __nv_bfloat16*)d.bias;
  const bool lead = threadIdx.x == 0;
  uint32_t ph = 0;   // parity of ebar's next completion
  float ss = 0.f;
  const int c1 = out_swap ? g : mt0, c2 = out_swap ? mt0 : g;   // the tile's row coordinates
  bool ok = done;
  constexpr int NBOX = BN / 32;
  // a bf16 residual arrives as boxes of 64 columns in the slots after the
  // group's output boxes (one per two of them)
  const bool res16 = d.res.base && !d.res.f32;
  const int gmax = res16 ? (2 * slots / 3) & ~1 : slots;
  for (int q0 = 0; q0 < NBOX; q0 += gmax) {
    const int nb = min(gmax, NBOX - q0);
    if (d.res.base) {
      if (lead) {
        if (res16) {
          mbar_expect_tx(ebar, (nb / 2) * 16384);
          for (int j = 0; j < nb / 2; ++j)
            tma_load_3d(tmRes, ebar, smem + (nb + j) * 16384, n0 + q0 * 32 + j * 64, c1, c2);
        } else {
          mbar_expect_tx(ebar, nb * 16384);
          for (int i = 0; i < nb; ++i) tma_load_3d(tmRes, ebar, smem + i * 16384, n0 + (q0 + i) * 32, c1, c2);
        }
      }
      ok = mbar_wait(ebar, ph) && ok;
      ph ^= 1;
    }
    for (int i = 0; i < nb; ++i) {
      const int c0 = (q0 + i) * 32, n = n0 + c0;
      float v[32];
      tmem_ld32(trow + c0, v);
      if (bias) {
        float bv[32];
        load_bf16x32(bias + (long long)grp * d.bias_sg + d.n_lo + n, bv);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] += bv[e];
      }
      if (d.act == ACT_GELU) {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = gelu_fast(v[e]);
      }
      if (d.res.base) {
        float rv[32];
        if (res16) ld_sw128_bf16_half(smem, nb + i / 2, r, i & 1, rv);
        else ld_sw128_f32(smem, i, r, rv);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] += rv[e];
      }
      if (n < d.scale_cols) {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= d.col_scale;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) ss = fmaf(v[e], v[e], ss);
      st_sw128_f32(smem, i, r, v);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (lead && ok) {
      for (int i = 0; i < nb; ++i) tma_store_3d(tmOut, smem + i * 16384, n0 + (q0 + i) * 32, c1, c2);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    // the stores have read the boxes before anyone writes them again (and,
    // for the RMSNorm pass, the rows are in global memory)
    if (lead) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  if (!d.rms.base) return;
  // pass 2: h = x r g, r = (mean(x^2) + eps)^(-1/2); per group of h boxes (64
  // bf16 columns) the two x boxes of each come back into slots 2j, 2j+1 and
  // h goes out of slots from 2 * per on
  const float rr = rsqrtf(ss / d.N + d.eps);
  const __nv_bfloat16* gm = (const __nv_bfloat16*)d.gamma;
  constexpr int NH = BN / 64;
  const int per = max(1, slots / 3);
  for (int j0 = 0; j0 < NH; j0 += per) {
    const int nj = min(per, NH - j0);
    if (lead) {
      // the rows were stored by this CTA's own TMA stores (complete above)
      asm volatile("fence.proxy.async.global;" ::: "memory");
      mbar_expect_tx(ebar, nj * 2 * 16384);
      for (int i = 0; i < 2 * nj; ++i) tma_load_3d(tmOut, ebar, smem + i * 16384, n0 + (2 * j0 + i) * 32, c1, c2);
    }
    ok = mbar_wait(ebar, ph) && ok;
    ph ^= 1;
    for (int j = 0; j < nj; ++j) {
      float xv[64], gv[64];
      ld_sw128_f32(smem, 2 * j, r, xv);
      ld_sw128_f32(smem, 2 * j + 1, r, xv + 32);
      load_bf16x32(gm + (j0 + j) * 64, gv);
      load_bf16x32(gm + (j0 + j) * 64 + 32, gv + 32);
#pragma unroll
      for (int e = 0; e < 64; ++e) xv[e] = xv[e] * rr * gv[e];
      st_sw128_32(smem + 2 * per * 16384 + j * 16384, 16384, r, 0, xv);
      st_sw128_32(smem + 2 * per * 16384 + j * 16384, 16384, r, 32, xv + 32);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (lead && ok) {
      for (int j = 0; j < nj; ++j) tma_store_3d(tmRms, smem + 2 * per * 16384 + j * 16384, n0 + (j0 + j) * 64, c1, c2);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    if (lead) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
}

template <int BN>
__global__ void __launch_bounds__(192, BN <= 256 ? 2 : 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmRes,
                   const __grid_constant__ CUtensorMap tmRms, const GemmDesc d, const int a_swap,
                   const int out_tma, const int out_swap) {
  using C = TcGemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* ebar = accf + 1;   // rows_tma epilogue: residual / row-block loads
  uint32_t* tmem_slot = (uint32_t*)(ebar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int mt0 = d.m_lo + blockIdx.y * 128;
  const int g = d.g_lo + blockIdx.z;
  const int grp = d.mode == TILE_SAMPLES ? g - d.grp_base : 0;
  const int KB = d.K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(ebar, 1);
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
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
      const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (kb / C::STAGES) & 1;
        if (kb >= C::STAGES && !mbar_wait(&empty[s], ph ^ 1)) break;
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        mbar_expect_tx(&full[s], C::STAGE_BYTES);
        if (a_swap) tma_load_3d_hint(&tmA, &full[s], sa, kb * 64, g, mt0, stream);
        else tma_load_3d_hint(&tmA, &full[s], sa, kb * 64, mt0, g, stream);
        if (d.w_mn) {
          // 64 columns of N x the k-block's 64 rows per box (MN-major)
#pragma unroll
          for (int c = 0; c < BN / 64; ++c)
            tma_load_3d_hint(&tmB, &full[s], sb + c * 8192, d.n_lo + n0 + c * 64, kb * 64, grp, keep);
        } else {
#pragma unroll
          for (int c = 0; c < BN / C::BOX_N; ++c)
            tma_load_3d_hint(&tmB, &full[s], sb + c * C::BOX_N * 128, kb * 64, d.n_lo + n0 + c * C::BOX_N, grp, keep);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc = d.w_mn ? idesc_bf16(128, C::UN, false, true) : idesc_bf16(128, C::UN);
      const uint64_t d0 = sdesc_k128(smem_u32(smem));  // stage 0's A tile
      // stage 0's B tile: K-major (16 k per 32 bytes), or MN-major (64-column
      // boxes 8 KB apart, 16 k per 2 KB)
      const uint64_t b0 = d.w_mn ? sdesc_mn128(smem_u32(smem + C::A_BYTES), 8192) : desc_add(d0, C::A_BYTES);
      const uint32_t kstep = d.w_mn ? 2048 : 32;
      bool ok = true;
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (kb / C::STAGES) & 1;
        ok = mbar_wait(&full[s], ph);
        if (!ok) break;
        tc_fence_after();
        const uint64_t da = desc_add(d0, s * C::STAGE_BYTES), db = desc_add(b0, s * C::STAGE_BYTES);
        const uint32_t acc0 = kb ? 1u : 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int j = 0; j < C::NSUB; ++j)
            umma_bf16(tmem + j * C::UN, desc_add(da, k * 32), desc_add(db, j * C::UN * 128 + k * kstep), idesc,
                      k ? 1u : acc0);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accf);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const bool done = mbar_wait(accf, 0);
    tc_fence_after();
    const int r = warp * 32 + lane;
    if (out_tma == 2) {
      rows_tma_epilogue<BN>(smem, C::STAGES * C::STAGE_BYTES / 16384, ebar, &tmOut, &tmRes, &tmRms, d,
                            tmem + ((uint32_t)(warp * 32) << 16), r, done, n0, mt0, g, grp, out_swap);
    } else {
    const int m = mt0 + r;
    const bool valid = done && m < d.m_lo + d.M;
    int b = 0, t = 0;
    if (valid) row_of(d, m, g, b, t);
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const __nv_bfloat16* bias = (const __nv_bfloat16*)d.bias;
    float ss = 0.f;
    for (int c0 = 0; c0 < BN; c0 += 32) {
      float v[32];
      tmem_ld32(trow + c0, v);
      if (!valid) continue;
      const int n = n0 + c0;
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
      if (d.res.base) {
        float rv[32];
        load_row32(d.res, rm_off(d.res, b, t, n), rv);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += rv[i];
      }
      if (n < d.scale_cols) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= d.col_scale;
      }
      if (d.out_kind == OUT_KV) {
        const int dm = d.kv.H * d.kv.dh;
        const int kind = n / dm, cc = n - kind * dm, head = cc / d.kv.dh, e = cc - head * d.kv.dh;
        const int p0 = d.kv.pos_off_u ? d.kv.pos_off_u[b] : d.kv.pos_off;
        store_bf16x32((__nv_bfloat16*)d.kv.pool + kv_off(d.kv, b, t + p0, kind, head, e), v);
      } else if (out_tma) {
        // every MMA is done: the stage buffers stage the tile for TMA stores
        if (d.out.f32) st_sw128_f32(smem, c0 >> 5, r, v);
        else st_sw128_32(smem, 16384, r, c0, v);
      } else {
        store_row32(d.out, rm_off(d.out, b, t, n), v);
      }
      if (d.rms.base) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float q = d.out.f32 ? v[i] : __bfloat162float(__float2bfloat16_rn(v[i]));
          ss += q * q;
        }
      }
    }
    if (out_tma) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (threadIdx.x == 0 && done) {
        const int bc = d.out.f32 ? 32 : 64;
        for (int i = 0; i < BN / bc; ++i) {
          if (out_swap) tma_store_3d(&tmOut, smem + i * 16384, n0 + i * bc, g, mt0);
          else tma_store_3d(&tmOut, smem + i * 16384, n0 + i * bc, mt0, g);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      }
    }
    if (valid && d.rms.base) {
      // the CTA owns the whole row (BN == N): normalise the stored row
      const float rr = rsqrtf(ss / d.N + d.eps);
      const __nv_bfloat16* gm = (const __nv_bfloat16*)d.gamma;
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32], gv[32];
        load_row32(d.out, rm_off(d.out, b, t, c0), v);
        load_bf16x32(gm + c0, gv);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = v[i] * rr * gv[i];
        store_row32(d.rms, rm_off(d.rms, b, t, c0), v);
      }
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
inline int tc_pick_bn(const GemmDesc& d) {
  if (d.rms.base) return (d.N == 128 || d.N == 256 || d.N == 384) ? d.N : 0;
  // a grid far below one wave with a long reduction: narrower tiles, more CTAs
  const long long tiles256 = (long long)((d.N + 255) / 256) * ((d.M + 127) / 128) * d.G;
  if (d.N % 128 == 0 && d.K >= 512 && 2 * tiles256 <= 148) return 128;
  if (d.N % 256 == 0) return 256;
  if (d.N % 384 == 0) return 384;
  if (d.N % 128 == 0) return 128;
  return 0;
}


inline bool tc_gemm_supported(const GemmDesc& d) {
  if (d.K <= 0 || d.K % 64 || !tc_pick_bn(d)) return false;
  if ((uintptr_t)d.A % 16 || (uintptr_t)d.W % 16) return false;
  if (d.a_sm % 8 || d.a_sg % 8 || d.w_sg % 8) return false;
  if (d.w_mn && (d.w_rows % 64 || d.n_lo % 64)) return false;
  if (d.bias && ((d.bias_sg % 8) || (d.n_lo % 8) || ((uintptr_t)d.bias % 16))) return false;
  if (d.res.base && !rowmap_vec_ok(d.res)) return false;
  if (d.rms.base && (!rowmap_vec_ok(d.rms) || (uintptr_t)d.gamma % 16)) return false;
  if (d.out_kind == OUT_KV) {
    if (d.kv.dh % 32 || (uintptr_t)d.kv.pool % 16) return false;
  } else if (!rowmap_vec_ok(d.out)) {
    return false;
  }
  return encode_fn() != nullptr;
}

// TMA map over the plain output rows of a GEMM (columns [0, N)), when the
// rows form a strided 2-D set and the whole tile fits in the stage buffers.
// TMA map over the rows of a GEMM (columns [0, N)) held by RowMap r, boxes
// of 128 rows x `bc` columns, when the rows form a strided 2-D set.
inline bool make_rows_tmap(CUtensorMap* map, const GemmDesc& d, const RowMap& r, uint32_t bc, int& swap) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !r.base || r.split < d.N || ((uintptr_t)r.base % 16)) return false;
  const uint64_t es = r.f32 ? 4 : 2;
  const uint64_t m_ext = (uint64_t)(d.m_lo + d.M), g_ext = (uint64_t)(d.g_lo + d.G);
  uint64_t s_m, s_g;
  if (d.mode == TILE_ROWS) { s_m = r.st; s_g = r.sb; }
  else if (d.mode == TILE_SAMPLES) { s_m = r.sb; s_g = r.st; }
  else {
    if (d.fold < d.m_lo + d.M && (long long)r.sb != (long long)d.fold * r.st) return false;
    s_m = r.st; s_g = m_ext * r.st;
  }
  if (g_ext == 1) s_g = m_ext * s_m;
  swap = (g_ext > 1 && s_g < s_m) ? 1 : 0;
  const cuuint64_t dims[3] = {(cuuint64_t)d.N, swap ? g_ext : m_ext, swap ? m_ext : g_ext};
  const cuuint64_t strides[2] = {(swap ? s_g : s_m) * es, (swap ? s_m : s_g) * es};
  const cuuint32_t box[3] = {bc, swap ? 1u : 128u, swap ? 128u : 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (strides[0] % 16 || strides[1] % 16) return false;
  return fn(map, r.f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, r.base, dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// TMA map over the plain output rows of a GEMM, when the whole tile fits in
// the stage buffers.
inline bool make_gemm_out_tmap(CUtensorMap* map, const GemmDesc& d, int bn, int stage_bytes, int& swap) {
  if (d.out_kind != OUT_ROWS || d.rms.base) return false;
  const uint64_t es = d.out.f32 ? 4 : 2;
  if ((uint64_t)128 * bn * es > (uint64_t)stage_bytes) return false;
  return make_rows_tmap(map, d, d.out, d.out.f32 ? 32 : 64, swap);
}

// The staged float32-rows epilogue (rows_tma): float32 output rows, an
// optional float32 residual, an optional RMSNorm of the whole row (bf16),
// all three TMA-addressable with the same row geometry.
inline bool make_rows_tma_maps(CUtensorMap* tout, CUtensorMap* tres, CUtensorMap* trms, const GemmDesc& d, int bn,
                               int& swap) {
  if (d.out_kind != OUT_ROWS || !d.out.f32 || d.act == ACT_GELU_BWD) return false;
  if (d.rms.base && (bn != d.N || d.rms.f32 || (uintptr_t)d.gamma % 16)) return false;
  int s_out = 0, s_res = 0, s_rms = 0;
  if (!make_rows_tmap(tout, d, d.out, 32, s_out)) return false;
  if (d.res.base && !make_rows_tmap(tres, d, d.res, d.res.f32 ? 32 : 64, s_res)) return false;
  if (d.rms.base && !make_rows_tmap(trms, d, d.rms, 64, s_rms)) return false;
  if ((d.res.base && s_res != s_out) || (d.rms.base && s_rms != s_out)) return false;
  swap = s_out;
  return true;
}

// A flat row set (rows of B samples back to back, `fold` per sample) as
// per-sample tiles, for an epilogue whose residual rows do not fold the same
// way (the pyramid's tail rows of a longer input).  Taken when the last tile
// of a sample wastes at most an eighth of the sample's rows.
inline bool flat_to_rows(GemmDesc& g) {
  if (g.mode != TILE_FLAT || g.G != 1 || g.m_lo != 0 || g.a_gext != 1 || g.fold < 128 || g.M % g.fold) return false;
  const int waste = (g.fold + 127) / 128 * 128 - g.fold;
  if (8 * waste > g.fold) return false;
  const int B = g.M / g.fold;
  g.mode = TILE_ROWS;
  g.a_sg = (long long)g.fold * g.a_sm;
  g.a_mext = g.fold;
  g.a_gext = B;
  g.M = g.fold;
  g.G = B;
  g.g_lo = 0;
  return true;
}

template <int BN>
inline onetrans_status tc_gemm_launch_bn(const GemmDesc& d_in, cudaStream_t st) {
  using C = TcGemmCfg<BN>;
  CUtensorMap ta, tb, tout, tres, trms;
  // the epilogue decides the row tiling: the staged float32 rows path where
  // the output (and residual / RMSNorm rows) allow it, else the plain staged
  // output, else per-thread stores
  GemmDesc d = d_in;
  int out_swap = 0, out_tma = 0;
  if (make_rows_tma_maps(&tout, &tres, &trms, d, BN, out_swap)) {
    out_tma = 2;
  } else {
    GemmDesc dr = d_in;
    if (dr.res.base && flat_to_rows(dr) && make_rows_tma_maps(&tout, &tres, &trms, dr, BN, out_swap)) {
      d = dr;
      out_tma = 2;
    } else if (make_gemm_out_tmap(&tout, d, BN, C::STAGES * C::STAGE_BYTES, out_swap)) {
      out_tma = 1;
    }
  }
  const uint64_t mext = (uint64_t)d.a_mext, gext = (uint64_t)d.a_gext;
  const uint64_t s_m = (uint64_t)d.a_sm, s_g = gext > 1 ? (uint64_t)d.a_sg : mext * (uint64_t)d.a_sm;
  const int a_swap = (gext > 1 && d.a_sg < d.a_sm) ? 1 : 0;
  bool ok = a_swap ? make_tmap_3d(&ta, d.A, d.K, gext, mext, s_g, s_m, 64, 1, 128)
                   : make_tmap_3d(&ta, d.A, d.K, mext, gext, s_m, s_g, 64, 128, 1);
  const uint64_t wg = (uint64_t)d.w_groups;
  const uint64_t w_sg = wg > 1 ? (uint64_t)d.w_sg : (uint64_t)d.w_rows * d.K;
  if (d.w_mn) ok = ok && make_tmap_3d(&tb, d.W, d.w_rows, d.K, wg, d.w_rows, w_sg, 64, 64, 1);
  else ok = ok && make_tmap_3d(&tb, d.W, d.K, d.w_rows, wg, d.K, w_sg, 64, C::BOX_N, 1);
  if (!ok) return ONETRANS_ERR_CUDA;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return ONETRANS_ERR_CUDA;
    attr_set = true;
  }
  if (!out_tma) tout = ta;
  if (!d.res.base || out_tma != 2) tres = ta;
  if (!d.rms.base || out_tma != 2) trms = ta;
  dim3 grid((unsigned)(d.N / BN), (unsigned)((d.M + 127) / 128), (unsigned)d.G);
  launch_dependent(gemm_tc_kernel<BN>, grid, dim3(192), C::SMEM, st, ta, tb, tout, tres, trms, d, a_swap, out_tma,
                   out_swap);
  return cudaGetLastError() == cudaSuccess ? ONETRANS_OK : ONETRANS_ERR_CUDA;
}

inline onetrans_status tc_gemm_launch(const GemmDesc& d, cudaStream_t st) {
  switch (tc_pick_bn(d)) {
    case 128: return tc_gemm_launch_bn<128>(d, st);
    case 256: return tc_gemm_launch_bn<256>(d, st);
    case 384: return tc_gemm_launch_bn<384>(d, st);
    default: return ONETRANS_ERR_UNSUPPORTED;
  }
}

}  // namespace ot
