// Fused tail of a OneTrans block for 128 rows (bf16 path, d = 256, sm_100a):
//
//   x_mid  = x + W^O a                      (a: attention output row)
//   h2     = RMSNorm(x_mid) * g_ffn
//   x_next = x_mid + W2 GELU(W1 h2 + b1) + b2       (mixed FFN: W1, W2 of the
//                                                     rows' weight group)
//   h_next = RMSNorm(x_next) * g_next               (next layer's pre-norm)
//
// Only a, x, x_next and h_next touch HBM; x_mid and the d_ff-wide hidden
// layer stay on chip.  TMEM (512 columns) holds D (256 fp32 columns: the
// residual rows, then + W^O a = x_mid, then + W2 hidden, since both products
// accumulate in place) and U (256 fp32 columns: the up-projection of one
// 256-unit hidden chunk).  Every product is a 128 x 256 tcgen05.mma, the
// shape that runs at the tensor pipe's full rate (narrower N issue at about
// the same cost per instruction).  Shared memory holds the attention tile
// (reused for h2 as the A operand of the up-projection) and a 5-stage ring of
// 32 KB tiles fed by TMA: first the residual rows, then W^O, then W1/W2
// chunk by chunk.  x_next and h_next leave by TMA stores staged through the
// then idle shared memory.  Row geometries TMA cannot express fall back to
// per-thread loads/stores.
//
// Per hidden chunk c: up(c) -> U; the compute warps apply b1 + GELU to U in
// four blocks of 64 units, packing each block's bf16 result over its own
// columns and signalling it at once, so down(c) (A = the packed hidden
// block, read from TMEM) runs block by block behind the GELU; up(c+1) follows
// once down(c) has read U.
//
// Warp roles (576 threads): warps 0-15 compute (four warps per row quarter:
// warps w, w+4, w+8, w+12 share TMEM lanes 32*(w%4).. and split each row's
// columns, exchanging row sums through shared memory), warp 16 TMA producer,
// warp 17 TMEM allocator and MMA issuer.
#pragma once
#include "tc_ptx.cuh"

namespace ot {

struct FfnDesc {
  int mode, M, m_lo, G, g_lo, fold, grp_base;  // row enumeration, as in GemmDesc
  const void* A;                                // attention rows, bf16 [.., 256]
  long long a_sm, a_sg, a_mext, a_gext;
  const void* Wo;                               // [256, 256]
  const void* W1; long long w1_sg;              // [G][dff, 256]
  const void* b1; long long b1_sg;              // [G][dff]
  const void* W2; long long w2_sg;              // [G][256, dff]
  const void* b2; long long b2_sg;              // [G][256]
  const void* g_ffn;                            // [256]
  const void* g_next;                           // [256] or null
  RowMap res, out, hout;                        // hout.base null = no next-layer norm
  int dff, w_groups;
  float eps;
};

// Which row tensors move by TMA (else per-thread accesses), and whether their
// maps list the fixed coordinate before the tiled one.
struct FfnIo {
  int res_tma, res_swap, res_f32;
  int out_tma, out_swap;
  int hout_tma, hout_swap;
};

struct FfnCfg {
  static constexpr int D = 256, BM = 128, HC = 256;  // hidden chunk width
  static constexpr int HB = 64;                      // GELU / down-projection block of a chunk
  static constexpr int A_BYTES = BM * D * 2;        // 64 KB: attention tile, then h2
  static constexpr int STAGE = 32768;               // one ring stage
  static constexpr int STAGES = 5;
  static constexpr int BAR_BYTES = 256 + 2048;       // barriers + per-row partial sums [4][128]
  static constexpr int SMEM = A_BYTES + STAGES * STAGE + BAR_BYTES;
  static constexpr int TMEM_COLS = 512;  // D 0..255, U 256..511 (GELU output packed over U, block by block)
};

constexpr int kFfnThreads = 576;

__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmWo,
                  const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                  const __grid_constant__ CUtensorMap tmRes, const __grid_constant__ CUtensorMap tmOut,
                  const __grid_constant__ CUtensorMap tmHout, const FfnDesc d, const int a_swap, const FfnIo io) {
  using C = FfnCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sA = smem;
  uint8_t* sW = sA + C::A_BYTES;  // [STAGES][32 KB]
  uint64_t* bars = (uint64_t*)(sW + C::STAGES * C::STAGE);
  uint64_t* a_full = bars;
  uint64_t* w_full = bars + 1;             // [STAGES]
  uint64_t* w_empty = w_full + C::STAGES;  // [STAGES]
  uint64_t* d_full = w_empty + C::STAGES;
  uint64_t* h2_ready = d_full + 1;
  uint64_t* u_full = h2_ready + 1;
  uint64_t* hid_full = u_full + 1;   // [HC / HB]: one per hidden block
  uint64_t* dn_done = hid_full + C::HC / C::HB;
  uint64_t* d_done = dn_done + 1;
  uint64_t* res_ready = d_done + 1;
  uint32_t* tmem_slot = (uint32_t*)(res_ready + 1);
  float* red = (float*)((uint8_t*)bars + 256);  // [4][128] partial row sums

  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt0 = d.m_lo + blockIdx.x * C::BM;
  const int g = d.g_lo + blockIdx.y;
  const int grp = d.mode == TILE_SAMPLES ? g - d.grp_base : 0;
  const int NC = d.dff / C::HC;
  // residual stages at the head of the ring: fp32 rows in 4 stages of 64
  // columns, bf16 rows in 2 stages of 128 columns (two 16 KB boxes each)
  const int RP = io.res_tma ? (io.res_f32 ? 4 : 2) : 0;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&w_full[s], 1); mbar_init(&w_empty[s], 1); }
    mbar_init(d_full, 1);
    mbar_init(h2_ready, 512);
    mbar_init(u_full, 1);
    mbar_init(dn_done, 1);
    for (int i = 0; i < C::HC / C::HB; ++i) mbar_init(&hid_full[i], 512);
    mbar_init(d_done, 1);
    mbar_init(res_ready, 512);
    fence_barrier_init();
  }
  if (warp == 16 && lane == 0) {
    prefetch_tmap(&tmA); prefetch_tmap(&tmWo); prefetch_tmap(&tmW1); prefetch_tmap(&tmW2);
    if (io.res_tma) prefetch_tmap(&tmRes);
  }
  if (warp == 17) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tD = tmem, tU = tmem + 256;
  // Ring stages in the order they are consumed: the residual rows (RP), W^O
  // (4 k-blocks), W1 of chunk 0 (4), then W2(c) (4) and W1(c+1) (4) chunk by
  // chunk.  Stage q goes to slot q % STAGES.
  const int n_stages = RP + 8 + NC * 4 + (NC - 1) * 4;
  auto issue_stage = [&](int q, uint64_t keep, uint64_t stream) {
    const int s = q % C::STAGES;
    uint8_t* dst = sW + s * C::STAGE;
    mbar_expect_tx(&w_full[s], C::STAGE);
    if (q < RP) {                    // residual rows, columns of part q
      const int bc = io.res_f32 ? 32 : 64;
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        const int col = (2 * q + bx) * bc;
        if (io.res_swap) tma_load_3d_hint(&tmRes, &w_full[s], dst + bx * 16384, col, g, mt0, stream);
        else tma_load_3d_hint(&tmRes, &w_full[s], dst + bx * 16384, col, mt0, g, stream);
      }
    } else if (q < RP + 4) {         // W^O k-block j: [256 out x 64]
      tma_load_3d_hint(&tmWo, &w_full[s], dst, (q - RP) * 64, 0, 0, keep);
    } else if (q < RP + 8) {         // W1 chunk 0, k-block j: [256 hidden x 64]
      tma_load_3d_hint(&tmW1, &w_full[s], dst, (q - RP - 4) * 64, 0, grp, keep);
    } else {
      const int t = q - RP - 8, c = t >> 3, j = t & 3;
      if ((t & 7) < 4)               // W2 chunk c, hidden block j: [256 out x 64 hidden]
        tma_load_3d_hint(&tmW2, &w_full[s], dst, c * C::HC + j * C::HB, 0, grp, keep);
      else                           // W1 chunk c + 1, k-block j
        tma_load_3d_hint(&tmW1, &w_full[s], dst, j * 64, (c + 1) * C::HC, grp, keep);
    }
  };
  // The weights, and the residual rows (written at least two launches back),
  // are final before the previous kernel ends; only the attention rows come
  // from it.  So the first ring stages load before the wait for that kernel.
  if (warp == 16 && lane == 0) {
    const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
    for (int q = 0; q < C::STAGES && q < n_stages; ++q) issue_stage(q, keep, stream);
  }
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
      mbar_expect_tx(a_full, C::A_BYTES);
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        if (a_swap) tma_load_3d_hint(&tmA, a_full, sA + kb * 16384, kb * 64, g, mt0, stream);
        else tma_load_3d_hint(&tmA, a_full, sA + kb * 16384, kb * 64, mt0, g, stream);
      }
      for (int q = C::STAGES; q < n_stages; ++q) {
        const int s = q % C::STAGES;
        if (!mbar_wait(&w_empty[s], ((q / C::STAGES) - 1) & 1)) break;
        issue_stage(q, keep, stream);
      }
    }
  } else if (warp == 17) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id256 = idesc_bf16(128, 256);
      const uint64_t dA = sdesc_k128(smem_u32(sA)), dW = sdesc_k128(smem_u32(sW));
      int q = RP;  // the residual stages are consumed by the compute warps
      auto wait_stage = [&](uint64_t& base) -> bool {
        const int s = q % C::STAGES;
        if (!mbar_wait(&w_full[s], (q / C::STAGES) & 1)) return false;
        tc_fence_after();
        base = desc_add(dW, s * C::STAGE);
        return true;
      };
      auto free_stage = [&]() { umma_commit(&w_empty[q % C::STAGES]); ++q; };
      // The weight stages of a chunk are waited for ahead of their use (each
      // barrier wait costs a few hundred cycles here): W2(c) right after
      // up(c) is issued, while GELU runs; W1(c+1) right after down(c) is
      // issued, while it runs.  Every awaited stage is freed by MMAs already
      // issued, so the ring keeps moving.
      auto wait_ahead = [&](uint64_t* base) -> bool {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int qq = q + j, s = qq % C::STAGES;
          if (!mbar_wait(&w_full[s], (qq / C::STAGES) & 1)) return false;
          base[j] = desc_add(dW, s * C::STAGE);
        }
        tc_fence_after();
        return true;
      };
      // U = h2 W1c^T, K = 256 in four staged k-blocks (stages waited by the caller)
      auto up = [&](const uint64_t* wb) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tU, desc_add(dA, j * 16384 + k * 32), desc_add(wb[j], k * 32), id256, (j | k) ? 1u : 0u);
          free_stage();
        }
        umma_commit(u_full);
      };
      bool ok = mbar_wait(a_full, 0) && mbar_wait(res_ready, 0);
      if (ok) tc_fence_after();
      // D holds the residual rows: x_mid = x + a W^O^T accumulates in place
      for (int j = 0; j < 4 && ok; ++j) {
        uint64_t wb;
        ok = wait_stage(wb);
        if (!ok) break;
        const uint64_t da = desc_add(dA, j * 16384);
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_bf16(tD, desc_add(da, k * 32), desc_add(wb, k * 32), id256, 1u);
        free_stage();
      }
      if (ok) umma_commit(d_full);
      uint64_t w1b[4], w2b[4];
      ok = ok && wait_ahead(w1b) && mbar_wait(h2_ready, 0);
      if (ok) {
        tc_fence_after();
        up(w1b);
      }
      for (int c = 0; c < NC && ok; ++c) {
        ok = wait_ahead(w2b);  // W2(c)
        // D += H W2c^T block by block as the GELU output appears: in block b
        // (units 64b..64b+63) units 64b+16k..+15 are packed over U columns
        // 64b+16k..+7, one k-step each
        for (int b = 0; b < C::HC / C::HB && ok; ++b) {
          ok = mbar_wait(&hid_full[b], c & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t tH = tU + b * C::HB;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(tD, tH + k * 16, desc_add(w2b[b], k * 32), id256, 1u);
          free_stage();
        }
        umma_commit(dn_done);
        // up(c+1) overwrites U: let down(c) finish reading it first, then
        // issue each k-block as soon as its W1 stage is in (the later stages
        // arrive while the first k-blocks run)
        if (ok && c + 1 < NC) {
          ok = mbar_wait(dn_done, c & 1);
          for (int j = 0; j < 4 && ok; ++j) {
            uint64_t wb;
            ok = wait_stage(wb);
            if (!ok) break;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(tU, desc_add(dA, j * 16384 + k * 32), desc_add(wb, k * 32), id256, (j | k) ? 1u : 0u);
            free_stage();
          }
          if (ok) umma_commit(u_full);
        }
      }
      umma_commit(d_done);
    }
  } else {
    // ------------------------------------------------------------- compute
    const int q4 = warp & 3, wq = warp >> 2;   // row quarter, column quarter
    const int r = q4 * 32 + lane;
    const int m = mt0 + r;
    const bool valid = m < d.m_lo + d.M;
    int b = 0, t = 0;
    if (valid) row_of_rows(d.mode, d.fold, m, g, b, t);
    const uint32_t lb = (uint32_t)(q4 * 32) << 16;
    const int cD = wq * (C::D / 4);            // this warp's 64 columns of a d-wide row
    const __nv_bfloat16* gffn = (const __nv_bfloat16*)d.g_ffn;
    // full-row sum from the four column quarters of row r
    auto row_sum = [&](float part) -> float {
      red[wq * 128 + r] = part;
      asm volatile("bar.sync 1, 512;" ::: "memory");
      const float s2 = (red[r] + red[128 + r]) + (red[256 + r] + red[384 + r]);
      asm volatile("bar.sync 1, 512;" ::: "memory");
      return s2;
    };
    bool ok = true;
    // residual rows into D (the W^O product accumulates on top)
    if (io.res_tma) {
      // every compute thread passes each named barrier, even after a failed wait
      for (int p = 0; p < RP; ++p) {
        const int s = p % C::STAGES;
        ok = ok && mbar_wait(&w_full[s], (p / C::STAGES) & 1);
        const uint8_t* st = sW + s * C::STAGE;
        const int bx = wq & 1;  // box of the stage this warp moves
        if (ok && io.res_f32 && (p & 1) == (wq >> 1)) {
          float v[32];
          ld_sw128_f32(st, bx, r, v);
          tmem_st32(tD + lb + (2 * p + bx) * 32, v);
        } else if (ok && !io.res_f32 && p == (wq >> 1)) {
          float v[64];
          ld_sw128_bf16(st, bx, r, v);
          tmem_st32(tD + lb + (2 * p + bx) * 64, v);
          tmem_st32(tD + lb + (2 * p + bx) * 64 + 32, v + 32);
        }
        // the stage may be refilled once every compute thread has read it
        asm volatile("bar.sync 1, 512;" ::: "memory");
        if (threadIdx.x == 0) mbar_arrive(&w_empty[s]);
      }
    } else {
      for (int c0 = cD; c0 < cD + C::D / 4; c0 += 32) {
        float v[32];
        if (valid) load_row32(d.res, rm_off(d.res, b, t, c0), v);
        else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        tmem_st32(tD + lb + c0, v);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(res_ready);
    ok = ok && mbar_wait(d_full, 0);
    tc_fence_after();
    // D = x_mid; its RMSNorm becomes h2 in sA
    float ss = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v[32];
      tmem_ld32(tD + lb + cD + h * 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
    }
    {
      const float rr = rsqrtf(row_sum(ss) / C::D + d.eps);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[32], gv[32];
        tmem_ld32(tD + lb + cD + h * 32, v);
        load_bf16x32(gffn + cD + h * 32, gv);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = v[i] * rr * gv[i];
        st_sw128_32(sA, 16384, r, cD + h * 32, v);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    mbar_arrive(h2_ready);
    // hidden chunks: b1 + GELU block by block; in each 64-unit block warp wq
    // takes units 16 wq .. 16 wq + 15 and packs them as bf16 pairs over the
    // first 8 of the columns it read, then signals the block
    const __nv_bfloat16* b1 = (const __nv_bfloat16*)d.b1 + (long long)grp * d.b1_sg;
    const int cH = wq * (C::HB / 4);
    for (int c = 0; c < NC; ++c) {
      // this chunk's b1 (bf16 pairs), fetched before the wait for up(c) so the
      // wait covers the load latency
      uint4 bq[C::HC / C::HB][2];
#pragma unroll
      for (int bb = 0; bb < C::HC / C::HB; ++bb)
#pragma unroll
        for (int i = 0; i < 2; ++i) bq[bb][i] = ((const uint4*)(b1 + c * C::HC + bb * C::HB + cH))[i];
      ok = ok && mbar_wait(u_full, c & 1);
      tc_fence_after();
#pragma unroll
      for (int bb = 0; bb < C::HC / C::HB; ++bb) {
        const uint32_t col = tU + lb + bb * C::HB + cH;
        float v[16];
        tmem_ld16(col, v);
        const uint32_t* bu = (const uint32_t*)bq[bb];
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 bf = __bfloat1622float2(*(const __nv_bfloat162*)&bu[i]);
          pk[i] = gelu_bias_bf16x2(v[2 * i], v[2 * i + 1], bf.x, bf.y);
        }
        tmem_st8(col, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&hid_full[bb]);
      }
    }
    // x_next = D + b2, and the next layer's RMSNorm; every MMA is done, so
    // the whole of shared memory can stage the outputs for TMA stores:
    // x_next in 8 boxes of 32 fp32 columns from offset 0, h_next in 4 boxes
    // of 64 bf16 columns from offset 128 KB
    const __nv_bfloat16* b2 = (const __nv_bfloat16*)d.b2 + (long long)grp * d.b2_sg;
    const __nv_bfloat16* gn = (const __nv_bfloat16*)d.g_next;
    // this warp's 64 columns of b2 and g_next into L1 before the wait
    if (lane < 2) asm volatile("prefetch.global.L1 [%0];" ::"l"(b2 + cD + lane * 32));
    if (d.hout.base && lane >= 2 && lane < 4) asm volatile("prefetch.global.L1 [%0];" ::"l"(gn + cD + (lane - 2) * 32));
    ok = ok && mbar_wait(d_done, 0);
    tc_fence_after();
    uint8_t* stage_x = smem;
    uint8_t* stage_h = smem + 8 * 16384;
    ss = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c0 = cD + h * 32;
      float v[32], bv[32];
      tmem_ld32(tD + lb + c0, v);
      load_bf16x32(b2 + c0, bv);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        v[i] += bv[i];
        ss = fmaf(v[i], v[i], ss);
      }
      if (io.out_tma) st_sw128_f32(stage_x, c0 >> 5, r, v);
      else if (valid && ok) store_row32(d.out, rm_off(d.out, b, t, c0), v);
    }
    // x_next leaves first, so its stores drain while the next layer's
    // RMSNorm is computed from the staged copy (reads only) into stage_h
    if (io.out_tma) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.sync 1, 512;" ::: "memory");
      if (threadIdx.x == 0 && ok) {
        for (int i = 0; i < 8; ++i) {
          if (io.out_swap) tma_store_3d(&tmOut, stage_x + i * 16384, i * 32, g, mt0);
          else tma_store_3d(&tmOut, stage_x + i * 16384, i * 32, mt0, g);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (d.hout.base) {
      const float r2 = rsqrtf(row_sum(ss) / C::D + d.eps);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c0 = cD + h * 32;
        float v[32], gv[32];
        if (io.out_tma) {
          ld_sw128_f32(stage_x, c0 >> 5, r, v);  // x_next as staged above (this thread's own row)
        } else {
          float bv[32];
          tmem_ld32(tD + lb + c0, v);
          load_bf16x32(b2 + c0, bv);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += bv[i];
        }
        load_bf16x32(gn + c0, gv);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= r2 * gv[i];
        if (io.hout_tma) st_sw128_32(stage_h, 16384, r, c0, v);
        else if (valid && ok) store_row32(d.hout, rm_off(d.hout, b, t, c0), v);
      }
      if (io.hout_tma) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("bar.sync 1, 512;" ::: "memory");
        if (threadIdx.x == 0 && ok) {
          for (int i = 0; i < 4; ++i) {
            if (io.hout_swap) tma_store_3d(&tmHout, stage_h + i * 16384, i * 64, g, mt0);
            else tma_store_3d(&tmHout, stage_h + i * 16384, i * 64, mt0, g);
          }
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
      }
    }
    // shared memory must stay valid until the stores have read it
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 17) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
inline bool tc_ffn_supported(const FfnDesc& d) {
  if (d.dff <= 0 || d.dff % FfnCfg::HC) return false;
  if ((uintptr_t)d.A % 16 || (uintptr_t)d.Wo % 16 || (uintptr_t)d.W1 % 16 || (uintptr_t)d.W2 % 16) return false;
  if ((uintptr_t)d.b1 % 16 || (uintptr_t)d.b2 % 16 || (uintptr_t)d.g_ffn % 16) return false;
  if (d.a_sm % 8 || d.a_sg % 8 || d.b1_sg % 8 || d.b2_sg % 8 || d.w1_sg % 8 || d.w2_sg % 8) return false;
  if (!rowmap_vec_ok(d.res) || !rowmap_vec_ok(d.out) || !d.out.f32) return false;
  if (d.hout.base && (!rowmap_vec_ok(d.hout) || d.hout.f32 || (uintptr_t)d.g_next % 16)) return false;
  return encode_fn() != nullptr;
}

// TMA map over the rows a FfnDesc enumerates for row map r (element size es,
// box of bc columns x 128 rows).  False when the rows are not a strided 2-D
// set (a flattened enumeration whose batches are not back to back).
inline bool make_rows_tmap(CUtensorMap* map, const FfnDesc& d, const RowMap& r, bool f32, int bc, int& swap) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !r.base || ((uintptr_t)r.base % 16) || r.split < FfnCfg::D) return false;
  const uint64_t es = f32 ? 4 : 2;
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
  const cuuint64_t dims[3] = {(cuuint64_t)FfnCfg::D, swap ? g_ext : m_ext, swap ? m_ext : g_ext};
  const cuuint64_t strides[2] = {(swap ? s_g : s_m) * es, (swap ? s_m : s_g) * es};
  const cuuint32_t box[3] = {(cuuint32_t)bc, swap ? 1u : 128u, swap ? 128u : 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (strides[0] % 16 || strides[1] % 16) return false;
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, r.base, dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline onetrans_status tc_ffn_launch(const FfnDesc& d, cudaStream_t st) {
  using C = FfnCfg;
  CUtensorMap ta, two, tw1, tw2, tres, tout, thout;
  const uint64_t mext = (uint64_t)d.a_mext, gext = (uint64_t)d.a_gext;
  const uint64_t s_m = (uint64_t)d.a_sm, s_g = gext > 1 ? (uint64_t)d.a_sg : mext * (uint64_t)d.a_sm;
  const int a_swap = (gext > 1 && d.a_sg < d.a_sm) ? 1 : 0;
  const uint64_t wg = (uint64_t)d.w_groups;
  bool ok = a_swap ? make_tmap_3d(&ta, d.A, C::D, gext, mext, s_g, s_m, 64, 1, 128)
                   : make_tmap_3d(&ta, d.A, C::D, mext, gext, s_m, s_g, 64, 128, 1);
  ok = ok && make_tmap_3d(&two, d.Wo, C::D, C::D, 1, C::D, (uint64_t)C::D * C::D, 64, 256, 1);
  ok = ok && make_tmap_3d(&tw1, d.W1, C::D, d.dff, wg, C::D, wg > 1 ? (uint64_t)d.w1_sg : (uint64_t)d.dff * C::D,
                          64, C::HC, 1);  // one k-block of a hidden chunk: [256 x 64]
  ok = ok && make_tmap_3d(&tw2, d.W2, d.dff, C::D, wg, d.dff, wg > 1 ? (uint64_t)d.w2_sg : (uint64_t)d.dff * C::D,
                          64, 256, 1);
  if (!ok) return ONETRANS_ERR_CUDA;
  FfnIo io;
  memset(&io, 0, sizeof(io));
  io.res_f32 = d.res.f32;
  io.res_tma = make_rows_tmap(&tres, d, d.res, d.res.f32, d.res.f32 ? 32 : 64, io.res_swap);
  io.out_tma = make_rows_tmap(&tout, d, d.out, true, 32, io.out_swap);
  io.hout_tma = d.hout.base ? make_rows_tmap(&thout, d, d.hout, false, 64, io.hout_swap) : 0;
  if (!io.res_tma) tres = ta;
  if (!io.out_tma) tout = ta;
  if (!io.hout_tma) thout = ta;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(ffn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return ONETRANS_ERR_CUDA;
    attr_set = true;
  }
  dim3 grid((unsigned)((d.M + C::BM - 1) / C::BM), (unsigned)d.G);
  launch_dependent(ffn_tc_kernel, grid, dim3(kFfnThreads), C::SMEM, st, ta, two, tw1, tw2, tres, tout, thout, d, a_swap, io);
  return cudaGetLastError() == cudaSuccess ? ONETRANS_OK : ONETRANS_ERR_CUDA;
}

}  // namespace ot
