// Tensor-core attention of the training step (sm_100a, d_h = 64), on the
// rows the backward recomputes: qkv [B, L, 3d] (q | k | v of every row, q
// unscaled, bf16); the Lq queries are the tail rows L - Lq .. L - 1, query t
// at key position L - Lq + t sees keys 0 .. that position.
//
//  * attn_train_fwd_kernel: one CTA per 128 queries of one head; per
//    128-key tile S = Q K^T (tcgen05, TMEM), online softmax in base 2 with
//    the lazy rescale, O += P V with P from TMEM; writes the output rows and
//    each row's log-sum-exp for the backward.
//  * attn_train_dq_kernel: per 64 keys S = Q K^T and dP = dO V^T, then
//    P = exp(S / sqrt(d_h) - lse) and dS = P (dP - D) per row (D = dO . O),
//    dQ += dS K with dS from TMEM; dQ / sqrt(d_h) into dqkv.
//  * attn_train_kv_kernel (dK, dV): one CTA per 128 keys of one head; per
//    64 queries S^T = K Q^T and dP^T = V dO^T, then P^T and dS^T per key
//    row, dV += P^T dO and dK += dS^T Q with P^T, dS^T from TMEM.
//
// Roles (192 threads): warps 0-3 own one TMEM lane (row) each, warp 4 loads
// tiles by TMA through a 2-stage ring, warp 5 issues the MMAs.  Every wait is
// bounded (a timeout sets the device status word and the CTA drains).  Two
// CTAs per SM, 256 TMEM columns each.
#pragma once
#include "tc_ptx.cuh"

namespace ot {

struct TrainAttnArgs {
  int B, L, Lq, H, d;
  const float* lse;      // [B, H, Lq] log-sum-exp, natural units (dQ, dK/dV)
  float* lse_out;        // forward: written
  const float* Dr;       // [B, H, Lq] dO . O per query row (dQ, dK/dV)
  __nv_bfloat16* o;      // forward: output rows [B, Lq, d]
  __nv_bfloat16* dqkv;   // [B, L, 3d]: dq into the q columns, dk / dv into k / v (bf16: the next GEMMs' operand)
};

struct TrainAttnCfg {
  static constexpr int DH = 64, BM = 128, BN = 128, BOX = 16384, STAGES = 2;
  static constexpr int BAR_BYTES = 256;
  // 6 tiles of 16 KB, the barriers, a query tile's log-sum-exp and D (1 KB):
  // two CTAs fit an SM
  static constexpr int SMEM = 6 * BOX + BAR_BYTES + 2 * BM * 4;
};

__device__ inline float ex2_t(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline float fmax3_t(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Forward: one CTA per 128 queries of one head, two CTAs per SM (S 0-127,
// O 128-191, P 192-255 of 256 TMEM columns).  S of key tile kt+1 is
// computed while the softmax of tile kt runs.
__global__ void __launch_bounds__(192, 2)
    attn_train_fwd_kernel(const __grid_constant__ CUtensorMap tmQKV, const TrainAttnArgs a) {
  using C = TrainAttnCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + 2 * C::BOX;   // [stage][K | V]
  uint64_t* bars = (uint64_t*)(smem + 6 * C::BOX);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;              // [STAGES]
  uint64_t* kv_empty = kv_full + C::STAGES;  // [STAGES]
  uint64_t* s_full = kv_empty + C::STAGES;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* p_free = s_full + 3;
  uint64_t* o_done = s_full + 4;
  uint32_t* tmem_slot = (uint32_t*)(s_full + 5);
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * C::BM, h = blockIdx.y, b = blockIdx.z;
  const int q_off = a.L - a.Lq;
  const int t_last = min(a.Lq, t0 + C::BM) - 1;
  const int nt = (q_off + t_last + 1 + C::BN - 1) / C::BN;   // key tiles
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_done, 1);
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) prefetch_tmap(&tmQKV);
  if (warp == 5) tmem_alloc(tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128, tP = tmem + 192;
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 4) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      mbar_expect_tx(q_full, C::BOX);
      tma_load_3d(&tmQKV, q_full, sQ, h * C::DH, q_off + t0, b);
      for (int kt = 0; kt < nt; ++kt) {
        const int s = kt % C::STAGES;
        if (kt >= C::STAGES && !mbar_wait(&kv_empty[s], ((kt / C::STAGES) - 1) & 1)) break;
        mbar_expect_tx(&kv_full[s], 2 * C::BOX);
        uint8_t* sk = sKV + s * 2 * C::BOX;
        tma_load_3d(&tmQKV, &kv_full[s], sk, a.d + h * C::DH, kt * C::BN, b);
        tma_load_3d(&tmQKV, &kv_full[s], sk + C::BOX, 2 * a.d + h * C::DH, kt * C::BN, b);
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_ss = idesc_bf16(128, 128);
      constexpr uint32_t id_ts = idesc_bf16(128, C::DH, false, true);
      const uint64_t dq = sdesc_k128(smem_u32(sQ));
      const uint64_t dk0 = sdesc_k128(smem_u32(sKV));
      const uint64_t dv0 = sdesc_mn128(smem_u32(sKV + C::BOX), 0);   // V as the MN-major B operand
      auto issue_s = [&](int kt) {
        const uint64_t dk = desc_add(dk0, (kt % C::STAGES) * 2 * C::BOX);
#pragma unroll
        for (int k = 0; k < C::DH / 16; ++k) umma_bf16(tS, desc_add(dq, k * 32), desc_add(dk, k * 32), id_ss, k ? 1u : 0u);
        umma_commit(s_full);
      };
      bool ok = mbar_wait(q_full, 0) && mbar_wait(&kv_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int kt = 0; kt < nt && ok; ++kt) {
        // S of tile kt is in registers: tile kt+1's may overwrite it
        if (kt + 1 < nt) {
          ok = mbar_wait(s_free, kt & 1) && mbar_wait(&kv_full[(kt + 1) % C::STAGES], ((kt + 1) / C::STAGES) & 1);
          if (!ok) break;
          tc_fence_after();
          issue_s(kt + 1);
        }
        ok = mbar_wait(p_full, kt & 1);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dv = desc_add(dv0, (kt % C::STAGES) * 2 * C::BOX);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tO, tP + kk * 8, desc_add(dv, kk * 2048), id_ts, (kt || kk) ? 1u : 0u);
        umma_commit(p_free);
        umma_commit(&kv_empty[kt % C::STAGES]);
      }
      umma_commit(o_done);
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int r = warp * 32 + lane;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    const int t = t0 + r, pos = q_off + t;
    const bool row_ok = t < a.Lq;
    const float c = 1.4426950408889634f * 0.125f;   // log2(e) / sqrt(64): base-2 logits
    const long long si = ((long long)b * a.H + h) * a.Lq + t;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = 0; kt < nt && ok; ++kt) {
      ok = mbar_wait(s_full, kt & 1);
      if (!ok) break;
      tc_fence_after();
      const int kbase = kt * C::BN;
      const int hi = row_ok ? min(max(pos + 1 - kbase, 0), C::BN) : 0;   // visible keys: [0, hi)
      float sv[128];
      tmem_ld128(tS + lb, sv);
      tc_fence_before();
      mbar_arrive(s_free);
#pragma unroll
      for (int i = 0; i < 128; ++i) sv[i] = i < hi ? sv[i] * c : -INFINITY;
      float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; i += 8) {
        m0 = fmax3_t(m0, sv[i], sv[i + 1]);
        m1 = fmax3_t(m1, sv[i + 2], sv[i + 3]);
        m2 = fmax3_t(m2, sv[i + 4], sv[i + 5]);
        m3 = fmax3_t(m3, sv[i + 6], sv[i + 7]);
      }
      const float mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m + 8.f) {
        if (m != -INFINITY) {
          alpha = ex2_t(m - mt);
          rescale = true;
        }
        m = mt;
      }
      const float mref = m == -INFINITY ? 0.f : m;
      float s0 = 0.f, s1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float pa = ex2_t(sv[2 * i] - mref), pb = ex2_t(sv[2 * i + 1] - mref);
        s0 += pa;
        s1 += pb;
        pk[i] = pack_bf16x2(pa, pb);
      }
      l = l * alpha + (s0 + s1);
      if (kt > 0) {
        ok = mbar_wait(p_free, (kt - 1) & 1);
        if (!ok) break;
        tc_fence_after();
      }
      // tcgen05.ld/st are warp-collective: the warp rescales when any row does
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int cc = 0; cc < C::DH / 32; ++cc) {
          float ov[32];
          tmem_ld32(tO + lb + cc * 32, ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tmem_st32(tO + lb + cc * 32, ov);
        }
      }
      tmem_st64(tP + lb, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    ok = ok && mbar_wait(o_done, 0);
    tc_fence_after();
    float o[C::DH];
#pragma unroll
    for (int cc = 0; cc < C::DH / 32; ++cc) tmem_ld32(tO + lb + cc * 32, o + cc * 32);
    if (ok && row_ok) {
      const float inv = 1.f / l;
#pragma unroll
      for (int e = 0; e < C::DH; ++e) o[e] *= inv;
      __nv_bfloat16* dst = a.o + ((long long)b * a.Lq + t) * a.d + h * C::DH;
#pragma unroll
      for (int cc = 0; cc < C::DH / 32; ++cc) store_bf16x32(dst + cc * 32, o + cc * 32);
      a.lse_out[si] = (m + log2f(l)) * 0.6931471805599453f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, 256);
}

// dQ: one CTA per 128 queries of one head, two CTAs per SM.  Each key tile is
// taken in two halves of 64 keys: S = Q K^T and dP = dO V^T (N = 64) into
// TMEM, then dS = P (dP - D), P = 2^(S c - lse), written as bf16 over the S
// columns already read (S 0-63, dP 64-127, dQ 128-191 of 256 columns), then
// dQ += dS K with dS from TMEM.  The next half's products wait for that one
// (its commit); the SM's other CTA fills the gaps.
__global__ void __launch_bounds__(192, 2)
    attn_train_dq_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                         const TrainAttnArgs a) {
  using C = TrainAttnCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::BOX;
  uint8_t* sKV = smem + 2 * C::BOX;   // [stage][K | V]
  uint64_t* bars = (uint64_t*)(smem + 6 * C::BOX);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;              // [STAGES]
  uint64_t* kv_empty = kv_full + C::STAGES;  // [STAGES]
  uint64_t* s_full = kv_empty + C::STAGES;   // S and dP of a half are in TMEM
  uint64_t* p_full = s_full + 1;             // dS of a half is in TMEM
  uint64_t* p_free = s_full + 2;             // dQ of a half is done
  uint64_t* o_done = s_full + 3;
  uint32_t* tmem_slot = (uint32_t*)(s_full + 4);
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * C::BM, h = blockIdx.y, b = blockIdx.z;
  const int q_off = a.L - a.Lq;
  const int t_last = min(a.Lq, t0 + C::BM) - 1;
  const int nt = (q_off + t_last + 1 + C::BN - 1) / C::BN;   // key tiles
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_done, 1);
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmQKV);
    prefetch_tmap(&tmDO);
  }
  if (warp == 5) tmem_alloc(tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tDP = tmem + 64, tQ = tmem + 128;
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 4) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      mbar_expect_tx(q_full, 2 * C::BOX);
      tma_load_3d(&tmQKV, q_full, sQ, h * C::DH, q_off + t0, b);
      tma_load_3d(&tmDO, q_full, sDO, h * C::DH, t0, b);
      for (int kt = 0; kt < nt; ++kt) {
        const int s = kt % C::STAGES;
        if (kt >= C::STAGES && !mbar_wait(&kv_empty[s], ((kt / C::STAGES) - 1) & 1)) break;
        mbar_expect_tx(&kv_full[s], 2 * C::BOX);
        uint8_t* sk = sKV + s * 2 * C::BOX;
        tma_load_3d(&tmQKV, &kv_full[s], sk, a.d + h * C::DH, kt * C::BN, b);
        tma_load_3d(&tmQKV, &kv_full[s], sk + C::BOX, 2 * a.d + h * C::DH, kt * C::BN, b);
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_ss = idesc_bf16(128, 64);
      constexpr uint32_t id_ts = idesc_bf16(128, C::DH, false, true);
      const uint64_t dq = sdesc_k128(smem_u32(sQ)), ddo = sdesc_k128(smem_u32(sDO));
      const uint64_t dk0 = sdesc_k128(smem_u32(sKV)), dv0 = sdesc_k128(smem_u32(sKV + C::BOX));
      const uint64_t mk0 = sdesc_mn128(smem_u32(sKV), 0);   // K as the MN-major B operand of dS K
      bool ok = mbar_wait(q_full, 0);
      for (int kt = 0; kt < nt && ok; ++kt) {
        const int s = kt % C::STAGES;
        ok = mbar_wait(&kv_full[s], (kt / C::STAGES) & 1);
        if (!ok) break;
        for (int kh = 0; kh < 2 && ok; ++kh) {
          const int hf = 2 * kt + kh;
          // the previous half's dQ has read dS from the S columns
          if (hf > 0) ok = mbar_wait(p_free, (hf - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          // keys kh*64 .. of the K and V tiles: 64 rows x 128 B further in
          const uint32_t so = s * 2 * C::BOX + kh * 8192;
#pragma unroll
          for (int k = 0; k < C::DH / 16; ++k)
            umma_bf16(tS, desc_add(dq, k * 32), desc_add(desc_add(dk0, so), k * 32), id_ss, k ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < C::DH / 16; ++k)
            umma_bf16(tDP, desc_add(ddo, k * 32), desc_add(desc_add(dv0, so), k * 32), id_ss, k ? 1u : 0u);
          umma_commit(s_full);
          ok = mbar_wait(p_full, hf & 1);
          if (!ok) break;
          tc_fence_after();
          const uint64_t mk = desc_add(mk0, so);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tQ, tS + kk * 8, desc_add(mk, kk * 2048), id_ts, (hf || kk) ? 1u : 0u);
          umma_commit(p_free);
        }
        umma_commit(&kv_empty[s]);
      }
      umma_commit(o_done);
    }
  } else {
    // ------------------------------------------------------ dS + epilogue
    const int r = warp * 32 + lane;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    const int t = t0 + r, pos = q_off + t;
    const bool row_ok = t < a.Lq;
    const float c = 1.4426950408889634f * 0.125f;
    const long long si = ((long long)b * a.H + h) * a.Lq + t;
    float lse2 = 0.f, Dv = 0.f;
    if (row_ok) {
      lse2 = a.lse[si] * 1.4426950408889634f;
      Dv = a.Dr[si];
    }
    bool ok = true;
    for (int kt = 0; kt < nt && ok; ++kt) {
      const int hi = row_ok ? min(max(pos + 1 - kt * C::BN, 0), C::BN) : 0;   // visible keys of the tile: [0, hi)
      for (int kh = 0; kh < 2 && ok; ++kh) {
        ok = mbar_wait(s_full, (2 * kt + kh) & 1);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          float sv[32], dp[32];
          tmem_ld32(tS + lb + qq * 32, sv);
          tmem_ld32(tDP + lb + qq * 32, dp);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = kh * 64 + qq * 32 + 2 * i;
            const float pa = c0 < hi ? ex2_t(fmaf(sv[2 * i], c, -lse2)) : 0.f;
            const float pb = c0 + 1 < hi ? ex2_t(fmaf(sv[2 * i + 1], c, -lse2)) : 0.f;
            pk[i] = pack_bf16x2(pa * (dp[2 * i] - Dv), pb * (dp[2 * i + 1] - Dv));
          }
          // over columns already read: chunk qq's 16 packed columns land on S columns 16 qq ..
          tmem_st16(tS + lb + qq * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
      }
    }
    ok = ok && mbar_wait(o_done, 0);
    tc_fence_after();
    float o[C::DH];
#pragma unroll
    for (int cc = 0; cc < C::DH / 32; ++cc) tmem_ld32(tQ + lb + cc * 32, o + cc * 32);
    if (ok && row_ok) {
      __nv_bfloat16* dst = a.dqkv + ((long long)b * a.L + pos) * 3 * a.d + h * C::DH;
#pragma unroll
      for (int e = 0; e < C::DH; ++e) o[e] *= 0.125f;
#pragma unroll
      for (int cc = 0; cc < C::DH / 32; ++cc) store_bf16x32(dst + cc * 32, o + cc * 32);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, 256);
}

// dK, dV: one CTA per 128 keys of one head, two CTAs per SM.  Each query
// tile is taken in two halves of 64 queries: S^T = K Q^T and dP^T = V dO^T
// (N = 64) into TMEM, then P^T and dS^T written as bf16 over the S^T and
// dP^T columns already read (so 256 TMEM columns hold S^T, dP^T, dV and
// dK), then dV += P^T dO and dK += dS^T Q with the A operands from TMEM.  The
// next half's products wait for those two (their commit), so one CTA runs
// its products and its softmax in turn and the SM's other CTA fills the gaps.
__global__ void __launch_bounds__(192, 2)
    attn_train_kv_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                         const TrainAttnArgs a) {
  using C = TrainAttnCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::BOX;
  uint8_t* sQD = smem + 2 * C::BOX;   // [stage][Q | dO]
  uint64_t* bars = (uint64_t*)(smem + 6 * C::BOX);
  uint64_t* kv_ready = bars;
  uint64_t* qd_full = bars + 1;              // [STAGES]
  uint64_t* qd_empty = qd_full + C::STAGES;  // [STAGES]
  uint64_t* s_full = qd_empty + C::STAGES;   // S^T and dP^T of a half are in TMEM
  uint64_t* p_full = s_full + 1;             // P^T and dS^T of a half are in TMEM
  uint64_t* p_free = s_full + 2;             // dV and dK of a half are done
  uint64_t* o_done = s_full + 3;
  uint32_t* tmem_slot = (uint32_t*)(s_full + 4);
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * C::BN, h = blockIdx.y, b = blockIdx.z;
  const int q_off = a.L - a.Lq;
  const int it0 = max(0, j0 - q_off) / C::BM;            // first query tile that sees a key of this tile
  const int nq = (a.Lq + C::BM - 1) / C::BM - it0;       // query tiles
  if (threadIdx.x == 0) {
    mbar_init(kv_ready, 1);
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&qd_full[i], 1); mbar_init(&qd_empty[i], 1); }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_done, 1);
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmQKV);
    prefetch_tmap(&tmDO);
  }
  if (warp == 5) tmem_alloc(tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S^T 0-63 (P^T over its first 32), dP^T 64-127 (dS^T over its first 32), dV 128-191, dK 192-255
  const uint32_t tS = tmem, tDP = tmem + 64, tDV = tmem + 128, tDK = tmem + 192;
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 4) {
    if (lane == 0) {
      mbar_expect_tx(kv_ready, 2 * C::BOX);
      tma_load_3d(&tmQKV, kv_ready, sK, a.d + h * C::DH, j0, b);
      tma_load_3d(&tmQKV, kv_ready, sV, 2 * a.d + h * C::DH, j0, b);
      for (int i = 0; i < nq; ++i) {
        const int s = i % C::STAGES, q0 = (it0 + i) * C::BM;
        if (i >= C::STAGES && !mbar_wait(&qd_empty[s], ((i / C::STAGES) - 1) & 1)) break;
        mbar_expect_tx(&qd_full[s], 2 * C::BOX);
        uint8_t* sq = sQD + s * 2 * C::BOX;
        tma_load_3d(&tmQKV, &qd_full[s], sq, h * C::DH, q_off + q0, b);
        tma_load_3d(&tmDO, &qd_full[s], sq + C::BOX, h * C::DH, q0, b);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t id_ss = idesc_bf16(128, 64);
      constexpr uint32_t id_ts = idesc_bf16(128, C::DH, false, true);
      const uint64_t dk = sdesc_k128(smem_u32(sK)), dv = sdesc_k128(smem_u32(sV));
      const uint64_t dq0 = sdesc_k128(smem_u32(sQD)), ddo0 = sdesc_k128(smem_u32(sQD + C::BOX));
      const uint64_t mq0 = sdesc_mn128(smem_u32(sQD), 0), mdo0 = sdesc_mn128(smem_u32(sQD + C::BOX), 0);
      bool ok = mbar_wait(kv_ready, 0);
      for (int i = 0; i < nq && ok; ++i) {
        const int s = i % C::STAGES;
        ok = mbar_wait(&qd_full[s], (i / C::STAGES) & 1);
        if (!ok) break;
        for (int qh = 0; qh < 2 && ok; ++qh) {
          const int hf = 2 * i + qh;
          // the previous half's dV, dK have read P^T and dS^T from these columns
          if (hf > 0) ok = mbar_wait(p_free, (hf - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          // rows qh*64 .. of the Q and dO tiles: 64 rows x 128 B further in
          const uint32_t so = s * 2 * C::BOX + qh * 8192;
          // S^T = K Q^T and dP^T = V dO^T: keys on the TMEM lanes, 64 queries on the columns
#pragma unroll
          for (int k = 0; k < C::DH / 16; ++k)
            umma_bf16(tS, desc_add(dk, k * 32), desc_add(desc_add(dq0, so), k * 32), id_ss, k ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < C::DH / 16; ++k)
            umma_bf16(tDP, desc_add(dv, k * 32), desc_add(desc_add(ddo0, so), k * 32), id_ss, k ? 1u : 0u);
          umma_commit(s_full);
          ok = mbar_wait(p_full, hf & 1);
          if (!ok) break;
          tc_fence_after();
          // dV += P^T dO, dK += dS^T Q: A from TMEM (16 queries per step), B MN-major
          const uint64_t mdo = desc_add(mdo0, so), mq = desc_add(mq0, so);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tDV, tS + kk * 8, desc_add(mdo, kk * 2048), id_ts, (hf || kk) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tDK, tDP + kk * 8, desc_add(mq, kk * 2048), id_ts, (hf || kk) ? 1u : 0u);
          umma_commit(p_free);
        }
        umma_commit(&qd_empty[s]);
      }
      umma_commit(o_done);
    }
  } else {
    const int r = warp * 32 + lane;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    const int j = j0 + r;
    const bool key_ok = j < a.L;
    const float c = 1.4426950408889634f * 0.125f;
    const float* lse = a.lse + ((long long)b * a.H + h) * a.Lq;
    const float* Dr = a.Dr + ((long long)b * a.H + h) * a.Lq;
    // the query tile's log-sum-exp (base 2) and D, one column per softmax thread
    float* s_lse = (float*)(smem + 6 * C::BOX + C::BAR_BYTES);
    float* s_D = s_lse + C::BM;
    bool ok = true;
    // every softmax thread passes both named barriers on every tile, even
    // after a wait that gave up, so that none is left waiting at one
    for (int i = 0; i < nq; ++i) {
      const int q0 = (it0 + i) * C::BM;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      s_lse[r] = q0 + r < a.Lq ? lse[q0 + r] * 1.4426950408889634f : 0.f;
      s_D[r] = q0 + r < a.Lq ? Dr[q0 + r] : 0.f;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // query column cc of the tile sees this key when q_off + q0 + cc >= j, and exists when q0 + cc < Lq
      const int lo = key_ok ? min(max(j - q_off - q0, 0), C::BM) : C::BM;
      const int hi = min(max(a.Lq - q0, 0), C::BM);
      for (int qh = 0; qh < 2; ++qh) {
        if (!ok) continue;
        ok = mbar_wait(s_full, (2 * i + qh) & 1);
        if (!ok) continue;
        tc_fence_after();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          float sv[32], dp[32];
          tmem_ld32(tS + lb + qq * 32, sv);
          tmem_ld32(tDP + lb + qq * 32, dp);
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p2[2], d2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int cc = qh * 64 + qq * 32 + 2 * e + u;
              const bool vis = cc >= lo && cc < hi;
              const float p = vis ? ex2_t(fmaf(sv[2 * e + u], c, -s_lse[cc])) : 0.f;
              p2[u] = p;
              d2[u] = p * (dp[2 * e + u] - s_D[cc]);
            }
            pk[e] = pack_bf16x2(p2[0], p2[1]);
            dk[e] = pack_bf16x2(d2[0], d2[1]);
          }
          // over columns already read: chunk qq's 16 packed columns land on S^T / dP^T columns 16 qq ..
          tmem_st16(tS + lb + qq * 16, pk);
          tmem_st16(tDP + lb + qq * 16, dk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
      }
    }
    ok = ok && mbar_wait(o_done, 0);
    tc_fence_after();
    float dv[C::DH], dkv[C::DH];
#pragma unroll
    for (int cc = 0; cc < C::DH / 32; ++cc) {
      tmem_ld32(tDV + lb + cc * 32, dv + cc * 32);
      tmem_ld32(tDK + lb + cc * 32, dkv + cc * 32);
    }
    if (ok && key_ok) {
      __nv_bfloat16* dst = a.dqkv + ((long long)b * a.L + j) * 3 * a.d + h * C::DH;
#pragma unroll
      for (int e = 0; e < C::DH; ++e) dkv[e] *= 0.125f;
#pragma unroll
      for (int cc = 0; cc < C::DH / 32; ++cc) {
        store_bf16x32(dst + a.d + cc * 32, dkv + cc * 32);
        store_bf16x32(dst + 2 * a.d + cc * 32, dv + cc * 32);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, 256);
}

// D[b][h][t] = sum over e of dO[b, t, h, e] O[b, t, h, e] (d_h = 64): one
// warp per row (b, t), each lane eight consecutive elements of dO and O (one
// 16-byte load each), the eight lanes of a head added by shuffles.
__global__ void __launch_bounds__(256) attn_train_delta_kernel(const __nv_bfloat16* __restrict__ dO,
                                                               const __nv_bfloat16* __restrict__ O,
                                                               float* __restrict__ Dr, int B, int Lq, int H) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= (long long)B * Lq) return;
  const int d = H * 64;
  const int b = (int)(row / Lq), t = (int)(row - (long long)b * Lq);
  for (int base = 0; base < d; base += 256) {   // the same trip count in every lane
    const int e0 = base + 8 * lane;
    float acc = 0.f;
    if (e0 < d) {
      const uint4 a = *(const uint4*)(dO + row * d + e0);
      const uint4 o = *(const uint4*)(O + row * d + e0);
      const __nv_bfloat162* ah = (const __nv_bfloat162*)&a;
      const __nv_bfloat162* oh = (const __nv_bfloat162*)&o;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x = __bfloat1622float2(ah[j]), y = __bfloat1622float2(oh[j]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if ((lane & 7) == 0 && e0 < d) Dr[((long long)b * H + e0 / 64) * Lq + t] = acc;
  }
}

}  // namespace ot
