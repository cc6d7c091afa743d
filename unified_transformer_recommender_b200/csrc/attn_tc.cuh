// Tensor-core attention for the bf16 path (sm_100a), head dims 64 and 96.
//
// One CTA owns 128 query rows of one head.  K/V tiles of 128 keys are
// streamed by TMA through a 3-stage shared-memory ring.  Per key tile:
//   S = Q K^T          tcgen05.mma into TMEM (fp32)
//   softmax            four warps read their query row back with tcgen05.ld
//                      (one row per thread, so the row max and sum stay in the
//                      thread), mask, and write P = 2^(S - m) as bf16 pairs
//                      into TMEM (online softmax in base 2: queries arrive
//                      pre-scaled by 1/sqrt(d_h)*log2(e))
//   O += P V           tcgen05.mma with P read from TMEM and V from shared
//                      memory (MN-major); O stays in TMEM for the whole row
// The running max m is raised only when a tile's max passes it by more than
// 2^8; then the thread rescales l, and its warp the O rows in TMEM (a
// warp-collective load and store, alpha = 1 for rows that keep their max).
// S of tile t+1 is computed while the softmax of tile t runs; two CTAs share
// an SM.
//
// Query kinds:
//  * MODE_CAUSAL  (Stage I, forward, append): query t of sequence b sits at
//    key position q_pos0 + t (q_pos0_u[b] + t when the sequences' cached
//    lengths differ, as in an append) and sees keys 0 .. that position, all
//    from 64-token KV-cache pages.  Only the tail rows are queries (the
//    pyramid's Q set); keys span the layer input.
//  * MODE_STAGE2: rows are NS tokens of up to floor(128/L_NS) candidates of one
//    user, candidate-major (row r = candidate r / L_NS, token r % L_NS).  They
//    see every cached S key of the user (s_len, or s_len_u[user] when users
//    hold different lengths), then one more key tile holding the
//    same candidates' own NS keys, masked to (same candidate, token <= own):
//    one softmax over the union, every product on tensor cores.
//
// Warp roles (192 threads): warps 0-3 softmax/epilogue, warp 4 TMA, warp 5 MMA.
#pragma once
#include "tc_ptx.cuh"

namespace ot {

enum : int { MODE_CAUSAL = 0, MODE_STAGE2 = 1 };

struct TcAttnArgs {
  int mode;
  // causal
  int Lq, q_pos0;
  const int* q_pos0_u;  // per batch, or null: q_pos0 for all
  RowMap o;
  // stage II
  const int* tiles;   // {user, c0, c1} per blockIdx.x
  __nv_bfloat16* o2;  // [C_tot, L_NS, d]
  int L_NS, s_len;
  const int* s_len_u;  // cached S keys per user, or null: s_len for all
  // shared
  KVStore kv;
  int H;
};

// Head dims 64 and 96.  A row of d_h bf16 is held as NB boxes of 64 columns
// (128-byte swizzle atoms); for d_h = 96 the second box's columns 96..127
// are the TMA's zero fill or a neighbouring head's values, which no product
// reads (Q K^T stops after d_h / 16 k-steps, P.V has N = d_h).
template <int DH_>
struct AttnCfgT {
  static constexpr int DH = DH_, BM = 128, BN = 128;
  static constexpr int NB = (DH + 63) / 64;
  static constexpr int BOX_BYTES = 128 * 128;     // 128 rows x 64 bf16
  static constexpr int Q_BYTES = NB * BOX_BYTES;
  static constexpr int KV_BYTES = NB * BOX_BYTES; // one of K or V for 128 keys
  static constexpr int PAGE_BYTES = 64 * 128;     // one 64-token page of one box
  // d_h = 64: S 0..127, O 128..191, P (bf16 pairs) 192..255, two CTAs per SM;
  // d_h = 96: S 0..127, O 128..223, P 224..287 of 512 columns, one CTA per SM
  static constexpr int T_O = 128, T_P = 128 + (DH + 31) / 32 * 32;
  static constexpr int TMEM_COLS = DH <= 64 ? 256 : 512;
  static constexpr int CTAS = DH <= 64 ? 2 : 1;
  // three K/V stages: the load of tile kt+1 may start while P.V of tile kt-1
  // still reads its stage (two CTAs of 115 KB share an SM's 228 KB at d_h = 64)
  static constexpr int STAGES = 3;
  static constexpr int BAR_BYTES = 128;
  static constexpr int MAX_PAGES = 128;           // page ids cached in shared memory (8192 keys)
  static constexpr int SMEM = Q_BYTES + STAGES * 2 * KV_BYTES + BAR_BYTES + MAX_PAGES * 4;
};

__device__ inline int kv_page_id(const KVStore& kv, int b, int page_idx) {
  return kv.table ? kv.table[kv.row_off[b] + page_idx] : b * kv.pps + page_idx;
}

// max(a, b, c) in one instruction (sm_100 three-input max.f32)
__device__ inline float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ inline float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


template <int DH>
__global__ void __launch_bounds__(192, AttnCfgT<DH>::CTAS)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                   const __grid_constant__ CUtensorMap tmNS, const TcAttnArgs a) {
  using C = AttnCfgT<DH>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + C::Q_BYTES;  // [stage][K|V][box][128 keys][64]
  uint64_t* bars = (uint64_t*)(sKV + C::STAGES * 2 * C::KV_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                // [STAGES]
  uint64_t* kv_empty = kv_full + C::STAGES;    // [STAGES]
  uint64_t* s_full = kv_empty + C::STAGES;
  uint64_t* p_full = s_full + 1;
  uint64_t* p_free = s_full + 2;
  uint64_t* o_done = s_full + 3;
  uint64_t* s_free = s_full + 4;               // the softmax has read S of the current tile
  uint32_t* tmem_slot = (uint32_t*)(s_full + 5);
  int* s_pages = (int*)((uint8_t*)bars + C::BAR_BYTES);

  // the swizzled tiles need 1024-byte alignment; refuse to run without it
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) flag_error(kErrSmemAlign);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_done, 1);
    mbar_init(s_free, 128);
    fence_barrier_init();
  }
  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKV);
      if (a.mode == MODE_STAGE2) prefetch_tmap(&tmNS);
    }
  }
  if (warp == 5) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + C::T_O, tP = tmem + C::T_P;
  grid_dep_wait();
  grid_dep_launch();

  // ---- work of this CTA
  int b, row0, n_keys_s, kmax, nt, n_rows = C::BM;
  int c0 = 0, q_pos0 = a.q_pos0;
  if (a.mode == MODE_CAUSAL) {
    b = blockIdx.z;
    if (a.q_pos0_u) q_pos0 = a.q_pos0_u[b];
    row0 = blockIdx.x * C::BM;
    const int t_last = min(a.Lq, row0 + C::BM) - 1;
    kmax = q_pos0 + t_last;
    n_keys_s = kmax + 1;
    nt = (n_keys_s + C::BN - 1) / C::BN;
  } else {
    b = a.tiles[blockIdx.x * 3 + 0];
    c0 = a.tiles[blockIdx.x * 3 + 1];
    const int c1 = a.tiles[blockIdx.x * 3 + 2];
    row0 = c0 * a.L_NS;
    n_rows = (c1 - c0) * a.L_NS;
    n_keys_s = a.s_len_u ? a.s_len_u[b] : a.s_len;
    kmax = n_keys_s - 1;
    nt = (n_keys_s + C::BN - 1) / C::BN + 1;  // + the tile of own NS keys
  }
  const int nt_s = (n_keys_s + C::BN - 1) / C::BN;  // tiles from the KV pages
  const int n_pages_used = (kmax + 1 + 63) / 64;

  if (warp == 4) {
    // page ids of every key page this CTA reads, fetched once (page ids past
    // the cached range read as the out-of-range page, which loads zeros)
    const int n_pg = min(2 * nt_s, C::MAX_PAGES);
    for (int i = lane; i < n_pg; i += 32) s_pages[i] = i < n_pages_used ? kv_page_id(a.kv, b, i) : a.kv.n_pages;
    __syncwarp();
    // ------------------------------------------------------------ producer
    if (lane == 0 && nt > 0) {
      const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
      mbar_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int i = 0; i < C::NB; ++i) {
        if (a.mode == MODE_CAUSAL)
          tma_load_3d_hint(&tmQ, q_full, sQ + i * C::BOX_BYTES, h * C::DH + i * 64, row0, b, stream);
        else
          tma_load_3d_hint(&tmQ, q_full, sQ + i * C::BOX_BYTES, h * C::DH + i * 64, row0, 0, stream);
      }
      for (int kt = 0; kt < nt; ++kt) {
        const int s = kt % C::STAGES;
        if (kt >= C::STAGES && !mbar_wait(&kv_empty[s], ((kt / C::STAGES) - 1) & 1)) break;
        mbar_expect_tx(&kv_full[s], 2 * C::KV_BYTES);
        uint8_t* sk = sKV + s * 2 * C::KV_BYTES;
        uint8_t* sv = sk + C::KV_BYTES;
        if (kt < nt_s) {
#pragma unroll
          for (int hp = 0; hp < 2; ++hp) {
            const int pi = kt * 2 + hp;
            const int pg = pi < C::MAX_PAGES ? s_pages[pi]
                                             : (pi < n_pages_used ? kv_page_id(a.kv, b, pi) : a.kv.n_pages);
#pragma unroll
            for (int i = 0; i < C::NB; ++i) {
              tma_load_4d_hint(&tmKV, &kv_full[s], sk + i * C::BOX_BYTES + hp * C::PAGE_BYTES, i * 64, 0, h, pg, keep);
              tma_load_4d_hint(&tmKV, &kv_full[s], sv + i * C::BOX_BYTES + hp * C::PAGE_BYTES, i * 64, 0, a.H + h, pg,
                               keep);
            }
          }
        } else {
          // own NS keys of this CTA's candidates: the K and V column blocks of the same rows
          const int d = a.H * C::DH;
#pragma unroll
          for (int i = 0; i < C::NB; ++i) {
            tma_load_3d_hint(&tmNS, &kv_full[s], sk + i * C::BOX_BYTES, d + h * C::DH + i * 64, row0, 0, stream);
            tma_load_3d_hint(&tmNS, &kv_full[s], sv + i * C::BOX_BYTES, 2 * d + h * C::DH + i * 64, row0, 0, stream);
          }
        }
      }
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0 && nt > 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128);
      constexpr uint32_t id_pv = idesc_bf16(128, C::DH, false, true);
      constexpr int KS = C::DH / 16;  // k-steps of Q K^T: 4 per 64-column box
      // base descriptors of Q and of each stage's K and V tiles
      const uint64_t dq = sdesc_k128(smem_u32(sQ));
      const uint64_t dk0 = sdesc_k128(smem_u32(sKV));                    // stage s: + s * 2 * KV_BYTES
      // V as the MN-major B operand: 64-column boxes (N atoms) BOX_BYTES apart
      const uint64_t dv0 = sdesc_mn128(smem_u32(sKV + C::KV_BYTES), C::NB > 1 ? C::BOX_BYTES : 0);
      bool ok = mbar_wait(q_full, 0) && mbar_wait(&kv_full[0], 0);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < KS; ++k) {
          const uint32_t off = (k >> 2) * C::BOX_BYTES + (k & 3) * 32;
          umma_bf16(tS, desc_add(dq, off), desc_add(dk0, off), id_qk, k ? 1u : 0u);
        }
        umma_commit(s_full);
      }
      for (int kt = 0; kt < nt && ok; ++kt) {
        // S of tile kt has been read into registers: S of tile kt+1 may
        // overwrite it while the softmax of tile kt runs
        if (kt + 1 < nt) {
          const int s1 = (kt + 1) % C::STAGES;
          ok = mbar_wait(s_free, kt & 1) && mbar_wait(&kv_full[s1], ((kt + 1) / C::STAGES) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dk = desc_add(dk0, s1 * 2 * C::KV_BYTES);
#pragma unroll
          for (int k = 0; k < KS; ++k) {
            const uint32_t off = (k >> 2) * C::BOX_BYTES + (k & 3) * 32;
            umma_bf16(tS, desc_add(dq, off), desc_add(dk, off), id_qk, k ? 1u : 0u);
          }
          umma_commit(s_full);
        }
        // P of tile kt is in TMEM
        ok = mbar_wait(p_full, kt & 1);
        if (!ok) break;
        tc_fence_after();
        // O += P V: P from TMEM (8 columns = 16 keys per step), V from shared memory
        const int s = kt % C::STAGES;
        const uint64_t dv = desc_add(dv0, s * 2 * C::KV_BYTES);
        const uint32_t acc0 = kt ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tO, tP + kk * 8, desc_add(dv, kk * 2048), id_pv, kk ? 1u : acc0);
        umma_commit(p_free);
        umma_commit(&kv_empty[s]);
      }
      umma_commit(o_done);
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int r = warp * 32 + lane;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    const int qpos = q_pos0 + row0 + r;  // causal: last visible key of this row
    const int cand = a.mode == MODE_STAGE2 ? r / a.L_NS : 0;
    const int tok = a.mode == MODE_STAGE2 ? r - cand * a.L_NS : 0;
    const int qpos_min = q_pos0 + row0;  // earliest query of the CTA: bounds the unmasked tiles
    // Running max m is only raised when a tile's max exceeds it by more than
    // 2^8 (then O and l are rescaled); below that, P = 2^(S - m) <= 256 is
    // exact enough in bf16 and the final O / l is unchanged.
    const float kThresh = 8.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = 0; kt < nt && ok; ++kt) {
      ok = mbar_wait(s_full, kt & 1);
      if (!ok) break;
      tc_fence_after();
      const int kbase = kt * C::BN;
      const bool ns_tile = kt >= nt_s;
      // visible keys of this row in this tile: [lo, hi)
      int lo = 0, hi = C::BN;
      if (ns_tile) {
        lo = cand * a.L_NS;
        hi = (r < n_rows) ? lo + tok + 1 : lo;
      } else {
        const int vis_end = a.mode == MODE_CAUSAL ? min(qpos + 1, n_keys_s) : n_keys_s;
        hi = min(max(vis_end - kbase, 0), C::BN);
      }
      const bool full = !ns_tile && (a.mode == MODE_CAUSAL ? (kbase + C::BN - 1 <= qpos_min && kbase + C::BN <= n_keys_s)
                                                          : (kbase + C::BN <= n_keys_s));
      // the row's 128 scores; keys it may not see become -inf
      float sv[128];
      tmem_ld128(tS + lb, sv);
      // S is in registers: release its TMEM columns to the next tile's Q K^T
      tc_fence_before();
      mbar_arrive(s_free);
      if (!full) {
#pragma unroll
        for (int i = 0; i < 128; ++i) sv[i] = (i >= lo && i < hi) ? sv[i] : -INFINITY;
      }
      // tile max over four independent chains of three-input maxima
      float mq0 = -INFINITY, mq1 = -INFINITY, mq2 = -INFINITY, mq3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; i += 8) {
        mq0 = fmax3(mq0, sv[i], sv[i + 1]);
        mq1 = fmax3(mq1, sv[i + 2], sv[i + 3]);
        mq2 = fmax3(mq2, sv[i + 4], sv[i + 5]);
        mq3 = fmax3(mq3, sv[i + 6], sv[i + 7]);
      }
      const float mt = fmaxf(fmaxf(mq0, mq1), fmaxf(mq2, mq3));
      // raise the reference only when this tile passes it by more than 2^kThresh
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m + kThresh) {
        if (m != -INFINITY) {
          alpha = ex2(m - mt);
          rescale = true;
        }
        m = mt;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      // P = 2^(S - m) pair by pair: the subtraction and the row sums on packed
      // fp32 pairs (half the issue slots), the exponentials on the MUFU
      const uint64_t nm2 = f2_pack(-mref, -mref);
      uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const uint64_t x2 = f2_add(f2_pack(sv[2 * i], sv[2 * i + 1]), nm2);
        float xa, xb;
        f2_unpack(x2, xa, xb);
        const uint64_t p2 = f2_pack(ex2(xa), ex2(xb));
        if (i & 1) acc1 = f2_add(acc1, p2);
        else acc0 = f2_add(acc0, p2);
        float pa, pb;
        f2_unpack(p2, pa, pb);
        pk[i] = pack_bf16x2(pa, pb);
      }
      {
        float s0, s1, s2, s3;
        f2_unpack(acc0, s0, s1);
        f2_unpack(acc1, s2, s3);
        l = l * alpha + ((s0 + s1) + (s2 + s3));
      }
      // P of the previous tile must be consumed before this one overwrites it
      if (kt > 0) {
        ok = mbar_wait(p_free, (kt - 1) & 1);
        if (!ok) break;
        tc_fence_after();
      }
      // tcgen05.ld/st are warp-collective: the whole warp rescales when any
      // of its rows does (alpha stays exactly 1 for the others)
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds the tiles before kt (p_free was awaited): bring it to the new max
#pragma unroll
        for (int c = 0; c < C::DH / 32; ++c) {
          float ov[32];
          tmem_ld32(tO + lb + c * 32, ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          uint32_t* ou = (uint32_t*)ov;
          tmem_st16(tO + lb + c * 32, ou);
          tmem_st16(tO + lb + c * 32 + 16, ou + 16);
        }
      }
      tmem_st64(tP + lb, pk);
      // keys past the last valid cache key may hold stale bits (P is 0 there,
      // but 0 * NaN is not): zero their V rows before P.V reads them
      if (kt == nt_s - 1 && kbase + r > kmax) {
#pragma unroll
        for (int i = 0; i < C::NB; ++i) {
          uint4* vrow = (uint4*)(sKV + (kt % C::STAGES) * 2 * C::KV_BYTES + C::KV_BYTES + i * C::BOX_BYTES + r * 128);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) vrow[ch] = make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    ok = ok && mbar_wait(o_done, 0);
    tc_fence_after();
    float o[C::DH];
#pragma unroll
    for (int c = 0; c < C::DH / 32; ++c) tmem_ld32(tO + lb + c * 32, o + c * 32);
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < C::DH; ++e) o[e] *= inv;
    if (ok && nt > 0) {
      __nv_bfloat16* dst = nullptr;
      if (a.mode == MODE_CAUSAL) {
        const int t = row0 + r;
        if (t < a.Lq) dst = (__nv_bfloat16*)a.o.base + rm_off(a.o, b, t, h * C::DH);
      } else if (r < n_rows) {
        dst = a.o2 + (long long)(row0 + r) * (a.H * C::DH) + h * C::DH;
      }
      if (dst) {
#pragma unroll
        for (int c = 0; c < C::DH / 32; ++c) store_bf16x32(dst + c * 32, o + c * 32);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
// 4-D bf16 map over a page pool: (d_h, token, kind*H + head, page).
inline bool make_tmap_pages(CUtensorMap* map, const KVStore& kv) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)kv.dh, (cuuint64_t)kv.P, (cuuint64_t)(2 * kv.H),
                              (cuuint64_t)kv.n_pages};
  const cuuint64_t strides[3] = {(cuuint64_t)kv.dh * 2, (cuuint64_t)kv.P * kv.dh * 2,
                                 (cuuint64_t)2 * kv.H * kv.P * kv.dh * 2};
  const cuuint32_t box[4] = {64, 64, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, kv.pool, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool tc_kv_ok(const KVStore& kv) {
  return (kv.dh == 64 || kv.dh == 96) && kv.P == 64 && kv.n_pages > 0 && ((uintptr_t)kv.pool % 16) == 0 && encode_fn();
}

inline bool tc_attn_supported(const AttnDesc& a) {
  return (a.dh == 64 || a.dh == 96) && a.kv.dh == a.dh && tc_kv_ok(a.kv) && ((uintptr_t)a.q.base % 16) == 0 && a.q.st % 8 == 0 &&
         a.q.sb % 8 == 0 && rowmap_vec_ok(a.o) && !a.o.f32;
}

template <int DH>
inline onetrans_status attn_launch_dh(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& tns,
                                      const TcAttnArgs& args, dim3 grid, cudaStream_t st) {
  using C = AttnCfgT<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return ONETRANS_ERR_CUDA;
    attr_set = true;
  }
  launch_dependent(attn_tc_kernel<DH>, grid, dim3(192), C::SMEM, st, tq, tkv, tns, args);
  return cudaGetLastError() == cudaSuccess ? ONETRANS_OK : ONETRANS_ERR_CUDA;
}

inline onetrans_status attn_launch_common(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& tns,
                                          const TcAttnArgs& args, int dh, dim3 grid, cudaStream_t st) {
  if (dh == 96) return attn_launch_dh<96>(tq, tkv, tns, args, grid, st);
  return attn_launch_dh<64>(tq, tkv, tns, args, grid, st);
}

inline onetrans_status tc_attn_launch(const AttnDesc& a, cudaStream_t st) {
  CUtensorMap tq, tkv;
  const uint64_t d = (uint64_t)a.H * a.dh;
  // Q rows of batch b: base + b*sb + t*st, d columns per row
  if (!make_tmap_3d(&tq, a.q.base, d, (uint64_t)a.Lq, (uint64_t)a.B, (uint64_t)a.q.st,
                    a.B > 1 ? (uint64_t)a.q.sb : (uint64_t)a.Lq * a.q.st, 64, 128, 1) ||
      !make_tmap_pages(&tkv, a.kv))
    return ONETRANS_ERR_CUDA;
  TcAttnArgs args;
  memset(&args, 0, sizeof(args));
  args.mode = MODE_CAUSAL;
  args.Lq = a.Lq;
  args.q_pos0 = a.q_pos0;
  args.q_pos0_u = a.q_pos0_u;
  args.o = a.o;
  args.kv = a.kv;
  args.H = a.H;
  dim3 grid((unsigned)((a.Lq + 127) / 128), (unsigned)a.H, (unsigned)a.B);
  return attn_launch_common(tq, tkv, tkv, args, a.dh, grid, st);
}

// Candidates per Stage II tile: whole candidates' NS rows fill at most 128 rows.
inline int stage2_cands_per_tile(int L_NS) { return L_NS <= 128 ? 128 / L_NS : 0; }

inline bool tc_stage2_supported(const Stage2Desc& a) {
  return (a.dh == 64 || a.dh == 96) && a.kv.dh == a.dh && stage2_cands_per_tile(a.L_NS) > 0 && tc_kv_ok(a.kv) && ((uintptr_t)a.qkv % 16) == 0 &&
         ((uintptr_t)a.o % 16) == 0;
}

inline onetrans_status tc_stage2_launch(const Stage2Desc& a, int n_tiles, cudaStream_t st) {
  CUtensorMap tq, tkv;
  const uint64_t d = (uint64_t)a.H * a.dh;
  const uint64_t rows = (uint64_t)a.C_tot * a.L_NS;
  // one map serves Q (columns h*64) and the own-NS K/V tile (columns d + h*64, 2d + h*64)
  if (!make_tmap_3d(&tq, a.qkv, 3 * d, rows, 1, 3 * d, rows * 3 * d, 64, 128, 1) || !make_tmap_pages(&tkv, a.kv))
    return ONETRANS_ERR_CUDA;
  TcAttnArgs args;
  memset(&args, 0, sizeof(args));
  args.mode = MODE_STAGE2;
  args.tiles = a.tiles;
  args.o2 = (__nv_bfloat16*)a.o;
  args.L_NS = a.L_NS;
  args.s_len = a.s_len;
  args.s_len_u = a.s_len_u;
  args.kv = a.kv;
  args.H = a.H;
  dim3 grid((unsigned)n_tiles, (unsigned)a.H, 1);
  return attn_launch_common(tq, tkv, tq, args, a.dh, grid, st);
}

}  // namespace ot
