// CUDA-core kernels: the float32 mode's whole path, and the fallback for
// shapes the tensor-core kernels do not take.  Same descriptors and memory
// layouts as the tensor-core path.
#pragma once
#include "common.cuh"

namespace ot {

// ------------------------------------------------------------------ GEMM --
// C[(b,t), n] = epilogue( sum_k A[(m,g), k] * W[grp][n_lo + n][k] )
// 64x64 output tile per CTA, 256 threads, 4x4 outputs per thread.
template <typename T>
__device__ inline void epilogue_store(const GemmDesc& d, int b, int t, int n, int grp, float v) {
  if (d.bias) v += to_f(((const T*)d.bias)[grp * d.bias_sg + d.n_lo + n]);
  if (d.act == ACT_GELU) v = gelu_tanh(v);
  if (d.res.base) v += rm_load<T>(d.res, rm_off(d.res, b, t, n));
  if (n < d.scale_cols) v *= d.col_scale;
  if (d.out_kind == OUT_KV) {
    const int dm = d.kv.H * d.kv.dh;
    const int kind = n / dm, c = n - kind * dm, head = c / d.kv.dh, e = c - head * d.kv.dh;
    ((T*)d.kv.pool)[kv_off(d.kv, b, t + (d.kv.pos_off_u ? d.kv.pos_off_u[b] : d.kv.pos_off), kind, head, e)] =
        from_f<T>(v);
  } else {
    rm_store<T>(d.out, rm_off(d.out, b, t, n), v);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc d) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int n0 = blockIdx.x * 64, m0 = d.m_lo + blockIdx.y * 64, g = d.g_lo + blockIdx.z;
  const int m_end = d.m_lo + d.M;
  const int grp = d.mode == TILE_SAMPLES ? g - d.grp_base : 0;
  const T* A = (const T*)d.A;
  const T* W = (const T*)d.W + (long long)grp * d.w_sg + (long long)d.n_lo * d.K;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d.K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i >> 4, kk = i & 15, k = k0 + kk;
      const int m = m0 + r, n = n0 + r;
      As[kk][r] = (m < m_end && k < d.K) ? to_f(A[(long long)m * d.a_sm + (long long)g * d.a_sg + k]) : 0.f;
      Bs[kk][r] = (n < d.N && k < d.K) ? to_f(W[(long long)n * d.K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; w[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= m_end) continue;
    int b, t;
    row_of(d, m, g, b, t);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < d.N) epilogue_store<T>(d, b, t, n, grp, acc[i][j]);
    }
  }
}

// -------------------------------------------------------------- RMSNorm --
// For every row the descriptor enumerates: dst = src * rsqrt(mean(src^2) + eps) * gamma
// over N columns; src = d.out, dst = d.rms.  One warp per row.
template <typename T>
__global__ void rms_rows_kernel(GemmDesc d) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = d.m_lo + blockIdx.x * (blockDim.x >> 5) + warp;
  const int g = d.g_lo + blockIdx.y;
  if (m >= d.m_lo + d.M) return;
  int b, t;
  row_of(d, m, g, b, t);
  float ss = 0.f;
  for (int n = lane; n < d.N; n += 32) {
    const float v = rm_load<T>(d.out, rm_off(d.out, b, t, n));
    ss += v * v;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / d.N + d.eps);
  const T* gm = (const T*)d.gamma;
  for (int n = lane; n < d.N; n += 32) {
    const float v = rm_load<T>(d.out, rm_off(d.out, b, t, n));
    rm_store<T>(d.rms, rm_off(d.rms, b, t, n), v * r * to_f(gm[n]));
  }
}

// RMSNorm of contiguous rows of D = 128 CH elements: dst = src * (mean(src^2)
// + eps)^-1/2 * gamma.  One warp per row, the row held in registers; each
// warp-wide access covers 128 consecutive elements (lane l: elements 4l ..
// 4l+3 of the chunk), so every byte is read and written once, coalesced.
template <typename T>
__device__ inline void load4(const T* p, float* v);
template <>
__device__ inline void load4<float>(const float* p, float* v) {
  const float4 f = *(const float4*)p;
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
template <>
__device__ inline void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
  const uint2 u = *(const uint2*)p;
  const float2 a = __bfloat1622float2(*(const __nv_bfloat162*)&u.x), b = __bfloat1622float2(*(const __nv_bfloat162*)&u.y);
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
template <typename T>
__device__ inline void store4(T* p, const float* v);
template <>
__device__ inline void store4<float>(float* p, const float* v) {
  *(float4*)p = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ inline void store4<__nv_bfloat16>(__nv_bfloat16* p, const float* v) {
  uint2 u;
  *(__nv_bfloat162*)&u.x = __floats2bfloat162_rn(v[0], v[1]);
  *(__nv_bfloat162*)&u.y = __floats2bfloat162_rn(v[2], v[3]);
  *(uint2*)p = u;
}
template <typename T, typename S, int CH>
__global__ void __launch_bounds__(256) rms_flat_kernel(const S* __restrict__ src, T* __restrict__ dst,
                                                       const T* __restrict__ gamma, long long rows, float eps) {
  constexpr int D = CH * 128;
  grid_dep_wait();
  grid_dep_launch();
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const S* x = src + row * D + lane * 4;
  float v[CH][4];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    load4<S>(x + c * 128, v[c]);
#pragma unroll
    for (int i = 0; i < 4; ++i) ss = fmaf(v[c][i], v[c][i], ss);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / D + eps);
  T* y = dst + row * D + lane * 4;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    float gv[4];
    load4<T>(gamma + c * 128 + lane * 4, gv);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[c][i] *= r * gv[i];
    store4<T>(y + c * 128, v[c]);
  }
}

// ------------------------------------------------------ causal attention --
constexpr int KT = 32;  // keys staged in shared memory per step
// Query t of batch b (key position p = q_pos0 + t) attends to keys 0..p of
// its K/V store.  One thread per query, 64 queries per CTA, keys staged in
// shared memory KT at a time, online softmax in base 2.
template <typename T, int DH>
__global__ void __launch_bounds__(64) attn_simt_kernel(AttnDesc a) {
  __shared__ float Ks[KT][DH + 1];
  __shared__ float Vs[KT][DH + 1];
  __shared__ float Ss[KT][65];
  const int tid = threadIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t = blockIdx.x * 64 + tid;
  const bool valid = t < a.Lq;
  const int q_pos0 = a.q_pos0_u ? a.q_pos0_u[b] : a.q_pos0;
  const int p = q_pos0 + t;
  const int t_last = min(a.Lq, (int)(blockIdx.x + 1) * 64) - 1;
  const int kmax = q_pos0 + t_last;
  float q[DH], o[DH];
  const T* qp = (const T*)a.q.base + rm_off(a.q, b, valid ? t : 0, h * DH);
#pragma unroll
  for (int e = 0; e < DH; ++e) { q[e] = valid ? to_f(qp[e]) : 0.f; o[e] = 0.f; }
  float mrow = -INFINITY, lrow = 0.f;
  const T* pool = (const T*)a.kv.pool;
  for (int k0 = 0; k0 <= kmax; k0 += KT) {
    __syncthreads();
    for (int i = tid; i < KT * DH; i += 64) {
      const int r = i / DH, e = i - r * DH, pos = k0 + r;
      float kv = 0.f, vv = 0.f;
      if (pos <= kmax) {
        kv = to_f(pool[kv_off(a.kv, b, pos, 0, h, e)]);
        vv = to_f(pool[kv_off(a.kv, b, pos, 1, h, e)]);
      }
      Ks[r][e] = kv;
      Vs[r][e] = vv;
    }
    __syncthreads();
    float mt = -INFINITY;
    for (int r = 0; r < KT; ++r) {
      float s = -INFINITY;
      if (valid && k0 + r <= p) {
        s = 0.f;
#pragma unroll
        for (int e = 0; e < DH; ++e) s = fmaf(q[e], Ks[r][e], s);
      }
      Ss[r][tid] = s;
      mt = fmaxf(mt, s);
    }
    if (!valid || mt == -INFINITY) continue;
    const float mn = fmaxf(mrow, mt);
    const float c = exp2f(mrow - mn);
    lrow *= c;
#pragma unroll
    for (int e = 0; e < DH; ++e) o[e] *= c;
    for (int r = 0; r < KT; ++r) {
      const float pr = exp2f(Ss[r][tid] - mn);
      lrow += pr;
#pragma unroll
      for (int e = 0; e < DH; ++e) o[e] = fmaf(pr, Vs[r][e], o[e]);
    }
    mrow = mn;
  }
  if (!valid) return;
  T* op = (T*)a.o.base + rm_off(a.o, b, t, h * DH);
  const float inv = 1.f / lrow;
#pragma unroll
  for (int e = 0; e < DH; ++e) op[e] = from_f<T>(o[e] * inv);
}

// ---------------------------------------------------- Stage II attention --
// NS token j of candidate c (one thread each, all candidates of the CTA from
// one user) attends in one softmax to the user's s_len cached S keys and to
// its own NS keys 0..j.
template <typename T, int DH>
__global__ void __launch_bounds__(64) stage2_attn_simt_kernel(Stage2Desc a) {
  __shared__ float Ks[KT][DH + 1];
  __shared__ float Vs[KT][DH + 1];
  __shared__ float Ss[KT][65];
  const int tid = threadIdx.x, h = blockIdx.y, j = blockIdx.z;
  const int user = a.tiles[blockIdx.x * 3 + 0];
  const int c = a.tiles[blockIdx.x * 3 + 1] + tid;
  const bool valid = c < a.tiles[blockIdx.x * 3 + 2];
  const int s_len = a.s_len_u ? a.s_len_u[user] : a.s_len;
  const int d = a.H * DH;
  const long long rs = 3LL * d;  // row stride of the packed Q|K|V rows
  const T* qkv = (const T*)a.qkv;
  float q[DH], o[DH];
  const T* qp = qkv + ((long long)(valid ? c : 0) * a.L_NS + j) * rs + h * DH;
#pragma unroll
  for (int e = 0; e < DH; ++e) { q[e] = valid ? to_f(qp[e]) : 0.f; o[e] = 0.f; }
  float mrow = -INFINITY, lrow = 0.f;
  const T* pool = (const T*)a.kv.pool;
  for (int k0 = 0; k0 < s_len; k0 += KT) {
    __syncthreads();
    for (int i = tid; i < KT * DH; i += 64) {
      const int r = i / DH, e = i - r * DH, pos = k0 + r;
      float kv = 0.f, vv = 0.f;
      if (pos < s_len) {
        kv = to_f(pool[kv_off(a.kv, user, pos, 0, h, e)]);
        vv = to_f(pool[kv_off(a.kv, user, pos, 1, h, e)]);
      }
      Ks[r][e] = kv;
      Vs[r][e] = vv;
    }
    __syncthreads();
    float mt = -INFINITY;
    for (int r = 0; r < KT; ++r) {
      float s = -INFINITY;
      if (k0 + r < s_len) {
        s = 0.f;
#pragma unroll
        for (int e = 0; e < DH; ++e) s = fmaf(q[e], Ks[r][e], s);
      }
      Ss[r][tid] = s;
      mt = fmaxf(mt, s);
    }
    const float mn = fmaxf(mrow, mt);
    if (mn == -INFINITY) continue;
    const float cf = exp2f(mrow - mn);
    lrow *= cf;
#pragma unroll
    for (int e = 0; e < DH; ++e) o[e] *= cf;
    for (int r = 0; r < KT; ++r) {
      const float pr = exp2f(Ss[r][tid] - mn);
      lrow += pr;
#pragma unroll
      for (int e = 0; e < DH; ++e) o[e] = fmaf(pr, Vs[r][e], o[e]);
    }
    mrow = mn;
  }
  if (!valid) return;
  // own NS keys 0..j of this candidate
  for (int i = 0; i <= j; ++i) {
    const T* kp = qkv + ((long long)c * a.L_NS + i) * rs + d + h * DH;
    const T* vp = kp + d;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) s = fmaf(q[e], to_f(kp[e]), s);
    const float mn = fmaxf(mrow, s);
    const float cf = exp2f(mrow - mn), pr = exp2f(s - mn);
    lrow = lrow * cf + pr;
#pragma unroll
    for (int e = 0; e < DH; ++e) o[e] = fmaf(pr, to_f(vp[e]), o[e] * cf);
    mrow = mn;
  }
  T* op = (T*)a.o + ((long long)c * a.L_NS + j) * d + h * DH;
  const float inv = 1.f / lrow;
#pragma unroll
  for (int e = 0; e < DH; ++e) op[e] = from_f<T>(o[e] * inv);
}

// ------------------------------------------------------ event tokenizer --
// out(b, t) = W2[ty] gelu(W1[ty] e + b1[ty]) + b2[ty] + type_emb[ty] for each
// appended event; one CTA per event, one thread per output feature.
struct EventMLP {
  const void* W1[8];
  const void* b1[8];
  const void* W2[8];
  const void* b2[8];
  const void* emb;  // [n_types, d] additive type identifiers, or null for none
  int n_types, e_dim, d;
};

// Intent-order layout of a user's behavior sequences: sequence i holds the
// flat input rows [end[i-1], end[i]) (end[-1] = 0), all of behavior type[i];
// its tokens land at output rows shifted by i, so that output row end[i] + i
// is left for the [SEP] vector after sequence i.  n = 0: no layout (per-row
// types from the device array, output row = input row).
constexpr int kMaxIntents = 8;
struct IntentLayout {
  int n;
  int end[kMaxIntents];
  int type[kMaxIntents];
  const void* sep;  // [d], written at the n - 1 gap rows
};

__device__ __forceinline__ int intent_seq_of(const IntentLayout& lay, int row) {
  int s = 0;
#pragma unroll
  for (int i = 0; i < kMaxIntents - 1; ++i) s += (i < lay.n - 1 && lay.end[i] <= row) ? 1 : 0;
  return s;
}

__device__ __forceinline__ int intent_type_of(const IntentLayout& lay, int s) {
  int ty = lay.type[0];
#pragma unroll
  for (int i = 1; i < kMaxIntents; ++i) ty = (i == s) ? lay.type[i] : ty;
  return ty;
}

// The [SEP] rows of a layout: one CTA, thread k writes column k of each.
template <typename T>
__device__ __forceinline__ void intent_write_seps(const IntentLayout& lay, int d, int dL, const RowMap& out) {
#pragma unroll
  for (int i = 0; i < kMaxIntents - 1; ++i) {
    if (i + 1 >= lay.n) break;
    const int orow = lay.end[i] + i, bb = orow / dL, tt = orow - bb * dL;
    for (int k = threadIdx.x; k < d; k += blockDim.x)
      rm_store<T>(out, rm_off(out, bb, tt, k), to_f(((const T*)lay.sep)[k]));
  }
}

template <typename T>
__global__ void event_tokenize_kernel(const T* ev, const int* types, int dL, EventMLP w, RowMap out,
                                      IntentLayout lay) {
  extern __shared__ float sm[];
  float* e = sm;              // [e_dim]
  float* hid = sm + w.e_dim;  // [d]
  if (lay.n > 1 && blockIdx.x == gridDim.x - 1) {  // the extra block of a layout: its [SEP] rows
    intent_write_seps<T>(lay, w.d, dL, out);
    return;
  }
  const int row = blockIdx.x;
  const int seq = lay.n ? intent_seq_of(lay, row) : 0;
  const int orow = row + seq, b = orow / dL, t = orow - b * dL;
  int ty = lay.n ? intent_type_of(lay, seq) : types[row];
  if (ty < 0 || ty >= w.n_types) {
    if (threadIdx.x == 0) flag_error(3);
    ty = 0;
  }
  for (int i = threadIdx.x; i < w.e_dim; i += blockDim.x) e[i] = to_f(ev[(long long)row * w.e_dim + i]);
  __syncthreads();
  const T* W1 = (const T*)w.W1[ty];
  const T* W2 = (const T*)w.W2[ty];
  for (int k = threadIdx.x; k < w.d; k += blockDim.x) {
    float s = to_f(((const T*)w.b1[ty])[k]);
    for (int i = 0; i < w.e_dim; ++i) s = fmaf(to_f(W1[(long long)k * w.e_dim + i]), e[i], s);
    hid[k] = gelu_tanh(s);
  }
  __syncthreads();
  for (int k = threadIdx.x; k < w.d; k += blockDim.x) {
    float s = to_f(((const T*)w.b2[ty])[k]);
    for (int i = 0; i < w.d; ++i) s = fmaf(to_f(W2[(long long)k * w.d + i]), hid[i], s);
    if (w.emb) s += to_f(((const T*)w.emb)[(long long)ty * w.d + k]);
    rm_store<T>(out, rm_off(out, b, t, k), s);
  }
}

// The same tokenizer for d = 256 and e_dim <= 96, 32 events per CTA: the
// events' inputs and hidden rows sit in shared memory, each thread owns one
// output column and streams its weight row once per type while updating the
// 32 events' accumulators from broadcast shared-memory reads.  Every type's
// MLP is evaluated for every event of the CTA and the event keeps its own
// type's result (n_types is small), so there is no data-dependent control flow.
constexpr int kEvBlock = 32, kEvD = 256, kEvEmax = 96;
// 8 consecutive weights (16-byte aligned) as fp32
__device__ inline void load8(const __nv_bfloat16* p, float* v) {
  const uint4 u = *(const uint4*)p;
  const __nv_bfloat162* h = (const __nv_bfloat162*)&u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ inline void load8(const float* p, float* v) {
  const float4 a = *(const float4*)p, b = *(const float4*)(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// acc[j] += sum_{i < 8} wv[i] * x[j][i0 + i] over the CTA's events
template <int LD>
__device__ inline void ev_fma8(float* acc, const float* wv, const float (*x)[LD], int i0) {
#pragma unroll
  for (int j = 0; j < kEvBlock; ++j) {
    const float4 a = *(const float4*)&x[j][i0], b = *(const float4*)&x[j][i0 + 4];
    float s = acc[j];
    s = fmaf(wv[0], a.x, s); s = fmaf(wv[1], a.y, s); s = fmaf(wv[2], a.z, s); s = fmaf(wv[3], a.w, s);
    s = fmaf(wv[4], b.x, s); s = fmaf(wv[5], b.y, s); s = fmaf(wv[6], b.z, s); s = fmaf(wv[7], b.w, s);
    acc[j] = s;
  }
}
template <typename T>
__global__ void __launch_bounds__(256) event_tokenize_tile_kernel(const T* ev, const int* types, int R, int dL,
                                                                  EventMLP w, RowMap out, IntentLayout lay) {
  __shared__ __align__(16) float se[kEvBlock][kEvEmax];
  __shared__ __align__(16) float shid[kEvBlock][kEvD];
  __shared__ int sty[kEvBlock];
  __shared__ int sseq[kEvBlock];
  grid_dep_wait();
  grid_dep_launch();
  if (lay.n > 1 && blockIdx.x == gridDim.x - 1) {  // the extra CTA of a layout: its [SEP] rows
    intent_write_seps<T>(lay, kEvD, dL, out);
    return;
  }
  const int r0 = blockIdx.x * kEvBlock;
  const int k = threadIdx.x;
  for (int idx = threadIdx.x; idx < kEvBlock * w.e_dim; idx += blockDim.x) {
    const int j = idx / w.e_dim, i = idx - j * w.e_dim;
    se[j][i] = (r0 + j < R) ? to_f(ev[(long long)(r0 + j) * w.e_dim + i]) : 0.f;
  }
  if (threadIdx.x < kEvBlock) {
    const int row = r0 + threadIdx.x;
    const int seq = (lay.n && row < R) ? intent_seq_of(lay, row) : 0;
    int ty = row < R ? (lay.n ? intent_type_of(lay, seq) : types[row]) : 0;
    if (ty < 0 || ty >= w.n_types) {
      flag_error(3);
      ty = 0;
    }
    sty[threadIdx.x] = ty;
    sseq[threadIdx.x] = seq;
  }
  __syncthreads();
  float acc[kEvBlock];
  for (int t = 0; t < w.n_types; ++t) {
    const T* W1r = (const T*)w.W1[t] + (long long)k * w.e_dim;
    const float b = to_f(((const T*)w.b1[t])[k]);
#pragma unroll
    for (int j = 0; j < kEvBlock; ++j) acc[j] = b;
    for (int i0 = 0; i0 < w.e_dim; i0 += 8) {
      float wv[8];
      load8(W1r + i0, wv);
      ev_fma8<kEvEmax>(acc, wv, se, i0);
    }
#pragma unroll
    for (int j = 0; j < kEvBlock; ++j)
      if (sty[j] == t) shid[j][k] = gelu_tanh(acc[j]);
  }
  __syncthreads();
  for (int t = 0; t < w.n_types; ++t) {
    const T* W2r = (const T*)w.W2[t] + (long long)k * kEvD;
    const float b = to_f(((const T*)w.b2[t])[k]) + (w.emb ? to_f(((const T*)w.emb)[(long long)t * kEvD + k]) : 0.f);
#pragma unroll
    for (int j = 0; j < kEvBlock; ++j) acc[j] = b;
    for (int i0 = 0; i0 < kEvD; i0 += 8) {
      float wv[8];
      load8(W2r + i0, wv);
      ev_fma8<kEvD>(acc, wv, shid, i0);
    }
#pragma unroll
    for (int j = 0; j < kEvBlock; ++j) {
      const int row = r0 + j;
      if (sty[j] == t && row < R) {
        const int orow = row + sseq[j], bb = orow / dL, tt = orow - bb * dL;
        rm_store<T>(out, rm_off(out, bb, tt, k), acc[j]);
      }
    }
  }
}

}  // namespace ot

namespace ot {

// ------------------------------------------------------------ scoring head --
// logit[c] = w . vec(h[c]) + b over the n = L_NS * d float32 entries of
// candidate c's final NS rows (token-major, as the stack writes them).  One
// warp per candidate, 16-byte loads of h, fp32 accumulation, a shuffle
// reduction.  HBM-bound: n * 4 bytes read per candidate (the rows were just
// written by the last layer, so mostly from L2).
template <typename T>
__global__ void __launch_bounds__(256) head_logits_kernel(const float* __restrict__ h, const T* __restrict__ w,
                                                          const T* __restrict__ b, int n, long long C,
                                                          float* __restrict__ logits) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const long long c = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (c >= C) return;
  const float4* hr = (const float4*)(h + c * (long long)n);
  float acc = 0.f;
  for (int i = lane; i < n / 4; i += 32) {
    const float4 x = hr[i];
    acc = fmaf(x.x, to_f(w[4 * i + 0]), acc);
    acc = fmaf(x.y, to_f(w[4 * i + 1]), acc);
    acc = fmaf(x.z, to_f(w[4 * i + 2]), acc);
    acc = fmaf(x.w, to_f(w[4 * i + 3]), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) logits[c] = acc + to_f(b[0]);
}

}  // namespace ot
