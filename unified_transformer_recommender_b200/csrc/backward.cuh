// Kernels of the training path: the backward pass of the block stack with
// activation recomputation.  The contractions run on the GEMM kernels of
// the forward path and, for the weight gradients, on the row-major
// weight-gradient GEMM (tcgen05 where the shape allows); these kernels supply
// the rest: operand transposes for the GEMMs that the tensor-core kernels do
// not take (K-major, zero-padded to a multiple of 64 rows), column sums (bias
// and gain gradients, two passes in a fixed order), the RMSNorm and GELU
// backward steps (with the gain and shared-bias column sums folded in), and
// attention forward / backward on CUDA cores for head widths the tensor-core
// training attention does not take.
#pragma once
#include "tc_ptx.cuh"

namespace ot {

// Row r of group g of a gathered row set: src + g*gs + (r / T)*sb + (r % T)*st
// (T rows per sample, sample stride sb, row stride st).
struct RowSet {
  long long gs, sb, st;
  int T, R;  // rows per sample, rows in the set
};

__device__ inline long long rowset_off(const RowSet& s, int g, int r) {
  const int b = r / s.T, t = r - b * s.T;
  return (long long)g * s.gs + (long long)b * s.sb + (long long)t * s.st;
}

// Four consecutive elements as one vector access (16 bytes of float32, 8 of
// bf16; the caller keeps the address aligned to that).
template <typename T> __device__ inline void ld4(const T* p, float v[4]);
template <> __device__ inline void ld4<float>(const float* p, float v[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
template <> __device__ inline void ld4<__nv_bfloat16>(const __nv_bfloat16* p, float v[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
template <typename T> __device__ inline void st4(T* p, const float v[4]);
template <> __device__ inline void st4<float>(float* p, const float v[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <> __device__ inline void st4<__nv_bfloat16>(__nv_bfloat16* p, const float v[4]) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 q;
  q.x = *reinterpret_cast<const uint32_t*>(&a);
  q.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = q;
}


// The K-major operand of a GEMM that contracts over rows: row r of group g,
// column c goes to dst[g][r / Kc][c][r % Kc] (R_pad = chunks x Kc; 0 for
// R <= r < R_pad), so that each chunk of Kc rows is its own K-major matrix
// (Kc = R_pad: one chunk).  32 x 32 tiles through shared memory, so both the
// reads and the writes are coalesced.
// Any shape: 32 x 32 tiles, one element per thread and pass.
template <typename Ti, typename To>
__global__ void __launch_bounds__(256) transpose_rows_scalar_kernel(const Ti* __restrict__ src, RowSet s, int C,
                                                                    To* __restrict__ dst, int R_pad, int Kc) {
  __shared__ float tile[32][33];
  const int g = blockIdx.z, c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty + 8 * i, c = c0 + tx;
    tile[ty + 8 * i][tx] = (r < s.R && c < C) ? to_f(src[rowset_off(s, g, r) + c]) : 0.f;
  }
  __syncthreads();
  To* out = dst + (long long)g * C * R_pad;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = c0 + ty + 8 * i, r = r0 + tx;
    if (c < C && r < R_pad) {
      const int ch = r / Kc;
      out[(long long)ch * C * Kc + (long long)c * Kc + (r - ch * Kc)] = from_f<To>(tile[tx][ty + 8 * i]);
    }
  }
}

// 64 x 64 tiles, 256 threads: each thread reads 4 columns of 4 rows (one
// vector load per row, one row-offset computation per row) and writes 4 rows
// of the transposed tile, 4 consecutive elements each.  Needs C % 4 == 0, the
// row strides % 4 == 0, R_pad % 64 == 0 and Kc % 64 == 0 (the host checks).
template <typename Ti, typename To>
__global__ void __launch_bounds__(256) transpose_rows_kernel(const Ti* __restrict__ src, RowSet s, int C,
                                                             To* __restrict__ dst, int R_pad, int Kc) {
  __shared__ float tile[64][65];
  const int g = blockIdx.z, c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
  const int cq = (threadIdx.x & 15) * 4, rq = threadIdx.x >> 4;   // 16 column quads x 16 row lanes
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = rq + 16 * i, r = r0 + rr, c = c0 + cq;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < s.R && c < C) {
      const Ti* p = src + rowset_off(s, g, r) + c;
      if (sizeof(Ti) == 4) {
        const float4 f = *(const float4*)p;
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      } else {
        const uint2 u = *(const uint2*)p;
        const __nv_bfloat162* h = (const __nv_bfloat162*)&u;
        const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[rr][cq + j] = v[j];
  }
  __syncthreads();
  To* out = dst + (long long)g * C * R_pad;
  const int ch = r0 / Kc, rin = r0 - ch * Kc + cq;   // the 64 rows of a tile lie in one chunk
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int cc = rq + 16 * i, c = c0 + cc;
    if (c < C && r0 < R_pad) {
      To* q = out + (long long)ch * C * Kc + (long long)c * Kc + rin;
      if (sizeof(To) == 4) {
        *(float4*)q = make_float4(tile[cq][cc], tile[cq + 1][cc], tile[cq + 2][cc], tile[cq + 3][cc]);
      } else {
        uint2 u;
        __nv_bfloat162* h = (__nv_bfloat162*)&u;
        h[0] = __floats2bfloat162_rn(tile[cq][cc], tile[cq + 1][cc]);
        h[1] = __floats2bfloat162_rn(tile[cq + 2][cc], tile[cq + 3][cc]);
        *(uint2*)q = u;
      }
    }
  }
}

// out[(i / n_inner) * out_stride + i % n_inner] = sum over the chunks k of
// part[k * n + i], chunk by chunk in order.  Few chunks (the row slices of a
// weight gradient): one thread per four outputs, vector loads.  Many chunks
// (the per-CTA partial rows of a gain or bias gradient): 32 outputs per CTA,
// warp w adding chunks w, w + NW, ..., the NW warp sums then added in warp
// order.  Both orders are fixed: the result does not depend on timing.
__global__ void __launch_bounds__(256) chunk_sum4_kernel(const float* __restrict__ part, int chunks, long long n,
                                                         float* __restrict__ out, long long out_stride,
                                                         long long n_inner) {
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int k = 0; k < chunks; ++k) {
    float v[4];
    ld4<float>(part + (long long)k * n + i, v);
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] += v[j];
  }
  st4<float>(out + (i / n_inner) * out_stride + i % n_inner, acc);
}

template <int NW>
__global__ void __launch_bounds__(NW * 32) chunk_sum_kernel(const float* __restrict__ part, int chunks, long long n,
                                                            float* __restrict__ out, long long out_stride,
                                                            long long n_inner) {
  __shared__ float red[NW][33];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const long long i = (long long)blockIdx.x * 32 + lane;
  float acc = 0.f;
  if (i < n) {
#pragma unroll 4
    for (int k = w; k < chunks; k += NW) acc += part[(long long)k * n + i];
  }
  red[w][lane] = acc;
  __syncthreads();
  if (w == 0 && i < n) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < NW; ++q) t += red[q][lane];
    out[(i / n_inner) * out_stride + i % n_inner] = t;
  }
}

// Column sums in two passes with a fixed order: this kernel sums chunk
// blockIdx.z (kColChunk rows) of group g's rows into part[g][chunk][c], 32
// columns per CTA and 8 row lanes per column; chunk_sum_kernel adds the chunks.
constexpr int kColChunk = 256;
template <typename Ti>
__global__ void __launch_bounds__(256) colsum_kernel(const Ti* __restrict__ src, RowSet s, int C,
                                                     float* __restrict__ part) {
  __shared__ float red[8][33];
  const int g = blockIdx.y, ch = blockIdx.z, tx = threadIdx.x & 31, ty = threadIdx.x >> 5, c = blockIdx.x * 32 + tx;
  const int r_end = min(s.R, (ch + 1) * kColChunk);
  float acc = 0.f;
  if (c < C)
    for (int r = ch * kColChunk + ty; r < r_end; r += 8) acc += to_f(src[rowset_off(s, g, r) + c]);
  red[ty][tx] = acc;
  __syncthreads();
  if (ty == 0 && c < C) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) t += red[i][tx];
    part[((long long)ch * gridDim.y + g) * C + c] = t;
  }
}

// The same, four columns per thread (one vector load per row): 128 columns
// per CTA.  Needs C % 4 == 0, strides % 4 == 0 and a vector-aligned base.
template <typename Ti>
__global__ void __launch_bounds__(256) colsum4_kernel(const Ti* __restrict__ src, RowSet s, int C,
                                                      float* __restrict__ part) {
  __shared__ float red[8][129];
  const int g = blockIdx.y, ch = blockIdx.z, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * 128 + 4 * lane;
  const int r_end = min(s.R, (ch + 1) * kColChunk);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (c < C)
    for (int r = ch * kColChunk + w; r < r_end; r += 8) {
      float v[4];
      ld4<Ti>(src + rowset_off(s, g, r) + c, v);
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] += v[j];
    }
#pragma unroll
  for (int j = 0; j < 4; ++j) red[w][4 * lane + j] = acc[j];
  __syncthreads();
  const int cc = blockIdx.x * 128 + threadIdx.x;
  if (threadIdx.x < 128 && cc < C) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][threadIdx.x];
    part[((long long)ch * gridDim.y + g) * C + cc] = t;
  }
}

// RMSNorm backward for y = x r g, r = (mean(x^2) + eps)^(-1/2), one warp per
// row (rows (b, t) through x's and dx's sample and row strides, `fold` rows
// per sample):  dx += r g dy - x r^3 sum(g dy x) / d, and pg = dy x r, the
// row's share of dg (summed over rows by colsum_kernel).
template <typename Tx, typename T>
__global__ void __launch_bounds__(256) rms_backward_kernel(const Tx* __restrict__ x, long long x_sb, long long x_st,
                                                           const T* __restrict__ gamma, const float* __restrict__ dy,
                                                           float* __restrict__ dx, long long dx_sb, long long dx_st,
                                                           float* __restrict__ pg, int rows, int fold, int d, float eps,
                                                           T* __restrict__ dx_copy) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int b = row / fold, t = row - b * fold;
  const Tx* xr = x + b * x_sb + t * x_st;
  const float* dyr = dy + (long long)row * d;
  float ss = 0.f, sg = 0.f;
  for (int k = lane; k < d; k += 32) {
    const float xv = to_f(xr[k]), gy = to_f(gamma[k]) * dyr[k];
    ss = fmaf(xv, xv, ss);
    sg = fmaf(gy, xv, sg);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    sg += __shfl_xor_sync(0xffffffffu, sg, o);
  }
  const float r = rsqrtf(ss / d + eps);
  const float c3 = r * r * r * sg / d;
  float* dxr = dx + b * dx_sb + t * dx_st;
  T* cpr = dx_copy ? dx_copy + b * dx_sb + t * dx_st : nullptr;
  float* pgr = pg + (long long)row * d;
  for (int k = lane; k < d; k += 32) {
    const float xv = to_f(xr[k]), g = to_f(gamma[k]), dv = dyr[k];
    const float v = dxr[k] + (r * g * dv - xv * c3);
    dxr[k] = v;
    if (cpr) cpr[k] = from_f<T>(v);   // the finished row, as the next GEMM's operand
    pgr[k] = dv * xv * r;
  }
}

// The same with the gain gradient folded in: warp w of CTA k takes rows
// k*8 + w, then every (gridDim.x * 8)-th row after it; lane l the columns
// 4l .. 4l+3 of every 128 (d = 128 NC4), as vector accesses.  The CTA's sums
// of dy x r leave as one partial row part[k][d], the warps added in warp
// order (chunk_sum_kernel then adds the CTAs' rows in CTA order).  dx is
// written, not accumulated: the gradient that reaches x around the norm (the
// residual branch) is read from `res`, row t - r_off of the sample (0 for
// t < r_off or without res).  With part_s, the CTA also leaves the column
// sums of the finished dx rows with t < s_rows as part_s[k][d] (the shared
// b2 gradient of the layer below, whose output x is).  Needs the row strides
// % 4 == 0 and vector-aligned bases.
template <typename Tx, typename T, int NC4>
__global__ void __launch_bounds__(256) rms_backward_dg_kernel(const Tx* __restrict__ x, long long x_sb, long long x_st,
                                                              const T* __restrict__ gamma,
                                                              const float* __restrict__ dy,
                                                              const float* __restrict__ res, long long r_sb,
                                                              long long r_st, int r_off, float* __restrict__ dx,
                                                              long long dx_sb, long long dx_st, float* __restrict__ part,
                                                              int rows, int fold, float eps, T* __restrict__ dx_copy,
                                                              float* __restrict__ part_s, int s_rows) {
  constexpr int d = 128 * NC4;
  __shared__ float red[8][d];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float gm[NC4][4], pg[NC4][4], ps[NC4][4];
#pragma unroll
  for (int i = 0; i < NC4; ++i) {
    ld4<T>(gamma + 128 * i + 4 * lane, gm[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) pg[i][j] = ps[i][j] = 0.f;
  }
  for (int row = blockIdx.x * 8 + w; row < rows; row += gridDim.x * 8) {
    const int b = row / fold, t = row - b * fold;
    const Tx* xr = x + b * x_sb + t * x_st;
    const float* dyr = dy + (long long)row * d;
    float xv[NC4][4], dv[NC4][4];
    float ss = 0.f, sg = 0.f;
#pragma unroll
    for (int i = 0; i < NC4; ++i) {
      ld4<Tx>(xr + 128 * i + 4 * lane, xv[i]);
      ld4<float>(dyr + 128 * i + 4 * lane, dv[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ss = fmaf(xv[i][j], xv[i][j], ss);
        sg = fmaf(gm[i][j] * dv[i][j], xv[i][j], sg);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      sg += __shfl_xor_sync(0xffffffffu, sg, o);
    }
    const float r = rsqrtf(ss / d + eps);
    const float c3 = r * r * r * sg / d;
    float* dxr = dx + b * dx_sb + t * dx_st;
    T* cpr = dx_copy ? dx_copy + b * dx_sb + t * dx_st : nullptr;
    const float* rr = (res && t >= r_off) ? res + b * r_sb + (t - r_off) * r_st : nullptr;
    const bool s_row = t < s_rows;
#pragma unroll
    for (int i = 0; i < NC4; ++i) {
      float o[4] = {0.f, 0.f, 0.f, 0.f};
      if (rr) ld4<float>(rr + 128 * i + 4 * lane, o);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        o[j] += r * gm[i][j] * dv[i][j] - xv[i][j] * c3;
        pg[i][j] = fmaf(dv[i][j], xv[i][j] * r, pg[i][j]);
        if (s_row) ps[i][j] += o[j];
      }
      st4<float>(dxr + 128 * i + 4 * lane, o);
      if (cpr) st4<T>(cpr + 128 * i + 4 * lane, o);   // the finished row, as the next GEMM's operand
    }
  }
#pragma unroll
  for (int i = 0; i < NC4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[w][128 * i + 4 * lane + j] = pg[i][j];
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += 256) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][c];
    part[(long long)blockIdx.x * d + c] = t;
  }
  if (!part_s) return;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NC4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[w][128 * i + 4 * lane + j] = ps[i][j];
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += 256) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][c];
    part_s[(long long)blockIdx.x * d + c] = t;
  }
}


// du = dz * GELU'(u) and z = GELU(u), both in the storage type (du: the
// operand of the next GEMMs and the rows whose column sums are db1; z: the
// activation operand of dW2).  Four elements per thread; the buffers start
// 16-byte aligned, so every full group of four is a vector access.
template <typename T>
__global__ void __launch_bounds__(256) gelu_backward_kernel(const float* __restrict__ dz, const T* __restrict__ u,
                                                            T* __restrict__ du, T* __restrict__ z, long long n) {
  const long long i0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i0 >= n) return;
  if (i0 + 4 <= n) {
    float uv[4], dv[4], zv[4], gv[4];
    ld4<T>(u + i0, uv);
    ld4<float>(dz + i0, dv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      gelu_tanh_and_grad(uv[k], zv[k], gv[k]);
      gv[k] *= dv[k];
    }
    st4<T>(du + i0, gv);
    st4<T>(z + i0, zv);
  } else {
    for (long long i = i0; i < n; ++i) {
      float zz, g;
      gelu_tanh_and_grad(to_f(u[i]), zz, g);
      du[i] = from_f<T>(dz[i] * g);
      z[i] = from_f<T>(zz);
    }
  }
}

// The same over whole rows of dff columns with the column sums of du over
// the S rows folded in (the gradient of the shared set's b1): CTA k takes
// rows [k*rows_per, (k+1)*rows_per) of the B x Lq rows (row t of a sample is
// an S row for t < sq), thread i the columns 4i .. 4i+3 of every 1024
// (dff <= 1024 J, dff % 4 == 0); the sums (of du before its rounding to the
// storage type) leave as part[k][dff].
template <typename T, int J>
__global__ void __launch_bounds__(256) gelu_backward_bias_kernel(const float* __restrict__ dz,
                                                                 const T* __restrict__ u, T* __restrict__ du,
                                                                 T* __restrict__ z, int rows, int Lq, int sq, int dff,
                                                                 int rows_per, float* __restrict__ part) {
  float acc[J][4];
#pragma unroll
  for (int j = 0; j < J; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
  const int r0 = blockIdx.x * rows_per, r1 = min(rows, r0 + rows_per);
#pragma unroll 2
  for (int r = r0; r < r1; ++r) {
    const bool s_row = (r % Lq) < sq;
    const long long base = (long long)r * dff;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int c = 1024 * j + 4 * threadIdx.x;
      if (c < dff) {
        float uv[4], dv[4], zv[4], gv[4];
        ld4<T>(u + base + c, uv);
        ld4<float>(dz + base + c, dv);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          gelu_tanh_and_grad(uv[q], zv[q], gv[q]);
          gv[q] *= dv[q];
          if (s_row) acc[j][q] += gv[q];
        }
        st4<T>(du + base + c, gv);
        st4<T>(z + base + c, zv);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int c = 1024 * j + 4 * threadIdx.x;
    if (c < dff) st4<float>(part + (long long)blockIdx.x * dff + c, acc[j]);
  }
}

template <typename T>
__global__ void cast_kernel(const float* __restrict__ src, T* __restrict__ dst, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = from_f<T>(src[i]);
}

// ------------------------------------------------ attention on plain rows --
// qkv [B, L, 3d] (q | k | v of every row, q unscaled); the Lq queries are the
// tail rows L - Lq .. L - 1, query t at key position L - Lq + t sees keys
// 0 .. that position.  One thread per (query or key, head), 64 per CTA.
struct AttnRows {
  const void* qkv;
  int B, L, Lq, H, d;
};

__device__ inline long long qkv_off(const AttnRows& a, int b, int row, int part, int h, int dh) {
  return ((long long)b * a.L + row) * 3 * a.d + (long long)part * a.d + (long long)h * dh;
}

// a = softmax(q k^T / sqrt(d_h)) v over the visible keys, and the row's
// log-sum-exp (natural units) for the backward.
template <typename T, int DH>
__global__ void __launch_bounds__(64) attn_rows_forward_kernel(AttnRows a, T* __restrict__ out, float* __restrict__ lse) {
  const int t = blockIdx.x * 64 + threadIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (t >= a.Lq) return;
  const T* qkv = (const T*)a.qkv;
  const int p = a.L - a.Lq + t;
  const float sc = rsqrtf((float)DH) * 1.4426950408889634f;   // base-2 logits
  float q[DH], o[DH];
  const T* qr = qkv + qkv_off(a, b, p, 0, h, DH);
#pragma unroll
  for (int e = 0; e < DH; ++e) { q[e] = to_f(qr[e]) * sc; o[e] = 0.f; }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j <= p; ++j) {
    const T* kr = qkv + qkv_off(a, b, j, 1, h, DH);
    const T* vr = qkv + qkv_off(a, b, j, 2, h, DH);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) s = fmaf(q[e], to_f(kr[e]), s);
    if (s > m) {
      const float c = exp2f(m - s);
      l *= c;
#pragma unroll
      for (int e = 0; e < DH; ++e) o[e] *= c;
      m = s;
    }
    const float w = exp2f(s - m);
    l += w;
#pragma unroll
    for (int e = 0; e < DH; ++e) o[e] = fmaf(w, to_f(vr[e]), o[e]);
  }
  T* orow = out + ((long long)b * a.Lq + t) * a.d + (long long)h * DH;
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < DH; ++e) orow[e] = from_f<T>(o[e] * inv);
  lse[((long long)b * a.H + h) * a.Lq + t] = (m + log2f(l)) * 0.6931471805599453f;
}

// Per query row: D = dO . O, then dQ = sum_j P_j (dO . v_j - D) k_j / sqrt(d_h)
// with P_j = exp(q . k_j / sqrt(d_h) - lse).  dO in the storage type; dq goes
// to dqkv's q columns in the storage type (the operand of the next GEMMs).
template <typename T, int DH>
__global__ void __launch_bounds__(64) attn_rows_dq_kernel(AttnRows a, const T* __restrict__ dout,
                                                          const T* __restrict__ out, const float* __restrict__ lse,
                                                          float* __restrict__ Dr, T* __restrict__ dqkv) {
  const int t = blockIdx.x * 64 + threadIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (t >= a.Lq) return;
  const T* qkv = (const T*)a.qkv;
  const int p = a.L - a.Lq + t;
  const float isq = rsqrtf((float)DH);
  const long long ro = ((long long)b * a.Lq + t) * a.d + (long long)h * DH;
  float q[DH], g[DH], dq[DH];
  float D = 0.f;
  const T* qr = qkv + qkv_off(a, b, p, 0, h, DH);
#pragma unroll
  for (int e = 0; e < DH; ++e) {
    q[e] = to_f(qr[e]) * isq;
    g[e] = to_f(dout[ro + e]);
    D = fmaf(g[e], to_f(out[ro + e]), D);
    dq[e] = 0.f;
  }
  const long long si = ((long long)b * a.H + h) * a.Lq + t;
  const float ls = lse[si];
  Dr[si] = D;
  for (int j = 0; j <= p; ++j) {
    const T* kr = qkv + qkv_off(a, b, j, 1, h, DH);
    const T* vr = qkv + qkv_off(a, b, j, 2, h, DH);
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) {
      s = fmaf(q[e], to_f(kr[e]), s);
      dp = fmaf(g[e], to_f(vr[e]), dp);
    }
    const float ds = __expf(s - ls) * (dp - D) * isq;
#pragma unroll
    for (int e = 0; e < DH; ++e) dq[e] = fmaf(ds, to_f(kr[e]), dq[e]);
  }
  T* dst = dqkv + ((long long)b * a.L + p) * 3 * a.d + (long long)h * DH;
#pragma unroll
  for (int e = 0; e < DH; ++e) dst[e] = from_f<T>(dq[e]);
}

// Per key row j: dV = sum_t P_tj dO_t, dK = sum_t P_tj (dO_t . v_j - D_t) q_t / sqrt(d_h)
// over the queries t that see key j.  dk, dv go to dqkv's k and v columns.
template <typename T, int DH>
__global__ void __launch_bounds__(64) attn_rows_dkdv_kernel(AttnRows a, const T* __restrict__ dout,
                                                            const float* __restrict__ lse, const float* __restrict__ Dr,
                                                            T* __restrict__ dqkv) {
  const int j = blockIdx.x * 64 + threadIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (j >= a.L) return;
  const T* qkv = (const T*)a.qkv;
  const float isq = rsqrtf((float)DH);
  float k[DH], v[DH], dk[DH], dv[DH];
  const T* kr = qkv + qkv_off(a, b, j, 1, h, DH);
  const T* vr = qkv + qkv_off(a, b, j, 2, h, DH);
#pragma unroll
  for (int e = 0; e < DH; ++e) {
    k[e] = to_f(kr[e]) * isq;
    v[e] = to_f(vr[e]);
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  const int q0 = a.L - a.Lq;
  for (int t = max(0, j - q0); t < a.Lq; ++t) {
    const T* qr = qkv + qkv_off(a, b, q0 + t, 0, h, DH);
    const T* gr = dout + ((long long)b * a.Lq + t) * a.d + (long long)h * DH;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) {
      s = fmaf(to_f(qr[e]), k[e], s);
      dp = fmaf(to_f(gr[e]), v[e], dp);
    }
    const long long si = ((long long)b * a.H + h) * a.Lq + t;
    const float pr = __expf(s - lse[si]);
    const float ds = pr * (dp - Dr[si]) * isq;
#pragma unroll
    for (int e = 0; e < DH; ++e) {
      dv[e] = fmaf(pr, to_f(gr[e]), dv[e]);
      dk[e] = fmaf(ds, to_f(qr[e]), dk[e]);
    }
  }
  T* dst = dqkv + ((long long)b * a.L + j) * 3 * a.d + (long long)h * DH;
#pragma unroll
  for (int e = 0; e < DH; ++e) {
    dst[a.d + e] = from_f<T>(dk[e]);
    dst[2 * a.d + e] = from_f<T>(dv[e]);
  }
}

}  // namespace ot
