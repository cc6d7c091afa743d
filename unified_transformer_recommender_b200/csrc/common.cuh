// Shared descriptors of the OneTrans CUDA library (host and device).
//
// Every activation row of the block stack is identified by (b, t): b is the
// batch index (sample, user or candidate) and t the row within it.  A GEMM
// tiles one of the two coordinates by 128 rows and fixes the other per CTA:
//   TILE_ROWS    tiled m = t, fixed g = b      (S rows of one sample/user)
//   TILE_SAMPLES tiled m = b, fixed g = t      (one NS token across samples;
//                                               weight group = t - grp_base)
//   TILE_FLAT    tiled m = b * fold + t        (rows contiguous across users)
#pragma once
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace ot {

enum TileMode : int { TILE_ROWS = 0, TILE_SAMPLES = 1, TILE_FLAT = 2 };
enum OutKind : int { OUT_ROWS = 0, OUT_KV = 1 };
// ACT_GELU_BWD (the FFN backward): the product is dz, the gradient of
// GELU's output; the epilogue reads the pre-activation u (act_in), stores
// du = dz * GELU'(u) as the output and GELU(u) through act_out.
enum Act : int { ACT_NONE = 0, ACT_GELU = 1, ACT_GELU_BWD = 2 };

// Address of element (b, t, n) = base + b*sb + t*st + (n / split)*sc + n % split
// (in elements).  `split` lets one GEMM write column blocks to separate
// planes (the token-major output of the auto-split tokenizer).  `f32` marks
// a float32 tensor (the residual stream and the stack's outputs); otherwise
// the element type is the model's storage type.
struct RowMap {
  void* base;
  long long sb, st, sc;
  int split;
  int f32;
};

// Paged K/V store.  A page holds P tokens of one (sequence, layer) laid out as
// [kind 0=K,1=V][head][token][d_h].  The page of token `pos` of batch row b is
//   table ? table[row_off[b] + pos / P] : b * pps + pos / P.
struct KVStore {
  void* pool;
  const int* table;
  const int* row_off;
  int P, H, dh, pps;
  int pos_off;  // written position = t + pos_off
  const int* pos_off_u;  // or, when set (device, per batch b): t + pos_off_u[b]
  int n_pages;  // pages in the pool (extent of the page dimension)
};

struct GemmDesc {
  int mode, M, m_lo, G, g_lo, fold;
  int N, K, n_lo, grp_base;
  // A element (m, g, k) = A + m*a_sm + g*a_sg + k; extents for the TMA map
  const void* A;
  long long a_sm, a_sg, a_mext, a_gext;
  // W element (grp, n, k) = W + grp*w_sg + (n_lo + n)*K + k, or with w_mn set
  // (a weight stored [K][w_rows], as dX = dY W reads the forward's W)
  // W + grp*w_sg + k*w_rows + n_lo + n
  const void* W;
  long long w_sg;
  int w_rows, w_groups;
  int w_mn;
  const void* bias;  // bias[grp*bias_sg + n_lo + n], or null
  long long bias_sg;
  int act;
  int out_kind;
  RowMap out;
  RowMap res;    // residual added after bias/activation (base null = none)
  RowMap rms;    // RMSNorm of the stored output row (base null = none)
  const void* gamma;
  float eps;
  KVStore kv;
  int scale_cols;     // output columns n < scale_cols are multiplied by col_scale
  float col_scale;    // (queries leave the GEMM pre-scaled by 1/sqrt(d_h) * log2(e))
  RowMap act_in, act_out;  // ACT_GELU_BWD: u read, GELU(u) written (storage type)
};

// Queries arrive pre-scaled by 1/sqrt(d_h) * log2(e) (the producing GEMM's
// epilogue), so q.k is already a base-2 logit.
struct AttnDesc {
  int B, H, dh, Lq, q_pos0;  // query t of batch b sits at key position q_pos0 + t
  const int* q_pos0_u;       // or, when set (device, per batch b): q_pos0_u[b] + t
  RowMap q, o;                // columns: head h occupies [h*dh, (h+1)*dh)
  KVStore kv;
};

// Stage II attention: candidates of one user share the user's cached S keys.
// Rows are candidate-major: row c*L_NS + j is NS token j of candidate c.
struct Stage2Desc {
  int H, dh, L_NS, C_tot, s_len, n_users;
  const int* s_len_u;  // cached S keys of each user at this layer (device, [n_users]), or null: s_len for all
  double s_sum;        // sum over candidates of their user's cached S keys (profiling)
  const int* tiles;    // n_tiles x {user, c0, c1}
  const void* qkv;     // [C_tot, L_NS, 3d] Q|K|V of the NS rows
  void* o;             // [C_tot, L_NS, d]
  KVStore kv;          // row_off indexed by user
};

__host__ __device__ inline void row_of_rows(int mode, int fold, int m, int g, int& b, int& t) {
  if (mode == TILE_ROWS) { t = m; b = g; }
  else if (mode == TILE_SAMPLES) { b = m; t = g; }
  else { b = m / fold; t = m - b * fold; }
}
__host__ __device__ inline void row_of(const GemmDesc& d, int m, int g, int& b, int& t) {
  row_of_rows(d.mode, d.fold, m, g, b, t);
}

__host__ __device__ inline long long rm_off(const RowMap& r, int b, int t, int n) {
  return (long long)b * r.sb + (long long)t * r.st + (long long)(n / r.split) * r.sc + (n % r.split);
}

__host__ __device__ inline long long kv_off(const KVStore& kv, int b, int pos, int kind, int head, int e) {
  int page = kv.table ? kv.table[kv.row_off[b] + pos / kv.P] : b * kv.pps + pos / kv.P;
  return (long long)page * (2LL * kv.H * kv.P * kv.dh) +
         ((long long)(kind * kv.H + head) * kv.P + (pos % kv.P)) * kv.dh + e;
}

template <typename T> __device__ inline float to_f(T v);
template <> __device__ inline float to_f<float>(float v) { return v; }
template <> __device__ inline float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ inline T from_f(float v);
template <> __device__ inline float from_f<float>(float v) { return v; }
template <> __device__ inline __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename T> __device__ inline float rm_load(const RowMap& r, long long off) {
  return r.f32 ? ((const float*)r.base)[off] : to_f(((const T*)r.base)[off]);
}
template <typename T> __device__ inline void rm_store(const RowMap& r, long long off, float v) {
  if (r.f32) ((float*)r.base)[off] = v;
  else ((T*)r.base)[off] = from_f<T>(v);
}

// GELU, tanh form (Hendrycks & Gimpel): 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3)))
__device__ inline float gelu_tanh(float x) {
  const float k0 = 0.7978845608028654f, k1 = 0.044715f;
  return 0.5f * x * (1.0f + tanhf(k0 * (x + k1 * x * x * x)));
}

// Device status word: kernels that detect a bounds or wait failure record a
// code here instead of trapping; the host reads and clears it.
__device__ int g_device_status = 0;  // one translation unit holds every kernel
__device__ inline void flag_error(int code) { atomicCAS(&g_device_status, 0, code); }

// Programmatic dependent launch.  Kernels of one call follow each other on a
// stream; launched with the programmatic-serialization attribute, a kernel's
// CTAs may start while its predecessor's last CTAs still run.  Each kernel
// therefore does only local set-up (barrier init, descriptor prefetch, TMEM
// allocation) before grid_dep_wait(), which returns once the predecessor grid
// has completed and its memory is visible; every global read or write of
// data that another kernel produces or consumes comes after it.  A kernel
// signals grid_dep_launch() only after its own TMEM allocation, so a
// dependent CTA that allocates before its wait never holds columns that a
// not-yet-started CTA of the predecessor needs.  Without the launch attribute
// both instructions are no-ops.
__device__ inline void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace ot
