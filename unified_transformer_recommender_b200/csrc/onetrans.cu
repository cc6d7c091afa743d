// Host side of the OneTrans C ABI: validation, schedules, workspace carving,
// paged-cache bookkeeping and the launch sequence of every entry point.
// All kernels live in this one translation unit (see the included headers).
#include "onetrans.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "simt.cuh"
#include "gemm_tc.cuh"
#include "gemm_persist.cuh"
#include "gemm_bres.cuh"
#include "attn_tc.cuh"
#include "ffn_tc.cuh"
#include "backward.cuh"
#include "attn_train.cuh"
#include "gemm_wgrad.cuh"

using namespace ot;

// ============================================================== model ====
struct onetrans_model {
  onetrans_config cfg;
  std::vector<int> pyr;
  int d, H, dh, dff, L_NS, NL, es;
  bool bf16;
  std::vector<const void*> g_attn, g_ffn, Wqkv_S, Wqkv_NS, Wo, W1_S, b1_S, W2_S, b2_S, W1_NS,
      b1_NS, W2_NS, b2_NS, Wb1, bb1, Wb2, bb2;
  const void *Wa1, *ba1, *Wa2, *ba2, *type_emb, *w_head, *b_head;
};

struct onetrans_cache {
  const onetrans_model* m;
  char* pool;
  size_t bytes;
  int n_slots, max_L_S, max_pages, n_pages;
  int* d_table;
  char* d_pages;
  std::vector<int> h_table;  // [slot][layer][max_pages], -1 = unassigned
  std::vector<int> len;      // cached S length per slot
  std::vector<int> free_pages;
};

static int g_policy = 0;

// ------------------------------------------------------------ profiling --
// When enabled, every launch is bracketed by CUDA events on its stream and
// tagged with a kernel kind and its algorithmic FLOPs and bytes.
enum ProfKind {
  PK_GEMM_QKV = 0, PK_GEMM_OPROJ, PK_GEMM_FFN_UP, PK_GEMM_FFN_DOWN, PK_GEMM_AUTOSPLIT, PK_ATTN_CAUSAL,
  PK_ATTN_STAGE2, PK_RMSNORM, PK_TOKENIZE, PK_BLOCK_TAIL, PK_HEAD, PK_TRAIN, PK_TRAIN_ATTN, PK_TRAIN_ELEM,
  PK_COUNT
};
static const char* kProfNames[PK_COUNT] = {"gemm_qkv", "gemm_oproj_rms", "gemm_ffn_up_gelu", "gemm_ffn_down_rms",
                                           "gemm_autosplit", "attn_causal", "attn_stage2", "rmsnorm",
                                           "tokenize_events", "fused_oproj_ffn", "score_head",
                                           "train_gemm", "train_attn_rows", "train_elementwise"};
struct ProfRec {
  int kind;
  cudaEvent_t e0, e1;
  double flops, bytes;
};
static struct {
  std::mutex mu;
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
} g_prof;

static cudaEvent_t prof_event() {
  if (g_prof.used < g_prof.pool.size()) return g_prof.pool[g_prof.used++];
  cudaEvent_t e;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  g_prof.pool.push_back(e);
  g_prof.used++;
  return e;
}

struct ProfScope {
  bool on;
  ProfRec rec;
  cudaStream_t st;
  ProfScope(int kind, double flops, double bytes, cudaStream_t s) : on(false), st(s) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (!g_prof.on) return;
    rec.kind = kind; rec.flops = flops; rec.bytes = bytes;
    rec.e0 = prof_event(); rec.e1 = prof_event();
    if (!rec.e0 || !rec.e1) return;
    on = cudaEventRecord(rec.e0, st) == cudaSuccess;
  }
  // the scope launched nothing after all (a kernel refused the shape): no record
  void cancel() { on = false; }
  ~ProfScope() {
    if (!on) return;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (cudaEventRecord(rec.e1, st) == cudaSuccess) g_prof.recs.push_back(rec);
  }
};
static const int kMaxUsers = 65536;  // users per Stage II call (workspace holds their table rows)

#define OT_TRY(x)                                  \
  do {                                             \
    onetrans_status _s = (x);                      \
    if (_s != ONETRANS_OK) return _s;              \
  } while (0)

static onetrans_status cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return ONETRANS_OK;
  return ONETRANS_ERR_CUDA;
}
static onetrans_status last_launch() { return cuda_ok(cudaGetLastError()); }

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
static long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// Query count of each layer for an input of L_S S rows.
static onetrans_status schedule_of(const onetrans_model* m, int L_S, std::vector<int>& Lq) {
  if (L_S < 0) return ONETRANS_ERR_SHAPE;
  Lq.assign(m->NL, 0);
  int L = L_S + m->L_NS;
  for (int n = 0; n < m->NL; ++n) {
    int q = m->pyr.empty() ? L : m->pyr[n];
    if (q < m->L_NS || q > L) return ONETRANS_ERR_SHAPE;
    Lq[n] = q;
    L = q;
  }
  return ONETRANS_OK;
}

// S rows per layer (s_n) and S rows among the queries (s'_n) for Stage I.
static onetrans_status s_rows_of(const onetrans_model* m, int L_S, std::vector<int>& s,
                                 std::vector<int>& sq) {
  std::vector<int> Lq;
  OT_TRY(schedule_of(m, L_S, Lq));
  s.assign(m->NL, 0);
  sq.assign(m->NL, 0);
  int cur = L_S;
  for (int n = 0; n < m->NL; ++n) {
    s[n] = cur;
    sq[n] = Lq[n] - m->L_NS;
    cur = sq[n];
  }
  return ONETRANS_OK;
}

// Bump allocator over the caller's workspace; with base == null it only sizes.
struct Carve {
  char* base;
  size_t cap, used = 0;
  bool overflow = false;
  Carve(void* b, size_t c) : base((char*)b), cap(c) {}
  void* take(size_t bytes) {
    used = (used + 255) & ~(size_t)255;
    void* p = base ? base + used : nullptr;
    used += bytes;
    if (base && used > cap) overflow = true;
    return p;
  }
};

static RowMap rmap(const void* base, long long sb, long long st) {
  RowMap r;
  r.base = (void*)base;
  r.sb = sb;
  r.st = st;
  r.sc = 0;
  r.split = 1 << 30;
  r.f32 = 0;
  return r;
}
// Map over a float32 tensor (residual stream, stack outputs).
static RowMap rmap32(const void* base, long long sb, long long st) {
  RowMap r = rmap(base, sb, st);
  r.f32 = 1;
  return r;
}

// Element pointer with an element offset (may be negative relative to a
// buffer start only when every address the map produces stays in bounds).
static void* eoff(const void* p, long long elems, int es) { return (char*)p + elems * es; }

static GemmDesc gdesc_base(const onetrans_model* m) {
  GemmDesc d;
  std::memset(&d, 0, sizeof(d));
  d.eps = m->cfg.rms_eps;
  d.w_groups = 1;
  d.fold = 1 << 30;
  return d;
}

// Queries leave their GEMM multiplied by 1/sqrt(d_h) * log2(e): the attention
// kernels then work on base-2 logits directly.
static void prescale_q(const onetrans_model* m, GemmDesc& g) {
  g.scale_cols = m->d;
  g.col_scale = (float)(1.4426950408889634 / std::sqrt((double)m->dh));
}

// ============================================================= launches ==
template <typename T>
static onetrans_status launch_rms(GemmDesc d, cudaStream_t st) {
  if (d.M <= 0 || d.G <= 0) return ONETRANS_OK;
  ProfScope prof(PK_RMSNORM, 0.0, (double)d.M * d.G * d.N * (sizeof(T) + (d.out.f32 ? 4 : sizeof(T))), st);
  dim3 grid((unsigned)cdiv(d.M, 8), (unsigned)d.G);
  rms_rows_kernel<T><<<grid, 256, 0, st>>>(d);
  return last_launch();
}

// Algorithmic bytes of one GEMM launch: A, W and every tensor the epilogue
// reads or writes, each once.
static double gemm_bytes(const onetrans_model* m, const GemmDesc& d) {
  const double rows = (double)d.M * d.G, es = m->es;
  double b = rows * d.K * es + (double)d.N * d.K * es * (d.mode == TILE_SAMPLES ? d.G : 1);
  b += rows * d.N * (d.out_kind == OUT_KV ? es : (d.out.f32 ? 4 : es));
  if (d.res.base) b += rows * d.N * (d.res.f32 ? 4 : es);
  if (d.rms.base) b += rows * d.N * es;
  if (d.act == ACT_GELU_BWD) b += 2.0 * rows * d.N * es;
  return b;
}

template <typename T>
static onetrans_status launch_gemm(const onetrans_model* m, const GemmDesc& d, cudaStream_t st,
                                   int kind = PK_GEMM_QKV) {
  if (d.M <= 0 || d.G <= 0 || d.N <= 0) return ONETRANS_OK;
  if (cdiv(d.M, 64) > 65535 || d.G > 65535) return ONETRANS_ERR_SHAPE;
  ProfScope prof(kind, 2.0 * d.M * d.G * (double)d.N * d.K, gemm_bytes(m, d), st);
  if (d.act == ACT_GELU_BWD) {
    // the GELU-backward epilogue exists in the weight-resident kernel only
    if (!(m->bf16 && g_policy == 0 && tc_gemm_supported(d) && tc_bres_supported(d))) {
      prof.cancel();
      return ONETRANS_ERR_UNSUPPORTED;
    }
    const onetrans_status r = tc_bres_launch(d, device_sm_count(), st);
    if (r == ONETRANS_ERR_UNSUPPORTED) prof.cancel();
    return r;
  }
  if (m->bf16 && g_policy == 0 && tc_gemm_supported(d)) {
    if (tc_bres_supported(d)) {
      const onetrans_status r = tc_bres_launch(d, device_sm_count(), st);
      if (r != ONETRANS_ERR_UNSUPPORTED) return r;
    }
    if (tc_persist_supported(d)) {
      const onetrans_status r = tc_persist_launch(d, st);
      if (r != ONETRANS_ERR_UNSUPPORTED) return r;
    }
    return tc_gemm_launch(d, st);
  }
  if (d.w_mn) {   // the callers transpose the weight instead
    prof.cancel();
    return ONETRANS_ERR_UNSUPPORTED;
  }
  dim3 grid((unsigned)cdiv(d.N, 64), (unsigned)cdiv(d.M, 64), (unsigned)d.G);
  gemm_simt_kernel<T><<<grid, 256, 0, st>>>(d);
  OT_TRY(last_launch());
  if (d.rms.base) OT_TRY(launch_rms<T>(d, st));
  return ONETRANS_OK;
}

template <typename T>
static onetrans_status launch_attn(const onetrans_model* m, const AttnDesc& a, cudaStream_t st) {
  if (a.Lq <= 0 || a.B <= 0) return ONETRANS_OK;
  // visible (query, key) pairs: query t sees q_pos0 + t + 1 keys
  const double pairs = (double)a.Lq * a.q_pos0 + 0.5 * (double)a.Lq * (a.Lq + 1);
  const double kv_bytes = 2.0 * (a.q_pos0 + a.Lq) * a.H * a.dh * m->es;
  ProfScope prof(PK_ATTN_CAUSAL, 4.0 * a.dh * a.H * a.B * pairs,
                 a.B * (kv_bytes + 2.0 * a.Lq * a.H * a.dh * m->es), st);
  if (m->bf16 && g_policy == 0 && tc_attn_supported(a)) return tc_attn_launch(a, st);
  dim3 grid((unsigned)cdiv(a.Lq, 64), (unsigned)a.H, (unsigned)a.B);
  switch (a.dh) {
    case 16: attn_simt_kernel<T, 16><<<grid, 64, 0, st>>>(a); break;
    case 32: attn_simt_kernel<T, 32><<<grid, 64, 0, st>>>(a); break;
    case 64: attn_simt_kernel<T, 64><<<grid, 64, 0, st>>>(a); break;
    case 96: attn_simt_kernel<T, 96><<<grid, 64, 0, st>>>(a); break;
    case 128: attn_simt_kernel<T, 128><<<grid, 64, 0, st>>>(a); break;
    default: return ONETRANS_ERR_UNSUPPORTED;
  }
  return last_launch();
}

// Tensor-core Stage II attention takes tiles of up to 128 candidates, the
// CUDA-core kernel up to 64.
static bool stage2_tc(const onetrans_model* m, const Stage2Desc& a) {
  return m->bf16 && g_policy == 0 && tc_stage2_supported(a);
}

template <typename T>
static onetrans_status launch_stage2_attn(const onetrans_model* m, const Stage2Desc& a, int n_tiles,
                                          cudaStream_t st) {
  if (n_tiles <= 0) return ONETRANS_OK;
  // per candidate: token j sees s_len + j + 1 keys; bytes: the users' cached
  // K/V once each, Q/K/V of the NS rows, the output
  const double pairs = a.L_NS * a.s_sum + (double)a.C_tot * 0.5 * a.L_NS * (a.L_NS + 1);
  const double es = m->es;
  ProfScope prof(PK_ATTN_STAGE2, 4.0 * a.dh * a.H * pairs,
                 a.n_users * 2.0 * a.s_len * a.H * a.dh * es + (double)a.L_NS * a.C_tot * a.H * a.dh * es * 4, st);
  if (stage2_tc(m, a)) return tc_stage2_launch(a, n_tiles, st);
  dim3 grid((unsigned)n_tiles, (unsigned)a.H, (unsigned)a.L_NS);
  switch (a.dh) {
    case 16: stage2_attn_simt_kernel<T, 16><<<grid, 64, 0, st>>>(a); break;
    case 32: stage2_attn_simt_kernel<T, 32><<<grid, 64, 0, st>>>(a); break;
    case 64: stage2_attn_simt_kernel<T, 64><<<grid, 64, 0, st>>>(a); break;
    case 96: stage2_attn_simt_kernel<T, 96><<<grid, 64, 0, st>>>(a); break;
    case 128: stage2_attn_simt_kernel<T, 128><<<grid, 64, 0, st>>>(a); break;
    default: return ONETRANS_ERR_UNSUPPORTED;
  }
  return last_launch();
}

// RMSNorm of `rows` contiguous rows of width d: dst = RMS(src) * gamma.
template <typename T>
static onetrans_status rms_flat(const onetrans_model* m, const void* src, bool src_f32, void* dst,
                                long long rows, const void* gamma, cudaStream_t st) {
  GemmDesc d = gdesc_base(m);
  d.mode = TILE_FLAT;
  d.M = (int)rows;
  d.G = 1;
  d.N = m->d;
  d.out = src_f32 ? rmap32(src, 0, m->d) : rmap(src, 0, m->d);
  d.rms = rmap(dst, 0, m->d);
  d.gamma = gamma;
  const int ch = m->d / 128;
  const bool aligned = ((uintptr_t)src % 16 == 0) && ((uintptr_t)dst % 16 == 0) && ((uintptr_t)gamma % 16 == 0);
  if (rows <= 0 || m->d % 128 || ch < 1 || ch > 4 || !aligned) return launch_rms<T>(d, st);
  ProfScope prof(PK_RMSNORM, 0.0, (double)rows * m->d * (sizeof(T) + (src_f32 ? 4 : sizeof(T))), st);
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  T* y = (T*)dst;
  const T* gm = (const T*)gamma;
  const float eps = m->cfg.rms_eps;
#define OT_RMS_FLAT(CH)                                                                                   \
  if (src_f32)                                                                                            \
    launch_dependent(rms_flat_kernel<T, float, CH>, dim3(blocks), dim3(256), 0, st, (const float*)src, y, gm, \
                     rows, eps);                                                                             \
  else                                                                                                     \
    launch_dependent(rms_flat_kernel<T, T, CH>, dim3(blocks), dim3(256), 0, st, (const T*)src, y, gm, rows, eps);
  switch (ch) {
    case 1: OT_RMS_FLAT(1) break;
    case 2: OT_RMS_FLAT(2) break;
    case 3: OT_RMS_FLAT(3) break;
    default: OT_RMS_FLAT(4) break;
  }
#undef OT_RMS_FLAT
  return last_launch();
}

// ------------------------------------------------------------ block tail --
// W^O + residual + RMSNorm + mixed FFN + residual (+ the next RMSNorm) over
// the rows that `f` (the FFN-up GEMM) enumerates.  `res` maps those rows to
// the block's residual input in f's (b, t) convention.
static FfnDesc ffn_desc(const onetrans_model* m, const GemmDesc& go, const GemmDesc& f, const GemmDesc& f2,
                        const RowMap& res) {
  FfnDesc fd;
  std::memset(&fd, 0, sizeof(fd));
  fd.mode = f.mode; fd.M = f.M; fd.m_lo = f.m_lo; fd.G = f.G; fd.g_lo = f.g_lo; fd.fold = f.fold;
  fd.grp_base = f.grp_base;
  fd.A = go.A;  // the attention output has the layout of h2
  fd.a_sm = f.a_sm; fd.a_sg = f.a_sg; fd.a_mext = f.a_mext; fd.a_gext = f.a_gext;
  fd.Wo = go.W;
  fd.W1 = f.W; fd.w1_sg = f.w_sg; fd.b1 = f.bias; fd.b1_sg = f.bias_sg;
  fd.W2 = f2.W; fd.w2_sg = f2.w_sg; fd.b2 = f2.bias; fd.b2_sg = f2.bias_sg;
  fd.g_ffn = go.gamma; fd.g_next = f2.gamma;
  fd.res = res; fd.out = f2.out; fd.hout = f2.rms;
  fd.dff = m->dff; fd.w_groups = f.w_groups; fd.eps = m->cfg.rms_eps;
  return fd;
}

static bool use_fused_tail(const onetrans_model* m, const FfnDesc& fd) {
  return m->bf16 && g_policy == 0 && m->d == FfnCfg::D && tc_ffn_supported(fd);
}

static onetrans_status launch_fused_tail(const onetrans_model* m, const FfnDesc& fd, cudaStream_t st) {
  if (fd.M <= 0 || fd.G <= 0) return ONETRANS_OK;
  const double rows = (double)fd.M * fd.G, d = m->d;
  ProfScope prof(PK_BLOCK_TAIL, 2.0 * rows * (d * d + 2.0 * d * m->dff),
                 rows * d * (2.0 + (fd.res.f32 ? 4 : 2) + 4 + (fd.hout.base ? 2 : 0)) +
                     2.0 * (d * d + (fd.mode == TILE_SAMPLES ? fd.G : 1) * 2.0 * d * m->dff),
                 st);
  return tc_ffn_launch(fd, st);
}

// ================================================================ forward =
template <typename T>
static onetrans_status forward_impl(const onetrans_model* m, const void* x0, int B, int L_S, void* out,
                                    void* ws, size_t ws_bytes, cudaStream_t st, size_t* need) {
  std::vector<int> Lq;
  OT_TRY(schedule_of(m, L_S, Lq));
  const int d = m->d, dff = m->dff, L_NS = m->L_NS, es = m->es, P = m->cfg.page_tokens;
  const int L0 = L_S + L_NS, Lq1 = Lq[0];
  const long long pps = cdiv(L0, P);
  Carve cv(ws, ws_bytes);
  void* xa = cv.take((size_t)B * Lq1 * d * 4);   // residual stream: float32
  void* xb = cv.take((size_t)B * Lq1 * d * 4);
  void* h = cv.take((size_t)B * L0 * d * es);
  void* q = cv.take((size_t)B * Lq1 * d * es);
  void* at = cv.take((size_t)B * Lq1 * d * es);
  void* xm = cv.take((size_t)B * Lq1 * d * 4);
  void* h2 = cv.take((size_t)B * Lq1 * d * es);
  void* hid = cv.take((size_t)B * Lq1 * dff * es);
  void* kvb = cv.take((size_t)B * pps * 2 * d * P * es);
  if (need) { *need = cv.used; return ONETRANS_OK; }
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;

  KVStore kv;
  std::memset(&kv, 0, sizeof(kv));
  kv.pool = kvb; kv.P = P; kv.H = m->H; kv.dh = m->dh; kv.pps = (int)pps; kv.n_pages = (int)(B * pps);

  OT_TRY(rms_flat<T>(m, x0, false, h, (long long)B * L0, m->g_attn[0], st));
  const void* x_in = x0;
  int L = L0;
  for (int n = 0; n < m->NL; ++n) {
    const int s = L - L_NS, Lqn = Lq[n], sq = Lqn - L_NS, off = L - Lqn;
    const bool last = n + 1 == m->NL;
    void* x_next = last ? out : (n % 2 == 0 ? xa : xb);
    // -- S rows: K,V of all S rows; Q of the tail S rows
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_ROWS; g.M = s; g.m_lo = 0; g.G = B; g.g_lo = 0;
    g.K = d; g.A = h; g.a_sm = d; g.a_sg = (long long)L * d; g.a_mext = L; g.a_gext = B;
    g.W = m->Wqkv_S[n]; g.w_rows = 3 * d; g.n_lo = d; g.N = 2 * d;
    g.out_kind = OUT_KV; g.kv = kv;
    OT_TRY(launch_gemm<T>(m, g, st));
    if (sq > 0) {
      g.m_lo = s - sq; g.M = sq; g.n_lo = 0; g.N = d; g.out_kind = OUT_ROWS;
      g.out = rmap(eoff(q, -(long long)off * d, es), (long long)Lqn * d, d);
      prescale_q(m, g);
      OT_TRY(launch_gemm<T>(m, g, st));
    }
    // -- NS rows: token j uses its own weights; tile across samples
    GemmDesc gn = gdesc_base(m);
    gn.mode = TILE_SAMPLES; gn.M = B; gn.m_lo = 0; gn.G = L_NS; gn.g_lo = s; gn.grp_base = s;
    gn.K = d; gn.A = h; gn.a_sm = (long long)L * d; gn.a_sg = d; gn.a_mext = B; gn.a_gext = L;
    gn.W = m->Wqkv_NS[n]; gn.w_sg = 3LL * d * d; gn.w_rows = 3 * d; gn.w_groups = L_NS;
    gn.n_lo = 0; gn.N = d; gn.out_kind = OUT_ROWS;
    gn.out = rmap(eoff(q, -(long long)off * d, es), (long long)Lqn * d, d);
    prescale_q(m, gn);
    OT_TRY(launch_gemm<T>(m, gn, st));
    gn.scale_cols = 0;
    gn.n_lo = d; gn.N = 2 * d; gn.out_kind = OUT_KV; gn.kv = kv;
    OT_TRY(launch_gemm<T>(m, gn, st));
    // -- attention of the Lqn tail queries over keys 0..p
    AttnDesc a;
    std::memset(&a, 0, sizeof(a));
    a.B = B; a.H = m->H; a.dh = m->dh; a.Lq = Lqn; a.q_pos0 = off;
    a.q = rmap(q, (long long)Lqn * d, d);
    a.o = rmap(at, (long long)Lqn * d, d);
    a.kv = kv;
    OT_TRY(launch_attn<T>(m, a, st));
    // -- W^O + residual, then RMSNorm for the FFN (all tail rows share W^O)
    GemmDesc go = gdesc_base(m);
    go.mode = TILE_FLAT; go.M = B * Lqn; go.fold = Lqn; go.G = 1;
    go.K = d; go.A = at; go.a_sm = d; go.a_mext = (long long)B * Lqn; go.a_gext = 1;
    go.W = m->Wo[n]; go.w_rows = d; go.N = d;
    go.res = n == 0 ? rmap(eoff(x_in, (long long)off * d, es), (long long)L * d, d)
                    : rmap32(eoff(x_in, (long long)off * d, 4), (long long)L * d, d);
    go.out = rmap32(xm, (long long)Lqn * d, d);
    go.rms = rmap(h2, (long long)Lqn * d, d);
    go.gamma = m->g_ffn[n];
    // -- mixed FFN: S tail rows shared, NS rows per token
    GemmDesc fs[2], f2s[2];
    bool has[2] = {false, false};
    for (int part = 0; part < 2; ++part) {
      GemmDesc f = gdesc_base(m);
      if (part == 0) {
        if (sq <= 0) continue;
        f.mode = TILE_ROWS; f.M = sq; f.G = B; f.a_sm = d; f.a_sg = (long long)Lqn * d;
        f.a_mext = Lqn; f.a_gext = B;
      } else {
        f.mode = TILE_SAMPLES; f.M = B; f.G = L_NS; f.g_lo = sq; f.grp_base = sq;
        f.a_sm = (long long)Lqn * d; f.a_sg = d; f.a_mext = B; f.a_gext = Lqn;
      }
      f.K = d; f.A = h2;
      f.W = part ? m->W1_NS[n] : m->W1_S[n]; f.w_rows = dff; f.N = dff;
      f.w_sg = part ? (long long)dff * d : 0; f.w_groups = part ? L_NS : 1;
      f.bias = part ? m->b1_NS[n] : m->b1_S[n]; f.bias_sg = part ? dff : 0;
      f.act = ACT_GELU;
      f.out = rmap(hid, (long long)Lqn * dff, dff);
      GemmDesc f2 = f;
      f2.K = dff; f2.A = hid; f2.act = ACT_NONE;
      if (part == 0) { f2.a_sm = dff; f2.a_sg = (long long)Lqn * dff; }
      else { f2.a_sm = (long long)Lqn * dff; f2.a_sg = dff; }
      f2.W = part ? m->W2_NS[n] : m->W2_S[n]; f2.w_rows = d; f2.N = d;
      f2.w_sg = part ? (long long)d * dff : 0;
      f2.bias = part ? m->b2_NS[n] : m->b2_S[n]; f2.bias_sg = part ? d : 0;
      f2.res = rmap32(xm, (long long)Lqn * d, d);
      f2.out = rmap32(x_next, (long long)Lqn * d, d);
      if (!last) { f2.rms = rmap(h, (long long)Lqn * d, d); f2.gamma = m->g_attn[n + 1]; }
      fs[part] = f; f2s[part] = f2; has[part] = true;
    }
    bool fused = true;
    FfnDesc fds[2];
    for (int part = 0; part < 2; ++part)
      if (has[part]) { fds[part] = ffn_desc(m, go, fs[part], f2s[part], go.res); fused = fused && use_fused_tail(m, fds[part]); }
    if (fused) {
      for (int part = 0; part < 2; ++part)
        if (has[part]) OT_TRY(launch_fused_tail(m, fds[part], st));
    } else {
      OT_TRY(launch_gemm<T>(m, go, st, PK_GEMM_OPROJ));
      for (int part = 0; part < 2; ++part) {
        if (!has[part]) continue;
        OT_TRY(launch_gemm<T>(m, fs[part], st, PK_GEMM_FFN_UP));
        OT_TRY(launch_gemm<T>(m, f2s[part], st, PK_GEMM_FFN_DOWN));
      }
    }
    x_in = x_next;
    L = Lqn;
  }
  return ONETRANS_OK;
}

// ============================================================== stage I ==
static void kv_for_cache(const onetrans_cache* c, int layer, const int* d_row_off, KVStore& kv) {
  std::memset(&kv, 0, sizeof(kv));
  kv.pool = c->d_pages;
  kv.table = c->d_table + (size_t)layer * c->max_pages;
  kv.row_off = d_row_off;
  kv.P = c->m->cfg.page_tokens;
  kv.H = c->m->H;
  kv.dh = c->m->dh;
  kv.n_pages = c->n_pages;
}

static onetrans_status upload_slot_table(onetrans_cache* c, int slot, cudaStream_t st) {
  const size_t row = (size_t)c->m->NL * c->max_pages;
  return cuda_ok(cudaMemcpyAsync(c->d_table + slot * row, c->h_table.data() + slot * row,
                                 row * sizeof(int), cudaMemcpyHostToDevice, st));
}

template <typename T>
static onetrans_status stage1_impl(const onetrans_model* m, onetrans_cache* c, const int* slots, int U,
                                   const void* s_tok, int L_S, void* ws, size_t ws_bytes,
                                   cudaStream_t st, size_t* need) {
  std::vector<int> s, sq;
  OT_TRY(s_rows_of(m, L_S, s, sq));
  const int d = m->d, dff = m->dff, es = m->es;
  const int sq1 = std::max(sq[0], 0);
  Carve cv(ws, ws_bytes);
  void* xa = cv.take((size_t)U * sq1 * d * 4);   // residual stream: float32
  void* xb = cv.take((size_t)U * sq1 * d * 4);
  void* h = cv.take((size_t)U * L_S * d * es);
  void* q = cv.take((size_t)U * sq1 * d * es);
  void* at = cv.take((size_t)U * sq1 * d * es);
  void* xm = cv.take((size_t)U * sq1 * d * 4);
  void* h2 = cv.take((size_t)U * sq1 * d * es);
  void* hid = cv.take((size_t)U * sq1 * dff * es);
  int* row_off = (int*)cv.take((size_t)U * sizeof(int));
  if (need) { *need = cv.used; return ONETRANS_OK; }
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;
  if (L_S > c->max_L_S) return ONETRANS_ERR_CAPACITY;

  // page assignment on the host: release the slots' pages, take new ones
  const int P = m->cfg.page_tokens;
  long long needed = 0, owned = 0;
  for (int u = 0; u < U; ++u) {
    for (int n = 0; n < m->NL; ++n) needed += cdiv(s[n], P);
    const size_t row = (size_t)slots[u] * m->NL * c->max_pages;
    for (size_t i = 0; i < (size_t)m->NL * c->max_pages; ++i) owned += c->h_table[row + i] >= 0;
  }
  if (needed > (long long)c->free_pages.size() + owned) return ONETRANS_ERR_CAPACITY;
  std::vector<int> h_row_off(U);
  for (int u = 0; u < U; ++u) {
    const size_t row = (size_t)slots[u] * m->NL * c->max_pages;
    for (size_t i = 0; i < (size_t)m->NL * c->max_pages; ++i) {
      if (c->h_table[row + i] >= 0) c->free_pages.push_back(c->h_table[row + i]);
      c->h_table[row + i] = -1;
    }
    for (int n = 0; n < m->NL; ++n)
      for (long long p = 0; p < cdiv(s[n], P); ++p) {
        c->h_table[row + (size_t)n * c->max_pages + p] = c->free_pages.back();
        c->free_pages.pop_back();
      }
    c->len[slots[u]] = L_S;
    h_row_off[u] = (int)row;
    OT_TRY(upload_slot_table(c, slots[u], st));
  }
  OT_TRY(cuda_ok(cudaMemcpyAsync(row_off, h_row_off.data(), U * sizeof(int), cudaMemcpyHostToDevice, st)));

  OT_TRY(rms_flat<T>(m, s_tok, false, h, (long long)U * L_S, m->g_attn[0], st));
  const void* x_in = s_tok;
  for (int n = 0; n < m->NL; ++n) {
    const int sn = s[n], sqn = sq[n];
    if (sn <= 0) break;
    KVStore kv;
    kv_for_cache(c, n, row_off, kv);
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_FLAT; g.M = U * sn; g.fold = sn; g.G = 1;
    g.K = d; g.A = h; g.a_sm = d; g.a_mext = (long long)U * sn; g.a_gext = 1;
    g.W = m->Wqkv_S[n]; g.w_rows = 3 * d; g.n_lo = d; g.N = 2 * d;
    g.out_kind = OUT_KV; g.kv = kv;
    OT_TRY(launch_gemm<T>(m, g, st));
    // the last layer's outputs feed nothing that is cached: only its K/V are needed
    if (sqn <= 0 || n + 1 == m->NL) break;
    void* x_next = n % 2 == 0 ? xa : xb;
    GemmDesc gq = gdesc_base(m);
    gq.mode = TILE_ROWS; gq.M = sqn; gq.m_lo = sn - sqn; gq.G = U;
    gq.K = d; gq.A = h; gq.a_sm = d; gq.a_sg = (long long)sn * d; gq.a_mext = sn; gq.a_gext = U;
    gq.W = m->Wqkv_S[n]; gq.w_rows = 3 * d; gq.n_lo = 0; gq.N = d;
    gq.out = rmap(eoff(q, -(long long)(sn - sqn) * d, es), (long long)sqn * d, d);
    prescale_q(m, gq);
    OT_TRY(launch_gemm<T>(m, gq, st));
    AttnDesc a;
    std::memset(&a, 0, sizeof(a));
    a.B = U; a.H = m->H; a.dh = m->dh; a.Lq = sqn; a.q_pos0 = sn - sqn;
    a.q = rmap(q, (long long)sqn * d, d);
    a.o = rmap(at, (long long)sqn * d, d);
    a.kv = kv;
    OT_TRY(launch_attn<T>(m, a, st));
    GemmDesc go = gdesc_base(m);
    go.mode = TILE_FLAT; go.M = U * sqn; go.fold = sqn; go.G = 1;
    go.K = d; go.A = at; go.a_sm = d; go.a_mext = (long long)U * sqn; go.a_gext = 1;
    go.W = m->Wo[n]; go.w_rows = d; go.N = d;
    go.res = n == 0 ? rmap(eoff(x_in, (long long)(sn - sqn) * d, es), (long long)sn * d, d)
                    : rmap32(eoff(x_in, (long long)(sn - sqn) * d, 4), (long long)sn * d, d);
    go.out = rmap32(xm, (long long)sqn * d, d);
    go.rms = rmap(h2, (long long)sqn * d, d);
    go.gamma = m->g_ffn[n];
    GemmDesc f = go;
    f.res.base = nullptr; f.rms.base = nullptr; f.gamma = nullptr;
    f.A = h2; f.W = m->W1_S[n]; f.w_rows = dff; f.N = dff; f.bias = m->b1_S[n]; f.act = ACT_GELU;
    f.out = rmap(hid, (long long)sqn * dff, dff);
    GemmDesc f2 = go;
    f2.K = dff; f2.A = hid; f2.a_sm = dff; f2.W = m->W2_S[n]; f2.w_rows = d; f2.N = d;
    f2.bias = m->b2_S[n];
    f2.res = rmap32(xm, (long long)sqn * d, d);
    f2.out = rmap32(x_next, (long long)sqn * d, d);
    f2.rms = rmap(h, (long long)sqn * d, d);
    f2.gamma = m->g_attn[n + 1];
    const FfnDesc fd = ffn_desc(m, go, f, f2, go.res);
    if (use_fused_tail(m, fd)) {
      OT_TRY(launch_fused_tail(m, fd, st));
    } else {
      OT_TRY(launch_gemm<T>(m, go, st, PK_GEMM_OPROJ));
      OT_TRY(launch_gemm<T>(m, f, st, PK_GEMM_FFN_UP));
      OT_TRY(launch_gemm<T>(m, f2, st, PK_GEMM_FFN_DOWN));
    }
    x_in = x_next;
  }
  return ONETRANS_OK;
}

// ========================================================= scoring head ==
// logit[c] = w_head . vec(final NS rows of candidate c) + b_head.
template <typename T>
static onetrans_status launch_head(const onetrans_model* m, const float* h, long long C, float* logits,
                                   cudaStream_t st) {
  if (C <= 0) return ONETRANS_OK;
  const int n = m->L_NS * m->d;
  ProfScope prof(PK_HEAD, 2.0 * C * n, (double)C * (n * 4.0 + 4.0) + (double)n * m->es, st);
  const unsigned blocks = (unsigned)cdiv(C, 8);
  launch_dependent(head_logits_kernel<T>, dim3(blocks), dim3(256), 0, st, h, (const T*)m->w_head,
                   (const T*)m->b_head, n, C, logits);
  return last_launch();
}

// ============================================================= stage II ==
template <typename T>
static onetrans_status stage2_impl(const onetrans_model* m, const onetrans_cache* c, const int* slots,
                                   int U, const int* offs, const void* ns_in, void* ns_out, float* logits,
                                   void* ws, size_t ws_bytes, cudaStream_t st, size_t* need, long long C_need,
                                   int L_S_need) {
  const int d = m->d, dff = m->dff, L_NS = m->L_NS, es = m->es;
  const long long C = need ? C_need : offs[U] - offs[0];
  const int L_S = need ? L_S_need : (U > 0 ? c->len[slots[0]] : 0);
  std::vector<int> s, sq;
  OT_TRY(s_rows_of(m, L_S, s, sq));
  // users may hold different cached lengths: each has its own schedule, so
  // its cached S keys per layer go into a table [NL][U] the attention reads
  bool ragged = false;
  std::vector<int> s_tab_h;
  std::vector<double> s_sum(m->NL, 0.0);
  std::vector<int> s_max(m->NL, 0);
  if (!need) {
    s_tab_h.assign((size_t)m->NL * U, 0);
    for (int u = 0; u < U; ++u) {
      const int Lu = c->len[slots[u]];
      ragged = ragged || Lu != L_S;
      std::vector<int> su, squ;
      OT_TRY(s_rows_of(m, Lu, su, squ));
      const double cu = (double)(offs[u + 1] - offs[u]);
      for (int n = 0; n < m->NL; ++n) {
        s_tab_h[(size_t)n * U + u] = su[n];
        s_sum[n] += cu * su[n];
        s_max[n] = std::max(s_max[n], su[n]);
      }
    }
  }
  // every candidate tile holds at least one candidate, so C tiles always
  // suffice; sizing and running carve the same layout
  const long long tile_cap = std::max<long long>(C, 1);
  Carve cv(ws, ws_bytes);
  void* xa = cv.take((size_t)L_NS * C * d * 4);   // residual stream: float32
  void* xb = cv.take((size_t)L_NS * C * d * 4);
  void* h = cv.take((size_t)L_NS * C * d * es);
  void* qkv = cv.take((size_t)L_NS * C * 3 * d * es);
  void* at = cv.take((size_t)L_NS * C * d * es);
  void* xm = cv.take((size_t)L_NS * C * d * 4);
  void* h2 = cv.take((size_t)L_NS * C * d * es);
  void* hid = cv.take((size_t)L_NS * C * dff * es);
  int* row_off = (int*)cv.take((size_t)kMaxUsers * sizeof(int));
  int* d_tiles = (int*)cv.take((size_t)tile_cap * 3 * sizeof(int));
  int* d_s_tab = (int*)cv.take((size_t)m->NL * kMaxUsers * sizeof(int));
  if (need) { *need = cv.used; return ONETRANS_OK; }
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;
  if (C == 0) return ONETRANS_OK;

  // candidate tiles, one user each; the attention kernel decides the tile size
  Stage2Desc probe;
  std::memset(&probe, 0, sizeof(probe));
  probe.H = m->H; probe.dh = m->dh; probe.L_NS = L_NS; probe.C_tot = (int)C;
  probe.qkv = qkv; probe.o = at;
  kv_for_cache(c, 0, row_off, probe.kv);
  const int TQ = stage2_tc(m, probe) ? stage2_cands_per_tile(L_NS) : 64;
  std::vector<int> tiles;
  for (int u = 0; u < U; ++u)
    for (int c0 = offs[u]; c0 < offs[u + 1]; c0 += TQ)
      tiles.insert(tiles.end(), {u, c0 - offs[0], std::min(c0 + TQ, offs[u + 1]) - offs[0]});
  const long long n_tiles = (long long)tiles.size() / 3;
  if (n_tiles > tile_cap) return ONETRANS_ERR_CAPACITY;

  std::vector<int> h_row_off(U);
  for (int u = 0; u < U; ++u) h_row_off[u] = slots[u] * m->NL * c->max_pages;
  OT_TRY(cuda_ok(cudaMemcpyAsync(row_off, h_row_off.data(), U * sizeof(int), cudaMemcpyHostToDevice, st)));
  OT_TRY(cuda_ok(cudaMemcpyAsync(d_tiles, tiles.data(), tiles.size() * sizeof(int), cudaMemcpyHostToDevice, st)));
  if (ragged)
    OT_TRY(cuda_ok(cudaMemcpyAsync(d_s_tab, s_tab_h.data(), s_tab_h.size() * sizeof(int), cudaMemcpyHostToDevice, st)));

  OT_TRY(rms_flat<T>(m, ns_in, false, h, (long long)L_NS * C, m->g_attn[0], st));
  const void* x_in = ns_in;
  const long long Ld = (long long)L_NS * d;   // candidate stride of [C, L_NS, d] rows
  for (int n = 0; n < m->NL; ++n) {
    const bool last = n + 1 == m->NL;
    void* x_next = last ? ns_out : (n % 2 == 0 ? xa : xb);
    // token j of every candidate through W_NS,j: fixed t = j, tiled over candidates
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_SAMPLES; g.M = (int)C; g.G = L_NS; g.g_lo = 0; g.grp_base = 0;
    g.K = d; g.A = h; g.a_sm = Ld; g.a_sg = d; g.a_mext = C; g.a_gext = L_NS;
    g.W = m->Wqkv_NS[n]; g.w_sg = 3LL * d * d; g.w_rows = 3 * d; g.w_groups = L_NS;
    g.n_lo = 0; g.N = 3 * d;
    g.out = rmap(qkv, 3LL * Ld, 3LL * d);
    prescale_q(m, g);
    OT_TRY(launch_gemm<T>(m, g, st));
    Stage2Desc a;
    std::memset(&a, 0, sizeof(a));
    a.H = m->H; a.dh = m->dh; a.L_NS = L_NS; a.C_tot = (int)C; a.n_users = U;
    a.s_len = ragged ? s_max[n] : s[n];
    a.s_len_u = ragged ? d_s_tab + (size_t)n * U : nullptr;
    a.s_sum = ragged ? s_sum[n] : (double)C * s[n];
    a.tiles = d_tiles; a.qkv = qkv; a.o = at;
    kv_for_cache(c, n, row_off, a.kv);
    OT_TRY(launch_stage2_attn<T>(m, a, (int)n_tiles, st));
    GemmDesc go = gdesc_base(m);
    go.mode = TILE_FLAT; go.M = (int)(L_NS * C); go.G = 1;
    go.K = d; go.A = at; go.a_sm = d; go.a_mext = L_NS * C; go.a_gext = 1;
    go.W = m->Wo[n]; go.w_rows = d; go.N = d;
    go.res = n == 0 ? rmap(x_in, 0, d) : rmap32(x_in, 0, d);
    go.out = rmap32(xm, 0, d);
    go.rms = rmap(h2, 0, d);
    go.gamma = m->g_ffn[n];
    GemmDesc f = g;
    f.scale_cols = 0;
    f.A = h2; f.W = m->W1_NS[n]; f.w_sg = (long long)dff * d; f.w_rows = dff; f.N = dff;
    f.bias = m->b1_NS[n]; f.bias_sg = dff; f.act = ACT_GELU;
    f.out = rmap(hid, (long long)L_NS * dff, dff);
    GemmDesc f2 = f;
    f2.K = dff; f2.A = hid; f2.a_sm = (long long)L_NS * dff; f2.a_sg = dff; f2.act = ACT_NONE;
    f2.W = m->W2_NS[n]; f2.w_sg = (long long)d * dff; f2.w_rows = d; f2.N = d;
    f2.bias = m->b2_NS[n]; f2.bias_sg = d;
    f2.res = rmap32(xm, Ld, d);
    f2.out = rmap32(x_next, Ld, d);
    if (!last) { f2.rms = rmap(h, Ld, d); f2.gamma = m->g_attn[n + 1]; }
    const RowMap res_bt = n == 0 ? rmap(x_in, Ld, d) : rmap32(x_in, Ld, d);  // (b = candidate, t = token)
    const FfnDesc fd = ffn_desc(m, go, f, f2, res_bt);
    if (use_fused_tail(m, fd)) {
      OT_TRY(launch_fused_tail(m, fd, st));
    } else {
      OT_TRY(launch_gemm<T>(m, go, st, PK_GEMM_OPROJ));
      OT_TRY(launch_gemm<T>(m, f, st, PK_GEMM_FFN_UP));
      OT_TRY(launch_gemm<T>(m, f2, st, PK_GEMM_FFN_DOWN));
    }
    x_in = x_next;
  }
  if (logits) OT_TRY(launch_head<T>(m, (const float*)ns_out, C, logits, st));
  return ONETRANS_OK;
}

// =============================================================== append ==
// The per-behavior MLPs and type embedding of the event tokenizer.
static EventMLP event_mlp_of(const onetrans_model* m) {
  EventMLP w;
  std::memset(&w, 0, sizeof(w));
  for (int t = 0; t < m->cfg.n_behaviors; ++t) {
    w.W1[t] = m->Wb1[t]; w.b1[t] = m->bb1[t]; w.W2[t] = m->Wb2[t]; w.b2[t] = m->bb2[t];
  }
  w.emb = m->type_emb; w.n_types = m->cfg.n_behaviors; w.e_dim = m->cfg.event_dim; w.d = m->d;
  return w;
}

// Tokenize R events (rows of `events`, type ids on the device) into `out`
// (row (r / dL, r % dL) of the row map).  With an intent layout (lay.n > 0)
// the types come from the layout, output rows are shifted past the [SEP] gaps,
// one more CTA writes the [SEP] rows, and `emb` decides whether the type
// identifiers are added.
template <typename T>
static onetrans_status launch_event_tokenizer(const onetrans_model* m, const void* events, const int* types,
                                              long long R, int dL, const RowMap& out, cudaStream_t st,
                                              const IntentLayout* layout = nullptr, bool emb = true) {
  IntentLayout lay;
  std::memset(&lay, 0, sizeof(lay));
  if (layout) lay = *layout;
  const int n_sep = lay.n > 1 ? 1 : 0;
  if (R < 0 || (R == 0 && !n_sep)) return ONETRANS_OK;
  if (R + lay.n > 0x7fffffff) return ONETRANS_ERR_SHAPE;
  EventMLP w = event_mlp_of(m);
  if (!emb) w.emb = nullptr;
  const int d = m->d;
  const size_t smem = (size_t)(w.e_dim + d) * sizeof(float);
  // the scope of the profiling record is the tokenizer launch alone
  ProfScope prof_tok(PK_TOKENIZE, 2.0 * R * ((double)w.e_dim * d + (double)d * d),
                     (double)R * (w.e_dim * m->es + d * (out.f32 ? 4 : m->es)), st);
  bool w_aligned = true;
  for (int t = 0; t < w.n_types; ++t)
    w_aligned = w_aligned && (uintptr_t)w.W1[t] % 16 == 0 && (uintptr_t)w.W2[t] % 16 == 0;
  if (d == kEvD && w.e_dim <= kEvEmax && w.e_dim % 8 == 0 && w_aligned)
    launch_dependent(event_tokenize_tile_kernel<T>, dim3((unsigned)(cdiv(R, kEvBlock) + n_sep)), dim3(kEvD), 0,
                     st, (const T*)events, types, (int)R, dL, w, out, lay);
  else
    event_tokenize_kernel<T><<<(unsigned)(R + n_sep), std::min(d, 512), smem, st>>>((const T*)events, types, dL,
                                                                                     w, out, lay);
  return last_launch();
}

template <typename T>
static onetrans_status append_impl(const onetrans_model* m, onetrans_cache* c, const int* slots, int U,
                                   const void* events, const int* types, int dL, void* ws,
                                   size_t ws_bytes, cudaStream_t st, size_t* need) {
  const int d = m->d, dff = m->dff, es = m->es, P = m->cfg.page_tokens;
  Carve cv(ws, ws_bytes);
  const long long R = (long long)U * dL;
  void* xa = cv.take((size_t)R * d * 4);   // residual stream: float32
  void* xb = cv.take((size_t)R * d * 4);
  void* h = cv.take((size_t)R * d * es);
  void* q = cv.take((size_t)R * d * es);
  void* at = cv.take((size_t)R * d * es);
  void* xm = cv.take((size_t)R * d * 4);
  void* h2 = cv.take((size_t)R * d * es);
  void* hid = cv.take((size_t)R * dff * es);
  int* row_off = (int*)cv.take((size_t)std::max(U, 1) * sizeof(int));
  int* d_pos0 = (int*)cv.take((size_t)std::max(U, 1) * sizeof(int));
  if (need) { *need = cv.used; return ONETRANS_OK; }
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;
  if (U == 0 || dL == 0) return ONETRANS_OK;
  // user u's new rows take positions [s_old[u], s_old[u] + dL); users may
  // hold different lengths (then the positions go to the kernels as a table)
  std::vector<int> s_old(U);
  bool ragged = false;
  long long needed = 0, sum_old = 0;
  for (int u = 0; u < U; ++u) {
    s_old[u] = c->len[slots[u]];
    if (s_old[u] + dL > c->max_L_S) return ONETRANS_ERR_CAPACITY;
    ragged = ragged || s_old[u] != s_old[0];
    sum_old += s_old[u];
    needed += (long long)m->NL * (cdiv(s_old[u] + dL, P) - cdiv(s_old[u], P));
  }
  if (needed > (long long)c->free_pages.size()) return ONETRANS_ERR_CAPACITY;
  std::vector<int> h_row_off(U);
  for (int u = 0; u < U; ++u) {
    const size_t row = (size_t)slots[u] * m->NL * c->max_pages;
    for (int n = 0; n < m->NL; ++n)
      for (long long p = cdiv(s_old[u], P); p < cdiv(s_old[u] + dL, P); ++p) {
        c->h_table[row + (size_t)n * c->max_pages + p] = c->free_pages.back();
        c->free_pages.pop_back();
      }
    c->len[slots[u]] = s_old[u] + dL;
    h_row_off[u] = (int)row;
    OT_TRY(upload_slot_table(c, slots[u], st));
  }
  OT_TRY(cuda_ok(cudaMemcpyAsync(row_off, h_row_off.data(), U * sizeof(int), cudaMemcpyHostToDevice, st)));
  if (ragged) OT_TRY(cuda_ok(cudaMemcpyAsync(d_pos0, s_old.data(), U * sizeof(int), cudaMemcpyHostToDevice, st)));

  if (R > 0x7fffffff) return ONETRANS_ERR_SHAPE;
  OT_TRY(launch_event_tokenizer<T>(m, events, types, R, dL, rmap32(xa, (long long)dL * d, d), st));
  OT_TRY(rms_flat<T>(m, xa, true, h, R, m->g_attn[0], st));
  const void* x_in = xa;
  for (int n = 0; n < m->NL; ++n) {
    const bool last = n + 1 == m->NL;
    void* x_next = (n % 2 == 0) ? xb : xa;
    KVStore kv;
    kv_for_cache(c, n, row_off, kv);
    kv.pos_off = s_old[0];
    kv.pos_off_u = ragged ? d_pos0 : nullptr;
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_FLAT; g.M = (int)R; g.fold = dL; g.G = 1;
    g.K = d; g.A = h; g.a_sm = d; g.a_mext = R; g.a_gext = 1;
    g.W = m->Wqkv_S[n]; g.w_rows = 3 * d; g.n_lo = d; g.N = 2 * d;
    g.out_kind = OUT_KV; g.kv = kv;
    OT_TRY(launch_gemm<T>(m, g, st));
    if (last) break;  // the last layer's outputs feed nothing that is cached
    g.n_lo = 0; g.N = d; g.out_kind = OUT_ROWS;
    g.out = rmap(q, (long long)dL * d, d);
    prescale_q(m, g);
    OT_TRY(launch_gemm<T>(m, g, st));
    AttnDesc a;
    std::memset(&a, 0, sizeof(a));
    a.B = U; a.H = m->H; a.dh = m->dh; a.Lq = dL;
    // the mean old length when they differ: used only for the profiling counts
    a.q_pos0 = ragged ? (int)(sum_old / U) : s_old[0];
    a.q_pos0_u = ragged ? d_pos0 : nullptr;
    a.q = rmap(q, (long long)dL * d, d);
    a.o = rmap(at, (long long)dL * d, d);
    a.kv = kv; a.kv.pos_off = 0; a.kv.pos_off_u = nullptr;
    OT_TRY(launch_attn<T>(m, a, st));
    GemmDesc go = gdesc_base(m);
    go.mode = TILE_FLAT; go.M = (int)R; go.fold = dL; go.G = 1;
    go.K = d; go.A = at; go.a_sm = d; go.a_mext = R; go.a_gext = 1;
    go.W = m->Wo[n]; go.w_rows = d; go.N = d;
    go.res = rmap32(x_in, (long long)dL * d, d);
    go.out = rmap32(xm, (long long)dL * d, d);
    go.rms = rmap(h2, (long long)dL * d, d);
    go.gamma = m->g_ffn[n];
    GemmDesc f = go;
    f.res.base = nullptr; f.rms.base = nullptr; f.gamma = nullptr;
    f.A = h2; f.W = m->W1_S[n]; f.w_rows = dff; f.N = dff; f.bias = m->b1_S[n]; f.act = ACT_GELU;
    f.out = rmap(hid, (long long)dL * dff, dff);
    GemmDesc f2 = go;
    f2.K = dff; f2.A = hid; f2.a_sm = dff; f2.W = m->W2_S[n]; f2.w_rows = d; f2.N = d;
    f2.bias = m->b2_S[n];
    f2.res = rmap32(xm, (long long)dL * d, d);
    f2.out = rmap32(x_next, (long long)dL * d, d);
    f2.rms = rmap(h, (long long)dL * d, d);
    f2.gamma = m->g_attn[n + 1];
    const FfnDesc fd = ffn_desc(m, go, f, f2, go.res);
    if (use_fused_tail(m, fd)) {
      OT_TRY(launch_fused_tail(m, fd, st));
    } else {
      OT_TRY(launch_gemm<T>(m, go, st, PK_GEMM_OPROJ));
      OT_TRY(launch_gemm<T>(m, f, st, PK_GEMM_FFN_UP));
      OT_TRY(launch_gemm<T>(m, f2, st, PK_GEMM_FFN_DOWN));
    }
    x_in = x_next;
  }
  return ONETRANS_OK;
}

// ============================================================ autosplit ==
template <typename T>
static onetrans_status autosplit_impl(const onetrans_model* m, const void* feats, long long N, void* out,
                                      void* ws, size_t ws_bytes, cudaStream_t st, size_t* need) {
  const int F = m->cfg.ns_feat_dim, Hh = m->cfg.ns_hidden, d = m->d, L_NS = m->L_NS, es = m->es;
  Carve cv(ws, ws_bytes);
  void* hid = cv.take((size_t)N * Hh * es);
  if (need) { *need = cv.used; return ONETRANS_OK; }
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;
  if (N == 0) return ONETRANS_OK;
  GemmDesc g = gdesc_base(m);
  g.mode = TILE_FLAT; g.M = (int)N; g.G = 1;
  g.K = F; g.A = feats; g.a_sm = F; g.a_mext = N; g.a_gext = 1;
  g.W = m->Wa1; g.w_rows = Hh; g.N = Hh; g.bias = m->ba1; g.act = ACT_GELU;
  g.out = rmap(hid, 0, Hh);
  OT_TRY(launch_gemm<T>(m, g, st, PK_GEMM_AUTOSPLIT));
  GemmDesc g2 = g;
  g2.K = Hh; g2.A = hid; g2.a_sm = Hh; g2.W = m->Wa2; g2.w_rows = L_NS * d; g2.N = L_NS * d;
  g2.bias = m->ba2; g2.act = ACT_NONE;
  g2.out = rmap(out, 0, (long long)L_NS * d);   // [N, L_NS, d]: token t = columns [t d, (t+1) d)
  return launch_gemm<T>(m, g2, st, PK_GEMM_AUTOSPLIT);
}

// Group-wise NS tokenizer: group g of every row through its own two-layer MLP
// (zero-padded to common widths F_max -> h_max -> d), token g = its output.
// Two grouped GEMMs: group g is the fixed coordinate that selects the weight
// set, the rows are tiled as samples; the hidden layer [N, G, h_max] lives in
// the workspace.
template <typename T>
static onetrans_status groupwise_impl(const onetrans_model* m, const void* feats, long long N, int F_max,
                                      int h_max, const void* W1, const void* b1, const void* W2, const void* b2,
                                      void* out, void* ws, size_t ws_bytes, cudaStream_t st, size_t* need) {
  const int G = m->L_NS, d = m->d, es = m->es;
  Carve cv(ws, ws_bytes);
  void* hid = cv.take((size_t)N * G * h_max * es);
  if (need) { *need = cv.used; return ONETRANS_OK; }
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;
  if (N == 0) return ONETRANS_OK;
  GemmDesc g = gdesc_base(m);
  g.mode = TILE_SAMPLES; g.M = (int)N; g.G = G; g.g_lo = 0; g.grp_base = 0;
  g.K = F_max; g.A = feats; g.a_sm = (long long)G * F_max; g.a_sg = F_max; g.a_mext = N; g.a_gext = G;
  g.W = W1; g.w_sg = (long long)h_max * F_max; g.w_rows = h_max; g.w_groups = G; g.n_lo = 0; g.N = h_max;
  g.bias = b1; g.bias_sg = h_max; g.act = ACT_GELU;
  g.out = rmap(hid, (long long)G * h_max, h_max);
  OT_TRY(launch_gemm<T>(m, g, st, PK_GEMM_AUTOSPLIT));
  GemmDesc g2 = g;
  g2.K = h_max; g2.A = hid; g2.a_sm = (long long)G * h_max; g2.a_sg = h_max;
  g2.W = W2; g2.w_sg = (long long)d * h_max; g2.w_rows = d; g2.N = d;
  g2.bias = b2; g2.bias_sg = d; g2.act = ACT_NONE;
  g2.out = rmap(out, (long long)G * d, d);   // [N, G, d]
  return launch_gemm<T>(m, g2, st, PK_GEMM_AUTOSPLIT);
}

// ============================================================== training ==
static long long pad64(long long r) { return (r + 63) / 64 * 64; }
// The backward pass of the stack with activation recomputation: the forward
// keeps only each layer's input; the backward recomputes a layer's
// intermediates from its input, then runs the chain rule in reverse order of
// the block.  Contractions run on the forward path's GEMM kernels: a GEMM
// over rows (dX = dY W) takes the transposed weights, a GEMM that reduces
// over rows (dW = dY^T X) takes both operands transposed (K-major), zero-
// padded to a multiple of 64 rows.
template <typename Ti, typename To>
static onetrans_status launch_transpose(const void* src, const RowSet& s, int G, int C, void* dst, int R_pad,
                                        cudaStream_t st, int Kc = 0) {
  if (G <= 0 || C <= 0 || R_pad <= 0) return ONETRANS_OK;
  const int kc = Kc > 0 ? Kc : R_pad;
  ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)G * C * ((double)s.R * sizeof(Ti) + (double)R_pad * sizeof(To)), st);
  const bool vec = C % 4 == 0 && s.st % 4 == 0 && s.sb % 4 == 0 && s.gs % 4 == 0 && R_pad % 64 == 0 &&
                   kc % 64 == 0 && (uintptr_t)src % 16 == 0 && (uintptr_t)dst % 16 == 0;
  if (vec)
    transpose_rows_kernel<Ti, To><<<dim3((unsigned)cdiv(C, 64), (unsigned)(R_pad / 64), (unsigned)G), 256, 0, st>>>(
        (const Ti*)src, s, C, (To*)dst, R_pad, kc);
  else
    transpose_rows_scalar_kernel<Ti, To><<<dim3((unsigned)cdiv(C, 32), (unsigned)cdiv(R_pad, 32), (unsigned)G), 256,
                                           0, st>>>((const Ti*)src, s, C, (To*)dst, R_pad, kc);
  return last_launch();
}

static onetrans_status launch_chunk_sum(const float* part, int chunks, long long n, float* out, long long out_stride,
                                        long long n_inner, cudaStream_t st) {
  if (n <= 0) return ONETRANS_OK;
  ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)n * (chunks + 1) * 4.0, st);
  if (chunks <= 32 && n % 4 == 0 && n_inner % 4 == 0 && out_stride % 4 == 0 && (uintptr_t)part % 16 == 0 &&
      (uintptr_t)out % 16 == 0)
    chunk_sum4_kernel<<<(unsigned)cdiv(n / 4, 256), 256, 0, st>>>(part, chunks, n, out, out_stride, n_inner);
  else if (chunks <= 64)
    chunk_sum_kernel<8><<<(unsigned)cdiv(n, 32), 256, 0, st>>>(part, chunks, n, out, out_stride, n_inner);
  else
    chunk_sum_kernel<32><<<(unsigned)cdiv(n, 32), 1024, 0, st>>>(part, chunks, n, out, out_stride, n_inner);
  return last_launch();
}

// CTAs of the row-parallel reductions that leave one partial row per CTA
// (gain and bias gradients): four per SM of a 148-SM part.
constexpr int kRedCtas = 4 * 148;

static bool vec4_ok(const void* p, size_t align, std::initializer_list<long long> strides) {
  if ((uintptr_t)p % align) return false;
  for (long long v : strides)
    if (v % 4) return false;
  return true;
}

// Column sums of G row sets (float32 or storage-type rows) into
// dst[g * dst_gs + c]: chunks of kColChunk rows in parallel into `part`
// (workspace), then the chunks added in order.
template <typename Ti>
static onetrans_status launch_colsum(const Ti* src, const RowSet& s, int G, int C, float* dst, long long dst_gs,
                                     float* part, cudaStream_t st) {
  if (G <= 0 || C <= 0) return ONETRANS_OK;
  const int chunks = (int)std::max<long long>(1, cdiv(s.R, kColChunk));
  {
    ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)G * C * (s.R * sizeof(Ti) + chunks * 4.0), st);
    if (C % 4 == 0 && vec4_ok(src, 4 * sizeof(Ti), {s.gs, s.sb, s.st}))
      colsum4_kernel<Ti><<<dim3((unsigned)cdiv(C, 128), (unsigned)G, (unsigned)chunks), 256, 0, st>>>(src, s, C,
                                                                                                      part);
    else
      colsum_kernel<Ti><<<dim3((unsigned)cdiv(C, 32), (unsigned)G, (unsigned)chunks), 256, 0, st>>>(src, s, C, part);
    OT_TRY(last_launch());
  }
  return launch_chunk_sum(part, chunks, (long long)G * C, dst, dst_gs, C, st);
}

// Row chunks of a weight-gradient GEMM: enough (weight tile, chunk) CTAs to
// fill one wave of 148 SMs (more chunks mean more partial gradients to add),
// chunks a multiple of 64 rows.
constexpr int kSplitCtas = 148;
static void split_rows(int R, int N_out, int K_in, int& chunks, int& Kc) {
  const int tiles = (int)(cdiv(N_out, 128) * cdiv(K_in, 256));
  const int want = std::max(1, std::min(kSplitCtas / std::max(tiles, 1), (int)(pad64(R) / 64)));
  Kc = (int)pad64(cdiv(R, want));
  chunks = (int)cdiv(R, Kc);
}

static RowSet rowset(long long gs, long long sb, long long st, int T, int R) {
  RowSet r;
  r.gs = gs; r.sb = sb; r.st = st; r.T = T; r.R = R;
  return r;
}

template <typename T>
static onetrans_status launch_cast(const float* src, void* dst, long long n, cudaStream_t st) {
  if (n <= 0) return ONETRANS_OK;
  ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)n * (4.0 + sizeof(T)), st);
  cast_kernel<T><<<(unsigned)cdiv(n, 256), 256, 0, st>>>(src, (T*)dst, n);
  return last_launch();
}

// Rows (b, t), t in [t_lo, t_hi) of a buffer with a_rows rows per sample: rows
// t < t_s use the shared S weights W_S [N, K], rows t >= t_s the set of NS
// token t - t_s of W_NS [L_NS, N, K].  A element (b, t, k) = A + b*a_samp +
// t*a_row + k; output rows through `out`; optional bias sets and residual.
// When the range is every row of densely stored samples, the shared-weight
// launch runs over all rows as one flat row set (whole 128-row tiles across
// sample boundaries, and one weight slice for the weight-resident kernel);
// the NS launch after it then rewrites the NS rows with their own weights.
// The output must not alias the residual or act_in rows.
template <typename T>
static onetrans_status mixed_rows_gemm(const onetrans_model* m, const void* A, long long a_row, long long a_samp,
                                       int a_rows, int B, int t_lo, int t_s, int t_hi, const void* W_S,
                                       const void* W_NS, int K, int N, RowMap out, cudaStream_t st,
                                       const void* bias_S = nullptr, const void* bias_NS = nullptr,
                                       RowMap res = RowMap{}, int act = ACT_NONE, RowMap act_in = RowMap{},
                                       RowMap act_out = RowMap{}, int w_mn = 0) {
  const bool flat = t_lo == 0 && t_hi == a_rows && a_samp == (long long)a_rows * a_row;
  if (t_s > t_lo && flat) {
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_FLAT; g.M = B * a_rows; g.fold = a_rows; g.G = 1;
    g.K = K; g.A = A; g.a_sm = a_row; g.a_mext = (long long)B * a_rows; g.a_gext = 1;
    g.W = W_S; g.w_rows = N; g.N = N; g.bias = bias_S; g.act = act; g.w_mn = w_mn;
    g.out = out; g.res = res; g.act_in = act_in; g.act_out = act_out;
    OT_TRY(launch_gemm<T>(m, g, st, PK_TRAIN));
  } else if (t_s > t_lo) {
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_ROWS; g.M = t_s - t_lo; g.m_lo = t_lo; g.G = B; g.g_lo = 0;
    g.K = K; g.A = A; g.a_sm = a_row; g.a_sg = a_samp; g.a_mext = a_rows; g.a_gext = B;
    g.W = W_S; g.w_rows = N; g.N = N; g.bias = bias_S; g.act = act; g.w_mn = w_mn;
    g.out = out; g.res = res; g.act_in = act_in; g.act_out = act_out;
    OT_TRY(launch_gemm<T>(m, g, st, PK_TRAIN));
  }
  if (t_hi > t_s) {
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_SAMPLES; g.M = B; g.G = t_hi - t_s; g.g_lo = t_s; g.grp_base = t_s;
    g.K = K; g.A = A; g.a_sm = a_samp; g.a_sg = a_row; g.a_mext = B; g.a_gext = a_rows;
    g.W = W_NS; g.w_sg = (long long)N * K; g.w_rows = N; g.w_groups = t_hi - t_s; g.N = N;
    g.bias = bias_NS; g.bias_sg = bias_NS ? N : 0; g.act = act; g.w_mn = w_mn;
    g.out = out; g.res = res; g.act_in = act_in; g.act_out = act_out;
    OT_TRY(launch_gemm<T>(m, g, st, PK_TRAIN));
  }
  return ONETRANS_OK;
}

// Weight gradient dW [N_out, K_in] = sum over a row set of dY^T X, the S set
// over all its rows and each NS set over its token's rows (one per sample).
// dY rows: src_y (float32) with y_cols columns starting at y_col0; X rows:
// src_x (storage type or float32) with x_cols columns.
struct GradRows {
  const void* p;     // element (b, t, c) = p + b*samp + t*row + c
  long long row, samp;
  bool f32;
};

// Scratch of the training step's reductions (workspace): the operand
// transposes, the row chunks' partial weight gradients, the column sums'
// partial sums.
struct TrainScratch {
  void *opA, *opW;
  float *split_part, *col_part;
};

// The same on the tensor cores straight from the row-major storage-type rows
// (no transposed copies): the S set's row tiles split into slices that fill
// one wave of CTAs, their partial gradients added in slice order; one slice
// per NS set.
static onetrans_status weight_grad_rows(GradRows Y, GradRows X, int N_out, int K_in, int B, int t_lo, int t_s,
                                        int t_hi, float* dW_S, float* dW_NS, const TrainScratch& sc,
                                        cudaStream_t st) {
  const int es = 2;
  const int tiles = (K_in / wgrad_pick_bn(K_in)) * (N_out / 128);
  if (t_s == t_lo && dW_S) OT_TRY(cuda_ok(cudaMemsetAsync(dW_S, 0, (size_t)N_out * K_in * 4, st)));
  if (t_s > t_lo && dW_S) {
    const int Tn = t_s - t_lo;
    WgradArgs wa;
    wa.TC = (int)cdiv(Tn, 64);
    wa.total = B * wa.TC;
    const int want = std::max(1, std::min(kSplitCtas / std::max(tiles, 1), wa.total));
    wa.per = (int)cdiv(wa.total, want);
    const int Z = (int)cdiv(wa.total, wa.per);
    CUtensorMap tY, tX, tO;
    float* out = Z > 1 ? sc.split_part : dW_S;
    int swx = 0;
    if (!wgrad_rows_tmap(&tY, (const char*)Y.p + (size_t)t_lo * Y.row * es, N_out, Tn, B, Y.row, Y.samp, wa.swap) ||
        !wgrad_rows_tmap(&tX, (const char*)X.p + (size_t)t_lo * X.row * es, K_in, Tn, B, X.row, X.samp, swx) ||
        swx != wa.swap || !wgrad_out_tmap(&tO, out, N_out, K_in, Z))
      return ONETRANS_ERR_CUDA;
    {
      ProfScope prof(PK_TRAIN, 2.0 * B * Tn * N_out * K_in, (double)B * Tn * (N_out + K_in) * es +
                     (double)Z * N_out * K_in * 4, st);
      OT_TRY(wgrad_launch(tY, tX, tO, N_out, K_in, Z, wa, st));
    }
    if (Z > 1) {
      const long long n = (long long)N_out * K_in;
      OT_TRY(launch_chunk_sum(sc.split_part, Z, n, dW_S, 0, n, st));
    }
  }
  if (t_hi > t_s && dW_NS) {
    const int G = t_hi - t_s;
    WgradArgs wa;
    wa.TC = (int)cdiv(B, 64);
    wa.per = wa.TC;
    wa.total = G * wa.TC;
    CUtensorMap tY, tX, tO;
    int swx = 0;
    if (!wgrad_rows_tmap(&tY, (const char*)Y.p + (size_t)t_s * Y.row * es, N_out, B, G, Y.samp, Y.row, wa.swap) ||
        !wgrad_rows_tmap(&tX, (const char*)X.p + (size_t)t_s * X.row * es, K_in, B, G, X.samp, X.row, swx) ||
        swx != wa.swap || !wgrad_out_tmap(&tO, dW_NS, N_out, K_in, G))
      return ONETRANS_ERR_CUDA;
    ProfScope prof(PK_TRAIN, 2.0 * B * G * N_out * K_in, (double)B * G * (N_out + K_in) * es +
                   (double)G * N_out * K_in * 4, st);
    OT_TRY(wgrad_launch(tY, tX, tO, N_out, K_in, G, wa, st));
  }
  return ONETRANS_OK;
}

template <typename T>
static onetrans_status weight_grad(const onetrans_model* m, GradRows Y, GradRows X, int N_out, int K_in, int B,
                                   int t_lo, int t_s, int t_hi, float* dW_S, float* dW_NS, const TrainScratch& sc,
                                   cudaStream_t st) {
  if (m->bf16 && g_policy == 0 && !Y.f32 && !X.f32 && wgrad_supported(N_out, K_in) && encode_fn() &&
      (uintptr_t)Y.p % 16 == 0 && (uintptr_t)X.p % 16 == 0 && Y.row % 8 == 0 && Y.samp % 8 == 0 &&
      X.row % 8 == 0 && X.samp % 8 == 0)
    return weight_grad_rows(Y, X, N_out, K_in, B, t_lo, t_s, t_hi, dW_S, dW_NS, sc, st);
  void *opA = sc.opA, *opW = sc.opW;
  const int es = m->es;
  auto transpose = [&](const GradRows& s, const RowSet& rs, int G, int C, void* dst, int R_pad, int Kc) {
    if (s.f32) return launch_transpose<float, T>(s.p, rs, G, C, dst, R_pad, st, Kc);
    return launch_transpose<T, T>(s.p, rs, G, C, dst, R_pad, st, Kc);
  };
  // a set with no rows (the S set of a layer that keeps only NS rows) has a zero gradient
  if (t_s == t_lo && dW_S) OT_TRY(cuda_ok(cudaMemsetAsync(dW_S, 0, (size_t)N_out * K_in * 4, st)));
  if (t_s > t_lo && dW_S) {
    // the reduction over rows is split into row chunks, each its own K-major
    // pair of operands: a grouped GEMM gives one partial gradient per chunk,
    // added in chunk order
    const int Tn = t_s - t_lo, R = B * Tn;
    int chunks, Kc;
    split_rows(R, N_out, K_in, chunks, Kc);
    const int Rp = chunks * Kc;
    const RowSet ry = rowset(0, Y.samp, Y.row, Tn, R), rx = rowset(0, X.samp, X.row, Tn, R);
    GradRows y0 = Y, x0 = X;
    y0.p = (const char*)Y.p + t_lo * Y.row * (Y.f32 ? 4 : es);
    x0.p = (const char*)X.p + t_lo * X.row * (X.f32 ? 4 : es);
    OT_TRY(transpose(y0, ry, 1, N_out, opA, Rp, Kc));
    OT_TRY(transpose(x0, rx, 1, K_in, opW, Rp, Kc));
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_SAMPLES; g.M = N_out; g.G = chunks; g.g_lo = 0; g.grp_base = 0;
    g.K = Kc; g.A = opA; g.a_sm = Kc; g.a_sg = (long long)N_out * Kc; g.a_mext = N_out; g.a_gext = chunks;
    g.W = opW; g.w_sg = (long long)K_in * Kc; g.w_rows = K_in; g.w_groups = chunks; g.N = K_in;
    float* out = chunks > 1 ? sc.split_part : dW_S;
    g.out = rmap32(out, K_in, (long long)N_out * K_in);
    OT_TRY(launch_gemm<T>(m, g, st, PK_TRAIN));
    if (chunks > 1) {
      const long long n = (long long)N_out * K_in;
      OT_TRY(launch_chunk_sum(sc.split_part, chunks, n, dW_S, 0, n, st));
    }
  }
  if (t_hi > t_s && dW_NS) {
    const int G = t_hi - t_s, Bp = (int)pad64(B);
    const RowSet ry = rowset(Y.row, Y.samp, 0, 1, B), rx = rowset(X.row, X.samp, 0, 1, B);
    GradRows y0 = Y, x0 = X;
    y0.p = (const char*)Y.p + t_s * Y.row * (Y.f32 ? 4 : es);
    x0.p = (const char*)X.p + t_s * X.row * (X.f32 ? 4 : es);
    OT_TRY(transpose(y0, ry, G, N_out, opA, Bp, Bp));
    OT_TRY(transpose(x0, rx, G, K_in, opW, Bp, Bp));
    GemmDesc g = gdesc_base(m);
    g.mode = TILE_SAMPLES; g.M = N_out; g.G = G; g.g_lo = 0; g.grp_base = 0;
    g.K = Bp; g.A = opA; g.a_sm = Bp; g.a_sg = (long long)N_out * Bp; g.a_mext = N_out; g.a_gext = G;
    g.W = opW; g.w_sg = (long long)K_in * Bp; g.w_rows = K_in; g.w_groups = G; g.N = K_in;
    g.out = rmap32(dW_NS, K_in, (long long)N_out * K_in);
    OT_TRY(launch_gemm<T>(m, g, st, PK_TRAIN));
  }
  return ONETRANS_OK;
}

// Bias gradient: column sums of rows (float32 or the storage type), the S set
// over all its rows and each NS set over its token's rows.
template <typename Ti>
static onetrans_status bias_grad(const Ti* rows, long long row, long long samp, int C, int B, int t_lo, int t_s,
                                 int t_hi, float* db_S, float* db_NS, float* part, cudaStream_t st) {
  if (t_s == t_lo && db_S) OT_TRY(cuda_ok(cudaMemsetAsync(db_S, 0, (size_t)C * 4, st)));
  if (t_s > t_lo && db_S)
    OT_TRY(launch_colsum(rows + t_lo * row, rowset(0, samp, row, t_s - t_lo, B * (t_s - t_lo)), 1, C, db_S, 0, part,
                         st));
  if (t_hi > t_s && db_NS)
    OT_TRY(launch_colsum(rows + t_s * row, rowset(row, samp, 0, 1, B), t_hi - t_s, C, db_NS, C, part, st));
  return ONETRANS_OK;
}

// RMSNorm backward of `rows` rows (`fold` per sample) into dx (dense
// [B][fold][d] rows): dx = (residual gradient: row t - r_off of `res`, 0 for
// t < r_off) + the norm's backward, with an optional storage-type copy of
// each finished row, and the gain gradient dg = sum over the rows of dy x r.
// Where d is a multiple of 128 up to 512 and the rows allow vector access
// one row kernel does it all (dg as one partial row per CTA, added in CTA
// order); else dx is filled from `res` first and the per-row products are
// column-summed.
template <typename T, typename Tx>
static onetrans_status launch_rms_backward(const void* x, long long x_sb, long long x_st, const void* gamma,
                                           const float* dy, const float* res, long long r_sb, long long r_st,
                                           int r_off, float* dx, float* pg, int rows, int fold, int d, float eps,
                                           void* dx_copy, float* dg, float* part, cudaStream_t st,
                                           float* db_s = nullptr, int s_rows = 0, bool* db_s_done = nullptr) {
  // db_s (optional): the column sums of the finished dx rows with t < s_rows,
  // taken in the fused row kernel only (*db_s_done tells the caller)
  if (db_s_done) *db_s_done = false;
  if (rows <= 0) return dg ? cuda_ok(cudaMemsetAsync(dg, 0, (size_t)d * 4, st)) : ONETRANS_OK;
  const long long dx_sb = (long long)fold * d, dx_st = d;
  const bool fused = d % 128 == 0 && d <= 512 && vec4_ok(x, 4 * sizeof(Tx), {x_sb, x_st}) &&
                     vec4_ok(dx, 16, {}) && vec4_ok(res, 16, {r_sb, r_st}) && vec4_ok(dy, 16, {}) &&
                     vec4_ok(gamma, 4 * sizeof(T), {}) && vec4_ok(dx_copy, 4 * sizeof(T), {});
  if (fused) {
    const int ctas = (int)std::min<long long>(cdiv(rows, 8), kRedCtas);
    float* part_s = db_s ? part + (size_t)kRedCtas * d : nullptr;
    {
      ProfScope prof(PK_TRAIN_ELEM, 0.0,
                     (double)rows * d * (sizeof(Tx) + 4.0 + 8.0 + (dx_copy ? sizeof(T) : 0)) + (double)ctas * d * 4,
                     st);
#define OT_RMS_DG(NC4)                                                                                             \
  rms_backward_dg_kernel<Tx, T, NC4><<<(unsigned)ctas, 256, 0, st>>>((const Tx*)x, x_sb, x_st, (const T*)gamma, dy, \
                                                                    res, r_sb, r_st, r_off, dx, dx_sb, dx_st, part, \
                                                                    rows, fold, eps, (T*)dx_copy, part_s, s_rows)
      switch (d / 128) {
        case 1: OT_RMS_DG(1); break;
        case 2: OT_RMS_DG(2); break;
        case 3: OT_RMS_DG(3); break;
        default: OT_RMS_DG(4); break;
      }
#undef OT_RMS_DG
      OT_TRY(last_launch());
    }
    OT_TRY(launch_chunk_sum(part, ctas, d, dg, 0, d, st));
    if (db_s) {
      OT_TRY(launch_chunk_sum(part_s, ctas, d, db_s, 0, d, st));
      if (db_s_done) *db_s_done = true;
    }
    return ONETRANS_OK;
  }
  // dx starts as the residual gradient
  OT_TRY(cuda_ok(cudaMemsetAsync(dx, 0, (size_t)rows * d * 4, st)));
  if (res && fold > r_off)
    OT_TRY(cuda_ok(cudaMemcpy2DAsync(dx + (size_t)r_off * d, (size_t)dx_sb * 4, res, (size_t)r_sb * 4,
                                     (size_t)(fold - r_off) * d * 4, rows / fold, cudaMemcpyDeviceToDevice, st)));
  {
    ProfScope prof(PK_TRAIN_ELEM, 0.0,
                   (double)rows * d * (sizeof(Tx) + 4.0 + 8.0 + 4.0 + (dx_copy ? sizeof(T) : 0)), st);
    rms_backward_kernel<Tx, T><<<(unsigned)cdiv(rows, 8), 256, 0, st>>>(
        (const Tx*)x, x_sb, x_st, (const T*)gamma, dy, dx, dx_sb, dx_st, pg, rows, fold, d, eps, (T*)dx_copy);
    OT_TRY(last_launch());
  }
  return launch_colsum(pg, rowset(0, (long long)fold * d, d, fold, rows), 1, d, dg, 0, part, st);
}

template <typename T>
static onetrans_status launch_attn_rows(const onetrans_model* m, int stage, const AttnRows& a, void* out,
                                        float* lse, const void* dout, float* Dr, void* dqkv, cudaStream_t st) {
  const int dh = m->dh;
  // visible (query, key) pairs x heads; FLOPs per pair: forward 2 x 2 d_h (q.k, p v), dq 3 x 2 d_h,
  // dk,dv 4 x 2 d_h; bytes: the q|k|v rows read once, the outputs written once
  const double pairs = (double)a.B * a.H * ((double)a.Lq * (a.L - a.Lq) + 0.5 * (double)a.Lq * (a.Lq + 1));
  const double fl = pairs * 2.0 * dh * (stage == 0 ? 2 : stage == 1 ? 3 : 4);
  ProfScope prof(PK_TRAIN_ATTN, fl, (double)a.B * a.L * 3 * a.d * m->es + (double)a.B * a.Lq * a.d * m->es, st);
#define OT_ATTN_ROWS(DH)                                                                                   \
  if (stage == 0) {                                                                                         \
    attn_rows_forward_kernel<T, DH><<<dim3((unsigned)cdiv(a.Lq, 64), a.H, a.B), 64, 0, st>>>(a, (T*)out, lse); \
  } else if (stage == 1) {                                                                                  \
    attn_rows_dq_kernel<T, DH><<<dim3((unsigned)cdiv(a.Lq, 64), a.H, a.B), 64, 0, st>>>(a, (const T*)dout,    \
                                                                                         (const T*)out, lse, Dr, \
                                                                                         (T*)dqkv);         \
  } else {                                                                                                  \
    attn_rows_dkdv_kernel<T, DH><<<dim3((unsigned)cdiv(a.L, 64), a.H, a.B), 64, 0, st>>>(a, (const T*)dout, lse, Dr, \
                                                                                         (T*)dqkv);         \
  }
  switch (dh) {
    case 16: OT_ATTN_ROWS(16) break;
    case 32: OT_ATTN_ROWS(32) break;
    case 64: OT_ATTN_ROWS(64) break;
    case 96: OT_ATTN_ROWS(96) break;
    case 128: OT_ATTN_ROWS(128) break;
    default: return ONETRANS_ERR_UNSUPPORTED;
  }
#undef OT_ATTN_ROWS
  return last_launch();
}

// Tensor-core attention of the training step (bf16, d_h = 64): stage 0 the
// forward with log-sum-exp, 1 dQ, 2 dK and dV.
static bool train_attn_tc(const onetrans_model* m) {
  return m->bf16 && g_policy == 0 && m->dh == TrainAttnCfg::DH && m->d % 64 == 0 && encode_fn() != nullptr;
}

static onetrans_status launch_attn_train_tc(const onetrans_model* m, int stage, const AttnRows& ar, void* o,
                                            float* lse, float* Dr, const void* dOb, void* dqkv, cudaStream_t st) {
  using C = TrainAttnCfg;
  const int d = ar.d;
  CUtensorMap tq, tdo;
  if (!make_tmap_3d(&tq, ar.qkv, 3 * (uint64_t)d, ar.L, ar.B, 3 * (uint64_t)d, (uint64_t)ar.L * 3 * d, 64, 128, 1))
    return ONETRANS_ERR_CUDA;
  if (stage > 0) {
    if (!make_tmap_3d(&tdo, dOb, d, ar.Lq, ar.B, d, (uint64_t)ar.Lq * d, 64, 128, 1)) return ONETRANS_ERR_CUDA;
  } else {
    tdo = tq;
  }
  TrainAttnArgs ta;
  std::memset(&ta, 0, sizeof(ta));
  ta.B = ar.B; ta.L = ar.L; ta.Lq = ar.Lq; ta.H = ar.H; ta.d = d;
  ta.lse = lse; ta.lse_out = lse; ta.Dr = Dr; ta.o = (__nv_bfloat16*)o; ta.dqkv = (__nv_bfloat16*)dqkv;
  const double pairs = (double)ar.B * ar.H * ((double)ar.Lq * (ar.L - ar.Lq) + 0.5 * (double)ar.Lq * (ar.Lq + 1));
  ProfScope prof(PK_TRAIN_ATTN, pairs * 2.0 * C::DH * (stage == 0 ? 2 : stage == 1 ? 3 : 4),
                 (double)ar.B * ar.L * 3 * d * 2 + (double)ar.B * ar.Lq * d * 2, st);
  static bool attr[3] = {false, false, false};
  if (!attr[stage]) {
    cudaError_t e = stage == 0 ? cudaFuncSetAttribute(attn_train_fwd_kernel,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)
                    : stage == 1 ? cudaFuncSetAttribute(attn_train_dq_kernel,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)
                                 : cudaFuncSetAttribute(attn_train_kv_kernel,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return ONETRANS_ERR_CUDA;
    attr[stage] = true;
  }
  if (stage == 0)
    attn_train_fwd_kernel<<<dim3((unsigned)cdiv(ar.Lq, C::BM), ar.H, ar.B), 192, C::SMEM, st>>>(tq, ta);
  else if (stage == 1)
    attn_train_dq_kernel<<<dim3((unsigned)cdiv(ar.Lq, C::BM), ar.H, ar.B), 192, C::SMEM, st>>>(tq, tdo, ta);
  else
    attn_train_kv_kernel<<<dim3((unsigned)cdiv(ar.L, C::BN), ar.H, ar.B), 192, C::SMEM, st>>>(tq, tdo, ta);
  return last_launch();
}

template <typename T>
static onetrans_status train_impl(const onetrans_model* m, const void* x0, int B, int L_S, const float* dy,
                                  float* out, float* dx0, const onetrans_grads* gr, void* ws, size_t ws_bytes,
                                  cudaStream_t st, size_t* need) {
  std::vector<int> Lq;
  OT_TRY(schedule_of(m, L_S, Lq));
  const int d = m->d, dff = m->dff, L_NS = m->L_NS, NL = m->NL, es = m->es, H = m->H;
  const int L0 = L_S + L_NS;
  std::vector<int> Ln(NL);  // input rows of each layer
  Ln[0] = L0;
  for (int n = 1; n < NL; ++n) Ln[n] = Lq[n - 1];
  const int Lq0 = Lq[0];
  const long long Mmax = pad64((long long)B * L0) + 64LL * kSplitCtas;   // row chunks pad each to 64 rows
  const long long op_elems = std::max<long long>(Mmax, (long long)L_NS * pad64(B)) * std::max(3 * d, dff);
  const long long split_elems = (long long)kSplitCtas * 128 * 256;      // chunks x N_out x K_in, at most
  const long long col_elems = std::max<long long>(cdiv((long long)B * L0, kColChunk) + cdiv(B, kColChunk) * L_NS,
                                                  kRedCtas) * std::max(3 * d, dff);
  const long long wt_elems = (long long)(1 + L_NS) * std::max(3 * d, dff) * d;
  Carve cv(ws, ws_bytes);
  std::vector<float*> X(NL, nullptr);   // float32 inputs of layers 1 .. NL-1
  for (int n = 1; n < NL; ++n) X[n] = (float*)cv.take((size_t)B * Ln[n] * d * 4);
  void* h = cv.take((size_t)B * L0 * d * es);
  void* qkv = cv.take((size_t)B * L0 * 3 * d * es);
  // each layer's attention output and log-sum-exp, kept from the forward
  std::vector<void*> Aout(NL);
  std::vector<float*> LSE(NL);
  for (int n = 0; n < NL; ++n) {
    Aout[n] = cv.take((size_t)B * Lq[n] * d * es);
    LSE[n] = (float*)cv.take((size_t)B * H * Lq[n] * 4);
  }
  float* Dr = (float*)cv.take((size_t)B * H * Lq0 * 4);
  float* x1 = (float*)cv.take((size_t)B * Lq0 * d * 4);
  void* h2 = cv.take((size_t)B * Lq0 * d * es);
  void* u = cv.take((size_t)B * Lq0 * dff * es);   // W1 h2 + b1, recomputed for the backward only
  void* z = cv.take((size_t)B * Lq0 * dff * es);
  float* gbuf[2] = {(float*)cv.take((size_t)B * L0 * d * 4), (float*)cv.take((size_t)B * L0 * d * 4)};
  void* gT = cv.take((size_t)B * L0 * d * es);      // the current output gradient in the storage type
  float* dx1 = (float*)cv.take((size_t)B * Lq0 * d * 4);
  void* dx1T = cv.take((size_t)B * Lq0 * d * es);
  float* dz = (float*)cv.take((size_t)B * Lq0 * dff * 4);
  void* du = cv.take((size_t)B * Lq0 * dff * es);
  float* dh2 = (float*)cv.take((size_t)B * Lq0 * d * 4);
  void* dqkv = cv.take((size_t)B * L0 * 3 * d * es);
  float* dh = (float*)cv.take((size_t)B * L0 * d * 4);
  float* pg = (float*)cv.take((size_t)B * L0 * d * 4);
  void* opA = cv.take((size_t)op_elems * es);
  void* opW = cv.take((size_t)op_elems * es);
  void* wT = cv.take((size_t)wt_elems * es);
  void* dOb = cv.take((size_t)B * Lq0 * d * es);   // the attention output's gradient in the storage type
  float* split_part = (float*)cv.take((size_t)split_elems * 4);
  float* col_part = (float*)cv.take((size_t)col_elems * 4);
  if (need) { *need = cv.used; return ONETRANS_OK; }
  TrainScratch sc;
  sc.opA = opA; sc.opW = opW; sc.split_part = split_part; sc.col_part = col_part;
  const bool tc_attn = train_attn_tc(m);
  if (cv.overflow) return ONETRANS_ERR_CAPACITY;

  // transposed weights of one layer's S set and NS sets: [N_out, K_in] -> [K_in, N_out]
  auto weights_T = [&](const void* W_S, const void* W_NS, int N_out, int K_in, void*& S_T, void*& NS_T) {
    S_T = wT;
    NS_T = (char*)wT + (size_t)N_out * K_in * es;
    OT_TRY((launch_transpose<T, T>(W_S, rowset(0, 0, K_in, N_out, N_out), 1, K_in, S_T, N_out, st)));
    if (W_NS)
      OT_TRY((launch_transpose<T, T>(W_NS, rowset((long long)N_out * K_in, 0, K_in, N_out, N_out), L_NS, K_in, NS_T,
                                    N_out, st)));
    return ONETRANS_OK;
  };

  // dX = dY W over a mixed row set (rows t < t_s use W_S, the others their NS
  // token's set of W_NS; W [N_out = K][K_in = N] as the forward stores it):
  // the tensor-core GEMMs read W as an MN-major operand; kernels that do not
  // take one get the weights transposed
  auto dx_gemm = [&](const void* A, long long a_row, long long a_samp, int rows, int t_s, const void* W_S,
                     const void* W_NS, int K, int N, RowMap out, int act = ACT_NONE, RowMap act_in = RowMap{},
                     RowMap act_out = RowMap{}) -> onetrans_status {
    const onetrans_status r = mixed_rows_gemm<T>(m, A, a_row, a_samp, rows, B, 0, t_s, rows, W_S, W_NS, K, N, out, st,
                                                 nullptr, nullptr, RowMap{}, act, act_in, act_out, 1);
    if (r != ONETRANS_ERR_UNSUPPORTED) return r;
    void *wS, *wNS;
    OT_TRY(weights_T(W_S, W_NS, K, N, wS, wNS));
    return mixed_rows_gemm<T>(m, A, a_row, a_samp, rows, B, 0, t_s, rows, wS, W_NS ? wNS : nullptr, K, N, out, st,
                              nullptr, nullptr, RowMap{}, act, act_in, act_out, 0);
  };

  // layer n's intermediates from its input x_in (L rows per sample).  The
  // forward pass computes the attention output and its log-sum-exp, kept
  // for the backward, and z = GELU(W1 h2 + b1); the backward recomputes the
  // rest (h, q | k | v, x1, h2 and the pre-activation u; z then comes out of
  // the GELU backward).
  auto recompute = [&](int n, const void* x_in, bool x_f32, bool fwd) -> onetrans_status {
    const int L = Ln[n], Lqn = Lq[n], s = L - L_NS, sq = Lqn - L_NS, off = L - Lqn;
    void* a = Aout[n];
    if (x_f32) OT_TRY(rms_flat<T>(m, x_in, true, h, (long long)B * L, m->g_attn[n], st));
    else OT_TRY(rms_flat<T>(m, x_in, false, h, (long long)B * L, m->g_attn[n], st));
    // q | k | v of every row (q unscaled)
    OT_TRY(mixed_rows_gemm<T>(m, h, d, (long long)L * d, L, B, 0, s, L, m->Wqkv_S[n], m->Wqkv_NS[n], d, 3 * d,
                              rmap(qkv, (long long)L * 3 * d, 3 * d), st));
    if (fwd) {
      AttnRows ar;
      ar.qkv = qkv; ar.B = B; ar.L = L; ar.Lq = Lqn; ar.H = H; ar.d = d;
      if (tc_attn) OT_TRY(launch_attn_train_tc(m, 0, ar, a, LSE[n], nullptr, nullptr, nullptr, st));
      else OT_TRY(launch_attn_rows<T>(m, 0, ar, a, LSE[n], nullptr, nullptr, nullptr, st));
    }
    // x1 = x[tail] + W^O a, h2 = RMSNorm(x1)
    GemmDesc go = gdesc_base(m);
    go.mode = TILE_FLAT; go.M = B * Lqn; go.fold = Lqn; go.G = 1;
    go.K = d; go.A = a; go.a_sm = d; go.a_mext = (long long)B * Lqn; go.a_gext = 1;
    go.W = m->Wo[n]; go.w_rows = d; go.N = d;
    go.res = x_f32 ? rmap32(eoff(x_in, (long long)off * d, 4), (long long)L * d, d)
                   : rmap(eoff(x_in, (long long)off * d, es), (long long)L * d, d);
    go.out = rmap32(x1, (long long)Lqn * d, d);
    go.rms = rmap(h2, (long long)Lqn * d, d);
    go.gamma = m->g_ffn[n];
    OT_TRY(launch_gemm<T>(m, go, st, PK_TRAIN));
    return mixed_rows_gemm<T>(m, h2, d, (long long)Lqn * d, Lqn, B, 0, sq, Lqn, m->W1_S[n], m->W1_NS[n], d, dff,
                              rmap(fwd ? z : u, (long long)Lqn * dff, dff), st, m->b1_S[n], m->b1_NS[n], RowMap{},
                              fwd ? ACT_GELU : ACT_NONE);
  };

  // ---- forward, keeping each layer's input
  for (int n = 0; n < NL; ++n) {
    const int Lqn = Lq[n], sq = Lqn - L_NS;
    OT_TRY(recompute(n, n == 0 ? x0 : (const void*)X[n], n > 0, true));
    float* y = n + 1 == NL ? out : X[n + 1];
    OT_TRY(mixed_rows_gemm<T>(m, z, dff, (long long)Lqn * dff, Lqn, B, 0, sq, Lqn, m->W2_S[n], m->W2_NS[n], dff, d,
                              rmap32(y, (long long)Lqn * d, d), st, m->b2_S[n], m->b2_NS[n],
                              rmap32(x1, (long long)Lqn * d, d)));
  }

  // ---- backward, layer by layer; the gradient of each layer's output is
  // kept in float32 (g_cur, for the residual and the bias sums) and in the
  // storage type (gT, the GEMM operand)
  const float* g_cur = dy;   // gradient of layer n's output, [B, Lq[n], d]
  bool b2s_done = false;     // db2 of the shared set of layer n already summed by the layer above
  OT_TRY(launch_cast<T>(dy, gT, (long long)B * Lq[NL - 1] * d, st));
  for (int n = NL - 1; n >= 0; --n) {
    const int L = Ln[n], Lqn = Lq[n], s = L - L_NS, sq = Lqn - L_NS, off = L - Lqn;
    void* a = Aout[n];
    float* lse = LSE[n];
    const bool x_f32 = n > 0;
    const void* x_in = n == 0 ? x0 : (const void*)X[n];
    float* g_in = n == 0 ? dx0 : gbuf[n % 2];   // gradient of layer n's input, [B, L, d]
    OT_TRY(recompute(n, x_in, x_f32, false));
    const long long Md = (long long)Lqn * d, Mf = (long long)Lqn * dff;
    // y = x1 + W2 z + b2
    OT_TRY(bias_grad(g_cur, d, Md, d, B, 0, sq, Lqn, b2s_done ? nullptr : gr->b2_S[n], gr->b2_NS[n], col_part, st));
    // z = GELU(u), u = W1 h2 + b1: the dz GEMM's epilogue applies the GELU
    // backward where the weight-resident kernel takes the shape (du and z
    // in the storage type, dz never stored); otherwise dz in float32 and a
    // GELU-backward pass that also sums the S rows' du
    const onetrans_status fz =
        m->bf16 && g_policy == 0
            ? dx_gemm(gT, d, Md, Lqn, sq, m->W2_S[n], m->W2_NS[n], d, dff, rmap(du, Mf, dff), ACT_GELU_BWD,
                      rmap(u, Mf, dff), rmap(z, Mf, dff))
            : ONETRANS_ERR_UNSUPPORTED;
    if (fz != ONETRANS_OK && fz != ONETRANS_ERR_UNSUPPORTED) return fz;
    const bool gelu_in_gemm = fz == ONETRANS_OK;
    bool gelu_fused = false;
    if (!gelu_in_gemm) {
      OT_TRY(dx_gemm(gT, d, Md, Lqn, sq, m->W2_S[n], m->W2_NS[n], d, dff, rmap32(dz, Mf, dff)));
      const long long nz = (long long)B * Mf;
      const int rows = B * Lqn;
      gelu_fused = gr->b1_S[n] && dff % 4 == 0 && dff <= 4096;
      if (gelu_fused) {
        // du, z and the S rows' column sums of du (db1 of the shared set) in one pass
        const int ctas0 = (int)std::min<long long>(cdiv(rows, 8), kRedCtas);
        const int rows_per = (int)cdiv(rows, ctas0), ctas = (int)cdiv(rows, rows_per);
        {
          ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)nz * (4.0 + 3.0 * es) + (double)ctas * dff * 4, st);
#define OT_GELU_B(J)                                                                                        \
  gelu_backward_bias_kernel<T, J><<<(unsigned)ctas, 256, 0, st>>>(dz, (const T*)u, (T*)du, (T*)z, rows, Lqn, sq, \
                                                                   dff, rows_per, col_part)
          switch ((dff + 1023) / 1024) {
            case 1: OT_GELU_B(1); break;
            case 2: OT_GELU_B(2); break;
            case 3: OT_GELU_B(3); break;
            default: OT_GELU_B(4); break;
          }
#undef OT_GELU_B
          OT_TRY(last_launch());
        }
        OT_TRY(launch_chunk_sum(col_part, ctas, dff, gr->b1_S[n], 0, dff, st));
      } else {
        ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)nz * (4.0 + 3.0 * es), st);
        gelu_backward_kernel<T><<<(unsigned)cdiv(nz, 1024), 256, 0, st>>>(dz, (const T*)u, (T*)du, (T*)z, nz);
        OT_TRY(last_launch());
      }
    }
    OT_TRY(weight_grad<T>(m, GradRows{gT, d, Md, false}, GradRows{z, dff, Mf, false}, d, dff, B, 0, sq, Lqn,
                          gr->W2_S[n], gr->W2_NS[n], sc, st));
    OT_TRY(bias_grad((const T*)du, dff, Mf, dff, B, 0, sq, Lqn, gelu_fused ? nullptr : gr->b1_S[n], gr->b1_NS[n],
                     col_part, st));
    OT_TRY(weight_grad<T>(m, GradRows{du, dff, Mf, false}, GradRows{h2, d, Md, false}, dff, d, B, 0, sq, Lqn,
                          gr->W1_S[n], gr->W1_NS[n], sc, st));
    OT_TRY(dx_gemm(du, dff, Mf, Lqn, sq, m->W1_S[n], m->W1_NS[n], dff, d, rmap32(dh2, Md, d)));
    // h2 = RMSNorm(x1; g_ffn), x1 = x[tail] + W^O a; y's gradient reaches x1 around the FFN
    OT_TRY((launch_rms_backward<T, float>(x1, Md, d, m->g_ffn[n], dh2, g_cur, Md, d, 0, dx1, pg, B * Lqn, Lqn, d,
                                         m->cfg.rms_eps, dx1T, gr->g_ffn[n], col_part, st)));
    OT_TRY(weight_grad<T>(m, GradRows{dx1T, d, Md, false}, GradRows{a, d, Md, false}, d, d, B, 0, Lqn, Lqn,
                          gr->Wo[n], nullptr, sc, st));
    OT_TRY(dx_gemm(dx1T, d, Md, Lqn, Lqn, m->Wo[n], nullptr, d, d, rmap(dOb, Md, d)));
    // attention: dq, dk, dv of the recomputed rows
    OT_TRY(cuda_ok(cudaMemsetAsync(dqkv, 0, (size_t)B * L * 3 * d * es, st)));
    AttnRows ar;
    ar.qkv = qkv; ar.B = B; ar.L = L; ar.Lq = Lqn; ar.H = H; ar.d = d;
    if (tc_attn) {
      {
        ProfScope prof(PK_TRAIN_ELEM, 0.0, (double)B * Lqn * d * 4.0 + (double)B * Lqn * H * 4.0, st);
        attn_train_delta_kernel<<<(unsigned)cdiv((long long)B * Lqn, 8), 256, 0, st>>>(
            (const __nv_bfloat16*)dOb, (const __nv_bfloat16*)a, Dr, B, Lqn, H);
      }
      OT_TRY(last_launch());
      OT_TRY(launch_attn_train_tc(m, 1, ar, a, lse, Dr, dOb, dqkv, st));
      OT_TRY(launch_attn_train_tc(m, 2, ar, a, lse, Dr, dOb, dqkv, st));
    } else {
      OT_TRY(launch_attn_rows<T>(m, 1, ar, a, lse, dOb, Dr, dqkv, st));
      OT_TRY(launch_attn_rows<T>(m, 2, ar, a, lse, dOb, Dr, dqkv, st));
    }
    // (q, k, v) = W_i^{QKV} h_i
    const long long Mq = (long long)L * 3 * d;
    OT_TRY(weight_grad<T>(m, GradRows{dqkv, 3 * d, Mq, false}, GradRows{h, d, (long long)L * d, false}, 3 * d, d,
                          B, 0, s, L, gr->Wqkv_S[n], gr->Wqkv_NS[n], sc, st));
    OT_TRY(dx_gemm(dqkv, 3 * d, Mq, L, s, m->Wqkv_S[n], m->Wqkv_NS[n], 3 * d, d, rmap32(dh, (long long)L * d, d)));
    // h = RMSNorm(x; g_attn); x1's gradient reaches the tail rows of x around
    // the attention; the lower layer's output gradient also as its GEMM operand
    void* g_copy = n > 0 ? gT : nullptr;
    // the lower layer's db2 (shared set: its S rows t < L - L_NS) from the same pass
    float* db2_below = n > 0 ? gr->b2_S[n - 1] : nullptr;
    if (x_f32)
      OT_TRY((launch_rms_backward<T, float>(x_in, (long long)L * d, d, m->g_attn[n], dh, dx1, Md, d, off, g_in, pg,
                                           B * L, L, d, m->cfg.rms_eps, g_copy, gr->g_attn[n], col_part, st,
                                           db2_below, L - L_NS, &b2s_done)));
    else
      OT_TRY((launch_rms_backward<T, T>(x_in, (long long)L * d, d, m->g_attn[n], dh, dx1, Md, d, off, g_in, pg,
                                       B * L, L, d, m->cfg.rms_eps, g_copy, gr->g_attn[n], col_part, st)));
    g_cur = g_in;
  }
  return ONETRANS_OK;
}

// Failure path of the bounded waits, without a fault: one thread waits on an
// mbarrier that nothing arrives at, with the same wait the tensor-core
// kernels use but limited to `limit` rounds; the wait gives up, records
// kErrWaitTimeout in the device status word, and the kernel returns.
__global__ void selftest_wait_kernel(uint32_t limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limited(&bar, 0, limit);
}

// ============================================================== C ABI ====
extern "C" {

int32_t onetrans_version(void) { return 100; }

const char* onetrans_status_string(int32_t s) {
  switch (s) {
    case ONETRANS_OK: return "ok";
    case ONETRANS_ERR_INVALID_ARG: return "invalid argument";
    case ONETRANS_ERR_SHAPE: return "shape mismatch";
    case ONETRANS_ERR_UNSUPPORTED: return "unsupported";
    case ONETRANS_ERR_CAPACITY: return "capacity exceeded";
    case ONETRANS_ERR_CUDA: return "CUDA error";
    case ONETRANS_ERR_DEVICE_CHECK: return "device-side check failed";
    default: return "unknown status";
  }
}

onetrans_status onetrans_set_kernel_policy(int32_t policy) {
  if (policy < 0 || policy > 1) return ONETRANS_ERR_INVALID_ARG;
  g_policy = policy;
  return ONETRANS_OK;
}

onetrans_status onetrans_model_create(const onetrans_config* cfg, const onetrans_weights* w,
                                      onetrans_model** out) {
  if (!cfg || !w || !out) return ONETRANS_ERR_INVALID_ARG;
  *out = nullptr;
  const int NL = cfg->n_layers, d = cfg->d_model, H = cfg->n_heads;
  if (NL < 1 || NL > 64 || d < 1 || H < 1 || cfg->d_ff < 1 || cfg->L_NS < 1 || cfg->L_NS > 256)
    return ONETRANS_ERR_SHAPE;
  if (d % H) return ONETRANS_ERR_SHAPE;
  const int dh = d / H;
  if (dh != 16 && dh != 32 && dh != 64 && dh != 96 && dh != 128) return ONETRANS_ERR_UNSUPPORTED;
  if (cfg->mode != ONETRANS_BF16 && cfg->mode != ONETRANS_FP32) return ONETRANS_ERR_INVALID_ARG;
  if (cfg->page_tokens != 64) return ONETRANS_ERR_UNSUPPORTED;
  if (!(cfg->rms_eps > 0.f)) return ONETRANS_ERR_INVALID_ARG;
  if (cfg->n_behaviors < 0 || cfg->n_behaviors > 8 || cfg->event_dim < 0 || cfg->ns_feat_dim < 0 ||
      cfg->ns_hidden < 0)
    return ONETRANS_ERR_SHAPE;
  if (cfg->event_dim > 4096) return ONETRANS_ERR_UNSUPPORTED;
  const void* const* per_layer[] = {w->g_attn, w->g_ffn, w->Wqkv_S, w->Wqkv_NS, w->Wo, w->W1_S, w->b1_S,
                                    w->W2_S, w->b2_S, w->W1_NS, w->b1_NS, w->W2_NS, w->b2_NS};
  for (auto arr : per_layer) {
    if (!arr) return ONETRANS_ERR_INVALID_ARG;
    for (int l = 0; l < NL; ++l)
      if (!arr[l] || !aligned(arr[l], 16)) return ONETRANS_ERR_INVALID_ARG;
  }
  if ((w->w_head != nullptr) != (w->b_head != nullptr) || (w->w_head && !aligned(w->w_head, 16)))
    return ONETRANS_ERR_INVALID_ARG;
  std::vector<int> pyr;
  if (cfg->pyramid_q) {
    for (int l = 0; l < NL; ++l) {
      const int q = cfg->pyramid_q[l];
      if (q < cfg->L_NS || (l > 0 && q > pyr.back())) return ONETRANS_ERR_SHAPE;
      pyr.push_back(q);
    }
  }
  onetrans_model* m = new (std::nothrow) onetrans_model();
  if (!m) return ONETRANS_ERR_CAPACITY;
  m->cfg = *cfg;
  m->cfg.pyramid_q = nullptr;
  m->pyr = pyr;
  m->d = d; m->H = H; m->dh = dh; m->dff = cfg->d_ff; m->L_NS = cfg->L_NS; m->NL = NL;
  m->bf16 = cfg->mode == ONETRANS_BF16;
  m->es = m->bf16 ? 2 : 4;
  auto cp = [NL](const void* const* a) { return std::vector<const void*>(a, a + NL); };
  m->g_attn = cp(w->g_attn); m->g_ffn = cp(w->g_ffn); m->Wqkv_S = cp(w->Wqkv_S);
  m->Wqkv_NS = cp(w->Wqkv_NS); m->Wo = cp(w->Wo); m->W1_S = cp(w->W1_S); m->b1_S = cp(w->b1_S);
  m->W2_S = cp(w->W2_S); m->b2_S = cp(w->b2_S); m->W1_NS = cp(w->W1_NS); m->b1_NS = cp(w->b1_NS);
  m->W2_NS = cp(w->W2_NS); m->b2_NS = cp(w->b2_NS);
  m->Wa1 = w->Wa1; m->ba1 = w->ba1; m->Wa2 = w->Wa2; m->ba2 = w->ba2; m->type_emb = w->type_emb;
  m->w_head = w->w_head; m->b_head = w->b_head;
  const int nb = cfg->n_behaviors;
  if (nb > 0 && w->Wb1 && w->bb1 && w->Wb2 && w->bb2) {
    m->Wb1.assign(w->Wb1, w->Wb1 + nb); m->bb1.assign(w->bb1, w->bb1 + nb);
    m->Wb2.assign(w->Wb2, w->Wb2 + nb); m->bb2.assign(w->bb2, w->bb2 + nb);
  }
  *out = m;
  return ONETRANS_OK;
}

onetrans_status onetrans_model_destroy(onetrans_model* m) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  delete m;
  return ONETRANS_OK;
}

onetrans_status onetrans_schedule(const onetrans_model* m, int32_t L_S, int32_t* out) {
  if (!m || !out) return ONETRANS_ERR_INVALID_ARG;
  std::vector<int> Lq;
  OT_TRY(schedule_of(m, L_S, Lq));
  std::copy(Lq.begin(), Lq.end(), out);
  return ONETRANS_OK;
}

onetrans_status onetrans_workspace_size(const onetrans_model* m, int32_t op, int64_t n, int32_t L,
                                        size_t* bytes) {
  if (!m || !bytes) return ONETRANS_ERR_INVALID_ARG;
  if (n < 0 || n > (1LL << 31) - 1 || L < 0) return ONETRANS_ERR_SHAPE;
  *bytes = 0;
  const int nn = (int)n;
  switch (op) {
    case ONETRANS_OP_FORWARD:
      return m->bf16 ? forward_impl<__nv_bfloat16>(m, nullptr, nn, L, nullptr, nullptr, 0, 0, bytes)
                     : forward_impl<float>(m, nullptr, nn, L, nullptr, nullptr, 0, 0, bytes);
    case ONETRANS_OP_STAGE1:
      return m->bf16 ? stage1_impl<__nv_bfloat16>(m, nullptr, nullptr, nn, nullptr, L, nullptr, 0, 0, bytes)
                     : stage1_impl<float>(m, nullptr, nullptr, nn, nullptr, L, nullptr, 0, 0, bytes);
    case ONETRANS_OP_STAGE2:
      return m->bf16 ? stage2_impl<__nv_bfloat16>(m, nullptr, nullptr, 1, nullptr, nullptr, nullptr, nullptr,
                                                  nullptr, 0, 0, bytes, n, L)
                     : stage2_impl<float>(m, nullptr, nullptr, 1, nullptr, nullptr, nullptr, nullptr, nullptr, 0,
                                          0, bytes, n, L);
    case ONETRANS_OP_APPEND:
      return m->bf16 ? append_impl<__nv_bfloat16>(m, nullptr, nullptr, nn, nullptr, nullptr, L, nullptr, 0, 0,
                                                  bytes)
                     : append_impl<float>(m, nullptr, nullptr, nn, nullptr, nullptr, L, nullptr, 0, 0, bytes);
    case ONETRANS_OP_AUTOSPLIT:
      return m->bf16 ? autosplit_impl<__nv_bfloat16>(m, nullptr, n, nullptr, nullptr, 0, 0, bytes)
                     : autosplit_impl<float>(m, nullptr, n, nullptr, nullptr, 0, 0, bytes);
    case ONETRANS_OP_TRAIN:
      return m->bf16 ? train_impl<__nv_bfloat16>(m, nullptr, nn, L, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0,
                                                 bytes)
                     : train_impl<float>(m, nullptr, nn, L, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0, bytes);
    case ONETRANS_OP_GROUPWISE:
      if (L < 1) return ONETRANS_ERR_SHAPE;
      return m->bf16 ? groupwise_impl<__nv_bfloat16>(m, nullptr, n, 1, L, nullptr, nullptr, nullptr, nullptr,
                                                     nullptr, nullptr, 0, 0, bytes)
                     : groupwise_impl<float>(m, nullptr, n, 1, L, nullptr, nullptr, nullptr, nullptr, nullptr,
                                             nullptr, 0, 0, bytes);
    default:
      return ONETRANS_ERR_INVALID_ARG;
  }
}

// ---------------------------------------------------------------- cache --
static void cache_layout(const onetrans_model* m, int n_slots, int max_L_S, int& max_pages, long long& n_pages,
                         size_t& table_bytes, size_t& page_bytes) {
  const int P = m->cfg.page_tokens;
  std::vector<int> s, sq;
  long long per_slot = 0;
  max_pages = (int)cdiv(max_L_S, P);
  if (s_rows_of(m, max_L_S, s, sq) == ONETRANS_OK) {
    for (int n = 0; n < m->NL; ++n) per_slot += cdiv(s[n], P);
  } else {
    per_slot = (long long)m->NL * max_pages;  // no valid schedule at this length: worst case
  }
  n_pages = per_slot * n_slots;
  table_bytes = (((size_t)n_slots * m->NL * max_pages * sizeof(int)) + 255) & ~(size_t)255;
  page_bytes = (size_t)2 * m->d * P * m->es;
}

onetrans_status onetrans_cache_size(const onetrans_model* m, int32_t n_slots, int32_t max_L_S, size_t* bytes) {
  if (!m || !bytes) return ONETRANS_ERR_INVALID_ARG;
  if (n_slots < 1 || max_L_S < 1) return ONETRANS_ERR_SHAPE;
  int max_pages;
  long long n_pages;
  size_t tb, pb;
  cache_layout(m, n_slots, max_L_S, max_pages, n_pages, tb, pb);
  *bytes = tb + (size_t)n_pages * pb;
  return ONETRANS_OK;
}

onetrans_status onetrans_cache_init(const onetrans_model* m, void* pool, size_t bytes, int32_t n_slots,
                                    int32_t max_L_S, onetrans_cache** out) {
  if (!m || !pool || !out) return ONETRANS_ERR_INVALID_ARG;
  *out = nullptr;
  if (!aligned(pool, 256)) return ONETRANS_ERR_INVALID_ARG;
  if (n_slots < 1 || max_L_S < 1) return ONETRANS_ERR_SHAPE;
  int max_pages;
  long long n_pages;
  size_t tb, pb;
  cache_layout(m, n_slots, max_L_S, max_pages, n_pages, tb, pb);
  if (tb + (size_t)n_pages * pb > bytes) return ONETRANS_ERR_CAPACITY;
  onetrans_cache* c = new (std::nothrow) onetrans_cache();
  if (!c) return ONETRANS_ERR_CAPACITY;
  c->m = m; c->pool = (char*)pool; c->bytes = bytes; c->n_slots = n_slots; c->max_L_S = max_L_S;
  c->max_pages = max_pages; c->n_pages = (int)n_pages;
  c->d_table = (int*)pool;
  c->d_pages = (char*)pool + tb;
  c->h_table.assign((size_t)n_slots * m->NL * max_pages, -1);
  c->len.assign(n_slots, 0);
  c->free_pages.resize(n_pages);
  for (long long i = 0; i < n_pages; ++i) c->free_pages[i] = (int)(n_pages - 1 - i);
  *out = c;
  return ONETRANS_OK;
}

onetrans_status onetrans_cache_destroy(onetrans_cache* c) {
  if (!c) return ONETRANS_ERR_INVALID_ARG;
  delete c;
  return ONETRANS_OK;
}

onetrans_status onetrans_cache_length(const onetrans_cache* c, int32_t slot, int32_t* len) {
  if (!c || !len) return ONETRANS_ERR_INVALID_ARG;
  if (slot < 0 || slot >= c->n_slots) return ONETRANS_ERR_SHAPE;
  *len = c->len[slot];
  return ONETRANS_OK;
}

onetrans_status onetrans_cache_row_ptr(const onetrans_cache* c, int32_t slot, int32_t layer, int32_t kind,
                                       int32_t head, int32_t token, void** ptr) {
  if (!c || !ptr) return ONETRANS_ERR_INVALID_ARG;
  const onetrans_model* m = c->m;
  if (slot < 0 || slot >= c->n_slots || layer < 0 || layer >= m->NL || kind < 0 || kind > 1 || head < 0 ||
      head >= m->H || token < 0 || token / m->cfg.page_tokens >= c->max_pages)
    return ONETRANS_ERR_SHAPE;
  const int P = m->cfg.page_tokens;
  const int page = c->h_table[((size_t)slot * m->NL + layer) * c->max_pages + token / P];
  if (page < 0) return ONETRANS_ERR_SHAPE;
  const size_t el = (size_t)page * 2 * m->d * P + ((size_t)(kind * m->H + head) * P + token % P) * m->dh;
  *ptr = c->d_pages + el * m->es;
  return ONETRANS_OK;
}

// ---------------------------------------------------------- entry points --
static onetrans_status check_ws(void* ws) {
  return (ws && aligned(ws, 256)) ? ONETRANS_OK : ONETRANS_ERR_INVALID_ARG;
}

onetrans_status onetrans_tokenize_autosplit(const onetrans_model* m, const void* feats, int64_t N,
                                            void* ns_tokens, void* ws, size_t ws_bytes, void* stream) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  if (N < 0 || N > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
  if (!m->Wa1 || !m->ba1 || !m->Wa2 || !m->ba2 || m->cfg.ns_feat_dim < 1 || m->cfg.ns_hidden < 1)
    return ONETRANS_ERR_UNSUPPORTED;
  if (N == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!feats || !ns_tokens || !aligned(feats, 16) || !aligned(ns_tokens, 16)) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? autosplit_impl<__nv_bfloat16>(m, feats, N, ns_tokens, ws, ws_bytes, st, nullptr)
                 : autosplit_impl<float>(m, feats, N, ns_tokens, ws, ws_bytes, st, nullptr);
}

onetrans_status onetrans_tokenize_groupwise(const onetrans_model* m, const void* feats, int64_t N,
                                            int32_t G, int32_t F_max, int32_t h_max, const void* W1,
                                            const void* b1, const void* W2, const void* b2, void* ns_tokens,
                                            void* ws, size_t ws_bytes, void* stream) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  if (N < 0 || N > (1LL << 31) - 1 || G != m->L_NS || F_max < 1 || h_max < 1) return ONETRANS_ERR_SHAPE;
  if (N == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!feats || !W1 || !b1 || !W2 || !b2 || !ns_tokens) return ONETRANS_ERR_INVALID_ARG;
  if (!aligned(feats, 16) || !aligned(ns_tokens, 16) || !aligned(W1, 16) || !aligned(W2, 16))
    return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? groupwise_impl<__nv_bfloat16>(m, feats, N, F_max, h_max, W1, b1, W2, b2, ns_tokens, ws,
                                                 ws_bytes, st, nullptr)
                 : groupwise_impl<float>(m, feats, N, F_max, h_max, W1, b1, W2, b2, ns_tokens, ws, ws_bytes, st,
                                         nullptr);
}

static onetrans_status check_slots(const onetrans_cache* c, const int32_t* slots, int U) {
  if (U < 0) return ONETRANS_ERR_SHAPE;
  if (U > 0 && !slots) return ONETRANS_ERR_INVALID_ARG;
  std::vector<char> seen(c->n_slots, 0);
  for (int u = 0; u < U; ++u) {
    if (slots[u] < 0 || slots[u] >= c->n_slots) return ONETRANS_ERR_SHAPE;
    if (seen[slots[u]]) return ONETRANS_ERR_INVALID_ARG;
    seen[slots[u]] = 1;
  }
  return ONETRANS_OK;
}

onetrans_status onetrans_stage1_encode(const onetrans_model* m, onetrans_cache* c, const int32_t* slots,
                                       int32_t U, const void* s_tokens, int32_t L_S, void* ws, size_t ws_bytes,
                                       void* stream) {
  if (!m || !c || c->m != m) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_slots(c, slots, U));
  if (L_S < 1) return ONETRANS_ERR_SHAPE;
  if ((long long)U * L_S > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
  if (U == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!s_tokens || !aligned(s_tokens, 16)) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? stage1_impl<__nv_bfloat16>(m, c, slots, U, s_tokens, L_S, ws, ws_bytes, st, nullptr)
                 : stage1_impl<float>(m, c, slots, U, s_tokens, L_S, ws, ws_bytes, st, nullptr);
}

onetrans_status onetrans_stage1_encode_ragged(const onetrans_model* m, onetrans_cache* c, const int32_t* slots,
                                              int32_t U, const void* s_tokens, const int32_t* lens, void* ws,
                                              size_t ws_bytes, void* stream) {
  if (!m || !c || c->m != m) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_slots(c, slots, U));
  if (U == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!lens) return ONETRANS_ERR_INVALID_ARG;
  long long R = 0;
  for (int u = 0; u < U; ++u) {
    if (lens[u] < 1) return ONETRANS_ERR_SHAPE;
    R += lens[u];
  }
  if (R > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
  if (!s_tokens || !aligned(s_tokens, 16)) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  // runs of consecutive users of one length: each is one uniform Stage I pass
  std::vector<std::pair<int, int>> runs;  // (first user, users)
  for (int u = 0; u < U;) {
    int v = u;
    while (v < U && lens[v] == lens[u]) ++v;
    runs.push_back({u, v - u});
    u = v;
  }
  // everything a pass can refuse is checked for every run before the first
  // launch; a run frees its slots' old pages before taking new ones, so page
  // capacity must hold for every prefix of the runs, in order
  const int P = m->cfg.page_tokens;
  const long long free0 = (long long)c->free_pages.size();
  long long need_pages = 0, owned_pages = 0;
  for (const auto& r : runs) {
    const int L = lens[r.first];
    if (L > c->max_L_S) return ONETRANS_ERR_CAPACITY;
    if ((long long)r.second * L > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
    std::vector<int> s, sq;
    OT_TRY(s_rows_of(m, L, s, sq));
    size_t need = 0;
    OT_TRY(m->bf16 ? stage1_impl<__nv_bfloat16>(m, c, slots + r.first, r.second, nullptr, L, nullptr, 0, 0, &need)
                   : stage1_impl<float>(m, c, slots + r.first, r.second, nullptr, L, nullptr, 0, 0, &need));
    if (need > ws_bytes) return ONETRANS_ERR_CAPACITY;
    for (int u = r.first; u < r.first + r.second; ++u) {
      for (int n = 0; n < m->NL; ++n) need_pages += cdiv(s[n], P);
      const size_t row = (size_t)slots[u] * m->NL * c->max_pages;
      for (size_t i = 0; i < (size_t)m->NL * c->max_pages; ++i) owned_pages += c->h_table[row + i] >= 0;
    }
    if (need_pages > free0 + owned_pages) return ONETRANS_ERR_CAPACITY;
  }
  cudaStream_t st = (cudaStream_t)stream;
  long long off = 0;
  for (const auto& r : runs) {
    const int L = lens[r.first];
    const void* tok = eoff(s_tokens, off * m->d, m->es);
    OT_TRY(m->bf16 ? stage1_impl<__nv_bfloat16>(m, c, slots + r.first, r.second, tok, L, ws, ws_bytes, st, nullptr)
                   : stage1_impl<float>(m, c, slots + r.first, r.second, tok, L, ws, ws_bytes, st, nullptr));
    off += (long long)r.second * L;
  }
  return ONETRANS_OK;
}

onetrans_status onetrans_stage2_score(const onetrans_model* m, const onetrans_cache* c, const int32_t* slots,
                                      int32_t U, const int32_t* cand_offsets, const void* ns_tokens,
                                      void* ns_out, float* logits, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !c || c->m != m) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_slots(c, slots, U));
  if (U == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (logits && !m->w_head) return ONETRANS_ERR_UNSUPPORTED;
  if (U > kMaxUsers) return ONETRANS_ERR_SHAPE;
  if (!cand_offsets) return ONETRANS_ERR_INVALID_ARG;
  for (int u = 0; u < U; ++u)
    if (cand_offsets[u + 1] < cand_offsets[u]) return ONETRANS_ERR_SHAPE;
  if (cand_offsets[0] != 0) return ONETRANS_ERR_SHAPE;
  for (int u = 0; u < U; ++u)
    if (c->len[slots[u]] == 0) return ONETRANS_ERR_SHAPE;
  if (cand_offsets[U] == 0) return ONETRANS_OK;  // no candidates
  if (!ns_tokens || !ns_out || !aligned(ns_tokens, 16) || !aligned(ns_out, 16)) return ONETRANS_ERR_INVALID_ARG;
  if (logits && !aligned(logits, 4)) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? stage2_impl<__nv_bfloat16>(m, c, slots, U, cand_offsets, ns_tokens, ns_out, logits, ws,
                                              ws_bytes, st, nullptr, 0, 0)
                 : stage2_impl<float>(m, c, slots, U, cand_offsets, ns_tokens, ns_out, logits, ws, ws_bytes, st,
                                      nullptr, 0, 0);
}

onetrans_status onetrans_cache_append(const onetrans_model* m, onetrans_cache* c, const int32_t* slots,
                                      int32_t U, const void* events, const int32_t* types, int32_t dL,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (!m || !c || c->m != m) return ONETRANS_ERR_INVALID_ARG;
  if (!m->pyr.empty()) return ONETRANS_ERR_UNSUPPORTED;
  if (m->cfg.n_behaviors < 1 || m->cfg.event_dim < 1 || m->Wb1.empty() || !m->type_emb)
    return ONETRANS_ERR_UNSUPPORTED;
  OT_TRY(check_slots(c, slots, U));
  if (dL < 0) return ONETRANS_ERR_SHAPE;
  if (U == 0 || dL == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!events || !types || !aligned(events, 16)) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  for (int u = 0; u < U; ++u)
    if (c->len[slots[u]] == 0) return ONETRANS_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? append_impl<__nv_bfloat16>(m, c, slots, U, events, types, dL, ws, ws_bytes, st, nullptr)
                 : append_impl<float>(m, c, slots, U, events, types, dL, ws, ws_bytes, st, nullptr);
}

onetrans_status onetrans_tokenize_events(const onetrans_model* m, const void* events, const int32_t* types,
                                         int64_t R, void* tokens, void* stream) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  if (m->cfg.n_behaviors < 1 || m->cfg.event_dim < 1 || m->Wb1.empty() || !m->type_emb)
    return ONETRANS_ERR_UNSUPPORTED;
  if (R < 0 || R > 0x7fffffff) return ONETRANS_ERR_SHAPE;
  if (R == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!events || !types || !tokens || !aligned(events, 16) || !aligned(tokens, 16))
    return ONETRANS_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? launch_event_tokenizer<__nv_bfloat16>(m, events, types, R, 1, rmap(tokens, m->d, m->d), st)
                 : launch_event_tokenizer<float>(m, events, types, R, 1, rmap(tokens, m->d, m->d), st);
}

onetrans_status onetrans_merge_intent_order(const onetrans_model* m, const void* events,
                                            const int64_t* seq_len, const int32_t* seq_type, int32_t n_seq,
                                            const void* sep, void* tokens, void* stream) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  if (m->cfg.n_behaviors < 1 || m->cfg.event_dim < 1 || m->Wb1.empty()) return ONETRANS_ERR_UNSUPPORTED;
  if (n_seq < 1) return ONETRANS_ERR_SHAPE;
  if (n_seq > kMaxIntents) return ONETRANS_ERR_UNSUPPORTED;
  if (!seq_len || !seq_type) return ONETRANS_ERR_INVALID_ARG;
  IntentLayout lay;
  std::memset(&lay, 0, sizeof(lay));
  lay.n = n_seq;
  lay.sep = sep;
  long long R = 0;
  for (int i = 0; i < n_seq; ++i) {
    if (seq_len[i] < 0) return ONETRANS_ERR_SHAPE;
    if (seq_type[i] < 0 || seq_type[i] >= m->cfg.n_behaviors) return ONETRANS_ERR_INVALID_ARG;
    R += seq_len[i];
    if (R + n_seq > 0x7fffffff) return ONETRANS_ERR_SHAPE;
    lay.end[i] = (int)R;
    lay.type[i] = seq_type[i];
  }
  const long long L_S = R + n_seq - 1;
  if (L_S == 0) return ONETRANS_OK;  // one empty sequence: no work
  if (!tokens || !aligned(tokens, 16) || (R > 0 && (!events || !aligned(events, 16))) || (n_seq > 1 && !sep))
    return ONETRANS_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? launch_event_tokenizer<__nv_bfloat16>(m, events, nullptr, R, 1, rmap(tokens, m->d, m->d), st,
                                                         &lay, false)
                 : launch_event_tokenizer<float>(m, events, nullptr, R, 1, rmap(tokens, m->d, m->d), st, &lay,
                                                 false);
}

onetrans_status onetrans_forward(const onetrans_model* m, const void* x0, int32_t B, int32_t L_S, void* out,
                                 void* ws, size_t ws_bytes, void* stream) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  if (B < 0 || L_S < 0) return ONETRANS_ERR_SHAPE;
  if ((long long)B * (L_S + m->L_NS) > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
  if (B == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!x0 || !out || !aligned(x0, 16) || !aligned(out, 16)) return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? forward_impl<__nv_bfloat16>(m, x0, B, L_S, out, ws, ws_bytes, st, nullptr)
                 : forward_impl<float>(m, x0, B, L_S, out, ws, ws_bytes, st, nullptr);
}

onetrans_status onetrans_forward_backward(const onetrans_model* m, const void* x0, int32_t B, int32_t L_S,
                                          const float* dy, float* out, float* dx0, const onetrans_grads* grads,
                                          void* ws, size_t ws_bytes, void* stream) {
  if (!m || !grads) return ONETRANS_ERR_INVALID_ARG;
  if (B < 0 || L_S < 0) return ONETRANS_ERR_SHAPE;
  if ((long long)B * (L_S + m->L_NS) * 3 * m->d > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
  float* const* per_layer[] = {grads->g_attn, grads->g_ffn, grads->Wqkv_S, grads->Wqkv_NS, grads->Wo,
                               grads->W1_S, grads->b1_S, grads->W2_S, grads->b2_S, grads->W1_NS,
                               grads->b1_NS, grads->W2_NS, grads->b2_NS};
  for (auto arr : per_layer) {
    if (!arr) return ONETRANS_ERR_INVALID_ARG;
    for (int l = 0; l < m->NL; ++l)
      if (!arr[l] || !aligned(arr[l], 16)) return ONETRANS_ERR_INVALID_ARG;
  }
  std::vector<int> Lq;
  OT_TRY(schedule_of(m, L_S, Lq));
  if (B == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!x0 || !dy || !out || !dx0 || !aligned(x0, 16) || !aligned(dy, 16) || !aligned(out, 16) || !aligned(dx0, 16))
    return ONETRANS_ERR_INVALID_ARG;
  OT_TRY(check_ws(ws));
  cudaStream_t st = (cudaStream_t)stream;
  return m->bf16 ? train_impl<__nv_bfloat16>(m, x0, B, L_S, dy, out, dx0, grads, ws, ws_bytes, st, nullptr)
                 : train_impl<float>(m, x0, B, L_S, dy, out, dx0, grads, ws, ws_bytes, st, nullptr);
}

onetrans_status onetrans_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.on = on != 0;
  g_prof.recs.clear();
  g_prof.used = 0;
  return ONETRANS_OK;
}

int32_t onetrans_profile_kinds(void) { return PK_COUNT; }

onetrans_status onetrans_profile_read(int32_t kind, const char** name, int64_t* launches, double* ms,
                                      double* flops, double* bytes) {
  if (kind < 0 || kind >= PK_COUNT || !name || !launches || !ms || !flops || !bytes)
    return ONETRANS_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  *name = kProfNames[kind];
  *launches = 0; *ms = 0; *flops = 0; *bytes = 0;
  for (const ProfRec& r : g_prof.recs) {
    if (r.kind != kind) continue;
    float t = 0.f;
    OT_TRY(cuda_ok(cudaEventSynchronize(r.e1)));
    OT_TRY(cuda_ok(cudaEventElapsedTime(&t, r.e0, r.e1)));
    *launches += 1; *ms += t; *flops += r.flops; *bytes += r.bytes;
  }
  return ONETRANS_OK;
}

onetrans_status onetrans_device_status(void* stream, int32_t* code) {
  if (!code) return ONETRANS_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  int v = 0;
  OT_TRY(cuda_ok(cudaMemcpyFromSymbolAsync(&v, ot::g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st)));
  OT_TRY(cuda_ok(cudaStreamSynchronize(st)));
  *code = v;
  if (v) {
    const int zero = 0;
    OT_TRY(cuda_ok(cudaMemcpyToSymbolAsync(ot::g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st)));
    OT_TRY(cuda_ok(cudaStreamSynchronize(st)));
    return ONETRANS_ERR_DEVICE_CHECK;
  }
  return ONETRANS_OK;
}

onetrans_status onetrans_selftest_bounded_wait(int32_t spin_limit, void* stream) {
  if (spin_limit < 1 || (uint32_t)spin_limit > ot::kSpinLimit) return ONETRANS_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint32_t)spin_limit);
  return last_launch();
}

}  // extern "C"

// ================================================= auto-split, no allocation
// Scratch for the auto-split tokenizer's hidden layer, in the library's own
// device memory: every GPU that loads the library holds these 16 MiB until
// the process exits.  All calls share it and it keeps the previous call's
// contents; nothing needs clearing because the first GEMM writes every
// element the second GEMM reads.  Calls whose kernels overlap on the GPU
// (two streams, two host threads) race on it.
static const size_t kStaticScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

static std::mutex g_static_mu;
static void* g_static_ptr[64];  // device address of g_static_scratch, per device

// Device address of the scratch on the current device, looked up once per
// device (host code cannot pass the symbol itself to a kernel).
static onetrans_status static_scratch(void** out) {
  int dev = -1;
  OT_TRY(cuda_ok(cudaGetDevice(&dev)));
  if (dev < 0 || dev >= 64) return ONETRANS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    OT_TRY(cuda_ok(cudaGetSymbolAddress(&p, g_static_scratch)));
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return ONETRANS_OK;
}

extern "C" onetrans_status onetrans_tokenize_autosplit_static(const onetrans_model* m, const void* feats,
                                                              int64_t N, void* ns_tokens, void* stream) {
  if (!m) return ONETRANS_ERR_INVALID_ARG;
  if (N < 0 || N > (1LL << 31) - 1) return ONETRANS_ERR_SHAPE;
  if (!m->Wa1 || !m->ba1 || !m->Wa2 || !m->ba2 || m->cfg.ns_feat_dim < 1 || m->cfg.ns_hidden < 1)
    return ONETRANS_ERR_UNSUPPORTED;
  if ((size_t)N * m->cfg.ns_hidden * m->es > kStaticScratchBytes) return ONETRANS_ERR_CAPACITY;
  if (N == 0) return ONETRANS_OK;  // no work: the data pointers may be NULL
  if (!feats || !ns_tokens || !aligned(feats, 16) || !aligned(ns_tokens, 16)) return ONETRANS_ERR_INVALID_ARG;
  void* scratch = nullptr;
  OT_TRY(static_scratch(&scratch));
  cudaStream_t st = (cudaStream_t)stream;
  // the workspace entry point's body with the scratch array as its workspace:
  // its capacity check also bounds every access to the array
  return m->bf16 ? autosplit_impl<__nv_bfloat16>(m, feats, N, ns_tokens, scratch, kStaticScratchBytes, st, nullptr)
                 : autosplit_impl<float>(m, feats, N, ns_tokens, scratch, kStaticScratchBytes, st, nullptr);
}
