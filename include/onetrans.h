/*
 * onetrans.h - C ABI of the OneTrans hot path on B200 (sm_100a).
 *
 * The library runs the forward pass of the OneTrans block stack and its
 * two-stage KV-cached scoring, as described in fun-rec mdbook 7.5, "OneTrans:
 * Unifying Sequence Modeling and Feature Interaction" (cited below as [FR]),
 * and in the paper-daily deep reading "OneTrans: Unified Feature Interaction
 * and Sequence Modeling with One Transformer in Industrial Recommender" ([PD]).
 *
 * Conventions shared by every call
 *  - Every pointer is a DEVICE pointer owned by the caller unless marked
 *    "host".  The library never allocates device memory: each call takes a
 *    caller-provided workspace whose size onetrans_workspace_size() reports,
 *    and the KV cache lives in a caller-provided pool (onetrans_cache_size()).
 *  - Tensors are dense row-major.  Inputs and weights follow the model's
 *    mode: ONETRANS_BF16 -> bfloat16 (fp32 accumulation inside kernels),
 *    ONETRANS_FP32 -> float32 with float32 arithmetic on CUDA cores.  The
 *    outputs of the stack (onetrans_forward's `out`, onetrans_stage2_score's
 *    `ns_out`) are float32 in both modes; inside, the residual stream is kept
 *    in float32 and only matrix operands and cached K/V use the mode's type.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream; inputs must stay valid
 *    and unmodified until the stream reaches the call's end.
 *  - Argument and shape errors are detected on the host before any launch and
 *    leave device memory untouched.  Launch failures return ONETRANS_ERR_CUDA.
 *  - A model is immutable after creation and may be used from several
 *    streams at once.  Calls that modify one cache slot must not overlap.
 *  - Buffers must be 16-byte aligned; the workspace and cache pool 256-byte.
 *  - A call with no work (N = 0, U = 0, B = 0, dL = 0, or no candidates at
 *    all) checks the model, cache, slots and offsets, returns ONETRANS_OK and
 *    launches nothing; its data pointers and workspace may then be NULL.
 */
#ifndef ONETRANS_H
#define ONETRANS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ONETRANS_API __attribute__((visibility("default")))
#else
#define ONETRANS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ONETRANS_OK = 0,
  ONETRANS_ERR_INVALID_ARG = -1, /* NULL pointer, bad enum, misaligned buffer */
  ONETRANS_ERR_SHAPE = -2,       /* sizes inconsistent with the model/schedule */
  ONETRANS_ERR_UNSUPPORTED = -3, /* e.g. append on a pyramid model */
  ONETRANS_ERR_CAPACITY = -4,    /* workspace or cache pool too small, slot full */
  ONETRANS_ERR_CUDA = -5,        /* a CUDA runtime/driver call failed */
  ONETRANS_ERR_DEVICE_CHECK = -6 /* a kernel's own bounds check fired */
} onetrans_status;

typedef enum { ONETRANS_BF16 = 0, ONETRANS_FP32 = 1 } onetrans_mode;

/* Model hyper-parameters.  [FR] 7.5.0-7.5.2 fix the structure; the widths,
 * head count, depth and schedule are the caller's choice.
 *  d_model % n_heads == 0, d_h = d_model / n_heads in {16, 32, 64, 96, 128}.
 *  pyramid_q (host, n_layers entries): L'_n, the number of tail rows kept as
 *    queries by layer n ([FR] 7.5.2, tail index set Q = {L-L'+1..L}).  NULL
 *    keeps every row.  Must be non-increasing and >= L_NS.
 *  ns_feat_dim / ns_hidden: F and H of the auto-split MLP (0 if unused).
 *  n_behaviors / event_dim: per-behavior event MLP used by cache append.
 *  page_tokens: KV-cache page size in tokens; must be 64. */
typedef struct {
  int32_t n_layers, d_model, n_heads, d_ff, L_NS;
  int32_t ns_feat_dim, ns_hidden;
  int32_t n_behaviors, event_dim;
  const int32_t* pyramid_q;
  float rms_eps;
  int32_t mode;
  int32_t page_tokens;
} onetrans_config;

/* Weights (device pointers, row-major W[out][in]; borrowed: the caller keeps
 * them alive while the model exists).  Per-layer entries are HOST arrays of
 * n_layers device pointers.  Mixed parameterization ([FR] 7.5.1): *_S is the
 * set shared by every S-token, *_NS holds one set per NS-token, stacked.
 *   g_attn, g_ffn      [d]              RMSNorm gains before attention / FFN
 *   Wqkv_S             [3d, d]          rows 0..d-1 = W^Q, d..2d-1 = W^K, 2d.. = W^V
 *   Wqkv_NS            [L_NS, 3d, d]
 *   Wo                 [d, d]           output projection shared by all tokens
 *   W1_S, b1_S         [d_ff, d], [d_ff]
 *   W2_S, b2_S         [d, d_ff], [d]
 *   W1_NS, b1_NS       [L_NS, d_ff, d], [L_NS, d_ff]
 *   W2_NS, b2_NS       [L_NS, d, d_ff], [L_NS, d]
 * Auto-split tokenizer ([FR] 7.5.0, NS-tokens = Split(MLP(Concat(NS)), L_NS)):
 *   Wa1 [H, F], ba1 [H], Wa2 [L_NS*d, H], ba2 [L_NS*d]      (may be NULL)
 * Per-behavior event MLP and type identifiers ([FR] 7.5.0, MLP_i and the
 * timestamp-aware merge): host arrays of n_behaviors device pointers
 *   Wb1[t] [d, event_dim], bb1[t] [d], Wb2[t] [d, d], bb2[t] [d];
 *   type_emb [n_behaviors, d]                                  (may be NULL)
 * Optional scoring head on the final NS states, the compact representation
 * the stack hands downstream ([FR] 7.5.2): logit = w_head . vec(h_NS) +
 * b_head, vec() token-major (token t = entries t*d .. t*d + d - 1):
 *   w_head [L_NS*d], b_head [1]                                (may be NULL) */
typedef struct {
  const void* const* g_attn;
  const void* const* g_ffn;
  const void* const* Wqkv_S;
  const void* const* Wqkv_NS;
  const void* const* Wo;
  const void* const* W1_S;
  const void* const* b1_S;
  const void* const* W2_S;
  const void* const* b2_S;
  const void* const* W1_NS;
  const void* const* b1_NS;
  const void* const* W2_NS;
  const void* const* b2_NS;
  const void* Wa1;
  const void* ba1;
  const void* Wa2;
  const void* ba2;
  const void* const* Wb1;
  const void* const* bb1;
  const void* const* Wb2;
  const void* const* bb2;
  const void* type_emb;
  const void* w_head;
  const void* b_head;
} onetrans_weights;

/* Weight gradients (float32 device pointers, laid out like onetrans_weights'
 * block-stack fields: per-layer fields are HOST arrays of n_layers device
 * pointers; each gradient has its weight's shape).  Written, not
 * accumulated, by onetrans_forward_backward. */
typedef struct {
  float* const* g_attn;
  float* const* g_ffn;
  float* const* Wqkv_S;
  float* const* Wqkv_NS;
  float* const* Wo;
  float* const* W1_S;
  float* const* b1_S;
  float* const* W2_S;
  float* const* b2_S;
  float* const* W1_NS;
  float* const* b1_NS;
  float* const* W2_NS;
  float* const* b2_NS;
} onetrans_grads;

typedef struct onetrans_model onetrans_model;
typedef struct onetrans_cache onetrans_cache;

/* Which call a workspace is sized for. */
typedef enum {
  ONETRANS_OP_FORWARD = 0,   /* n = B samples, L = L_S */
  ONETRANS_OP_STAGE1 = 1,    /* n = U users,   L = L_S */
  ONETRANS_OP_STAGE2 = 2,    /* n = total candidates, L = cached L_S */
  ONETRANS_OP_APPEND = 3,    /* n = U users,   L = dL */
  ONETRANS_OP_AUTOSPLIT = 4, /* n = N feature rows, L unused */
  ONETRANS_OP_GROUPWISE = 5, /* n = N feature rows, L = h_max (padded hidden width) */
  ONETRANS_OP_TRAIN = 6      /* n = B samples, L = L_S (onetrans_forward_backward) */
} onetrans_op;

/* Validate `cfg`/`w` and create a model.  Copies the config and the pointer
 * tables (not the weights).  Does not touch the GPU. */
ONETRANS_API onetrans_status onetrans_model_create(const onetrans_config* cfg,
                                      const onetrans_weights* w,
                                      onetrans_model** out);
ONETRANS_API onetrans_status onetrans_model_destroy(onetrans_model* m);

/* Bytes of workspace `op` needs for n rows of length L (see onetrans_op). */
ONETRANS_API onetrans_status onetrans_workspace_size(const onetrans_model* m, int32_t op,
                                        int64_t n, int32_t L, size_t* bytes);

/* Query counts of the stack for an input of L0 = L_S + L_NS rows: writes
 * n_layers values L'_n to `out` (host).  With no pyramid every L'_n = L0.
 * Returns SHAPE if the schedule does not fit L0 ([FR] 7.5.2). */
ONETRANS_API onetrans_status onetrans_schedule(const onetrans_model* m, int32_t L_S,
                                  int32_t* out);

/* ---------------------------------------------------------------- cache --
 * Paged, append-only KV cache of the S-side keys/values of every layer
 * ([FR] 7.5.3 Stage I and cross-request caching; [PD] 6.2 on paged
 * attention).  A page holds page_tokens consecutive tokens of one
 * (slot, layer) as [K|V][head][token][d_h].  The pool starts with the page
 * table (int32 [n_slots][n_layers][max_pages]) followed by the pages.  Page
 * assignment and per-slot lengths are tracked on the host, so capacity errors
 * never need a device read. */
ONETRANS_API onetrans_status onetrans_cache_size(const onetrans_model* m, int32_t n_slots,
                                    int32_t max_L_S, size_t* bytes);
ONETRANS_API onetrans_status onetrans_cache_init(const onetrans_model* m, void* pool,
                                    size_t bytes, int32_t n_slots,
                                    int32_t max_L_S, onetrans_cache** out);
ONETRANS_API onetrans_status onetrans_cache_destroy(onetrans_cache* c);
/* Cached S length of `slot` (host); 0 = empty. */
ONETRANS_API onetrans_status onetrans_cache_length(const onetrans_cache* c, int32_t slot,
                                      int32_t* len);
/* Device address of the first element of (slot, layer, kind 0=K/1=V, head,
 * token): lets callers read back cached rows.  Host-side arithmetic only. */
ONETRANS_API onetrans_status onetrans_cache_row_ptr(const onetrans_cache* c, int32_t slot,
                                       int32_t layer, int32_t kind,
                                       int32_t head, int32_t token,
                                       void** ptr);

/* ---------------------------------------------------------- entry points --
 * Auto-split NS tokenizer ([FR] 7.5.0): ns = Split(MLP(feats), L_NS) with
 * MLP = Linear(F->H) + ba1 -> GELU-tanh -> Linear(H->L_NS*d) + ba2.
 *   feats     [N, F]
 *   ns_tokens [N, L_NS, d]  (token t of row i = MLP output columns t*d..t*d+d-1) */
ONETRANS_API onetrans_status onetrans_tokenize_autosplit(const onetrans_model* m,
                                            const void* feats, int64_t N,
                                            void* ns_tokens, void* ws,
                                            size_t ws_bytes, void* stream);

/* Group-wise NS tokenizer (paper-daily reading "OneTrans: Unified Feature
 * Interaction and Sequence Modeling with One Transformer in Industrial
 * Recommender", 2.1 Unified Tokenization; listeners-pseudolab "OneTrans
 * 정리", 3.1 Non-Sequential Token): the non-sequential features come split
 * into G = L_NS semantic groups; group g's features go through the group's
 * own MLP (Linear F_g -> h_g, GELU-tanh, Linear h_g -> d) and give NS token g.
 * Every group is zero-padded to common widths F_max and h_max (zero feature
 * columns, zero weight rows and columns, zero bias entries), which leaves
 * the result unchanged since GELU(0) = 0.
 *   feats [N, G, F_max]; W1 [G, h_max, F_max]; b1 [G, h_max];
 *   W2 [G, d, h_max]; b2 [G, d]; ns_tokens [N, G, d] (all device, the mode's
 *   element type), the layout onetrans_stage2_score takes.
 * The weights are arguments, not part of the model, and stay the caller's.
 * G != L_NS, F_max < 1 or h_max < 1 is SHAPE; the workspace holds the hidden
 * layer (onetrans_workspace_size with ONETRANS_OP_GROUPWISE, n = N,
 * L = h_max). */
ONETRANS_API onetrans_status onetrans_tokenize_groupwise(
    const onetrans_model* m, const void* feats, int64_t N, int32_t G,
    int32_t F_max, int32_t h_max, const void* W1, const void* b1,
    const void* W2, const void* b2, void* ns_tokens, void* ws,
    size_t ws_bytes, void* stream);

/* The auto-split tokenizer for callers that cannot allocate device memory:
 * a plugin inside an inference server whose device memory all belongs to the
 * server's own pool, or a latency-bound serving loop where a cudaMalloc would
 * synchronize the device.  Same computation and output as
 * onetrans_tokenize_autosplit, but no workspace: the hidden layer lives in a
 * fixed 16 MiB array in the library's own device memory, held by every GPU
 * that loads the library until the process exits.  N * ns_hidden * element
 * size must not exceed 16 MiB (N <= 2730 rows at H = 3072 in bf16), else
 * ONETRANS_ERR_CAPACITY.  The first call on a device looks up the array's
 * address with that device current; make that first call before any stream
 * capture.  All calls share the array: calls whose kernels overlap on the GPU
 * race.  Nothing is allocated.  The pages have no counterpart of this call. */
ONETRANS_API onetrans_status onetrans_tokenize_autosplit_static(
    const onetrans_model* m, const void* feats, int64_t N, void* ns_tokens,
    void* stream);

/* S-side tokenizer, timestamp-aware merge ([FR] 7.5.0): each event is
 * aligned to d by the MLP of its behavior type (Linear e->d, GELU-tanh,
 * Linear d->d) plus the type's additive identifier.  The caller lays the
 * events of a user's behavior sequences out in time order (one flat row per
 * event); the tokens then feed onetrans_stage1_encode or onetrans_forward.
 *   events [R, event_dim] (the mode's element type); types [R] int32
 *   (device, each in 0 .. n_behaviors-1; an out-of-range id sets the device
 *   status word and is read as 0); tokens [R, d] (the mode's element type).
 * UNSUPPORTED when the model has no behavior MLPs. */
ONETRANS_API onetrans_status onetrans_tokenize_events(const onetrans_model* m,
                                        const void* events,
                                        const int32_t* types, int64_t R,
                                        void* tokens, void* stream);

/* S-side tokenizer, timestamp-agnostic merge ([FR] 7.5.0): a user's n_seq
 * behavior sequences, given in intent order (for example purchase, then
 * add-to-cart, then click), are each aligned to d by their behavior's MLP
 * (Linear e->d, GELU-tanh, Linear d->d; no type identifier) and laid out one
 * after another with the learnable [SEP] vector between consecutive ones.
 *   events [R, event_dim] (the mode's element type, device): the sequences'
 *     events back to back, R = sum of seq_len;
 *   seq_len [n_seq] int64, seq_type [n_seq] int32 (host): each sequence's
 *     length (0 allowed) and behavior id (0 .. n_behaviors-1);
 *   sep [d] (the mode's element type, device; may be NULL when n_seq = 1);
 *   tokens [L_S, d] (the mode's element type, device), L_S = R + n_seq - 1:
 *     sequence i at rows from (sum of earlier lengths) + i, its [SEP] right
 *     after it.
 * 1 <= n_seq <= 8, else SHAPE (below 1) or UNSUPPORTED (above 8); a negative
 * length is SHAPE, an out-of-range behavior id INVALID_ARG, both before any
 * launch.  UNSUPPORTED when the model has no behavior MLPs. */
ONETRANS_API onetrans_status onetrans_merge_intent_order(
    const onetrans_model* m, const void* events, const int64_t* seq_len,
    const int32_t* seq_type, int32_t n_seq, const void* sep, void* tokens,
    void* stream);

/* Stage I ([FR] 7.5.3): run each user's S-tokens through the stack (pyramid
 * tail queries included) and store every layer's S-side K/V in cache slot
 * slots[u] (host array of U slot ids, distinct).  The slot's previous
 * contents are replaced.  s_tokens [U, L_S, d]. */
ONETRANS_API onetrans_status onetrans_stage1_encode(const onetrans_model* m,
                                       onetrans_cache* c, const int32_t* slots,
                                       int32_t U, const void* s_tokens,
                                       int32_t L_S, void* ws, size_t ws_bytes,
                                       void* stream);

/* Stage I for users of different lengths in one call: user u's lens[u]
 * (host) S-tokens lie back to back in s_tokens [sum of lens, d], in the
 * order of slots.  Each run of consecutive users with one length is one
 * onetrans_stage1_encode pass over its slice (ordering users by length makes
 * fewer passes).  Every check a pass can fail (length against the pool, the
 * schedule, the workspace, page capacity over the runs in order) is made for
 * all runs before the first launch.  A workspace sized for
 * ONETRANS_OP_STAGE1 with n = U, L = the largest length is enough. */
ONETRANS_API onetrans_status onetrans_stage1_encode_ragged(
    const onetrans_model* m, onetrans_cache* c, const int32_t* slots,
    int32_t U, const void* s_tokens, const int32_t* lens, void* ws,
    size_t ws_bytes, void* stream);

/* Stage II ([FR] 7.5.3): score candidates against the cached S side.  User u
 * owns candidates cand_offsets[u] .. cand_offsets[u+1]-1 (host CSR, U+1
 * entries) and cache slot slots[u] (host).  Per layer, NS token j of a
 * candidate attends in one softmax to the slot's cached S keys and its own
 * NS keys 0..j, then passes through its token-specific FFN.  Slots may hold
 * different S lengths (encoded by separate Stage I calls): each user's layers
 * then see that user's own pyramid schedule of cached keys.  A slot with no
 * cached sequence is ONETRANS_ERR_SHAPE.  At most 65536 users per call.
 *   ns_tokens [C_tot, L_NS, d] (candidate-major, as the tokenizer writes it);
 *   ns_out    [C_tot, L_NS, d] float32;
 *   logits    [C_tot] float32 or NULL: w_head . vec(ns_out[c]) + b_head per
 *             candidate; non-NULL needs the model's head weights
 *             (ONETRANS_ERR_UNSUPPORTED otherwise). */
ONETRANS_API onetrans_status onetrans_stage2_score(const onetrans_model* m,
                                      const onetrans_cache* c,
                                      const int32_t* slots, int32_t U,
                                      const int32_t* cand_offsets,
                                      const void* ns_tokens, void* ns_out,
                                      float* logits, void* ws, size_t ws_bytes,
                                      void* stream);

/* Cross-request append ([FR] 7.5.3): tokenize dL new events per user with the
 * per-behavior MLP plus type identifier, run only those rows through every
 * layer (keys: cached + new, causal), and append their K/V to slots[u].
 * Non-pyramid models only (UNSUPPORTED otherwise).  Slots may hold
 * different lengths: user u's events take positions len(slots[u]) ..
 * len(slots[u]) + dL - 1.  A slot with no cached sequence is
 * ONETRANS_ERR_SHAPE.  events [U, dL, event_dim]; types [U, dL] int32
 * (device). */
ONETRANS_API onetrans_status onetrans_cache_append(const onetrans_model* m,
                                      onetrans_cache* c, const int32_t* slots,
                                      int32_t U, const void* events,
                                      const int32_t* types, int32_t dL,
                                      void* ws, size_t ws_bytes, void* stream);

/* One-pass forward of the stack on X^(0) = [S-tokens; NS-tokens] ([FR] 7.5.0
 * eq. for X^(0), 7.5.1, 7.5.2).  x0 [B, L_S + L_NS, d]; out [B, L'_N, d]
 * float32, the rows the last layer keeps. */
ONETRANS_API onetrans_status onetrans_forward(const onetrans_model* m, const void* x0,
                                 int32_t B, int32_t L_S, void* out, void* ws,
                                 size_t ws_bytes, void* stream);

/* Training step of the stack (the pages train it end to end and cut training
 * time and memory with mixed precision and activation recomputation: [FR]
 * 7.5.3 system optimizations; paper-daily 4.3, the "+ mixed precision +
 * recomputation" row).  Forward over x0 [B, L_S + L_NS, d] (the mode's
 * type) keeping each layer's input and its attention output and
 * log-sum-exp (O(L) per layer), then the backward layer by layer with the
 * rest of each layer's intermediates (the normalised rows, q | k | v, the
 * residual sum and the FFN pre-activation) recomputed from its input: a
 * selective recomputation that skips the attention's second forward.  The
 * loss gradient
 * enters as dy [B, L'_N, d] float32, the gradient of the output out
 * [B, L'_N, d] float32 (the rows onetrans_forward returns).  Writes out,
 * dx0 [B, L_S + L_NS, d] float32 (gradient of x0) and every weight gradient
 * of `grads`.  In BF16 mode every matrix operand is bf16 with float32
 * accumulation and every gradient float32; FP32 mode is float32
 * throughout.  Workspace: ONETRANS_OP_TRAIN with n = B, L = L_S. */
ONETRANS_API onetrans_status onetrans_forward_backward(const onetrans_model* m, const void* x0,
                                          int32_t B, int32_t L_S, const float* dy,
                                          float* out, float* dx0,
                                          const onetrans_grads* grads, void* ws,
                                          size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- plumbing --
 * Kernel selection for tests: 0 = automatic (tensor-core kernels where the
 * shape allows), 1 = CUDA-core kernels only.  Process-wide. */
ONETRANS_API onetrans_status onetrans_set_kernel_policy(int32_t policy);
/* Reads and clears the device status word that kernels set, instead of
 * trapping, when a bounds check or a bounded wait fails.  *code: 0 = no
 * failure, 101 = an mbarrier wait gave up (its kernel drained and returned),
 * 102 = dynamic shared memory not 1024-byte aligned (the kernel returned
 * without work), 3 = a CUDA-core kernel's bounds check skipped an access.
 * Returns ONETRANS_ERR_DEVICE_CHECK when *code != 0.  Synchronizes `stream`. */
ONETRANS_API onetrans_status onetrans_device_status(void* stream, int32_t* code);
/* Exercises the failure path of the bounded waits without a GPU fault: one
 * thread waits on an mbarrier that nothing arrives at, with the wait every
 * tensor-core kernel uses, limited to spin_limit try_wait rounds (1 ..
 * 2^20, else INVALID_ARG).  The wait gives up, records code 101 in the
 * device status word and the kernel returns; onetrans_device_status then
 * reports it. */
ONETRANS_API onetrans_status onetrans_selftest_bounded_wait(int32_t spin_limit, void* stream);
/* Per-kernel timing for measurement.  While enabled, every launch is
 * bracketed by CUDA events on its stream and tagged with its kernel kind and
 * its algorithmic FLOPs and bytes (each operand and result once).  Enabling
 * clears earlier records.  onetrans_profile_read synchronizes on the
 * recorded events and sums one kind: launches, device milliseconds, FLOPs,
 * bytes; `name` points to static storage. */
ONETRANS_API onetrans_status onetrans_profile_enable(int32_t on);
ONETRANS_API int32_t onetrans_profile_kinds(void);
ONETRANS_API onetrans_status onetrans_profile_read(int32_t kind, const char** name,
                                                   int64_t* launches, double* ms,
                                                   double* flops, double* bytes);
/* Human-readable name of a status code (static storage). */
ONETRANS_API const char* onetrans_status_string(int32_t status);
/* Library version as major*10000 + minor*100 + patch. */
ONETRANS_API int32_t onetrans_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ONETRANS_H */
