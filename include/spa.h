/*
 * spa.h -- C ABI of libspa, the SPA-Cache cached transformer-block update on
 * one NVIDIA B200 (sm_100a).
 *
 * SPA-Cache ("Singular Proxies for Adaptive Caching in Diffusion Language
 * Models") refreshes only the k = ceil(N * rho(l)) tokens of layer l whose
 * low-rank proxy drifted most since they were last refreshed, and reuses
 * cached rows for the rest.  The operations below follow the three phases of
 * the method's Algorithm 1 as given on the papernotes.org page (方法详解 >
 * 整体框架) and the gist.science technical summary (Methodology, items 1-3).
 *
 * Conventions for every call:
 *   - Returns a spa_status (0 = SPA_OK).  Arguments and shapes are checked
 *     before anything is launched; a failing call launches nothing.
 *   - Device work is enqueued on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and is asynchronous: no call below
 *     synchronises the host unless it says so.
 *   - Pointers marked "device" must point to device memory of the current
 *     device; "host" pointers to host memory.  Matrices are row-major.
 *     Weight matrices are stored [out, in] (y = W x).
 *   - Element type: dtype SPA_F32 (float) or SPA_BF16 (__nv_bfloat16) for
 *     weights, hidden states, K^c, V^c and H^c.  Proxies P^c, scores and the
 *     proxy weights given from the host are always float.  Index sets are
 *     int32, ascending.
 *   - Ownership: the caller owns activations, caches and weights (borrowed:
 *     they must outlive the handles that use them).  The library owns what
 *     its create/init calls allocate and frees it in the matching free call.
 *   - Device-side checks (gather/scatter indices out of range, a bounded wait
 *     that ran out) do not fault: they set an error word in the workspace,
 *     which spa_workspace_status() reads and clears.
 *   - Handles are not thread-safe.  Calls that share a workspace must be
 *     ordered on one stream.
 */
#ifndef SPA_H
#define SPA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPA_OK = 0,
  SPA_ERR_INVALID = -1,     /* null pointer or a bad argument value */
  SPA_ERR_SHAPE = -2,       /* a size outside what the handle was created for */
  SPA_ERR_CUDA = -3,        /* a CUDA runtime/driver call or a launch failed */
  SPA_ERR_NOMEM = -4,       /* device or host allocation failed */
  SPA_ERR_UNSUPPORTED = -5, /* valid, but not built for this configuration */
  SPA_ERR_TIMEOUT = -6,     /* a device-side bounded wait ran out */
  SPA_ERR_DEVICE = -7       /* a device-side index check failed */
} spa_status;

enum { SPA_F32 = 0, SPA_BF16 = 1 };

/* Static, NUL-terminated name of a status.  Thread-safe. */
const char *spa_status_string(int status);
/* Detail message of the last failing call on this host thread ("" if none). */
const char *spa_last_error(void);
/* Library version, 100*major + minor. */
int spa_version(void);

/* ---------------------------------------------------------------- budget --
 * rho(l): piecewise-Gaussian update ratio of layer l (1-based) of L layers,
 * peak rho_p at layer l_p, rho_1 at layer 1, rho_L at layer L (papernotes.org,
 * 关键设计 3).  For l <= l_p: rho_p*exp(ln(rho_1/rho_p)*((l-l_p)/(l_p-1))^2);
 * for l > l_p the same with rho_L and (L-l_p) (the branch the page calls
 * symmetric, read so that rho(L) = rho_L).  Returns NaN on invalid input. */
double spa_rho(int l, int L, double rho_p, int l_p, double rho_1, double rho_L);
/* k = ceil(N * rho) clamped to [1, N] (Algorithm 1, phase 1: "k = N rho").
 * Returns -1 on invalid input (N < 1, rho not finite or <= 0). */
int spa_budget_k(int N, double rho);

/* ------------------------------------------------------------ layer setup -- */
typedef struct {
  int d;          /* model width; multiple of 256 for SPA_BF16, of 4 for SPA_F32 */
  int n_heads;    /* d = n_heads * head_dim */
  int head_dim;   /* even; <= 128 */
  int ffn;        /* SwiGLU hidden width F; multiple of 128 for SPA_BF16 */
  int r;          /* proxy rank, 1 <= r <= d; SPA_BF16: r > 256 (up to r = d, the full-d
                   * Value identifier) must be a multiple of 4; SPA_F32: r <= 128 */
  int dtype;      /* SPA_F32 or SPA_BF16 */
  float rms_eps;  /* RMSNorm epsilon */
  float rope_theta;
} spa_layer_desc;

/* Device pointers of one layer's weights, dtype elements, borrowed.
 * wq, wk, wv, wo: [d, d]; w_gate, w_up: [F, d]; w_down: [d, F];
 * attn_norm, ffn_norm: [d] RMSNorm gains. */
typedef struct {
  const void *wq, *wk, *wv, *wo, *w_gate, *w_up, *w_down, *attn_norm, *ffn_norm;
} spa_layer_weights;

/* Host routine: W_r = Lambda_r V_r^T (r x d) from the truncated SVD of the
 * Value weights, W_v ~= U Lambda V^T (papernotes.org, 关键设计 2).  w_v is the
 * host [d, d] float matrix as stored ([out, in]); w_r_out receives r*d
 * floats, each row's largest-magnitude entry made positive.  Randomised
 * subspace iteration in double precision with oversampling; accuracy ~1e-6
 * relative for spectra with a gap beyond r.  Synchronous, host only. */
int spa_singular_proxy_host(const float *w_v, int d, int r, float *w_r_out);

/* Scratch for the layer calls: sized for at most max_B sequences of max_N
 * tokens.  One workspace can serve many layers of the same shape. */
typedef struct spa_workspace spa_workspace;
int spa_workspace_create(const spa_layer_desc *desc, int max_B, int max_N, spa_workspace **out);
void spa_workspace_free(spa_workspace *ws);
/* Synchronises `stream`, then reads and clears the device error word:
 * SPA_OK, SPA_ERR_TIMEOUT or SPA_ERR_DEVICE. */
int spa_workspace_status(spa_workspace *ws, void *stream);

/* Device addresses of the workspace buffers that hold the intermediates of
 * the last layer call, for inspection (valid until the workspace is freed;
 * overwritten by the next call).  Rows t = b*k + i are the selected tokens in
 * index-set order (k = N for spa_full_block): x = RMSNorm(H[I]) [B*k, d],
 * q = RoPE(Q_I) [B*k, d], o = attention output [B*k, d], h1 = H[I] + o W_o^T
 * [B*k, d], x2 = RMSNorm(h1) [B*k, d], a = silu(x2 W_gate^T) * (x2 W_up^T)
 * [B*k, F] (dtype elements); a_hat [B*N, r] and score [B*N] (float) from
 * the last spa_proxy_select. */
typedef struct {
  void *x, *q, *o, *h1, *x2, *a;
  float *a_hat, *score;
} spa_intermediates;
int spa_workspace_intermediates(const spa_workspace *ws, spa_intermediates *out);

/* Kernel timing.  While enabled, every kernel the library launches for this
 * workspace (layers, and models built on it) is bracketed by two CUDA events
 * on its stream.  spa_profile_read synchronises on the recorded events and
 * fills, per kernel class (arrays of SPA_PROF_CLASSES entries), the number
 * of launches, their summed device time in ms, and the algorithmic bytes and
 * flops those launches move and perform (computed from the shapes: each
 * operand read once, each result written once), then clears the record. */
enum {
  SPA_PROF_PROXY = 0, /* phase 1 proxy GEMM + norm + score */
  SPA_PROF_TOPK,      /* top-k select + P^c scatter */
  SPA_PROF_NORM,      /* RMSNorm (gathered rows) */
  SPA_PROF_QKV,       /* Q/K/V GEMM + RoPE + K^c/V^c scatter */
  SPA_PROF_ATTN,      /* sparse-query attention */
  SPA_PROF_OPROJ,     /* output projection + residual */
  SPA_PROF_GATEUP,    /* gate/up GEMM + SwiGLU */
  SPA_PROF_DOWN,      /* down GEMM + residual + H^c scatter */
  SPA_PROF_LMHEAD,    /* LM head GEMM + per-tile argmax */
  SPA_PROF_MISC,      /* embedding rows, final norm, argmax reduction */
  SPA_PROF_FFN,       /* the persistent FFN half: O-proj + FFN norm + gate/up + down in one launch */
  SPA_PROF_CLASSES
};
int spa_profile_enable(spa_workspace *ws, int enable);
int spa_profile_read(spa_workspace *ws, int *launches, double *ms, double *bytes, double *flops);
/* Number of kernels the library has launched in this process so far. */
long long spa_launch_count(void);

/* A layer handle: borrows `w` and `ws`, owns its proxy weights W_r (stored in
 * the layer dtype) and the RoPE table.  w_r_host (host, [r, d] float) is a
 * proxy computed offline; NULL makes the library copy W_v to the host and run
 * spa_singular_proxy_host (synchronous). */
typedef struct spa_layer spa_layer;
int spa_init_layer(const spa_layer_desc *desc, const spa_layer_weights *w, const float *w_r_host,
                   spa_workspace *ws, spa_layer **out);
void spa_free_layer(spa_layer *layer);
/* Copies the stored proxy weights (as float) to host w_r_out [r, d]. */
int spa_layer_proxy_weights(const spa_layer *layer, float *w_r_out);

/* Caches of one layer for B sequences of N tokens (device, caller-owned):
 * k_cache, v_cache: [B, N, d] post-RoPE keys and values; h_cache: [B, N, d]
 * layer outputs; p_cache: [B, N, r] float unit proxies. */
typedef struct {
  void *k_cache, *v_cache, *h_cache;
  float *p_cache;
  int B, N;
} spa_layer_cache;

/* ----------------------------------------------------------- layer step --
 * Phase 1, update identification (Algorithm 1; gist.science Methodology
 * item 1): a = W_r h for every token of H ([B, N, d] device, the layer
 * input), a_hat = a/|a|, s = 1/2 |a_hat - P^c|^2 (= 1 - cosine to the cached
 * proxy), I = the k largest s per sequence with ties to the lowest index,
 * written ascending to idx ([B, k] int32 device); then P^c[I] <- a_hat[I].
 * score ([B, N] float device) receives s when non-NULL. */
int spa_proxy_select(spa_layer *layer, const void *H, const spa_layer_cache *cache, int k,
                     int32_t *idx, float *score, void *stream);

/* Phases 2 and 3 for a given index set idx ([B, k] int32 device, ascending,
 * entries in [0, N)): x = RMSNorm(H[I]); Q, K, V = x W^T; RoPE on Q, K at
 * positions I; K^c[I] <- K, V^c[I] <- V; O = softmax(Q K^cT / sqrt(d_h)) V^c
 * over all N cached rows; H1 = H[I] + O W_o^T;
 * H^c[I] <- H1 + W_down(silu(W_gate x2) * W_up x2), x2 = RMSNorm(H1).
 * Rows of H^c outside I are not touched. */
int spa_partial_block(spa_layer *layer, const void *H, const int32_t *idx, int k,
                      const spa_layer_cache *cache, void *stream);

/* Phases 1-3 in one call: spa_proxy_select then spa_partial_block. */
int spa_layer_step(spa_layer *layer, const void *H, const spa_layer_cache *cache, int k,
                   int32_t *idx, void *stream);

/* rho = 1 pass (the uncached forward): every row of K^c, V^c and H^c is
 * recomputed from H.  fill_proxy = 1 also writes P^c = a_hat of every row
 * (the cache fill that starts a decode); 0 skips the proxy entirely; 2 fills
 * P^c with every row's unit attention output instead, the fill of the
 * attention-output identifier below (needs r = d). */
int spa_full_block(spa_layer *layer, const void *H, const spa_layer_cache *cache, int fill_proxy,
                   void *stream);

/* A cached layer step with the attention output as the update identifier,
 * the variant the pages compare with the Value proxy (papernotes.org, 关键设计
 * 1 and Table 1: Query, Key, Value or attention output as identifier).  Its
 * cost is the point: scoring a token by the drift of its attention output
 * needs that output for every token, so phase 1 runs the attention
 * sub-layer for all N rows: x = RMSNorm(H), Q/K/V of every row with RoPE,
 * K^c, V^c rewritten at every row, O = softmax(Q K^cT / sqrt(d_h)) V^c; then
 * o_hat = O / |O|, s = 1/2 |o_hat - P^c|^2 against the cached unit outputs
 * P^c ([B, N, r] with r = d), I = the k largest s (ties to the lowest index,
 * ascending) into idx ([B, k] int32 device), P^c[I] <- o_hat[I].  Phase 3 runs
 * on the selected rows: H1 = H[I] + O[I] W_o^T, H^c[I] <- H1 + FFN(RMSNorm(H1)).
 * The layer must have r = d (its W_r is not used); start from
 * spa_full_block(..., fill_proxy = 2).  Errors: SPA_ERR_INVALID,
 * SPA_ERR_SHAPE (k outside [1, N], r != d), SPA_ERR_CUDA. */
int spa_layer_step_attn_identifier(spa_layer *layer, const void *H, const spa_layer_cache *cache, int k,
                                   int32_t *idx, void *stream);

/* ---------------------------------------------------------- decode loop -- */
typedef struct {
  int n_layers, vocab, B, N;
  double rho_p, rho_1, rho_L; /* rho(l) parameters; uniform budget: all equal */
  int l_p;
} spa_model_desc;

/* A model: n_layers layer handles (borrowed, all sharing one workspace), a
 * cache per layer (caches[l], borrowed), the layer-0 input buffer h0
 * ([B, N, d] device, borrowed), token embeddings embed [vocab, d], final
 * RMSNorm gain final_norm [d] and LM head lm_head [vocab, d] (device,
 * borrowed).  The per-layer budgets k_l come from rho(l) at creation. */
typedef struct spa_model spa_model;
int spa_model_create(const spa_model_desc *desc, spa_layer *const *layers,
                     const spa_layer_cache *caches, void *h0, const void *embed,
                     const void *final_norm, const void *lm_head, spa_model **out);
void spa_model_free(spa_model *model);
/* k_l of layer l (0-based), or -1. */
int spa_model_layer_k(const spa_model *model, int layer);
/* The index set I of layer `layer` (0-based) from the last cached decode
 * step (Algorithm 1, phase 1: the k_l tokens per sequence whose proxy drifted
 * most, ascending): copies B * k_l int32 values, [B, k_l], into idx_out
 * (device), asynchronously on `stream`.  Undefined before the first cached
 * step (a rho = 1 step selects every row and does not write it). */
int spa_model_index_set(const spa_model *model, int layer, int32_t *idx_out, void *stream);
/* h0[b, i] <- embed[tokens[b, i]] for every position (tokens: [B, N] int32 device). */
int spa_model_embed(spa_model *model, const int32_t *tokens, void *stream);

/* One decoding step: full = 0 runs the cached layer step with k_l at every
 * layer; full = 1 runs every layer at rho = 1 and fills all caches, P^c
 * included (step 0); full = 2 runs every layer at rho = 1 without the proxy
 * (vanilla decoding, the uncached baseline).  Then the final RMSNorm and LM head at the u
 * positions pos ([B, u] int32 device) give argmax ids (lowest id on ties)
 * into tok_out ([B, u] int32 device).  The ids written back into h0 at pos
 * for the next step are tok_in ([B, u] device) when non-NULL (teacher
 * forcing), else the argmax. */
int spa_decode_step(spa_model *model, const int32_t *pos, const int32_t *tok_in, int u, int full,
                    int32_t *tok_out, void *stream);

/* The same step in three calls, for callers that choose the positions to
 * unmask from the logits (confidence-based parallel unmasking: [NOTES]
 * 实验关键数据 > 叠加并行解码 (Table 3); [GIST] Key Findings, "Integration
 * with Parallel Decoding"; the threshold rule is the caller's):
 * - spa_decode_layers runs the L layers of one step (full as above);
 * - spa_decode_confidence takes the final RMSNorm and the LM head at u
 *   positions pos ([B, u] int32 device, e.g. every still-masked position) and
 *   writes per position the argmax id (lowest on ties) into tok_out ([B, u]
 *   int32) and its softmax probability 1 / sum_v exp(l_v - max_v l) into
 *   conf_out ([B, u] float);
 * - spa_model_write_tokens puts embed[tok] ([B, u] int32 device) into h0 at
 *   pos ([B, u]), the next step's layer-0 input (with the incremental proxy,
 *   these are the rows the next step's layer 0 projects again).
 * spa_decode_step is spa_decode_layers, the argmax at pos, and
 * spa_model_write_tokens.  u <= N; errors as spa_decode_step. */
int spa_decode_layers(spa_model *model, int full, void *stream);
int spa_decode_confidence(spa_model *model, const int32_t *pos, int u, int32_t *tok_out, float *conf_out,
                          void *stream);
int spa_model_write_tokens(spa_model *model, const int32_t *pos, const int32_t *tok, int u, void *stream);

/* CUDA-graph form of the cached decode step (full = 0).  Capture records one
 * step with fixed device buffers pos ([B, u]), tok_in ([B, u] or NULL) and
 * tok_out ([B, u]) on `stream` (must not be the legacy default stream; the
 * step must not be running elsewhere), replacing any earlier capture.  Each
 * launch replays it: the caller writes the step's positions (and forced ids)
 * into those buffers first.  Kernel timing events are not recorded inside the
 * graph.  The graph belongs to the model and is freed with it. */
int spa_decode_graph_capture(spa_model *model, const int32_t *pos, const int32_t *tok_in, int u,
                             int32_t *tok_out, void *stream);
int spa_decode_graph_launch(spa_model *model, void *stream);
/* Number of kernel nodes in the captured step's graph (the library kernels
 * one launch of it runs); 0 when nothing has been captured, -1 for a null
 * model. */
int spa_decode_graph_kernel_nodes(const spa_model *model);

/* Incremental proxy (enable = 1; 0 restores the plain path).  Phase 1 of
 * Algorithm 1 ([NOTES] 方法详解 > 整体框架; [GIST] Methodology 1) scores every
 * token with the unit proxy of its current layer input against P^c.  A
 * token's layer input changes in a decoding step only if the previous layer
 * rewrote its row (I_{l-1}), or, at layer 0, if it was unmasked at the end of
 * the last step; the other rows keep their proxy, and their score changes
 * only where P^c was rewritten, to exactly 0 (P^c = a_hat there).  In this
 * mode the model keeps, per layer, a_hat [B, N, r] and the score [B, N]
 * (fp32, library-owned, allocated here: L*B*N*(r + 1)*4 bytes, plus a compact
 * [B*N, d] buffer of changed rows), and a cached step projects only the
 * changed rows (B*k_{l-1} per layer, B*u at layer 0) instead of all B*N.
 * The scores, index sets and outputs are bit-identical to the plain path:
 * the proxy GEMM reduces each row in a fixed order that does not depend on
 * the other rows.  The first cached step after enabling, after
 * spa_model_embed or after a vanilla step (full = 2) projects every row once;
 * a fill (full = 1) sets the state directly.  A graph captured while the
 * state is current replays the incremental step and refuses to launch
 * (SPA_ERR_INVALID) once the state has gone stale.  Errors: SPA_ERR_INVALID
 * (null model), SPA_ERR_NOMEM. */
int spa_model_set_incremental_proxy(spa_model *model, int enable);

/* ------------------------------------------------------- testing hooks --
 * No counterpart on the pages: hooks that let tests drive the failure paths
 * without faulting or hanging a GPU.
 *
 * spa_debug_fail_alloc_after(n): after n more successful device allocations
 * made by the library (workspaces, layer proxy weights, model buffers, the
 * incremental-proxy state), the next one fails once, as if the device were
 * out of memory; the call that made it returns SPA_ERR_NOMEM having freed
 * what it had allocated.  n < 0 switches the injection off.  Process-wide;
 * returns SPA_OK.
 *
 * spa_debug_bounded_wait(ws, flag, expect, limit_us, stream): launches one
 * bounded device-side wait that records a time-out in the workspace's error
 * word (spa_workspace_status then returns SPA_ERR_TIMEOUT) if it has not
 * completed after limit_us microseconds (0 <= limit_us <= 1e6).  flag NULL:
 * the wait is on a shared-memory barrier that nothing completes, the kind of
 * wait every pipelined kernel of the library bounds; otherwise it waits
 * until the device int *flag equals expect.  Errors: SPA_ERR_INVALID,
 * SPA_ERR_CUDA. */
int spa_debug_fail_alloc_after(long long n);
int spa_debug_bounded_wait(spa_workspace *ws, const int *flag, int expect, double limit_us, void *stream);

/* ------------------------------------------------- allocation-free variant --
 * No counterpart on the pages: an engineering addition for callers that may
 * not allocate device memory (custom memory managers and allocator hooks that
 * must not re-enter the CUDA allocator, hosts that give the library a fixed
 * memory budget up front, loops where an allocation's implicit device
 * synchronisation is not allowed).
 *
 * The sparse-query attention of spa_partial_block on its own, bf16, head_dim
 * 128: O = softmax(Q K^cT / sqrt(head_dim)) V^c per head over all N cached
 * rows.  Q [B, k, n_heads * 128] (the compact selected queries, post-RoPE),
 * k_cache, v_cache [B, N, n_heads * 128], O [B, k, n_heads * 128]: device,
 * bf16, row-major, caller-owned.  It allocates nothing: the split-over-keys
 * partials, the per-query-tile split counters and a device error word live
 * in one fixed 8 MiB array inside the library (held on every GPU that loads
 * it until the process exits).  The keys of a query tile are split across
 * CTAs only as far as that array holds the partials (B * k * (n_heads * 130)
 * fp32 values within 2 Mi floats, and B * n_heads * ceil(k / 128) query tiles
 * within 4096 counters); a larger call is not refused but splits less, down to
 * no split, which needs no scratch (it is then slower for long caches).  The
 * first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call on a device shares the array: calls
 * whose work overlaps on the GPU (other streams, other host threads) race, so
 * order them on one stream.  Errors: SPA_ERR_INVALID (null pointer),
 * SPA_ERR_SHAPE (k > N, or B, n_heads or the cache beyond the launch limits:
 * B, n_heads <= 65535 and fewer than 2^31 elements per cache),
 * SPA_ERR_UNSUPPORTED (head_dim != 128), SPA_ERR_CUDA; details in
 * spa_last_error().  Device-side failures (a bounded wait that ran out) are
 * kept in the error word until spa_attention_noalloc_status reads them. */
int spa_attention_noalloc(const void *Q, const void *k_cache, const void *v_cache, void *O, int B,
                          int k, int N, int n_heads, int head_dim, void *stream);
/* Synchronises `stream`, then reads and clears the error word of the
 * allocation-free attention on the current device (into host stack memory:
 * it allocates nothing either): SPA_OK, SPA_ERR_TIMEOUT (a bounded wait of
 * some call since the last read ran out; that call's O rows are not valid)
 * or SPA_ERR_DEVICE; SPA_ERR_CUDA if the stream or the copy failed. */
int spa_attention_noalloc_status(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SPA_H */
