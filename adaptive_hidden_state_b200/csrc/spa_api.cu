// Host side of libspa: argument checks, workspace and handle management,
// tensor-map encoding and the launch sequence of each C-ABI call.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include <cuda_bf16.h>

#include "../../include/spa.h"
#include "spa_internal.h"

namespace spa {
int singular_proxy_host(const float* w_v, int d, int r, float* w_r, int iters);
}

using namespace spa;

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
static thread_local char g_last_error[512] = "";

static int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

#define SPA_CK(call)                                                                     \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess) return fail(SPA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define SPA_TRY(expr)          \
  do {                         \
    int s_ = (expr);           \
    if (s_ != SPA_OK) return s_; \
  } while (0)

// ---------------------------------------------------------------------------
// kernel timing (events per launch, off by default) and the launch counter
// ---------------------------------------------------------------------------
static long long g_launches = 0;

struct ProfRec {
  int cls;
  cudaEvent_t a, b;
  double bytes, flops;
};

struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> free_events;
  std::vector<ProfRec> recs;
  cudaEvent_t get() {
    if (!free_events.empty()) {
      cudaEvent_t e = free_events.back();
      free_events.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return e;
  }
  void release_all() {
    for (auto& r : recs) {
      free_events.push_back(r.a);
      free_events.push_back(r.b);
    }
    recs.clear();
  }
  ~Profiler() {
    release_all();
    for (cudaEvent_t e : free_events) cudaEventDestroy(e);
  }
};

// Brackets one kernel launch with events when profiling is on; counts it.
struct ProfScope {
  Profiler* p;
  int cls;
  double bytes, flops;
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  ProfScope(Profiler* prof, int c, double by, double fl, cudaStream_t st)
      : p(prof), cls(c), bytes(by), flops(fl), s(st) {
    ++g_launches;
    if (p && p->on) {
      a = p->get();
      b = p->get();
      if (a && b) cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    if (a && b) {
      cudaEventRecord(b, s);
      p->recs.push_back({cls, a, b, bytes, flops});
    }
  }
};

extern "C" const char* spa_status_string(int status) {
  switch (status) {
    case SPA_OK: return "SPA_OK";
    case SPA_ERR_INVALID: return "SPA_ERR_INVALID";
    case SPA_ERR_SHAPE: return "SPA_ERR_SHAPE";
    case SPA_ERR_CUDA: return "SPA_ERR_CUDA";
    case SPA_ERR_NOMEM: return "SPA_ERR_NOMEM";
    case SPA_ERR_UNSUPPORTED: return "SPA_ERR_UNSUPPORTED";
    case SPA_ERR_TIMEOUT: return "SPA_ERR_TIMEOUT";
    case SPA_ERR_DEVICE: return "SPA_ERR_DEVICE";
    default: return "SPA_ERR_UNKNOWN";
  }
}

extern "C" const char* spa_last_error(void) { return g_last_error; }

int spa::set_last_error(int status, const char* msg) { return fail(status, "%s", msg); }
extern "C" int spa_version(void) { return 100; }

// ---------------------------------------------------------------------------
// budget
// ---------------------------------------------------------------------------
extern "C" double spa_rho(int l, int L, double rho_p, int l_p, double rho_1, double rho_L) {
  if (L < 1 || l < 1 || l > L || l_p < 1 || l_p > L || !(rho_p > 0) || !(rho_1 > 0) ||
      !(rho_L > 0) || !std::isfinite(rho_p) || !std::isfinite(rho_1) || !std::isfinite(rho_L))
    return NAN;
  if (l <= l_p) {
    if (l_p == 1) return rho_p;
    const double t = (double)(l - l_p) / (double)(l_p - 1);
    return rho_p * std::exp(std::log(rho_1 / rho_p) * t * t);
  }
  const double t = (double)(l - l_p) / (double)(L - l_p);
  return rho_p * std::exp(std::log(rho_L / rho_p) * t * t);
}

extern "C" int spa_budget_k(int N, double rho) {
  if (N < 1 || !std::isfinite(rho) || !(rho > 0)) return -1;
  const double x = std::ceil((double)N * rho);
  if (x >= (double)N) return N;
  if (x < 1.0) return 1;
  return (int)x;
}

extern "C" int spa_singular_proxy_host(const float* w_v, int d, int r, float* w_r_out) {
  if (!w_v || !w_r_out) return fail(SPA_ERR_INVALID, "spa_singular_proxy_host: null pointer");
  if (d < 1 || r < 1 || r > d) return fail(SPA_ERR_SHAPE, "spa_singular_proxy_host: bad d=%d r=%d", d, r);
  try {
    if (singular_proxy_host(w_v, d, r, w_r_out, 24) != 0)
      return fail(SPA_ERR_INVALID, "spa_singular_proxy_host failed");
  } catch (const std::bad_alloc&) {
    return fail(SPA_ERR_NOMEM, "spa_singular_proxy_host: host allocation failed");
  }
  return SPA_OK;
}

// ---------------------------------------------------------------------------
// handles
// ---------------------------------------------------------------------------
// SMs of the device, recorded when a workspace is created (GEMM planning).
static int ws_num_sms_hint = 148;

struct spa_workspace {
  spa_layer_desc desc;
  int device = 0;
  int max_B = 0, max_N = 0, cap = 0;  // cap = max_B * max_N token rows
  size_t elem = 4;
  float* a_hat = nullptr;   // [cap, r]
  float* score = nullptr;   // [cap]
  float* proxy_raw = nullptr;  // [cap, r] raw proxies when r > 256 (bf16)
  int32_t* idx = nullptr;   // [cap]
  void* X = nullptr;        // [cap, d]
  void* Q = nullptr;        // [cap, d]
  void* O = nullptr;        // [cap, d]
  void* H1 = nullptr;       // [cap, d]
  void* X2 = nullptr;       // [cap, d]
  void* A = nullptr;        // [cap, F]
  float* part_o = nullptr;  // attention split partials
  float* part_ml = nullptr;
  int part_rows = 0;
  int* attn_sync = nullptr;  // per query tile: attention key splits finished
  int attn_sync_len = 0;
  int* err = nullptr;       // [2]
  float* sk_part = nullptr;  // stream-K GEMM: the segments' partial tiles (fp32)
  size_t sk_part_floats = 0;
  float* ffn_part = nullptr;  // persistent FFN: the three phases' partial tiles (fp32)
  size_t ffn_part_floats = 0;
  int* ffn_sync = nullptr;    // persistent FFN: [8] phase counters
  float* ss_part = nullptr;   // folded FFN RMSNorm: per (token, 128-feature tile) sums of H1^2
  float* gs_part = nullptr;   // weight-stationary split-K through global memory: the splits' partial tiles
  size_t gs_part_floats = 0;
  int* gs_counter = nullptr;  // [2 * kWsCounters] its per-tile arrival and departure counts
  float* rope_cos = nullptr;  // [max_N, hd/2]
  float* rope_sin = nullptr;
  CUtensorMap tmX, tmO, tmX2, tmA;
  int num_sms = 148;
  std::vector<void*> allocs;
  Profiler prof;
};

struct spa_layer {
  spa_layer_desc desc;
  spa_layer_weights w;
  spa_workspace* ws = nullptr;
  void* w_r = nullptr;      // [r, d] dtype
  CUtensorMap tm_wq, tm_wk, tm_wv, tm_wo, tm_wg, tm_wu, tm_wd, tm_wr;
  CUtensorMap tm_wg64, tm_wu64;  // W_gate, W_up with 64-row boxes (stream-K gate/up tiles)
};

struct spa_model {
  spa_model_desc desc;
  std::vector<spa_layer*> layers;
  std::vector<spa_layer_cache> caches;
  std::vector<int> k;
  void* h0 = nullptr;
  const void* embed = nullptr;
  const void* final_norm = nullptr;
  const void* lm_head = nullptr;
  int32_t* idx_all = nullptr;  // [L, B, N] index sets of the last step
  float* amax_val = nullptr;   // [B*N, n_tiles]
  int32_t* amax_idx = nullptr;
  float* amax_sum = nullptr;   // [B*N, n_tiles] sums of exp for the argmax probability
  int lm_tiles = 0;
  CUtensorMap tm_lm;
  cudaGraphExec_t graph = nullptr;  // a captured cached decode step
  int graph_u = 0;
  // incremental proxy: per layer, the unit proxy of every row's current input
  // and its drift score, kept across steps; only rows whose input changed are
  // projected again (the previous layer's index set, or the unmasked rows at
  // layer 0), whose new input rows the previous kernels leave compact in chg_rows
  bool inc = false;           // incremental proxy enabled
  bool inc_valid = false;     // ahat_all / score_all / chg_rows describe the current state
  int graph_inc = 0;          // the captured step: 0 plain, 1 proxy state refreshed, 2 incremental
  int graph_kernels = 0;      // kernel nodes of the captured step
  float* ahat_all = nullptr;  // [L, B, N, r]
  float* score_all = nullptr; // [L, B, N]
  void* chg_rows = nullptr;   // [B*N, d] compact changed rows (layer input of the next proxy)
  int32_t* chg0_idx = nullptr;  // [B*N] rows changed at layer 0 (the last unmasked positions)
  int chg0_u = 0;
};

static int check_desc(const spa_layer_desc* d) {
  if (!d) return fail(SPA_ERR_INVALID, "null layer descriptor");
  if (d->dtype != SPA_F32 && d->dtype != SPA_BF16) return fail(SPA_ERR_INVALID, "dtype must be SPA_F32 or SPA_BF16");
  if (d->d < 4 || d->n_heads < 1 || d->head_dim < 2 || d->ffn < 4 || d->r < 1)
    return fail(SPA_ERR_SHAPE, "non-positive dimension");
  if (d->n_heads * d->head_dim != d->d) return fail(SPA_ERR_SHAPE, "d != n_heads * head_dim");
  if (d->head_dim % 8 != 0 || d->head_dim > 128) return fail(SPA_ERR_UNSUPPORTED, "head_dim must be a multiple of 8, <= 128");
  if (d->r > d->d) return fail(SPA_ERR_SHAPE, "r > d");
  if (d->d > 8192) return fail(SPA_ERR_UNSUPPORTED, "d must be <= 8192");
  if (!(d->rms_eps > 0.f) || !(d->rope_theta > 0.f)) return fail(SPA_ERR_INVALID, "eps and theta must be positive");
  if (d->dtype == SPA_BF16) {
    if (d->d % 256 != 0) return fail(SPA_ERR_UNSUPPORTED, "bf16: d must be a multiple of 256");
    if (d->ffn % 128 != 0) return fail(SPA_ERR_UNSUPPORTED, "bf16: ffn must be a multiple of 128");
    if (d->r > 256 && d->r % 4 != 0) return fail(SPA_ERR_UNSUPPORTED, "bf16: r > 256 must be a multiple of 4");
  } else {
    if (d->d % 4 != 0 || d->ffn % 4 != 0) return fail(SPA_ERR_UNSUPPORTED, "f32: d and ffn must be multiples of 4");
    if (d->r > 128) return fail(SPA_ERR_UNSUPPORTED, "f32: r must be <= 128");
    if (128 % d->head_dim != 0) return fail(SPA_ERR_UNSUPPORTED, "f32: head_dim must divide 128");
  }
  return SPA_OK;
}

// Failure injection for tests of the error paths: after this many more
// successful device allocations, the next one fails once (negative: never).
static std::atomic<long long> g_fail_alloc_after{-1};

// Every device allocation of the library goes through here.
static cudaError_t dev_alloc(void** p, size_t bytes) {
  long long n = g_fail_alloc_after.load();
  while (n >= 0) {
    if (g_fail_alloc_after.compare_exchange_weak(n, n - 1)) {
      if (n == 0) {
        *p = nullptr;
        return cudaErrorMemoryAllocation;
      }
      break;
    }
  }
  return cudaMalloc(p, bytes);
}

extern "C" int spa_debug_fail_alloc_after(long long n) {
  g_fail_alloc_after.store(n < 0 ? -1 : n);
  return SPA_OK;
}

static int ws_alloc(spa_workspace* ws, void** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  cudaError_t e = dev_alloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(SPA_ERR_NOMEM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  }
  ws->allocs.push_back(*p);
  return SPA_OK;
}

// Stream-K plan of one weight-streaming GEMM: `tiles128` tiles of 128 weight
// rows, K / 64 k-blocks, NT tokens per MMA, on `sms` SMs.
struct SkPlan {
  int nacc, nbuf, n_tiles, KB, grid, maxseg;
};

static SkPlan sk_plan(int tiles128, int K, int NT, int sms, bool overrides) {
  SkPlan pl;
  // two 128-row tiles per unit halve the token-box traffic and the stages per
  // weight byte; GEMMs with few tiles keep one (their tiles split over more
  // CTAs, and two per unit would double the partials to sum)
  pl.nacc = (tiles128 % 2 == 0 && tiles128 >= 64) ? 2 : 1;
  if (overrides)
    if (const char* env = std::getenv("SPA_SK_NACC")) {  // tuning override, 1 or 2
      const int v = std::atoi(env);
      if ((v == 1 || v == 2) && tiles128 % v == 0) pl.nacc = v;
    }
  pl.nbuf = 2 * pl.nacc * NT <= 512 ? 2 : 1;
  pl.n_tiles = tiles128 / pl.nacc;
  pl.KB = K / 64;
  const int units = pl.n_tiles * pl.KB;
  // one CTA per SM, at least four k-blocks each
  pl.grid = std::max(1, std::min(sms, units / 4));
  if (overrides)
    if (const char* env = std::getenv("SPA_SK_GRID")) {  // tuning / test override, 1..SMs and <= units
      const int v = std::atoi(env);
      if (v >= 1 && v <= sms && v <= units) pl.grid = v;
    }
  // the reduce kernel takes at most sk_reduce_max_seg() segments per tile
  int mc = 0, mt = 0;
  for (;;) {
    sk_partition_bounds(pl.n_tiles, pl.KB, pl.grid, &mc, &mt);
    if (mt <= sk_reduce_max_seg() || pl.grid == 1) break;
    --pl.grid;
  }
  pl.maxseg = mc;
  return pl;
}

// Scratch floats the stream-K GEMMs of a layer of width d and FFN width F need
// at the widest token count (256) with either tile width.
static size_t sk_scratch_floats(int sms, int d, int F) {
  const int gemm[4][2] = {{3 * d / 128, d}, {d / 128, d}, {F / 64, d}, {d / 128, F}};
  size_t need = 0;
  for (const auto& gk : gemm)
    for (int nacc = 1; nacc <= 2; ++nacc) {
      if (gk[0] % nacc) continue;
      for (int NT = 32; NT <= 256; NT += 32) {
        SkPlan pl = sk_plan(gk[0], gk[1], NT, sms, false);
        pl.nacc = nacc;  // both widths, whatever the default
        pl.n_tiles = gk[0] / nacc;
        const int units = pl.n_tiles * pl.KB;
        for (int grid = 1; grid <= std::min(sms, units); ++grid) {
          int mc = 0, mt = 0;
          sk_partition_bounds(pl.n_tiles, pl.KB, grid, &mc, &mt);
          need = std::max(need, (size_t)grid * mc * NT * nacc * 128);
        }
      }
    }
  return need;
}

// Plan of the persistent FFN for NT tokens per MMA on `sms` SMs: per phase
// (O-proj, gate/up, down) the tile width, tiles, k-blocks, units, the
// busiest CTA's segments and the total; one grid for all three phases.
struct FfnPlan {
  int nacc[3], n_tiles[3], KB[3], units[3], maxseg[3], seg_total[3], grid;
  size_t part_floats[3];
  bool ok;
};

static FfnPlan ffn_plan(int d, int F, int NT, int sms) {
  FfnPlan pl;
  std::memset(&pl, 0, sizeof(pl));
  const int tiles128[3] = {d / 128, F / 64, d / 128}, K[3] = {d, d, F};
  int min_units = 1 << 30;
  for (int ph = 0; ph < 3; ++ph) {
    // two 128-row gate/up tiles per unit while two TMEM buffers of both fit
    pl.nacc[ph] = (ph == 1 && NT <= 128 && tiles128[ph] % 2 == 0) ? 2 : 1;
    if (const char* env = std::getenv("SPA_FFN_NACC"))  // tuning override of the gate/up width
      if (ph == 1 && env[0] == '1') pl.nacc[ph] = 1;
    pl.n_tiles[ph] = tiles128[ph] / pl.nacc[ph];
    pl.KB[ph] = K[ph] / 64;
    pl.units[ph] = pl.n_tiles[ph] * pl.KB[ph];
    min_units = std::min(min_units, pl.units[ph]);
  }
  pl.grid = std::max(1, std::min(sms, min_units / 4));
  if (const char* env = std::getenv("SPA_FFN_GRID")) {  // tuning / test override, 1..SMs and <= units
    const int v = std::atoi(env);
    if (v >= 1 && v <= sms && v <= min_units) pl.grid = v;
  }
  pl.ok = true;
  for (;;) {
    bool fits = true;
    for (int ph = 0; ph < 3; ++ph) {
      int mc = 0, mt = 0;
      sk_partition_bounds(pl.n_tiles[ph], pl.KB[ph], pl.grid, &mc, &mt);
      if (mt > ffn_max_seg()) fits = false;
      pl.maxseg[ph] = mc;
    }
    if (fits || pl.grid == 1) {
      pl.ok = fits;
      break;
    }
    --pl.grid;
  }
  for (int ph = 0; ph < 3; ++ph) {
    if (pl.n_tiles[ph] > ffn_max_tiles()) pl.ok = false;
    // every CTA's segments of the phase
    const int U = pl.units[ph], KB = pl.KB[ph];
    int tot = 0;
    for (int g = 0; g < pl.grid; ++g) {
      const int a = (int)(((long long)g * U) / pl.grid), b = (int)(((long long)(g + 1) * U) / pl.grid);
      if (b > a) tot += (b - 1) / KB - a / KB + 1;
    }
    pl.seg_total[ph] = tot;
    pl.part_floats[ph] = (size_t)pl.grid * pl.maxseg[ph] * NT * pl.nacc[ph] * 128;
  }
  return pl;
}

static size_t ffn_scratch_floats(int sms, int d, int F) {
  size_t need = 0;
  for (int NT = 32; NT <= 256; NT += 32) {
    const FfnPlan pl = ffn_plan(d, F, NT, sms);
    need = std::max(need, pl.part_floats[0] + pl.part_floats[1] + pl.part_floats[2]);
  }
  return need;
}

extern "C" void spa_workspace_free(spa_workspace* ws) {
  if (!ws) return;
  for (void* p : ws->allocs) cudaFree(p);
  delete ws;
}

extern "C" int spa_workspace_create(const spa_layer_desc* desc, int max_B, int max_N,
                                    spa_workspace** out) {
  if (!out) return fail(SPA_ERR_INVALID, "null output handle");
  *out = nullptr;
  SPA_TRY(check_desc(desc));
  if (max_B < 1 || max_N < 1) return fail(SPA_ERR_SHAPE, "max_B and max_N must be >= 1");
  if (max_N > 8192) return fail(SPA_ERR_UNSUPPORTED, "N > 8192 is not supported by the top-k select");
  if ((long long)max_B * max_N > (1ll << 24)) return fail(SPA_ERR_SHAPE, "max_B * max_N too large");
  spa_workspace* ws = new (std::nothrow) spa_workspace();
  if (!ws) return fail(SPA_ERR_NOMEM, "host allocation failed");
  ws->desc = *desc;
  ws->max_B = max_B;
  ws->max_N = max_N;
  ws->cap = max_B * max_N;
  ws->elem = desc->dtype == SPA_BF16 ? 2 : 4;
  cudaGetDevice(&ws->device);
  cudaDeviceGetAttribute(&ws->num_sms, cudaDevAttrMultiProcessorCount, ws->device);
  if (ws->num_sms > 0) ws_num_sms_hint = ws->num_sms;
  const size_t cap = ws->cap, d = desc->d, F = desc->ffn, r = desc->r, e = ws->elem;
  ws->part_rows = (int)std::min<size_t>(cap, 4096) * 4;
  int st = SPA_OK;
  void* p;
#define WS_ALLOC(field, bytes) \
  if (st == SPA_OK) { st = ws_alloc(ws, &p, (bytes)); if (st == SPA_OK) ws->field = (decltype(ws->field))p; }
  WS_ALLOC(a_hat, cap * r * 4)
  WS_ALLOC(score, cap * 4)
  if (desc->dtype == SPA_BF16 && r > 256) WS_ALLOC(proxy_raw, cap * r * 4)
  WS_ALLOC(idx, cap * 4)
  WS_ALLOC(X, cap * d * e)
  WS_ALLOC(Q, cap * d * e)
  WS_ALLOC(O, cap * d * e)
  WS_ALLOC(H1, cap * d * e)
  WS_ALLOC(X2, cap * d * e)
  WS_ALLOC(A, cap * F * e)
  WS_ALLOC(part_o, (size_t)ws->part_rows * d * 4)
  WS_ALLOC(part_ml, (size_t)ws->part_rows * desc->n_heads * 2 * 4)
  ws->attn_sync_len = max_B * desc->n_heads * ((max_N + 127) / 128);
  WS_ALLOC(attn_sync, (size_t)ws->attn_sync_len * sizeof(int))
  WS_ALLOC(err, 2 * sizeof(int))
  if (desc->dtype == SPA_BF16) {
    ws->sk_part_floats = sk_scratch_floats(ws->num_sms, (int)d, (int)F);
    WS_ALLOC(sk_part, ws->sk_part_floats * 4)
    ws->ffn_part_floats = ffn_scratch_floats(ws->num_sms, (int)d, (int)F);
    WS_ALLOC(ffn_part, ws->ffn_part_floats * 4)
    WS_ALLOC(ffn_sync, 8 * sizeof(int))
    WS_ALLOC(ss_part, std::min<size_t>(cap, 256) * ((d + 127) / 128) * 4)
    // one partial tile of at most 512 accumulator columns x 128 rows per SM
    ws->gs_part_floats = (size_t)ws->num_sms * 512 * 128;
    WS_ALLOC(gs_part, ws->gs_part_floats * 4)
    WS_ALLOC(gs_counter, 2 * kWsCounters * sizeof(int))
  }
  WS_ALLOC(rope_cos, (size_t)max_N * (desc->head_dim / 2) * 4)
  WS_ALLOC(rope_sin, (size_t)max_N * (desc->head_dim / 2) * 4)
#undef WS_ALLOC
  if (st != SPA_OK) {
    spa_workspace_free(ws);
    return st;
  }
  // RoPE table in double precision: angle = pos * theta^(-2i/hd)
  const int hh = desc->head_dim / 2;
  std::vector<float> cs((size_t)max_N * hh), sn((size_t)max_N * hh);
  for (int pos = 0; pos < max_N; ++pos)
    for (int i = 0; i < hh; ++i) {
      const double inv = std::pow((double)desc->rope_theta, -2.0 * i / (double)desc->head_dim);
      const double a = (double)pos * inv;
      cs[(size_t)pos * hh + i] = (float)std::cos(a);
      sn[(size_t)pos * hh + i] = (float)std::sin(a);
    }
  if (cudaMemcpy(ws->rope_cos, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(ws->rope_sin, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(ws->err, 0, 2 * sizeof(int)) != cudaSuccess ||
      cudaMemset(ws->attn_sync, 0, (size_t)ws->attn_sync_len * sizeof(int)) != cudaSuccess ||
      (ws->ffn_sync && cudaMemset(ws->ffn_sync, 0, 8 * sizeof(int)) != cudaSuccess) ||
      (ws->gs_counter && cudaMemset(ws->gs_counter, 0, 2 * kWsCounters * sizeof(int)) != cudaSuccess)) {
    spa_workspace_free(ws);
    return fail(SPA_ERR_CUDA, "workspace initialisation copy failed");
  }
  if (desc->dtype == SPA_BF16) {
    if (encode_bf16_map(&ws->tmX, ws->X, cap, d) || encode_bf16_map(&ws->tmO, ws->O, cap, d) ||
        encode_bf16_map(&ws->tmX2, ws->X2, cap, d) || encode_bf16_map(&ws->tmA, ws->A, cap, F)) {
      spa_workspace_free(ws);
      return fail(SPA_ERR_CUDA, "tensor map encoding failed");
    }
  }
  *out = ws;
  return SPA_OK;
}

extern "C" int spa_workspace_status(spa_workspace* ws, void* stream) {
  if (!ws) return fail(SPA_ERR_INVALID, "null workspace");
  SPA_CK(cudaStreamSynchronize((cudaStream_t)stream));
  int h[2] = {0, 0};
  SPA_CK(cudaMemcpy(h, ws->err, sizeof(h), cudaMemcpyDeviceToHost));
  if (h[0] == 0) return SPA_OK;
  SPA_CK(cudaMemset(ws->err, 0, sizeof(h)));
  // a kernel that gave up may have left split counters behind: start them afresh
  SPA_CK(cudaMemset(ws->attn_sync, 0, (size_t)ws->attn_sync_len * sizeof(int)));
  if (ws->ffn_sync) SPA_CK(cudaMemset(ws->ffn_sync, 0, 8 * sizeof(int)));
  if (ws->gs_counter) SPA_CK(cudaMemset(ws->gs_counter, 0, 2 * kWsCounters * sizeof(int)));
  if (h[0] & DEVERR_TIMEOUT) return fail(SPA_ERR_TIMEOUT, "device wait timed out (site %d)", h[1]);
  return fail(SPA_ERR_DEVICE, "device check failed: bits 0x%x site %d", h[0], h[1]);
}

extern "C" int spa_debug_bounded_wait(spa_workspace* ws, const int* flag, int expect, double limit_us,
                                      void* stream) {
  if (!ws) return fail(SPA_ERR_INVALID, "null workspace");
  if (!(limit_us >= 0.0) || limit_us > 1e6) return fail(SPA_ERR_INVALID, "limit_us must be in [0, 1e6]");
  const cudaError_t e = launch_wait_probe(flag, expect, (unsigned long long)(limit_us * 1e3), ws->err,
                                          (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "wait probe launch: %s", cudaGetErrorString(e));
  ++g_launches;
  return SPA_OK;
}

extern "C" int spa_workspace_intermediates(const spa_workspace* ws, spa_intermediates* out) {
  if (!ws || !out) return fail(SPA_ERR_INVALID, "null argument");
  out->x = ws->X;
  out->q = ws->Q;
  out->o = ws->O;
  out->h1 = ws->H1;
  out->x2 = ws->X2;
  out->a = ws->A;
  out->a_hat = ws->a_hat;
  out->score = ws->score;
  return SPA_OK;
}

extern "C" int spa_profile_enable(spa_workspace* ws, int enable) {
  if (!ws) return fail(SPA_ERR_INVALID, "null workspace");
  ws->prof.on = enable != 0;
  return SPA_OK;
}

extern "C" int spa_profile_read(spa_workspace* ws, int* launches, double* ms, double* bytes,
                                double* flops) {
  if (!ws || !launches || !ms || !bytes || !flops) return fail(SPA_ERR_INVALID, "null argument");
  for (int c = 0; c < SPA_PROF_CLASSES; ++c) {
    launches[c] = 0;
    ms[c] = bytes[c] = flops[c] = 0.0;
  }
  int st = SPA_OK;
  for (auto& r : ws->prof.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();
      st = fail(SPA_ERR_CUDA, "reading kernel timing events failed");
      continue;
    }
    launches[r.cls] += 1;
    ms[r.cls] += t;
    bytes[r.cls] += r.bytes;
    flops[r.cls] += r.flops;
  }
  ws->prof.release_all();
  return st;
}

extern "C" long long spa_launch_count(void) { return g_launches; }

extern "C" void spa_free_layer(spa_layer* layer) {
  if (!layer) return;
  if (layer->w_r) cudaFree(layer->w_r);
  delete layer;
}

extern "C" int spa_init_layer(const spa_layer_desc* desc, const spa_layer_weights* w,
                              const float* w_r_host, spa_workspace* ws, spa_layer** out) {
  if (!out) return fail(SPA_ERR_INVALID, "null output handle");
  *out = nullptr;
  SPA_TRY(check_desc(desc));
  if (!w || !ws) return fail(SPA_ERR_INVALID, "null weights or workspace");
  if (!w->wq || !w->wk || !w->wv || !w->wo || !w->w_gate || !w->w_up || !w->w_down ||
      !w->attn_norm || !w->ffn_norm)
    return fail(SPA_ERR_INVALID, "null weight pointer");
  if (std::memcmp(desc, &ws->desc, sizeof(spa_layer_desc)) != 0)
    return fail(SPA_ERR_SHAPE, "layer descriptor differs from the workspace's");
  const int d = desc->d, r = desc->r;
  std::vector<float> wr;
  try {
    wr.resize((size_t)r * d);
    if (w_r_host) {
      std::memcpy(wr.data(), w_r_host, wr.size() * 4);
    } else {
      std::vector<float> wv((size_t)d * d);
      if (desc->dtype == SPA_BF16) {
        std::vector<__nv_bfloat16> tmp((size_t)d * d);
        SPA_CK(cudaMemcpy(tmp.data(), w->wv, tmp.size() * 2, cudaMemcpyDeviceToHost));
        for (size_t i = 0; i < tmp.size(); ++i) wv[i] = __bfloat162float(tmp[i]);
      } else {
        SPA_CK(cudaMemcpy(wv.data(), w->wv, wv.size() * 4, cudaMemcpyDeviceToHost));
      }
      SPA_TRY(spa_singular_proxy_host(wv.data(), d, r, wr.data()));
    }
  } catch (const std::bad_alloc&) {
    return fail(SPA_ERR_NOMEM, "host allocation failed");
  }
  spa_layer* L = new (std::nothrow) spa_layer();
  if (!L) return fail(SPA_ERR_NOMEM, "host allocation failed");
  L->desc = *desc;
  L->w = *w;
  L->ws = ws;
  const size_t e = desc->dtype == SPA_BF16 ? 2 : 4;
  if (dev_alloc(&L->w_r, (size_t)r * d * e) != cudaSuccess) {
    cudaGetLastError();
    delete L;
    return fail(SPA_ERR_NOMEM, "cudaMalloc of the proxy weights failed");
  }
  int st = SPA_OK;
  if (desc->dtype == SPA_BF16) {
    std::vector<__nv_bfloat16> b((size_t)r * d);
    for (size_t i = 0; i < b.size(); ++i) b[i] = __float2bfloat16_rn(wr[i]);
    if (cudaMemcpy(L->w_r, b.data(), b.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess)
      st = fail(SPA_ERR_CUDA, "proxy weight upload failed");
    const uint64_t D = d, F = desc->ffn;
    if (st == SPA_OK &&
        (encode_bf16_map(&L->tm_wq, w->wq, D, D) || encode_bf16_map(&L->tm_wk, w->wk, D, D) ||
         encode_bf16_map(&L->tm_wv, w->wv, D, D) || encode_bf16_map(&L->tm_wo, w->wo, D, D) ||
         encode_bf16_map(&L->tm_wg, w->w_gate, F, D) || encode_bf16_map(&L->tm_wu, w->w_up, F, D) ||
         encode_bf16_map(&L->tm_wd, w->w_down, D, F) || encode_bf16_map(&L->tm_wr, L->w_r, r, D) ||
         encode_bf16_map_box(&L->tm_wg64, w->w_gate, F, D, 64) || encode_bf16_map_box(&L->tm_wu64, w->w_up, F, D, 64)))
      st = fail(SPA_ERR_CUDA, "tensor map encoding failed (weights must be 16-byte aligned)");
  } else {
    if (cudaMemcpy(L->w_r, wr.data(), wr.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      st = fail(SPA_ERR_CUDA, "proxy weight upload failed");
  }
  if (st != SPA_OK) {
    spa_free_layer(L);
    return st;
  }
  *out = L;
  return SPA_OK;
}

extern "C" int spa_layer_proxy_weights(const spa_layer* layer, float* w_r_out) {
  if (!layer || !w_r_out) return fail(SPA_ERR_INVALID, "null argument");
  const size_t n = (size_t)layer->desc.r * layer->desc.d;
  if (layer->desc.dtype == SPA_BF16) {
    std::vector<__nv_bfloat16> b(n);
    SPA_CK(cudaMemcpy(b.data(), layer->w_r, n * 2, cudaMemcpyDeviceToHost));
    for (size_t i = 0; i < n; ++i) w_r_out[i] = __bfloat162float(b[i]);
  } else {
    SPA_CK(cudaMemcpy(w_r_out, layer->w_r, n * 4, cudaMemcpyDeviceToHost));
  }
  return SPA_OK;
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------
static EpiParams base_epi(const spa_layer* L, int M, int tps, int N, const int32_t* idx) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.M = M;
  ep.d = L->desc.d;
  ep.head_dim = L->desc.head_dim;
  ep.tokens_per_seq = tps;
  ep.N = N;
  ep.idx = idx;
  ep.rope_cos = L->ws->rope_cos;
  ep.rope_sin = L->ws->rope_sin;
  ep.err = L->ws->err;
  return ep;
}

// Number of K-splits for a weight-streaming GEMM: as many CTAs as fit one
// wave of the SMs, at least 4 k-blocks of 64 per CTA, cluster size <= 8.
static int choose_splits(int tiles, int KB, int sms) {
  int best = 1;
  for (int s = 1; s <= 8; ++s) {
    if (KB / s < 4) break;
    if (tiles * s <= sms) best = s;
  }
  return best;
}

// Algorithmic work of one launch, for the kernel timing record.
struct Work {
  int cls;
  double bytes, flops;
};

// Tiled tcgen05 GEMM over M token rows.  With KB (the k-blocks of 64) given,
// a layer GEMM of at least 512 rows takes 256-row tiles (twice the MMA work
// per staged byte) and its split-K is re-planned for the halved tile count;
// SPA_TC_BM=128 keeps 128-row tiles (tuning override).
static int run_tc(int mode, int BN, TcGemmParams& p, int M, int n_tiles, int splits, cudaStream_t s,
                  Profiler* prof, Work w, int KB = 0, int sms = 148) {
  int BM = 128;
  if (KB > 0 && BN == 256 && M >= 512 &&
      (mode == EPI_STORE || mode == EPI_QKV || mode == EPI_RESID || mode == EPI_SWIGLU ||
       mode == EPI_RESID_SCATTER)) {
    const char* env = std::getenv("SPA_TC_BM");
    if (!(env && std::atoi(env) == 128)) BM = 256;
  }
  const int m_tiles = (M + BM - 1) / BM;
  if (m_tiles == 0) return SPA_OK;
  if (BM == 256) splits = choose_splits(n_tiles * m_tiles, KB, sms);
  ProfScope ps(prof, w.cls, w.bytes, w.flops, s);
  if (m_tiles > 65535 || n_tiles > 65535) return fail(SPA_ERR_SHAPE, "GEMM grid too large");
  cudaError_t e = launch_tc_gemm(mode, BN, BM, p, m_tiles, n_tiles, splits, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "tc GEMM launch (mode %d): %s", mode, cudaGetErrorString(e));
  return SPA_OK;
}

// Weight-stationary tcgen05 GEMM for M <= 256 tokens: X is the [M, K] bf16
// token operand (row-major, 16-byte aligned); `rows` weight rows (for
// gate/up: features, each with a W_gate and a W_up row).  Each CTA keeps NACC
// accumulators of 128 rows so one token tile feeds up to 512 weight rows
// (NACC * NT <= 512 TMEM columns).
//
// ws_shape is its plan: NT tokens per MMA, NACC, the column tiles and the
// split-K cluster size.  Two 128-row blocks per CTA (gate/up: a W_gate and a
// W_up block) halve the token-tile traffic per weight byte: each CTA's TMA
// stream then moves 48 KB per stage for 32 KB of weights instead of 32 KB for
// 16 KB, which lets ~96 CTAs stream near the HBM rate.  A GEMM with fewer rows
// (O-proj, down: 32 blocks of 128) keeps one block per CTA so that its split-K
// clusters still cover the SMs.  Only a GEMM with many more weight rows than
// the SMs can cover (the LM head) takes four.  `fold`: the folded FFN norm
// sums a row's squares over 128-feature tiles, so one block.
struct WsShape {
  int NT, nacc, n_tiles, splits;
  bool global;  // the splits are separate CTAs that reduce through global memory
};
// g_floats: the global split-K scratch (0: none).
static WsShape ws_shape(int mode, bool gateup, bool fold, int M, int K, int rows, size_t g_floats = 0) {
  WsShape sh;
  sh.NT = ((M + 31) / 32) * 32;
  const int NT = sh.NT;
  const int min_nacc = gateup ? 2 : 1;
  int nacc = min_nacc;
  if (!gateup && rows % 256 == 0 && rows / 128 >= 64 && 2 * NT <= 512) nacc = 2;
  if (rows / 128 > 4 * ws_num_sms_hint)
    for (int n = 4; n > min_nacc; n /= 2) {
      const int feat = gateup ? n / 2 * 128 : n * 128;
      if (n * NT <= 512 && (rows + feat - 1) / feat >= 16) {
        nacc = n;
        break;
      }
    }
  if (const char* env = std::getenv("SPA_WS_NACC")) {  // tuning override
    const int v = std::atoi(env);
    if ((v == 1 || v == 2 || v == 4) && v >= min_nacc && v * NT <= 512) nacc = v;
  }
  if (fold) nacc = 1;
  const int feat = gateup ? nacc / 2 * 128 : nacc * 128;
  sh.nacc = nacc;
  sh.n_tiles = (rows + feat - 1) / feat;
  sh.splits = plan_ws_splits(mode, nacc, sh.n_tiles, K / 64);
  sh.global = false;
  // a split-K through global memory where it covers more SMs than the
  // clusters can (QKV: 48 two-block tiles x 3 splits = 144 CTAs, where only 45
  // clusters of 3 fit).  Tuning override SPA_WS_GLOBAL: 0 keeps the clusters;
  // 2..8 takes that many global splits when the grid is resident at once.
  const char* genv = std::getenv("SPA_WS_GLOBAL");
  const int gforce = genv ? std::atoi(genv) : -1;
  if (g_floats > 0 && sh.n_tiles <= kWsCounters && gforce != 0) {
    const size_t per = (size_t)sh.n_tiles * NT * nacc * 128;
    const int g_max = (int)std::min<size_t>(8, g_floats / per);
    int sg = plan_ws_global_splits(mode, nacc, sh.n_tiles, K / 64, g_max);
    if (gforce >= 2 && gforce <= g_max && K / 64 >= gforce && ws_resident_ctas(mode, nacc) >= sh.n_tiles * gforce)
      sg = gforce;
    if (sg > 1) {
      sh.splits = sg;
      sh.global = true;
    }
  }
  if (const char* env = std::getenv("SPA_WS_SPLITS")) {  // tuning override, 1..8 (clusters)
    const int v = std::atoi(env);
    if (v >= 1 && v <= 8 && K / 64 >= v) {
      sh.splits = v;
      sh.global = false;
    }
  }
  return sh;
}

static int run_ws(int mode, bool gateup, TcWsParams& p, spa_workspace* ws, const void* X, int M, int K,
                  int rows, cudaStream_t s, Profiler* prof, Work w) {
  if (M <= 0) return SPA_OK;
  if (M > 256) return fail(SPA_ERR_SHAPE, "weight-stationary GEMM takes at most 256 tokens");
  const WsShape sh = ws_shape(mode, gateup, p.ep.x2 != nullptr, M, K, rows, ws->gs_part ? ws->gs_part_floats : 0);
  const int NT = sh.NT, nacc = sh.nacc, n_tiles = sh.n_tiles;
  p.part = sh.global ? ws->gs_part : nullptr;
  p.counter = sh.global ? ws->gs_counter : nullptr;
  if (encode_bf16_map_box(&p.tmX, X, (uint64_t)M, (uint64_t)K, (uint32_t)NT))
    return fail(SPA_ERR_CUDA, "tensor map for the token operand failed");
  int cols = 32;
  while (cols < nacc * NT) cols *= 2;
  p.NT = NT;
  p.tmem_cols = cols;
  p.K = K;
  if (mode == EPI_ARGMAX) p.ep.n_tiles = n_tiles;
  ProfScope ps(prof, w.cls, w.bytes, w.flops, s);
  cudaError_t e = launch_tc_ws(mode, nacc, p, n_tiles, sh.splits, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "weight-stationary GEMM launch (mode %d): %s", mode, cudaGetErrorString(e));
  return SPA_OK;
}

// Stream-K weight-streaming GEMM (M <= 256 tokens): `tiles` weight tiles of
// 128 output features (gate/up: 64 features, 64 gate + 64 up rows) times the
// [M, K] bf16 token operand X, K / 64 k-blocks each, over one CTA per SM.
static bool streamk_enabled() {
  // opt-in (SPA_STREAMK=1): measured slower than the cluster split-K kernel on
  // the LLaDA-shaped layer, because the fp32 partials it writes and re-reads
  // cost more than its even spread over the SMs gains
  const char* e = std::getenv("SPA_STREAMK");
  return e && e[0] == '1';
}

static int run_sk(int mode, SkParams& p, spa_workspace* ws, const void* X, int M, int K, int tiles128,
                  cudaStream_t s, Profiler* prof, Work w, const void* gamma = nullptr, void* x2 = nullptr,
                  float eps = 0.f) {
  if (M <= 0) return SPA_OK;
  if (M > 256) return fail(SPA_ERR_SHAPE, "stream-K GEMM takes at most 256 tokens");
  const int NT = ((M + 31) / 32) * 32;
  if (encode_bf16_map_box(&p.tmX, X, (uint64_t)M, (uint64_t)K, (uint32_t)NT))
    return fail(SPA_ERR_CUDA, "tensor map for the token operand failed");
  const SkPlan pl = sk_plan(tiles128, K, NT, ws->num_sms, true);
  if (pl.n_tiles > sk_reduce_max_tiles()) return fail(SPA_ERR_SHAPE, "stream-K GEMM: too many weight tiles");
  const size_t slot_floats = (size_t)NT * pl.nacc * 128;
  if ((size_t)pl.grid * pl.maxseg * slot_floats > ws->sk_part_floats)
    return fail(SPA_ERR_SHAPE, "stream-K GEMM: scratch too small for the partition");
  int cols = 32;
  while (cols < pl.nbuf * pl.nacc * NT) cols *= 2;
  p.K = K;
  p.KB = pl.KB;
  p.NT = NT;
  p.nacc = pl.nacc;
  p.nbuf = pl.nbuf;
  p.n_tiles = pl.n_tiles;
  p.units = pl.n_tiles * pl.KB;
  p.tmem_cols = cols;
  p.maxseg = pl.maxseg;
  p.part = ws->sk_part;
  SkReduceParams r;
  std::memset(&r, 0, sizeof(r));
  r.part = ws->sk_part;
  r.slot_floats = slot_floats;
  r.feat = pl.nacc * 128;
  r.nacc = pl.nacc;
  r.n_tiles = pl.n_tiles;
  r.KB = pl.KB;
  r.G = pl.grid;
  r.U = p.units;
  r.maxseg = pl.maxseg;
  r.gamma = gamma;
  r.x2 = x2;
  r.eps = eps;
  r.ep = p.ep;
  ProfScope ps(prof, w.cls, w.bytes, w.flops, s);
  g_launches += 1;  // the reduce kernel (the scope counts the GEMM)
  cudaError_t e = launch_tc_sk(mode, p, pl.grid, r, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "stream-K GEMM launch (mode %d): %s", mode, cudaGetErrorString(e));
  return SPA_OK;
}

static int run_simt(int mode, SimtGemmParams& p, int M, int n_tiles, cudaStream_t s, Profiler* prof,
                    Work w) {
  const int m_tiles = (M + 63) / 64;
  if (m_tiles == 0) return SPA_OK;
  ProfScope ps(prof, w.cls, w.bytes, w.flops, s);
  cudaError_t e = launch_simt_gemm(mode, p, m_tiles, n_tiles, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "SIMT GEMM launch (mode %d): %s", mode, cudaGetErrorString(e));
  return SPA_OK;
}

static int check_cache(const spa_layer* L, const spa_layer_cache* c) {
  if (!c) return fail(SPA_ERR_INVALID, "null cache");
  if (!c->k_cache || !c->v_cache || !c->h_cache || !c->p_cache) return fail(SPA_ERR_INVALID, "null cache buffer");
  if (c->B < 1 || c->N < 1 || c->B > L->ws->max_B || c->N > L->ws->max_N ||
      (long long)c->B * c->N > L->ws->cap)
    return fail(SPA_ERR_SHAPE, "cache B=%d N=%d exceeds the workspace (B<=%d, N<=%d)", c->B, c->N,
                L->ws->max_B, L->ws->max_N);
  return SPA_OK;
}

// Phase 1: proxy GEMM with the fused norm / score epilogue (or the P^c fill).
// X holds tps token rows per sequence: every cache row (rows == null, tps = N)
// or the rows listed in `rows` ([B, tps] cache rows), compact.  a_hat and
// score are [B*N, r] and [B*N], written at the tokens' cache rows.
static int run_proxy_rows(spa_layer* L, const void* H, const int32_t* rows, int tps,
                          const spa_layer_cache* c, float* a_hat, float* score, int fill,
                          cudaStream_t s) {
  const int M = c->B * tps, d = L->desc.d, r = L->desc.r;
  if (M <= 0) return SPA_OK;
  EpiParams ep = base_epi(L, M, tps, c->N, rows);
  ep.n_out = r;
  ep.a_hat = a_hat;
  ep.p_cache = c->p_cache;
  ep.score = score;
  ep.proxy_fill = fill;
  const double e = L->desc.dtype == SPA_BF16 ? 2.0 : 4.0;
  // H read, W_r read, P^c read + a_hat write (or P^c write), scores
  const Work w{SPA_PROF_PROXY,
               (double)M * d * e + (double)r * d * e + (fill ? 1.0 : 2.0) * M * r * 4 + (fill ? 0 : 4.0 * M),
               2.0 * M * d * r};
  if (L->desc.dtype == SPA_BF16) {
    TcGemmParams p;
    std::memset(&p, 0, sizeof(p));
    if (encode_bf16_map(&p.tmA, H, (uint64_t)M, (uint64_t)d))
      return fail(SPA_ERR_CUDA, "tensor map for H failed (H must be 16-byte aligned)");
    p.tmB[0] = L->tm_wr;
    p.K = d;
    p.b_mode = B_SINGLE;
    p.b_rows_per_src = r;
    p.ep = ep;
    // split count depends on d only, so a row's proxy bits never depend on B or N
    int splits = std::max(1, std::min(16, (d / 64) / 4));
    if (const char* env = std::getenv("SPA_PROXY_SPLITS")) {  // tuning override (depends on d only)
      const int v = std::atoi(env);
      if (v >= 1 && v <= 16 && (d / 64) / v >= 1) splits = v;
    }
    if (r <= 256) return run_tc(EPI_PROXY, r <= 128 ? 128 : 256, p, M, 1, splits, s, &L->ws->prof, w);
    // wide r: raw proxies in 256-column tiles, then norms and scores per row
    p.ep.out = L->ws->proxy_raw;
    SPA_TRY(run_tc(EPI_PROXY_RAW, 256, p, M, (r + 255) / 256, splits, s, &L->ws->prof, w));
    ProfScope ps(&L->ws->prof, SPA_PROF_PROXY, (double)M * r * 4 * 3, 0.0, s);
    const cudaError_t e2 = launch_proxy_finish(L->ws->proxy_raw, M, r, tps, c->N, rows, a_hat, c->p_cache,
                                               score, fill, L->ws->err, s);
    if (e2 != cudaSuccess) return fail(SPA_ERR_CUDA, "proxy finish launch: %s", cudaGetErrorString(e2));
    return SPA_OK;
  }
  SimtGemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.A = (const float*)H;
  p.B[0] = (const float*)L->w_r;
  p.K = d;
  p.b_mode = B_SINGLE;
  p.b_rows_per_src = r;
  p.ep = ep;
  return run_simt(EPI_PROXY, p, M, 1, s, &L->ws->prof, w);
}

static int run_proxy(spa_layer* L, const void* H, const spa_layer_cache* c, float* score, int fill,
                     cudaStream_t s) {
  return run_proxy_rows(L, H, nullptr, c->N, c, fill ? nullptr : L->ws->a_hat, score, fill, s);
}

// Phases 2 and 3 for M = B * tps tokens; idx == null means every row (rho = 1).
// Phase 2: x = RMSNorm(H[I]), Q/K/V with RoPE, K^c/V^c[I] <- K, V, and the
// attention of the M = B * tps selected queries over the whole cache into
// ws->O (compact rows); idx == null means every row (rho = 1).
static int run_attn_half(spa_layer* L, const void* H, const int32_t* idx, int tps,
                         const spa_layer_cache* c, cudaStream_t s, bool x_ready) {
  spa_workspace* ws = L->ws;
  const spa_layer_desc& D = L->desc;
  const int d = D.d, M = c->B * tps, N = c->N;
  const bool bf = D.dtype == SPA_BF16;
  const double es = bf ? 2.0 : 4.0, Md = (double)M * d, Bn = (double)c->B * N;
  Profiler* prof = &ws->prof;
  cudaError_t e;
  // x = RMSNorm(H[I]) (already in ws->X when the select wrote it)
  if (!x_ready) {
    {
      ProfScope ps(prof, SPA_PROF_NORM, 2.0 * Md * es + d * es, 4.0 * Md, s);
      e = launch_rmsnorm_rows(D.dtype, H, 1, idx, tps, N, M, d, L->w.attn_norm, D.rms_eps, ws->X, ws->err, s);
    }
    if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "rmsnorm launch: %s", cudaGetErrorString(e));
  }
  // Q, K, V with RoPE; K, V scattered into the caches
  {
    EpiParams ep = base_epi(L, M, tps, N, idx);
    ep.n_out = 3 * d;
    ep.out = ws->Q;
    ep.k_cache = c->k_cache;
    ep.v_cache = c->v_cache;
    const int hd = D.head_dim;
    if (bf && M <= 256 && streamk_enabled() && (hd == 32 || hd == 64 || hd == 128)) {
      SkParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wq; p.tmW[1] = L->tm_wk; p.tmW[2] = L->tm_wv;
      p.b_mode = B_CONCAT3; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_sk(EPI_QKV, p, ws, ws->X, M, d, 3 * d / 128, s, prof,
                     Work{SPA_PROF_QKV, 3.0 * d * d * es + Md * es + 3.0 * Md * es, 6.0 * Md * d}));
    } else if (bf && M <= 256) {
      TcWsParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wq; p.tmW[1] = L->tm_wk; p.tmW[2] = L->tm_wv;
      p.b_mode = B_CONCAT3; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_ws(EPI_QKV, false, p, ws, ws->X, M, d, 3 * d, s, prof,
                     Work{SPA_PROF_QKV, 3.0 * d * d * es + Md * es + 3.0 * Md * es, 6.0 * Md * d}));
    } else if (bf) {
      TcGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmA = ws->tmX;
      p.tmB[0] = L->tm_wq; p.tmB[1] = L->tm_wk; p.tmB[2] = L->tm_wv;
      p.K = d; p.b_mode = B_CONCAT3; p.b_rows_per_src = d; p.ep = ep;
      const int nt = 3 * d / 256, mt = (M + 127) / 128;
      SPA_TRY(run_tc(EPI_QKV, 256, p, M, nt, choose_splits(nt * mt, d / 64, ws->num_sms), s, prof,
                     Work{SPA_PROF_QKV, 3.0 * d * d * es + Md * es + 3.0 * Md * es, 6.0 * Md * d}, d / 64, ws->num_sms));
    } else {
      SimtGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.A = (const float*)ws->X;
      p.B[0] = (const float*)L->w.wq; p.B[1] = (const float*)L->w.wk; p.B[2] = (const float*)L->w.wv;
      p.K = d; p.b_mode = B_CONCAT3; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_simt(EPI_QKV, p, M, (3 * d + 127) / 128, s, prof,
                       Work{SPA_PROF_QKV, 3.0 * d * d * es + Md * es + 3.0 * Md * es, 6.0 * Md * d}));
    }
  }
  // O = attention over the whole cache
  {
    ProfScope ps(prof, SPA_PROF_ATTN, 2.0 * Md * es + 2.0 * Bn * d * es, 4.0 * Md * N, s);
    e = launch_attention(D.dtype, ws->Q, c->k_cache, c->v_cache, ws->O, c->B, tps, N, D.n_heads,
                         D.head_dim, ws->part_o, ws->part_ml, ws->part_rows, ws->attn_sync,
                         ws->attn_sync_len, ws->err, 1, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
  return SPA_OK;
}

// Phase 3 for the M = B * tps selected rows whose attention outputs are the
// compact rows of Ob (tmOb: its tensor map, bf16): H1 = H[I] + O W_o^T,
// x2 = RMSNorm(H1), A = SwiGLU, H^c[I] = H1 + A W_down^T.
static bool ffn_persistent_enabled() {
  const char* e = std::getenv("SPA_FFN");
  return e && e[0] == '1';
}

// The persistent FFN half (M <= 256 bf16 tokens): one launch for the O-proj,
// the FFN RMSNorm, gate/up + SwiGLU and down + H^c scatter.  Returns
// SPA_ERR_UNSUPPORTED (nothing launched) when the shapes do not fit its plan.
static int run_ffn_persistent(spa_layer* L, const void* H, const int32_t* idx, int tps, const spa_layer_cache* c,
                              cudaStream_t s, const void* Ob, void* row_copy, float* score_zero) {
  spa_workspace* ws = L->ws;
  const spa_layer_desc& D = L->desc;
  const int d = D.d, F = D.ffn, M = c->B * tps;
  const int NT = ((M + 31) / 32) * 32;
  const FfnPlan pl = ffn_plan(d, F, NT, ws->num_sms);
  if (!pl.ok || pl.part_floats[0] + pl.part_floats[1] + pl.part_floats[2] > ws->ffn_part_floats)
    return SPA_ERR_UNSUPPORTED;
  FfnParams p;
  std::memset(&p, 0, sizeof(p));
  p.tmWo = L->tm_wo;
  p.tmWg = L->tm_wg64;
  p.tmWu = L->tm_wu64;
  p.tmWd = L->tm_wd;
  if (encode_bf16_map_box(&p.tmX[0], Ob, (uint64_t)M, (uint64_t)d, (uint32_t)NT) ||
      encode_bf16_map_box(&p.tmX[1], ws->X2, (uint64_t)M, (uint64_t)d, (uint32_t)NT) ||
      encode_bf16_map_box(&p.tmX[2], ws->A, (uint64_t)M, (uint64_t)F, (uint32_t)NT))
    return fail(SPA_ERR_CUDA, "tensor maps of the FFN token operands failed");
  p.d = d; p.F = F; p.M = M; p.NT = NT; p.tps = tps; p.N = c->N; p.idx = idx;
  p.H = (const __nv_bfloat16*)H;
  p.gamma = (const __nv_bfloat16*)L->w.ffn_norm;
  p.eps = D.rms_eps;
  p.H1 = (__nv_bfloat16*)ws->H1;
  p.X2 = (__nv_bfloat16*)ws->X2;
  p.A = (__nv_bfloat16*)ws->A;
  p.Hc = (__nv_bfloat16*)c->h_cache;
  p.row_copy = (__nv_bfloat16*)row_copy;
  p.score_zero = score_zero;
  size_t off = 0;
  for (int ph = 0; ph < 3; ++ph) {
    p.KB[ph] = pl.KB[ph]; p.nacc[ph] = pl.nacc[ph]; p.n_tiles[ph] = pl.n_tiles[ph];
    p.units[ph] = pl.units[ph]; p.maxseg[ph] = pl.maxseg[ph]; p.seg_total[ph] = pl.seg_total[ph];
    p.part[ph] = ws->ffn_part + off;
    off += pl.part_floats[ph];
    p.max_nacc = std::max(p.max_nacc, pl.nacc[ph]);
  }
  p.acc_cols = p.max_nacc * NT;
  int cols = 32;
  while (cols < 2 * p.acc_cols) cols *= 2;
  p.tmem_cols = cols;
  p.sync = ws->ffn_sync;
  p.err = ws->err;
  const double es = 2.0, Md = (double)M * d;
  const double wbytes = ((double)d * d + 3.0 * d * F) * es;
  ProfScope ps(&ws->prof, SPA_PROF_FFN, wbytes + 6.0 * Md * es + 2.0 * (double)M * F * es,
               2.0 * Md * d + 6.0 * Md * F, s);
  const cudaError_t e = launch_ffn_persistent(p, pl.grid, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "persistent FFN launch: %s", cudaGetErrorString(e));
  return SPA_OK;
}

// The FFN RMSNorm folded into the O-proj and gate/up epilogues of the
// weight-stationary path (SPA_NORM_FOLD=0: a separate norm kernel instead).
static bool norm_fold_enabled() {
  const char* e = std::getenv("SPA_NORM_FOLD");
  return !(e && e[0] == '0');
}

static int run_ffn_half(spa_layer* L, const void* H, const int32_t* idx, int tps,
                        const spa_layer_cache* c, cudaStream_t s, const void* Ob, const CUtensorMap* tmOb,
                        void* row_copy, float* score_zero) {
  spa_workspace* ws = L->ws;
  const spa_layer_desc& D = L->desc;
  const int d = D.d, F = D.ffn, M = c->B * tps, N = c->N;
  const bool bf = D.dtype == SPA_BF16;
  const double es = bf ? 2.0 : 4.0, Md = (double)M * d;
  Profiler* prof = &ws->prof;
  cudaError_t e;
  if (bf && M <= 256 && ffn_persistent_enabled()) {
    const int st = run_ffn_persistent(L, H, idx, tps, c, s, Ob, row_copy, score_zero);
    if (st != SPA_ERR_UNSUPPORTED) return st;  // otherwise the separate kernels below
  }
  // H1 = H[I] + O W_o^T
  {
    EpiParams ep = base_epi(L, M, tps, N, idx);
    ep.n_out = d;
    ep.out = ws->H1;
    ep.resid = H;
    if (bf && M <= 256 && streamk_enabled()) {
      SkParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wo; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      // the reduce kernel also takes the FFN RMSNorm of each row: x2 = RMSNorm(H1)
      SPA_TRY(run_sk(EPI_RESID, p, ws, Ob, M, d, d / 128, s, prof,
                     Work{SPA_PROF_OPROJ, (double)d * d * es + 4.0 * Md * es + d * es, 2.0 * Md * d + 4.0 * Md},
                     L->w.ffn_norm, ws->X2, D.rms_eps));
    } else if (bf && M <= 256) {
      TcWsParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wo; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      if (norm_fold_enabled()) {
        // the FFN RMSNorm folded in: x2 = gamma * H1 and the rows' partial sums of squares
        p.ep.gamma = L->w.ffn_norm;
        p.ep.x2 = ws->X2;
        p.ep.ss_part = ws->ss_part;
        p.ep.ss_tiles = (d + 127) / 128;
      }
      SPA_TRY(run_ws(EPI_RESID, false, p, ws, Ob, M, d, d, s, prof,
                     Work{SPA_PROF_OPROJ, (double)d * d * es + 4.0 * Md * es + d * es, 2.0 * Md * d + 3.0 * Md}));
    } else if (bf) {
      TcGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmA = *tmOb; p.tmB[0] = L->tm_wo;
      p.K = d; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      const int nt = d / 256, mt = (M + 127) / 128;
      SPA_TRY(run_tc(EPI_RESID, 256, p, M, nt, choose_splits(nt * mt, d / 64, ws->num_sms), s, prof,
                     Work{SPA_PROF_OPROJ, (double)d * d * es + 3.0 * Md * es, 2.0 * Md * d}, d / 64, ws->num_sms));
    } else {
      SimtGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.A = (const float*)Ob; p.B[0] = (const float*)L->w.wo;
      p.K = d; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_simt(EPI_RESID, p, M, (d + 127) / 128, s, prof,
                       Work{SPA_PROF_OPROJ, (double)d * d * es + 3.0 * Md * es, 2.0 * Md * d}));
    }
  }
  // x2 = RMSNorm(H1) (the stream-K O-proj's reduce kernel wrote it already;
  // the weight-stationary GEMMs fold it into their epilogues)
  const bool ws_path = bf && M <= 256 && !streamk_enabled();
  const bool fold = ws_path && norm_fold_enabled();
  if (!(bf && M <= 256) || (ws_path && !fold)) {
    {
      ProfScope ps(prof, SPA_PROF_NORM, 2.0 * Md * es + d * es, 4.0 * Md, s);
      e = launch_rmsnorm_rows(D.dtype, ws->H1, 0, nullptr, tps, N, M, d, L->w.ffn_norm, D.rms_eps, ws->X2, ws->err, s);
    }
    if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "rmsnorm launch: %s", cudaGetErrorString(e));
  }
  // A = silu(x2 W_gate^T) * (x2 W_up^T)
  {
    EpiParams ep = base_epi(L, M, tps, N, idx);
    ep.n_out = F;
    ep.out = ws->A;
    if (bf && M <= 256 && streamk_enabled()) {
      SkParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wg64; p.tmW[1] = L->tm_wu64; p.b_mode = B_GATEUP; p.b_rows_per_src = F; p.ep = ep;
      SPA_TRY(run_sk(EPI_SWIGLU, p, ws, ws->X2, M, d, F / 64, s, prof,
                     Work{SPA_PROF_GATEUP, 2.0 * F * d * es + Md * es + (double)M * F * es, 4.0 * Md * F}));
    } else if (ws_path) {
      TcWsParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wg; p.tmW[1] = L->tm_wu; p.b_mode = B_GATEUP; p.b_rows_per_src = F; p.ep = ep;
      if (fold) {  // x2 holds gamma * H1: each token's 1 / rms(H1) scales its accumulators
        p.ep.ss_part = ws->ss_part;
        p.ep.ss_tiles = (d + 127) / 128;
        p.ep.eps = D.rms_eps;
      }
      SPA_TRY(run_ws(EPI_SWIGLU, true, p, ws, ws->X2, M, d, F, s, prof,
                     Work{SPA_PROF_GATEUP, 2.0 * F * d * es + Md * es + (double)M * F * es, 4.0 * Md * F}));
    } else if (bf) {
      TcGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmA = ws->tmX2; p.tmB[0] = L->tm_wg; p.tmB[1] = L->tm_wu;
      p.K = d; p.b_mode = B_GATEUP; p.b_rows_per_src = F; p.ep = ep;
      const int nt = F / 128, mt = (M + 127) / 128;
      SPA_TRY(run_tc(EPI_SWIGLU, 256, p, M, nt, choose_splits(nt * mt, d / 64, ws->num_sms), s, prof,
                     Work{SPA_PROF_GATEUP, 2.0 * F * d * es + Md * es + (double)M * F * es, 4.0 * Md * F}, d / 64, ws->num_sms));
    } else {
      SimtGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.A = (const float*)ws->X2; p.B[0] = (const float*)L->w.w_gate; p.B[1] = (const float*)L->w.w_up;
      p.K = d; p.b_mode = B_GATEUP; p.b_rows_per_src = F; p.ep = ep;
      SPA_TRY(run_simt(EPI_SWIGLU, p, M, (F + 63) / 64, s, prof,
                       Work{SPA_PROF_GATEUP, 2.0 * F * d * es + Md * es + (double)M * F * es, 4.0 * Md * F}));
    }
  }
  // H^c[I] = H1 + A W_down^T
  {
    EpiParams ep = base_epi(L, M, tps, N, idx);
    ep.n_out = d;
    ep.out = c->h_cache;
    ep.resid = ws->H1;
    ep.row_copy = row_copy;
    ep.score_zero = score_zero;
    if (bf && M <= 256 && streamk_enabled()) {
      SkParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wd; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_sk(EPI_RESID_SCATTER, p, ws, ws->A, M, F, d / 128, s, prof,
                     Work{SPA_PROF_DOWN, (double)d * F * es + (double)M * F * es + 2.0 * Md * es, 2.0 * Md * F}));
    } else if (bf && M <= 256) {
      TcWsParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmW[0] = L->tm_wd; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_ws(EPI_RESID_SCATTER, false, p, ws, ws->A, M, F, d, s, prof,
                     Work{SPA_PROF_DOWN, (double)d * F * es + (double)M * F * es + 2.0 * Md * es, 2.0 * Md * F}));
    } else if (bf) {
      TcGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.tmA = ws->tmA; p.tmB[0] = L->tm_wd;
      p.K = F; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      const int nt = d / 256, mt = (M + 127) / 128;
      SPA_TRY(run_tc(EPI_RESID_SCATTER, 256, p, M, nt, choose_splits(nt * mt, F / 64, ws->num_sms), s, prof,
                     Work{SPA_PROF_DOWN, (double)d * F * es + (double)M * F * es + 2.0 * Md * es, 2.0 * Md * F}, F / 64, ws->num_sms));
    } else {
      SimtGemmParams p;
      std::memset(&p, 0, sizeof(p));
      p.A = (const float*)ws->A; p.B[0] = (const float*)L->w.w_down;
      p.K = F; p.b_mode = B_SINGLE; p.b_rows_per_src = d; p.ep = ep;
      SPA_TRY(run_simt(EPI_RESID_SCATTER, p, M, (d + 127) / 128, s, prof,
                       Work{SPA_PROF_DOWN, (double)d * F * es + (double)M * F * es + 2.0 * Md * es, 2.0 * Md * F}));
    }
  }
  return SPA_OK;
}

// Phases 2 and 3 for M = B * tps tokens; idx == null means every row (rho = 1).
static int run_block(spa_layer* L, const void* H, const int32_t* idx, int tps,
                     const spa_layer_cache* c, cudaStream_t s, bool x_ready = false,
                     void* row_copy = nullptr, float* score_zero = nullptr) {
  SPA_TRY(run_attn_half(L, H, idx, tps, c, s, x_ready));
  return run_ffn_half(L, H, idx, tps, c, s, L->ws->O, &L->ws->tmO, row_copy, score_zero);
}

static int check_H(const void* H) {
  if (!H) return fail(SPA_ERR_INVALID, "null H");
  if (reinterpret_cast<uintptr_t>(H) % 16 != 0) return fail(SPA_ERR_INVALID, "H must be 16-byte aligned");
  return SPA_OK;
}

extern "C" int spa_proxy_select(spa_layer* L, const void* H, const spa_layer_cache* c, int k,
                                int32_t* idx, float* score, void* stream) {
  if (!L) return fail(SPA_ERR_INVALID, "null layer");
  SPA_TRY(check_H(H));
  SPA_TRY(check_cache(L, c));
  if (!idx) return fail(SPA_ERR_INVALID, "null idx");
  if (k < 1 || k > c->N) return fail(SPA_ERR_SHAPE, "k=%d outside [1, N=%d]", k, c->N);
  cudaStream_t s = (cudaStream_t)stream;
  float* sc = score ? score : L->ws->score;
  SPA_TRY(run_proxy(L, H, c, sc, 0, s));
  cudaError_t e;
  {
    const double Bn = (double)c->B * c->N, Bk = (double)c->B * k;
    ProfScope ps(&L->ws->prof, SPA_PROF_TOPK, 4.0 * Bn + 8.0 * Bk * L->desc.r + 4.0 * Bk, 0.0, s);
    e = launch_topk_select(sc, c->B, c->N, k, idx, L->ws->a_hat, c->p_cache, L->desc.r, L->ws->err, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "top-k launch: %s", cudaGetErrorString(e));
  return SPA_OK;
}

extern "C" int spa_partial_block(spa_layer* L, const void* H, const int32_t* idx, int k,
                                 const spa_layer_cache* c, void* stream) {
  if (!L) return fail(SPA_ERR_INVALID, "null layer");
  SPA_TRY(check_H(H));
  SPA_TRY(check_cache(L, c));
  if (!idx) return fail(SPA_ERR_INVALID, "null idx");
  if (k < 1 || k > c->N) return fail(SPA_ERR_SHAPE, "k=%d outside [1, N=%d]", k, c->N);
  return run_block(L, H, idx, k, c, (cudaStream_t)stream);
}

// One cached layer step.  Plain: the proxy of every row into the workspace,
// then the select.  With a_hat / score given (the model's per-layer proxy
// state, incremental mode): chg == null projects every row into them; else
// only the chg_tps rows per sequence listed in chg_idx, whose new input rows
// `chg` holds compact, and the other rows keep their proxy and score (their
// input is unchanged, and a row selected last step scores 0 because
// P^c = a_hat there).  The down GEMM then leaves this step's rewritten rows
// compact in row_copy (the next layer's changed rows) and zeroes their
// scores (P^c[I] = a_hat[I] now).
static int layer_step_impl(spa_layer* L, const void* H, const spa_layer_cache* c, int k, int32_t* idx,
                           cudaStream_t s, float* a_hat, float* score, const void* chg,
                           const int32_t* chg_idx, int chg_tps, void* row_copy) {
  const spa_layer_desc& D = L->desc;
  spa_workspace* ws = L->ws;
  if (!idx) return fail(SPA_ERR_INVALID, "null idx");
  if (k < 1 || k > c->N) return fail(SPA_ERR_SHAPE, "k=%d outside [1, N=%d]", k, c->N);
  const bool state = a_hat != nullptr;
  if (!state) {
    a_hat = ws->a_hat;
    score = ws->score;
  }
  if (chg) SPA_TRY(run_proxy_rows(L, chg, chg_idx, chg_tps, c, a_hat, score, 0, s));
  else SPA_TRY(run_proxy_rows(L, H, nullptr, c->N, c, a_hat, score, 0, s));
  const double Bn = (double)c->B * c->N, Bk = (double)c->B * k;
  const double es = D.dtype == SPA_BF16 ? 2.0 : 4.0;
  cudaError_t e;
  bool x_ready = false;
  if (select_norm_supported(D.dtype, c->N, D.d)) {
    // one launch for the select, the P^c scatter and RMSNorm(H[I])
    ProfScope ps(&ws->prof, SPA_PROF_TOPK, 4.0 * Bn + 8.0 * Bk * D.r + 4.0 * Bk + 2.0 * Bk * D.d * es, 0.0, s);
    e = launch_select_norm(D.dtype, score, c->B, c->N, k, idx, a_hat, c->p_cache, D.r, H, L->w.attn_norm,
                           D.rms_eps, D.d, ws->X, ws->err, s);
    x_ready = true;
  } else {
    ProfScope ps(&ws->prof, SPA_PROF_TOPK, 4.0 * Bn + 8.0 * Bk * D.r + 4.0 * Bk, 0.0, s);
    e = launch_topk_select(score, c->B, c->N, k, idx, a_hat, c->p_cache, D.r, ws->err, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "select launch: %s", cudaGetErrorString(e));
  return run_block(L, H, idx, k, c, s, x_ready, row_copy, state ? score : nullptr);
}

extern "C" int spa_layer_step(spa_layer* L, const void* H, const spa_layer_cache* c, int k,
                              int32_t* idx, void* stream) {
  if (!L) return fail(SPA_ERR_INVALID, "null layer");
  SPA_TRY(check_H(H));
  SPA_TRY(check_cache(L, c));
  return layer_step_impl(L, H, c, k, idx, (cudaStream_t)stream, nullptr, nullptr, nullptr, nullptr, 0,
                         nullptr);
}

// Unit rows of the attention outputs ws->O (M rows of r = d elements) into
// P^c (fill) or into a_hat with their drift scores against P^c.
static int score_attn_rows(spa_layer* L, const spa_layer_cache* c, int fill, cudaStream_t s) {
  spa_workspace* ws = L->ws;
  const int M = c->B * c->N, d = L->desc.d;
  const double e = L->desc.dtype == SPA_BF16 ? 2.0 : 4.0;
  ProfScope ps(&ws->prof, SPA_PROF_PROXY, (double)M * d * e + (fill ? 1.0 : 3.0) * M * d * 4, 0.0, s);
  const cudaError_t er = launch_unit_rows_score(L->desc.dtype, ws->O, M, d, c->N, c->N, nullptr,
                                                fill ? nullptr : ws->a_hat, c->p_cache, fill ? nullptr : ws->score,
                                                fill, ws->err, s);
  if (er != cudaSuccess) return fail(SPA_ERR_CUDA, "attention-output score launch: %s", cudaGetErrorString(er));
  return SPA_OK;
}

extern "C" int spa_full_block(spa_layer* L, const void* H, const spa_layer_cache* c, int fill_proxy,
                              void* stream) {
  if (!L) return fail(SPA_ERR_INVALID, "null layer");
  SPA_TRY(check_H(H));
  SPA_TRY(check_cache(L, c));
  if (fill_proxy < 0 || fill_proxy > 2) return fail(SPA_ERR_INVALID, "fill_proxy must be 0, 1 or 2");
  cudaStream_t s = (cudaStream_t)stream;
  if (fill_proxy == 2) {
    // the attention-output identifier's fill: P^c = unit attention output of every row
    if (L->desc.r != L->desc.d) return fail(SPA_ERR_SHAPE, "the attention-output identifier needs r = d");
    SPA_TRY(run_attn_half(L, H, nullptr, c->N, c, s, false));
    SPA_TRY(score_attn_rows(L, c, 1, s));
    return run_ffn_half(L, H, nullptr, c->N, c, s, L->ws->O, &L->ws->tmO, nullptr, nullptr);
  }
  if (fill_proxy) SPA_TRY(run_proxy(L, H, c, nullptr, 1, s));
  return run_block(L, H, nullptr, c->N, c, s);
}

extern "C" int spa_layer_step_attn_identifier(spa_layer* L, const void* H, const spa_layer_cache* c, int k,
                                              int32_t* idx, void* stream) {
  if (!L) return fail(SPA_ERR_INVALID, "null layer");
  SPA_TRY(check_H(H));
  SPA_TRY(check_cache(L, c));
  if (!idx) return fail(SPA_ERR_INVALID, "null idx");
  if (k < 1 || k > c->N) return fail(SPA_ERR_SHAPE, "k=%d outside [1, N=%d]", k, c->N);
  if (L->desc.r != L->desc.d) return fail(SPA_ERR_SHAPE, "the attention-output identifier needs r = d");
  cudaStream_t s = (cudaStream_t)stream;
  spa_workspace* ws = L->ws;
  const spa_layer_desc& D = L->desc;
  // phase 1: every row's attention output from fresh Q/K/V (K^c, V^c rewritten
  // at every row), its drift score, the top-k and P^c[I] <- unit output
  SPA_TRY(run_attn_half(L, H, nullptr, c->N, c, s, false));
  SPA_TRY(score_attn_rows(L, c, 0, s));
  cudaError_t e;
  const double Bn = (double)c->B * c->N, Bk = (double)c->B * k, es = D.dtype == SPA_BF16 ? 2.0 : 4.0;
  {
    ProfScope ps(&ws->prof, SPA_PROF_TOPK, 4.0 * Bn + 8.0 * Bk * D.r + 4.0 * Bk, 0.0, s);
    e = launch_topk_select(ws->score, c->B, c->N, k, idx, ws->a_hat, c->p_cache, D.r, ws->err, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "select launch: %s", cudaGetErrorString(e));
  // phase 2 is done: the selected rows' outputs, compact, feed phase 3
  {
    ProfScope ps(&ws->prof, SPA_PROF_MISC, 2.0 * Bk * D.d * es, 0.0, s);
    e = launch_gather_rows(D.dtype, ws->O, idx, c->B, k, c->N, D.d, ws->X, ws->err, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "gather launch: %s", cudaGetErrorString(e));
  return run_ffn_half(L, H, idx, k, c, s, ws->X, &ws->tmX, nullptr, nullptr);
}

// ---------------------------------------------------------------------------
// model / decode
// ---------------------------------------------------------------------------
extern "C" void spa_model_free(spa_model* m) {
  if (!m) return;
  if (m->graph) cudaGraphExecDestroy(m->graph);
  if (m->idx_all) cudaFree(m->idx_all);
  if (m->amax_val) cudaFree(m->amax_val);
  if (m->amax_idx) cudaFree(m->amax_idx);
  if (m->amax_sum) cudaFree(m->amax_sum);
  if (m->ahat_all) cudaFree(m->ahat_all);
  if (m->score_all) cudaFree(m->score_all);
  if (m->chg_rows) cudaFree(m->chg_rows);
  if (m->chg0_idx) cudaFree(m->chg0_idx);
  delete m;
}

extern "C" int spa_model_create(const spa_model_desc* desc, spa_layer* const* layers,
                                const spa_layer_cache* caches, void* h0, const void* embed,
                                const void* final_norm, const void* lm_head, spa_model** out) {
  if (!out) return fail(SPA_ERR_INVALID, "null output handle");
  *out = nullptr;
  if (!desc || !layers || !caches || !h0 || !embed || !final_norm || !lm_head)
    return fail(SPA_ERR_INVALID, "null argument");
  if (desc->n_layers < 1 || desc->vocab < 2 || desc->B < 1 || desc->N < 1)
    return fail(SPA_ERR_SHAPE, "bad model sizes");
  spa_workspace* ws = layers[0] ? layers[0]->ws : nullptr;
  if (!ws) return fail(SPA_ERR_INVALID, "null layer");
  for (int l = 0; l < desc->n_layers; ++l) {
    if (!layers[l] || layers[l]->ws != ws) return fail(SPA_ERR_INVALID, "every layer must share one workspace");
    SPA_TRY(check_cache(layers[l], &caches[l]));
    if (caches[l].B != desc->B || caches[l].N != desc->N) return fail(SPA_ERR_SHAPE, "cache shape differs from the model's");
  }
  spa_model* m = new (std::nothrow) spa_model();
  if (!m) return fail(SPA_ERR_NOMEM, "host allocation failed");
  m->desc = *desc;
  m->layers.assign(layers, layers + desc->n_layers);
  m->caches.assign(caches, caches + desc->n_layers);
  m->h0 = h0;
  m->embed = embed;
  m->final_norm = final_norm;
  m->lm_head = lm_head;
  for (int l = 1; l <= desc->n_layers; ++l) {
    const double rho = spa_rho(l, desc->n_layers, desc->rho_p, desc->l_p, desc->rho_1, desc->rho_L);
    const int k = spa_budget_k(desc->N, rho);
    if (k < 1) {
      delete m;
      return fail(SPA_ERR_INVALID, "invalid rho parameters");
    }
    m->k.push_back(k);
  }
  const spa_layer_desc& D = ws->desc;
  m->lm_tiles = (desc->vocab + 127) / 128;  // the widest split: 128-column tiles
  const size_t rows = (size_t)desc->B * desc->N;
  if (dev_alloc((void**)&m->idx_all, (size_t)desc->n_layers * rows * 4) != cudaSuccess ||
      dev_alloc((void**)&m->amax_val, rows * m->lm_tiles * 4) != cudaSuccess ||
      dev_alloc((void**)&m->amax_idx, rows * m->lm_tiles * 4) != cudaSuccess ||
      dev_alloc((void**)&m->amax_sum, rows * m->lm_tiles * 4) != cudaSuccess) {
    cudaGetLastError();
    spa_model_free(m);
    return fail(SPA_ERR_NOMEM, "model buffers: cudaMalloc failed");
  }
  if (D.dtype == SPA_BF16 && encode_bf16_map(&m->tm_lm, lm_head, desc->vocab, D.d)) {
    spa_model_free(m);
    return fail(SPA_ERR_CUDA, "tensor map for the LM head failed");
  }
  *out = m;
  return SPA_OK;
}

extern "C" int spa_model_layer_k(const spa_model* m, int layer) {
  if (!m || layer < 0 || layer >= (int)m->k.size()) return -1;
  return m->k[layer];
}

extern "C" int spa_model_index_set(const spa_model* m, int layer, int32_t* idx_out, void* stream) {
  if (!m || !idx_out) return fail(SPA_ERR_INVALID, "null argument");
  if (layer < 0 || layer >= (int)m->k.size()) return fail(SPA_ERR_SHAPE, "layer %d outside [0, %d)", layer, (int)m->k.size());
  const size_t rows = (size_t)m->desc.B * m->desc.N;
  SPA_CK(cudaMemcpyAsync(idx_out, m->idx_all + (size_t)layer * rows, (size_t)m->desc.B * m->k[layer] * sizeof(int32_t),
                         cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return SPA_OK;
}

extern "C" int spa_model_set_incremental_proxy(spa_model* m, int enable) {
  if (!m) return fail(SPA_ERR_INVALID, "null model");
  if (enable && !m->ahat_all) {
    const spa_layer_desc& D = m->layers[0]->desc;
    const size_t rows = (size_t)m->desc.B * m->desc.N, L = m->desc.n_layers;
    const size_t es = D.dtype == SPA_BF16 ? 2 : 4;
    if (dev_alloc((void**)&m->ahat_all, L * rows * D.r * 4) != cudaSuccess ||
        dev_alloc((void**)&m->score_all, L * rows * 4) != cudaSuccess ||
        dev_alloc(&m->chg_rows, rows * D.d * es) != cudaSuccess ||
        dev_alloc((void**)&m->chg0_idx, rows * 4) != cudaSuccess) {
      cudaGetLastError();
      for (void** q : {(void**)&m->ahat_all, (void**)&m->score_all, &m->chg_rows, (void**)&m->chg0_idx}) {
        if (*q) cudaFree(*q);
        *q = nullptr;
      }
      return fail(SPA_ERR_NOMEM, "incremental proxy buffers: cudaMalloc failed");
    }
  }
  m->inc = enable != 0;
  m->inc_valid = false;  // the next step projects every row once
  return SPA_OK;
}

extern "C" int spa_model_embed(spa_model* m, const int32_t* tokens, void* stream) {
  if (!m || !tokens) return fail(SPA_ERR_INVALID, "null argument");
  m->inc_valid = false;  // every row of the layer-0 input may change
  spa_workspace* ws = m->layers[0]->ws;
  ProfScope ps(&ws->prof, SPA_PROF_MISC, 0.0, 0.0, (cudaStream_t)stream);
  cudaError_t e = launch_embed_rows(ws->desc.dtype, m->embed, tokens, nullptr, m->desc.B, m->desc.N,
                                    m->desc.N, ws->desc.d, m->desc.vocab, m->h0, ws->err,
                                    (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "embed launch: %s", cudaGetErrorString(e));
  return SPA_OK;
}

// The L layers of one decoding step (full: 0 cached, 1 rho = 1 fill, 2 vanilla).
static int decode_layers_impl(spa_model* m, int full, cudaStream_t s) {
  spa_workspace* ws = m->layers[0]->ws;
  const spa_layer_desc& D = ws->desc;
  const int L = m->desc.n_layers, B = m->desc.B, N = m->desc.N;
  const size_t rows = (size_t)B * N;
  void* stream = (void*)s;
  const bool inc = m->inc;
  const bool use_chg = inc && m->inc_valid && !full;
  const int r = D.r;
  for (int l = 0; l < L; ++l) {
    const void* H = (l == 0) ? m->h0 : m->caches[l - 1].h_cache;
    spa_layer* ly = m->layers[l];
    const spa_layer_cache* c = &m->caches[l];
    float* A = inc ? m->ahat_all + (size_t)l * rows * r : nullptr;
    float* S = inc ? m->score_all + (size_t)l * rows : nullptr;
    if (full == 1 && inc) {
      // the rho = 1 fill also sets the proxy state: a_hat = P^c, score 0
      SPA_TRY(run_proxy_rows(ly, H, nullptr, N, c, A, S, 1, s));
      SPA_TRY(run_block(ly, H, nullptr, N, c, s));
    } else if (full) {
      SPA_TRY(spa_full_block(ly, H, c, full == 1 ? 1 : 0, stream));
    } else if (inc) {
      const int32_t* ci = l == 0 ? m->chg0_idx : m->idx_all + (size_t)(l - 1) * rows;
      const int ctps = l == 0 ? m->chg0_u : m->k[l - 1];
      SPA_TRY(check_H(H));
      SPA_TRY(check_cache(ly, c));
      SPA_TRY(layer_step_impl(ly, H, c, m->k[l], m->idx_all + (size_t)l * rows, s, A, S,
                              use_chg ? m->chg_rows : nullptr, use_chg ? ci : nullptr, use_chg ? ctps : 0,
                              m->chg_rows));
    } else {
      SPA_TRY(spa_layer_step(ly, H, c, m->k[l], m->idx_all + (size_t)l * rows, stream));
    }
  }
  // the proxy state follows the caches after a fill or a cached step in
  // incremental mode; no layer-0 row has changed since (until tokens are written)
  m->chg0_u = 0;
  m->inc_valid = inc && full != 2;
  return SPA_OK;
}

// Final RMSNorm at the u positions pos ([B, u]) of the last layer's output,
// LM head, and per row the argmax id (lowest on ties) into tok_out; with
// conf_out, also that id's softmax probability.
static int lm_head_impl(spa_model* m, const int32_t* pos, int u, int32_t* tok_out, float* conf_out,
                        cudaStream_t s) {
  spa_workspace* ws = m->layers[0]->ws;
  const spa_layer_desc& D = ws->desc;
  const int L = m->desc.n_layers, B = m->desc.B, N = m->desc.N, d = D.d;
  // final RMSNorm at the u positions, LM head, argmax
  const double es = D.dtype == SPA_BF16 ? 2.0 : 4.0;
  cudaError_t e;
  {
    ProfScope ps(&ws->prof, SPA_PROF_MISC, 2.0 * B * u * d * es, 0.0, s);
    e = launch_gather_final(D.dtype, m->caches[L - 1].h_cache, pos, B, u, N, d, m->final_norm,
                            D.rms_eps, ws->X, ws->err, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "final norm launch: %s", cudaGetErrorString(e));
  const int M = B * u;
  const Work wl{SPA_PROF_LMHEAD, (double)m->desc.vocab * d * es + (double)M * d * es,
                2.0 * M * d * m->desc.vocab};
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.M = M;
  ep.n_out = m->desc.vocab;
  ep.d = d;
  ep.tokens_per_seq = u;
  ep.N = N;
  ep.amax_val = m->amax_val;
  ep.amax_idx = m->amax_idx;
  ep.amax_sum = conf_out ? m->amax_sum : nullptr;
  ep.err = ws->err;
  int tiles = m->lm_tiles;
  if (D.dtype == SPA_BF16 && M <= 256) {
    TcWsParams p;
    std::memset(&p, 0, sizeof(p));
    p.tmW[0] = m->tm_lm; p.b_mode = B_SINGLE; p.b_rows_per_src = m->desc.vocab; p.ep = ep;
    SPA_TRY(run_ws(EPI_ARGMAX, false, p, ws, ws->X, M, d, m->desc.vocab, s, &ws->prof, wl));
    tiles = p.ep.n_tiles;
  } else if (D.dtype == SPA_BF16) {
    tiles = (m->desc.vocab + 255) / 256;
    ep.n_tiles = tiles;
    TcGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.tmA = ws->tmX;
    p.tmB[0] = m->tm_lm;
    p.K = d; p.b_mode = B_SINGLE; p.b_rows_per_src = m->desc.vocab; p.ep = ep;
    SPA_TRY(run_tc(EPI_ARGMAX, 256, p, M, tiles, 1, s, &ws->prof, wl));
  } else {
    ep.n_tiles = tiles;
    SimtGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.A = (const float*)ws->X; p.B[0] = (const float*)m->lm_head;
    p.K = d; p.b_mode = B_SINGLE; p.b_rows_per_src = m->desc.vocab; p.ep = ep;
    SPA_TRY(run_simt(EPI_ARGMAX, p, M, m->lm_tiles, s, &ws->prof, wl));
  }
  {
    ProfScope ps(&ws->prof, SPA_PROF_MISC, 8.0 * M * m->lm_tiles, 0.0, s);
    e = conf_out ? launch_confidence_reduce(m->amax_val, m->amax_idx, m->amax_sum, M, tiles, tok_out, conf_out, s)
                 : launch_argmax_reduce(m->amax_val, m->amax_idx, M, tiles, tok_out, s);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "argmax launch: %s", cudaGetErrorString(e));
  return SPA_OK;
}

// h0[b, pos] <- embed[tok] ([B, u]): the next step's layer-0 input.
static int write_tokens_impl(spa_model* m, const int32_t* pos, const int32_t* tok, int u, cudaStream_t s) {
  spa_workspace* ws = m->layers[0]->ws;
  const spa_layer_desc& D = ws->desc;
  const int B = m->desc.B, N = m->desc.N, d = D.d;
  const double es = D.dtype == SPA_BF16 ? 2.0 : 4.0;
  const bool inc = m->inc;
  const int M = B * u;
  cudaError_t e;
  {
    ProfScope ps(&ws->prof, SPA_PROF_MISC, 2.0 * M * d * es, 0.0, s);
    e = launch_embed_rows(D.dtype, m->embed, tok, pos, B, u, N, d, m->desc.vocab, m->h0, ws->err, s,
                          inc ? m->chg_rows : nullptr, inc ? m->chg0_idx : nullptr);
  }
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, "embed launch: %s", cudaGetErrorString(e));
  m->chg0_u = u;  // these rows of the layer-0 input changed
  return SPA_OK;
}

extern "C" int spa_decode_step(spa_model* m, const int32_t* pos, const int32_t* tok_in, int u,
                               int full, int32_t* tok_out, void* stream) {
  if (!m || !pos || !tok_out) return fail(SPA_ERR_INVALID, "null argument");
  if (full < 0 || full > 2) return fail(SPA_ERR_INVALID, "full must be 0, 1 or 2");
  if (u < 1 || u > m->desc.N) return fail(SPA_ERR_SHAPE, "u=%d outside [1, N]", u);
  cudaStream_t s = (cudaStream_t)stream;
  SPA_TRY(decode_layers_impl(m, full, s));
  SPA_TRY(lm_head_impl(m, pos, u, tok_out, nullptr, s));
  return write_tokens_impl(m, pos, tok_in ? tok_in : tok_out, u, s);
}

extern "C" int spa_decode_layers(spa_model* m, int full, void* stream) {
  if (!m) return fail(SPA_ERR_INVALID, "null model");
  if (full < 0 || full > 2) return fail(SPA_ERR_INVALID, "full must be 0, 1 or 2");
  return decode_layers_impl(m, full, (cudaStream_t)stream);
}

extern "C" int spa_decode_confidence(spa_model* m, const int32_t* pos, int u, int32_t* tok_out,
                                     float* conf_out, void* stream) {
  if (!m || !pos || !tok_out || !conf_out) return fail(SPA_ERR_INVALID, "null argument");
  if (u < 1 || u > m->desc.N) return fail(SPA_ERR_SHAPE, "u=%d outside [1, N]", u);
  return lm_head_impl(m, pos, u, tok_out, conf_out, (cudaStream_t)stream);
}

extern "C" int spa_model_write_tokens(spa_model* m, const int32_t* pos, const int32_t* tok, int u,
                                      void* stream) {
  if (!m || !pos || !tok) return fail(SPA_ERR_INVALID, "null argument");
  if (u < 1 || u > m->desc.N) return fail(SPA_ERR_SHAPE, "u=%d outside [1, N]", u);
  return write_tokens_impl(m, pos, tok, u, (cudaStream_t)stream);
}

extern "C" int spa_decode_graph_capture(spa_model* m, const int32_t* pos, const int32_t* tok_in,
                                        int u, int32_t* tok_out, void* stream) {
  if (!m || !pos || !tok_out) return fail(SPA_ERR_INVALID, "null argument");
  if (!stream) return fail(SPA_ERR_INVALID, "capture needs a non-default stream");
  cudaStream_t s = (cudaStream_t)stream;
  spa_workspace* ws = m->layers[0]->ws;
  const bool prof_on = ws->prof.on;
  ws->prof.on = false;  // no timing events inside the graph
  // the launches captured depend on the proxy state; capture runs nothing, so the state is unchanged
  const bool saved_valid = m->inc_valid;
  const int variant = !m->inc ? 0 : (m->inc_valid ? 2 : 1);
  SPA_CK(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
  const int st = spa_decode_step(m, pos, tok_in, u, 0, tok_out, stream);
  m->inc_valid = saved_valid;
  cudaGraph_t g = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(s, &g);
  ws->prof.on = prof_on;
  if (st != SPA_OK) {
    if (g) cudaGraphDestroy(g);
    return st;
  }
  if (ec != cudaSuccess) return fail(SPA_ERR_CUDA, "stream capture failed: %s", cudaGetErrorString(ec));
  // count the kernel nodes the step recorded
  int kernels = 0;
  size_t n_nodes = 0;
  if (cudaGraphGetNodes(g, nullptr, &n_nodes) == cudaSuccess && n_nodes > 0) {
    std::vector<cudaGraphNode_t> nodes(n_nodes);
    if (cudaGraphGetNodes(g, nodes.data(), &n_nodes) == cudaSuccess)
      for (size_t i = 0; i < n_nodes; ++i) {
        cudaGraphNodeType t;
        if (cudaGraphNodeGetType(nodes[i], &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++kernels;
      }
  }
  cudaGetLastError();
  cudaGraphExec_t ex = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&ex, g, 0);
  cudaGraphDestroy(g);
  if (ei != cudaSuccess) return fail(SPA_ERR_CUDA, "graph instantiation failed: %s", cudaGetErrorString(ei));
  if (m->graph) cudaGraphExecDestroy(m->graph);
  m->graph = ex;
  m->graph_u = u;
  m->graph_inc = variant;
  m->graph_kernels = kernels;
  return SPA_OK;
}

extern "C" int spa_decode_graph_kernel_nodes(const spa_model* m) {
  if (!m) return -1;
  return m->graph ? m->graph_kernels : 0;
}

extern "C" int spa_decode_graph_launch(spa_model* m, void* stream) {
  if (!m) return fail(SPA_ERR_INVALID, "null model");
  if (!m->graph) return fail(SPA_ERR_INVALID, "no decode step has been captured");
  if (m->graph_inc == 2 && !m->inc_valid)
    return fail(SPA_ERR_INVALID, "the captured step projects only changed rows, but the proxy state is stale "
                                 "(a fill, a vanilla step or an embedding came in between): run one step "
                                 "directly first");
  SPA_CK(cudaGraphLaunch(m->graph, (cudaStream_t)stream));
  m->inc_valid = m->graph_inc != 0;
  return SPA_OK;
}
