// Internal interfaces between the host API (spa_api.cu) and the kernel files.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace spa {

// Bits of the device error word.
enum : int {
  DEVERR_TIMEOUT = 1,  // a bounded wait ran out
  DEVERR_INDEX = 2,    // a gather/scatter index fell outside [0, N)
  DEVERR_SHAPE = 4,    // a launch saw a shape it cannot handle
};

// What a GEMM does with its fp32 accumulator tile (rows = tokens, columns =
// output features).  Every mode is a step of the cached layer update.
enum EpiMode : int {
  EPI_STORE = 0,          // out[t, n] = acc (dtype)                    - tests
  EPI_QKV = 1,            // RoPE(Q) -> compact Q; RoPE(K), V -> K^c, V^c rows I
  EPI_RESID = 2,          // H1[t] = acc + H[b, I[t]]
  EPI_SWIGLU = 3,         // A[t, f] = silu(acc_gate) * acc_up
  EPI_RESID_SCATTER = 4,  // H^c[b, I[t]] = acc + H1[t]
  EPI_PROXY = 5,          // a_hat = acc/|acc|; s = 1/2|a_hat - P^c|^2 (or fill P^c)
  EPI_ARGMAX = 6,         // per-tile (max, argmax) of the logits of each row
  EPI_PROXY_RAW = 7,      // out[t, n] = acc (fp32): the proxy of a wide r, finished per row
};

// How column tile n maps to rows of the weight sources.
enum BMode : int {
  B_SINGLE = 0,   // one matrix, rows n*BN ...
  B_CONCAT3 = 1,  // [W_q; W_k; W_v] stacked, rows_per_src rows each
  B_GATEUP = 2,   // first half of the tile from W_gate, second from W_up (same rows)
};

struct EpiParams {
  int M;               // valid rows (tokens) of the GEMM
  int n_out;           // logical output width (STORE: n; QKV: 3d; SWIGLU: F; PROXY: r; ARGMAX: vocab)
  int d;               // model width (row stride of caches and compact buffers)
  int head_dim;
  int tokens_per_seq;  // token t belongs to sequence t / tokens_per_seq
  int N;               // cache rows per sequence
  const int32_t* idx;  // [B * tokens_per_seq] cache row of each token; null: row = t % tokens_per_seq
  void* out;
  void* k_cache;
  void* v_cache;
  const void* resid;
  const float* rope_cos;  // [N, head_dim / 2]
  const float* rope_sin;
  float* a_hat;        // PROXY: [B*N, r] (rows addressed through the token's cache row)
  float* p_cache;      // PROXY: [B*N, r]
  float* score;        // PROXY: [B*N]
  int proxy_fill;      // PROXY: 1 = write the unit proxy into p_cache (and into a_hat, score = 0,
                       // when those are given)
  void* row_copy;      // RESID_SCATTER: also store the result rows compactly [M, d] (or null)
  float* score_zero;   // RESID_SCATTER: score_zero[b*N + row] = 0 for the tile's rows (or null)
  float* amax_val;     // ARGMAX: [M, n_tiles]
  int32_t* amax_idx;
  float* amax_sum;     // ARGMAX: sum over the tile of exp(logit - tile max) [M, n_tiles], or null
  int n_tiles;
  // The FFN RMSNorm folded into the GEMMs around it (weight-stationary path):
  // RESID (128-feature tiles) also writes x2[t] = gamma * H1[t] (bf16) and
  // ss_part[t * ss_tiles + tile] = the sum of H1[t]^2 over the tile's
  // features; SWIGLU scales both accumulators of token t by 1 / sqrt(sum over
  // tiles of ss_part[t] / d + eps) before silu(g) * u.  Null: not folded.
  const void* gamma;
  void* x2;
  float* ss_part;
  int ss_tiles;
  float eps;
  int* err;            // device error word
};

struct alignas(64) TcGemmParams {
  CUtensorMap tmA;     // [M, K] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap tmB[3];  // weight sources, box 64 x 128, 128-byte swizzle
  int K;
  int b_mode;
  int b_rows_per_src;
  EpiParams ep;
};

struct alignas(64) TcWsParams {
  CUtensorMap tmW[3];  // weight sources, box 64 x 128, 128-byte swizzle
  CUtensorMap tmX;     // token rows [M, K], box 64 x NT, 128-byte swizzle
  int K;
  int NT;              // tokens per MMA (multiple of 32, <= 256)
  int tmem_cols;       // power of two >= NACC * NT
  int b_mode;
  int b_rows_per_src;
  // Split-K across separate CTAs (no cluster; the whole grid resident at
  // once): every split stores its fp32 partial tile [NT][NACC * 128] at part +
  // ((tile * splits + split) * NT) * NACC * 128, counts itself in on
  // counter[tile], waits (bounded) for the tile's other splits, then sums the
  // splits in order 0..splits-1 for its share of the token rows and runs their
  // epilogue; the last split out (counter[kWsCounters + tile]) resets both.
  float* part;         // null: the splits of a tile form a cluster (DSMEM reduction)
  int* counter;        // [2 * kWsCounters], zero between launches
  EpiParams ep;
};
constexpr int kWsCounters = 4096;  // tiles of a split-K through global memory

// Stream-K weight-streaming GEMM (spa_streamk.cu): units (tile of nacc x 128
// output features, 64-column k-block) split evenly over the grid's CTAs; each
// CTA writes every segment's fp32 partial tile to its scratch slots, and a
// reduce kernel sums them per token row in k-block order and applies the
// fused epilogue.
struct alignas(64) SkParams {
  CUtensorMap tmW[3];  // weight sources, box 64 x 128 rows (B_GATEUP: 64 rows)
  CUtensorMap tmX;     // token rows [M, K], box 64 x NT, 128-byte swizzle
  int K, KB;           // reduction length and its 64-column blocks
  int NT;              // tokens per MMA (multiple of 32, <= 256)
  int n_tiles;         // unit tiles (nacc x 128 weight rows each)
  int units;           // n_tiles * KB
  int tmem_cols;       // power of two >= nbuf * nacc * NT
  int nacc;            // 128-row weight tiles per unit (1 or 2), sharing the token box
  int nbuf;            // TMEM accumulator buffers (2: a segment's epilogue overlaps the next)
  int maxseg;          // scratch slots per CTA (its most segments)
  int b_mode;
  int b_rows_per_src;
  float* part;         // scratch: slot (g * maxseg + j) = [NT][nacc * 128] fp32
  EpiParams ep;
};

struct SkReduceParams {
  const float* part;   // the GEMM's scratch slots
  size_t slot_floats;  // NT * feat
  int feat;            // nacc * 128
  int nacc, n_tiles, KB, G, U, maxseg;
  const void* gamma;   // EPI_RESID: FFN RMSNorm gain [d] and output x2 [M, d] (null: no norm)
  void* x2;
  float eps;
  EpiParams ep;
};

// Persistent FFN half of a cached layer step (spa_ffn.cu): O-proj (+ the FFN
// RMSNorm), gate/up with SwiGLU and down with the H^c scatter in one launch;
// phase p in 0..2, each split stream-K over the grid.
struct alignas(64) FfnParams {
  CUtensorMap tmWo, tmWg, tmWu, tmWd;  // W_o, W_down: 128-row boxes; W_gate, W_up: 64-row boxes
  CUtensorMap tmX[3];  // token operands: O [M, d], X2 [M, d], A [M, F]; box 64 x NT
  int d, F, M, NT, tps, N;
  const int32_t* idx;  // [B * tps] cache rows of the tokens (null: t % tps)
  const __nv_bfloat16* H;      // layer input [B, N, d] (residual of the O-proj)
  const __nv_bfloat16* gamma;  // FFN RMSNorm gain [d]
  float eps;
  __nv_bfloat16 *H1, *X2, *A, *Hc, *row_copy;  // outputs (row_copy may be null)
  float* score_zero;   // or null
  int KB[3], nacc[3], n_tiles[3], units[3], maxseg[3], seg_total[3];
  int max_nacc, acc_cols, tmem_cols;  // acc_cols = max nacc * NT; tmem_cols >= 2 * acc_cols
  float* part[3];      // per-phase scratch slots (g * maxseg + j) = [NT][nacc * 128] fp32
  int* sync;           // [8] segments counted, rows finished (per phase), CTAs done
  int* err;
};

struct SimtGemmParams {
  const float* A;      // [M, K]
  const float* B[3];
  int K;
  int b_mode;
  int b_rows_per_src;  // rows of each source matrix
  EpiParams ep;
};

// tcgen05 GEMM: D[M, n] = A[M, K] . B[n, K]^T, BM = 128, BN = 128 or 256,
// split-K across a thread-block cluster of `splits` CTAs with a fixed-order
// reduction through distributed shared memory.
// Tiled tcgen05 GEMM: BM x BN tiles (BM = 128, or 256 with BN = 256 for the
// layer GEMMs' epilogues), split-K across a cluster of `splits` CTAs.
cudaError_t launch_tc_gemm(int mode, int BN, int BM, const TcGemmParams& p, int m_tiles, int n_tiles,
                           int splits, cudaStream_t stream);
// Weight-stationary tcgen05 GEMM for M <= 256 tokens: 128 weight rows per
// CTA (NACC = 2: gate and up rows) against all tokens; same epilogues.
cudaError_t launch_tc_ws(int mode, int nacc, const TcWsParams& p, int n_tiles, int splits,
                         cudaStream_t stream);  // p.part set: splits of separate CTAs (no cluster)
int plan_ws_splits(int mode, int nacc, int n_tiles, int KB);
// Split count for a split-K through global memory (0: none fits): the whole
// grid resident at once, at most g_max splits (the scratch), and cheaper than
// the cluster plan of plan_ws_splits by the same estimate.
int plan_ws_global_splits(int mode, int nacc, int n_tiles, int KB, int g_max);
// CTAs of this weight-stationary GEMM the current device holds at once.
int ws_resident_ctas(int mode, int nacc);
// The persistent FFN kernel over `grid` CTAs (at most one per SM).
cudaError_t launch_ffn_persistent(const FfnParams& p, int grid, cudaStream_t stream);
int ffn_max_seg();    // segments per tile the reducers take
int ffn_max_tiles();  // unit tiles per phase
// Stream-K weight-streaming GEMM over `grid` CTAs (one per SM), then its
// per-row reduce + epilogue kernel (M CTAs).
cudaError_t launch_tc_sk(int mode, const SkParams& p, int grid, const SkReduceParams& r, cudaStream_t stream);
int sk_stages(int nacc, int NT);
// Segments of the busiest CTA and of the most split tile of a partition.
void sk_partition_bounds(int n_tiles, int KB, int G, int* max_seg_per_cta, int* max_seg_per_tile);
int sk_reduce_max_seg();    // segments per tile the reduce kernel takes
int sk_reduce_max_tiles();  // unit tiles the reduce kernel takes
// Encodes a 2D bf16 tensor map with a 64 x box_rows box.
int encode_bf16_map_box(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows);
// fp32 CUDA-core GEMM with the same epilogues, BM = 64, BN = 128.
cudaError_t launch_simt_gemm(int mode, const SimtGemmParams& p, int m_tiles, int n_tiles,
                             cudaStream_t stream);

// Encodes a 2D bf16 tensor map (rows x cols, row-major) with a 64 x 128 box.
int encode_bf16_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols);

// Records `msg` as this host thread's last error (read by spa_last_error)
// and returns `status`.
int set_last_error(int status, const char* msg);

// ---- small kernels (spa_kernels.cu) ----
// X[t] = RMSNorm(src[row(t)]) * gamma, row(t) = b * N + (idx ? idx[t] : t % tps) when
// src_is_cache, else t.
cudaError_t launch_rmsnorm_rows(int dtype, const void* src, int src_is_cache, const int32_t* idx,
                                int tokens_per_seq, int N, int M, int d, const void* gamma,
                                float eps, void* X, int* err, cudaStream_t stream);
// Per sequence: top-k of score (ties to the lowest index) -> idx ascending,
// then P^c[I] <- a_hat[I].
cudaError_t launch_topk_select(const float* score, int B, int N, int k, int32_t* idx,
                               const float* a_hat, float* p_cache, int r, int* err,
                               cudaStream_t stream);
// The top-k above fused with the gathered RMSNorm of the selected rows
// (X[b*k + j] = RMSNorm(H[b, idx[b, j]]) * gamma), bit-identical to running
// launch_topk_select then launch_rmsnorm_rows; for N <= 2048 and rows of at
// most 512 16-byte chunks (select_norm_supported).
// Rows of raw proxies a [M, r] fp32 (token t: sequence t / tps, cache row
// idx[t], or t % tps when idx is null) -> unit proxies and drift scores, as
// the EPI_PROXY epilogue computes them for r <= 256: fill = 1 writes P^c (and
// a_hat, score = 0 when given), else a_hat and score = 1/2 |a_hat - P^c|^2.
cudaError_t launch_proxy_finish(const float* raw, int M, int r, int tps, int N, const int32_t* idx,
                                float* a_hat, float* p_cache, float* score, int fill, int* err,
                                cudaStream_t stream);
// The same per-row finish on rows of dtype elements (1 = bf16, 0 = fp32):
// the attention-output identifier scores every row's attention output.
cudaError_t launch_unit_rows_score(int dtype, const void* rows, int M, int r, int tps, int N,
                                   const int32_t* idx, float* a_hat, float* p_cache, float* score, int fill,
                                   int* err, cudaStream_t stream);
// dst[b * k + j] = src[b * N + idx[b * k + j]] (rows of d dtype elements; d * size a multiple of 16 bytes).
cudaError_t launch_gather_rows(int dtype, const void* src, const int32_t* idx, int B, int k, int N, int d,
                               void* dst, int* err, cudaStream_t stream);
bool select_norm_supported(int dtype, int N, int d);
cudaError_t launch_select_norm(int dtype, const float* score, int B, int N, int k, int32_t* idx,
                               const float* a_hat, float* p_cache, int r, const void* H,
                               const void* gamma, float eps, int d, void* X, int* err,
                               cudaStream_t stream);
// Sparse-query attention: O[t] = softmax(Q_t K^cT / sqrt(hd)) V^c per head.
// allow_cluster = 1: key splits run as thread-block clusters and combine in
// distributed shared memory (the scratch arguments are unused).  Otherwise
// key splits use part_o / part_ml (max_rows partial rows of n_heads * hd and
// of 2 * n_heads floats) and `sync` (sync_len ints, zero between launches).
cudaError_t launch_attention(int dtype, const void* Q, const void* Kc, const void* Vc, void* O,
                             int B, int k, int N, int n_heads, int head_dim, float* part_o,
                             float* part_ml, int max_rows, int* sync, int sync_len, int* err,
                             int allow_cluster, cudaStream_t stream);
// h0[b, pos] <- embed[tok] for the listed (or all) positions.
cudaError_t launch_embed_rows(int dtype, const void* embed, const int32_t* tokens,
                              const int32_t* pos, int B, int u, int N, int d, int vocab,
                              void* h0, int* err, cudaStream_t stream, void* row_copy = nullptr,
                              int32_t* pos_copy = nullptr);
// Gathers final-layer rows at pos and applies the final RMSNorm.
cudaError_t launch_gather_final(int dtype, const void* hc, const int32_t* pos, int B, int u, int N,
                                int d, const void* gamma, float eps, void* X, int* err,
                                cudaStream_t stream);
// Reduces per-tile (max, argmax) partials to one id per row, lowest id on ties.
cudaError_t launch_argmax_reduce(const float* val, const int32_t* idx, int rows, int n_tiles,
                                 int32_t* out, cudaStream_t stream);
// Per row: the argmax id (lowest on ties) and its softmax probability
// 1 / sum_v exp(l_v - max) from per-tile (max, argmax, sum of exp) partials.
cudaError_t launch_confidence_reduce(const float* val, const int32_t* idx, const float* sum, int rows,
                                     int n_tiles, int32_t* tok, float* conf, cudaStream_t stream);
// A bounded wait that nothing completes (flag == null: an mbarrier no thread
// arrives on; else until *flag == expect), for tests of the time-out path.
cudaError_t launch_wait_probe(const int* flag, int expect, unsigned long long limit_ns, int* err,
                              cudaStream_t stream);
// Copies a [rows] int32 array (device) element-wise.
cudaError_t launch_copy_i32(const int32_t* src, int32_t* dst, int n, cudaStream_t stream);

}  // namespace spa
