// Memory- and latency-bound kernels of the SPA-Cache layer step: gathered
// RMSNorm, the per-sequence top-k select with the proxy-cache scatter (alone,
// or fused with the gather and RMSNorm of the selected rows), the per-row
// finish of wide proxies, embedding row updates, the final-norm gather and
// the LM-head argmax reduction.
#include <cfloat>

#include "spa_device.cuh"
#include "spa_internal.h"
#include "spa_select.cuh"

namespace spa {

// ---------------------------------------------------------------------------
// RMSNorm of gathered rows: X[t] = src[row(t)] / sqrt(mean(src^2) + eps) * gamma
// One CTA of 128 threads per row; every 16-byte chunk of the row (and of
// gamma) is loaded up front into registers, so a row costs one round trip.
// d must be a multiple of 16 bytes' worth of elements and <= 1024 chunks.
// ---------------------------------------------------------------------------
constexpr int kNormMaxChunks = 8;  // per thread: d <= 8 * 128 * 8 bf16 (8192) / 4096 f32

template <typename T>
__global__ void __launch_bounds__(128) rmsnorm_rows_kernel(const T* src, int src_is_cache,
                                                           const int32_t* idx, int tps, int N,
                                                           int M, int d, const T* gamma, float eps,
                                                           T* X, int* err) {
  griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.x;
  if (t >= M) return;
  size_t row;
  if (src_is_cache) {
    const int b = t / tps;
    const int pos = idx ? idx[t] : (t % tps);
    if (pos < 0 || pos >= N) {
      if (threadIdx.x == 0) report_error(err, DEVERR_INDEX, 301);
      return;
    }
    row = (size_t)b * N + pos;
  } else {
    row = (size_t)t;
  }
  __shared__ float red[4];
  rmsnorm_one_row<T, kNormMaxChunks>(src + row * d, gamma, d, eps, X + (size_t)t * d, threadIdx.x, red,
                                     []() { __syncthreads(); });
}

cudaError_t launch_rmsnorm_rows(int dtype, const void* src, int src_is_cache, const int32_t* idx,
                                int tps, int N, int M, int d, const void* gamma, float eps, void* X,
                                int* err, cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  const int vec = dtype == 1 ? 8 : 4;
  if (d % vec != 0 || d / vec > 128 * kNormMaxChunks) return cudaErrorInvalidValue;
  if (dtype == 1)
    return launch_k(rmsnorm_rows_kernel<__nv_bfloat16>, dim3(M), dim3(128), 0, stream,
                    (const __nv_bfloat16*)src, src_is_cache, idx, tps, N, M, d,
                    (const __nv_bfloat16*)gamma, eps, (__nv_bfloat16*)X, err);
  return launch_k(rmsnorm_rows_kernel<float>, dim3(M), dim3(128), 0, stream, (const float*)src,
                  src_is_cache, idx, tps, N, M, d, (const float*)gamma, eps, (float*)X, err);
}

constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads) topk_select_kernel(const float* score, int N, int k,
                                                                   int32_t* idx_out,
                                                                   const float* a_hat,
                                                                   float* p_cache, int r, int* err) {
  __shared__ SelectSmem<kTopkThreads> sm;
  __shared__ int32_t list[kSelMaxPerThread * kTopkThreads];
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  block_select<kTopkThreads>(score + (size_t)b * N, N, k, list, idx_out + (size_t)b * k, sm, err);
  __syncthreads();
  // P^c[b, I] <- a_hat[b, I], flattened over (selected row, 16-byte chunk):
  // up to kScatterBatch loads per thread in flight before any store
  if (p_cache != nullptr) {
    constexpr int kScatterBatch = 8;
    if ((r & 3) == 0) {
      const int r4 = r / 4, total = k * r4;
      const float4* src = reinterpret_cast<const float4*>(a_hat);
      float4* dst = reinterpret_cast<float4*>(p_cache);
      for (int base = tid; base < total; base += kTopkThreads * kScatterBatch) {
        float4 v[kScatterBatch];
        size_t off[kScatterBatch];
#pragma unroll
        for (int u = 0; u < kScatterBatch; ++u) {
          const int it = base + u * kTopkThreads;
          off[u] = it < total ? ((size_t)b * N + list[it / r4]) * r4 + (it % r4) : 0;
          if (it < total) v[u] = src[off[u]];
        }
#pragma unroll
        for (int u = 0; u < kScatterBatch; ++u)
          if (base + u * kTopkThreads < total) dst[off[u]] = v[u];
      }
    } else {
      const int total = k * r;
      for (int base = tid; base < total; base += kTopkThreads * kScatterBatch) {
        float v[kScatterBatch];
        size_t off[kScatterBatch];
#pragma unroll
        for (int u = 0; u < kScatterBatch; ++u) {
          const int it = base + u * kTopkThreads;
          off[u] = it < total ? ((size_t)b * N + list[it / r]) * r + (it % r) : 0;
          if (it < total) v[u] = a_hat[off[u]];
        }
#pragma unroll
        for (int u = 0; u < kScatterBatch; ++u)
          if (base + u * kTopkThreads < total) p_cache[off[u]] = v[u];
      }
    }
  }
}

cudaError_t launch_topk_select(const float* score, int B, int N, int k, int32_t* idx,
                               const float* a_hat, float* p_cache, int r, int* err,
                               cudaStream_t stream) {
  if (N > kTopkThreads * kSelMaxPerThread || k < 1 || k > N) return cudaErrorInvalidValue;
  return launch_k(topk_select_kernel, dim3(B), dim3(kTopkThreads), 0, stream, score, N, k, idx,
                  a_hat, p_cache, r, err);
}

// ---------------------------------------------------------------------------
// Select + gather + RMSNorm in one launch (the cached layer step): CTA (c, b)
// runs the top-k of sequence b itself (its scores are a few KB, and every
// CTA of the sequence computes the same index set), then each group
// of 128 threads takes one selected row j = 2c + group: writes idx[b, j], copies the
// proxy row a_hat -> P^c, and writes X[b*k + j] = RMSNorm(H[b, I_j]).  The
// select and the row arithmetic are the ones of the two separate kernels, so
// the results are bit-identical to theirs.
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 256;
constexpr int kSelRows = kSelThreads / 128;               // selected rows per CTA
constexpr int kSelMaxChunks = 4;                          // d <= 512 16-byte chunks
constexpr int kSelMaxN = kSelThreads * kSelMaxPerThread;  // 2048 scores

template <typename T>
__global__ void __launch_bounds__(kSelThreads, 2) select_norm_kernel(
    const float* score, int N, int k, int32_t* idx_out, const float* a_hat, float* p_cache, int r,
    const T* H, const T* gamma, float eps, int d, T* X, int* err) {
  __shared__ SelectSmem<kSelThreads> sm;
  __shared__ int32_t list[kSelMaxN];
  __shared__ float red[kSelRows][4];
  griddep_launch_dependents();
  griddep_wait();
  const int c = blockIdx.x, b = blockIdx.y;
  block_select<kSelThreads>(score + (size_t)b * N, N, k, list, nullptr, sm, c == 0 ? err : nullptr);
  __syncthreads();
  const int g = threadIdx.x >> 7, gt = threadIdx.x & 127;
  const int j = c * kSelRows + g;
  if (j >= k) return;  // whole groups only: the row barriers below are per group
  const int pos = list[j];
  const size_t row = (size_t)b * N + pos;
  if (gt == 0) idx_out[(size_t)b * k + j] = pos;
  if ((r & 3) == 0) {
    const float4* src = reinterpret_cast<const float4*>(a_hat) + row * (r / 4);
    float4* dst = reinterpret_cast<float4*>(p_cache) + row * (r / 4);
    for (int q = gt; q < r / 4; q += 128) dst[q] = src[q];
  } else {
    for (int q = gt; q < r; q += 128) p_cache[row * r + q] = a_hat[row * r + q];
  }
  rmsnorm_one_row<T, kSelMaxChunks>(H + row * d, gamma, d, eps, X + ((size_t)b * k + j) * d, gt, red[g],
                                    [g]() { asm volatile("bar.sync %0, 128;" ::"r"(g + 1) : "memory"); });
}

bool select_norm_supported(int dtype, int N, int d) {
  const int vec = dtype == 1 ? 8 : 4;
  return N <= kSelMaxN && d % vec == 0 && d / vec <= 128 * kSelMaxChunks;
}

cudaError_t launch_select_norm(int dtype, const float* score, int B, int N, int k, int32_t* idx,
                               const float* a_hat, float* p_cache, int r, const void* H,
                               const void* gamma, float eps, int d, void* X, int* err,
                               cudaStream_t stream) {
  if (!select_norm_supported(dtype, N, d) || k < 1 || k > N || !p_cache) return cudaErrorInvalidValue;
  const dim3 grid((k + kSelRows - 1) / kSelRows, B);
  if (dtype == 1)
    return launch_k(select_norm_kernel<__nv_bfloat16>, grid, dim3(kSelThreads), 0, stream, score, N, k,
                    idx, a_hat, p_cache, r, (const __nv_bfloat16*)H, (const __nv_bfloat16*)gamma, eps, d,
                    (__nv_bfloat16*)X, err);
  return launch_k(select_norm_kernel<float>, grid, dim3(kSelThreads), 0, stream, score, N, k, idx, a_hat,
                  p_cache, r, (const float*)H, (const float*)gamma, eps, d, (float*)X, err);
}

// ---------------------------------------------------------------------------
// Proxy rows of a wide r (> 256): the GEMM leaves the raw proxies a; one CTA
// of 256 threads per token row takes the norm, the unit proxy and the drift
// score (block sums in a fixed order), and writes them at the token's cache
// row.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) proxy_finish_kernel(const T* raw, int M, int r, int tps, int N,
                                                           const int32_t* idx, float* a_hat,
                                                           float* p_cache, float* score, int fill,
                                                           int* err) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float red[8];
  const int t = blockIdx.x;
  if (t >= M) return;
  const int b = t / tps;
  const int pos = idx ? idx[t] : (t % tps);
  if (pos < 0 || pos >= N) {
    if (threadIdx.x == 0) report_error(err, DEVERR_INDEX, 701);
    return;
  }
  const size_t dst = ((size_t)b * N + pos) * r;
  const T* a = raw + (size_t)t * r;
  auto block_sum = [&](float v) {
    v = warp_sum(v);
    __syncthreads();  // red[] is reused by the next sum
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w];
    return s;
  };
  float ss = 0.f;
  for (int c = threadIdx.x; c < r; c += 256) {
    const float x = to_f(a[c]);
    ss += x * x;
  }
  ss = block_sum(ss);
  const float nrm = sqrtf(ss);
  float sd = 0.f;
  for (int c = threadIdx.x; c < r; c += 256) {
    const float ah = ss > 0.f ? to_f(a[c]) / nrm : 0.f;
    if (fill) {
      p_cache[dst + c] = ah;
      if (a_hat) a_hat[dst + c] = ah;
    } else {
      const float df = ah - p_cache[dst + c];
      a_hat[dst + c] = ah;
      sd += df * df;
    }
  }
  if (!fill) {
    sd = block_sum(sd);
    if (threadIdx.x == 0) score[(size_t)b * N + pos] = 0.5f * sd;
  } else if (score && threadIdx.x == 0) {
    score[(size_t)b * N + pos] = 0.f;
  }
}

cudaError_t launch_proxy_finish(const float* raw, int M, int r, int tps, int N, const int32_t* idx,
                                float* a_hat, float* p_cache, float* score, int fill, int* err,
                                cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  return launch_k(proxy_finish_kernel<float>, dim3(M), dim3(256), 0, stream, raw, M, r, tps, N, idx, a_hat,
                  p_cache, score, fill, err);
}

cudaError_t launch_unit_rows_score(int dtype, const void* rows, int M, int r, int tps, int N,
                                   const int32_t* idx, float* a_hat, float* p_cache, float* score, int fill,
                                   int* err, cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  if (dtype == 1)
    return launch_k(proxy_finish_kernel<__nv_bfloat16>, dim3(M), dim3(256), 0, stream,
                    (const __nv_bfloat16*)rows, M, r, tps, N, idx, a_hat, p_cache, score, fill, err);
  return launch_k(proxy_finish_kernel<float>, dim3(M), dim3(256), 0, stream, (const float*)rows, M, r, tps,
                  N, idx, a_hat, p_cache, score, fill, err);
}

// ---------------------------------------------------------------------------
// Gather: dst[t] = src[b * N + idx[t]] for the M = B * k selected rows
// (t = b * k + j), 16 bytes per thread step.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) gather_rows_kernel(const T* src, const int32_t* idx, int k, int N,
                                                         int M, int d, T* dst, int* err) {
  griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.x;
  if (t >= M) return;
  const int b = t / k, pos = idx[t];
  if (pos < 0 || pos >= N) {
    if (threadIdx.x == 0) report_error(err, DEVERR_INDEX, 702);
    return;
  }
  const uint4* s4 = reinterpret_cast<const uint4*>(src + ((size_t)b * N + pos) * d);
  uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)t * d);
  const int nch = d * (int)sizeof(T) / 16;
  for (int c = threadIdx.x; c < nch; c += 128) d4[c] = s4[c];
}

cudaError_t launch_gather_rows(int dtype, const void* src, const int32_t* idx, int B, int k, int N, int d,
                               void* dst, int* err, cudaStream_t stream) {
  const int M = B * k;
  if (M <= 0) return cudaSuccess;
  if (dtype == 1)
    return launch_k(gather_rows_kernel<__nv_bfloat16>, dim3(M), dim3(128), 0, stream,
                    (const __nv_bfloat16*)src, idx, k, N, M, d, (__nv_bfloat16*)dst, err);
  return launch_k(gather_rows_kernel<float>, dim3(M), dim3(128), 0, stream, (const float*)src, idx, k, N, M,
                  d, (float*)dst, err);
}

// ---------------------------------------------------------------------------
// Embedding rows, final-norm gather, argmax reduction
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_rows_kernel(const T* embed, const int32_t* tokens, const int32_t* pos, int u,
                                  int N, int d, int vocab, T* h0, int* err, T* row_copy,
                                  int32_t* pos_copy) {
  griddep_launch_dependents();
  griddep_wait();
  const int j = blockIdx.x;  // row among B*u (or B*N when pos is null)
  const int b = j / u;
  const int p = pos ? pos[j] : (j % u);
  const int tok = tokens[j];
  if (p < 0 || p >= N || tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) report_error(err, DEVERR_INDEX, 501);
    if (pos_copy && threadIdx.x == 0) pos_copy[j] = -1;
    return;
  }
  const T* src = embed + (size_t)tok * d;
  T* dst = h0 + ((size_t)b * N + p) * d;
  T* cpy = row_copy ? row_copy + (size_t)j * d : nullptr;  // the changed rows, compact
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 v = load4(src + c);
    store4(dst + c, v);
    if (cpy) store4(cpy + c, v);
  }
  if (pos_copy && threadIdx.x == 0) pos_copy[j] = p;
}

cudaError_t launch_embed_rows(int dtype, const void* embed, const int32_t* tokens,
                              const int32_t* pos, int B, int u, int N, int d, int vocab, void* h0,
                              int* err, cudaStream_t stream, void* row_copy, int32_t* pos_copy) {
  const int rows = B * u;
  if (rows <= 0) return cudaSuccess;
  if (dtype == 1)
    return launch_k(embed_rows_kernel<__nv_bfloat16>, dim3(rows), dim3(128), 0, stream,
                    (const __nv_bfloat16*)embed, tokens, pos, u, N, d, vocab, (__nv_bfloat16*)h0, err,
                    (__nv_bfloat16*)row_copy, pos_copy);
  return launch_k(embed_rows_kernel<float>, dim3(rows), dim3(128), 0, stream, (const float*)embed,
                  tokens, pos, u, N, d, vocab, (float*)h0, err, (float*)row_copy, pos_copy);
}

cudaError_t launch_gather_final(int dtype, const void* hc, const int32_t* pos, int B, int u, int N,
                                int d, const void* gamma, float eps, void* X, int* err,
                                cudaStream_t stream) {
  return launch_rmsnorm_rows(dtype, hc, 1, pos, u, N, B * u, d, gamma, eps, X, err, stream);
}

__global__ void argmax_reduce_kernel(const float* val, const int32_t* idx, int rows, int n_tiles,
                                     int32_t* out) {
  griddep_launch_dependents();
  griddep_wait();
  const int row = blockIdx.x;
  const int lane = threadIdx.x;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int t = lane; t < n_tiles; t += 32) {
    const float v = val[(size_t)row * n_tiles + t];
    const int i = idx[(size_t)row * n_tiles + t];
    if (v > best || (v == best && i < bi)) { best = v; bi = i; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  if (lane == 0) out[row] = bi;
}

cudaError_t launch_argmax_reduce(const float* val, const int32_t* idx, int rows, int n_tiles,
                                 int32_t* out, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(argmax_reduce_kernel, dim3(rows), dim3(32), 0, stream, val, idx, rows, n_tiles, out);
}

// One warp per row: the row's max over the tiles and its argmax (lowest id on
// ties, as argmax_reduce_kernel), then total = sum_t sum_t * exp(max_t - max)
// (lane-strided partial sums, a fixed tree), conf = 1 / total.
__global__ void confidence_reduce_kernel(const float* val, const int32_t* idx, const float* sum, int rows,
                                         int n_tiles, int32_t* tok, float* conf) {
  griddep_launch_dependents();
  griddep_wait();
  const int row = blockIdx.x;
  const int lane = threadIdx.x;
  const float* v = val + (size_t)row * n_tiles;
  const int32_t* ix = idx + (size_t)row * n_tiles;
  const float* sm = sum + (size_t)row * n_tiles;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int t = lane; t < n_tiles; t += 32) {
    if (v[t] > best || (v[t] == best && ix[t] < bi)) { best = v[t]; bi = ix[t]; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  float total = 0.f;
  for (int t = lane; t < n_tiles; t += 32) total += sm[t] * expf(v[t] - best);
  total = warp_sum(total);
  if (lane == 0) {
    tok[row] = bi;
    conf[row] = total > 0.f ? 1.0f / total : 0.f;
  }
}

cudaError_t launch_confidence_reduce(const float* val, const int32_t* idx, const float* sum, int rows,
                                     int n_tiles, int32_t* tok, float* conf, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(confidence_reduce_kernel, dim3(rows), dim3(32), 0, stream, val, idx, sum, rows, n_tiles,
                  tok, conf);
}

__global__ void copy_i32_kernel(const int32_t* src, int32_t* dst, int n) {
  griddep_launch_dependents();
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[i];
}

cudaError_t launch_copy_i32(const int32_t* src, int32_t* dst, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  return launch_k(copy_i32_kernel, dim3((n + 255) / 256), dim3(256), 0, stream, src, dst, n);
}

// ---------------------------------------------------------------------------
// Bounded waits that nothing completes, for tests of the time-out path: with
// flag == null an mbarrier of count 1 that no thread arrives on, otherwise
// the global flag compared with `expect`.  Either way the wait gives up
// after limit_ns and records DEVERR_TIMEOUT in the error word; no copy or
// tensor-core operation is in flight, so the kernel then simply returns.
// ---------------------------------------------------------------------------
__global__ void wait_probe_kernel(const int* flag, int expect, unsigned long long limit_ns, int* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (flag == nullptr) mbar_wait(&bar, 0, &abort_flag, err, 901, limit_ns);
  else flag_wait(flag, expect, err, 902, limit_ns);
}

cudaError_t launch_wait_probe(const int* flag, int expect, unsigned long long limit_ns, int* err,
                              cudaStream_t stream) {
  wait_probe_kernel<<<1, 32, 0, stream>>>(flag, expect, limit_ns, err);
  return cudaPeekAtLastError();
}

}  // namespace spa
