// Memory-bound kernels of the SPA-Cache layer step: gathered RMSNorm, the
// per-sequence top-k select with the proxy-cache scatter, embedding row
// updates, the final-norm gather and the LM-head argmax reduction.
#include <cfloat>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

// ---------------------------------------------------------------------------
// RMSNorm of gathered rows: X[t] = src[row(t)] / sqrt(mean(src^2) + eps) * gamma
// One CTA of 128 threads per row; every 16-byte chunk of the row (and of
// gamma) is loaded up front into registers, so a row costs one round trip.
// d must be a multiple of 16 bytes' worth of elements and <= 1024 chunks.
// ---------------------------------------------------------------------------
constexpr int kNormMaxChunks = 8;  // per thread: d <= 8 * 128 * 8 bf16 (8192) / 4096 f32

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& u, float* f);
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    const float2 t = __bfloat1622float2(b);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& u, float* f) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
template <typename T>
__device__ __forceinline__ uint4 pack16(const float* f);
template <>
__device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ uint4 pack16<float>(const float* f) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

template <typename T>
__global__ void __launch_bounds__(128) rmsnorm_rows_kernel(const T* src, int src_is_cache,
                                                           const int32_t* idx, int tps, int N,
                                                           int M, int d, const T* gamma, float eps,
                                                           T* X, int* err) {
  constexpr int VEC = 16 / sizeof(T);
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
  const uint4* x = reinterpret_cast<const uint4*>(src + row * d);
  const uint4* g = reinterpret_cast<const uint4*>(gamma);
  const int nch = d / VEC;
  uint4 xv[kNormMaxChunks], gv[kNormMaxChunks];
#pragma unroll
  for (int i = 0; i < kNormMaxChunks; ++i) {
    const int c = threadIdx.x + 128 * i;
    if (c < nch) {
      xv[i] = x[c];
      gv[i] = g[c];
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kNormMaxChunks; ++i) {
    if (threadIdx.x + 128 * i < nch) {
      float f[VEC];
      unpack16<T>(xv[i], f);
#pragma unroll
      for (int e = 0; e < VEC; ++e) ss += f[e] * f[e];
    }
  }
  __shared__ float red[4];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  const float tot = (red[0] + red[1]) + (red[2] + red[3]);
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  uint4* out = reinterpret_cast<uint4*>(X + (size_t)t * d);
#pragma unroll
  for (int i = 0; i < kNormMaxChunks; ++i) {
    const int c = threadIdx.x + 128 * i;
    if (c < nch) {
      float f[VEC], gg[VEC];
      unpack16<T>(xv[i], f);
      unpack16<T>(gv[i], gg);
#pragma unroll
      for (int e = 0; e < VEC; ++e) f[e] = f[e] * inv * gg[e];
      out[c] = pack16<T>(f);
    }
  }
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

// ---------------------------------------------------------------------------
// Top-k select, one CTA of 1024 threads per sequence (N <= 8192).
//
// Scores are non-negative floats, so their bit patterns order like the
// values.  A 4-pass MSB-first radix select (8 bits per pass) finds the k-th
// largest key T and how many keys equal to T are still needed (`need`).  A
// token is selected if its key is > T, or == T and fewer than `need` equal
// keys precede it by index (ties to the lowest index).  Block-wide exclusive
// scans in index order then give each selected token its slot, so the index
// set comes out ascending.  Finally P^c[I] <- a_hat[I], flattened over
// (row, column) with several copies per thread in flight.
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkPerThread = 8;  // N <= 8192

// Exclusive scan of one int per thread across the block; returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int w = warp_tot[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  const int res = warp_tot[wid] + incl - v;
  total = warp_tot[32];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kTopkThreads) topk_select_kernel(const float* score, int N, int k,
                                                                   int32_t* idx_out,
                                                                   const float* a_hat,
                                                                   float* p_cache, int r, int* err) {
  __shared__ int hist[256];
  __shared__ int warp_tot[33];
  __shared__ int sel_digit, sel_above;
  __shared__ int32_t list[kTopkPerThread * kTopkThreads];
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const float* s = score + (size_t)b * N;
  const int E = (N + kTopkThreads - 1) / kTopkThreads;
  const int i0 = tid * E;

  uint32_t key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = i0 + j;
    const uint32_t bits = (j < E && i < N) ? __float_as_uint(s[i]) : 0u;
    key[j] = (bits & 0x80000000u) ? 0u : bits;  // s >= 0; -0 and negatives order as 0
  }

  uint32_t prefix = 0, mask = 0;
  int need = k;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    // one shared-memory atomic per distinct digit per warp (scores cluster in
    // a few top-byte values, so per-thread atomics would serialise)
#pragma unroll
    for (int j = 0; j < kTopkPerThread; ++j) {
      const int i = i0 + j;
      const bool act = j < E && i < N && (key[j] & mask) == prefix;
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const unsigned dig = (key[j] >> shift) & 255u;
        const unsigned peers = __match_any_sync(am, dig);
        if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[dig], __popc(peers));
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits [8l, 8l+8); scan from the top digit downwards
      int c[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[tid * 8 + j]; lsum += c[j]; }
      // suffix sum over lanes above this one (higher digits)
      int suf = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_down_sync(0xffffffffu, suf, o);
        if (tid + o < 32) suf += n;
      }
      int above = suf - lsum;  // count in lanes with higher digits
      // the lane whose range contains the boundary
      if (above < need && need <= suf) {
        int acc = above;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          if (acc < need && need <= acc + c[j]) { sel_digit = tid * 8 + j; sel_above = acc; }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)sel_digit << shift;
    mask |= 255u << shift;
    need -= sel_above;
    __syncthreads();
  }
  const uint32_t T = prefix;

  // selected = key > T, or key == T among the first `need` equal keys by index
  int n_eq = 0;
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = i0 + j;
    if (j < E && i < N && key[j] == T) ++n_eq;
  }
  int tot;
  int eq_before = block_exclusive_scan(n_eq, warp_tot, tot);
  int flags = 0, n_sel = 0;
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = i0 + j;
    if (j < E && i < N) {
      bool sel = key[j] > T;
      if (key[j] == T) {
        sel = eq_before < need;
        ++eq_before;
      }
      if (sel) { flags |= 1 << j; ++n_sel; }
    }
  }
  int slot = block_exclusive_scan(n_sel, warp_tot, tot);
  if (tid == 0 && tot != k) report_error(err, DEVERR_SHAPE, 401);
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    if (flags & (1 << j)) {
      if (slot < k) {
        list[slot] = i0 + j;
        idx_out[(size_t)b * k + slot] = i0 + j;
      }
      ++slot;
    }
  }
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
  if (N > kTopkThreads * kTopkPerThread || k < 1 || k > N) return cudaErrorInvalidValue;
  return launch_k(topk_select_kernel, dim3(B), dim3(kTopkThreads), 0, stream, score, N, k, idx,
                  a_hat, p_cache, r, err);
}

// ---------------------------------------------------------------------------
// Embedding rows, final-norm gather, argmax reduction
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_rows_kernel(const T* embed, const int32_t* tokens, const int32_t* pos, int u,
                                  int N, int d, int vocab, T* h0, int* err) {
  griddep_launch_dependents();
  griddep_wait();
  const int j = blockIdx.x;  // row among B*u (or B*N when pos is null)
  const int b = j / u;
  const int p = pos ? pos[j] : (j % u);
  const int tok = tokens[j];
  if (p < 0 || p >= N || tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) report_error(err, DEVERR_INDEX, 501);
    return;
  }
  const T* src = embed + (size_t)tok * d;
  T* dst = h0 + ((size_t)b * N + p) * d;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) store4(dst + c, load4(src + c));
}

cudaError_t launch_embed_rows(int dtype, const void* embed, const int32_t* tokens,
                              const int32_t* pos, int B, int u, int N, int d, int vocab, void* h0,
                              int* err, cudaStream_t stream) {
  const int rows = B * u;
  if (rows <= 0) return cudaSuccess;
  if (dtype == 1)
    return launch_k(embed_rows_kernel<__nv_bfloat16>, dim3(rows), dim3(128), 0, stream,
                    (const __nv_bfloat16*)embed, tokens, pos, u, N, d, vocab, (__nv_bfloat16*)h0, err);
  return launch_k(embed_rows_kernel<float>, dim3(rows), dim3(128), 0, stream, (const float*)embed,
                  tokens, pos, u, N, d, vocab, (float*)h0, err);
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

}  // namespace spa
