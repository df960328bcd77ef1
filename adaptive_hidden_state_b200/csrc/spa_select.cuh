// Block-level helpers of the select kernels and of row RMSNorm: 16-byte
// (un)packing, RMSNorm of one row by 128 threads, and the per-sequence top-k
// (ties to the lowest index, indices ascending).
#pragma once
#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

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

// One row, 128 threads (gt = thread index within the group, red = 4 floats
// of shared memory for the group, bar = the group's barrier).  The sum of
// squares is taken in the same order by every caller, so a row's output bits
// do not depend on the kernel that normalises it.
template <typename T, int MAXC, typename Bar>
__device__ __forceinline__ void rmsnorm_one_row(const T* src_row, const T* gamma, int d, float eps,
                                                T* out_row, int gt, float* red, Bar bar) {
  constexpr int VEC = 16 / sizeof(T);
  const uint4* x = reinterpret_cast<const uint4*>(src_row);
  const uint4* g = reinterpret_cast<const uint4*>(gamma);
  const int nch = d / VEC;
  uint4 xv[MAXC], gv[MAXC];  // the row and gamma, all loads issued up front
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = gt + 128 * i;
    if (c < nch) {
      xv[i] = x[c];
      gv[i] = g[c];
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    if (gt + 128 * i < nch) {
      float f[VEC];
      unpack16<T>(xv[i], f);
#pragma unroll
      for (int e = 0; e < VEC; ++e) ss += f[e] * f[e];
    }
  }
  ss = warp_sum(ss);
  if ((gt & 31) == 0) red[gt >> 5] = ss;
  bar();
  const float tot = (red[0] + red[1]) + (red[2] + red[3]);
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  uint4* out = reinterpret_cast<uint4*>(out_row);
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    const int c = gt + 128 * i;
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


// ---------------------------------------------------------------------------
// Top-k select (per sequence; ties to the lowest index; indices ascending).
//
// Scores are non-negative floats, so their bit patterns order like the
// values (-0 and negatives are taken as 0).  Thread t of an NT-thread block
// holds keys [t*E, t*E + E) in registers (E = ceil(N / NT) <= 8).  The k-th
// largest key T, the largest value with #{key >= T} >= k, is found two bits
// per round from the top: a round counts the keys >= each of the three
// candidates T | d << b (d = 1, 2, 3) with warp reductions and one block
// barrier, and keeps the largest candidate that still has k keys at or above
// it.  One block-wide exclusive scan of each thread's counts of keys > T and
// == T (packed into one int) then places every selected key: with
// need = k - #{key > T}, a key == T is taken while fewer than `need` equal
// keys precede it, and a taken key's slot is (#keys > T before it) +
// min(#keys == T before it, need), so the list comes out ascending without a
// sort.  Per-thread key counts stay below 2^16, so the packed sums cannot
// carry.
// ---------------------------------------------------------------------------
constexpr int kSelMaxPerThread = 8;  // N <= 8 * block size

__device__ __forceinline__ uint32_t score_key(float v) {
  const uint32_t bits = __float_as_uint(v);
  return (bits & 0x80000000u) ? 0u : bits;
}

// Exclusive scan of one int per thread across an NT-thread block; `total`
// gets the block sum.  warp_tot holds 33 ints.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  constexpr int NW = NT / 32;
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
    const int w = lane < NW ? warp_tot[lane] : 0;
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

// Shared memory of block_select.
template <int NT>
struct SelectSmem {
  unsigned cnt[2][NT / 32];  // per round (double-buffered), per warp: three packed key counts
  int warp_tot[33];
};

// list[0..k) (and idx_out, when not null) <- the selected indices, ascending.
// MAXE (2, 4 or 8) bounds the keys a thread holds (E = ceil(N / NT) <= MAXE);
// block_select below picks the smallest that fits, so a round compares only
// the keys there can be.  A round's three counts per thread (<= 8 each) and
// per warp (<= 256) are packed 10 bits apart into one word, so one warp
// reduction and one shared word per warp carry all three.
template <int NT, int MAXE>
__device__ void block_select_e(const float* s, int N, int k, int32_t* list, int32_t* idx_out,
                               SelectSmem<NT>& sm, int* err) {
  constexpr int NW = NT / 32;
  static_assert(MAXE <= kSelMaxPerThread && MAXE * 32 < 1024, "packed counts must not carry");
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int E = (N + NT - 1) / NT;
  const int i0 = tid * E;
  uint32_t key[MAXE];
#pragma unroll
  for (int j = 0; j < MAXE; ++j)
    key[j] = (j < E && i0 + j < N) ? score_key(s[i0 + j]) : 0u;  // 0 is below every candidate
  uint32_t t = 0;
#pragma unroll 1
  for (int r = 0; r < 16; ++r) {
    const int shift = 30 - 2 * r;  // bits (31, 30), (29, 28), ..., (1, 0)
    const uint32_t c1 = t | (1u << shift), c2 = t | (2u << shift), c3 = t | (3u << shift);
    unsigned packed = 0;
#pragma unroll
    for (int j = 0; j < MAXE; ++j)
      packed += (key[j] >= c1 ? 1u : 0u) + (key[j] >= c2 ? 1u << 10 : 0u) + (key[j] >= c3 ? 1u << 20 : 0u);
    packed = __reduce_add_sync(0xffffffffu, packed);
    if (lane == 0) sm.cnt[r & 1][wid] = packed;
    __syncthreads();  // double-buffered counts: one barrier per round
    unsigned s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const unsigned v = sm.cnt[r & 1][w];
      s1 += v & 1023u;
      s2 += (v >> 10) & 1023u;
      s3 += v >> 20;
    }
    const unsigned kk = (unsigned)k;
    t = s3 >= kk ? c3 : s2 >= kk ? c2 : s1 >= kk ? c1 : t;
  }
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int j = 0; j < MAXE; ++j) {
    const bool v = j < E && i0 + j < N;
    n_gt += (v && key[j] > t) ? 1 : 0;
    n_eq += (v && key[j] == t) ? 1 : 0;
  }
  int tot;
  const int pre = block_exclusive_scan<NT>((n_gt << 16) | n_eq, sm.warp_tot, tot);
  const int need = k - (tot >> 16);
  if (tid == 0 && (tot >> 16) + min(tot & 0xffff, need) != k) report_error(err, DEVERR_SHAPE, 401);
  int gb = pre >> 16, eb = pre & 0xffff;
#pragma unroll
  for (int j = 0; j < MAXE; ++j) {
    if (!(j < E && i0 + j < N)) continue;
    int slot = -1;
    if (key[j] > t) {
      slot = gb + min(eb, need);
      ++gb;
    } else if (key[j] == t) {
      if (eb < need) slot = gb + eb;
      ++eb;
    }
    if (slot >= 0 && slot < k) {
      list[slot] = i0 + j;
      if (idx_out) idx_out[slot] = i0 + j;
    }
  }
}

template <int NT>
__device__ void block_select(const float* s, int N, int k, int32_t* list, int32_t* idx_out,
                             SelectSmem<NT>& sm, int* err) {
  const int E = (N + NT - 1) / NT;  // block-uniform
  if (E <= 2) block_select_e<NT, 2>(s, N, k, list, idx_out, sm, err);
  else if (E <= 4) block_select_e<NT, 4>(s, N, k, list, idx_out, sm, err);
  else block_select_e<NT, 8>(s, N, k, list, idx_out, sm, err);
}

}  // namespace spa
