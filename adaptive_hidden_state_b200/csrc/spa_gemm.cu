// GEMMs of the SPA-Cache layer step with their fused epilogues.
//
// tc_gemm_kernel (bf16, sm_100a tensor cores): one CTA computes a 128 x BN
// fp32 tile of D = A . B^T in TMEM.  Warp 0 streams A (token rows) and B
// (weight rows) tiles of 64 columns through a STAGES-deep TMA ring with
// 128-byte swizzling; one thread of warp 1 issues tcgen05.mma (M = 128,
// N = BN, K = 16) and frees each stage with tcgen05.commit.  Split-K runs
// across the CTAs of a thread-block cluster: each CTA stages its partial tile
// in shared memory, and CTA q sums rows [q*128/S, (q+1)*128/S) of all S
// partials through distributed shared memory in the fixed order 0..S-1, so
// results are deterministic and each output row depends only on its own
// input row.  The epilogue then applies the step's fused operation.
//
// simt_gemm_kernel (fp32, CUDA cores): 64 x 128 tiles with the same epilogues,
// for the fp32 configurations.
#include <cstdio>

#include <cudaTypedefs.h>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

// ---------------------------------------------------------------------------
// Epilogues over an fp32 tile held in shared memory (row-major, stride ld).
//
// The epilogues are latency-bound (a few dependent global accesses per
// output), so each thread works on kUnroll items at a time with all their
// global loads issued before any result is used, and the cache row of every
// tile row (b, position in I) is staged in shared memory once per tile.
// ---------------------------------------------------------------------------
constexpr int kUnroll = 8;

// silu(g) = g / (1 + e^-g) with the fast exponential and fast divide
// intrinsics: relative error a few 1e-7, far below the bf16 rounding of the
// result; for g below about -88, e^-g overflows and the quotient is -0, the
// limit of silu.  (A correctly rounded reciprocal here cost ~4 us per gate/up
// launch: its slow path serialises the epilogue's 64 silu per thread.)
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// s_rows[row] = (sequence b, cache row) of token t = gm0 + row; (0, -1) when
// t >= M or the index is out of range (the latter is reported).
__device__ void stage_rows(const EpiParams& ep, int gm0, int row_begin, int row_end, int2* s_rows,
                           int tid, int nthr) {
  for (int row = row_begin + tid; row < row_end; row += nthr) {
    const int t = gm0 + row;
    int2 v = make_int2(0, -1);
    if (t < ep.M) {
      v.x = t / ep.tokens_per_seq;
      v.y = ep.idx ? ep.idx[t] : (t % ep.tokens_per_seq);
      if (v.y < 0 || v.y >= ep.N) {
        report_error(ep.err, DEVERR_INDEX, 101);
        v.y = -1;
      }
    }
    s_rows[row] = v;
  }
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// While the main loop streams the weights, pull into L2 the global operands
// that the epilogue of rows gm0 .. gm0 + nrows - 1 will read: the residual
// rows' slice of this column tile (EPI_RESID: H[b, I_t]), the rotary table
// rows of the tokens' positions (EPI_QKV, Q and K tiles) and the cached proxy
// rows (EPI_PROXY).  One prefetch per 128-byte line; a hint, so no result
// depends on it.
template <int MODE, int FEAT, typename T>
__device__ void prefetch_epilogue_rows(const EpiParams& ep, int gm0, int nrows, int n_tile, int tid,
                                       int nthr) {
  if constexpr (MODE == EPI_RESID || MODE == EPI_QKV || MODE == EPI_PROXY) {
    for (int row = tid; row < nrows; row += nthr) {
      const int t = gm0 + row;
      if (t >= ep.M) break;
      const int b = t / ep.tokens_per_seq;
      const int pos = ep.idx ? ep.idx[t] : t % ep.tokens_per_seq;
      if (pos < 0 || pos >= ep.N) continue;
      const size_t cr = (size_t)b * ep.N + pos;
      if constexpr (MODE == EPI_RESID) {
        const char* src = reinterpret_cast<const char*>(reinterpret_cast<const T*>(ep.resid) + cr * ep.d +
                                                        (size_t)n_tile * FEAT);
        for (int o = 0; o < FEAT * (int)sizeof(T); o += 128) prefetch_l2(src + o);
      } else if constexpr (MODE == EPI_QKV) {
        if ((size_t)n_tile * FEAT < 2 * (size_t)ep.d) {
          const int hh = ep.head_dim / 2;
          const char* c = reinterpret_cast<const char*>(ep.rope_cos + (size_t)pos * hh);
          const char* sn = reinterpret_cast<const char*>(ep.rope_sin + (size_t)pos * hh);
          for (int o = 0; o < hh * 4; o += 128) {
            prefetch_l2(c + o);
            prefetch_l2(sn + o);
          }
        }
      } else {
        if (!ep.proxy_fill) {
          const char* pc = reinterpret_cast<const char*>(ep.p_cache + cr * ep.n_out);
          for (int o = 0; o < ep.n_out * 4; o += 128) prefetch_l2(pc + o);
        }
      }
    }
  }
}

template <int MODE, int BN, typename T>
__device__ void run_epilogue(const float* tile, int ld, int row_begin, int row_end, int gm0,
                             int n_tile, const EpiParams& ep, const int2* s_rows, int tid,
                             int nthr, const float* s_scale = nullptr) {
  const int nrows = row_end - row_begin;
  if (nrows <= 0) return;

  if constexpr (MODE == EPI_STORE || MODE == EPI_RESID || MODE == EPI_RESID_SCATTER) {
    constexpr int C4 = BN / 4;
    const int gn0 = n_tile * BN;
    const int total = nrows * C4;
    for (int base = tid; base < total; base += nthr * kUnroll) {
      float4 v[kUnroll], h[kUnroll];
      int row[kUnroll], c[kUnroll];
      bool ok[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int it = base + u * nthr;
        row[u] = row_begin + it / C4;
        c[u] = (it % C4) * 4;
        const int t = gm0 + row[u], gn = gn0 + c[u];
        ok[u] = it < total && t < ep.M && gn < ep.n_out;
        if (MODE != EPI_STORE && ok[u]) ok[u] = s_rows[row[u]].y >= 0;
        if (ok[u]) {
          v[u] = *reinterpret_cast<const float4*>(tile + row[u] * ld + c[u]);
          if constexpr (MODE == EPI_RESID) {
            const int2 br = s_rows[row[u]];
            h[u] = load4(reinterpret_cast<const T*>(ep.resid) + ((size_t)br.x * ep.N + br.y) * ep.d + gn);
          } else if constexpr (MODE == EPI_RESID_SCATTER) {
            h[u] = load4(reinterpret_cast<const T*>(ep.resid) + (size_t)t * ep.d + gn);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (!ok[u]) continue;
        const int t = gm0 + row[u], gn = gn0 + c[u];
        float4 r = v[u];
        if constexpr (MODE == EPI_STORE) {
          store4(reinterpret_cast<T*>(ep.out) + (size_t)t * ep.n_out + gn, r);
        } else {
          r.x += h[u].x; r.y += h[u].y; r.z += h[u].z; r.w += h[u].w;
          if constexpr (MODE == EPI_RESID) {
            store4(reinterpret_cast<T*>(ep.out) + (size_t)t * ep.d + gn, r);
          } else {
            const int2 br = s_rows[row[u]];
            store4(reinterpret_cast<T*>(ep.out) + ((size_t)br.x * ep.N + br.y) * ep.d + gn, r);
            if (ep.row_copy) store4(reinterpret_cast<T*>(ep.row_copy) + (size_t)t * ep.d + gn, r);
            if (ep.score_zero && gn == 0) ep.score_zero[(size_t)br.x * ep.N + br.y] = 0.f;
          }
        }
      }
      if constexpr (MODE == EPI_RESID && BN == 128 && sizeof(T) == 2) {
        // the FFN RMSNorm, folded: a warp holds one row's 128 features (32
        // float4 items), so its sum of squares is a warp sum in a fixed order
        if (ep.x2 != nullptr) {
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            const int t = gm0 + row[u], gn = gn0 + c[u];
            float ss = 0.f;
            if (ok[u]) {
              float4 q = v[u];
              q.x += h[u].x; q.y += h[u].y; q.z += h[u].z; q.w += h[u].w;
              // H1 as stored (bf16), times gamma
              q.x = __bfloat162float(__float2bfloat16_rn(q.x)); q.y = __bfloat162float(__float2bfloat16_rn(q.y));
              q.z = __bfloat162float(__float2bfloat16_rn(q.z)); q.w = __bfloat162float(__float2bfloat16_rn(q.w));
              ss = q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
              const float4 gm = load4(reinterpret_cast<const T*>(ep.gamma) + gn);
              store4(reinterpret_cast<T*>(ep.x2) + (size_t)t * ep.d + gn,
                     make_float4(q.x * gm.x, q.y * gm.y, q.z * gm.z, q.w * gm.w));
            }
            ss = warp_sum(ss);  // every lane of the warp runs the same items
            if ((tid & 31) == 0 && ok[u]) ep.ss_part[(size_t)t * ep.ss_tiles + n_tile] = ss;
          }
        }
      }
    }
  } else if constexpr (MODE == EPI_SWIGLU) {
    constexpr int HALF = BN / 2, C4 = HALF / 4;
    const int f0 = n_tile * HALF;
    for (int it = tid; it < nrows * C4; it += nthr) {
      const int row = row_begin + it / C4, c = (it % C4) * 4;
      const int t = gm0 + row, f = f0 + c;
      if (t >= ep.M || f >= ep.n_out) continue;
      float4 g = *reinterpret_cast<const float4*>(tile + row * ld + c);
      float4 u = *reinterpret_cast<const float4*>(tile + row * ld + HALF + c);
      if (s_scale != nullptr) {  // the folded FFN RMSNorm of token t
        const float sc = s_scale[row];
        g.x *= sc; g.y *= sc; g.z *= sc; g.w *= sc;
        u.x *= sc; u.y *= sc; u.z *= sc; u.w *= sc;
      }
      const float4 a = make_float4(silu(g.x) * u.x, silu(g.y) * u.y, silu(g.z) * u.z, silu(g.w) * u.w);
      store4(reinterpret_cast<T*>(ep.out) + (size_t)t * ep.n_out + f, a);
    }
  } else if constexpr (MODE == EPI_QKV) {
    constexpr int kUnrollQ = 4;  // four float4 operands per item, all loads of 4 items in flight
    // Item = 4 rotary pairs (j..j+3, j+hd/2..j+hd/2+3) of one head of one row.
    const int hd = ep.head_dim, hh = hd / 2;
    const int items_per_head = hh / 4;
    const int items = (BN / hd) * items_per_head;
    const int gn0 = n_tile * BN;
    const int total = nrows * items;
    for (int base = tid; base < total; base += nthr * kUnrollQ) {
      float4 x1[kUnrollQ], x2[kUnrollQ], cs[kUnrollQ], sn[kUnrollQ];
      int row[kUnrollQ], c1[kUnrollQ], j[kUnrollQ];
      bool ok[kUnrollQ];
#pragma unroll
      for (int u = 0; u < kUnrollQ; ++u) {
        const int it = base + u * nthr;
        row[u] = row_begin + it / items;
        const int w = it % items;
        const int hl = w / items_per_head;
        j[u] = (w % items_per_head) * 4;
        c1[u] = hl * hd + j[u];
        const int g1 = gn0 + c1[u];
        ok[u] = it < total && gm0 + row[u] < ep.M && g1 < ep.n_out && s_rows[row[u]].y >= 0;
        if (ok[u]) {
          x1[u] = *reinterpret_cast<const float4*>(tile + row[u] * ld + c1[u]);
          x2[u] = *reinterpret_cast<const float4*>(tile + row[u] * ld + c1[u] + hh);
          if (g1 / ep.d < 2) {
            const size_t off = (size_t)s_rows[row[u]].y * hh + j[u];
            cs[u] = *reinterpret_cast<const float4*>(ep.rope_cos + off);
            sn[u] = *reinterpret_cast<const float4*>(ep.rope_sin + off);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnrollQ; ++u) {
        if (!ok[u]) continue;
        const int g1 = gn0 + c1[u];
        const int part = g1 / ep.d, col1 = g1 % ep.d, col2 = col1 + hh;
        float4 a = x1[u], bb = x2[u];
        if (part < 2) {
          const float4 c = cs[u], s_ = sn[u];
          a = make_float4(x1[u].x * c.x - x2[u].x * s_.x, x1[u].y * c.y - x2[u].y * s_.y,
                          x1[u].z * c.z - x2[u].z * s_.z, x1[u].w * c.w - x2[u].w * s_.w);
          bb = make_float4(x2[u].x * c.x + x1[u].x * s_.x, x2[u].y * c.y + x1[u].y * s_.y,
                           x2[u].z * c.z + x1[u].z * s_.z, x2[u].w * c.w + x1[u].w * s_.w);
        }
        const int t = gm0 + row[u];
        const int2 br = s_rows[row[u]];
        T* dst;
        if (part == 0) dst = reinterpret_cast<T*>(ep.out) + (size_t)t * ep.d;
        else dst = reinterpret_cast<T*>(part == 1 ? ep.k_cache : ep.v_cache) +
                   ((size_t)br.x * ep.N + br.y) * ep.d;
        store4(dst + col1, a);
        store4(dst + col2, bb);
      }
    }
  } else if constexpr (MODE == EPI_PROXY) {
    // One warp per token row: norm, unit proxy, drift score.  r <= 256, so a
    // lane holds at most 8 columns (c = lane + 32 j).  Results go to the
    // token's cache row (b, s_rows[row].y): the tokens may be every row of
    // the caches or a compact list of rows.
    const int lane = tid & 31, wid = tid >> 5, nw = nthr >> 5;
    const int r = ep.n_out;
    for (int row = row_begin + wid; row < row_end; row += nw) {
      const int t = gm0 + row;
      if (t >= ep.M || s_rows[row].y < 0) continue;
      const size_t dst = (size_t)s_rows[row].x * ep.N + s_rows[row].y;
      const float* src = tile + row * ld;
      float a[8], pc[8];
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = lane + 32 * j;
        a[j] = c < r ? src[c] : 0.f;
        pc[j] = (!ep.proxy_fill && c < r) ? ep.p_cache[dst * r + c] : 0.f;
        ss += a[j] * a[j];
      }
      ss = warp_sum(ss);
      const float nrm = sqrtf(ss);
      float sd = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = lane + 32 * j;
        if (c >= r) continue;
        const float ah = ss > 0.f ? a[j] / nrm : 0.f;
        if (ep.proxy_fill) {
          ep.p_cache[dst * r + c] = ah;
          if (ep.a_hat) ep.a_hat[dst * r + c] = ah;
        } else {
          ep.a_hat[dst * r + c] = ah;
          const float df = ah - pc[j];
          sd += df * df;
        }
      }
      if (!ep.proxy_fill) {
        sd = warp_sum(sd);
        if (lane == 0) ep.score[dst] = 0.5f * sd;
      } else if (ep.score && lane == 0) {
        ep.score[dst] = 0.f;  // P^c = a_hat on this row
      }
    }
  } else if constexpr (MODE == EPI_PROXY_RAW) {
    constexpr int C4 = BN / 4;
    const int gn0 = n_tile * BN;
    float* out = reinterpret_cast<float*>(ep.out);
    for (int it = tid; it < nrows * C4; it += nthr) {
      const int row = row_begin + it / C4, c = (it % C4) * 4;
      const int t = gm0 + row, gn = gn0 + c;
      if (t >= ep.M || gn >= ep.n_out) continue;  // n_out is a multiple of 4
      *reinterpret_cast<float4*>(out + (size_t)t * ep.n_out + gn) =
          *reinterpret_cast<const float4*>(tile + row * ld + c);
    }
  } else if constexpr (MODE == EPI_ARGMAX) {
    const int lane = tid & 31, wid = tid >> 5, nw = nthr >> 5;
    const int gn0 = n_tile * BN;
    for (int row = row_begin + wid; row < row_end; row += nw) {
      const int t = gm0 + row;
      if (t >= ep.M) continue;
      float best = -INFINITY;
      int bi = 0x7fffffff;
      for (int c = lane; c < BN; c += 32) {
        const int gn = gn0 + c;
        if (gn >= ep.n_out) break;
        const float v = tile[row * ld + c];
        if (v > best) { best = v; bi = gn; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
      }
      if (lane == 0) {
        ep.amax_val[(size_t)t * ep.n_tiles + n_tile] = best;
        ep.amax_idx[(size_t)t * ep.n_tiles + n_tile] = bi;
      }
      if (ep.amax_sum) {  // for the softmax probability of the argmax
        float se = 0.f;
        for (int c = lane; c < BN; c += 32) {
          if (gn0 + c >= ep.n_out) break;
          se += expf(tile[row * ld + c] - best);
        }
        se = warp_sum(se);
        if (lane == 0) ep.amax_sum[(size_t)t * ep.n_tiles + n_tile] = se;
      }
    }
  }
}

// Rows [r0, r1) of the cluster's S partial tiles summed in the fixed order
// 0..S-1 into this CTA's tile.  With S <= 4 a thread takes four 16-byte
// items at once and issues all of their remote loads (up to 16) before using
// any; with more splits, eight loads of one item at a time.
template <int W>
__device__ void cluster_reduce_rows(float* tile, int ld, int r0, int r1, int S, int tid, int nthr) {
  constexpr int C4 = W / 4;
  const int total = (r1 - r0) * C4;
  if (S <= 4) {
    for (int base = tid; base < total; base += 4 * nthr) {
      float4 v[4][4];
      uint32_t local[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = base + u * nthr;
        const int row = r0 + it / C4, c = (it % C4) * 4;
        local[u] = smem_u32(tile + row * ld + c);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (it < total && q < S) v[u][q] = ld_dsmem_f4(mapa_shared(local[u], (uint32_t)q));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = base + u * nthr;
        if (it >= total) continue;
        float4 acc = v[u][0];  // split 0 first, then 1..S-1 in order
#pragma unroll
        for (int q = 1; q < 4; ++q)
          if (q < S) { acc.x += v[u][q].x; acc.y += v[u][q].y; acc.z += v[u][q].z; acc.w += v[u][q].w; }
        const int row = r0 + it / C4, c = (it % C4) * 4;
        *reinterpret_cast<float4*>(tile + row * ld + c) = acc;
      }
    }
    return;
  }
  for (int it = tid; it < total; it += nthr) {
    const int row = r0 + it / C4, c = (it % C4) * 4;
    const uint32_t local = smem_u32(tile + row * ld + c);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q0 = 0; q0 < 16; q0 += 8) {  // eight loads in flight, summed in order
      if (q0 >= S) break;
      float4 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q0 + q < S) v[q] = ld_dsmem_f4(mapa_shared(local, (uint32_t)(q0 + q)));
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q0 + q < S) { acc.x += v[q].x; acc.y += v[q].y; acc.z += v[q].z; acc.w += v[q].w; }
    }
    *reinterpret_cast<float4*>(tile + row * ld + c) = acc;
  }
}

// ---------------------------------------------------------------------------
// tcgen05 GEMM (token rows on the MMA's M side; used for M > 256 and the proxy)
// ---------------------------------------------------------------------------
template <int BN>
__device__ __forceinline__ void b_source(const TcGemmParams& p, int n_tile, int half, int& src,
                                         int& row) {
  if (p.b_mode == B_GATEUP) {
    src = half;
    row = n_tile * 128;
  } else if (p.b_mode == B_CONCAT3) {
    const int g = n_tile * BN + half * 128;
    src = g / p.b_rows_per_src;
    row = g % p.b_rows_per_src;
  } else {
    src = 0;
    row = n_tile * BN + half * 128;
  }
}

constexpr int kTcABytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kThreads = 256;         // 8 warps: producer, MMA issuer, all 8 in the epilogue

// BM = 256 (two 128-row A boxes and two TMEM accumulators of 128 x 256 per
// CTA) doubles the MMA work per byte staged: a 64-column k-block moves 64 KB
// through the ring for 2 x 128 x 256 x 64 MACs instead of 48 KB for half of
// that, which lifts the TMA-fill-bound rate of a CTA (one per SM: it holds
// tensor memory) by ~1.5x.  The epilogue runs the two 128-row halves in turn.
__host__ __device__ constexpr int tc_stages(int BN, int BM = 128) { return BM == 256 ? 3 : BN == 256 ? 4 : 3; }
__host__ __device__ constexpr int tc_smem_bytes(int BN, int BM = 128) {
  return tc_stages(BN, BM) * ((BM / 128) * kTcABytes + BN * 128) + 1024;
}

// A CTA that gave up (a bounded wait ran out) must not release its shared and
// tensor memory while its copies or tensor-core operations are in flight:
// thread 0 waits (bounded, ignoring the abort) for the accumulator commit and
// for every requested stage the MMA did not consume; then all threads proceed.
__device__ __forceinline__ void ws_drain_on_abort(int abort, uint64_t* accum_bar, uint64_t* full_bar, int stages,
                                                  int consumed, int issued, int* err) {
  if (abort && threadIdx.x == 0) {
    mbar_drain_bounded(accum_bar, 0, err, 215);
    for (int it = consumed; it < issued; ++it) mbar_drain_bounded(&full_bar[it % stages], (it / stages) & 1, err, 216);
  }
  __syncthreads();
}

template <int MODE, int BN, int BM>
__global__ void __launch_bounds__(kThreads, BN == 128 ? 2 : 1) tc_gemm_kernel(const __grid_constant__ TcGemmParams p) {
  constexpr int STAGES = tc_stages(BN, BM);
  constexpr int NA = BM / 128;  // A boxes (and accumulators) per stage
  constexpr int A_BYTES = NA * kTcABytes;
  constexpr int B_BYTES = BN * 128;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int LD = BN + 4;
  static_assert(BM == 128 || (BM == 256 && BN == 256), "256-row tiles take 256 columns");
  static_assert(128 * LD * 4 <= STAGES * STAGE_BYTES, "epilogue tile must fit the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t accum_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_issued, s_consumed;  // stages whose boxes were requested / consumed by the MMA
  __shared__ int2 s_rows[128];

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, S = gridDim.x;
  const int n_tile = blockIdx.y, m_tile = blockIdx.z;
  const int KB = p.K / 64;
  const int kb0 = (split * KB) / S, kb1 = ((split + 1) * KB) / S;
  const int nk = kb1 - kb0;
  int* err = p.ep.err;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&accum_bar, 1);
    abort_flag = 0;
    s_issued = 0;
    s_consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, NA * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // The B operand is always a weight matrix, which no earlier kernel writes:
  // the weight boxes of the first stages are requested before
  // griddepcontrol.wait, so they stream while the previous kernel finishes;
  // the token rows (A) follow the wait.
  const int pre = nk < STAGES ? nk : STAGES;
  if (warp == 0 && lane == 0) {
    s_issued = pre;
    for (int it = 0; it < pre; ++it) {
      uint8_t* sb = smem + it * STAGE_BYTES + A_BYTES;
      mbar_arrive_expect_tx(&full_bar[it], STAGE_BYTES);
      const int kx = (kb0 + it) * 64;
#pragma unroll
      for (int h = 0; h < BN / 128; ++h) {
        int src, row;
        b_source<BN>(p, n_tile, h, src, row);
        tma_load_2d(sb + h * 128 * 128, &p.tmB[src], &full_bar[it], kx, row);
      }
    }
  }
  griddep_wait();  // the token rows and the epilogue operands come from earlier kernels

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    for (int it = 0; it < pre; ++it) {
      uint8_t* sa = smem + it * STAGE_BYTES;
      const int kx = (kb0 + it) * 64;
#pragma unroll
      for (int a = 0; a < NA; ++a) tma_load_2d(sa + a * kTcABytes, &p.tmA, &full_bar[it], kx, m_tile * BM + a * 128);
    }
    for (int it = pre; it < nk; ++it) {
      const int s = it % STAGES;
      if (!mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, &abort_flag, err, 201)) break;
      uint8_t* sa = smem + s * STAGE_BYTES;
      uint8_t* sb = sa + A_BYTES;
      mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
      const int kx = (kb0 + it) * 64;
#pragma unroll
      for (int a = 0; a < NA; ++a) tma_load_2d(sa + a * kTcABytes, &p.tmA, &full_bar[s], kx, m_tile * BM + a * 128);
#pragma unroll
      for (int h = 0; h < BN / 128; ++h) {
        int src, row;
        b_source<BN>(p, n_tile, h, src, row);
        tma_load_2d(sb + h * 128 * 128, &p.tmB[src], &full_bar[s], kx, row);
      }
      s_issued = it + 1;
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
    for (int it = 0; it < nk; ++it) {
      const int s = it % STAGES;
      if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, &abort_flag, err, 202)) break;
      s_consumed = it + 1;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
      const uint64_t db = smem_desc_sw128(sa + A_BYTES);
#pragma unroll
      for (int a = 0; a < NA; ++a) {
        const uint64_t da = smem_desc_sw128(sa + a * kTcABytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem + (uint32_t)(a * BN), da + 2 * kk, db + 2 * kk, idesc, (it > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&empty_bar[s]);
    }
    umma_commit(&accum_bar);
  } else if (warp >= 2) {
    // idle during the main loop: the epilogue's operands into L2
    for (int a = 0; a < NA; ++a)
      prefetch_epilogue_rows<MODE, BN, __nv_bfloat16>(p.ep, m_tile * BM + a * 128, 128, n_tile, threadIdx.x - 64,
                                                      kThreads - 64);
  }
  __syncwarp();

  mbar_wait(&accum_bar, 0, &abort_flag, err, 203);
  __syncthreads();
  const bool good = (abort_flag == 0);
  tc_fence_after();

  float* tile = reinterpret_cast<float*>(smem);
#pragma unroll 1
  for (int a = 0; a < NA; ++a) {
    // the a-th 128-row half of the tile: accumulator -> shared memory, split-K
    // reduction across the cluster, epilogue
    if (a > 0) __syncthreads();  // the previous half's epilogue is done with the tile
    const int gm0 = m_tile * BM + a * 128;
    // rows of this half that hold tokens: the rest are never read, so they are
    // neither moved out of TMEM nor reduced
    const int mv = min(128, max(0, p.ep.M - gm0));
    if (good && (warp & 3) * 32 < mv) {
      const int q = warp & 3, half = warp >> 2;
      float* dst = tile + (q * 32 + lane) * LD;
#pragma unroll 1
      for (int c = 32 * half; c < BN; c += 64) {
        float v[32];
        if (nk > 0) {
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * BN + c), v);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + c + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (a == NA - 1) {
      ws_drain_on_abort(abort_flag, &accum_bar, full_bar, STAGES, s_consumed, s_issued, err);
      tc_fence_after();
      if (warp == 0) tmem_dealloc(tmem, NA * BN);
    }

    int r0 = 0, r1 = 128;
    if (S > 1) {
      cluster_sync();
      const int q = (int)cluster_ctarank();
      r0 = (q * mv) / S;
      r1 = ((q + 1) * mv) / S;
      if (good) cluster_reduce_rows<BN>(tile, LD, r0, r1, S, threadIdx.x, kThreads);
      cluster_sync();
    }
    if (good) {
      stage_rows(p.ep, gm0, r0, r1, s_rows, threadIdx.x, kThreads);
      __syncthreads();
      run_epilogue<MODE, BN, __nv_bfloat16>(tile, LD, r0, r1, gm0, n_tile, p.ep, s_rows, threadIdx.x,
                                            kThreads);
    }
  }
}

template <int MODE, int BN, int BM>
static cudaError_t launch_tc_typed(const TcGemmParams& p, int m_tiles, int n_tiles, int splits,
                                   cudaStream_t stream) {
  auto kern = tc_gemm_kernel<MODE, BN, BM>;
  const int smem = tc_smem_bytes(BN, BM);
  cudaError_t ec = configure_kernel((const void*)kern, smem, true);
  if (ec != cudaSuccess) return ec;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits, n_tiles, m_tiles);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_tc_gemm(int mode, int BN, int BM, const TcGemmParams& p, int m_tiles, int n_tiles,
                           int splits, cudaStream_t stream) {
  if (BM == 256) {
#define SPA_TC_CASE(M_)                                                                               \
  if (mode == M_ && BN == 256) return launch_tc_typed<M_, 256, 256>(p, m_tiles, n_tiles, splits, stream);
    SPA_TC_CASE(EPI_STORE)
    SPA_TC_CASE(EPI_QKV)
    SPA_TC_CASE(EPI_RESID)
    SPA_TC_CASE(EPI_SWIGLU)
    SPA_TC_CASE(EPI_RESID_SCATTER)
#undef SPA_TC_CASE
    return cudaErrorInvalidValue;
  }
  if (BM != 128) return cudaErrorInvalidValue;
#define SPA_TC_CASE(M_, BN_)                                           \
  if (mode == M_ && BN == BN_) return launch_tc_typed<M_, BN_, 128>(p, m_tiles, n_tiles, splits, stream);
  SPA_TC_CASE(EPI_STORE, 128)
  SPA_TC_CASE(EPI_STORE, 256)
  SPA_TC_CASE(EPI_QKV, 256)
  SPA_TC_CASE(EPI_RESID, 256)
  SPA_TC_CASE(EPI_SWIGLU, 256)
  SPA_TC_CASE(EPI_RESID_SCATTER, 256)
  SPA_TC_CASE(EPI_PROXY, 128)
  SPA_TC_CASE(EPI_PROXY, 256)
  SPA_TC_CASE(EPI_ARGMAX, 256)
  SPA_TC_CASE(EPI_PROXY_RAW, 256)
#undef SPA_TC_CASE
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// tcgen05 GEMM, weight-stationary (swap-AB) for few tokens (M <= 256)
//
// The MMA's M side (128 TMEM lanes) is a tile of 128 weight rows (output
// features) and its N side is all NT tokens, so every weight byte is streamed
// from HBM once per call however many tokens there are.  NACC = 2 keeps two
// accumulators (W_gate and W_up rows of the same features) side by side in
// TMEM.  The TMA ring is as deep as a fixed shared-memory budget allows for
// the stage size (fewer tokens -> more stages in flight).  The epilogue moves
// the transposed accumulator to shared memory in chunks of up to 128 tokens
// (tile[token][feature]) and reuses run_epilogue.
// ---------------------------------------------------------------------------
constexpr int kWsW = 128 * 128;          // one 128-row x 64-column weight tile (bytes)
constexpr int kWsRing = 200 * 1024;      // bytes of the TMA ring (one CTA per SM)
constexpr int kWsMaxStages = 8;
constexpr int kWsSmem = kWsRing + 1024;

// Tokens per epilogue chunk: the fp32 chunk tile [tokens][FEAT + 4] reuses the ring.
__host__ __device__ constexpr int ws_chunk(int nacc) {
  return (kWsRing / ((nacc * 128 + 4) * 4)) / 32 * 32 < 256 ? (kWsRing / ((nacc * 128 + 4) * 4)) / 32 * 32
                                                            : 256;
}

__host__ __device__ inline int ws_stages(int nacc, int NT) {
  const int st = kWsRing / (nacc * kWsW + NT * 128);
  return st < kWsMaxStages ? st : kWsMaxStages;
}

// tile[row][0..FEAT) <- sum over splits q = 0..S-1 (in that order) of the
// partial rows c0 + row, row < nt, from base + q * slot ([NT][FEAT] fp32
// each), except split `own` (>= 0), whose partial rows are already in the
// tile: U items of QMAX loads in flight per thread (S <= QMAX).
template <int U, int QMAX, int FEAT>
__device__ __forceinline__ void ws_sum_splits(const float* base, size_t slot, int S, int own, int c0, int nt,
                                              float* tile, int ld, int tid, int nthr) {
  constexpr int C4 = FEAT / 4;
  const int total = nt * C4;
  for (int it0 = tid; it0 < total; it0 += U * nthr) {
    float4 v[U][QMAX];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int it = it0 + u * nthr;
      const size_t off = (size_t)(c0 + it / C4) * FEAT + (it % C4) * 4;
#pragma unroll
      for (int q = 0; q < QMAX; ++q)
        if (q < S && it < total)
          v[u][q] = q == own ? *reinterpret_cast<const float4*>(tile + (it / C4) * ld + (it % C4) * 4)
                             : __ldcg(reinterpret_cast<const float4*>(base + q * slot + off));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int it = it0 + u * nthr;
      if (it >= total) continue;
      float4 acc = v[u][0];
#pragma unroll
      for (int q = 1; q < QMAX; ++q)
        if (q < S) { acc.x += v[u][q].x; acc.y += v[u][q].y; acc.z += v[u][q].z; acc.w += v[u][q].w; }
      *reinterpret_cast<float4*>(tile + (it / C4) * ld + (it % C4) * 4) = acc;
    }
  }
}

// The NACC weight boxes (128 rows x 64 columns each) of one k-block of
// column tile n_tile: GATEUP -> the first NACC/2 from W_gate, the rest the
// same rows of W_up; otherwise 128 consecutive rows per accumulator.
template <int NACC>
__device__ __forceinline__ void ws_load_weights(const TcWsParams& p, int n_tile, uint8_t* sw,
                                                uint64_t* bar, int kx) {
  constexpr int FEAT = NACC * 128;
#pragma unroll
  for (int a = 0; a < NACC; ++a) {
    int src, row;
    if (p.b_mode == B_GATEUP) {
      const int hal = NACC / 2 > 0 ? NACC / 2 : 1;  // gate/up blocks come in pairs (NACC >= 2)
      src = a < hal ? 0 : 1;
      row = n_tile * (FEAT / 2) + (a % hal) * 128;
    } else if (p.b_mode == B_CONCAT3) {
      const int g = n_tile * FEAT + a * 128;
      src = g / p.b_rows_per_src;
      row = g % p.b_rows_per_src;
      if (src > 2) {  // past the last matrix: a box wholly out of range reads zeros
        src = 2;
        row = p.b_rows_per_src;
      }
    } else {
      src = 0;
      row = n_tile * FEAT + a * 128;
    }
    tma_load_2d(sw + a * kWsW, &p.tmW[src], bar, kx, row);
  }
}

template <int MODE, int NACC>
__global__ void __launch_bounds__(kThreads, 1) tc_ws_kernel(const __grid_constant__ TcWsParams p) {
  constexpr int W_BYTES = NACC * kWsW;
  constexpr int FEAT = NACC * 128;
  constexpr int LD = FEAT + 4;
  constexpr int CHUNK = ws_chunk(NACC);
  static_assert(CHUNK * LD * 4 <= kWsRing, "epilogue tile must fit the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kWsMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kWsMaxStages];
  __shared__ __align__(8) uint64_t accum_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_issued, s_consumed;  // stages whose boxes were requested / consumed by the MMA
  __shared__ int s_all_in;
  __shared__ int2 s_rows[256];  // >= CHUNK
  __shared__ float s_scale[MODE == EPI_SWIGLU ? 256 : 1];  // the folded FFN RMSNorm, per token

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, S = gridDim.x;
  const int n_tile = blockIdx.y;
  const int NT = p.NT;  // tokens per MMA, multiple of 32, <= 256
  const int STAGES = ws_stages(NACC, NT);
  const int X_BYTES = NT * 128;
  const int STAGE_BYTES = W_BYTES + X_BYTES;  // multiple of 1024
  const int KB = p.K / 64;
  const int kb0 = (split * KB) / S, kb1 = ((split + 1) * KB) / S;
  const int nk = kb1 - kb0;
  // CTAs start their k-loop at staggered blocks so they do not all read the
  // same token tile at once (the sum order stays fixed per tile)
  const int rot = nk > 0 ? (n_tile * 5) % nk : 0;
  int* err = p.ep.err;
  // token rows whose epilogue this CTA runs first: with split-K through
  // global memory, split q takes rows [q*NT/S, (q+1)*NT/S); otherwise from 0
  const bool g_split = p.part != nullptr && S > 1;
  const int g_r0 = g_split ? (split * NT) / S : 0;
  const int g_r1 = g_split ? ((split + 1) * NT) / S : NT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&accum_bar, 1);
    abort_flag = 0;
    s_issued = 0;
    s_consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // The weights do not depend on earlier kernels: the weight boxes of the
  // first stages are requested before griddepcontrol.wait, so they stream
  // while the previous kernel finishes; the token tiles follow the wait.
  const int pre = nk < STAGES ? nk : STAGES;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmX);
    s_issued = pre;
    for (int it = 0; it < pre; ++it) {
      uint8_t* sw = smem + it * STAGE_BYTES;
      mbar_arrive_expect_tx(&full_bar[it], (uint32_t)STAGE_BYTES);
      int kit = it + rot;
      if (kit >= nk) kit -= nk;
      const int kx = (kb0 + kit) * 64;
      ws_load_weights<NACC>(p, n_tile, sw, &full_bar[it], kx);
    }
  }
  if (warp == 0 && lane == 0) {
    griddep_wait();
    for (int it = 0; it < pre; ++it) {
      int kit = it + rot;
      if (kit >= nk) kit -= nk;
      tma_load_2d(smem + it * STAGE_BYTES + W_BYTES, &p.tmX, &full_bar[it], (kb0 + kit) * 64, 0);
    }
    for (int it = pre; it < nk; ++it) {
      const int s = it % STAGES;
      if (it >= STAGES && !mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, &abort_flag, err, 211))
        break;
      uint8_t* sw = smem + s * STAGE_BYTES;
      uint8_t* sx = sw + W_BYTES;
      mbar_arrive_expect_tx(&full_bar[s], (uint32_t)STAGE_BYTES);
      int kit = it + rot;
      if (kit >= nk) kit -= nk;
      const int kx = (kb0 + kit) * 64;
      ws_load_weights<NACC>(p, n_tile, sw, &full_bar[s], kx);
      tma_load_2d(sx, &p.tmX, &full_bar[s], kx, 0);
      s_issued = it + 1;
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, NT);
    for (int it = 0; it < nk; ++it) {
      const int s = it % STAGES;
      if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, &abort_flag, err, 212)) break;
      s_consumed = it + 1;
      tc_fence_after();
      const uint32_t sw = smem_u32(smem + s * STAGE_BYTES);
      const uint64_t dx = smem_desc_sw128(sw + W_BYTES);
#pragma unroll
      for (int a = 0; a < NACC; ++a) {
        const uint64_t dw = smem_desc_sw128(sw + a * kWsW);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem + (uint32_t)(a * NT), dw + 2 * kk, dx + 2 * kk, idesc,
                    (it > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&empty_bar[s]);
    }
    umma_commit(&accum_bar);
  } else if (warp >= 2) {
    // idle during the main loop: fetch the first chunk's row indices now
    griddep_wait();
    stage_rows(p.ep, g_r0, 0, min(CHUNK, g_r1 - g_r0), s_rows, threadIdx.x - 64, kThreads - 64);
    prefetch_epilogue_rows<MODE, FEAT, __nv_bfloat16>(p.ep, g_r0, min(CHUNK, g_r1 - g_r0), n_tile,
                                                      threadIdx.x - 64, kThreads - 64);
    if constexpr (MODE == EPI_SWIGLU) {
      // and the per-token scale of the folded FFN RMSNorm: 1 / sqrt(mean(H1^2)
      // + eps), the tiles' partial sums added in tile order
      if (p.ep.ss_part != nullptr)
        for (int t = threadIdx.x - 64; t < NT; t += kThreads - 64) {
          float tot = 0.f;
          if (t < p.ep.M) {
            const float* sp = p.ep.ss_part + (size_t)t * p.ep.ss_tiles;
            for (int j0 = 0; j0 < p.ep.ss_tiles; j0 += 8) {
              float v[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = j0 + j < p.ep.ss_tiles ? sp[j0 + j] : 0.f;
#pragma unroll
              for (int j = 0; j < 8; ++j) tot += v[j];
            }
          }
          s_scale[t] = 1.0f / sqrtf(tot / (float)p.ep.d + p.ep.eps);
        }
    }
  }
  __syncwarp();

  mbar_wait(&accum_bar, 0, &abort_flag, err, 213);
  __syncthreads();
  const bool good = (abort_flag == 0);
  griddep_wait();  // the epilogue reads and writes rows that earlier kernels use
  tc_fence_after();

  float* tile = reinterpret_cast<float*>(smem);
  const int M = p.ep.M;
  const int q4 = warp & 3, half = warp >> 2;
  if (g_split) {
    // ---- split-K through global memory: publish this split's partial tile,
    // wait until every split of the tile has, then reduce this split's share
    // of the token rows (summed in split order 0..S-1) and run its epilogue
    // this split's own share of the rows stays in shared memory (the tile,
    // row c - g_r0) when it fits one epilogue chunk; only the other rows go out
    const bool own_in_tile = g_r1 - g_r0 <= CHUNK;
    {
      const int f = q4 * 32 + lane;
      float* mine = p.part + ((size_t)n_tile * S + split) * (size_t)NT * FEAT + f;
#pragma unroll 1
      for (int a = 0; a < NACC; ++a) {
#pragma unroll 1
        for (int c = 32 * half; c < NT; c += 64) {
          float v[32];
          if (good && nk > 0) {
            tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(a * NT + c), v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = c + j;
            if (own_in_tile && t >= g_r0 && t < g_r1) tile[(t - g_r0) * LD + a * 128 + f] = v[j];
            else __stcg(mine + (size_t)t * FEAT + a * 128, v[j]);
          }
        }
      }
    }
    tc_fence_before();
    __threadfence();
    __syncthreads();
    int* arrive = p.counter + n_tile;
    int* leave = p.counter + kWsCounters + n_tile;
    if (threadIdx.x == 0) {
      atomicAdd(arrive, 1);
      // every split of the tile is resident (the host keeps the grid within
      // one wave), so this wait ends unless a split gave up
      s_all_in = flag_wait(arrive, S, err, 217) ? 1 : 0;
      if (!s_all_in) abort_flag = 1;
    }
    __syncthreads();
    const bool all_in = s_all_in != 0;
    __threadfence();
    const float* base = p.part + (size_t)n_tile * S * (size_t)NT * FEAT;
    const size_t slot = (size_t)NT * FEAT;
    for (int c0 = g_r0; c0 < g_r1; c0 += CHUNK) {
      const int nt = min(CHUNK, g_r1 - c0);
      if (all_in) {
        const int own = own_in_tile ? split : -1;
        if (S <= 4)
          ws_sum_splits<4, 4, FEAT>(base, slot, S, own, c0, nt, tile, LD, threadIdx.x, kThreads);
        else
          ws_sum_splits<2, 8, FEAT>(base, slot, S, own, c0, nt, tile, LD, threadIdx.x, kThreads);
      }
      if (c0 > g_r0) stage_rows(p.ep, c0, 0, nt, s_rows, threadIdx.x, kThreads);  // first: staged above
      __syncthreads();
      // the partial rows just summed are dead: drop their L2 lines without a
      // write-back (otherwise the next kernels pay for writing them to HBM);
      // each 128-byte line of these rows is read by this CTA alone
      if (all_in) {
        constexpr int LINES = FEAT * 4 / 128;  // per row of one split's partial
        for (int it = threadIdx.x; it < S * nt * LINES; it += kThreads) {
          const int q = it / (nt * LINES), rl = it % (nt * LINES);
          const float* line = base + q * slot + (size_t)(c0 + rl / LINES) * FEAT + (rl % LINES) * 32;
          asm volatile("discard.global.L2 [%0], 128;" ::"l"(line) : "memory");
        }
      }
      if (good && all_in && c0 < M)
        run_epilogue<MODE, FEAT, __nv_bfloat16>(tile, LD, 0, nt, c0, n_tile, p.ep, s_rows, threadIdx.x, kThreads,
                                                (MODE == EPI_SWIGLU && p.ep.ss_part) ? s_scale + c0 : nullptr);
      __syncthreads();
    }
    if (threadIdx.x == 0 && atomicAdd(leave, 1) == S - 1) {
      // the last split out: every split has passed its wait, so the counters
      // can start afresh for the next launch
      *arrive = 0;
      *leave = 0;
    }
    ws_drain_on_abort(abort_flag, &accum_bar, full_bar, STAGES, s_consumed, s_issued, err);
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
    return;
  }
  if constexpr (MODE == EPI_SWIGLU && NACC == 2) {
    if (S == 1) {
      // no reduction: thread (quadrant, lane) owns feature q4*32 + lane, whose
      // gate and up accumulators sit in the same TMEM lane; silu(g) * u is
      // rounded to bf16 into a [token][128-feature] tile in the (idle) ring,
      // which then leaves as 16-byte row chunks (two 256-byte row slabs per
      // warp store instead of 64-byte pieces)
      __nv_bfloat16* T = reinterpret_cast<__nv_bfloat16*>(smem);
      if (good && nk > 0) {
        const uint32_t row_base = tmem + ((uint32_t)(q4 * 32) << 16);
#pragma unroll 1
        for (int c = 32 * half; c < NT; c += 64) {
          float g[32], u[32];
          tmem_ld32(row_base + (uint32_t)c, g);
          tmem_ld32(row_base + (uint32_t)(NT + c), u);
          if (p.ep.ss_part != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              g[j] *= s_scale[c + j];
              u[j] *= s_scale[c + j];
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) T[(c + j) * 128 + q4 * 32 + lane] = __float2bfloat16_rn(silu(g[j]) * u[j]);
        }
      }
      __syncthreads();
      if (good && nk > 0) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.ep.out);
        const int n_out = p.ep.n_out;
        for (int it = threadIdx.x; it < M * 16; it += kThreads) {
          const int t = it >> 4, f0 = n_tile * 128 + (it & 15) * 8;
          const __nv_bfloat16* src = T + t * 128 + (it & 15) * 8;
          __nv_bfloat16* dst = out + (size_t)t * n_out + f0;
          if ((n_out & 7) == 0 && f0 + 8 <= n_out) {
            *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
          } else {
            for (int e = 0; e < 8 && f0 + e < n_out; ++e) dst[e] = src[e];
          }
        }
      }
      tc_fence_before();
      __syncthreads();
      ws_drain_on_abort(abort_flag, &accum_bar, full_bar, STAGES, s_consumed, s_issued, err);
      tc_fence_after();
      if (warp == 0) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
      return;
    }
  }
  for (int c0 = 0; c0 < NT; c0 += CHUNK) {
    const int nt = min(CHUNK, NT - c0);
    if (good) {
      const int f = q4 * 32 + lane;
#pragma unroll 1
      for (int a = 0; a < NACC; ++a) {
#pragma unroll 1
        for (int c = 32 * half; c < nt; c += 64) {
          float v[32];
          if (nk > 0) {
            tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(a * NT + c0 + c), v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) tile[(c + j) * LD + a * 128 + f] = v[j];
        }
      }
    }
    tc_fence_before();
    int r0 = 0, r1 = nt;
    if (S > 1) {
      cluster_sync();
      const int q = (int)cluster_ctarank();
      r0 = (q * nt) / S;
      r1 = ((q + 1) * nt) / S;
      if (good) cluster_reduce_rows<FEAT>(tile, LD, r0, r1, S, threadIdx.x, kThreads);
      cluster_sync();
    } else {
      __syncthreads();
    }
    if (good && c0 + r0 < M) {
      if (c0 > 0) {  // the first chunk's rows were staged during the main loop
        stage_rows(p.ep, c0, r0, r1, s_rows, threadIdx.x, kThreads);
        __syncthreads();
      }
      run_epilogue<MODE, FEAT, __nv_bfloat16>(tile, LD, r0, r1, c0, n_tile, p.ep, s_rows, threadIdx.x, kThreads,
                                              (MODE == EPI_SWIGLU && p.ep.ss_part) ? s_scale + c0 : nullptr);
    }
    __syncthreads();
  }
  ws_drain_on_abort(abort_flag, &accum_bar, full_bar, STAGES, s_consumed, s_issued, err);
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
}

template <int MODE, int NACC>
static cudaError_t launch_ws_typed(const TcWsParams& p, int n_tiles, int splits,
                                   cudaStream_t stream) {
  auto kern = tc_ws_kernel<MODE, NACC>;
  cudaError_t ec = configure_kernel((const void*)kern, kWsSmem, false);
  if (ec != cudaSuccess) return ec;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits, n_tiles, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kWsSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.part ? 1 : splits;  // global split-K: separate CTAs
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int MODE, int NACC>
static int ws_max_clusters(int splits) {
  static int cache_all[kMaxDevices][9] = {{0}};  // per device, filled once (benign race: same value)
  if (splits < 1 || splits > 8) return 0;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int* cache = cache_all[dev];
  if (cache[splits] == 0) {
    auto kern = tc_ws_kernel<MODE, NACC>;
    if (configure_kernel((const void*)kern, kWsSmem, false) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kWsSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cache[splits] = n > 0 ? n : -1;
  }
  return cache[splits] > 0 ? cache[splits] : 0;
}

#define SPA_WS_MODES(X)                                                   \
  X(EPI_STORE, 1) X(EPI_STORE, 2) X(EPI_STORE, 4)                         \
  X(EPI_QKV, 1) X(EPI_QKV, 2) X(EPI_QKV, 4)                               \
  X(EPI_RESID, 1) X(EPI_RESID, 2) X(EPI_RESID, 4)                         \
  X(EPI_SWIGLU, 2) X(EPI_SWIGLU, 4)                                       \
  X(EPI_RESID_SCATTER, 1) X(EPI_RESID_SCATTER, 2) X(EPI_RESID_SCATTER, 4) \
  X(EPI_ARGMAX, 1) X(EPI_ARGMAX, 2) X(EPI_ARGMAX, 4)

cudaError_t launch_tc_ws(int mode, int nacc, const TcWsParams& p, int n_tiles, int splits,
                         cudaStream_t stream) {
  if (p.part && (p.counter == nullptr || n_tiles > kWsCounters || splits > 8)) return cudaErrorInvalidValue;
#define SPA_WS_CASE(M_, A_) \
  if (mode == M_ && nacc == A_) return launch_ws_typed<M_, A_>(p, n_tiles, splits, stream);
  SPA_WS_MODES(SPA_WS_CASE)
#undef SPA_WS_CASE
  return cudaErrorInvalidValue;
}

int ws_resident_ctas(int mode, int nacc) {
  int resident = 0;
#define SPA_WS_FIT(M_, A_) \
  if (mode == M_ && nacc == A_) resident = ws_max_clusters<M_, A_>(1);
  SPA_WS_MODES(SPA_WS_FIT)
#undef SPA_WS_FIT
  return resident;
}

int plan_ws_global_splits(int mode, int nacc, int n_tiles, int KB, int g_max) {
  const int resident = ws_resident_ctas(mode, nacc);
  // the cluster plan's estimate (see plan_ws_splits)
  const int sc = plan_ws_splits(mode, nacc, n_tiles, KB);
  int fit = 0;
#define SPA_WS_FIT(M_, A_) \
  if (mode == M_ && nacc == A_) fit = ws_max_clusters<M_, A_>(sc);
  SPA_WS_MODES(SPA_WS_FIT)
#undef SPA_WS_FIT
  const double c_cost = fit > 0 ? ((n_tiles + fit - 1) / fit) * ((KB + sc - 1) / sc + 12.0) : 1e30;
  int best = 0;
  double best_cost = c_cost;
  for (int s = 2; s <= 8 && s <= g_max; ++s) {
    if (KB / s < 4 || n_tiles * s > resident) continue;
    // one wave; each split also stores its partial tile and reduces its share
    // of the rows from every split's (about six k-blocks' time)
    const double cost = (KB + s - 1) / s + 12.0 + 6.0;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

// Split-K plan for the weight-stationary GEMM: estimated time ~ waves x
// (k-blocks per CTA + fixed per-CTA cost in k-block units), waves from how
// many clusters of `splits` CTAs the GPU holds at once.
int plan_ws_splits(int mode, int nacc, int n_tiles, int KB) {
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 8; ++s) {
    if (KB / s < 2) break;
    int fit = 0;
#define SPA_WS_FIT(M_, A_) \
  if (mode == M_ && nacc == A_) fit = ws_max_clusters<M_, A_>(s);
    SPA_WS_MODES(SPA_WS_FIT)
#undef SPA_WS_FIT
    if (fit <= 0) continue;
    const int waves = (n_tiles + fit - 1) / fit;
    const double cost = waves * ((KB + s - 1) / s + 12.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

// ---------------------------------------------------------------------------
// fp32 CUDA-core GEMM (64 x 128 tiles, 256 threads, 4 x 8 outputs per thread)
// ---------------------------------------------------------------------------
constexpr int kSBM = 64, kSBN = 128, kSBK = 16;

__device__ __forceinline__ const float* simt_b_row(const SimtGemmParams& p, int n_tile, int c) {
  int src, row;
  if (p.b_mode == B_GATEUP) {
    src = c < kSBN / 2 ? 0 : 1;
    row = n_tile * (kSBN / 2) + (c % (kSBN / 2));
  } else if (p.b_mode == B_CONCAT3) {
    const int g = n_tile * kSBN + c;
    src = g / p.b_rows_per_src;
    row = g % p.b_rows_per_src;
    if (src > 2) return nullptr;
  } else {
    src = 0;
    row = n_tile * kSBN + c;
  }
  if (row >= p.b_rows_per_src) return nullptr;
  return p.B[src] + (size_t)row * p.K;
}

template <int MODE>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtGemmParams p) {
  __shared__ __align__(16) float As[kSBK][kSBM + 4];
  __shared__ __align__(16) float Bs[kSBK][kSBN + 4];
  __shared__ __align__(16) float tile[kSBM * (kSBN + 4)];
  griddep_launch_dependents();
  griddep_wait();
  const int tid = threadIdx.x;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y;
  const int ty = tid / 16, tx = tid % 16;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  // loaders: A: 64 rows x 16 k (4 per thread); B: 128 rows x 16 k (8 per thread)
  const int a_row = tid / 4, a_k = (tid % 4) * 4;
  const int ga = m_tile * kSBM + a_row;
  const float* a_ptr = ga < p.ep.M ? p.A + (size_t)ga * p.K : nullptr;
  const int b_row = tid / 2, b_k = (tid % 2) * 8;
  const float* b_ptr = simt_b_row(p, n_tile, b_row);

  for (int k0 = 0; k0 < p.K; k0 += kSBK) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + a_k + j;
      As[a_k + j][a_row] = (a_ptr && k < p.K) ? a_ptr[k] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = k0 + b_k + j;
      Bs[b_k + j][b_row] = (b_ptr && k < p.K) ? b_ptr[k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kSBK; ++k) {
      float a[4], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[k][tx * 8 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  constexpr int LD = kSBN + 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) tile[(ty * 4 + i) * LD + tx * 8 + j] = acc[i][j];
  __shared__ int2 s_rows[kSBM];
  stage_rows(p.ep, m_tile * kSBM, 0, kSBM, s_rows, tid, 256);
  __syncthreads();
  run_epilogue<MODE, kSBN, float>(tile, LD, 0, kSBM, m_tile * kSBM, n_tile, p.ep, s_rows, tid, 256);
}

cudaError_t launch_simt_gemm(int mode, const SimtGemmParams& p, int m_tiles, int n_tiles,
                             cudaStream_t stream) {
  dim3 grid(n_tiles, m_tiles), block(256);
  switch (mode) {
    case EPI_STORE: return launch_k(simt_gemm_kernel<EPI_STORE>, grid, block, 0, stream, p);
    case EPI_QKV: return launch_k(simt_gemm_kernel<EPI_QKV>, grid, block, 0, stream, p);
    case EPI_RESID: return launch_k(simt_gemm_kernel<EPI_RESID>, grid, block, 0, stream, p);
    case EPI_SWIGLU: return launch_k(simt_gemm_kernel<EPI_SWIGLU>, grid, block, 0, stream, p);
    case EPI_RESID_SCATTER: return launch_k(simt_gemm_kernel<EPI_RESID_SCATTER>, grid, block, 0, stream, p);
    case EPI_PROXY: return launch_k(simt_gemm_kernel<EPI_PROXY>, grid, block, 0, stream, p);
    case EPI_ARGMAX: return launch_k(simt_gemm_kernel<EPI_ARGMAX>, grid, block, 0, stream, p);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// Tensor maps
// ---------------------------------------------------------------------------
int encode_bf16_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  return encode_bf16_map_box(map, base, rows, cols, 128);
}

int encode_bf16_map_box(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return -1;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

}  // namespace spa
