// Stream-K weight-streaming GEMM for the cached layer step (bf16, sm_100a).
//
// The four GEMMs of a cached layer step (QKV, O-proj, gate/up, down) multiply
// a large weight matrix by the few selected tokens (M <= 256): they are bound
// by streaming the weights from HBM, so every SM has to stream its share of
// them all the time.  The weights are cut into tiles of 128 output features
// (the 128 TMEM lanes of one tcgen05.mma, M = 128) and k-blocks of 64 input
// columns; the tile-major list of (tile, k-block) units is split evenly over
// one CTA per SM (stream-K), so no SM idles whatever the tile count is.
//
// A CTA's range is a run of segments: the tail of one tile, whole tiles, the
// head of another.  Roles (8 warps):
//   warp 0      TMA producer: for every unit the weight box (128 x 64) and the
//               token box (NT x 64) into a ring of stages, running straight
//               across segment boundaries.  The weight boxes of the first
//               stages are requested before griddepcontrol.wait (weights do
//               not depend on earlier kernels).
//   warp 1      one thread issues tcgen05.mma (D[f, t] += W[f, k] X[t, k]) into
//               one of two TMEM accumulators (segment j uses j % 2), so the
//               epilogue of a segment overlaps the main loop of the next.
// A unit may also hold NACC = 2 consecutive 128-row tiles that share the
// token box of the stage (half the token-tile traffic per weight byte); then
// two accumulators per buffer, and one buffer when 4 * NT > 512 TMEM columns.
//   warps 2-3   stage every token's (sequence, cache row), then idle.
//   warps 4-7   epilogue: thread (quadrant q, lane) owns feature row
//               f = 32 q + lane of the tile (its TMEM lane).
// A tile split over several CTAs is fixed up without any CTA waiting for
// another: each segment's CTA writes its fp32 partial tile [128][NT] to a
// scratch slot and counts it in the tile's counter; the CTA that brings the
// counter to the number of segments (or finds all other segments counted
// before writing its own) sums every segment's partial in k-block order
// (own partial straight from TMEM) and runs the fused epilogue, then resets
// the counter.  The summation order is fixed by the partition, which depends
// only on the weight shape and the SM count, so results are deterministic and
// every output row depends only on its own token.
//
// Fused epilogues (from registers, one bf16 per thread and token; a warp
// writes 32 consecutive features = 64 bytes of a row):
//   EPI_QKV            RoPE on Q and K (the pair partner of feature f is
//                      f ^ (head_dim / 2), exchanged through shared memory),
//                      Q to the compact buffer, K and V into K^c, V^c rows I
//   EPI_RESID          H1[t] = acc + H[b, I[t]]
//   EPI_SWIGLU         tile = 64 gate rows (lanes 0-63) + the same 64 up rows
//                      (lanes 64-127); A[t, f] = silu(gate) * up
//   EPI_RESID_SCATTER  H^c[b, I[t]] = acc + H1[t] (+ compact copy, score zero)
//   EPI_STORE          out[t, n] = acc
#include <cstdio>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

constexpr int kSkThreads = 256;
constexpr int kSkRing = 196 * 1024;     // bytes of the TMA ring
constexpr int kSkMaxStages = 16;
constexpr int kSkSmem = kSkRing + 1024;  // + alignment slack
constexpr int kSkW = 128 * 128;          // one weight stage: 128 rows x 64 columns bf16
constexpr int kSkXLd = 33;               // exchange tile row stride (floats)

__device__ __forceinline__ float sk_silu(float g) { return g * __frcp_rn(1.0f + __expf(-g)); }

// First unit of CTA g of G over U units.
__host__ __device__ __forceinline__ int sk_start(int g, int G, int U) {
  return (int)(((long long)g * U) / G);
}
// The CTA whose range holds unit u.
__device__ __forceinline__ int sk_owner(int u, int G, int U) {
  int g = (int)(((long long)u * G) / U);
  while (g + 1 < G && sk_start(g + 1, G, U) <= u) ++g;
  while (g > 0 && sk_start(g, G, U) > u) --g;
  return g;
}
// Scratch slot of CTA g's partial of tile t: slot 2g for the CTA's first
// segment, 2g + 1 for its last (a CTA has at most two partial segments).
__device__ __forceinline__ int sk_slot(int g, int t, int G, int U, int KB) {
  return 2 * g + (sk_start(g, G, U) / KB == t ? 0 : 1);
}

// The weight boxes of unit (tile t, k-block kb) into sw (one 128-row stage).
__device__ __forceinline__ void sk_load_w(const SkParams& p, int t, int kb, uint8_t* sw, uint64_t* bar) {
  const int kx = kb * 64;
  if (p.b_mode == B_GATEUP) {  // 64 gate rows, then the same 64 up rows
    tma_load_2d(sw, &p.tmW[0], bar, kx, t * 64);
    tma_load_2d(sw + kSkW / 2, &p.tmW[1], bar, kx, t * 64);
  } else if (p.b_mode == B_CONCAT3) {
    const int g = t * 128;
    tma_load_2d(sw, &p.tmW[g / p.b_rows_per_src], bar, kx, g % p.b_rows_per_src);
  } else {
    tma_load_2d(sw, &p.tmW[0], bar, kx, t * 128);
  }
}

// s_rows[t] = (sequence, cache row) of token t for every t < NT: (0, -1) past
// the last token or for an index outside [0, N) (reported).
__device__ void stage_rows_sk(const EpiParams& ep, int2* s_rows, int tid, int nthr) {
  for (int t = tid; t < 256; t += nthr) {
    int2 v = make_int2(0, -1);
    if (t < ep.M) {
      v.x = t / ep.tokens_per_seq;
      v.y = ep.idx ? ep.idx[t] : (t % ep.tokens_per_seq);
      if (v.y < 0 || v.y >= ep.N) {
        report_error(ep.err, DEVERR_INDEX, 807);
        v.y = -1;
      }
    }
    s_rows[t] = v;
  }
}

template <int MODE>
__device__ __forceinline__ void sk_store_chunk(const SkParams& p, int t, int f, int c0, const float* acc,
                                               const float* partner, const int2* s_rows) {
  const EpiParams& ep = p.ep;
  const int M = ep.M;
  __nv_bfloat16* const outb = reinterpret_cast<__nv_bfloat16*>(ep.out);
  if constexpr (MODE == EPI_STORE) {
    const int n = t * 128 + f;
    if (n >= ep.n_out) return;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < M) outb[(size_t)(c0 + j) * ep.n_out + n] = __float2bfloat16_rn(acc[j]);
  } else if constexpr (MODE == EPI_RESID) {
    const int n = t * 128 + f;
    if (n >= ep.n_out) return;
    const __nv_bfloat16* res = reinterpret_cast<const __nv_bfloat16*>(ep.resid);
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int2 br = s_rows[c0 + j];
      h[j] = (c0 + j < M && br.y >= 0) ? __bfloat162float(res[((size_t)br.x * ep.N + br.y) * ep.d + n]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < M && s_rows[c0 + j].y >= 0)
        outb[(size_t)(c0 + j) * ep.d + n] = __float2bfloat16_rn(acc[j] + h[j]);
  } else if constexpr (MODE == EPI_RESID_SCATTER) {
    const int n = t * 128 + f;
    if (n >= ep.n_out) return;
    const __nv_bfloat16* res = reinterpret_cast<const __nv_bfloat16*>(ep.resid);
    __nv_bfloat16* rc = reinterpret_cast<__nv_bfloat16*>(ep.row_copy);
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      h[j] = c0 + j < M ? __bfloat162float(res[(size_t)(c0 + j) * ep.d + n]) : 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int2 br = s_rows[c0 + j];
      if (c0 + j >= M || br.y < 0) continue;
      const __nv_bfloat16 v = __float2bfloat16_rn(acc[j] + h[j]);
      outb[((size_t)br.x * ep.N + br.y) * ep.d + n] = v;
      if (rc) rc[(size_t)(c0 + j) * ep.d + n] = v;
      if (ep.score_zero && n == 0) ep.score_zero[(size_t)br.x * ep.N + br.y] = 0.f;
    }
  } else if constexpr (MODE == EPI_SWIGLU) {
    if (f >= 64) return;  // the up rows only feed their gate partners
    const int fo = t * 64 + f;
    if (fo >= ep.n_out) return;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < M) outb[(size_t)(c0 + j) * ep.n_out + fo] = __float2bfloat16_rn(sk_silu(acc[j]) * partner[j]);
  } else if constexpr (MODE == EPI_QKV) {
    const int n = t * 128 + f;
    if (n >= ep.n_out) return;
    const int part = n / ep.d, col = n % ep.d;
    const int hd = ep.head_dim, hh = hd / 2;
    const int jj = col % hd, i = jj % hh;
    const bool first = jj < hh;
    float cs[32], sn[32];
    if (part < 2) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int2 br = s_rows[c0 + j];
        const bool ok = c0 + j < M && br.y >= 0;
        cs[j] = ok ? ep.rope_cos[(size_t)br.y * hh + i] : 0.f;
        sn[j] = ok ? ep.rope_sin[(size_t)br.y * hh + i] : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int2 br = s_rows[c0 + j];
      if (c0 + j >= M || br.y < 0) continue;
      float v = acc[j];
      if (part < 2) {
        // first half: x1 c - x2 s; second half: x2 c + x1 s (x1 = first-half value)
        v = first ? acc[j] * cs[j] - partner[j] * sn[j] : acc[j] * cs[j] + partner[j] * sn[j];
      }
      const __nv_bfloat16 b = __float2bfloat16_rn(v);
      if (part == 0) outb[(size_t)(c0 + j) * ep.d + col] = b;
      else reinterpret_cast<__nv_bfloat16*>(part == 1 ? ep.k_cache : ep.v_cache)[((size_t)br.x * ep.N + br.y) * ep.d + col] = b;
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(kSkThreads, 1) tc_sk_kernel(const __grid_constant__ SkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kSkMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kSkMaxStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, prod_issued, mma_consumed, s_flag, s_ok;
  __shared__ int2 s_rows[256];
  __shared__ float xch[4][32 * kSkXLd];

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int KB = p.KB, U = p.units, NT = p.NT;
  const int u0 = sk_start(g, G, U), u1 = sk_start(g + 1, G, U);
  const int n_units = u1 - u0;
  const int NACC = p.nacc, NBUF = p.nbuf;
  const int W_BYTES = NACC * kSkW;
  const int X_BYTES = NT * 128;
  const int STAGE_BYTES = W_BYTES + X_BYTES;  // multiple of 1024
  int STAGES = kSkRing / STAGE_BYTES;
  if (STAGES > kSkMaxStages) STAGES = kSkMaxStages;
  int* err = p.ep.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 1);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    s_ok = 1;
    prod_issued = mma_consumed = 0;
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

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tmX);
      const int pre = n_units < STAGES ? n_units : STAGES;
      for (int it = 0; it < pre; ++it) {
        const int u = u0 + it;
        mbar_arrive_expect_tx(&full_bar[it], (uint32_t)STAGE_BYTES);
        for (int a = 0; a < NACC; ++a)
          sk_load_w(p, (u / KB) * NACC + a, u % KB, smem + it * STAGE_BYTES + a * kSkW, &full_bar[it]);
      }
      griddep_wait();  // the token rows come from earlier kernels
      for (int it = 0; it < pre; ++it)
        tma_load_2d(smem + it * STAGE_BYTES + W_BYTES, &p.tmX, &full_bar[it], ((u0 + it) % KB) * 64, 0);
      int it = pre;
      for (; it < n_units; ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, &abort_flag, err, 801)) break;
        const int u = u0 + it;
        uint8_t* sw = smem + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)STAGE_BYTES);
        for (int a = 0; a < NACC; ++a) sk_load_w(p, (u / KB) * NACC + a, u % KB, sw + a * kSkW, &full_bar[s]);
        tma_load_2d(sw + W_BYTES, &p.tmX, &full_bar[s], (u % KB) * 64, 0);
      }
      prod_issued = it;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, NT);
      int it = 0, j = 0;
      bool ok = true;
      for (int u = u0; ok && u < u1; ++j) {
        const int kb0 = u % KB;
        const int kb1 = kb0 + (u1 - u < KB - kb0 ? u1 - u : KB - kb0);
        const int a = j % NBUF;
        if (j >= NBUF && !mbar_wait(&acc_empty[a], ((j / NBUF) - 1) & 1, &abort_flag, err, 802)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * NACC * NT);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, &abort_flag, err, 803)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t dx = smem_desc_sw128(sa + W_BYTES);
          for (int sub = 0; sub < NACC; ++sub) {
            const uint64_t dw = smem_desc_sw128(sa + sub * kSkW);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(d_tmem + (uint32_t)(sub * NT), dw + 2 * kk, dx + 2 * kk, idesc,
                        (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[a]);
        u += kb1 - kb0;
      }
      mma_consumed = it;
      umma_commit(&mma_done);  // every MMA issued by this thread has completed
    }
  } else if (warp < 4) {
    griddep_wait();
    stage_rows_sk(p.ep, s_rows, threadIdx.x - 64, 64);
    named_bar_sync(1, 192);
  } else {
    // ------------------------------------------------------------ epilogue
    griddep_wait();
    named_bar_sync(1, 192);  // s_rows staged
    const int q = warp - 4, f = q * 32 + lane;
    const int et = threadIdx.x - 128;  // 0..127
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // the RoPE / SwiGLU partner of feature f
    const int half = MODE == EPI_SWIGLU ? 64 : p.ep.head_dim / 2;
    const int pf = f ^ half;
    const int pq = pf >> 5, pl = pf & 31;
    const int M = p.ep.M;
    int j = 0;
    for (int u = u0; u < u1; ++j) {
      const int t = u / KB, kb0 = u % KB;
      const int kb1 = kb0 + (u1 - u < KB - kb0 ? u1 - u : KB - kb0);
      u += kb1 - kb0;
      const int a = j % NBUF;
      const bool got = mbar_wait(&acc_full[a], (j / NBUF) & 1, &abort_flag, err, 804);
      __syncwarp();
      // the four epilogue warps agree on whether to go on, so every named
      // barrier below is reached by all 128 threads or by none
      const bool warp_ok = __all_sync(0xffffffffu, got);
      if (lane == 0 && !warp_ok) atomicAnd(&s_ok, 0);
      named_bar_sync(2, 128);
      if (!s_ok) break;
      tc_fence_after();
      const uint32_t buf_tmem = lane_base + (uint32_t)(a * NACC * NT);
      // the tile's segments: CTAs g_first..g_last, own index own_s
      const int g_first = sk_owner(t * KB, G, U), g_last = sk_owner(t * KB + KB - 1, G, U);
      const int nseg = g_last - g_first + 1, own_s = g - g_first;
      bool finisher = true;
      if (nseg > 1) {
        if (et == 0) {
          int c;
          asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(c) : "l"(p.count + t) : "memory");
          s_flag = (c == nseg - 1) ? 1 : 0;  // every other segment is in: no need to publish ours
        }
        named_bar_sync(2, 128);
        finisher = s_flag != 0;
        named_bar_sync(2, 128);
        if (!finisher) {
          for (int sub = 0; sub < NACC; ++sub) {
            float* dst = p.part + (((size_t)sk_slot(g, t, G, U, KB) * NACC + sub) * 128 + f) * NT;
            const uint32_t acc_tmem = buf_tmem + (uint32_t)(sub * NT);
            for (int c0 = 0; c0 < NT; c0 += 32) {
              float v[32];
              tmem_ld32(acc_tmem + (uint32_t)c0, v);
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                __stcg(reinterpret_cast<float4*>(dst + c0 + i), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
            }
          }
          __threadfence();
          named_bar_sync(2, 128);
          if (et == 0) s_flag = (atomicAdd(p.count + t, 1) == nseg - 1) ? 1 : 0;
          named_bar_sync(2, 128);
          finisher = s_flag != 0;
          named_bar_sync(2, 128);
        }
      }
      if (finisher) {
        __threadfence();
        for (int sub = 0; sub < NACC; ++sub)
        for (int c0 = 0; c0 < NT && c0 < M; c0 += 32) {
          const uint32_t acc_tmem = buf_tmem + (uint32_t)(sub * NT);
          const int vt = t * NACC + sub;  // 128-row tile of the weights
          float acc[32];
          tmem_ld32(acc_tmem + (uint32_t)c0, acc);  // own partial
          if (nseg > 1) {
            float sum[32];
            for (int s = 0; s < nseg; ++s) {  // k-block order
              float x[32];
              if (s == own_s) {
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = acc[i];
              } else {
                const float4* src = reinterpret_cast<const float4*>(
                    p.part + (((size_t)sk_slot(g_first + s, t, G, U, KB) * NACC + sub) * 128 + f) * NT + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float4 w = __ldcg(src + i);
                  x[4 * i] = w.x; x[4 * i + 1] = w.y; x[4 * i + 2] = w.z; x[4 * i + 3] = w.w;
                }
              }
              if (s == 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) sum[i] = x[i];
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) sum[i] += x[i];
              }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = sum[i];
          }
          float partner[32];
          if constexpr (MODE == EPI_QKV || MODE == EPI_SWIGLU) {
            float* mine = xch[q];
#pragma unroll
            for (int i = 0; i < 32; ++i) mine[i * kSkXLd + lane] = acc[i];
            named_bar_sync(3, 128);
            const float* theirs = xch[pq];
#pragma unroll
            for (int i = 0; i < 32; ++i) partner[i] = theirs[i * kSkXLd + pl];
            named_bar_sync(3, 128);
          }
          sk_store_chunk<MODE>(p, vt, f, c0, acc, partner, s_rows);
        }
        if (nseg > 1 && et == 0) p.count[t] = 0;  // every segment has counted: ready for the next launch
      }
      // the accumulator buffer may be overwritten by segment j + 2
      tc_fence_before();
      named_bar_sync(2, 128);
      if (et == 0) mbar_arrive_cta(&acc_empty[a]);
    }
  }
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) {
    // MMAs still in flight must finish before TMEM is released; after an
    // abort, so must the copies issued into stages nobody consumed
    mbar_drain_bounded(&mma_done, 0, err, 805);
    if (abort_flag != 0)
      for (int it = mma_consumed; it < prod_issued; ++it)
        mbar_drain_bounded(&full_bar[it % STAGES], (it / STAGES) & 1, err, 806);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
}

cudaError_t launch_tc_sk(int mode, const SkParams& p, int grid, cudaStream_t stream) {
  const void* kern = nullptr;
  switch (mode) {
    case EPI_STORE: kern = (const void*)tc_sk_kernel<EPI_STORE>; break;
    case EPI_QKV: kern = (const void*)tc_sk_kernel<EPI_QKV>; break;
    case EPI_RESID: kern = (const void*)tc_sk_kernel<EPI_RESID>; break;
    case EPI_SWIGLU: kern = (const void*)tc_sk_kernel<EPI_SWIGLU>; break;
    case EPI_RESID_SCATTER: kern = (const void*)tc_sk_kernel<EPI_RESID_SCATTER>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = configure_kernel(kern, kSkSmem, false);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kSkThreads, 1, 1);
  cfg.dynamicSmemBytes = kSkSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  void* args[] = {const_cast<SkParams*>(&p)};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

int sk_stages(int nacc, int NT) {
  const int st = kSkRing / (nacc * kSkW + NT * 128);
  return st < kSkMaxStages ? st : kSkMaxStages;
}

}  // namespace spa
