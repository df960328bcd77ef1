// Stream-K weight-streaming GEMM for the cached layer step (bf16, sm_100a).
//
// The four GEMMs of a cached layer step (QKV, O-proj, gate/up, down) multiply
// a large weight matrix by the few selected tokens (M <= 256): they are bound
// by streaming the weights from HBM, so every SM has to stream its share of
// them all the time.  The weights are cut into tiles of NACC x 128 output
// features (the 128 TMEM lanes of one tcgen05.mma, M = 128, times NACC
// accumulators sharing one token box) and k-blocks of 64 input columns; the
// tile-major list of (tile, k-block) units is split evenly over one CTA per
// SM (stream-K), so no SM idles whatever the tile count is.
//
// tc_sk_kernel.  A CTA's range is a run of segments (the tail of one tile,
// maybe whole tiles, the head of another).  Roles (8 warps):
//   warp 0      TMA producer: for every unit the NACC weight boxes (128 x 64
//               each) and the token box (NT x 64) into a ring of stages,
//               straight across segment boundaries.  The weight boxes of the
//               first stages are requested before griddepcontrol.wait
//               (weights do not depend on earlier kernels).
//   warp 1      one thread issues tcgen05.mma (D[f, t] += W[f, k] X[t, k]) into
//               the accumulators of buffer j % NBUF for segment j; with two
//               buffers the epilogue of a segment overlaps the next main loop.
//   warps 4-7   epilogue: thread (quadrant q, lane) reads TMEM lane f = 32 q +
//               lane (feature f of the tile) and stores the segment's fp32
//               partial sums into its own scratch slot, token-major
//               [NT][NACC x 128], so a warp writes 128 contiguous bytes per
//               token.
// No CTA waits for another and none sums other CTAs' partials.
//
// sk_reduce_kernel<MODE>: one CTA per token row sums, for every feature, the
// partials of the tile's segments in k-block order (the order is fixed by the
// partition, which depends only on the weight shape and the grid: results are
// deterministic, and each row depends only on its own token), then applies the
// fused epilogue of the step:
//   EPI_QKV            RoPE on Q and K (pairs f, f + head_dim/2 of a head), Q
//                      to the compact buffer, K and V into K^c, V^c rows I
//   EPI_RESID          H1[t] = acc + H[b, I[t]]; with x2 given also the FFN
//                      RMSNorm of the row, x2 = RMSNorm(H1) (no separate norm
//                      kernel)
//   EPI_SWIGLU         tile = 64 gate rows (lanes 0-63) + the same 64 up rows
//                      (lanes 64-127); A[t, f] = silu(gate) * up
//   EPI_RESID_SCATTER  H^c[b, I[t]] = acc + H1[t] (+ compact copy, score zero)
//   EPI_STORE          out[t, n] = acc
// The reduce kernel is launched with programmatic dependent launch right
// behind the GEMM; its CTAs are small enough to sit beside the GEMM's, and the
// next GEMM's CTAs start prefetching their weights as soon as the GEMM's exit.
#include <algorithm>
#include <cstdio>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

constexpr int kSkThreads = 256;
constexpr int kSkRing = 200 * 1024;      // bytes of the TMA ring (leaves room for a reduce CTA beside it)
constexpr int kSkMaxStages = 16;
constexpr int kSkSmem = kSkRing + 1024;  // + alignment slack
constexpr int kSkW = 128 * 128;          // one weight box: 128 rows x 64 columns bf16
constexpr int kRedThreads = 256;
constexpr int kRedMaxSeg = 8;     // segments per tile (the host keeps the grid within it)
constexpr int kRedJobs = 4;       // feature groups summed per thread at once (all their loads in flight)
constexpr int kRedMaxTiles = 256;

__device__ __forceinline__ float sk_silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// First unit of CTA g of G over U units.
__host__ __device__ __forceinline__ int sk_start(int g, int G, int U) {
  return (int)(((long long)g * U) / G);
}
// The CTA whose range holds unit u.
__host__ __device__ __forceinline__ int sk_owner(int u, int G, int U) {
  int g = (int)(((long long)u * G) / U);
  while (g + 1 < G && sk_start(g + 1, G, U) <= u) ++g;
  while (g > 0 && sk_start(g, G, U) > u) --g;
  return g;
}

// The weight box of 128-row tile vt, k-block kb into sw.
__device__ __forceinline__ void sk_load_w(const SkParams& p, int vt, int kb, uint8_t* sw, uint64_t* bar) {
  const int kx = kb * 64;
  if (p.b_mode == B_GATEUP) {  // 64 gate rows, then the same 64 up rows
    tma_load_2d(sw, &p.tmW[0], bar, kx, vt * 64);
    tma_load_2d(sw + kSkW / 2, &p.tmW[1], bar, kx, vt * 64);
  } else if (p.b_mode == B_CONCAT3) {
    const int g = vt * 128;
    tma_load_2d(sw, &p.tmW[g / p.b_rows_per_src], bar, kx, g % p.b_rows_per_src);
  } else {
    tma_load_2d(sw, &p.tmW[0], bar, kx, vt * 128);
  }
}

__global__ void __launch_bounds__(kSkThreads, 1) tc_sk_kernel(const __grid_constant__ SkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kSkMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kSkMaxStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, prod_issued, mma_consumed, s_ok;

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int KB = p.KB, U = p.units, NT = p.NT;
  const int u0 = sk_start(g, G, U), u1 = sk_start(g + 1, G, U);
  const int n_units = u1 - u0;
  const int NACC = p.nacc, NBUF = p.nbuf, FEAT = NACC * 128;
  const int W_BYTES = NACC * kSkW;
  const int STAGE_BYTES = W_BYTES + NT * 128;  // multiple of 1024
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
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    // the scratch slots were read by the previous launch's reduce kernel
    griddep_wait();
    const int q = warp - 4, f = q * 32 + lane;
    const int et = threadIdx.x - 128;  // 0..127
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int M = p.ep.M;
    const int mt = M < NT ? M : NT;
    int j = 0;
    for (int u = u0; u < u1; ++j) {
      const int kb0 = u % KB;
      u += (u1 - u < KB - kb0 ? u1 - u : KB - kb0);
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
      // segment j of this CTA -> scratch slot g * maxseg + j, [NT][FEAT] fp32
      float* dst = p.part + ((size_t)g * p.maxseg + j) * (size_t)NT * FEAT + f;
      for (int sub = 0; sub < NACC; ++sub) {
        const uint32_t acc_tmem = lane_base + (uint32_t)((a * NACC + sub) * NT);
        for (int c0 = 0; c0 < mt; c0 += 32) {
          float v[32];
          tmem_ld32(acc_tmem + (uint32_t)c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < mt) __stcg(dst + (size_t)(c0 + i) * FEAT + sub * 128, v[i]);
        }
      }
      // the accumulator buffer may be overwritten by segment j + NBUF
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

// ---------------------------------------------------------------------------
// Reduce + fused epilogue: one CTA per token row.
// ---------------------------------------------------------------------------

// Sums of kRedJobs feature groups (4 features at 4 * f4[j] of 128-row tile
// vt[j]; skipped where ok[j] is false) over their tiles' segments, each in
// k-block order.  Every load of the jobs is issued before any sum, so a
// thread keeps up to kRedJobs * kRedMaxSeg 16-byte loads in flight.
__device__ __forceinline__ void sk_sum_jobs(const SkReduceParams& r, const int* s_nseg,
                                            const int (*s_slot)[kRedMaxSeg], int t, const int* vt,
                                            const int* f4, const bool* ok, float4* out) {
  float4 v[kRedJobs][kRedMaxSeg];
  int n[kRedJobs];
#pragma unroll
  for (int j = 0; j < kRedJobs; ++j) {
    n[j] = 0;
    if (!ok[j]) continue;
    const int tu = vt[j] / r.nacc, sub = vt[j] % r.nacc;
    n[j] = s_nseg[tu];
    const size_t off = (size_t)t * r.feat + sub * 128 + f4[j] * 4;
#pragma unroll
    for (int s = 0; s < kRedMaxSeg; ++s)
      if (s < n[j]) v[j][s] = __ldcg(reinterpret_cast<const float4*>(r.part + (size_t)s_slot[tu][s] * r.slot_floats + off));
  }
#pragma unroll
  for (int j = 0; j < kRedJobs; ++j) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n[j] > 0) acc = v[j][0];
#pragma unroll
    for (int s = 1; s < kRedMaxSeg; ++s)
      if (s < n[j]) {
        acc.x += v[j][s].x; acc.y += v[j][s].y; acc.z += v[j][s].z; acc.w += v[j][s].w;
      }
    out[j] = acc;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kRedThreads) sk_reduce_kernel(const __grid_constant__ SkReduceParams r) {
  __shared__ int s_nseg[kRedMaxTiles];
  __shared__ int s_slot[kRedMaxTiles][kRedMaxSeg];
  __shared__ float s_red[kRedThreads / 32];
  griddep_launch_dependents();
  const int t = blockIdx.x;
  const EpiParams& ep = r.ep;
  // the segments of every tile (the same integer arithmetic as the GEMM's partition)
  for (int tu = threadIdx.x; tu < r.n_tiles; tu += kRedThreads) {
    const int gf = sk_owner(tu * r.KB, r.G, r.U), gl = sk_owner(tu * r.KB + r.KB - 1, r.G, r.U);
    s_nseg[tu] = gl - gf + 1;
    for (int s = 0; s <= gl - gf && s < kRedMaxSeg; ++s) {
      const int gg = gf + s;
      s_slot[tu][s] = gg * r.maxseg + (tu - sk_start(gg, r.G, r.U) / r.KB);
    }
  }
  __syncthreads();
  griddep_wait();  // the GEMM's partials, and the rows earlier kernels wrote
  if (t >= ep.M) return;
  const int b = t / ep.tokens_per_seq;
  const int row = ep.idx ? ep.idx[t] : (t % ep.tokens_per_seq);
  if (row < 0 || row >= ep.N) {
    if (threadIdx.x == 0) report_error(ep.err, DEVERR_INDEX, 808);
    return;
  }
  const size_t crow = (size_t)b * ep.N + row;  // the token's cache row
  __nv_bfloat16* const outb = reinterpret_cast<__nv_bfloat16*>(ep.out);
  const int nv = r.n_tiles * r.nacc;          // 128-row tiles
  int vt[kRedJobs], f4[kRedJobs];
  bool ok[kRedJobs];
  float4 sum[kRedJobs];
  if constexpr (MODE == EPI_QKV || MODE == EPI_SWIGLU) {
    // two groups per item: QKV 4 rotary pairs (features f1.. and f1 + hd/2..)
    // of one head; SwiGLU 4 gate features and their 4 up features
    constexpr int IPB = kRedJobs / 2;  // items per batch
    const int hd = ep.head_dim, hh = hd / 2, per_head = hd / 8;
    const int n_items = nv * 16;
#pragma unroll 1
    for (int base = threadIdx.x; base < n_items; base += IPB * kRedThreads) {
      int it[IPB];
#pragma unroll
      for (int i = 0; i < IPB; ++i) {
        it[i] = base + i * kRedThreads;
        const int v_ = it[i] / 16, jt = it[i] % 16;
        int fa, fb;
        if constexpr (MODE == EPI_QKV) {
          const int hl = jt / per_head, jj = jt % per_head;
          fa = hl * hd + 4 * jj;
          fb = fa + hh;
        } else {
          fa = 4 * jt;
          fb = fa + 64;
        }
        const bool in = it[i] < n_items &&
                        (MODE == EPI_QKV ? v_ * 128 + fa < ep.n_out : v_ * 64 + 4 * jt < ep.n_out);
        vt[2 * i] = vt[2 * i + 1] = v_;
        f4[2 * i] = fa / 4;
        f4[2 * i + 1] = fb / 4;
        ok[2 * i] = ok[2 * i + 1] = in;
      }
      sk_sum_jobs(r, s_nseg, s_slot, t, vt, f4, ok, sum);
#pragma unroll
      for (int i = 0; i < IPB; ++i) {
        if (!ok[2 * i]) continue;
        const float4 x1 = sum[2 * i], x2 = sum[2 * i + 1];
        if constexpr (MODE == EPI_QKV) {
          const int n1 = vt[2 * i] * 128 + 4 * f4[2 * i];
          const int part = n1 / ep.d, col1 = n1 % ep.d, col2 = col1 + hh;
          const int jj = (col1 % hd) / 4;
          float4 a = x1, bb = x2;
          if (part < 2) {
            const float4 c = *reinterpret_cast<const float4*>(ep.rope_cos + (size_t)row * hh + 4 * jj);
            const float4 s_ = *reinterpret_cast<const float4*>(ep.rope_sin + (size_t)row * hh + 4 * jj);
            a = make_float4(x1.x * c.x - x2.x * s_.x, x1.y * c.y - x2.y * s_.y, x1.z * c.z - x2.z * s_.z,
                            x1.w * c.w - x2.w * s_.w);
            bb = make_float4(x2.x * c.x + x1.x * s_.x, x2.y * c.y + x1.y * s_.y, x2.z * c.z + x1.z * s_.z,
                             x2.w * c.w + x1.w * s_.w);
          }
          __nv_bfloat16* dst = part == 0 ? outb + (size_t)t * ep.d
                                         : reinterpret_cast<__nv_bfloat16*>(part == 1 ? ep.k_cache : ep.v_cache) +
                                               crow * ep.d;
          store4(dst + col1, a);
          store4(dst + col2, bb);
        } else {
          const int fo = vt[2 * i] * 64 + 4 * f4[2 * i];
          store4(outb + (size_t)t * ep.n_out + fo,
                 make_float4(sk_silu(x1.x) * x2.x, sk_silu(x1.y) * x2.y, sk_silu(x1.z) * x2.z, sk_silu(x1.w) * x2.w));
        }
      }
    }
  } else {
    // STORE, RESID (+ the FFN RMSNorm), RESID_SCATTER: 4 consecutive features per item
    const __nv_bfloat16* res = reinterpret_cast<const __nv_bfloat16*>(ep.resid);
    __nv_bfloat16* rc = reinterpret_cast<__nv_bfloat16*>(ep.row_copy);
    const int n_items = nv * 32;
    float ss = 0.f;
#pragma unroll 1
    for (int base = threadIdx.x; base < n_items; base += kRedJobs * kRedThreads) {
#pragma unroll
      for (int j = 0; j < kRedJobs; ++j) {
        const int it = base + j * kRedThreads;
        vt[j] = it / 32;
        f4[j] = it % 32;
        ok[j] = it < n_items && vt[j] * 128 + 4 * f4[j] < ep.n_out;
      }
      sk_sum_jobs(r, s_nseg, s_slot, t, vt, f4, ok, sum);
#pragma unroll
      for (int j = 0; j < kRedJobs; ++j) {
        if (!ok[j]) continue;
        const int n = vt[j] * 128 + 4 * f4[j];
        float4 v = sum[j];
        if constexpr (MODE == EPI_STORE) {
          store4(outb + (size_t)t * ep.n_out + n, v);
        } else if constexpr (MODE == EPI_RESID) {
          const float4 h = load4(res + crow * ep.d + n);
          v = make_float4(v.x + h.x, v.y + h.y, v.z + h.z, v.w + h.w);
          store4(outb + (size_t)t * ep.d + n, v);
          if (r.x2) {  // sum of squares of the stored (bf16-rounded) values
            const float qx = __bfloat162float(__float2bfloat16_rn(v.x)), qy = __bfloat162float(__float2bfloat16_rn(v.y));
            const float qz = __bfloat162float(__float2bfloat16_rn(v.z)), qw = __bfloat162float(__float2bfloat16_rn(v.w));
            ss += qx * qx + qy * qy + qz * qz + qw * qw;
          }
        } else {  // EPI_RESID_SCATTER
          const float4 h = load4(res + (size_t)t * ep.d + n);
          v = make_float4(v.x + h.x, v.y + h.y, v.z + h.z, v.w + h.w);
          store4(outb + crow * ep.d + n, v);
          if (rc) store4(rc + (size_t)t * ep.d + n, v);
          if (ep.score_zero && n == 0) ep.score_zero[crow] = 0.f;
        }
      }
    }
    if constexpr (MODE == EPI_RESID) {
      if (r.x2) {
        // x2 = RMSNorm(H1) * gamma over the whole row (block sum in a fixed order)
        ss = warp_sum(ss);
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kRedThreads / 32; ++w) tot += s_red[w];
        const float inv = 1.0f / sqrtf(tot / (float)ep.d + r.eps);
        const __nv_bfloat16* gam = reinterpret_cast<const __nv_bfloat16*>(r.gamma);
        __nv_bfloat16* x2 = reinterpret_cast<__nv_bfloat16*>(r.x2);
#pragma unroll 1
        for (int it = threadIdx.x; it < n_items; it += kRedThreads) {
          const int n = (it / 32) * 128 + 4 * (it % 32);  // items this thread stored above
          if (n >= ep.n_out) continue;
          const float4 h = load4(outb + (size_t)t * ep.d + n);
          const float4 gm = load4(gam + n);
          store4(x2 + (size_t)t * ep.d + n,
                 make_float4(h.x * inv * gm.x, h.y * inv * gm.y, h.z * inv * gm.z, h.w * inv * gm.w));
        }
      }
    }
  }
}

cudaError_t launch_tc_sk(int mode, const SkParams& p, int grid, const SkReduceParams& r, cudaStream_t stream) {
  cudaError_t e = configure_kernel((const void*)tc_sk_kernel, kSkSmem, false);
  if (e != cudaSuccess) return e;
  e = launch_k(tc_sk_kernel, dim3(grid), dim3(kSkThreads), kSkSmem, stream, p);
  if (e != cudaSuccess) return e;
  const dim3 rg(p.ep.M), rb(kRedThreads);
  switch (mode) {
    case EPI_STORE: return launch_k(sk_reduce_kernel<EPI_STORE>, rg, rb, 0, stream, r);
    case EPI_QKV: return launch_k(sk_reduce_kernel<EPI_QKV>, rg, rb, 0, stream, r);
    case EPI_RESID: return launch_k(sk_reduce_kernel<EPI_RESID>, rg, rb, 0, stream, r);
    case EPI_SWIGLU: return launch_k(sk_reduce_kernel<EPI_SWIGLU>, rg, rb, 0, stream, r);
    case EPI_RESID_SCATTER: return launch_k(sk_reduce_kernel<EPI_RESID_SCATTER>, rg, rb, 0, stream, r);
    default: return cudaErrorInvalidValue;
  }
}

int sk_stages(int nacc, int NT) {
  const int st = kSkRing / (nacc * kSkW + NT * 128);
  return st < kSkMaxStages ? st : kSkMaxStages;
}

void sk_partition_bounds(int n_tiles, int KB, int G, int* max_seg_per_cta, int* max_seg_per_tile) {
  const int U = n_tiles * KB;
  int mc = 0, mt = 0;
  for (int g = 0; g < G; ++g) {
    const int a = sk_start(g, G, U), b = sk_start(g + 1, G, U);
    if (b > a) mc = std::max(mc, (b - 1) / KB - a / KB + 1);
  }
  for (int tu = 0; tu < n_tiles; ++tu)
    mt = std::max(mt, sk_owner(tu * KB + KB - 1, G, U) - sk_owner(tu * KB, G, U) + 1);
  *max_seg_per_cta = mc;
  *max_seg_per_tile = mt;
}

int sk_reduce_max_seg() { return kRedMaxSeg; }
int sk_reduce_max_tiles() { return kRedMaxTiles; }

}  // namespace spa
