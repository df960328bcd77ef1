// Persistent FFN half of the cached layer step (bf16, sm_100a): the O-proj,
// the FFN RMSNorm, the gate/up GEMM with SwiGLU and the down GEMM with the
// H^c scatter in one launch of one CTA per SM.
//
// Separate launches pay, per GEMM, a start-up (~4 us until the first weight
// tile lands) and a tail (epilogue) during which HBM idles.  Here each CTA's
// producer streams the weights of its share of the three GEMMs back to back:
// the weights do not depend on the activations, so while the previous GEMM is
// being finished the ring already fills with the next GEMM's weights, and only
// the token boxes wait for their activations.
//
// Each GEMM ("phase") is split stream-K over the CTAs: tiles of nacc x 128
// weight rows (gate/up: 64 gate rows + the same 64 up rows per 128), units of
// one tile and 64 input columns, the tile-major unit list cut evenly over the
// grid.  Roles (12 warps):
//   warp 0        TMA producer over all three phases; a phase's token boxes
//                 wait for that phase's activations (a global row counter),
//                 its weight boxes do not.
//   warp 1        tcgen05.mma issuer (two TMEM accumulator buffers).
//   warps 4-7     epilogue: every segment's fp32 partial tile into its scratch
//                 slot ([NT][nacc x 128], token-major), then counted.
//   warps 2,3,8-11 reducers: once every segment of a phase is counted, the
//                 CTA's rows (t = g, g + G, ...) are summed over the segments
//                 in k-block order and finished: phase 0 H1 = H[b, I[t]] + .,
//                 and x2 = RMSNorm(H1) over the whole row; phase 1 A = silu(g) u;
//                 phase 2 H^c[b, I[t]] = H1 + . (+ compact copy, score zero).
//                 Then the phase's row counter is advanced.
// Every wait on another CTA is bounded (1 s) and records a time-out; the grid
// never exceeds the SMs and a CTA fills an SM, so all CTAs are resident once
// the previous kernel's CTAs have left.  The last CTA to finish zeroes the
// counters for the next launch.  Results are deterministic: the partition and
// the summation order depend only on the shapes and the grid.
#include <algorithm>
#include <cstdio>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

constexpr int kFfThreads = 384;
constexpr int kFfRing = 192 * 1024;
constexpr int kFfMaxStages = 16;
constexpr int kFfW = 128 * 128;     // one 128-row x 64-column weight box
constexpr int kFfMaxSeg = 6;        // segments per tile (the host keeps the grid within it)
constexpr int kFfMaxTiles = 192;    // unit tiles per phase
constexpr int kFfTableBytes = 3 * kFfMaxTiles * (1 + kFfMaxSeg) * 2;
constexpr int kFfSmem = kFfRing + kFfTableBytes + 1024;
constexpr int kFfRed = 192;         // reducer threads
constexpr int kFfJobs = 4;          // feature groups summed per reducer thread at once

__device__ __forceinline__ float ff_silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__host__ __device__ __forceinline__ int ff_start(int g, int G, int U) { return (int)(((long long)g * U) / G); }
__host__ __device__ __forceinline__ int ff_owner(int u, int G, int U) {
  int g = (int)(((long long)u * G) / U);
  while (g + 1 < G && ff_start(g + 1, G, U) <= u) ++g;
  while (g > 0 && ff_start(g, G, U) > u) --g;
  return g;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Wait until *ctr >= target, bounded; true when reached.
__device__ __forceinline__ bool ff_wait_count(const int* ctr, int target, volatile int* abort, int* err, int site) {
  if (ld_acquire(ctr) >= target) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (ld_acquire(ctr) >= target) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort = 1;
      report_error(err, DEVERR_TIMEOUT, site);
      return false;
    }
  }
}

// The weight boxes of unit (phase ph, unit tile tu, sub-tile a, k-block kb).
__device__ __forceinline__ void ff_load_w(const FfnParams& p, int ph, int tu, int a, int kb, uint8_t* sw,
                                          uint64_t* bar) {
  const int kx = kb * 64;
  const int vt = tu * p.nacc[ph] + a;
  if (ph == 0) {
    tma_load_2d(sw, &p.tmWo, bar, kx, vt * 128);
  } else if (ph == 1) {
    tma_load_2d(sw, &p.tmWg, bar, kx, vt * 64);
    tma_load_2d(sw + kFfW / 2, &p.tmWu, bar, kx, vt * 64);
  } else {
    tma_load_2d(sw, &p.tmWd, bar, kx, vt * 128);
  }
}

// Unit `it` of this CTA's concatenated phase ranges -> (phase, unit).
__device__ __forceinline__ void ff_unit(const int* lo, const int* hi, int it, int& ph, int& u) {
  ph = 0;
  while (ph < 2 && it >= hi[ph] - lo[ph]) {
    it -= hi[ph] - lo[ph];
    ++ph;
  }
  u = lo[ph] + it;
}

__global__ void __launch_bounds__(kFfThreads, 1) ffn_persistent_kernel(const __grid_constant__ FfnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint16_t* tab = reinterpret_cast<uint16_t*>(smem + kFfRing);  // [3][tiles][1 + kFfMaxSeg]
  __shared__ __align__(8) uint64_t full_bar[kFfMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kFfMaxStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, prod_issued, mma_consumed, s_ok, r_ok;
  __shared__ float s_red[kFfRed / 32];

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int NT = p.NT, M = p.M;
  int lo[3], hi[3];
#pragma unroll
  for (int ph = 0; ph < 3; ++ph) {
    lo[ph] = ff_start(g, G, p.units[ph]);
    hi[ph] = ff_start(g + 1, G, p.units[ph]);
  }
  const int n_its = (hi[0] - lo[0]) + (hi[1] - lo[1]) + (hi[2] - lo[2]);
  const int W_SLOT = p.max_nacc * kFfW;          // room for the widest phase's weight boxes
  const int STAGE_BYTES = W_SLOT + NT * 128;     // multiple of 1024
  int STAGES = kFfRing / STAGE_BYTES;
  if (STAGES > kFfMaxStages) STAGES = kFfMaxStages;
  int* err = p.err;
  int* seg_done = p.sync;       // [3]
  int* rows_done = p.sync + 3;  // [3]
  int* ctas_done = p.sync + 6;

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
    s_ok = r_ok = 1;
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
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmX[0]);
      tma_prefetch_desc(&p.tmX[1]);
      tma_prefetch_desc(&p.tmX[2]);
      // weights run ahead of the token boxes: w_it stages have their weight
      // boxes requested, x_it their token boxes
      int w_it = 0, x_it = 0;
      bool ready[3] = {false, false, false};
      bool waited = false;
      const unsigned long long t0 = globaltimer();
      volatile int* abort_v = &abort_flag;
      while (x_it < n_its && !*abort_v) {
        bool progress = false;
        // weights of the next stage, once its slot is free (never more than
        // STAGES ahead of the token boxes)
        if (w_it < n_its && w_it < x_it + STAGES) {
          const int s = w_it % STAGES;
          if (w_it < STAGES || mbar_try_wait(smem_u32(&empty_bar[s]), ((w_it / STAGES) - 1) & 1)) {
            int ph, u;
            ff_unit(lo, hi, w_it, ph, u);
            const int KB = p.KB[ph], tu = u / KB, kb = u % KB;
            uint8_t* sw = smem + s * STAGE_BYTES;
            mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(p.nacc[ph] * kFfW + NT * 128));
            for (int a = 0; a < p.nacc[ph]; ++a) ff_load_w(p, ph, tu, a, kb, sw + a * kFfW, &full_bar[s]);
            ++w_it;
            progress = true;
          }
        }
        // token box of the oldest stage, once its phase's activations are ready
        if (x_it < w_it) {
          int ph, u;
          ff_unit(lo, hi, x_it, ph, u);
          if (!ready[ph]) {
            if (ph == 0) {
              if (!waited) griddep_wait();  // the attention output and H come from earlier kernels
              waited = true;
              ready[0] = true;
            } else if (ld_acquire(rows_done + ph - 1) >= M) {
              ready[ph] = true;
            }
            if (ready[ph]) fence_proxy_async_global();  // written by other CTAs' reducers
          }
          if (ready[ph]) {
            const int s = x_it % STAGES;
            tma_load_2d(smem + s * STAGE_BYTES + W_SLOT, &p.tmX[ph], &full_bar[s], (u % p.KB[ph]) * 64, 0);
            ++x_it;
            progress = true;
          }
        }
        if (!progress && globaltimer() - t0 > 4 * kWaitLimitNs) {
          abort_flag = 1;
          report_error(err, DEVERR_TIMEOUT, 901);
        }
      }
      prod_issued = x_it;  // stages with both boxes requested
      if (!waited) griddep_wait();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int ph = 0; ok && ph < 3; ++ph) {
        const int KB = p.KB[ph], nacc = p.nacc[ph];
        const uint32_t idesc = idesc_bf16_f32(128, NT);
        for (int u = lo[ph]; ok && u < hi[ph]; ++j) {
          const int kb0 = u % KB;
          const int kb1 = kb0 + (hi[ph] - u < KB - kb0 ? hi[ph] - u : KB - kb0);
          const int a = j & 1;
          if (j >= 2 && !mbar_wait(&acc_empty[a], ((j >> 1) - 1) & 1, &abort_flag, err, 902)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + (uint32_t)(a * p.acc_cols);
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, &abort_flag, err, 903)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
            const uint64_t dx = smem_desc_sw128(sa + W_SLOT);
            for (int sub = 0; sub < nacc; ++sub) {
              const uint64_t dw = smem_desc_sw128(sa + sub * kFfW);
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
      }
      mma_consumed = it;
      umma_commit(&mma_done);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------- epilogue
    griddep_wait();  // the scratch was read by the previous launch's reducers
    const int q = warp - 4, f = q * 32 + lane, et = threadIdx.x - 128;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int mt = M < NT ? M : NT;
    int j = 0;
    bool go = true;
    for (int ph = 0; go && ph < 3; ++ph) {
      const int KB = p.KB[ph], nacc = p.nacc[ph], FEAT = nacc * 128;
      int jp = 0;  // segment index within the phase
      for (int u = lo[ph]; u < hi[ph]; ++j, ++jp) {
        const int kb0 = u % KB;
        u += (hi[ph] - u < KB - kb0 ? hi[ph] - u : KB - kb0);
        const int a = j & 1;
        const bool got = mbar_wait(&acc_full[a], (j >> 1) & 1, &abort_flag, err, 904);
        __syncwarp();
        const bool warp_ok = __all_sync(0xffffffffu, got);
        if (lane == 0 && !warp_ok) atomicAnd(&s_ok, 0);
        named_bar_sync(2, 128);
        if (!s_ok) { go = false; break; }
        tc_fence_after();
        float* dst = p.part[ph] + ((size_t)g * p.maxseg[ph] + jp) * (size_t)NT * FEAT + f;
        for (int sub = 0; sub < nacc; ++sub) {
          const uint32_t acc_tmem = lane_base + (uint32_t)(a * p.acc_cols + sub * NT);
          for (int c0 = 0; c0 < mt; c0 += 32) {
            float v[32];
            tmem_ld32(acc_tmem + (uint32_t)c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i < mt) __stcg(dst + (size_t)(c0 + i) * FEAT + sub * 128, v[i]);
          }
        }
        tc_fence_before();
        __threadfence();
        named_bar_sync(2, 128);
        if (et == 0) {
          mbar_arrive_cta(&acc_empty[a]);
          atomicAdd(seg_done + ph, 1);  // this segment's partial is published
        }
      }
    }
  } else {
    // ------------------------------------------------------------- reducers
    const int rt = (warp < 4) ? (warp - 2) * 32 + lane : 64 + (warp - 8) * 32 + lane;  // 0..191
    // segment tables: tab[ph][tu] = {nseg, slot_0 .. slot_{nseg-1}}
    for (int ph = 0; ph < 3; ++ph)
      for (int tu = rt; tu < p.n_tiles[ph]; tu += kFfRed) {
        const int KB = p.KB[ph], U = p.units[ph];
        const int gf = ff_owner(tu * KB, G, U), gl = ff_owner(tu * KB + KB - 1, G, U);
        uint16_t* e = tab + ((size_t)ph * kFfMaxTiles + tu) * (1 + kFfMaxSeg);
        e[0] = (uint16_t)(gl - gf + 1);
        for (int s = 0; s <= gl - gf && s < kFfMaxSeg; ++s)
          e[1 + s] = (uint16_t)((gf + s) * p.maxseg[ph] + (tu - ff_start(gf + s, G, U) / KB));
      }
    named_bar_sync(3, kFfRed);
    griddep_wait();
    const __nv_bfloat16* Hin = p.H;
    for (int ph = 0; ph < 3; ++ph) {
      // every segment of the phase is published
      if (rt == 0 && !ff_wait_count(seg_done + ph, p.seg_total[ph], &abort_flag, err, 905 + ph)) r_ok = 0;
      named_bar_sync(3, kFfRed);
      if (!r_ok) break;
      __threadfence();
      const int nacc = p.nacc[ph], FEAT = nacc * 128;
      const size_t slot_floats = (size_t)NT * FEAT;
      const float* part = p.part[ph];
      const uint16_t* tb = tab + (size_t)ph * kFfMaxTiles * (1 + kFfMaxSeg);
      const int nv = p.n_tiles[ph] * nacc;  // 128-row tiles
      int my_rows = 0;
      for (int t = g; t < M; t += G) {
        ++my_rows;
        const int b = t / p.tps;
        const int row = p.idx ? p.idx[t] : (t % p.tps);
        const bool row_ok = row >= 0 && row < p.N;
        if (!row_ok && rt == 0) report_error(err, DEVERR_INDEX, 909);
        const size_t crow = (size_t)b * p.N + (row_ok ? row : 0);
        // jobs: (128-row tile vt, feature group f4 of 4 features); phase 1
        // pairs each gate group with its up group (f4 + 16)
        const int per_tile = ph == 1 ? 16 : 32;
        const int n_items = nv * per_tile;
        float ss = 0.f;
#pragma unroll 1
        for (int base = rt; base < n_items; base += (ph == 1 ? kFfJobs / 2 : kFfJobs) * kFfRed) {
          int vt[kFfJobs], f4[kFfJobs];
          bool ok[kFfJobs];
#pragma unroll
          for (int jb = 0; jb < kFfJobs; ++jb) {
            const int it = ph == 1 ? base + (jb / 2) * kFfRed : base + jb * kFfRed;
            vt[jb] = it / per_tile;
            f4[jb] = (it % per_tile) + (ph == 1 && (jb & 1) ? 16 : 0);
            ok[jb] = row_ok && it < n_items;
          }
          float4 v[kFfJobs][kFfMaxSeg];
          int n[kFfJobs];
#pragma unroll
          for (int jb = 0; jb < kFfJobs; ++jb) {
            n[jb] = 0;
            if (!ok[jb]) continue;
            const int tu = vt[jb] / nacc, sub = vt[jb] % nacc;
            const uint16_t* e = tb + (size_t)tu * (1 + kFfMaxSeg);
            n[jb] = e[0];
            const size_t off = (size_t)t * FEAT + sub * 128 + f4[jb] * 4;
#pragma unroll
            for (int s = 0; s < kFfMaxSeg; ++s)
              if (s < n[jb]) v[jb][s] = __ldcg(reinterpret_cast<const float4*>(part + (size_t)e[1 + s] * slot_floats + off));
          }
          float4 sum[kFfJobs];
#pragma unroll
          for (int jb = 0; jb < kFfJobs; ++jb) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n[jb] > 0) acc = v[jb][0];
#pragma unroll
            for (int s = 1; s < kFfMaxSeg; ++s)
              if (s < n[jb]) {
                acc.x += v[jb][s].x; acc.y += v[jb][s].y; acc.z += v[jb][s].z; acc.w += v[jb][s].w;
              }
            sum[jb] = acc;
          }
          if (ph == 0) {
#pragma unroll
            for (int jb = 0; jb < kFfJobs; ++jb) {
              if (!ok[jb]) continue;
              const int n_ = vt[jb] * 128 + 4 * f4[jb];
              const float4 h = load4(Hin + crow * p.d + n_);
              const float4 r = make_float4(sum[jb].x + h.x, sum[jb].y + h.y, sum[jb].z + h.z, sum[jb].w + h.w);
              store4(p.H1 + (size_t)t * p.d + n_, r);
              const float qx = __bfloat162float(__float2bfloat16_rn(r.x)), qy = __bfloat162float(__float2bfloat16_rn(r.y));
              const float qz = __bfloat162float(__float2bfloat16_rn(r.z)), qw = __bfloat162float(__float2bfloat16_rn(r.w));
              ss += qx * qx + qy * qy + qz * qz + qw * qw;
            }
          } else if (ph == 1) {
#pragma unroll
            for (int jb = 0; jb < kFfJobs; jb += 2) {
              if (!ok[jb]) continue;
              const float4 gt = sum[jb], up = sum[jb + 1];
              const int fo = vt[jb] * 64 + 4 * f4[jb];
              store4(p.A + (size_t)t * p.F + fo,
                     make_float4(ff_silu(gt.x) * up.x, ff_silu(gt.y) * up.y, ff_silu(gt.z) * up.z, ff_silu(gt.w) * up.w));
            }
          } else {
#pragma unroll
            for (int jb = 0; jb < kFfJobs; ++jb) {
              if (!ok[jb]) continue;
              const int n_ = vt[jb] * 128 + 4 * f4[jb];
              const float4 h = load4(p.H1 + (size_t)t * p.d + n_);
              const float4 r = make_float4(sum[jb].x + h.x, sum[jb].y + h.y, sum[jb].z + h.z, sum[jb].w + h.w);
              store4(p.Hc + crow * p.d + n_, r);
              if (p.row_copy) store4(p.row_copy + (size_t)t * p.d + n_, r);
              if (p.score_zero && n_ == 0) p.score_zero[crow] = 0.f;
            }
          }
        }
        if (ph == 0) {
          // x2 = RMSNorm(H1) * gamma over the whole row (block sum in a fixed order)
          ss = warp_sum(ss);
          if (lane == 0) s_red[rt >> 5] = ss;
          named_bar_sync(3, kFfRed);
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < kFfRed / 32; ++w) tot += s_red[w];
          named_bar_sync(3, kFfRed);  // s_red is reused by the next row
          const float inv = 1.0f / sqrtf(tot / (float)p.d + p.eps);
          if (row_ok) {
#pragma unroll 1
            for (int it = rt; it < n_items; it += kFfRed) {
              const int n_ = (it / 32) * 128 + 4 * (it % 32);
              const float4 h = load4(p.H1 + (size_t)t * p.d + n_);  // this thread's own stores
              const float4 gm = load4(p.gamma + n_);
              store4(p.X2 + (size_t)t * p.d + n_,
                     make_float4(h.x * inv * gm.x, h.y * inv * gm.y, h.z * inv * gm.z, h.w * inv * gm.w));
            }
          }
        }
      }
      // publish this CTA's rows of the phase (TMA reads them in other CTAs)
      fence_proxy_async_global();
      __threadfence();
      named_bar_sync(3, kFfRed);
      if (rt == 0 && my_rows > 0) atomicAdd(rows_done + ph, my_rows);
    }
  }
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_drain_bounded(&mma_done, 0, err, 910);
    if (abort_flag != 0)
      for (int it = mma_consumed; it < prod_issued; ++it)
        mbar_drain_bounded(&full_bar[it % STAGES], (it / STAGES) & 1, err, 911);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
  if (threadIdx.x == 0) {
    // the last CTA to leave zeroes the counters for the next launch
    __threadfence();
    if (atomicAdd(ctas_done, 1) == G - 1) {
      for (int i = 0; i < 6; ++i) p.sync[i] = 0;
      __threadfence();
      *ctas_done = 0;
    }
  }
}

cudaError_t launch_ffn_persistent(const FfnParams& p, int grid, cudaStream_t stream) {
  cudaError_t e = configure_kernel((const void*)ffn_persistent_kernel, kFfSmem, false);
  if (e != cudaSuccess) return e;
  return launch_k(ffn_persistent_kernel, dim3(grid), dim3(kFfThreads), kFfSmem, stream, p);
}

int ffn_max_seg() { return kFfMaxSeg; }
int ffn_max_tiles() { return kFfMaxTiles; }

}  // namespace spa
