// Sparse-query attention of the SPA-Cache layer step: the k refreshed
// queries of each sequence attend to all N cached keys and values (the
// bidirectional cache K^c, V^c, already holding this step's fresh rows).
//
// attn_tc_kernel (bf16, head_dim 128): tcgen05 tensor cores with TMEM
// accumulators, described below.
//
// attn_simt_kernel: one warp per (query, head), online softmax over chunks of
// 32 keys (one key per lane), fp32 throughout.  Used for the fp32
// configurations and for head sizes the tensor-core kernel does not cover.
#include <cstdlib>
#include <cstring>

#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

template <typename T>
__global__ void __launch_bounds__(128) attn_simt_kernel(const T* Q, const T* Kc, const T* Vc, T* O,
                                                        int k, int N, int n_heads, int hd,
                                                        float scale) {
  __shared__ float qs[4][128];
  griddep_launch_dependents();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 4 + warp;  // query within the sequence
  const int h = blockIdx.y, b = blockIdx.z;
  const int d = n_heads * hd;
  if (i >= k) return;
  const size_t qrow = ((size_t)b * k + i) * d + (size_t)h * hd;
  for (int c = lane; c < hd; c += 32) qs[warp][c] = to_f(Q[qrow + c]);
  __syncwarp();
  const T* Kb = Kc + (size_t)b * N * d + (size_t)h * hd;
  const T* Vb = Vc + (size_t)b * N * d + (size_t)h * hd;
  float m = -INFINITY, l = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 < N; j0 += 32) {
    const int j = j0 + lane;
    float dot = -INFINITY;
    if (j < N) {
      const T* kr = Kb + (size_t)j * d;
      float s = 0.f;
      for (int c = 0; c < hd; ++c) s = fmaf(qs[warp][c], to_f(kr[c]), s);
      dot = s * scale;
    }
    const float m_new = fmaxf(m, warp_max(dot));
    const float p = (j < N) ? expf(dot - m_new) : 0.f;
    const float corr = expf(m - m_new);
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] *= corr;
    const int nj = min(32, N - j0);
    for (int jj = 0; jj < nj; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T* vr = Vb + (size_t)(j0 + jj) * d;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = lane + 32 * q;
        if (c < hd) acc[q] = fmaf(pj, to_f(vr[c]), acc[q]);
      }
    }
    m = m_new;
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = lane + 32 * q;
    if (c < hd) O[qrow + c] = from_f<T>(acc[q] * inv);
  }
}

// ---------------------------------------------------------------------------
// tensor-core attention (tcgen05, TMEM), bf16, head_dim 128
//
// One CTA = one head of one sequence, one tile of 128 selected queries, one
// contiguous range of the N cached keys (split-KV).  Q (128 x 128) is loaded
// once; K and V tiles of 128 keys stream through a 2-stage TMA ring.
//   warp 0      TMA producer
//   warp 1      one thread issues tcgen05.mma: S_j = Q K_j^T into one of two
//               TMEM score buffers, then O += P_{j-1} V_{j-1} (P from shared
//               memory, V as an MN-major operand), so the tensor core works on
//               the next scores while the softmax warps work on these
//   warps 4-7   softmax: thread i owns query row i (TMEM lane i).  It reads
//               its 128 scores from TMEM twice, 32 columns at a time (the
//               row max, then the probabilities), keeps the running max m
//               and sum l in registers, writes P = 2^(s*log2e/sqrt(d_h) - m) as bf16 into
//               the 128-byte-swizzled K-major layout the MMA reads, and
//               rescales O in TMEM only when the max grows by more than 2^8
//               (the result is exact for any reference max: the final
//               division by l uses the same one).
// With several key splits the S CTAs of a query tile form a thread-block
// cluster: each leaves its unnormalised O rows, m and l in its own shared
// memory, and after a cluster barrier CTA q combines rows [q*128/S,
// (q+1)*128/S) of all S splits through distributed shared memory, in split
// order 0..S-1, so the result does not depend on timing.  Where clusters are
// not allowed (the allocation-free entry point) each CTA writes (O, m, l) to
// scratch instead and the last CTA of the query tile to finish (an atomic
// counter) combines them in the same order and resets the counter.
// ---------------------------------------------------------------------------
constexpr int kAT = 128;                 // queries per CTA and keys per tile
constexpr int kAQBytes = 2 * 16384;      // Q: two 64-column boxes of 128 rows
constexpr int kAKVBytes = 4 * 16384;     // K and V tiles, two boxes each
constexpr int kAPBytes = 2 * 16384;      // P: 128 x 128 bf16
constexpr int kAStages = 2;
constexpr int kASmem = kAQBytes + kAStages * kAKVBytes + kAPBytes + 1024;
constexpr int kAThreads = 256;
constexpr float kARescale = 8.0f;        // rescale O when the max grows by > 2^8

struct alignas(64) AttnTcParams {
  CUtensorMap tmQ;  // compact Q [B*k, d], box 64 x 128
  CUtensorMap tmK;  // K^c [B*N, d], box 64 x 128
  CUtensorMap tmV;  // V^c [B*N, d], box 64 x 128
  __nv_bfloat16* O; // [B*k, d]
  float* part_o;    // split partials: slot -> [128][128] fp32
  float* part_ml;   // slot -> m[128], l[128]
  int* sync;        // per query tile: splits finished (zero between launches)
  int* err;
  int B, k, N, n_heads, q_tiles, splits;
  int cluster;       // splits > 1: 1 = combine in distributed shared memory
  float scale_log2;  // log2(e) / sqrt(head_dim)
};

// Shared-memory descriptor of an MN-major operand tile with 128-byte
// swizzling: 64 contiguous MN elements (128 B) per K row, 8-row atoms of
// 1024 B (stride byte offset), the next 64 MN elements `lbo` bytes further
// (leading byte offset).
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)64 << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
// Bounded wait that ignores the abort flag (copies/MMAs in flight after an abort).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, int* err, int site) {
  const uint32_t a = smem_u32(bar);
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      report_error(err, DEVERR_TIMEOUT, site);
      return;
    }
  }
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Rows [r0, r0 + 128/S) of the cluster's S split partials (unnormalised O in
// each CTA's shared memory, 16-byte chunk c of row r at chunk c ^ (r % 32)),
// weighted by w[row][q] and summed in split order, to bf16 rows of O (query
// q0 + row, skipped past k).  128/S rows x 32 chunks = 4096/S tasks over the
// block's 256 threads: 16/S tasks and 16 remote loads per thread, all issued
// before any is used.
template <int S>
__device__ __forceinline__ void attn_cluster_combine(const float* sO, const float (*w)[8], int r0, int q0,
                                                     int k, int d, __nv_bfloat16* Ob) {
  constexpr int T = 16 / S;
  float4 v[T][S];
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int task = threadIdx.x + kAThreads * t;
    const int rl = task >> 5, ch = task & 31, row = r0 + rl;
    const uint32_t la = smem_u32(sO + row * 128 + ((ch ^ (row & 31)) << 2));
#pragma unroll
    for (int q = 0; q < S; ++q)
      v[t][q] = q0 + row < k ? ld_dsmem_f4(mapa_shared(la, (uint32_t)q)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int task = threadIdx.x + kAThreads * t;
    const int rl = task >> 5, ch = task & 31, row = r0 + rl;
    if (q0 + row >= k) continue;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < S; ++q) {
      const float wq = w[rl][q];
      acc.x += wq * v[t][q].x; acc.y += wq * v[t][q].y; acc.z += wq * v[t][q].z; acc.w += wq * v[t][q].w;
    }
    store4(Ob + (size_t)(q0 + row) * d + ch * 4, acc);
  }
}

__global__ void __launch_bounds__(kAThreads, 1) attn_tc_kernel(const __grid_constant__ AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kAQBytes;
  uint8_t* sP = sKV + kAStages * kAKVBytes;
  __shared__ __align__(8) uint64_t q_full, kv_full[kAStages], kv_empty[kAStages];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full, pv_done, o_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, last_flag;
  __shared__ int kv_issued, kv_consumed, tile_ok;
  __shared__ float s_m[kAT], s_l[kAT];  // this split's row max and sum (cluster combine)
  __shared__ float s_w[kAT / 2][8];     // combine weights of this CTA's rows, per split

  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.splits;
  const int qt = blockIdx.x / S, sp = blockIdx.x % S, h = blockIdx.y, b = blockIdx.z;
  const int n_kt = (p.N + kAT - 1) / kAT;
  const int kt0 = (sp * n_kt) / S, kt1 = ((sp + 1) * n_kt) / S;
  const int nkt = kt1 - kt0;
  int* err = p.err;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 128);
    }
    mbar_init(&p_full, 128);
    mbar_init(&pv_done, 1);
    mbar_init(&o_done, 1);
    abort_flag = 0;
    last_flag = 0;
    kv_issued = kv_consumed = 0;
    tile_ok = 1;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;  // S buffers at columns 0 and 128, O at 256
  griddep_wait();  // Q, K^c and V^c come from the previous kernel

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
    const int qrow = b * p.k + qt * kAT, col = h * kAT;
    mbar_arrive_expect_tx(&q_full, kAQBytes);
    tma_load_2d(sQ, &p.tmQ, &q_full, col, qrow);
    tma_load_2d(sQ + 16384, &p.tmQ, &q_full, col + 64, qrow);
    for (int j = 0; j < nkt; ++j) {
      const int s = j % kAStages;
      if (j >= kAStages && !mbar_wait(&kv_empty[s], ((j / kAStages) - 1) & 1, &abort_flag, err, 601)) break;
      uint8_t* kv = sKV + s * kAKVBytes;
      const int krow = b * p.N + (kt0 + j) * kAT;
      mbar_arrive_expect_tx(&kv_full[s], kAKVBytes);
      tma_load_2d(kv, &p.tmK, &kv_full[s], col, krow);
      tma_load_2d(kv + 16384, &p.tmK, &kv_full[s], col + 64, krow);
      tma_load_2d(kv + 32768, &p.tmV, &kv_full[s], col, krow);
      tma_load_2d(kv + 49152, &p.tmV, &kv_full[s], col + 64, krow);
      kv_issued = j + 1;
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128);                 // both K-major
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128) | (1u << 16);    // B (V) MN-major
    const uint64_t dq = smem_desc_sw128(smem_u32(sQ));
    const uint64_t dp = smem_desc_sw128(smem_u32(sP));
    bool ok = mbar_wait(&q_full, 0, &abort_flag, err, 602);
    for (int j = 0; ok && j <= nkt; ++j) {
      if (j < nkt) {
        // S_j = Q K_j^T into score buffer j % 2
        const int s = j % kAStages, sb = j & 1;
        if (!mbar_wait(&kv_full[s], (j / kAStages) & 1, &abort_flag, err, 603)) break;
        kv_consumed = j + 1;
        if (j >= 2 && !mbar_wait(&s_empty[sb], ((j / 2) - 1) & 1, &abort_flag, err, 604)) break;
        tc_fence_after();
        const uint64_t dk = smem_desc_sw128(smem_u32(sKV + s * kAKVBytes));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
          umma_bf16(tmem + (uint32_t)(sb * 128), dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[sb]);
      }
      if (j >= 1) {
        // O += P_{j-1} V_{j-1}
        const int jj = j - 1, s = jj % kAStages;
        if (!mbar_wait(&p_full, jj & 1, &abort_flag, err, 605)) break;
        tc_fence_after();
        const uint64_t dv = smem_desc_sw128_mn(smem_u32(sKV + s * kAKVBytes + 32768), 16384);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t offp = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
          umma_bf16(tmem + 256u, dp + offp, dv + (uint64_t)(kk * 128), idesc_pv,
                    (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done);
        umma_commit(&kv_empty[s]);
      }
    }
    umma_commit(&o_done);
  } else if (warp >= 4) {
    const int q4 = warp - 4, row = q4 * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      const int sb = j & 1;
      // every lane waits, then the warp reconverges before the warp-wide
      // (.sync.aligned) TMEM instructions
      const bool got = mbar_wait(&s_full[sb], (j / 2) & 1, &abort_flag, err, 606);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      // two passes over the scores in TMEM, 32 columns at a time (compact
      // code and 32 registers instead of a 128-wide unrolled row): the row
      // max, then the probabilities
      const int key0 = (kt0 + j) * kAT;
      const uint32_t s_base = lane_base + (uint32_t)(sb * 128);
      float tmax = -INFINITY;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float x[32];
        tmem_ld32(s_base + (uint32_t)c0, x);
#pragma unroll
        for (int c = 0; c < 32; ++c)
          tmax = fmaxf(tmax, (key0 + c0 + c < p.N) ? x[c] * p.scale_log2 : -INFINITY);
      }
      // O and P may be rewritten only once the previous PV product is done
      const bool pv_ok = j == 0 || mbar_wait(&pv_done, (j - 1) & 1, &abort_flag, err, 607);
      __syncwarp();
      if (!__all_sync(0xffffffffu, pv_ok)) { ok = false; break; }
      if (j == 0) {
        m_used = tmax;
      } else if (__any_sync(0xffffffffu, tmax > m_used + kARescale)) {
        // some row's max grew by more than 2^8: the whole warp rescales (the
        // TMEM instructions are warp-wide), each row to its own new max
        const float m_new = fmaxf(m_used, tmax);
        const float f = exp2f(m_used - m_new);
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          float o[32];
          tmem_ld32(lane_base + 256u + (uint32_t)c, o);
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] *= f;
          tmem_st32(lane_base + 256u + (uint32_t)c, o);
        }
        tmem_st_wait();
        l *= f;
        m_used = m_new;
      }
      float sum = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float x[32];
        tmem_ld32(s_base + (uint32_t)c0, x);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = (key0 + c0 + c < p.N) ? x[c] * p.scale_log2 : -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = exp2f(x[c + 2 * q] - m_used), bb = exp2f(x[c + 2 * q + 1] - m_used);
            sum += a + bb;
            __nv_bfloat162 v2 = __floats2bfloat162_rn(a, bb);
            w[q] = *reinterpret_cast<uint32_t*>(&v2);
          }
          // 16-byte chunk of row `row`, 128-byte swizzle, two 64-key halves
          const int chunk = (c0 + c) >> 3, half = chunk >> 3, cc = chunk & 7;
          uint8_t* dst = sP + half * 16384 + row * 128 + ((cc ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // the score buffer is free once both passes have read it
      tc_fence_before();
      mbar_arrive1(&s_empty[sb]);
      l += sum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive1(&p_full);
    }
    // final O row
    const bool fin = ok && mbar_wait(&o_done, 0, &abort_flag, err, 608);
    __syncwarp();
    const bool warp_ok = __all_sync(0xffffffffu, fin);
    // the four softmax warps agree on whether the tile is usable, so the
    // named barriers below are reached by all 128 threads or by none
    if (lane == 0) atomicAnd(&tile_ok, warp_ok ? 1 : 0);
    named_bar(1, 128);
    if (tile_ok) {
      tc_fence_after();
      const int d = p.n_heads * kAT;
      const int qi = qt * kAT + row;  // query within the sequence
      if (S == 1) {
        const float inv = l > 0.f ? 1.0f / l : 0.f;
        __nv_bfloat16* dst = p.O + ((size_t)b * p.k + qi) * d + (size_t)h * kAT;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float o[32];
          tmem_ld32(lane_base + 256u + (uint32_t)c0, o);
          if (qi < p.k) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint32_t w[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 v2 = __floats2bfloat162_rn(o[c + 2 * q] * inv, o[c + 2 * q + 1] * inv);
                w[q] = *reinterpret_cast<uint32_t*>(&v2);
              }
              *reinterpret_cast<uint4*>(dst + c0 + c) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else if (p.cluster) {
        // unnormalised O row into the (now idle) K/V ring, 16-byte chunk c
        // of row r at chunk position c ^ (r % 32)
        float* sO = reinterpret_cast<float*>(sKV);
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float o[32];
          tmem_ld32(lane_base + 256u + (uint32_t)c0, o);
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const int ch = (c0 + c) >> 2;
            *reinterpret_cast<float4*>(sO + row * 128 + ((ch ^ (row & 31)) << 2)) =
                make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
          }
        }
        s_m[row] = m_used;
        s_l[row] = l;
      } else {
        const size_t grp = ((size_t)b * p.n_heads + h) * p.q_tiles + qt;
        const size_t slot = grp * S + sp;
        float* po = p.part_o + slot * (kAT * kAT) + (size_t)row * kAT;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float o[32];
          tmem_ld32(lane_base + 256u + (uint32_t)c0, o);
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(po + c0 + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        }
        p.part_ml[slot * 256 + row] = m_used;
        p.part_ml[slot * 256 + 128 + row] = l;
        __threadfence();
        named_bar(1, 128);
        if (row == 0) last_flag = (atomicAdd(p.sync + grp, 1) == S - 1) ? 1 : 0;
        named_bar(1, 128);
        if (last_flag) {
          __threadfence();
          // combine the S splits of this row in split order 0..S-1
          float mm = -INFINITY;
          for (int q = 0; q < S; ++q) mm = fmaxf(mm, __ldcg(p.part_ml + (grp * S + q) * 256 + row));
          float wsum = 0.f;
          for (int q = 0; q < S; ++q) {
            const size_t sl = grp * S + q;
            wsum += __ldcg(p.part_ml + sl * 256 + 128 + row) * exp2f(__ldcg(p.part_ml + sl * 256 + row) - mm);
          }
          const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
          // 32 columns at a time, splits in order (8 loads in flight per split)
          __nv_bfloat16* dst = p.O + ((size_t)b * p.k + qi) * d + (size_t)h * kAT;
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            float acc[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = 0.f;
#pragma unroll 1
            for (int q = 0; q < S; ++q) {
              const size_t sl = grp * S + q;
              const float pw = exp2f(__ldcg(p.part_ml + sl * 256 + row) - mm);
              const float4* src =
                  reinterpret_cast<const float4*>(p.part_o + sl * (kAT * kAT) + (size_t)row * kAT + c0);
              float4 v[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) v[c] = __ldcg(src + c);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                acc[4 * c] += pw * v[c].x; acc[4 * c + 1] += pw * v[c].y;
                acc[4 * c + 2] += pw * v[c].z; acc[4 * c + 3] += pw * v[c].w;
              }
            }
            if (qi < p.k) {
#pragma unroll
              for (int c = 0; c < 32; c += 8) {
                uint32_t w4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  __nv_bfloat162 v2 = __floats2bfloat162_rn(acc[c + 2 * q] * inv, acc[c + 2 * q + 1] * inv);
                  w4[q] = *reinterpret_cast<uint32_t*>(&v2);
                }
                *reinterpret_cast<uint4*>(dst + c0 + c) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
            }
          }
          if (row == 0) p.sync[grp] = 0;  // ready for the next launch
        }
      }
    }
  }
  __syncwarp();
  __syncthreads();
  if (abort_flag != 0 && threadIdx.x == 0) {
    // after a bounded wait gave up: MMAs and copies in flight must finish
    // before TMEM and shared memory are released
    mbar_drain(&o_done, 0, err, 609);
    mbar_drain(&q_full, 0, err, 610);
    for (int j = kv_consumed; j < kv_issued; ++j) mbar_drain(&kv_full[j % kAStages], (j / kAStages) & 1, err, 611);
  }
  __syncthreads();
  if (S > 1 && p.cluster) {
    // every thread of every CTA of the cluster passes both cluster barriers,
    // whatever happened before, so none waits for a CTA that left
    cluster_sync();
    const bool good = abort_flag == 0 && tile_ok;
    const int RS = kAT / S, r0 = sp * RS;
    if (good) {
      if ((int)threadIdx.x < RS) {
        const int row = r0 + threadIdx.x;
        const uint32_t am = smem_u32(&s_m[row]), al = smem_u32(&s_l[row]);
        float mq[8], lq[8], mm = -INFINITY;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) {
            mq[q] = ld_dsmem_f32(mapa_shared(am, (uint32_t)q));
            lq[q] = ld_dsmem_f32(mapa_shared(al, (uint32_t)q));
            mm = fmaxf(mm, mq[q]);
          }
        float w[8], L = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) {
            w[q] = mq[q] == -INFINITY ? 0.f : exp2f(mq[q] - mm);
            L += w[q] * lq[q];
          }
        const float inv = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) s_w[threadIdx.x][q] = w[q] * inv;
      }
      __syncthreads();
      // one warp per row, 32 lanes x 4 columns; each thread has all of its
      // 16 remote loads in flight at once
      const float* sO = reinterpret_cast<const float*>(sKV);
      __nv_bfloat16* Ob = p.O + (size_t)b * p.k * (p.n_heads * kAT) + (size_t)h * kAT;
      if (S == 2) attn_cluster_combine<2>(sO, s_w, r0, qt * kAT, p.k, p.n_heads * kAT, Ob);
      else if (S == 4) attn_cluster_combine<4>(sO, s_w, r0, qt * kAT, p.k, p.n_heads * kAT, Ob);
      else attn_cluster_combine<8>(sO, s_w, r0, qt * kAT, p.k, p.n_heads * kAT, Ob);
    }
    cluster_sync();
  }
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// How many clusters of `splits` attention CTAs the GPU holds at once (0: none).
static int attn_max_clusters(int splits) {
  static int cache_all[kMaxDevices][9] = {{0}};  // per device, filled once (benign race: same value)
  if (splits < 2 || splits > 8) return 0;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int* cache = cache_all[dev];
  if (cache[splits] == 0) {
    if (configure_kernel((const void*)attn_tc_kernel, kASmem, false) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, 1, 1);
    cfg.blockDim = dim3(kAThreads, 1, 1);
    cfg.dynamicSmemBytes = kASmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cache[splits] = n > 0 ? n : -1;
  }
  return cache[splits] > 0 ? cache[splits] : 0;
}

cudaError_t launch_attention(int dtype, const void* Q, const void* Kc, const void* Vc, void* O,
                             int B, int k, int N, int n_heads, int head_dim, float* part_o,
                             float* part_ml, int max_rows, int* sync, int sync_len, int* err,
                             int allow_cluster, cudaStream_t stream) {
  if (head_dim > 128) return cudaErrorInvalidValue;
  const float scale = 1.0f / sqrtf((float)head_dim);
  if (dtype == 1 && head_dim == kAT) {
    const int q_tiles = (k + kAT - 1) / kAT;
    const int n_kt = (N + kAT - 1) / kAT;
    const long long groups = (long long)B * n_heads * q_tiles;
    // capacity of the scratch in (128-row, one-head) partial slots
    const long long slots = (long long)max_rows * n_heads / kAT;
    const cudaError_t ec = configure_kernel((const void*)attn_tc_kernel, kASmem, false);
    if (ec != cudaSuccess) return ec;
    int splits = 1;
    if (allow_cluster) {
      // split the keys while every cluster of the grid is resident at once and
      // each split keeps >= 1 key tile (one tile per CTA measured fastest at
      // N = 512: 16.9 against 18.8 us with two)
      while (splits < 8 && n_kt >= splits * 2 && groups <= attn_max_clusters(splits * 2)) splits *= 2;
      if (const char* env = std::getenv("SPA_ATTN_SPLITS")) {  // tuning override: 1, 2, 4 or 8 key splits
        const int v = std::atoi(env);
        if ((v == 1 || v == 2 || v == 4 || v == 8) && v <= n_kt) splits = v;
      }
    } else {
      // split the keys while the grid is small, each split keeps >= 2 key tiles
      while (splits < 8 && groups * splits * 2 <= 160 && n_kt >= splits * 4 &&
             groups * splits * 2 <= slots && groups <= sync_len)
        splits *= 2;
    }
    AttnTcParams p;
    std::memset(&p, 0, sizeof(p));
    if (encode_bf16_map(&p.tmQ, Q, (uint64_t)B * k, (uint64_t)n_heads * kAT) ||
        encode_bf16_map(&p.tmK, Kc, (uint64_t)B * N, (uint64_t)n_heads * kAT) ||
        encode_bf16_map(&p.tmV, Vc, (uint64_t)B * N, (uint64_t)n_heads * kAT))
      return cudaErrorInvalidValue;
    p.O = (__nv_bfloat16*)O;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.sync = sync;
    p.err = err;
    p.B = B; p.k = k; p.N = N; p.n_heads = n_heads; p.q_tiles = q_tiles; p.splits = splits;
    p.cluster = allow_cluster && splits > 1;
    p.scale_log2 = scale * 1.4426950408889634f;
    dim3 grid(q_tiles * splits, n_heads, B);
    if (!p.cluster) return launch_k(attn_tc_kernel, grid, dim3(kAThreads), kASmem, stream, p);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kAThreads, 1, 1);
    cfg.dynamicSmemBytes = kASmem;
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
    return cudaLaunchKernelEx(&cfg, attn_tc_kernel, p);
  }
  dim3 grid((k + 3) / 4, n_heads, B), block(128);
  if (dtype == 1)
    return launch_k(attn_simt_kernel<__nv_bfloat16>, grid, block, 0, stream, (const __nv_bfloat16*)Q,
                    (const __nv_bfloat16*)Kc, (const __nv_bfloat16*)Vc, (__nv_bfloat16*)O, k, N,
                    n_heads, head_dim, scale);
  return launch_k(attn_simt_kernel<float>, grid, block, 0, stream, (const float*)Q, (const float*)Kc,
                  (const float*)Vc, (float*)O, k, N, n_heads, head_dim, scale);
}

}  // namespace spa
