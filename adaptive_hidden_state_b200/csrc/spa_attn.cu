// Sparse-query attention of the SPA-Cache layer step: the k refreshed
// queries of each sequence attend to all N cached keys and values (the
// bidirectional cache K^c, V^c, already holding this step's fresh rows).
//
// attn_mma_kernel (bf16, head_dim 128): flash-style, 64 queries x 1 head per
// CTA (16 per warp), key/value tiles of 64 rows double-buffered in shared
// memory with cp.async, S = Q K^T and O += P V on the tensor cores
// (mma.sync m16n8k16, fp32 accumulate), online softmax in fp32 registers.
// Keys are split across CTAs when the grid would not fill the GPU; each split
// writes (O_s / l_s, m_s, l_s) and attn_combine_kernel merges them in a fixed
// order.
//
// attn_simt_kernel: one warp per (query, head), online softmax over chunks of
// 32 keys (one key per lane), fp32 throughout.  Used for the fp32
// configurations and for head sizes the tensor-core kernel does not cover.
#include "spa_device.cuh"
#include "spa_internal.h"

namespace spa {

template <typename T>
__global__ void __launch_bounds__(128) attn_simt_kernel(const T* Q, const T* Kc, const T* Vc, T* O,
                                                        int k, int N, int n_heads, int hd,
                                                        float scale) {
  __shared__ float qs[4][128];
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
// tensor-core attention, head_dim = 128
// ---------------------------------------------------------------------------
constexpr int kBQ = 64, kBK = 64, kHD = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk c of row `row` in a [rows][128] bf16 tile whose
// chunks are XOR-swizzled by (row & 7) so ldmatrix reads are conflict-free.
__device__ __forceinline__ uint32_t swz(int row, int c) {
  return (uint32_t)(row * 256 + ((c ^ (row & 7)) << 4));
}

// Loads rows [row0, row0 + 64) (head h) of a [., n_rows, d] bf16 matrix into a
// swizzled 64 x 128 tile; rows >= n_rows are zero-filled.
__device__ __forceinline__ void load_tile64(uint32_t sbase, const __nv_bfloat16* g, int row0,
                                            int n_rows, int d, int tid) {
#pragma unroll
  for (int i = 0; i < (kBK * 16) / 128; ++i) {
    const int id = tid + i * 128;
    const int row = id >> 4, c = id & 15;
    const int gr = row0 + row;
    const bool ok = gr < n_rows;
    const __nv_bfloat16* src = g + (size_t)(ok ? gr : 0) * d + c * 8;
    cp_async16(sbase + swz(row, c), src, ok);
  }
}

__global__ void __launch_bounds__(128) attn_mma_kernel(const __nv_bfloat16* __restrict__ Q,
                                                       const __nv_bfloat16* __restrict__ Kc,
                                                       const __nv_bfloat16* __restrict__ Vc,
                                                       __nv_bfloat16* __restrict__ O, float* part_o,
                                                       float* part_ml, int k, int N, int n_heads,
                                                       int splits, float scale_log2) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + kBQ * 256;
  const uint32_t sV0 = sK0 + 2 * kBK * 256;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y;
  const int b = blockIdx.z / splits, split = blockIdx.z % splits;
  const int d = n_heads * kHD;
  const int n_kt = (N + kBK - 1) / kBK;
  const int kt0 = (split * n_kt) / splits, kt1 = ((split + 1) * n_kt) / splits;

  const __nv_bfloat16* Qg = Q + ((size_t)b * k) * d + (size_t)h * kHD;
  const __nv_bfloat16* Kg = Kc + ((size_t)b * N) * d + (size_t)h * kHD;
  const __nv_bfloat16* Vg = Vc + ((size_t)b * N) * d + (size_t)h * kHD;

  load_tile64(sQ, Qg, qt * kBQ, k, d, tid);
  if (kt0 < kt1) {
    load_tile64(sK0, Kg, kt0 * kBK, N, d, tid);
    load_tile64(sV0, Vg, kt0 * kBK, N, d, tid);
  }
  cp_async_commit();

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qf[8][4];

  for (int kt = kt0; kt < kt1; ++kt) {
    const int stage = (kt - kt0) & 1;
    if (kt + 1 < kt1) {
      const int ns = stage ^ 1;
      load_tile64(sK0 + ns * kBK * 256, Kg, (kt + 1) * kBK, N, d, tid);
      load_tile64(sV0 + ns * kBK * 256, Vg, (kt + 1) * kBK, N, d, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (kt == kt0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int row = warp * 16 + (lane & 15), c = 2 * kk + (lane >> 4);
        ldsm_x4(sQ + swz(row, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t sK = sK0 + stage * kBK * 256, sV = sV0 + stage * kBK * 256;
    // S = Q K^T  (16 x 64 per warp)
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const int key = j * 8 + ((lane >> 4) << 3) + (lane & 7);
        const int c = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(key, c), b0, b1, b2, b3);
        mma_bf16(s[j], qf[kk], b0, b1);
        mma_bf16(s[j + 1], qf[kk], b2, b3);
      }
    }
    // scale, mask keys >= N, online softmax (rows lane/4 and lane/4 + 8)
    const int key_base = kt * kBK + 2 * (lane & 3);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key_base + j * 8 + (e & 1);
        float v = s[j][e] * scale_log2;
        if (key >= N) v = -INFINITY;
        s[j][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float corr[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
      const float mn = fmaxf(m_r[rr], mx[rr]);
      corr[rr] = exp2f(m_r[rr] - mn);
      m_r[rr] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[j][e] - m_r[e >> 1]);
        s[j][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      rs[rr] += __shfl_xor_sync(0xffffffffu, rs[rr], 1);
      rs[rr] += __shfl_xor_sync(0xffffffffu, rs[rr], 2);
      l_r[rr] = l_r[rr] * corr[rr] + rs[rr];
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= corr[0]; o[i][1] *= corr[0];
      o[i][2] *= corr[1]; o[i][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        const int key = kk * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
        const int ch = c + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz(key, ch), b0, b1, b2, b3);
        mma_bf16(o[c], pa, b0, b1);
        mma_bf16(o[c + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // write: rows r = lane/4 (+8) of this warp's 16 queries
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int qi = qt * kBQ + warp * 16 + (lane >> 2) + rr * 8;
    if (qi >= k) continue;
    const float inv = l_r[rr] > 0.f ? 1.0f / l_r[rr] : 0.f;
    const size_t t = (size_t)b * k + qi;
    if (splits == 1) {
      __nv_bfloat16* dst = O + t * d + (size_t)h * kHD + 2 * (lane & 3);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        *reinterpret_cast<uint32_t*>(dst + c * 8) =
            pack_bf16(o[c][2 * rr] * inv, o[c][2 * rr + 1] * inv);
      }
    } else {
      const size_t rows = gridDim.z / splits * (size_t)k;  // B * k
      float* dst = part_o + ((size_t)split * rows + t) * d + (size_t)h * kHD + 2 * (lane & 3);
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<float2*>(dst + c * 8) = make_float2(o[c][2 * rr] * inv, o[c][2 * rr + 1] * inv);
      if ((lane & 3) == 0) {
        float* ml = part_ml + (((size_t)split * rows + t) * n_heads + h) * 2;
        ml[0] = m_r[rr];
        ml[1] = l_r[rr];
      }
    }
  }
}

// O[t, h] = sum_s w_s O_s / sum_s w_s with w_s = l_s 2^(m_s - max m), in order s = 0..S-1.
__global__ void attn_combine_kernel(const float* part_o, const float* part_ml,
                                    __nv_bfloat16* O, int rows, int n_heads, int splits) {
  const int t = blockIdx.x, h = blockIdx.y, c = threadIdx.x;  // 128 threads = head_dim
  const int d = n_heads * kHD;
  float mmax = -INFINITY;
  for (int s = 0; s < splits; ++s)
    mmax = fmaxf(mmax, part_ml[(((size_t)s * rows + t) * n_heads + h) * 2]);
  float num = 0.f, den = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* ml = part_ml + (((size_t)s * rows + t) * n_heads + h) * 2;
    const float w = ml[1] * exp2f(ml[0] - mmax);
    num += w * part_o[((size_t)s * rows + t) * d + (size_t)h * kHD + c];
    den += w;
  }
  O[(size_t)t * d + (size_t)h * kHD + c] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
}

cudaError_t launch_attention(int dtype, const void* Q, const void* Kc, const void* Vc, void* O,
                             int B, int k, int N, int n_heads, int head_dim, float* part_o,
                             float* part_ml, int max_rows, int* err, cudaStream_t stream) {
  (void)err;
  if (head_dim > 128) return cudaErrorInvalidValue;
  const float scale = 1.0f / sqrtf((float)head_dim);
  if (dtype == 1 && head_dim == kHD) {
    const int q_tiles = (k + kBQ - 1) / kBQ;
    const int n_kt = (N + kBK - 1) / kBK;
    const int base = q_tiles * n_heads * B;
    int splits = 1;
    // split the keys until about two CTAs per SM are busy, >= 2 key tiles per split
    while (splits < 16 && base * splits < 2 * 148 && n_kt / (splits * 2) >= 2 &&
           (long long)(splits * 2) * B * k <= max_rows)
      splits *= 2;
    const int smem = (kBQ + 4 * kBK) * 256;
    static bool configured = false;
    if (!configured) {
      cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      configured = true;
    }
    dim3 grid(q_tiles, n_heads, B * splits);
    attn_mma_kernel<<<grid, 128, smem, stream>>>(
        (const __nv_bfloat16*)Q, (const __nv_bfloat16*)Kc, (const __nv_bfloat16*)Vc,
        (__nv_bfloat16*)O, part_o, part_ml, k, N, n_heads, splits, scale * 1.4426950408889634f);
    if (splits > 1) {
      cudaError_t e = cudaPeekAtLastError();
      if (e != cudaSuccess) return e;
      attn_combine_kernel<<<dim3(B * k, n_heads), kHD, 0, stream>>>(part_o, part_ml,
                                                                   (__nv_bfloat16*)O, B * k,
                                                                   n_heads, splits);
    }
    return cudaPeekAtLastError();
  }
  dim3 grid((k + 3) / 4, n_heads, B), block(128);
  if (dtype == 1)
    attn_simt_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
        (const __nv_bfloat16*)Q, (const __nv_bfloat16*)Kc, (const __nv_bfloat16*)Vc,
        (__nv_bfloat16*)O, k, N, n_heads, head_dim, scale);
  else
    attn_simt_kernel<float><<<grid, block, 0, stream>>>((const float*)Q, (const float*)Kc,
                                                        (const float*)Vc, (float*)O, k, N, n_heads,
                                                        head_dim, scale);
  return cudaPeekAtLastError();
}

}  // namespace spa
