// Sparse-query attention of the SPA-Cache layer step: the k refreshed
// queries of each sequence attend to all N cached keys and values (the
// bidirectional cache K^c, V^c, already holding this step's fresh rows).
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

cudaError_t launch_attention(int dtype, const void* Q, const void* Kc, const void* Vc, void* O,
                             int B, int k, int N, int n_heads, int head_dim, float* part_o,
                             float* part_ml, int max_splits, int* err, cudaStream_t stream) {
  (void)part_o; (void)part_ml; (void)max_splits; (void)err;
  if (head_dim > 128) return cudaErrorInvalidValue;
  dim3 grid((k + 3) / 4, n_heads, B), block(128);
  const float scale = 1.0f / sqrtf((float)head_dim);
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
