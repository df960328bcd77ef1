// Sparse-query attention for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc: custom memory
// managers and allocator hooks that must not re-enter the CUDA allocator,
// hosts that hand the library a fixed device-memory budget up front, and
// latency-critical loops where an allocation (which can synchronise the
// device) is not allowed.  The attention step needs scratch beyond its inputs
// and outputs when it splits the keys across CTAs: each split writes partial
// outputs and softmax statistics that a second kernel combines.  The regular
// path takes that scratch from a workspace the library allocated; the entry
// point here takes it from one fixed array in the library's own device image
// instead, so it allocates nothing.
//
// The array is a file-scope __device__ variable of 8 MiB: every GPU that
// loads the library holds it until the process exits.  Its device address is
// fetched with cudaGetSymbolAddress once per device, by the first call made
// with that device current.
#include <cstdio>
#include <mutex>

#include "../../include/spa.h"
#include "spa_internal.h"

namespace {

// 8 MiB: fp32 split-KV partials, B * k * (d + 2 * n_heads) floats at most,
// then kNoAllocSyncInts counters (per query tile: splits finished).
constexpr size_t kNoAllocScratchFloats = (size_t)2 << 20;
constexpr int kNoAllocSyncInts = 4096;
constexpr size_t kNoAllocPartialFloats = kNoAllocScratchFloats - kNoAllocSyncInts;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {nullptr};

int fail(int status, const char* msg) { return spa::set_last_error(status, msg); }

}  // namespace

extern "C" int spa_attention_noalloc(const void* Q, const void* k_cache, const void* v_cache,
                                     void* O, int B, int k, int N, int n_heads, int head_dim,
                                     void* stream) {
  if (!Q || !k_cache || !v_cache || !O) return fail(SPA_ERR_INVALID, "null pointer");
  if (B < 1 || k < 1 || N < 1 || n_heads < 1 || head_dim < 1 || k > N)
    return fail(SPA_ERR_SHAPE, "bad sizes (need B, k, N, n_heads, head_dim >= 1 and k <= N)");
  if (head_dim != 128)
    return fail(SPA_ERR_UNSUPPORTED, "the allocation-free attention takes head_dim = 128 (bf16)");
  const long long d = (long long)n_heads * head_dim;
  const long long row_floats = d + 2LL * n_heads;  // one partial output row + its (m, l) pairs
  const long long rows = (long long)B * k;
  const long long tiles = (long long)B * n_heads * ((k + 127) / 128);
  if (rows * row_floats > (long long)kNoAllocPartialFloats || tiles > kNoAllocSyncInts)
    return fail(SPA_ERR_SHAPE,
                "B * k * (n_heads * head_dim + 2 * n_heads) exceeds the fixed scratch "
                "(2 Mi floats = 8 MiB), or B * n_heads * ceil(k / 128) exceeds 4096");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return fail(SPA_ERR_CUDA, "cudaGetDevice failed or device ordinal out of range");
  }
  float* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
      // once per device, with that device current: the device address of the array
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return fail(SPA_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch failed");
      }
      g_scratch_ptr[dev] = static_cast<float*>(p);
    }
    scratch = g_scratch_ptr[dev];
  }
  // split partials first, then their (m, l) pairs; the launcher splits the
  // keys only as far as max_rows partial rows fit
  const int max_rows = (int)(kNoAllocPartialFloats / row_floats);
  float* part_o = scratch;
  float* part_ml = scratch + (size_t)max_rows * d;
  int* sync = reinterpret_cast<int*>(scratch + kNoAllocPartialFloats);
  // the split counters must start at zero (a completed call leaves them so)
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(sync, 0, (size_t)tiles * sizeof(int), s) != cudaSuccess) {
    cudaGetLastError();
    return fail(SPA_ERR_CUDA, "clearing the split counters failed");
  }
  const cudaError_t e = spa::launch_attention(1, Q, k_cache, v_cache, O, B, k, N, n_heads, head_dim,
                                              part_o, part_ml, max_rows, sync, (int)tiles, nullptr, 0, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, cudaGetErrorString(e));
  return SPA_OK;
}
