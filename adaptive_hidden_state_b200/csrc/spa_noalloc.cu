// Sparse-query attention for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc: custom memory
// managers and allocator hooks that must not re-enter the CUDA allocator,
// hosts that hand the library a fixed device-memory budget up front, and
// latency-critical loops where an allocation (which can synchronise the
// device) is not allowed.  The attention step needs scratch beyond its inputs
// and outputs when it splits the keys across CTAs: each split writes partial
// outputs and softmax statistics that the last CTA of the query tile
// combines.  The regular path takes that scratch from a workspace the library
// allocated; the entry point here takes it from one fixed array in the
// library's own device image instead, so it allocates nothing.
//
// The array is a file-scope __device__ variable of 8 MiB: every GPU that
// loads the library holds it until the process exits.  Its device address is
// fetched with cudaGetSymbolAddress once per device, by the first call made
// with that device current.  Layout: split partials, then the per-query-tile
// split counters, then a two-int device error word (the same word the
// workspace calls use: bits of timed-out waits and failed index checks, and
// the site of the first one).
#include <cstdio>
#include <mutex>

#include "../../include/spa.h"
#include "spa_internal.h"

namespace {

// 8 MiB: fp32 split-KV partials, B * k * (d + 2 * n_heads) floats at most,
// then kNoAllocSyncInts counters (per query tile: splits finished), then the
// error word.
constexpr size_t kNoAllocScratchFloats = (size_t)2 << 20;
constexpr int kNoAllocSyncInts = 4096;
constexpr int kNoAllocErrInts = 2;
constexpr size_t kNoAllocPartialFloats = kNoAllocScratchFloats - kNoAllocSyncInts - kNoAllocErrInts;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {nullptr};

int fail(int status, const char* msg) { return spa::set_last_error(status, msg); }

// The device address of the fixed array on the current device (looked up
// once per device, with that device current), or null with the error set.
float* scratch_on_current_device(int* status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    *status = fail(SPA_ERR_CUDA, "cudaGetDevice failed or device ordinal out of range");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      *status = fail(SPA_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch failed");
      return nullptr;
    }
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *status = SPA_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int spa_attention_noalloc(const void* Q, const void* k_cache, const void* v_cache,
                                     void* O, int B, int k, int N, int n_heads, int head_dim,
                                     void* stream) {
  if (!Q || !k_cache || !v_cache || !O) return fail(SPA_ERR_INVALID, "null pointer");
  if (B < 1 || k < 1 || N < 1 || n_heads < 1 || head_dim < 1 || k > N)
    return fail(SPA_ERR_SHAPE, "bad sizes (need B, k, N, n_heads, head_dim >= 1 and k <= N)");
  if (head_dim != 128)
    return fail(SPA_ERR_UNSUPPORTED, "the allocation-free attention takes head_dim = 128 (bf16)");
  // launch grid (query tiles x key splits, heads, sequences) and 32-bit row indices
  if (B > 65535 || n_heads > 65535 || (long long)B * N * n_heads * head_dim >= (1LL << 31) ||
      (long long)B * k * n_heads * head_dim >= (1LL << 31))
    return fail(SPA_ERR_SHAPE, "B, n_heads or the cache size beyond the launch limits");
  int st = SPA_OK;
  float* scratch = scratch_on_current_device(&st);
  if (!scratch) return st;
  const long long d = (long long)n_heads * head_dim;
  const long long row_floats = d + 2LL * n_heads;  // one partial output row + its (m, l) pairs
  const long long tiles = (long long)B * n_heads * ((k + 127) / 128);
  // The keys are split only as far as the fixed array holds the partials
  // (max_rows rows) and the counters (one per query tile); a call beyond that
  // runs with fewer splits, down to none, which uses no scratch at all.
  const int max_rows = (int)(kNoAllocPartialFloats / row_floats);
  float* part_o = scratch;
  float* part_ml = scratch + (size_t)max_rows * d;
  int* sync = reinterpret_cast<int*>(scratch + kNoAllocPartialFloats);
  int* err = sync + kNoAllocSyncInts;
  const int sync_len = (int)(tiles < kNoAllocSyncInts ? tiles : kNoAllocSyncInts);
  // the split counters must start at zero (a completed call leaves them so);
  // the error word keeps its bits until spa_attention_noalloc_status reads it
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(sync, 0, (size_t)sync_len * sizeof(int), s) != cudaSuccess) {
    cudaGetLastError();
    return fail(SPA_ERR_CUDA, "clearing the split counters failed");
  }
  const cudaError_t e = spa::launch_attention(1, Q, k_cache, v_cache, O, B, k, N, n_heads, head_dim,
                                              part_o, part_ml, max_rows, sync, sync_len, err, 0, s);
  if (e != cudaSuccess) return fail(SPA_ERR_CUDA, cudaGetErrorString(e));
  return SPA_OK;
}

extern "C" int spa_attention_noalloc_status(void* stream) {
  int st = SPA_OK;
  float* scratch = scratch_on_current_device(&st);
  if (!scratch) return st;
  int* err = reinterpret_cast<int*>(scratch + kNoAllocPartialFloats) + kNoAllocSyncInts;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return fail(SPA_ERR_CUDA, "stream synchronisation failed");
  }
  int h[kNoAllocErrInts] = {0, 0};  // host stack memory: nothing is allocated
  if (cudaMemcpy(h, err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return fail(SPA_ERR_CUDA, "reading the error word failed");
  }
  if (h[0] == 0) return SPA_OK;
  if (cudaMemset(err, 0, sizeof(h)) != cudaSuccess) {
    cudaGetLastError();
    return fail(SPA_ERR_CUDA, "clearing the error word failed");
  }
  char msg[96];
  if (h[0] & spa::DEVERR_TIMEOUT) {
    snprintf(msg, sizeof(msg), "device wait timed out (site %d)", h[1]);
    return fail(SPA_ERR_TIMEOUT, msg);
  }
  snprintf(msg, sizeof(msg), "device check failed: bits 0x%x site %d", h[0], h[1]);
  return fail(SPA_ERR_DEVICE, msg);
}
