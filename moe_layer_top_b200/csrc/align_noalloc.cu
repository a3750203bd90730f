// moe_align_noalloc: the expert alignment for callers that cannot allocate
// device memory.
//
// Some callers may not call cudaMalloc (or any allocator) at the point where
// they align tokens: code that runs while a CUDA graph is being captured
// into a fixed memory plan, plug-ins whose host framework owns every device
// allocation and hands out none, and latency-critical serving loops that
// forbid allocator calls after start-up.  moe_align needs a few hundred
// kilobytes of scratch (per-chunk expert histograms, counts, offsets and a
// status word); this variant keeps that scratch in one file-scope device
// array instead, so the caller passes only its inputs and outputs.
//
// The array is MOE_ALIGN_NOALLOC_SCRATCH_BYTES long and lives on every GPU
// that loads the library until the process exits.  Its device address is
// looked up once per device (cudaGetSymbolAddress, with that device current)
// on the first call made on that device and cached for the life of the
// process; after a cudaDeviceReset of that device the cached address is
// stale, so the entry point must not be called on it again.  Every call on a
// device shares the array: calls that overlap on the GPU (different streams
// without ordering) race on it.
#include <cstdio>
#include <mutex>

#include "kernels.h"
#include "moe_b200.h"

namespace {

static __device__ __align__(256) unsigned char g_align_scratch[MOE_ALIGN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDev] = {nullptr};

inline size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

// Device address of g_align_scratch on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_align_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" MOE_API int moe_align_noalloc(const int32_t* topk_ids, int32_t T, int32_t topk, int32_t E,
                                         int32_t block_m, int32_t* sorted_token_ids, int32_t* expert_ids,
                                         int32_t* num_tokens_post_padded, int32_t* expert_counts,
                                         int32_t* expert_offsets, void* stream) {
  // everything is checked on the host before the device is touched
  if (T < 0 || topk < 1 || E < 1 || E > 1024 || block_m < 1 || block_m > 4096)
    return moe::record_error(MOE_ERR_INVALID, "align_noalloc: bad sizes (T, topk, E, block_m)");
  if (!sorted_token_ids || !expert_ids || !num_tokens_post_padded || (T > 0 && !topk_ids))
    return moe::record_error(MOE_ERR_INVALID, "align_noalloc: NULL pointer");
  const size_t need = moe_align_workspace_size(T, topk, E);
  if (need == 0 || need > static_cast<size_t>(MOE_ALIGN_NOALLOC_SCRATCH_BYTES))
    return moe::record_error(MOE_ERR_INVALID,
                             "align_noalloc: T * topk and E need more scratch than the static "
                             "MOE_ALIGN_NOALLOC_SCRATCH_BYTES array holds; use moe_align with a workspace");
  void* scratch = nullptr;
  const cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    char msg[192];
    snprintf(msg, sizeof msg, "align_noalloc: no device address for the static scratch (%s: %s)",
             cudaGetErrorName(e), cudaGetErrorString(e));
    return moe::record_error(MOE_ERR_CUDA, msg);
  }
  // moe_align clears the status word it owns and writes every other scratch
  // entry it reads, so no stale contents of the previous call are used
  return moe_align(topk_ids, T, topk, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded,
                   expert_counts, expert_offsets, scratch, need, stream);
}
