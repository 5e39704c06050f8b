// fa_noalloc.cu -- fa_fwd_kvcache_noalloc: the paged split-KV decode with its
// split partials kept in a fixed device array owned by this library, so the
// caller passes no workspace and nothing is allocated per call.
//
// For callers that cannot allocate device memory themselves: a plain C host
// program or plugin that has no device allocator of its own, a component
// living inside another runtime whose memory pool already holds the free
// device memory (so a cudaMalloc of its own would fail), or a latency-bound
// decode loop that must not call cudaMalloc, which can synchronise the
// device.
//
// The array below is a file-scope __device__ variable: every GPU that loads
// this library holds FA_NOALLOC_SCRATCH_BYTES of it until the process exits.
// In host code its name is only a host-side stand-in, so the device address
// is looked up with cudaGetSymbolAddress once per device (on the first call
// made with that device current) and that address is what the kernels get.
// Only a successful lookup is kept: after a failed one (say, made during a
// stream capture) the next call on that device looks the address up again.
#include "fa.h"
#include "fa_internal.h"

#include <cuda_runtime.h>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = FA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_split_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // set once a lookup on the device succeeded

// Device address of g_split_scratch on the current device.
fa_status scratch_for_current_device(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  if (dev >= kMaxDevices) return FA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_split_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // clear the (non-sticky) error so a later call starts clean
      return FA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_fwd_kvcache_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                            const int* block_table, const int* cache_seqlens, void* out, float* lse,
                                            int B, int H, int d, int num_pages, int page_size, int max_blocks,
                                            fa_dtype dtype, float scale, int window_left,
                                            const float* alibi_slopes, float softcap, int num_splits,
                                            cudaStream_t stream) {
  // Same sizes, split count and partial layout as fa_fwd_kvcache; only the
  // place the partials live differs.
  const size_t need = fa_kvcache_workspace_size(B, H, d, max_blocks, page_size, num_splits);
  if (need > kScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const fa_status st = scratch_for_current_device(&scratch);
    if (st != FA_OK) return st;
  }
  // Every split writes all of its partial (empty splits write O = 0 and
  // LSE = -inf) before the merge reads it, so nothing left in the array by
  // an earlier call is ever read and nothing needs clearing.
  return fa_fwd_kvcache(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, B, H, d, num_pages, page_size,
                        max_blocks, dtype, scale, window_left, alibi_slopes, softcap, num_splits, scratch,
                        need > 0 ? kScratchBytes : 0, stream);
}
