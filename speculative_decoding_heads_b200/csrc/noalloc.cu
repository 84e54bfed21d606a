// medusa_heads_topk_noalloc: the heads + top-k call for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: a host that
// reserves all device memory up front and gives plugins no allocator, or
// code that runs where allocating is not allowed.  This entry point keeps
// the scratch that medusa_heads_topk normally takes from the caller's
// workspace in a fixed array that lives in the library's own device memory
// (every GPU that loads the library holds kNoAllocScratchBytes of it until
// the process exits).  The caller still passes every input and output.
//
// In host code the array's name only stands for the symbol; the device
// address is fetched with cudaGetSymbolAddress once per device, with that
// device current, on the first call made on it, and kept for the life of the
// process.  After a device reset (cudaDeviceReset, or the primary context
// torn down) the array may sit elsewhere, so this entry point must not be
// used across a reset.
#include <mutex>
#include <string>

#include "common.cuh"

namespace medusa {
namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;   // 4 MiB per device

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDev];

// Device address of the scratch array on the current device (set up on first use).
medusa_status_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("medusa_heads_topk_noalloc: cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDev) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_heads_topk_noalloc: device index");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail("medusa_heads_topk_noalloc: cudaGetSymbolAddress", e);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MEDUSA_OK;
}

}  // namespace
}  // namespace medusa

using namespace medusa;

extern "C" medusa_status_t medusa_heads_topk_noalloc(const void* h, const void* W1, const void* b1,
                                                     const void* Wout, int B, int d, int V, int K, int topk,
                                                     medusa_dtype_t dtype, float* head_logits, int32_t* topk_ids,
                                                     float* topk_vals, cudaStream_t stream) {
  if (sm_count() <= 0) return fail(MEDUSA_ERR_CUDA, "medusa_heads_topk_noalloc: no usable CUDA device");
  if (B < 1 || d < 1 || V < 1 || K < 1 || topk < 1)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_topk_noalloc: B, d, V, K and topk must be positive");
  const size_t need = heads_workspace_bytes(B, d, V, K, topk);
  if (need > kNoAllocScratchBytes)
    return fail(MEDUSA_ERR_UNSUPPORTED,
                "medusa_heads_topk_noalloc: this shape needs " + std::to_string(need) +
                    " bytes of scratch, above the fixed " + std::to_string(kNoAllocScratchBytes) +
                    "-byte array; use medusa_heads_topk with a workspace");
  void* scratch = nullptr;
  medusa_status_t st = scratch_address(&scratch);
  if (st != MEDUSA_OK) return st;
  // Every argument is checked before the shared array is touched: a call that
  // is refused enqueues nothing, not even the clearing below.
  st = check_heads(h, W1, b1, Wout, B, d, V, K, topk, dtype, head_logits, topk_ids, topk_vals, scratch,
                   kNoAllocScratchBytes);
  if (st != MEDUSA_OK) return st;
  // The array keeps whatever the previous call left.  The kernel's completion
  // counters must start at zero, so the part of the array this call uses is
  // cleared on the stream first (a memset, not an allocation).
  cudaError_t e = cudaMemsetAsync(scratch, 0, need, stream);
  if (e != cudaSuccess) return cuda_fail("medusa_heads_topk_noalloc: clearing the scratch", e);
  return launch_heads(h, W1, b1, Wout, B, d, V, K, topk, dtype, head_logits, topk_ids, topk_vals, scratch, stream);
}
