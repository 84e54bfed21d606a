// S7: keep the accepted prefix's K/V ("Medusa — 让大模型自己同时猜好几个 token",
// 实践案例 case 1 step 4: keep the accepted prefix, re-guess the rest).
// For every (layer, sequence, head) slice the a+1 accepted tree rows
// L+n_0 .. L+n_a move to L .. L+a.  A source row can be the destination of
// an earlier j (n_j >= j, so row L+n_j may be overwritten by j' = n_j), so
// each warp first reads all its source rows into shared memory, then writes.
// A second, one-block launch advances seq_lens once every slice is done.
#include "common.cuh"

namespace medusa {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) accept_rows_kernel(
    const TreeDev t, int n_slices, int B, int H, int row_bytes, unsigned char* __restrict__ k_cache,
    unsigned char* __restrict__ v_cache, int Lcap, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ best_path, const int32_t* __restrict__ accept_len, int* status) {
  extern __shared__ __align__(16) unsigned char buf[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slice = blockIdx.x * kWarps + warp;
  if (slice >= n_slices) return;
  const int b = (slice / H) % B;
  const int L = seq_lens[b];
  const int a = accept_len[b];
  const int best = best_path[b];
  if (L < 0 || L + t.T > Lcap || a < 0 || a > t.D || best < 0 || best >= t.P) {
    if (lane == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailAcceptSeqLen);
    return;
  }
  const int D1 = t.D + 1;
  if (t.retrieve[best * D1 + a] < 0) {   // accept_len longer than the chosen path
    if (lane == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailAcceptSeqLen);
    return;
  }
  unsigned char* mine = buf + static_cast<size_t>(warp) * D1 * row_bytes;
  const int chunks = row_bytes / 16;
  for (int which = 0; which < 2; ++which) {
    unsigned char* base = (which == 0 ? k_cache : v_cache) + static_cast<size_t>(slice) * Lcap * row_bytes;
    for (int j = 0; j <= a; ++j) {
      const int src = L + t.retrieve[best * D1 + j];
      const uint4* s = reinterpret_cast<const uint4*>(base + static_cast<size_t>(src) * row_bytes);
      uint4* d = reinterpret_cast<uint4*>(mine + static_cast<size_t>(j) * row_bytes);
      for (int c = lane; c < chunks; c += 32) d[c] = s[c];
    }
    __syncwarp();
    for (int j = 0; j <= a; ++j) {
      const uint4* s = reinterpret_cast<const uint4*>(mine + static_cast<size_t>(j) * row_bytes);
      uint4* d = reinterpret_cast<uint4*>(base + static_cast<size_t>(L + j) * row_bytes);
      for (int c = lane; c < chunks; c += 32) d[c] = s[c];
    }
    __syncwarp();
  }
}

__global__ void advance_lens_kernel(int B, int32_t* seq_lens, const int32_t* accept_len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) seq_lens[b] += accept_len[b] + 1;
}

}  // namespace

medusa_status_t launch_accept_kv(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype,
                                 void* k_cache, void* v_cache, int Lcap, int32_t* seq_lens,
                                 const int32_t* best_path, const int32_t* accept_len,
                                 cudaStream_t stream) {
  const int row_bytes = hd * (dtype == MEDUSA_BF16 ? 2 : 4);
  const int n_slices = layers * B * H;
  const size_t smem = static_cast<size_t>(kWarps) * (t.D + 1) * row_bytes;
  accept_rows_kernel<<<(n_slices + kWarps - 1) / kWarps, kWarps * 32, smem, stream>>>(
      t, n_slices, B, H, row_bytes, static_cast<unsigned char*>(k_cache), static_cast<unsigned char*>(v_cache),
      Lcap, seq_lens, best_path, accept_len, device_status_ptr());
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("medusa_accept_kv: rows launch", e);
  advance_lens_kernel<<<(B + 63) / 64, 64, 0, stream>>>(B, seq_lens, accept_len);
  e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_accept_kv: lens launch", e);
}

}  // namespace medusa
