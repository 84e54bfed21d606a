// S7: keep the accepted prefix's K/V ("Medusa — 让大模型自己同时猜好几个 token",
// 实践案例 case 1 step 4: keep the accepted prefix, re-guess the rest).
// For every (layer, sequence, head) slice the a+1 accepted tree rows
// L+n_0 .. L+n_a move to L .. L+a.  A source row can be the destination of
// an earlier j (n_j >= j, so row L+n_j may be overwritten by j' = n_j), so
// each thread owns one 16-byte column of one slice's K or V and loads all of
// its accepted source rows into registers before it writes any of them.
// A second, one-block launch advances seq_lens once every slice is done.
#include "common.cuh"

namespace medusa {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxRows = MEDUSA_MAX_K + 1;   // a <= D <= K

__global__ void __launch_bounds__(kThreads) accept_rows_kernel(
    const TreeDev t, int n_slices, int B, int H, int chunks, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, int Lcap, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ best_path, const int32_t* __restrict__ accept_len, int* status) {
  allow_dependents();
  wait_prior_grids();   // best path and accept length; attention done with the cache
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_slice = 2 * chunks;
  const long long slice = gid / per_slice;
  if (slice >= n_slices) return;
  const int rem = static_cast<int>(gid - slice * per_slice);
  const int which = rem / chunks, c = rem - which * chunks;
  const int b = static_cast<int>((slice / H) % B);
  const int L = seq_lens[b];
  const int a = accept_len[b];
  const int best = best_path[b];
  const int D1 = t.D + 1;
  if (L < 0 || L + t.T > Lcap || a < 0 || a > t.D || best < 0 || best >= t.P || t.retrieve[best * D1 + a] < 0) {
    if (rem == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailAcceptSeqLen);
    return;
  }
  uint4* base = (which == 0 ? k_cache : v_cache) + static_cast<size_t>(slice) * Lcap * chunks + c;
  const int32_t* path = t.retrieve + best * D1;
  uint4 r[kMaxRows];
#pragma unroll
  for (int j = 0; j < kMaxRows; ++j)
    if (j <= a && path[j] != j) r[j] = base[static_cast<size_t>(L + path[j]) * chunks];
#pragma unroll
  for (int j = 0; j < kMaxRows; ++j)
    if (j <= a && path[j] != j) base[static_cast<size_t>(L + j) * chunks] = r[j];
}

__global__ void advance_lens_kernel(int B, int32_t* seq_lens, const int32_t* accept_len) {
  wait_prior_grids();   // every slice has read seq_lens
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) seq_lens[b] += accept_len[b] + 1;
}

}  // namespace

medusa_status_t launch_accept_kv(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype,
                                 void* k_cache, void* v_cache, int Lcap, int32_t* seq_lens,
                                 const int32_t* best_path, const int32_t* accept_len,
                                 cudaStream_t stream, bool pdl) {
  const int row_bytes = hd * (dtype == MEDUSA_BF16 ? 2 : 4);
  const int chunks = row_bytes / 16;
  const long long n_slices = static_cast<long long>(layers) * B * H;
  const long long threads = n_slices * 2 * chunks;
  cudaError_t e = launch_kernel(accept_rows_kernel, dim3(static_cast<unsigned>((threads + kThreads - 1) / kThreads)),
                                dim3(kThreads), 0, stream, pdl, t, static_cast<int>(n_slices), B, H, chunks,
                                static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), Lcap,
                                static_cast<const int32_t*>(seq_lens), best_path, accept_len, device_status_ptr());
  if (e != cudaSuccess) return cuda_fail("medusa_accept_kv: rows launch", e);
  e = launch_kernel(advance_lens_kernel, dim3((B + 63) / 64), dim3(64), 0, stream, pdl, B, seq_lens, accept_len);
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_accept_kv: lens launch", e);
}

}  // namespace medusa
