// S3 over a vocabulary split across ranks: the global top-k of every
// (sequence, head) from the per-shard top-k lists.
//
// "Medusa — 让大模型自己同时猜好几个 token", 核心要点: each head keeps the k
// most probable tokens of its own vocabulary projection.  When the rows of
// Wout are spread over G ranks, the k best rows of the whole vocabulary are
// among the union of each shard's k best (every shard holds at least k rows,
// and a shard keeps its rows in global id order), so selecting k from the
// G*k gathered candidates gives exactly the unsplit result.
//
// One CTA per (sequence, head): the G*k candidates go to shared memory with
// their global ids (shard's first row + local id); k rounds each pick the
// best remaining candidate (value descending, lower id first on equal
// values; NaN ranks below every number) with a block arg-max.
#include <cmath>
#include <climits>

#include "common.cuh"

namespace medusa {
namespace {

constexpr int kMergeThreads = 128;
constexpr int kMergeWarps = kMergeThreads / 32;

struct MergeArgs {
  const float* vals;      // [G, B*K, topk]
  const int32_t* ids;     // [G, B*K, topk], shard-local
  float* out_vals;        // [B*K, topk]
  int32_t* out_ids;       // [B*K, topk], global
  int G, BK, topk;
  int row0[MEDUSA_MAX_SHARDS];
};

// Candidate a ranks before candidate b.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  const bool na = isnan(va), nb = isnan(vb);
  if (na || nb) return nb && (!na || ia < ib);
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(const MergeArgs a) {
  __shared__ float cv[MEDUSA_MAX_SHARDS * MEDUSA_MAX_TOPK];
  __shared__ int ci[MEDUSA_MAX_SHARDS * MEDUSA_MAX_TOPK];   // -1 once taken
  __shared__ float wv[kMergeWarps];
  __shared__ int wi[kMergeWarps], wp[kMergeWarps];
  const int bk = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = a.G * a.topk;
  for (int c = tid; c < n; c += kMergeThreads) {
    const int g = c / a.topk, j = c - g * a.topk;
    const size_t src = (static_cast<size_t>(g) * a.BK + bk) * a.topk + j;
    cv[c] = a.vals[src];
    ci[c] = a.row0[g] + a.ids[src];
  }
  __syncthreads();
  for (int r = 0; r < a.topk; ++r) {
    float bv = 0.f;
    int bi = INT_MAX, bp = -1;   // bp < 0: nothing found yet
    for (int c = tid; c < n; c += kMergeThreads) {
      const int id = ci[c];
      if (id >= 0 && (bp < 0 || ranks_before(cv[c], id, bv, bi))) {
        bv = cv[c];
        bi = id;
        bp = c;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      const int op = __shfl_xor_sync(0xffffffffu, bp, off);
      if (op >= 0 && (bp < 0 || ranks_before(ov, oi, bv, bi))) {
        bv = ov;
        bi = oi;
        bp = op;
      }
    }
    if (lane == 0) {
      wv[warp] = bv;
      wi[warp] = bi;
      wp[warp] = bp;
    }
    __syncthreads();
    if (tid == 0) {
      float v = wv[0];
      int i = wi[0], pos = wp[0];
      for (int w = 1; w < kMergeWarps; ++w)
        if (wp[w] >= 0 && (pos < 0 || ranks_before(wv[w], wi[w], v, i))) {
          v = wv[w];
          i = wi[w];
          pos = wp[w];
        }
      // n >= topk candidates, so every round finds one.
      a.out_vals[static_cast<size_t>(bk) * a.topk + r] = v;
      a.out_ids[static_cast<size_t>(bk) * a.topk + r] = i;
      ci[pos] = -1;
    }
    __syncthreads();
  }
}

}  // namespace

medusa_status_t launch_topk_merge(const float* vals, const int32_t* ids, const int32_t* row0, int G, int B,
                                  int K, int topk, float* out_vals, int32_t* out_ids, cudaStream_t stream) {
  MergeArgs a{};
  a.vals = vals;
  a.ids = ids;
  a.out_vals = out_vals;
  a.out_ids = out_ids;
  a.G = G;
  a.BK = B * K;
  a.topk = topk;
  for (int g = 0; g < G; ++g) a.row0[g] = row0[g];
  topk_merge_kernel<<<a.BK, kMergeThreads, 0, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_topk_merge", e);
}

}  // namespace medusa
