// S4: candidate assembly ("Medusa API参考：核心函数与类详解", 核心功能函数:
// generate_candidates gathers the flat candidate list through tree_indices and
// reads per-path candidates through retrieve_indices; tree_decoding takes
// medusa_position_ids).  One thread per output element; the flat list
// [root, head1 top-k, ..., headK top-k] is never materialised.
#include "common.cuh"

namespace medusa {
namespace {

__device__ __forceinline__ int32_t flat_token(const TreeDev& t, int b, int fi, const int32_t* root,
                                              const int32_t* topk_ids) {
  if (fi == 0) return root[b];
  return topk_ids[static_cast<size_t>(b) * t.K * t.topk + (fi - 1)];
}

__global__ void build_tree_kernel(const TreeDev t, int B, const int32_t* __restrict__ root,
                                  const int32_t* __restrict__ topk_ids,
                                  const int32_t* __restrict__ seq_lens, int32_t* __restrict__ tree_tokens,
                                  int32_t* __restrict__ candidates, int32_t* __restrict__ position_ids) {
  const int per_b = 2 * t.T + t.P * (t.D + 1);
  const int total = B * per_b;
  for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < total; g += gridDim.x * blockDim.x) {
    const int b = g / per_b;
    int o = g % per_b;
    if (o < t.T) {
      tree_tokens[b * t.T + o] = flat_token(t, b, t.tree_indices[o], root, topk_ids);
    } else if (o < 2 * t.T) {
      o -= t.T;
      position_ids[b * t.T + o] = seq_lens[b] + t.depth[o];
    } else {
      o -= 2 * t.T;
      const int node = t.retrieve[o];
      candidates[static_cast<size_t>(b) * t.P * (t.D + 1) + o] =
          node < 0 ? -1 : flat_token(t, b, t.tree_indices[node], root, topk_ids);
    }
  }
}

}  // namespace

medusa_status_t launch_build_tree(const TreeDev& t, int B, const int32_t* root_tokens,
                                  const int32_t* topk_ids, const int32_t* seq_lens,
                                  int32_t* tree_tokens, int32_t* candidates, int32_t* position_ids,
                                  cudaStream_t stream) {
  const int total = B * (2 * t.T + t.P * (t.D + 1));
  const int threads = 256;
  const int blocks = (total + threads - 1) / threads;
  build_tree_kernel<<<blocks, threads, 0, stream>>>(t, B, root_tokens, topk_ids, seq_lens, tree_tokens,
                                                    candidates, position_ids);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_build_tree: launch", e);
}

}  // namespace medusa
