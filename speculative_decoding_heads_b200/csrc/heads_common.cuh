// Device pieces shared by the two heads kernels (heads.cu on the CUDA cores,
// heads_tc.cu on the tensor cores): the warp-cooperative insertion into a
// sorted top-k list, the merge of the per-CTA lists of one (sequence, head),
// and the candidate-tree build (S4) done by the last CTA of medusa_step's
// heads launch.
#pragma once

#include <cfloat>
#include <cstdint>

#include "common.cuh"

namespace medusa {

// One warp: insert (v, id) into the sorted list (lv, lid, *cnt) of capacity
// topk (larger value first, lower id first on equal values).
__device__ __forceinline__ void list_insert(float* lv, int* lid, int* cnt_p, int topk, float v, int id, int lane) {
  const int cnt = *cnt_p;
  float ev = -FLT_MAX;
  int ei = -1;
  if (lane < cnt) {
    ev = lv[lane];
    ei = lid[lane];
  }
  const bool before = lane < cnt && ranks_before(ev, ei, v, id);
  const int pos = __popc(__ballot_sync(0xffffffffu, before));
  const float pv = __shfl_up_sync(0xffffffffu, ev, 1);
  const int pi = __shfl_up_sync(0xffffffffu, ei, 1);
  __syncwarp();
  if (pos < topk && lane < topk && lane >= pos && lane <= cnt) {
    lv[lane] = (lane == pos) ? v : pv;
    lid[lane] = (lane == pos) ? id : pi;
  }
  __syncwarp();
  if (lane == 0 && pos < topk && cnt < topk) *cnt_p = cnt + 1;
  __syncwarp();
}

constexpr int kMergeRegs = 16;   // candidates per lane held in registers by the merge

// One warp: the topk best of ncand published candidates (vals/ids, entries
// with id < 0 are empty), written to out_ids / out_vals in order.  Each of
// the topk rounds picks the best candidate that ranks strictly after the
// previous pick.
__device__ __forceinline__ void merge_candidates(const float* vals, const int32_t* ids, int ncand, int topk,
                                                 int32_t* out_ids, float* out_vals, int lane) {
  float cv[kMergeRegs];
  int ci[kMergeRegs];
#pragma unroll
  for (int m = 0; m < kMergeRegs; ++m) {
    const int i = lane + 32 * m;
    cv[m] = -FLT_MAX;
    ci[m] = -1;
    if (i < ncand) {
      cv[m] = __ldcg(vals + i);
      ci[m] = __ldcg(ids + i);
    }
  }
  float prev_v = FLT_MAX;
  int prev_i = -1;
  for (int r = 0; r < topk; ++r) {
    float bv = -FLT_MAX;
    int bi = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < kMergeRegs; ++m)
      if (ci[m] >= 0 && ranks_before(prev_v, prev_i, cv[m], ci[m]) && ranks_before(cv[m], ci[m], bv, bi)) {
        bv = cv[m];
        bi = ci[m];
      }
    for (int i = lane + 32 * kMergeRegs; i < ncand; i += 32) {   // large lists only
      const float v = __ldcg(vals + i);
      const int id = __ldcg(ids + i);
      if (id >= 0 && ranks_before(prev_v, prev_i, v, id) && ranks_before(v, id, bv, bi)) {
        bv = v;
        bi = id;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ranks_before(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      out_ids[r] = bi;
      out_vals[r] = bv;
    }
    prev_v = bv;
    prev_i = bi;
  }
}

// S4 for all B sequences from the final top-k (all threads of one CTA): the
// flat list [root, head 1 top-k, ..., head K top-k] gathered through
// tree_indices and retrieve, and the position ids.
__device__ __forceinline__ void build_tree_block(const TreeBuild& bd, int B, const int32_t* topk_ids) {
  const TreeDev& t = bd.t;
  const int per_b = 2 * t.T + t.P * (t.D + 1);
  for (int g = threadIdx.x; g < B * per_b; g += blockDim.x) {
    const int b = g / per_b;
    int o = g - b * per_b;
    auto flat = [&](int fi) -> int32_t {
      return fi == 0 ? bd.root_tokens[b] : __ldcg(topk_ids + (static_cast<size_t>(b) * t.K) * t.topk + (fi - 1));
    };
    if (o < t.T) {
      bd.tree_tokens[b * t.T + o] = flat(t.tree_indices[o]);
    } else if (o < 2 * t.T) {
      o -= t.T;
      bd.position_ids[b * t.T + o] = bd.seq_lens[b] + t.depth[o];
    } else {
      o -= 2 * t.T;
      const int node = t.retrieve[o];
      bd.candidates[static_cast<size_t>(b) * t.P * (t.D + 1) + o] = node < 0 ? -1 : flat(t.tree_indices[node]);
    }
  }
}

}  // namespace medusa
