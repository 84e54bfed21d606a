// S6: evaluate the posterior of every candidate path and pick the best one
// ("Medusa API参考：核心函数与类详解", 核心功能函数: evaluate_posterior with
// posterior_threshold = 0.09 and posterior_alpha = 0.3 by default;
// "Medusa — 让大模型自己同时猜好几个 token", 核心要点: typical acceptance, and
// 实践案例 case 1 step 4: keep the longest acceptable prefix from the root).
//
// Kernel 1, one CTA per (sequence, tree node): one pass over the node's V
// base logits for the arg-max (lower id on ties) and, for typical
// acceptance, a second pass for the tempered softmax statistics
//     m = max z/T,  S = sum exp(z/T - m),  E = sum exp(z/T - m) (z/T - m)
// so that H = ln S - E / S and thr = min(eps, alpha exp(-H)).
// Kernel 2, one CTA per sequence, one thread per path: walk the path from
// the root, count the leading accepted depths, then reduce (max count,
// lowest path index) and write the step's outputs.
#include <cfloat>

#include "common.cuh"

namespace medusa {
namespace {

constexpr int kStatThreads = 256;

struct NodeStat {
  int argmax;
  float m;
  float S;
  float thr;
};

__device__ __forceinline__ void argmax_merge(float& v, int& i, float ov, int oi) {
  if (ranks_before(ov, oi, v, i)) {
    v = ov;
    i = oi;
  }
}

__global__ void __launch_bounds__(kStatThreads) node_stats_kernel(const float* __restrict__ logits, int V,
                                                                  int typical, float inv_t_unused,
                                                                  float temperature, float eps, float alpha,
                                                                  NodeStat* __restrict__ stats) {
  (void)inv_t_unused;
  const int row = blockIdx.x;
  const float* z = logits + static_cast<size_t>(row) * V;
  __shared__ float red_v[kStatThreads / 32];
  __shared__ int red_i[kStatThreads / 32];
  __shared__ float red_s[kStatThreads / 32], red_e[kStatThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  float bv = -FLT_MAX;
  int bi = 0x7fffffff;
  const bool vec_ok = (V % 4) == 0 && (reinterpret_cast<uintptr_t>(z) & 15) == 0;
  if (vec_ok) {
    const float4* z4 = reinterpret_cast<const float4*>(z);
    for (int q = tid; q < V / 4; q += blockDim.x) {
      const float4 c = __ldg(z4 + q);
      argmax_merge(bv, bi, c.x, 4 * q);
      argmax_merge(bv, bi, c.y, 4 * q + 1);
      argmax_merge(bv, bi, c.z, 4 * q + 2);
      argmax_merge(bv, bi, c.w, 4 * q + 3);
    }
  } else {
    for (int v = tid; v < V; v += blockDim.x) argmax_merge(bv, bi, __ldg(z + v), v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    argmax_merge(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
  if (lane == 0) {
    red_v[warp] = bv;
    red_i[warp] = bi;
  }
  __syncthreads();
  if (warp == 0) {
    bv = lane < (int)(blockDim.x / 32) ? red_v[lane] : -FLT_MAX;
    bi = lane < (int)(blockDim.x / 32) ? red_i[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      argmax_merge(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
    if (lane == 0) {
      red_v[0] = bv;
      red_i[0] = bi;
    }
  }
  __syncthreads();
  const float zmax = red_v[0];
  const int amax = red_i[0];
  if (!typical) {
    if (tid == 0) stats[row] = NodeStat{amax, 0.f, 0.f, 0.f};
    return;
  }
  // m = max(z / T) = max(z) / T for T > 0 (division is monotone).
  const float m = zmax / temperature;
  float s = 0.f, e = 0.f;
  for (int v = tid; v < V; v += blockDim.x) {
    const float y = __ldg(z + v) / temperature - m;
    const float p = expf(y);
    s += p;
    e = fmaf(p, y, e);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    e += __shfl_xor_sync(0xffffffffu, e, o);
  }
  __syncthreads();
  if (lane == 0) {
    red_s[warp] = s;
    red_e[warp] = e;
  }
  __syncthreads();
  if (tid == 0) {
    float S = 0.f, Es = 0.f;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
      S += red_s[w];
      Es += red_e[w];
    }
    const float H = logf(S) - Es / S;
    const float thr = fminf(eps, alpha * expf(-H));
    stats[row] = NodeStat{amax, m, S, thr};
  }
}

__global__ void paths_kernel(const TreeDev t, int V, const float* __restrict__ logits,
                             const int32_t* __restrict__ candidates, const NodeStat* __restrict__ stats,
                             int typical, float temperature, int32_t* __restrict__ best_path,
                             int32_t* __restrict__ accept_len, int32_t* __restrict__ accepted_tokens,
                             int32_t* __restrict__ next_token, int* status) {
  const int b = blockIdx.x;
  const int p = threadIdx.x;
  const int D1 = t.D + 1;
  __shared__ int red_a[32], red_p[32];
  __shared__ int s_best, s_a;
  int acc = -1;  // threads without a path never win
  if (p < t.P) {
    acc = 0;
    const int32_t* cand = candidates + (static_cast<size_t>(b) * t.P + p) * D1;
    for (int j = 1; j <= t.D; ++j) {
      const int node = t.retrieve[p * D1 + j];
      if (node < 0) break;
      const int par = t.retrieve[p * D1 + j - 1];
      const int tok = cand[j];
      if (tok < 0 || tok >= V) {
        set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailPosteriorArgs);
        break;
      }
      const NodeStat st = stats[b * t.T + par];
      bool ok;
      if (!typical) {
        ok = tok == st.argmax;
      } else {
        const float y = logits[(static_cast<size_t>(b) * t.T + par) * V + tok] / temperature - st.m;
        ok = expf(y) / st.S > st.thr;
      }
      if (!ok) break;
      ++acc;
    }
  }
  // (max acc, then lowest p)
  int ba = acc, bp = p;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const int oa = __shfl_xor_sync(0xffffffffu, ba, o);
    const int op = __shfl_xor_sync(0xffffffffu, bp, o);
    if (oa > ba || (oa == ba && op < bp)) {
      ba = oa;
      bp = op;
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  if (lane == 0) {
    red_a[warp] = ba;
    red_p[warp] = bp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < nw; ++w)
      if (red_a[w] > ba || (red_a[w] == ba && red_p[w] < bp)) {
        ba = red_a[w];
        bp = red_p[w];
      }
    s_best = bp;
    s_a = ba;
    best_path[b] = bp;
    accept_len[b] = ba;
    const int last = t.retrieve[bp * D1 + ba];
    next_token[b] = stats[b * t.T + last].argmax;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < D1; j += blockDim.x)
    accepted_tokens[b * D1 + j] =
        j <= s_a ? candidates[(static_cast<size_t>(b) * t.P + s_best) * D1 + j] : -1;
}

}  // namespace

size_t posterior_workspace_bytes(const TreeDev& t, int B) {
  return align_up(static_cast<size_t>(B) * t.T * sizeof(NodeStat), 256);
}

medusa_status_t launch_posterior(const TreeDev& t, int B, int V, const float* logits,
                                 const int32_t* candidates, medusa_mode_t mode, float temperature,
                                 float eps, float alpha, int32_t* best_path, int32_t* accept_len,
                                 int32_t* accepted_tokens, int32_t* next_token, void* ws,
                                 cudaStream_t stream) {
  NodeStat* stats = static_cast<NodeStat*>(ws);
  const int typical = mode == MEDUSA_TYPICAL ? 1 : 0;
  node_stats_kernel<<<B * t.T, kStatThreads, 0, stream>>>(logits, V, typical, 0.f, temperature, eps, alpha,
                                                          stats);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("medusa_evaluate_posterior: stats launch", e);
  const int threads = ((t.P + 31) / 32) * 32;
  paths_kernel<<<B, threads, 0, stream>>>(t, V, logits, candidates, stats, typical, temperature, best_path,
                                          accept_len, accepted_tokens, next_token, device_status_ptr());
  e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_evaluate_posterior: paths launch", e);
}

}  // namespace medusa
