// S6: evaluate the posterior of every candidate path and pick the best one
// ("Medusa API参考：核心函数与类详解", 核心功能函数: evaluate_posterior with
// posterior_threshold = 0.09 and posterior_alpha = 0.3 by default;
// "Medusa — 让大模型自己同时猜好几个 token", 核心要点: typical acceptance, and
// 实践案例 case 1 step 4: keep the longest acceptable prefix from the root).
//
// One kernel, one CTA of 1024 threads per (sequence, tree node): the node's
// V base logits are loaded once into registers (8 float4 per thread, all in
// flight together), giving the arg-max (lower id on ties) and, for typical
// acceptance, the tempered softmax statistics
//     m = max z/T,  S = sum exp(z/T - m),  E = sum exp(z/T - m) (z/T - m)
// so that H = ln S - E / S and thr = min(eps, alpha exp(-H)).
// The last CTA of a sequence to finish (a self-resetting counter in the
// workspace) then walks every path from the root with one thread per path,
// counts the leading accepted depths, reduces (max count, lowest path index)
// and writes the step's outputs.
#include <cfloat>

#include "common.cuh"

namespace medusa {
namespace {

constexpr int kThreads = 1024;
constexpr int kVecPerThread = 8;          // float4 per thread held in registers per chunk
constexpr int kChunk = kThreads * kVecPerThread * 4;   // logits per chunk (32768)

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

// Block-wide reductions through a 32-entry shared array (all threads call).
__device__ __forceinline__ void block_argmax(float& v, int& i, float* sv, int* si) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    argmax_merge(v, i, __shfl_xor_sync(0xffffffffu, v, o), __shfl_xor_sync(0xffffffffu, i, o));
  if (lane == 0) {
    sv[warp] = v;
    si[warp] = i;
  }
  __syncthreads();
  v = sv[lane];
  i = si[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    argmax_merge(v, i, __shfl_xor_sync(0xffffffffu, v, o), __shfl_xor_sync(0xffffffffu, i, o));
  __syncthreads();
}

__device__ __forceinline__ void block_sum2(float& a, float& b, float* sa, float* sb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (lane == 0) {
    sa[warp] = a;
    sb[warp] = b;
  }
  __syncthreads();
  a = 0.f;
  b = 0.f;
  if (threadIdx.x == 0)
    for (int w = 0; w < kThreads / 32; ++w) {   // fixed order
      a += sa[w];
      b += sb[w];
    }
  __syncthreads();
}

// Loads logits c0 + 4 (tid + i kThreads) + j of row z into c[i] (-inf past
// V): 16-byte loads when the row allows them, else one value at a time.
__device__ __forceinline__ void load_chunk(const float* z, int V, int c0, bool vec, float4 (&c)[kVecPerThread]) {
#pragma unroll
  for (int i = 0; i < kVecPerThread; ++i) {
    const int v0 = c0 + 4 * (threadIdx.x + i * kThreads);
    if (vec) {
      c[i] = v0 < V ? __ldg(reinterpret_cast<const float4*>(z + v0))
                    : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    } else {
      c[i].x = v0 < V ? __ldg(z + v0) : -INFINITY;
      c[i].y = v0 + 1 < V ? __ldg(z + v0 + 1) : -INFINITY;
      c[i].z = v0 + 2 < V ? __ldg(z + v0 + 2) : -INFINITY;
      c[i].w = v0 + 3 < V ? __ldg(z + v0 + 3) : -INFINITY;
    }
  }
}

__global__ void __launch_bounds__(kThreads) posterior_kernel(
    const TreeDev t, int V, const float* __restrict__ logits, const int32_t* __restrict__ candidates, int typical,
    float temperature, float eps, float alpha, NodeStat* stats, unsigned* counters, int32_t* __restrict__ best_path,
    int32_t* __restrict__ accept_len, int32_t* __restrict__ accepted_tokens, int32_t* __restrict__ next_token,
    int* status) {
  __shared__ float red_v[32], red_s[32];
  __shared__ int red_i[32];
  __shared__ int s_last;
  allow_dependents();
  const int row = blockIdx.x;           // b * T + node
  const int b = row / t.T;
  const float* z = logits + static_cast<size_t>(row) * V;
  const int tid = threadIdx.x;

  // ---- node statistics
  const bool vec = (V % 4) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
  float4 c[kVecPerThread];
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  const bool one_chunk = V <= kChunk;
  for (int c0 = 0; c0 < V; c0 += kChunk) {
    load_chunk(z, V, c0, vec, c);
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
      const int v0 = c0 + 4 * (tid + i * kThreads);
      argmax_merge(bv, bi, c[i].x, v0);
      argmax_merge(bv, bi, c[i].y, v0 + 1);
      argmax_merge(bv, bi, c[i].z, v0 + 2);
      argmax_merge(bv, bi, c[i].w, v0 + 3);
    }
  }
  block_argmax(bv, bi, red_v, red_i);
  if (!typical) {
    if (tid == 0) stats[row] = NodeStat{bi, 0.f, 0.f, 0.f};
  } else {
    // m = max(z / T) = max(z) / T for T > 0 (division is monotone).
    const float m = bv / temperature;
    float s = 0.f, e = 0.f;
    for (int c0 = 0; c0 < V; c0 += kChunk) {
      if (!one_chunk) load_chunk(z, V, c0, vec, c);
#pragma unroll
      for (int i = 0; i < kVecPerThread; ++i) {
        const float zz[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (zz[j] != -INFINITY) {   // past the row's end (or a zero-probability logit)
            const float y = zz[j] / temperature - m;
            const float pp = expf(y);
            s += pp;
            e = fmaf(pp, y, e);
          }
        }
      }
    }
    block_sum2(s, e, red_s, red_v);
    if (tid == 0) {
      const float H = logf(s) - e / s;
      const float thr = fminf(eps, alpha * expf(-H));
      stats[row] = NodeStat{bi, m, s, thr};
    }
  }

  // ---- the last node of sequence b to finish evaluates the paths (the
  // candidates come from an earlier kernel of the step)
  wait_prior_grids();
  if (tid == 0) {
    __threadfence();
    const unsigned done = atom_add_acq_rel_gpu(&counters[b], 1u);
    s_last = done == static_cast<unsigned>(t.T - 1);
    if (s_last) counters[b] = 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int D1 = t.D + 1;
  const int p = tid;
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
      const NodeStat* sp = stats + b * t.T + par;
      bool ok;
      if (!typical) {
        ok = tok == __ldcg(&sp->argmax);
      } else {
        const float y = logits[(static_cast<size_t>(b) * t.T + par) * V + tok] / temperature - __ldcg(&sp->m);
        ok = expf(y) / __ldcg(&sp->S) > __ldcg(&sp->thr);
      }
      if (!ok) break;
      ++acc;
    }
  }
  // (max acc, then lowest p)
  float av = static_cast<float>(acc);
  int ap = p;
  // ranks_before orders by larger value, then lower index: exactly (max acc, lowest p).
  block_argmax(av, ap, red_v, red_i);
  const int ba = static_cast<int>(av), bp = ap;
  if (tid == 0) {
    best_path[b] = bp;
    accept_len[b] = ba;
    const int last = t.retrieve[bp * D1 + ba];
    next_token[b] = __ldcg(&stats[b * t.T + last].argmax);
  }
  for (int j = tid; j < D1; j += blockDim.x)
    accepted_tokens[b * D1 + j] = j <= ba ? candidates[(static_cast<size_t>(b) * t.P + bp) * D1 + j] : -1;
}

}  // namespace

size_t posterior_workspace_bytes(const TreeDev& t, int B) {
  return align_up(static_cast<size_t>(B) * t.T * sizeof(NodeStat), 256) +
         align_up(static_cast<size_t>(B) * sizeof(unsigned), 256);
}

medusa_status_t launch_posterior(const TreeDev& t, int B, int V, const float* logits,
                                 const int32_t* candidates, medusa_mode_t mode, float temperature,
                                 float eps, float alpha, int32_t* best_path, int32_t* accept_len,
                                 int32_t* accepted_tokens, int32_t* next_token, void* ws,
                                 cudaStream_t stream, bool pdl) {
  if (t.P > kThreads) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_evaluate_posterior: more than 1024 paths");
  NodeStat* stats = static_cast<NodeStat*>(ws);
  unsigned* counters = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(ws) +
                                                   align_up(static_cast<size_t>(B) * t.T * sizeof(NodeStat), 256));
  const int typical = mode == MEDUSA_TYPICAL ? 1 : 0;
  const cudaError_t e = launch_kernel(posterior_kernel, dim3(B * t.T), dim3(kThreads), 0, stream, pdl, t, V, logits,
                                     candidates, typical, temperature, eps, alpha, stats, counters, best_path,
                                     accept_len, accepted_tokens, next_token, device_status_ptr());
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_evaluate_posterior: launch", e);
}

}  // namespace medusa
