// S6: evaluate the posterior of every candidate path and pick the best one
// ("Medusa API参考：核心函数与类详解", 核心功能函数: evaluate_posterior with
// posterior_threshold = 0.09, posterior_alpha = 0.3, top_p = 0.8 and
// sampling = 'typical' by default; "Medusa — 让大模型自己同时猜好几个 token",
// 核心要点: typical acceptance, and 实践案例 case 1 step 4: keep the longest
// acceptable prefix from the root), and inside medusa_step also S7 (keep the
// accepted path's K/V; 实践案例 case 1 step 4) in the same launch.
//
// One kernel of 1024-thread CTAs.  Each CTA takes a ticket when it starts:
//  * tickets 0 .. B*T-1 are tree nodes.  The node's V base logits are loaded
//    once into registers (8 float4 per thread, all in flight together),
//    giving the arg-max (lower id on ties) and the tempered softmax
//    statistics  m = max z/T,  S = sum exp(z/T - m),  E = sum exp(z/T - m)(z/T - m),
//    so that H = ln S - E/S and thr = min(eps, alpha exp(-H)).  In nucleus
//    mode the node also decides, for each child, whether the child's token
//    lies in its top-p nucleus: the tempered mass of the tokens that rank
//    before it (larger logit, or equal logit and lower id) must stay below
//    top_p * S.  The last node of a sequence to finish (a self-resetting
//    counter) walks every path from the root with one thread per path,
//    counts the leading accepted depths, reduces (max count, lowest path
//    index), writes the step's outputs and, given a uniform per sequence,
//    draws the next token by inverse CDF in token-id order from the last
//    accepted node's tempered distribution (or its nucleus).
//  * with the compaction on (medusa_step), tickets from B*T on move the
//    accepted rows: each waits (bounded) until every sequence's walk has
//    published (L, a, best path), then copies cache rows L+n_j -> L+j for
//    j = 0..a of its share of the (layer, sequence, head) slices, K and V.
//    The walk also advances seq_lens.
// Tickets are handed out in the order CTAs start, so every node ticket is
// held by a running CTA before any compaction CTA begins to wait: the wait
// always ends, whatever the number of resident CTAs.
#include <cfloat>

#include "common.cuh"

namespace medusa {
namespace {

constexpr int kThreads = 1024;
constexpr int kVecPerThread = 8;          // float4 per thread held in registers per chunk
constexpr int kChunk = kThreads * kVecPerThread * 4;   // logits per chunk (32768)
constexpr int kChildBatch = 4;            // children whose nucleus mass one pass accumulates
constexpr int kMaxRowsInFlight = 4;       // compaction rows loaded before they are stored

struct NodeStat {
  int argmax;
  float m;
  float S;
  float thr;
};

struct PostArgs {
  TreeDev t;
  int B, V;
  const float* logits;         // [B, T, V]
  const int32_t* candidates;   // [B, P, D+1]
  int mode;                    // MEDUSA_GREEDY / MEDUSA_TYPICAL / MEDUSA_NUCLEUS
  float temperature, eps, alpha, top_p;
  const float* uniforms;       // [B] or null: next token by arg-max
  NodeStat* stats;             // workspace [B*T]
  int32_t* edge_ok;            // workspace [B*T]: node's token lies in its parent's nucleus
  unsigned* done;              // workspace [B]: nodes finished per sequence
  unsigned* ctrs;              // workspace [2]: [0] ticket, [1] CTAs exited
  int32_t* best_path;
  int32_t* accept_len;
  int32_t* accepted_tokens;
  int32_t* next_token;
  int* status;
  // S7 (medusa_step only; n_comp = 0 turns it off)
  int n_comp;                  // compaction CTAs
  int layers, H, chunks, Lcap; // chunks: 16-byte columns per cache row
  uint4* k_cache;
  uint4* v_cache;
  int32_t* seq_lens;           // [B], advanced by a+1
  int* walk;                   // workspace [B][3]: L, a (-1: skipped), best path
  unsigned* ready;             // workspace [B]: walk published
};

struct Shared {
  float red_v[32 * (kChildBatch + 1)];
  float red_scan[64];
  int red_i[32];
  int kids[MEDUSA_MAX_TOPK];      // a node has at most topk children
  int kid_tok[MEDUSA_MAX_TOPK];
  int n_kids;
  int flag;
  int best, acc;
  int walk[3 * MEDUSA_MAX_B];
};

__device__ __forceinline__ void argmax_merge(float& v, int& i, float ov, int oi) {
  if (ranks_before(ov, oi, v, i)) {
    v = ov;
    i = oi;
  }
}

// Block-wide reductions through shared arrays (all threads call).
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

// Sums N values over the block in a fixed order; every thread receives the totals.
template <int N>
__device__ __forceinline__ void block_sum(float (&v)[N], float* red /* [32 * (N + 1)] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) red[warp * N + i] = v[i];
  __syncthreads();
  if (threadIdx.x < N) {
    float s = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) s += red[w * N + threadIdx.x];
    red[32 * N + threadIdx.x] = s;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = red[32 * N + i];
  __syncthreads();
}

// Exclusive prefix over threads (in thread order) of one value per thread;
// returns the exclusive prefix of this thread.  Fixed order.
__device__ __forceinline__ float block_exclusive_scan(float x, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    float w = red[lane];
    float wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    red[32 + lane] = wi - w;   // exclusive prefix of warp totals
  }
  __syncthreads();
  const float r = red[32 + warp] + incl - x;
  __syncthreads();
  return r;
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

__device__ __forceinline__ float comp(const float4& c, int j) {
  return j == 0 ? c.x : (j == 1 ? c.y : (j == 2 ? c.z : c.w));
}

// Node statistics of row `row` = b*T + node, and (nucleus) the nucleus
// membership of each child's token.  All threads.  kMode is a.mode.
template <int kMode>
__device__ void node_phase(const PostArgs& a, int row, Shared& sh) {
  const TreeDev& t = a.t;
  const int V = a.V, tid = threadIdx.x;
  const int b = row / t.T, node = row - b * t.T;
  const float* z = a.logits + static_cast<size_t>(row) * V;
  const bool vec = (V % 4) == 0 && (reinterpret_cast<uintptr_t>(a.logits) & 15) == 0;
  const bool one_chunk = V <= kChunk;
  float4 c[kVecPerThread];
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int c0 = 0; c0 < V; c0 += kChunk) {
    load_chunk(z, V, c0, vec, c);
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
      const int v0 = c0 + 4 * (tid + i * kThreads);
#pragma unroll
      for (int j = 0; j < 4; ++j) argmax_merge(bv, bi, comp(c[i], j), v0 + j);
    }
  }
  block_argmax(bv, bi, sh.red_v, sh.red_i);
  if constexpr (kMode == MEDUSA_GREEDY) {
    if (tid == 0) a.stats[row] = NodeStat{bi, 0.f, 0.f, 0.f};
    return;
  }
  // m = max(z / T) = max(z) / T for T > 0 (division is monotone).
  const float m = bv / a.temperature;
  float se[2] = {0.f, 0.f};
  for (int c0 = 0; c0 < V; c0 += kChunk) {
    if (!one_chunk) load_chunk(z, V, c0, vec, c);
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float zz = comp(c[i], j);
        if (zz != -INFINITY) {   // past the row's end (or a zero-probability logit)
          const float y = zz / a.temperature - m;
          const float pp = expf(y);
          se[0] += pp;
          se[1] = fmaf(pp, y, se[1]);
        }
      }
  }
  block_sum<2>(se, sh.red_v);
  const float S = se[0];
  if (tid == 0) {
    const float H = logf(S) - se[1] / S;
    a.stats[row] = NodeStat{bi, m, S, fminf(a.eps, a.alpha * expf(-H))};
  }
  if constexpr (kMode != MEDUSA_NUCLEUS) return;

  // Nucleus membership of each child's token (the tokens come from an
  // earlier kernel of the step).
  wait_prior_grids();
  const int D1 = t.D + 1;
  if (tid == 0) {
    int n = 0;
    for (int k = node + 1; k < t.T && n < MEDUSA_MAX_TOPK; ++k)
      if (t.parent[k] == node) {
        sh.kids[n] = k;
        sh.kid_tok[n] = a.candidates[(static_cast<size_t>(b) * t.P + t.path_of[k]) * D1 + t.depth[k]];
        ++n;
      }
    sh.n_kids = n;
  }
  __syncthreads();
  const int n_kids = sh.n_kids;
  const float cut = a.top_p * S;
  for (int k0 = 0; k0 < n_kids; k0 += kChildBatch) {
    float zc[kChildBatch];
    int tc[kChildBatch];
#pragma unroll
    for (int q = 0; q < kChildBatch; ++q) {
      tc[q] = k0 + q < n_kids ? sh.kid_tok[k0 + q] : -1;
      zc[q] = (tc[q] >= 0 && tc[q] < V) ? __ldg(z + tc[q]) : INFINITY;   // a bad token: nothing ranks before it
    }
    float mass[kChildBatch] = {};
    for (int c0 = 0; c0 < V; c0 += kChunk) {
      if (!one_chunk) load_chunk(z, V, c0, vec, c);
#pragma unroll
      for (int i = 0; i < kVecPerThread; ++i) {
        const int v0 = c0 + 4 * (tid + i * kThreads);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float zz = comp(c[i], j);
          const float w = expf(zz / a.temperature - m);   // 0 past the row's end
#pragma unroll
          for (int q = 0; q < kChildBatch; ++q)
            if (zz > zc[q] || (zz == zc[q] && v0 + j < tc[q])) mass[q] += w;
        }
      }
    }
    block_sum<kChildBatch>(mass, sh.red_v);
    if (tid < kChildBatch && k0 + tid < n_kids) {
      float mq = mass[0];
#pragma unroll
      for (int q = 1; q < kChildBatch; ++q)
        if (q == tid) mq = mass[q];
      a.edge_ok[b * t.T + sh.kids[k0 + tid]] = mq < cut ? 1 : 0;
    }
  }
}

// Inverse-CDF draw of the next token at node `last` of sequence b (all
// threads): weights exp(z/T - m) in token-id order, restricted in nucleus mode
// to the tokens at or above the nucleus cut-off.  Every thread gets the token.
template <int kMode>
__device__ int draw_next(const PostArgs& a, int b, int last, float u, Shared& sh) {
  const int V = a.V, tid = threadIdx.x;
  const float* z = a.logits + (static_cast<size_t>(b) * a.t.T + last) * V;
  const bool vec = (V % 4) == 0 && (reinterpret_cast<uintptr_t>(a.logits) & 15) == 0;
  const bool one_chunk = V <= kChunk;
  // Written by another CTA of this launch; visible after the completion counter.
  const NodeStat* sp = a.stats + b * a.t.T + last;
  const float m = __ldcg(&sp->m), S = __ldcg(&sp->S);
  const int amax = __ldcg(&sp->argmax);
  float4 c[kVecPerThread];
  // Weights of one chunk, in place of the logits (w is monotone in z, so
  // comparing weights ranks tokens as the logits do).
  auto weights = [&](int c0) {
    load_chunk(z, V, c0, vec, c);
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
      c[i].x = expf(c[i].x / a.temperature - m);
      c[i].y = expf(c[i].y / a.temperature - m);
      c[i].z = expf(c[i].z / a.temperature - m);
      c[i].w = expf(c[i].w / a.temperature - m);
    }
  };
  if (one_chunk) weights(0);
  // Nucleus cut-off: the largest weight key t with sum(w : key(w) >= t) >= top_p * S
  // (bisection over the bit patterns of non-negative floats, which order like their values).
  uint32_t cut = 0;
  if constexpr (kMode == MEDUSA_NUCLEUS) {
    const float target = a.top_p * S;
    uint64_t lo = 0, hi = 0x80000000ull;   // mass(lo) >= target, mass(hi) < target
    while (hi - lo > 1) {
      const uint32_t mid = static_cast<uint32_t>((lo + hi) / 2);
      float s[1] = {0.f};
      for (int c0 = 0; c0 < V; c0 += kChunk) {
        if (!one_chunk) weights(c0);
#pragma unroll
        for (int i = 0; i < kVecPerThread; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float w = comp(c[i], j);
            if (__float_as_uint(w) >= mid) s[0] += w;
          }
      }
      block_sum<1>(s, sh.red_v);
      if (s[0] >= target) lo = mid; else hi = mid;
    }
    cut = static_cast<uint32_t>(lo);
  }
  auto keep = [&](float w) { return __float_as_uint(w) >= cut ? w : 0.f; };
  // Chunk totals, then the chunk holding u * total, then the thread and the token.
  float x = 0.f;
  int found = -1;
  float before = 0.f, tot_all = 0.f;
  {
    float tot[1] = {0.f};
    // total over every chunk
    for (int c0 = 0; c0 < V; c0 += kChunk) {
      if (!one_chunk) weights(c0);
#pragma unroll
      for (int i = 0; i < kVecPerThread; ++i) {
        tot[0] += keep(c[i].x);
        tot[0] += keep(c[i].y);
        tot[0] += keep(c[i].z);
        tot[0] += keep(c[i].w);
      }
    }
    block_sum<1>(tot, sh.red_v);
    tot_all = tot[0];
    x = u * tot_all;
  }
  // Walk the id order: chunk c0, group i, thread, component j.
  for (int c0 = 0; c0 < V && found < 0; c0 += kChunk) {
    if (!one_chunk) weights(c0);
    for (int i = 0; i < kVecPerThread && found < 0; ++i) {
      const float g = keep(c[i].x) + keep(c[i].y) + keep(c[i].z) + keep(c[i].w);
      const float ex = block_exclusive_scan(g, sh.red_scan);
      float grp[1] = {g};
      block_sum<1>(grp, sh.red_v);
      if (tid == 0) sh.flag = -1;
      __syncthreads();
      if (before + ex <= x && x < before + ex + g) {
        float cum = before + ex;
        int pick = -1;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float w = keep(comp(c[i], j));
          cum += w;
          if (pick < 0 && w > 0.f && cum > x) pick = c0 + 4 * (tid + i * kThreads) + j;
        }
        if (pick < 0) pick = c0 + 4 * (tid + i * kThreads) + 3;   // rounding at the group's end
        atomicMax(&sh.flag, pick);   // at most one thread's interval holds x; max keeps it deterministic
      }
      __syncthreads();
      found = sh.flag;
      before += grp[0];
      __syncthreads();
    }
  }
  if (found < 0 || found >= V) found = amax;   // u * total at the very end (rounding): the arg-max
  return found;
}

// The last CTA of sequence b walks the paths and writes the step's outputs.
template <int kMode>
__device__ void walk_paths(const PostArgs& a, int b, Shared& sh) {
  const TreeDev& t = a.t;
  const int tid = threadIdx.x, D1 = t.D + 1, V = a.V;
  const int p = tid;
  int acc = -1;  // threads without a path never win
  if (p < t.P) {
    acc = 0;
    const int32_t* cand = a.candidates + (static_cast<size_t>(b) * t.P + p) * D1;
    for (int j = 1; j <= t.D; ++j) {
      const int node = t.retrieve[p * D1 + j];
      if (node < 0) break;
      const int par = t.retrieve[p * D1 + j - 1];
      const int tok = cand[j];
      if (tok < 0 || tok >= V) {
        set_device_status(a.status, MEDUSA_ERR_DEVICE_CHECK, kDetailPosteriorArgs);
        break;
      }
      const NodeStat* sp = a.stats + b * t.T + par;
      bool ok;
      if constexpr (kMode == MEDUSA_GREEDY) {
        ok = tok == __ldcg(&sp->argmax);
      } else if constexpr (kMode == MEDUSA_TYPICAL) {
        const float y = a.logits[(static_cast<size_t>(b) * t.T + par) * V + tok] / a.temperature - __ldcg(&sp->m);
        ok = expf(y) / __ldcg(&sp->S) > __ldcg(&sp->thr);
      } else {
        ok = __ldcg(a.edge_ok + b * t.T + node) != 0;
      }
      if (!ok) break;
      ++acc;
    }
  }
  // (max acc, then lowest p): ranks_before orders by larger value, then lower index.
  float av = static_cast<float>(acc);
  int ap = p;
  block_argmax(av, ap, sh.red_v, sh.red_i);
  const int ba = static_cast<int>(av), bp = ap;
  const int last = t.retrieve[bp * D1 + ba];
  int nxt = __ldcg(&a.stats[b * t.T + last].argmax);
  if constexpr (kMode != MEDUSA_GREEDY) {
    if (a.uniforms != nullptr) nxt = draw_next<kMode>(a, b, last, __ldg(a.uniforms + b), sh);
  }
  if (tid == 0) {
    a.best_path[b] = bp;
    a.accept_len[b] = ba;
    a.next_token[b] = nxt;
    sh.best = bp;
    sh.acc = ba;
  }
  for (int j = tid; j < D1; j += blockDim.x)
    a.accepted_tokens[b * D1 + j] = j <= ba ? a.candidates[(static_cast<size_t>(b) * t.P + bp) * D1 + j] : -1;
  __syncthreads();
}

template <int kMode>
__global__ void __launch_bounds__(kThreads) posterior_kernel(const PostArgs a) {
  __shared__ Shared sh;
  __shared__ int s_ticket;
  allow_dependents();
  const TreeDev& t = a.t;
  const int tid = threadIdx.x;
  if (tid == 0) s_ticket = static_cast<int>(atomicAdd(&a.ctrs[0], 1u));
  __syncthreads();
  const int ticket = s_ticket;
  const int n_nodes = a.B * t.T;

  if (ticket < n_nodes) {
    // ---- a tree node
    node_phase<kMode>(a, ticket, sh);
    wait_prior_grids();   // candidates, and (with the compaction) attention done with the caches
    const int b = ticket / t.T;
    if (tid == 0) {
      __threadfence();
      const unsigned done = atom_add_acq_rel_gpu(&a.done[b], 1u);
      sh.flag = done == static_cast<unsigned>(t.T - 1);
      if (sh.flag) a.done[b] = 0u;
    }
    __syncthreads();
    if (sh.flag) {
      __threadfence();
      walk_paths<kMode>(a, b, sh);
      if (a.n_comp > 0 && tid == 0) {
        // Publish the walk for the compaction CTAs, then advance the length.
        const int L = a.seq_lens[b];
        int acc = sh.acc;
        if (L < 0 || L + t.T > a.Lcap) {
          set_device_status(a.status, MEDUSA_ERR_DEVICE_CHECK, kDetailAcceptSeqLen);
          acc = -1;
        }
        a.walk[3 * b] = L;
        a.walk[3 * b + 1] = acc;
        a.walk[3 * b + 2] = sh.best;
        if (acc >= 0) a.seq_lens[b] = L + acc + 1;
        __threadfence();
        atom_add_release_gpu(&a.ready[b], 1u);
      }
    }
  } else {
    // ---- compaction of the accepted rows (S7)
    wait_prior_grids();
    if (tid == 0) {
      int ok = 1;
      const uint64_t t0 = globaltimer_ns();
      for (int b = 0; b < a.B && ok; ++b) {
        while (ld_acquire_gpu(&a.ready[b]) == 0u) {
          if (globaltimer_ns() - t0 > kSpinLimitNs) {
            set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailPosteriorWait);
            ok = 0;
            break;
          }
          __nanosleep(256);
        }
      }
      for (int i = 0; ok && i < 3 * a.B; ++i) sh.walk[i] = __ldcg(a.walk + i);
      sh.flag = ok;
    }
    __syncthreads();
    if (sh.flag) {
      const int D1 = t.D + 1;
      const long long per_slice = 2ll * a.chunks;
      const long long total = static_cast<long long>(a.layers) * a.B * a.H * per_slice;
      for (long long g = static_cast<long long>(ticket - n_nodes) * kThreads + tid; g < total;
           g += static_cast<long long>(a.n_comp) * kThreads) {
        const long long slice = g / per_slice;
        const int rem = static_cast<int>(g - slice * per_slice);
        const int which = rem / a.chunks, col = rem - which * a.chunks;
        const int b = static_cast<int>((slice / a.H) % a.B);
        const int L = sh.walk[3 * b], acc = sh.walk[3 * b + 1], best = sh.walk[3 * b + 2];
        if (acc < 0) continue;
        uint4* base = (which == 0 ? a.k_cache : a.v_cache) + static_cast<size_t>(slice) * a.Lcap * a.chunks + col;
        const int32_t* path = t.retrieve + best * D1;
        // In increasing j: the source of j is row L+n_j with n_j >= j (a node's
        // index is at least its depth), so no destination written earlier is a
        // source read later; a batch loads its sources before its stores.
        for (int j0 = 0; j0 <= acc; j0 += kMaxRowsInFlight) {
          uint4 r[kMaxRowsInFlight];
#pragma unroll
          for (int q = 0; q < kMaxRowsInFlight; ++q) {
            const int j = j0 + q;
            if (j <= acc && path[j] != j) r[q] = base[static_cast<size_t>(L + path[j]) * a.chunks];
          }
#pragma unroll
          for (int q = 0; q < kMaxRowsInFlight; ++q) {
            const int j = j0 + q;
            if (j <= acc && path[j] != j) base[static_cast<size_t>(L + j) * a.chunks] = r[q];
          }
        }
      }
    }
  }

  // The last CTA to leave resets the ticket and the walk flags for the next call.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned left = atom_add_acq_rel_gpu(&a.ctrs[1], 1u);
    if (left == gridDim.x - 1) {
      a.ctrs[0] = 0u;
      a.ctrs[1] = 0u;
      if (a.n_comp > 0)
        for (int b = 0; b < a.B; ++b) a.ready[b] = 0u;
      __threadfence();
    }
  }
}

struct PostLayout {
  size_t stats, edge_ok, done, ctrs, walk, ready, total;
};

PostLayout post_layout(const TreeDev& t, int B) {
  PostLayout l{};
  size_t o = 0;
  l.stats = o;
  o += align_up(static_cast<size_t>(B) * t.T * sizeof(NodeStat), 256);
  l.edge_ok = o;
  o += align_up(static_cast<size_t>(B) * t.T * sizeof(int32_t), 256);
  l.done = o;
  o += align_up(static_cast<size_t>(B) * sizeof(unsigned), 256);
  l.ctrs = o;
  o += 256;
  l.walk = o;
  o += align_up(static_cast<size_t>(B) * 3 * sizeof(int), 256);
  l.ready = o;
  o += align_up(static_cast<size_t>(B) * sizeof(unsigned), 256);
  l.total = o;
  return l;
}

cudaError_t launch_mode(const PostArgs& a, int grid, cudaStream_t stream, bool pdl) {
  if (a.mode == MEDUSA_GREEDY)
    return launch_kernel(posterior_kernel<MEDUSA_GREEDY>, dim3(grid), dim3(kThreads), 0, stream, pdl, a);
  if (a.mode == MEDUSA_TYPICAL)
    return launch_kernel(posterior_kernel<MEDUSA_TYPICAL>, dim3(grid), dim3(kThreads), 0, stream, pdl, a);
  return launch_kernel(posterior_kernel<MEDUSA_NUCLEUS>, dim3(grid), dim3(kThreads), 0, stream, pdl, a);
}

PostArgs post_args(const TreeDev& t, int B, int V, const float* logits, const int32_t* candidates, medusa_mode_t mode,
                   float temperature, float eps, float alpha, float top_p, const float* uniforms, int32_t* best_path,
                   int32_t* accept_len, int32_t* accepted_tokens, int32_t* next_token, void* ws) {
  const PostLayout l = post_layout(t, B);
  unsigned char* w = static_cast<unsigned char*>(ws);
  PostArgs a{};
  a.t = t;
  a.B = B;
  a.V = V;
  a.logits = logits;
  a.candidates = candidates;
  a.mode = static_cast<int>(mode);
  a.temperature = temperature;
  a.eps = eps;
  a.alpha = alpha;
  a.top_p = top_p;
  a.uniforms = uniforms;
  a.stats = reinterpret_cast<NodeStat*>(w + l.stats);
  a.edge_ok = reinterpret_cast<int32_t*>(w + l.edge_ok);
  a.done = reinterpret_cast<unsigned*>(w + l.done);
  a.ctrs = reinterpret_cast<unsigned*>(w + l.ctrs);
  a.walk = reinterpret_cast<int*>(w + l.walk);
  a.ready = reinterpret_cast<unsigned*>(w + l.ready);
  a.best_path = best_path;
  a.accept_len = accept_len;
  a.accepted_tokens = accepted_tokens;
  a.next_token = next_token;
  a.status = device_status_ptr();
  return a;
}

}  // namespace

size_t posterior_workspace_bytes(const TreeDev& t, int B) { return post_layout(t, B).total; }

medusa_status_t launch_posterior(const TreeDev& t, int B, int V, const float* logits,
                                 const int32_t* candidates, medusa_mode_t mode, float temperature,
                                 float eps, float alpha, float top_p, const float* uniforms, int32_t* best_path,
                                 int32_t* accept_len, int32_t* accepted_tokens, int32_t* next_token, void* ws,
                                 cudaStream_t stream, bool pdl) {
  if (t.P > kThreads) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_evaluate_posterior: more than 1024 paths");
  const PostArgs a = post_args(t, B, V, logits, candidates, mode, temperature, eps, alpha, top_p, uniforms, best_path,
                               accept_len, accepted_tokens, next_token, ws);
  const cudaError_t e = launch_mode(a, B * t.T, stream, pdl);
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_evaluate_posterior: launch", e);
}

medusa_status_t launch_posterior_accept(const TreeDev& t, int B, int V, const float* logits,
                                        const int32_t* candidates, medusa_mode_t mode, float temperature, float eps,
                                        float alpha, float top_p, const float* uniforms, int32_t* best_path,
                                        int32_t* accept_len, int32_t* accepted_tokens, int32_t* next_token,
                                        int layers, int H, int hd, medusa_dtype_t dtype, void* k_cache,
                                        void* v_cache, int Lcap, int32_t* seq_lens, void* ws, cudaStream_t stream,
                                        bool pdl) {
  if (t.P > kThreads) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_step: more than 1024 paths");
  PostArgs a = post_args(t, B, V, logits, candidates, mode, temperature, eps, alpha, top_p, uniforms, best_path,
                         accept_len, accepted_tokens, next_token, ws);
  const int row_bytes = hd * (dtype == MEDUSA_BF16 ? 2 : 4);
  a.chunks = row_bytes / 16;
  a.layers = layers;
  a.H = H;
  a.Lcap = Lcap;
  a.k_cache = static_cast<uint4*>(k_cache);
  a.v_cache = static_cast<uint4*>(v_cache);
  a.seq_lens = seq_lens;
  const long long threads = static_cast<long long>(layers) * B * H * 2 * a.chunks;
  const long long want = (threads + kThreads - 1) / kThreads;
  const long long cap = 2ll * (sm_count() > 0 ? sm_count() : 1);
  a.n_comp = static_cast<int>(want < cap ? want : cap);
  const cudaError_t e = launch_mode(a, B * t.T + a.n_comp, stream, pdl);
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_step: posterior and compaction launch", e);
}

}  // namespace medusa
