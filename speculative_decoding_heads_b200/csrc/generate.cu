// Medusa generation of one sequence on the GPU (greedy, typical or nucleus
// acceptance, as medusa_evaluate_posterior): the loop of
// "Medusa API参考：核心函数与类详解" (MedusaModelABC, medusa_generate: each step
// proposes with the heads, verifies the tree with one base-model forward and
// keeps the accepted prefix) and "Medusa — 让大模型自己同时猜好几个 token"
// (实践案例 case 1: read the hidden state, guess with the heads, verify the
// tree in one forward, keep the longest acceptable prefix; 学到什么: every
// step also yields the base model's own next token).
//
// The prompt is run through the base model in chains of at most 17 tokens
// (a chain is a tree whose nodes each have one child).  Then, per step:
//   heads on h (the final-norm hidden state of the last accepted token) and
//   the candidate tree rooted at the base model's next token (one launch);
//   the base model's forward over the tree tokens at the cache length, which
//   writes the tree's K/V rows into the cache;
//   acceptance with the compaction of the accepted rows (one launch; the
//   next token drawn with the step's uniform when the caller gives them);
//   h for the next step: the final-norm row of the last accepted node.
// The host reads the accept length and the accepted tokens after each step.
#include <vector>

#include "common.cuh"

namespace medusa {
namespace {

constexpr int kChain = 17;   // longest chain of prompt tokens per forward (MEDUSA_MAX_K + 1)

__global__ void set_len_kernel(int32_t* seq_lens, int L) { seq_lens[0] = L; }

// h = the final-norm row `row` of the forward's output, where row is the last
// accepted node (retrieve[best, a]) or `fixed_row`; with root set, also the
// arg-max of that row's logits (lower id on ties).  One CTA of 256 threads.
__global__ void next_input_kernel(const uint16_t* rows, const float* logits, int D, int V, int fixed_row,
                                  const int32_t* retrieve, int P, int dp1, const int32_t* best, const int32_t* alen,
                                  uint16_t* h, int32_t* root, int* status) {
  __shared__ float sv[8];
  __shared__ int si[8];
  int row = fixed_row;
  if (retrieve) {
    const int bp = best[0], a = alen[0];
    row = (bp >= 0 && bp < P && a >= 0 && a < dp1) ? retrieve[bp * dp1 + a] : -1;
    if (row < 0) {   // the step's outputs are not a path: leave h alone
      if (threadIdx.x == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailPosteriorArgs);
      return;
    }
  }
  for (int i = threadIdx.x; i < D; i += blockDim.x) h[i] = rows[static_cast<size_t>(row) * D + i];
  if (!root) return;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  const float* z = logits + static_cast<size_t>(row) * V;
  for (int v = threadIdx.x; v < V; v += blockDim.x)
    if (z[v] > bv) {   // increasing v per thread: the first maximum wins
      bv = z[v];
      bi = v;
    }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) {
      bv = ov;
      bi = oi;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    sv[threadIdx.x >> 5] = bv;
    si[threadIdx.x >> 5] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w)
      if (sv[w] > bv || (sv[w] == bv && si[w] < bi)) {
        bv = sv[w];
        bi = si[w];
      }
    // bv/bi of thread 0 started as warp 0's result
    root[0] = bi;
  }
}

struct GenLayout {
  size_t dec, heads, post, tokens, pos, cand, ids, vals, logits, h, small, total;
};

GenLayout gen_layout(const medusa_tree_t* tree, const medusa_decoder_t* m) {
  GenLayout l{};
  const int T = tree->T > kChain ? tree->T : kChain;
  size_t o = 0;
  auto take = [&](size_t n) {
    const size_t at = o;
    o += align_up(n, 256);
    return at;
  };
  const size_t dec_a = decoder_workspace_bytes(tree->T, m->D, m->F, m->V);
  const size_t dec_b = decoder_workspace_bytes(kChain, m->D, m->F, m->V);
  l.dec = take(dec_a > dec_b ? dec_a : dec_b);
  l.heads = take(heads_workspace_bytes(1, m->D, m->V, tree->K, tree->topk));
  l.post = take(posterior_workspace_bytes(tree->dev, 1));
  l.tokens = take(static_cast<size_t>(T) * 4);
  l.pos = take(static_cast<size_t>(T) * 4);
  l.cand = take(static_cast<size_t>(tree->P) * (tree->D + 1) * 4);
  l.ids = take(static_cast<size_t>(tree->K) * tree->topk * 4);
  l.vals = take(static_cast<size_t>(tree->K) * tree->topk * 4);
  l.logits = take(static_cast<size_t>(T) * m->V * 4);
  l.h = take(static_cast<size_t>(m->D) * 2);
  l.small = take(static_cast<size_t>(8 + tree->D + 1) * 4);   // root, seq_len, best, alen, uniform, -, accepted tokens
  l.total = o;
  return l;
}

// The chain tree of n tokens (n - 1 nodes, node i the rank tuple of i zeros).
medusa_status_t chain_tree(int n, medusa_tree_t** out) {
  const int nodes = n - 1, K = nodes > 0 ? nodes : 1;
  std::vector<int32_t> ranks(static_cast<size_t>(nodes > 0 ? nodes : 1) * K, 0), lens(nodes > 0 ? nodes : 1, 0);
  for (int i = 0; i < nodes; ++i) lens[i] = i + 1;
  return medusa_tree_create(ranks.data(), lens.data(), nodes, K, 1, 1, out);
}

struct TreeGuard {
  medusa_tree_t* t = nullptr;
  ~TreeGuard() {
    if (t) medusa_tree_destroy(t);
  }
};

}  // namespace
}  // namespace medusa

using namespace medusa;

extern "C" size_t medusa_generate_workspace_size(const medusa_tree_t* tree, const medusa_decoder_t* model) {
  if (!tree || !tree->dev_block || !model || sm_count() <= 0) return 0;
  return gen_layout(tree, model).total;
}

extern "C" medusa_status_t medusa_generate(const medusa_tree_t* tree, const medusa_decoder_t* model,
                                           const void* W1, const void* b1, const void* Wout, medusa_mode_t mode,
                                           float temperature, float eps, float alpha, float top_p,
                                           const float* uniforms, const int32_t* prompt, int n_prompt, int n_new,
                                           void* k_cache, void* v_cache, int Lcap, int32_t* out_tokens,
                                           int32_t* out_accept, int max_steps, int32_t* n_steps, void* workspace,
                                           size_t workspace_bytes, cudaStream_t stream) {
  const char* fn = "medusa_generate";
  medusa_status_t st = check_decoder(tree, model, 1, fn);
  if (st != MEDUSA_OK) return st;
  if (!W1 || !b1 || !Wout || !prompt || !k_cache || !v_cache || !out_tokens || !out_accept || !n_steps || !workspace)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (n_prompt < 1 || n_new < 1 || max_steps < 1)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": n_prompt, n_new and max_steps must be positive");
  if (static_cast<long long>(n_prompt) + tree->T > Lcap)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": Lcap holds neither the prompt nor one tree after it");
  for (int i = 0; i < n_prompt; ++i)
    if (prompt[i] < 0 || prompt[i] >= model->V) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": prompt token outside [0, V)");
  const GenLayout l = gen_layout(tree, model);
  if (workspace_bytes < l.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": workspace too small or misaligned");
  unsigned char* w = static_cast<unsigned char*>(workspace);
  // the heads' own checks (d, V, K, topk, alignment), on the buffers of this workspace
  st = check_heads(w + l.h, W1, b1, Wout, 1, model->D, model->V, tree->K, tree->topk, MEDUSA_BF16, nullptr,
                   reinterpret_cast<const int32_t*>(w + l.ids), reinterpret_cast<const float*>(w + l.vals),
                   w + l.heads, heads_workspace_bytes(1, model->D, model->V, tree->K, tree->topk));
  if (st != MEDUSA_OK) return st;
  st = check_posterior(tree, 1, model->V, reinterpret_cast<const float*>(w + l.logits),
                       reinterpret_cast<const int32_t*>(w + l.cand), mode, temperature, eps, alpha, top_p,
                       reinterpret_cast<const int32_t*>(w + l.small), reinterpret_cast<const int32_t*>(w + l.small),
                       reinterpret_cast<const int32_t*>(w + l.small), reinterpret_cast<const int32_t*>(w + l.small),
                       w + l.post, posterior_workspace_bytes(tree->dev, 1));
  if (st != MEDUSA_OK) return st;
  if (uniforms)
    for (int i = 0; i < max_steps; ++i)
      if (!(uniforms[i] >= 0.f && uniforms[i] < 1.f))
        return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": uniforms outside [0, 1)");

  void* ws_dec = w + l.dec;
  void* ws_heads = w + l.heads;
  void* ws_post = w + l.post;
  int32_t* tokens = reinterpret_cast<int32_t*>(w + l.tokens);
  int32_t* pos = reinterpret_cast<int32_t*>(w + l.pos);
  int32_t* cand = reinterpret_cast<int32_t*>(w + l.cand);
  int32_t* ids = reinterpret_cast<int32_t*>(w + l.ids);
  float* vals = reinterpret_cast<float*>(w + l.vals);
  float* logits = reinterpret_cast<float*>(w + l.logits);
  uint16_t* h = reinterpret_cast<uint16_t*>(w + l.h);
  int32_t* small = reinterpret_cast<int32_t*>(w + l.small);
  int32_t *root = small, *seq_len = small + 1, *best = small + 2, *alen = small + 3, *acc = small + 8;
  float* u_dev = reinterpret_cast<float*>(small + 4);   // this step's uniform
  const int D = model->D, V = model->V, H = D / 128;
  cudaError_t e;

  // The prompt, in chains of at most kChain tokens.
  int L = 0, last_n = 0;
  TreeGuard full, rest;
  for (int at = 0; at < n_prompt; at += kChain) {
    const int n = n_prompt - at < kChain ? n_prompt - at : kChain;
    TreeGuard& g = n == kChain ? full : rest;
    if (!g.t) {
      st = chain_tree(n, &g.t);
      if (st != MEDUSA_OK) return st;
    }
    e = cudaMemcpyAsync(tokens, prompt + at, static_cast<size_t>(n) * 4, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail("medusa_generate: prompt copy", e);
    set_len_kernel<<<1, 1, 0, stream>>>(seq_len, L);
    st = launch_tree_decode(g.t->dev, model, 1, tokens, k_cache, v_cache, Lcap, seq_len, logits, nullptr, ws_dec,
                            stream);
    if (st != MEDUSA_OK) return st;
    L += n;
    last_n = n;
  }
  next_input_kernel<<<1, 256, 0, stream>>>(decoder_final_rows(ws_dec, last_n, D, model->F, V), logits, D, V,
                                           last_n - 1, nullptr, 0, 0, nullptr, nullptr, h, root, device_status_ptr());
  set_len_kernel<<<1, 1, 0, stream>>>(seq_len, L);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("medusa_generate: launch", e);

  TreeBuild tb{};
  tb.t = tree->dev;
  tb.root_tokens = root;
  tb.seq_lens = seq_len;
  tb.tree_tokens = tokens;
  tb.candidates = cand;
  tb.position_ids = pos;
  const int dp1 = tree->D + 1;
  std::vector<int32_t> host(dp1 + 1);
  int produced = 0, steps = 0;
  while (produced < n_new && steps < max_steps && L + tree->T <= Lcap) {
    st = launch_heads(h, W1, b1, Wout, 1, D, V, tree->K, tree->topk, MEDUSA_BF16, nullptr, ids, vals, ws_heads,
                      stream, &tb);
    if (st != MEDUSA_OK) return st;
    st = launch_tree_decode(tree->dev, model, 1, tokens, k_cache, v_cache, Lcap, seq_len, logits, nullptr, ws_dec,
                            stream);
    if (st != MEDUSA_OK) return st;
    // acceptance; the next token (drawn with this step's uniform, if any) goes where the next
    // step's root is read
    if (uniforms) {
      e = cudaMemcpyAsync(u_dev, uniforms + steps, 4, cudaMemcpyHostToDevice, stream);
      if (e != cudaSuccess) return cuda_fail("medusa_generate: uniform copy", e);
    }
    st = launch_posterior_accept(tree->dev, 1, V, logits, cand, mode, temperature, eps, alpha, top_p,
                                 uniforms ? u_dev : nullptr, best, alen, acc, root, model->layers, H, 128, MEDUSA_BF16,
                                 k_cache, v_cache, Lcap, seq_len, ws_post, stream, false);
    if (st != MEDUSA_OK) return st;
    next_input_kernel<<<1, 256, 0, stream>>>(decoder_final_rows(ws_dec, tree->T, D, model->F, V), logits, D, V, 0,
                                             tree->dev.retrieve, tree->P, dp1, best, alen, h, nullptr,
                                             device_status_ptr());
    e = cudaMemcpyAsync(host.data(), alen, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(host.data() + 1, acc, static_cast<size_t>(dp1) * 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail("medusa_generate: step", e);
    const int a = host[0];
    if (a < 0 || a >= dp1) return fail(MEDUSA_ERR_DEVICE_CHECK, std::string(fn) + ": accept length out of range");
    for (int j = 0; j <= a && produced < n_new; ++j) out_tokens[produced++] = host[1 + j];
    out_accept[steps++] = a;
    L += a + 1;
  }
  *n_steps = steps;
  if (produced < n_new)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": stopped before n_new tokens (Lcap or max_steps)");
  return MEDUSA_OK;
}

extern "C" medusa_status_t medusa_generate_greedy(const medusa_tree_t* tree, const medusa_decoder_t* model,
                                                  const void* W1, const void* b1, const void* Wout,
                                                  const int32_t* prompt, int n_prompt, int n_new, void* k_cache,
                                                  void* v_cache, int Lcap, int32_t* out_tokens,
                                                  int32_t* out_accept, int max_steps, int32_t* n_steps,
                                                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return medusa_generate(tree, model, W1, b1, Wout, MEDUSA_GREEDY, 0.f, 0.09f, 0.3f, 0.8f, nullptr, prompt, n_prompt,
                         n_new, k_cache, v_cache, Lcap, out_tokens, out_accept, max_steps, n_steps, workspace,
                         workspace_bytes, stream);
}
