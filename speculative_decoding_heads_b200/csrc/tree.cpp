// Host side of the candidate tree: the rank-sum construction, validation and
// the index tables (tree_indices, parent, depth, retrieve, ancestor bitmask)
// that the kernels read.  The tables follow the candidate-assembly step of
// "Medusa API参考：核心函数与类详解" (generate_candidates: tree_indices and
// retrieve_indices) and the mask of "Medusa — 让大模型自己同时猜好几个 token"
// (实践案例 case 3: a node sees the prefix, its ancestors and itself).
#include <algorithm>
#include <cstring>
#include <map>
#include <new>
#include <vector>

#include <cuda_runtime_api.h>

#include "internal.h"

namespace {

using Tuple = std::vector<int32_t>;

// Appends, in lexicographic order, tuples of `len` entries in [0, topk) with
// entry sum `sum`, until `out` holds `want` tuples.
void enumerate_sum(int len, int sum, int topk, Tuple& cur, std::vector<Tuple>& out, size_t want) {
  if (out.size() >= want) return;
  if (len == 0) {
    if (sum == 0) out.push_back(cur);
    return;
  }
  for (int r = 0; r < topk && r <= sum; ++r) {
    const long rest = sum - r;
    if (rest > static_cast<long>(len - 1) * (topk - 1)) continue;  // cannot reach the sum
    cur.push_back(r);
    enumerate_sum(len - 1, static_cast<int>(rest), topk, cur, out, want);
    cur.pop_back();
    if (out.size() >= want) return;
  }
}

bool lex_less(const Tuple& a, const Tuple& b) {
  if (a.size() != b.size()) return a.size() < b.size();
  return a < b;
}

}  // namespace

extern "C" medusa_status_t medusa_tree_choices_ranksum(int K, int topk, int n_nodes,
                                                       int32_t* ranks, int32_t* lens) {
  using medusa::fail;
  if (K < 1 || K > MEDUSA_MAX_K || topk < 1 || topk > MEDUSA_MAX_TOPK)
    return fail(MEDUSA_ERR_INVALID_ARG, "ranksum: K or topk out of range");
  if (n_nodes < 0 || n_nodes > MEDUSA_MAX_T - 1)
    return fail(MEDUSA_ERR_INVALID_ARG, "ranksum: n_nodes out of range");
  if (n_nodes > 0 && (!ranks || !lens)) return fail(MEDUSA_ERR_INVALID_ARG, "ranksum: null output");
  std::vector<Tuple> out;
  Tuple cur;
  const size_t want = static_cast<size_t>(n_nodes);
  for (int s = 0; s <= K * (topk - 1) && out.size() < want; ++s)
    for (int len = 1; len <= K && out.size() < want; ++len) enumerate_sum(len, s, topk, cur, out, want);
  if (out.size() < want) return fail(MEDUSA_ERR_INVALID_ARG, "ranksum: fewer tuples than n_nodes");
  for (int i = 0; i < n_nodes; ++i) {
    lens[i] = static_cast<int32_t>(out[i].size());
    for (int j = 0; j < K; ++j) ranks[i * K + j] = j < lens[i] ? out[i][j] : 0;
  }
  return MEDUSA_OK;
}

extern "C" medusa_status_t medusa_tree_create(const int32_t* ranks, const int32_t* lens,
                                              int n_nodes, int K, int topk, int upload,
                                              medusa_tree_t** out) {
  using medusa::fail;
  if (!out) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: out is null");
  *out = nullptr;
  if (K < 1 || K > MEDUSA_MAX_K) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: K out of range");
  if (topk < 1 || topk > MEDUSA_MAX_TOPK)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: topk out of range");
  if (n_nodes < 0 || n_nodes + 1 > MEDUSA_MAX_T)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: n_nodes out of range");
  if (n_nodes > 0 && (!ranks || !lens)) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: null input");

  std::vector<Tuple> nodes;
  nodes.reserve(n_nodes);
  for (int i = 0; i < n_nodes; ++i) {
    const int len = lens[i];
    if (len < 1 || len > K) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: tuple length outside 1..K");
    Tuple t(ranks + static_cast<size_t>(i) * K, ranks + static_cast<size_t>(i) * K + len);
    for (int r : t)
      if (r < 0 || r >= topk) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: rank outside [0, topk)");
    nodes.push_back(std::move(t));
  }
  std::sort(nodes.begin(), nodes.end(), lex_less);
  for (size_t i = 1; i < nodes.size(); ++i)
    if (nodes[i] == nodes[i - 1]) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: duplicate tuple");
  nodes.insert(nodes.begin(), Tuple{});

  std::map<Tuple, int> index;
  for (size_t i = 0; i < nodes.size(); ++i) index[nodes[i]] = static_cast<int>(i);

  medusa_tree* t = new (std::nothrow) medusa_tree();
  if (!t) return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: out of host memory");
  const int T = static_cast<int>(nodes.size());
  t->T = T;
  t->K = K;
  t->topk = topk;
  t->W = (T + 63) / 64;
  t->tree_indices.assign(T, 0);
  t->parent.assign(T, -1);
  t->depth.assign(T, 0);
  std::vector<char> has_child(T, 0);
  int D = 0;
  for (int i = 1; i < T; ++i) {
    const Tuple& c = nodes[i];
    Tuple par(c.begin(), c.end() - 1);
    auto it = index.find(par);
    if (it == index.end()) {
      delete t;
      return fail(MEDUSA_ERR_INVALID_ARG, "tree_create: a tuple's parent is missing");
    }
    t->parent[i] = it->second;
    has_child[it->second] = 1;
    const int len = static_cast<int>(c.size());
    t->depth[i] = len;
    t->tree_indices[i] = 1 + (len - 1) * topk + c.back();
    D = std::max(D, len);
  }
  t->D = D;
  std::vector<int> leaves;
  for (int i = 0; i < T; ++i)
    if (!has_child[i]) leaves.push_back(i);
  t->P = static_cast<int>(leaves.size());
  t->retrieve.assign(static_cast<size_t>(t->P) * (D + 1), -1);
  for (int p = 0; p < t->P; ++p) {
    // walk up from the leaf; fill depth slots from the bottom
    int n = leaves[p];
    while (n >= 0) {
      t->retrieve[static_cast<size_t>(p) * (D + 1) + t->depth[n]] = n;
      n = t->parent[n];
    }
  }
  t->anc.assign(static_cast<size_t>(T) * t->W, 0ull);
  for (int i = 0; i < T; ++i) {
    int n = i;
    while (n >= 0) {
      t->anc[static_cast<size_t>(i) * t->W + n / 64] |= 1ull << (n % 64);
      n = t->parent[n];
    }
  }
  // Lowest path through each node (the posterior reads a node's token from it).
  t->path_of.assign(T, -1);
  for (int p = t->P - 1; p >= 0; --p)
    for (int j = 0; j <= D; ++j) {
      const int n = t->retrieve[static_cast<size_t>(p) * (D + 1) + j];
      if (n >= 0) t->path_of[n] = p;
    }
  t->nodes = std::move(nodes);

  if (upload) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
      delete t;
      return medusa::cuda_fail("tree_create: cudaGetDevice", e);
    }
    const size_t n32 = static_cast<size_t>(4 * T) + t->retrieve.size();
    const size_t off_anc = medusa::align_up(n32 * sizeof(int32_t), 256);
    const size_t bytes = off_anc + t->anc.size() * sizeof(uint64_t);
    std::vector<unsigned char> host(bytes, 0);
    int32_t* h32 = reinterpret_cast<int32_t*>(host.data());
    std::memcpy(h32, t->tree_indices.data(), T * sizeof(int32_t));
    std::memcpy(h32 + T, t->parent.data(), T * sizeof(int32_t));
    std::memcpy(h32 + 2 * T, t->depth.data(), T * sizeof(int32_t));
    std::memcpy(h32 + 3 * T, t->retrieve.data(), t->retrieve.size() * sizeof(int32_t));
    std::memcpy(h32 + 3 * T + t->retrieve.size(), t->path_of.data(), T * sizeof(int32_t));
    std::memcpy(host.data() + off_anc, t->anc.data(), t->anc.size() * sizeof(uint64_t));
    e = cudaMalloc(&t->dev_block, bytes);
    if (e == cudaSuccess) e = cudaMemcpy(t->dev_block, host.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      if (t->dev_block) cudaFree(t->dev_block);
      delete t;
      return medusa::cuda_fail("tree_create: upload", e);
    }
    t->device = dev;
    const int32_t* d32 = static_cast<const int32_t*>(t->dev_block);
    t->dev = medusa::TreeDev{T, t->P, t->D, K, topk, t->W, d32, d32 + T, d32 + 2 * T, d32 + 3 * T,
                             reinterpret_cast<const uint64_t*>(
                                 static_cast<const unsigned char*>(t->dev_block) + off_anc),
                             d32 + 3 * T + t->retrieve.size()};
  }
  *out = t;
  return MEDUSA_OK;
}

extern "C" void medusa_tree_destroy(medusa_tree_t* tree) {
  if (!tree) return;
  if (tree->dev_block) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != tree->device) cudaSetDevice(tree->device);
    cudaFree(tree->dev_block);
    if (cur >= 0 && cur != tree->device) cudaSetDevice(cur);
  }
  delete tree;
}

extern "C" medusa_status_t medusa_tree_info(const medusa_tree_t* tree, int32_t* T, int32_t* P,
                                            int32_t* D) {
  if (!tree) return medusa::fail(MEDUSA_ERR_INVALID_ARG, "tree_info: tree is null");
  if (T) *T = tree->T;
  if (P) *P = tree->P;
  if (D) *D = tree->D;
  return MEDUSA_OK;
}

extern "C" medusa_status_t medusa_tree_tables(const medusa_tree_t* tree, int32_t* tree_indices,
                                              int32_t* parent, int32_t* depth, int32_t* retrieve,
                                              uint64_t* anc) {
  if (!tree) return medusa::fail(MEDUSA_ERR_INVALID_ARG, "tree_tables: tree is null");
  if (tree_indices) std::copy(tree->tree_indices.begin(), tree->tree_indices.end(), tree_indices);
  if (parent) std::copy(tree->parent.begin(), tree->parent.end(), parent);
  if (depth) std::copy(tree->depth.begin(), tree->depth.end(), depth);
  if (retrieve) std::copy(tree->retrieve.begin(), tree->retrieve.end(), retrieve);
  if (anc) std::copy(tree->anc.begin(), tree->anc.end(), anc);
  return MEDUSA_OK;
}
