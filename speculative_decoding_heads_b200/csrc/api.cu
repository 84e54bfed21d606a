// The C ABI of libmedusa_b200: argument checks, the per-device status word,
// and the step that chains S1..S7 on one stream.  Every check happens on the
// host before any launch.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"

namespace medusa {

namespace {
thread_local std::string g_last_error;

__device__ int g_device_status[2];   // [0] status code, [1] detail

constexpr int kMaxDevices = 64;
int g_status_dev[kMaxDevices];
int* g_status_ptr[kMaxDevices];
int g_sms[kMaxDevices];
std::once_flag g_once[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

void init_device(int dev) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) == cudaSuccess) g_status_ptr[dev] = static_cast<int*>(p);
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) g_sms[dev] = sms;
  g_status_dev[dev] = 1;
}

bool ensure_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(g_once[dev], init_device, dev);
  return g_status_ptr[dev] != nullptr && g_sms[dev] > 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

medusa_status_t fail(medusa_status_t st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

medusa_status_t cuda_fail(const char* what, int err) {
  g_last_error = std::string(what) + ": " + cudaGetErrorName(static_cast<cudaError_t>(err)) + " (" +
                 cudaGetErrorString(static_cast<cudaError_t>(err)) + ")";
  return MEDUSA_ERR_CUDA;
}

int* device_status_ptr() {
  const int dev = current_device();
  return ensure_device(dev) ? g_status_ptr[dev] : nullptr;
}

int sm_count() {
  const int dev = current_device();
  return ensure_device(dev) ? g_sms[dev] : 0;
}

medusa_status_t device_status_read(int32_t* status, int32_t* detail, int clear) {
  const int dev = current_device();
  if (!ensure_device(dev)) return fail(MEDUSA_ERR_CUDA, "medusa_device_status: no usable CUDA device");
  int host[2] = {0, 0};
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(host, g_status_ptr[dev], sizeof(host), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) {
    const int zero[2] = {0, 0};
    e = cudaMemcpy(g_status_ptr[dev], zero, sizeof(zero), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) return cuda_fail("medusa_device_status", e);
  if (status) *status = host[0];
  if (detail) *detail = host[1];
  return MEDUSA_OK;
}

// Checks shared by the calls that take a tree.
static medusa_status_t check_tree(const medusa_tree_t* tree, const char* fn) {
  if (!tree) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": tree is null");
  if (!tree->dev_block) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": tree was created without upload");
  const int dev = current_device();
  if (dev != tree->device)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": tree belongs to another device");
  if (!ensure_device(dev)) return fail(MEDUSA_ERR_CUDA, std::string(fn) + ": no usable CUDA device");
  return MEDUSA_OK;
}

}  // namespace medusa

using namespace medusa;

extern "C" const char* medusa_last_error(void) { return g_last_error.c_str(); }

extern "C" int medusa_abi_version(void) { return MEDUSA_ABI_VERSION; }

extern "C" medusa_status_t medusa_device_status(int32_t* status, int32_t* detail, int clear) {
  return device_status_read(status, detail, clear);
}

extern "C" size_t medusa_heads_workspace_size(int B, int d, int V, int K, int topk) {
  if (B < 1 || d < 1 || V < 1 || K < 1 || topk < 1) return 0;
  if (sm_count() <= 0) return 0;
  return heads_workspace_bytes(B, d, V, K, topk);
}

medusa_status_t medusa::check_heads(const void* h, const void* W1, const void* b1, const void* Wout, int B,
                                    int d, int V, int K, int topk, medusa_dtype_t dtype, const float* head_logits,
                                    const int32_t* topk_ids, const float* topk_vals, const void* ws,
                                    size_t ws_bytes) {
  const char* fn = "medusa_heads_topk";
  if (!h || !W1 || !b1 || !Wout || !topk_ids || !topk_vals || !ws)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (B < 1 || B > MEDUSA_MAX_B || K < 1 || K > MEDUSA_MAX_K || V < 1 || d < 1)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": B, K, V or d out of range");
  if (topk < 1 || topk > MEDUSA_MAX_TOPK || topk > V)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": topk out of range");
  if (dtype != MEDUSA_BF16 && dtype != MEDUSA_F32)
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": dtype");
  const int unit = dtype == MEDUSA_BF16 ? 256 : 128;
  const int dmax = dtype == MEDUSA_BF16 ? 8192 : 4096;
  if (d % unit != 0 || d > dmax)
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": d must be a multiple of 256 (bf16) / 128 (f32) "
                                                          "and at most 8192 (bf16) / 4096 (f32)");
  if (!aligned16(h) || !aligned16(W1) || !aligned16(b1) || !aligned16(Wout) ||
      (head_logits && !aligned16(head_logits)) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned pointer");
  if (static_cast<long long>(K) * V * d >= (1ll << 40))
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": weights too large");
  if (ws_bytes < heads_workspace_bytes(B, d, V, K, topk))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": workspace too small");
  return MEDUSA_OK;
}

extern "C" medusa_status_t medusa_heads_topk(const void* h, const void* W1, const void* b1, const void* Wout,
                                             int B, int d, int V, int K, int topk, medusa_dtype_t dtype,
                                             float* head_logits, int32_t* topk_ids, float* topk_vals,
                                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (sm_count() <= 0) return fail(MEDUSA_ERR_CUDA, "medusa_heads_topk: no usable CUDA device");
  medusa_status_t st = check_heads(h, W1, b1, Wout, B, d, V, K, topk, dtype, head_logits, topk_ids, topk_vals,
                                   workspace, workspace_bytes);
  if (st != MEDUSA_OK) return st;
  return launch_heads(h, W1, b1, Wout, B, d, V, K, topk, dtype, head_logits, topk_ids, topk_vals, workspace,
                      stream);
}

extern "C" medusa_status_t medusa_topk_merge(const float* vals, const int32_t* ids, const int32_t* row0, int G,
                                             int V, int B, int K, int topk, float* out_vals, int32_t* out_ids,
                                             cudaStream_t stream) {
  const char* fn = "medusa_topk_merge";
  if (!vals || !ids || !row0 || !out_vals || !out_ids) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (G < 1 || G > MEDUSA_MAX_SHARDS || B < 1 || B > MEDUSA_MAX_B || K < 1 || K > MEDUSA_MAX_K)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": G, B or K out of range");
  if (topk < 1 || topk > MEDUSA_MAX_TOPK) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": topk out of range");
  if (row0[0] != 0) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": row0[0] must be 0");
  for (int g = 0; g < G; ++g) {
    const long long end = g + 1 < G ? row0[g + 1] : V;
    if (end - row0[g] < topk)
      return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": shard " + std::to_string(g) + " holds fewer than topk rows");
  }
  if (sm_count() <= 0) return fail(MEDUSA_ERR_CUDA, std::string(fn) + ": no usable CUDA device");
  return launch_topk_merge(vals, ids, row0, G, B, K, topk, out_vals, out_ids, stream);
}

extern "C" medusa_status_t medusa_build_tree(const medusa_tree_t* tree, int B, const int32_t* root_tokens,
                                             const int32_t* topk_ids, const int32_t* seq_lens,
                                             int32_t* tree_tokens, int32_t* candidates, int32_t* position_ids,
                                             cudaStream_t stream) {
  medusa_status_t st = check_tree(tree, "medusa_build_tree");
  if (st != MEDUSA_OK) return st;
  if (B < 1 || B > MEDUSA_MAX_B) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_build_tree: B out of range");
  if (!root_tokens || !topk_ids || !seq_lens || !tree_tokens || !candidates || !position_ids)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_build_tree: null pointer");
  return launch_build_tree(tree->dev, B, root_tokens, topk_ids, seq_lens, tree_tokens, candidates, position_ids,
                           stream);
}

static medusa_status_t check_attention(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                       medusa_dtype_t dtype, const void* q, const void* k, const void* v, int Lcap,
                                       const int32_t* seq_lens, float scale, const void* out) {
  const char* fn = "medusa_tree_attention";
  medusa_status_t st = check_tree(tree, fn);
  if (st != MEDUSA_OK) return st;
  if (!q || !k || !v || !seq_lens || !out) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (layers < 1 || B < 1 || B > MEDUSA_MAX_B || H < 1 || Lcap < tree->T)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": layers, B, H or Lcap out of range");
  if (dtype != MEDUSA_BF16 && dtype != MEDUSA_F32) return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": dtype");
  if (hd < 32 || hd > 256 || hd % 32 != 0)
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": hd must be a multiple of 32 in [32, 256]");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": scale");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned pointer");
  if (static_cast<long long>(layers) * B * H >= (1ll << 31) / 2)
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": too many slices");
  return MEDUSA_OK;
}

extern "C" size_t medusa_attention_workspace_size(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                                  medusa_dtype_t dtype) {
  if (!tree || !tree->dev_block) return 0;
  return attention_workspace_bytes(tree->dev, layers, B, H, hd, dtype);
}

extern "C" medusa_status_t medusa_tree_attention(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                                 medusa_dtype_t dtype, const void* q, const void* k_cache,
                                                 const void* v_cache, int Lcap, const int32_t* seq_lens,
                                                 float scale, void* out, void* workspace, size_t workspace_bytes,
                                                 cudaStream_t stream) {
  medusa_status_t st =
      check_attention(tree, layers, B, H, hd, dtype, q, k_cache, v_cache, Lcap, seq_lens, scale, out);
  if (st != MEDUSA_OK) return st;
  const size_t need = attention_workspace_bytes(tree->dev, layers, B, H, hd, dtype);
  if (workspace_bytes < need || (need && !workspace))
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_attention: workspace too small");
  return launch_attention(tree->dev, layers, B, H, hd, dtype, q, k_cache, v_cache, Lcap, seq_lens, scale, out,
                          workspace, stream);
}

extern "C" medusa_status_t medusa_tree_attention_split(const medusa_tree_t* tree, int layers, int B, int H,
                                                       int hd, medusa_dtype_t dtype, const void* q,
                                                       const void* k_cache, const void* v_cache, int Lcap,
                                                       const int32_t* seq_lens, float scale, int rank, int G,
                                                       float* out, float* lse, cudaStream_t stream) {
  const char* fn = "medusa_tree_attention_split";
  medusa_status_t st =
      check_attention(tree, layers, B, H, hd, dtype, q, k_cache, v_cache, Lcap, seq_lens, scale, out);
  if (st != MEDUSA_OK) return st;
  if (!lse) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (G < 1 || G > MEDUSA_MAX_SHARDS || rank < 0 || rank >= G)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": rank or G out of range");
  return launch_attention_split(tree->dev, layers, B, H, hd, dtype, q, k_cache, v_cache, Lcap, seq_lens, scale, rank,
                                G, out, lse, stream);
}

extern "C" medusa_status_t medusa_attention_combine(int G, int64_t rows, int hd, const float* outs,
                                                    const float* lses, float* out, float* lse_out,
                                                    cudaStream_t stream) {
  const char* fn = "medusa_attention_combine";
  if (!outs || !lses || !out) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (G < 1 || G > MEDUSA_MAX_SHARDS || rows < 1 || hd < 4 || hd > 1024 || hd % 4 != 0)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": G, rows or hd out of range");
  if (!aligned16(outs) || !aligned16(out)) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned pointer");
  const uintptr_t o0 = reinterpret_cast<uintptr_t>(out), o1 = o0 + static_cast<uintptr_t>(rows) * hd * 4;
  const uintptr_t i0 = reinterpret_cast<uintptr_t>(outs), i1 = i0 + static_cast<uintptr_t>(rows) * hd * 4 * G;
  if (o0 < i1 && i0 < o1) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": out overlaps outs");
  if (sm_count() <= 0) return fail(MEDUSA_ERR_CUDA, std::string(fn) + ": no usable CUDA device");
  return launch_attention_combine(G, static_cast<size_t>(rows), hd, outs, lses, out, lse_out, stream);
}

extern "C" medusa_status_t medusa_attention_rescale(int G, int rank, int64_t rows, int hd, const float* lses,
                                                    float* part, float* lse_out, cudaStream_t stream) {
  const char* fn = "medusa_attention_rescale";
  if (!lses || !part) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (G < 1 || G > MEDUSA_MAX_SHARDS || rank < 0 || rank >= G || rows < 1 || hd < 4 || hd > 1024 || hd % 4 != 0)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": G, rank, rows or hd out of range");
  if (!aligned16(part)) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned pointer");
  if (sm_count() <= 0) return fail(MEDUSA_ERR_CUDA, std::string(fn) + ": no usable CUDA device");
  return launch_attention_rescale(G, rank, static_cast<size_t>(rows), hd, lses, part, lse_out, stream);
}

extern "C" size_t medusa_posterior_workspace_size(const medusa_tree_t* tree, int B) {
  if (!tree || B < 1) return 0;
  medusa::TreeDev t{};
  t.T = tree->T;
  return posterior_workspace_bytes(t, B);
}

medusa_status_t medusa::check_posterior(const medusa_tree_t* tree, int B, int V, const float* logits,
                                       const int32_t* candidates, medusa_mode_t mode, float temperature,
                                       float eps, float alpha, float top_p, const int32_t* best_path,
                                       const int32_t* accept_len, const int32_t* accepted_tokens,
                                       const int32_t* next_token, const void* ws, size_t ws_bytes) {
  const char* fn = "medusa_evaluate_posterior";
  medusa_status_t st = check_tree(tree, fn);
  if (st != MEDUSA_OK) return st;
  if (!logits || !candidates || !best_path || !accept_len || !accepted_tokens || !next_token || !ws)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (B < 1 || B > MEDUSA_MAX_B || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": B or V");
  if (mode != MEDUSA_GREEDY && mode != MEDUSA_TYPICAL && mode != MEDUSA_NUCLEUS)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": mode");
  if (mode != MEDUSA_GREEDY) {
    if (!(temperature > 0.f) || !std::isfinite(temperature))
      return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": typical and nucleus acceptance need temperature > 0");
    if (!std::isfinite(eps) || !std::isfinite(alpha) || eps < 0.f || alpha < 0.f)
      return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": eps and alpha must be finite and >= 0");
  }
  if (mode == MEDUSA_NUCLEUS && !(top_p > 0.f && top_p <= 1.f))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": nucleus acceptance needs 0 < top_p <= 1");
  if (ws_bytes < posterior_workspace_bytes(tree->dev, B))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": workspace too small");
  return MEDUSA_OK;
}

extern "C" medusa_status_t medusa_evaluate_posterior(const medusa_tree_t* tree, int B, int V, const float* logits,
                                                     const int32_t* candidates, medusa_mode_t mode,
                                                     float temperature, float eps, float alpha, float top_p,
                                                     const float* uniforms, int32_t* best_path,
                                                     int32_t* accept_len, int32_t* accepted_tokens,
                                                     int32_t* next_token, void* workspace, size_t workspace_bytes,
                                                     cudaStream_t stream) {
  medusa_status_t st = check_posterior(tree, B, V, logits, candidates, mode, temperature, eps, alpha, top_p,
                                       best_path, accept_len, accepted_tokens, next_token, workspace,
                                       workspace_bytes);
  if (st != MEDUSA_OK) return st;
  return launch_posterior(tree->dev, B, V, logits, candidates, mode, temperature, eps, alpha, top_p, uniforms,
                          best_path, accept_len, accepted_tokens, next_token, workspace, stream);
}

static medusa_status_t check_accept(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                    medusa_dtype_t dtype, const void* k, const void* v, int Lcap,
                                    const int32_t* seq_lens, const int32_t* best_path, const int32_t* accept_len) {
  const char* fn = "medusa_accept_kv";
  medusa_status_t st = check_tree(tree, fn);
  if (st != MEDUSA_OK) return st;
  if (!k || !v || !seq_lens || !best_path || !accept_len)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (layers < 1 || B < 1 || B > MEDUSA_MAX_B || H < 1 || Lcap < tree->T)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": layers, B, H or Lcap out of range");
  if (dtype != MEDUSA_BF16 && dtype != MEDUSA_F32) return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": dtype");
  if (hd < 8 || hd > 256 || (hd * (dtype == MEDUSA_BF16 ? 2 : 4)) % 16 != 0)
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": hd");
  if (!aligned16(k) || !aligned16(v)) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned pointer");
  return MEDUSA_OK;
}

extern "C" medusa_status_t medusa_accept_kv(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                            medusa_dtype_t dtype, void* k_cache, void* v_cache, int Lcap,
                                            int32_t* seq_lens, const int32_t* best_path, const int32_t* accept_len,
                                            cudaStream_t stream) {
  medusa_status_t st = check_accept(tree, layers, B, H, hd, dtype, k_cache, v_cache, Lcap, seq_lens, best_path,
                                    accept_len);
  if (st != MEDUSA_OK) return st;
  return launch_accept_kv(tree->dev, layers, B, H, hd, dtype, k_cache, v_cache, Lcap, seq_lens, best_path,
                          accept_len, stream);
}

// ---- the base model's forward over the tree -------------------------------

extern "C" medusa_status_t medusa_decoder_pack_rows(int which, int n, int32_t* out) {
  const char* fn = "medusa_decoder_pack_rows";
  if (!out || n <= 0 || (which != 0 && which != 1)) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": arguments");
  if (which == 0) {
    if (n % 128 != 0) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": D must be a multiple of 128");
    for (int r = 0; r < n; ++r) {
      const int head = r / 128, lr = r % 128;
      out[r] = head * 128 + (lr >> 1) + (lr & 1) * 64;
    }
  } else {
    if (n % 2 != 0) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": 2F rows");
    for (int r = 0; r < n; ++r) out[r] = (r & 1) ? n / 2 + (r >> 1) : (r >> 1);
  }
  return MEDUSA_OK;
}

medusa_status_t medusa::check_decoder(const medusa_tree_t* tree, const medusa_decoder_t* m, int B, const char* fn) {
  medusa_status_t st = check_tree(tree, fn);
  if (st != MEDUSA_OK) return st;
  if (!m || !m->layer || !m->embed || !m->final_norm || !m->lm_head)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null model pointer");
  if (m->layers < 1 || m->D < 128 || m->D % 128 != 0 || m->D > 8192 || m->F < 128 || m->F % 128 != 0 || m->V < 1 ||
      B < 1 || B > MEDUSA_MAX_B)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": layers, D, F, V or B out of range");
  if (static_cast<long long>(B) * tree->T > (1 << 20))
    return fail(MEDUSA_ERR_UNSUPPORTED, std::string(fn) + ": too many tree tokens");
  for (int l = 0; l < m->layers; ++l) {
    const medusa_decoder_layer_t& y = m->layer[l];
    if (!y.attn_norm || !y.wqkv || !y.wo || !y.mlp_norm || !y.wgu || !y.wdown)
      return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null layer pointer");
    if (!aligned16(y.wqkv) || !aligned16(y.wo) || !aligned16(y.wgu) || !aligned16(y.wdown) ||
        !aligned16(y.attn_norm) || !aligned16(y.mlp_norm))
      return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned weights");
  }
  if (!aligned16(m->embed) || !aligned16(m->lm_head) || !aligned16(m->final_norm))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned");
  return MEDUSA_OK;
}

extern "C" size_t medusa_tree_decode_workspace_size(const medusa_tree_t* tree, const medusa_decoder_t* m, int B) {
  if (!tree || !m || B < 1 || sm_count() <= 0) return 0;
  return decoder_workspace_bytes(B * tree->T, m->D, m->F, m->V);
}

extern "C" medusa_status_t medusa_tree_decode(const medusa_tree_t* tree, const medusa_decoder_t* m, int B,
                                              const int32_t* tree_tokens, void* k_cache, void* v_cache, int Lcap,
                                              const int32_t* seq_lens, float* logits, float* hidden,
                                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const char* fn = "medusa_tree_decode";
  medusa_status_t st = check_decoder(tree, m, B, fn);
  if (st != MEDUSA_OK) return st;
  if (!tree_tokens || !k_cache || !v_cache || !seq_lens || !logits || !workspace)
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (Lcap < tree->T) return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": Lcap smaller than the tree");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(logits) || (hidden && !aligned16(hidden)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": misaligned pointer");
  if (workspace_bytes < decoder_workspace_bytes(B * tree->T, m->D, m->F, m->V))
    return fail(MEDUSA_ERR_INVALID_ARG, std::string(fn) + ": workspace too small");
  return launch_tree_decode(tree->dev, m, B, tree_tokens, k_cache, v_cache, Lcap, seq_lens, logits, hidden, workspace,
                            stream);
}

// ---- the whole step ------------------------------------------------------

namespace {
struct StepLayout {
  size_t heads, attn, post, total;
};

StepLayout step_layout(const medusa_step_args_t* a) {
  StepLayout l{};
  l.heads = align_up(heads_workspace_bytes(a->B, a->d, a->V, a->K, a->topk), 256);
  l.attn = align_up(attention_workspace_bytes(a->tree->dev, a->layers, a->B, a->H, a->hd, a->dtype), 256);
  l.post = align_up(posterior_workspace_bytes(a->tree->dev, a->B), 256);
  l.total = l.heads + l.attn + l.post;
  return l;
}
}  // namespace

extern "C" size_t medusa_step_workspace_size(const medusa_step_args_t* args) {
  if (!args || !args->tree || !args->tree->dev_block || sm_count() <= 0) return 0;
  return step_layout(args).total;
}

medusa_status_t medusa::check_step(const medusa_step_args_t* a, const void* workspace, size_t workspace_bytes) {
  if (!a) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step: args is null");
  medusa_status_t st = check_tree(a->tree, "medusa_step");
  if (st != MEDUSA_OK) return st;
  if (a->K != a->tree->K || a->topk != a->tree->topk)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step: K / topk differ from the tree's");
  if (!workspace) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step: workspace is null");
  const StepLayout l = step_layout(a);
  if (workspace_bytes < l.total) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step: workspace too small");
  unsigned char* ws = static_cast<unsigned char*>(const_cast<void*>(workspace));
  void* ws_heads = ws;
  void* ws_post = ws + l.heads + l.attn;
  // Validate every stage before launching any of them.
  st = check_heads(a->h, a->W1, a->b1, a->Wout, a->B, a->d, a->V, a->K, a->topk, a->dtype, a->head_logits,
                   a->topk_ids, a->topk_vals, ws_heads, l.heads);
  if (st != MEDUSA_OK) return st;
  if (!a->root_tokens || !a->tree_tokens || !a->candidates || !a->position_ids)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step: null tree output");
  st = check_attention(a->tree, a->layers, a->B, a->H, a->hd, a->dtype, a->q, a->k_cache, a->v_cache, a->Lcap,
                       a->seq_lens, a->scale, a->attn_out);
  if (st != MEDUSA_OK) return st;
  st = check_posterior(a->tree, a->B, a->V, a->base_logits, a->candidates, a->mode, a->temperature, a->eps, a->alpha,
                       a->top_p, a->best_path, a->accept_len, a->accepted_tokens, a->next_token, ws_post, l.post);
  if (st != MEDUSA_OK) return st;
  return check_accept(a->tree, a->layers, a->B, a->H, a->hd, a->dtype, a->k_cache, a->v_cache, a->Lcap,
                      a->seq_lens, a->best_path, a->accept_len);
}

extern "C" medusa_status_t medusa_step(const medusa_step_args_t* a, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream) {
  medusa_status_t st = check_step(a, workspace, workspace_bytes);
  if (st != MEDUSA_OK) return st;
  const StepLayout l = step_layout(a);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  void* ws_heads = ws;
  void* ws_attn = ws + l.heads;
  void* ws_post = ws + l.heads + l.attn;

  // S1-S4 in one launch per batch group: the heads kernel's last CTA also
  // builds the candidate tree from the final top-k.
  TreeBuild tb{};
  tb.t = a->tree->dev;
  tb.root_tokens = a->root_tokens;
  tb.seq_lens = a->seq_lens;
  tb.tree_tokens = a->tree_tokens;
  tb.candidates = a->candidates;
  tb.position_ids = a->position_ids;
  st = launch_heads(a->h, a->W1, a->b1, a->Wout, a->B, a->d, a->V, a->K, a->topk, a->dtype, a->head_logits,
                    a->topk_ids, a->topk_vals, ws_heads, stream, &tb);
  if (st != MEDUSA_OK) return st;
  // Attention, posterior and compaction start while the kernel before them
  // drains (programmatic dependent launch); each waits for its predecessor
  // before it touches that kernel's outputs.
  if (a->attn_inputs_ready) {
    const cudaError_t e = cudaStreamWaitEvent(stream, a->attn_inputs_ready, 0);
    if (e != cudaSuccess) return cuda_fail("medusa_step: wait for the attention inputs", e);
  }
  st = launch_attention(a->tree->dev, a->layers, a->B, a->H, a->hd, a->dtype, a->q, a->k_cache, a->v_cache, a->Lcap,
                        a->seq_lens, a->scale, a->attn_out, ws_attn, stream, true);
  if (st != MEDUSA_OK) return st;
  if (a->posterior_inputs_ready) {
    const cudaError_t e = cudaStreamWaitEvent(stream, a->posterior_inputs_ready, 0);
    if (e != cudaSuccess) return cuda_fail("medusa_step: wait for the posterior inputs", e);
  }
  // S6 and S7 in one launch: node statistics, the path walk (which advances
  // seq_lens), then the compaction of the accepted rows.
  return launch_posterior_accept(a->tree->dev, a->B, a->V, a->base_logits, a->candidates, a->mode, a->temperature,
                                 a->eps, a->alpha, a->top_p, a->uniforms, a->best_path, a->accept_len,
                                 a->accepted_tokens, a->next_token, a->layers, a->H, a->hd, a->dtype, a->k_cache,
                                 a->v_cache, a->Lcap, a->seq_lens, ws_post, stream, true);
}
