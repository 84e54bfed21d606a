// Internal declarations shared by the host-side sources of libmedusa_b200.
#pragma once

#include <cstdint>
#include <string>
#include <vector>
#include <utility>

#include <cuda_runtime.h>

#include "medusa_b200.h"

namespace medusa {

// Device-side view of a tree, passed to kernels by value.
struct TreeDev {
  int T, P, D, K, topk, W;        // W = 64-bit words per ancestor-mask row
  const int32_t* tree_indices;    // [T]
  const int32_t* parent;          // [T]
  const int32_t* depth;           // [T]
  const int32_t* retrieve;        // [P * (D+1)]
  const uint64_t* anc;            // [T * W]
  const int32_t* path_of;         // [T] lowest path index through each node
};

}  // namespace medusa

struct medusa_tree {
  int T = 0, P = 0, D = 0, K = 0, topk = 0, W = 0;
  int device = -1;                // device holding the uploaded tables, -1 if none
  std::vector<std::vector<int32_t>> nodes;   // rank tuple of every node, nodes[0] empty
  std::vector<int32_t> tree_indices, parent, depth, retrieve, path_of;
  std::vector<uint64_t> anc;
  void* dev_block = nullptr;      // one device allocation holding every table
  medusa::TreeDev dev{};
};

namespace medusa {

// Thread-local error text; returns the status for convenient `return fail(...)`.
medusa_status_t fail(medusa_status_t st, const std::string& msg);
medusa_status_t cuda_fail(const char* what, int err);

// Status word on the current device (set by kernels, read by medusa_device_status).
medusa_status_t device_status_read(int32_t* status, int32_t* detail, int clear);

// Number of SMs of the current device (cached per device).
int sm_count();

// S4 outputs, when the heads kernel also builds the candidate tree (medusa_step).
struct TreeBuild {
  TreeDev t;
  const int32_t* root_tokens;   // [B]
  const int32_t* seq_lens;      // [B]
  int32_t* tree_tokens;         // [B, T]
  int32_t* candidates;          // [B, P, D+1]
  int32_t* position_ids;        // [B, T]
};

// Host-side argument checks of medusa_heads_topk (api.cu); nothing is enqueued.
medusa_status_t check_heads(const void* h, const void* W1, const void* b1, const void* Wout, int B, int d, int V,
                            int K, int topk, medusa_dtype_t dtype, const float* head_logits, const int32_t* topk_ids,
                            const float* topk_vals, const void* ws, size_t ws_bytes);

// Every host-side check of medusa_step (api.cu); nothing is enqueued.
medusa_status_t check_step(const medusa_step_args_t* args, const void* ws, size_t ws_bytes);

// Host-side checks of the base model and the tree for medusa_tree_decode (api.cu).
medusa_status_t check_decoder(const medusa_tree_t* tree, const medusa_decoder_t* m, int B, const char* fn);

// Host-side checks of medusa_evaluate_posterior (api.cu).
medusa_status_t check_posterior(const medusa_tree_t* tree, int B, int V, const float* logits,
                                const int32_t* candidates, medusa_mode_t mode, float temperature, float eps,
                                float alpha, float top_p, const int32_t* best_path, const int32_t* accept_len,
                                const int32_t* accepted_tokens, const int32_t* next_token, const void* ws,
                                size_t ws_bytes);

// Kernel launchers (heads.cu, tree_kernels.cu, attention.cu, posterior.cu, accept.cu).
size_t heads_workspace_bytes(int B, int d, int V, int K, int topk);
medusa_status_t launch_heads(const void* h, const void* W1, const void* b1, const void* Wout,
                             int B, int d, int V, int K, int topk, medusa_dtype_t dtype,
                             float* head_logits, int32_t* topk_ids, float* topk_vals, void* ws,
                             cudaStream_t stream, const TreeBuild* build = nullptr);

// The tensor-core heads (heads_tc.cu) for 2..16 sequences per pass, bf16, d a
// multiple of 128; launch_heads dispatches to it.
bool heads_tc_supported(int B, int d, medusa_dtype_t dtype);
size_t heads_tc_workspace_bytes(int B, int d, int V, int K, int topk);
medusa_status_t launch_heads_tc(const void* h, const void* W1, const void* b1, const void* Wout, int B, int d, int V,
                                int K, int topk, float* head_logits, int32_t* topk_ids, float* topk_vals, void* ws,
                                cudaStream_t stream, const TreeBuild* build);

medusa_status_t launch_build_tree(const TreeDev& t, int B, const int32_t* root_tokens,
                                  const int32_t* topk_ids, const int32_t* seq_lens,
                                  int32_t* tree_tokens, int32_t* candidates,
                                  int32_t* position_ids, cudaStream_t stream);

size_t attention_workspace_bytes(const TreeDev& t, int layers, int B, int H, int hd,
                                 medusa_dtype_t dtype);
// `pdl`: launch with programmatic stream serialisation (only inside medusa_step,
// where the preceding kernel is this library's own and the kernel waits for it
// before it touches that kernel's outputs).
medusa_status_t launch_attention(const TreeDev& t, int layers, int B, int H, int hd,
                                 medusa_dtype_t dtype, const void* q, const void* k_cache,
                                 const void* v_cache, int Lcap, const int32_t* seq_lens,
                                 float scale, void* out, void* ws, cudaStream_t stream, bool pdl = false);
// bf16, hd 128 only: the base forward's attention, its output bf16 [B, T, H, 128],
// launched to overlap the preceding kernel (AttnOut).
medusa_status_t launch_attention_bf16_out(const TreeDev& t, int B, int H, const void* q, const void* k_cache,
                                          const void* v_cache, int Lcap, const int32_t* seq_lens, float scale,
                                          uint16_t* out, cudaStream_t stream);

size_t posterior_workspace_bytes(const TreeDev& t, int B);
medusa_status_t launch_posterior(const TreeDev& t, int B, int V, const float* logits,
                                 const int32_t* candidates, medusa_mode_t mode, float temperature,
                                 float eps, float alpha, float top_p, const float* uniforms, int32_t* best_path,
                                 int32_t* accept_len, int32_t* accepted_tokens, int32_t* next_token, void* ws,
                                 cudaStream_t stream, bool pdl = false);
// S6 and S7 in one launch (medusa_step): the posterior's node CTAs, then
// compaction CTAs that wait for every sequence's walk; the walk advances seq_lens.
medusa_status_t launch_posterior_accept(const TreeDev& t, int B, int V, const float* logits,
                                        const int32_t* candidates, medusa_mode_t mode, float temperature, float eps,
                                        float alpha, float top_p, const float* uniforms, int32_t* best_path,
                                        int32_t* accept_len, int32_t* accepted_tokens, int32_t* next_token,
                                        int layers, int H, int hd, medusa_dtype_t dtype, void* k_cache,
                                        void* v_cache, int Lcap, int32_t* seq_lens, void* ws, cudaStream_t stream,
                                        bool pdl);

medusa_status_t launch_accept_kv(const TreeDev& t, int layers, int B, int H, int hd,
                                 medusa_dtype_t dtype, void* k_cache, void* v_cache, int Lcap,
                                 int32_t* seq_lens, const int32_t* best_path,
                                 const int32_t* accept_len, cudaStream_t stream, bool pdl = false);

// Tree attention over window `rank` of G of each slice's cached prefix (the
// tree's rows with the last window), writing the window's normalised output
// and its lse; then the combine of G such partials.
medusa_status_t launch_attention_split(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype,
                                       const void* q, const void* k_cache, const void* v_cache, int Lcap,
                                       const int32_t* seq_lens, float scale, int rank, int G, float* out,
                                       float* lse, cudaStream_t stream);
medusa_status_t launch_attention_combine(int G, size_t rows, int hd, const float* outs, const float* lses,
                                         float* out, float* lse_out, cudaStream_t stream);

medusa_status_t launch_attention_rescale(int G, int rank, size_t rows, int hd, const float* lses, float* part,
                                         float* lse_out, cudaStream_t stream);

medusa_status_t launch_topk_merge(const float* vals, const int32_t* ids, const int32_t* row0, int G, int B,
                                  int K, int topk, float* out_vals, int32_t* out_ids, cudaStream_t stream);

// The tree-token forward of the base model (decoder.cu).
size_t decoder_workspace_bytes(int ntok, int D, int F, int V);
// The final RMSNorm's bf16 output rows [ntok, D] inside a forward's workspace.
uint16_t* decoder_final_rows(void* ws, int ntok, int D, int F, int V);
medusa_status_t launch_tree_decode(const TreeDev& t, const medusa_decoder_t* m, int B, const int32_t* tree_tokens,
                                   void* k_cache, void* v_cache, int Lcap, const int32_t* seq_lens,
                                   float* logits, float* hidden, void* ws, cudaStream_t stream);

// cuTensorMapEncodeTiled (PFN_cuTensorMapEncodeTiled_v12000), or null.
void* tensor_map_encoder();

// Inside the base forward: the output as bf16 (the next product's operand)
// instead of fp32, and a launch that overlaps the preceding kernel, whose
// outputs (q, the tree's K/V rows) the kernel waits for before its first load.
struct AttnOut {
  uint16_t* bf16 = nullptr;
  bool wait_first = false;
};

// split_r / split_G: attend only to window split_r of split_G of each slice's
// cached prefix (the tree's own rows with the last window); lse, if not null,
// receives ln sum exp(scale q.k) over the window per (layer, seq, node, head).
medusa_status_t launch_attention_tc64(const TreeDev& t, int layers, int B, int H, const void* q,
                                      const void* k_cache, const void* v_cache, int Lcap, const int32_t* seq_lens,
                                      float scale_log2, float* out, int* status, cudaStream_t stream, bool pdl,
                                      int row_lo, int row_hi, int split_r = 0, int split_G = 1,
                                      float* lse = nullptr, const AttnOut& dec = AttnOut{});

medusa_status_t launch_attention_tc128(const TreeDev& t, int layers, int B, int H, const void* q,
                                       const void* k_cache, const void* v_cache, int Lcap, const int32_t* seq_lens,
                                       float scale_log2, float* out, int* status, cudaStream_t stream, bool pdl,
                                       int row_lo, int row_hi, const AttnOut& dec = AttnOut{});

// cudaLaunchKernelEx with programmatic stream serialisation when `pdl` is set.
template <typename... Params, typename... Args>
cudaError_t launch_kernel(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace medusa
