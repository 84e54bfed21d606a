/*
 * libmedusa_b200 -- one Medusa verification step on NVIDIA B200 (sm_100a).
 *
 * The step (sources are cited by page title and section):
 *   S1-S3  medusa_heads_topk        K residual heads on the last hidden state,
 *                                   each with its own vocabulary projection,
 *                                   and the top-k tokens of every head.
 *          ["Medusa API参考：核心函数与类详解", MedusaConfig / MedusaModelABC;
 *           "Medusa — 让大模型自己同时猜好几个 token", 是什么 and 核心要点]
 *   S4     medusa_build_tree        candidate tree tokens (tree_indices gather),
 *                                   per-path candidates (retrieve_indices) and
 *                                   position ids.
 *          ["Medusa API参考", 核心功能函数: generate_candidates, tree_decoding]
 *   S5     medusa_tree_attention    attention of the T tree tokens against the
 *                                   cached prefix and their own ancestors.
 *          ["Medusa — 让大模型…", 核心要点 (tree attention) and 实践案例 case 3]
 *   S6     medusa_evaluate_posterior greedy or typical acceptance, best path,
 *                                   accept length, accepted tokens, next token.
 *          ["Medusa API参考", evaluate_posterior; "Medusa — 让大模型…", 核心要点,
 *           实践案例 case 1 step 4, 学到什么]
 *   S7     medusa_accept_kv         move the accepted path's K/V rows to the
 *                                   end of the cached prefix.
 *          ["Medusa — 让大模型…", 实践案例 case 1 step 4]
 *   S3 over G ranks  medusa_topk_merge  the global top-k from the top-k lists
 *                                   of G vocabulary shards (rows of Wout
 *                                   split across ranks, lists all-gathered).
 *   S5 over G ranks  medusa_tree_attention_split, medusa_attention_combine
 *                                   attention over one window of the cached
 *                                   prefix per rank, then the log-sum-exp
 *                                   combine of the gathered partials.
 *   medusa_step                     S1..S7 in order on one stream.
 *
 * Conventions shared by every call:
 *   - Tensors are caller-owned DEVICE pointers unless a comment says "host".
 *     No call allocates device memory, except medusa_tree_create (which owns
 *     the tree tables it uploads).  No call synchronises its stream; all work
 *     is enqueued on the caller's cudaStream_t.
 *   - Arguments are checked on the host before any launch; a bad argument
 *     returns MEDUSA_ERR_INVALID_ARG / MEDUSA_ERR_UNSUPPORTED and launches
 *     nothing.  A launch failure returns MEDUSA_ERR_CUDA.  Conditions that
 *     only the device can see (a sequence length that overflows the cache, a
 *     bounded wait that ran out) set a per-device status word that
 *     medusa_device_status() reads back; such a call still returns MEDUSA_OK.
 *   - medusa_last_error() gives a thread-local message for the last failure.
 *   - Index tensors are int32.  Logits (head and base) are always fp32.
 *   - "workspace" buffers are caller-owned device memory of at least the size
 *     the matching *_workspace_size() call returns, 256-byte aligned.  They
 *     must be zero-filled once before their first use (cudaMemsetAsync); each
 *     call leaves its counters at zero again when it completes.  After a call
 *     that reported a device-side error, zero the workspace again.  Calls
 *     that share a workspace must not run concurrently.
 *
 * Shapes (contiguous, row-major):
 *   h       [B, d]            hidden state at the last cached position
 *   W1      [K, d, d]         residual-block weight, out x in
 *   b1      [K, d]            residual-block bias
 *   Wout    [K, V, d]         per-head vocabulary projection, no bias
 *   q, out  [layers, B, T, H, hd]           tree queries / attention output (fp32)
 *   k_cache, v_cache [layers, B, H, Lcap, hd] with the tree's own K/V already
 *                     at rows seq_lens[b] .. seq_lens[b]+T-1 of every slice
 *   base logits [B, T, V]     base-model logits at every tree node (fp32)
 */
#ifndef MEDUSA_B200_H
#define MEDUSA_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MEDUSA_ABI_VERSION 7
#define MEDUSA_MAX_T 256     /* tree tokens including the root */
#define MEDUSA_MAX_K 16      /* heads (so tree depth <= 16) */
#define MEDUSA_MAX_TOPK 32   /* candidates per head */
#define MEDUSA_MAX_B 64      /* sequences per call */
#define MEDUSA_MAX_SHARDS 64 /* vocabulary shards merged by medusa_topk_merge */

typedef enum medusa_status {
  MEDUSA_OK = 0,
  MEDUSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad tree, bad mode */
  MEDUSA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels handle */
  MEDUSA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  MEDUSA_ERR_TIMEOUT = 4,       /* device status: a bounded wait ran out */
  MEDUSA_ERR_DEVICE_CHECK = 5   /* device status: a device-side check failed */
} medusa_status_t;

typedef enum medusa_dtype { MEDUSA_F32 = 0, MEDUSA_BF16 = 1 } medusa_dtype_t;

/* Acceptance rule of the posterior (S6).  NUCLEUS is the API's
 * sampling='nucleus' with top_p ("Medusa API参考", evaluate_posterior); the
 * pages name it without defining it, and this library reads it in the form
 * of the typical rule: a child is accepted when its token lies in the top_p
 * nucleus of its parent's tempered distribution. */
typedef enum medusa_mode { MEDUSA_GREEDY = 0, MEDUSA_TYPICAL = 1, MEDUSA_NUCLEUS = 2 } medusa_mode_t;

typedef struct medusa_tree medusa_tree_t;

/* Thread-local text of the last error raised by a call on this thread. */
const char* medusa_last_error(void);

/* MEDUSA_ABI_VERSION of the loaded library. */
int medusa_abi_version(void);

/* Reads (and, when clear != 0, resets) the current device's status word:
 * MEDUSA_OK, MEDUSA_ERR_TIMEOUT or MEDUSA_ERR_DEVICE_CHECK.  Synchronises the
 * device.  *detail receives a kernel-specific code (may be NULL). */
medusa_status_t medusa_device_status(int32_t* status, int32_t* detail, int clear);

/* Test hook of the failure-detection path; not for production use.  Later
 * launches of the batch-1 / fp32 heads kernel (medusa_heads_topk with B = 1,
 * or fp32 weights) wait, between the residual block and the vocabulary
 * projection, for extra_arrivals more CTAs than the launch has, so with
 * extra_arrivals > 0 that wait cannot be satisfied, and that wait gives up
 * after limit_ns (0: the default of about 2 s).  A wait that gives up sets
 * the device status (MEDUSA_ERR_TIMEOUT, detail 1 for this wait), the
 * kernel's other roles stop waiting as soon as they see it, its copies in
 * flight land, and it returns without writing the top-k; zero the workspace
 * before the next call.
 * medusa_test_heads_wait(0, 0) restores the defaults.  Process-wide.
 * Errors: INVALID_ARG unless 0 <= extra_arrivals <= 1024 and limit_ns >= 0.
 * The pages have no counterpart. */
medusa_status_t medusa_test_heads_wait(int extra_arrivals, long long limit_ns);

/* ------------------------------------------------------------------------ */
/* Candidate tree                                                            */
/* ------------------------------------------------------------------------ */

/* Host.  The static tree used by the Vicuna-shaped workloads: all rank tuples
 * of length 1..K with entries in [0, topk), ordered by (rank sum, length,
 * lexicographic), first n_nodes kept (a prefix-closed set).
 * ranks: host [n_nodes * K], tuple i in ranks[i*K .. i*K+lens[i]-1], rest 0;
 * lens: host [n_nodes].  The pages name the tree (medusa_choices of
 * medusa_generate, "Medusa API参考") but not this construction; it is the
 * reading used for the Vicuna-shaped workloads.  Errors: INVALID_ARG when
 * n_nodes exceeds the number of tuples or MEDUSA_MAX_T-1. */
medusa_status_t medusa_tree_choices_ranksum(int K, int topk, int n_nodes,
                                            int32_t* ranks, int32_t* lens);

/* Host (+ device when upload != 0).  Builds the tree tables from n_nodes rank
 * tuples (same packing as above; any order).  Node 0 is the root; nodes are
 * laid out breadth first, (length, lexicographic).  Node (r1..rj) takes head
 * j's rank-rj token ["Medusa — 让大模型…", 核心要点; 实践案例 case 3].
 * Checks: 1 <= len <= K <= MEDUSA_MAX_K, 0 <= rank < topk <= MEDUSA_MAX_TOPK,
 * no duplicates, every tuple's parent present, T = n_nodes+1 <= MEDUSA_MAX_T.
 * With upload != 0 the tables are copied (synchronously) to the current
 * device and the tree may only be used on that device.  The caller owns
 * *out and frees it with medusa_tree_destroy. */
medusa_status_t medusa_tree_create(const int32_t* ranks, const int32_t* lens, int n_nodes,
                                   int K, int topk, int upload, medusa_tree_t** out);

void medusa_tree_destroy(medusa_tree_t* tree);

/* Host.  T tree tokens (root included), P root-to-leaf paths, D max depth. */
medusa_status_t medusa_tree_info(const medusa_tree_t* tree, int32_t* T, int32_t* P, int32_t* D);

/* Host copies of the tables (any pointer may be NULL):
 *   tree_indices [T]  index into [root, head1 top-k, ..., headK top-k]
 *   parent [T] (-1 for the root), depth [T]
 *   retrieve [P * (D+1)]  node ids along each path, leaf order, padded -1
 *   anc [T * ((T+63)/64)] bit j of row i set when node j is i or an ancestor */
medusa_status_t medusa_tree_tables(const medusa_tree_t* tree, int32_t* tree_indices,
                                   int32_t* parent, int32_t* depth, int32_t* retrieve,
                                   uint64_t* anc);

/* ------------------------------------------------------------------------ */
/* S1-S3: heads and top-k                                                    */
/* ------------------------------------------------------------------------ */

size_t medusa_heads_workspace_size(int B, int d, int V, int K, int topk);

/* u[b,k] = h[b] + SiLU(W1[k] h[b] + b1[k])   (fp32, kept unrounded)
 * z[b,k] = Wout[k] u[b,k]                     (fp32 head logits)
 * topk_ids/vals[b,k,:] = the topk largest z[b,k,:], value descending, lower
 * token id first on equal values.
 * dtype: element type of h, W1, b1, Wout (MEDUSA_F32 or MEDUSA_BF16); all
 * arithmetic is fp32.  head_logits [B,K,V] fp32 may be NULL (not written).
 * topk_ids [B,K,topk] int32, topk_vals [B,K,topk] fp32.
 * Supported: d a multiple of 256 (bf16) / 128 (f32), d <= 8192 (bf16) /
 * 4096 (f32), topk <= min(V, MEDUSA_MAX_TOPK), 1 <= B <= MEDUSA_MAX_B,
 * 1 <= K <= MEDUSA_MAX_K.  Pointers must be 16-byte aligned. */
medusa_status_t medusa_heads_topk(const void* h, const void* W1, const void* b1,
                                  const void* Wout, int B, int d, int V, int K, int topk,
                                  medusa_dtype_t dtype, float* head_logits, int32_t* topk_ids,
                                  float* topk_vals, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* The same computation as medusa_heads_topk for callers that cannot allocate
 * device memory: a host that reserves all device memory up front and gives
 * this library no allocator, or code running where allocating is not
 * allowed.  Instead of a caller workspace it uses a fixed 4 MiB scratch array
 * that the library keeps in device memory (every GPU that loads the library
 * holds those 4 MiB until the process exits); it calls no cudaMalloc,
 * cudaFree or allocating routine.  The paper has no counterpart: this is an
 * interface choice of this library.
 *  - Arguments, layouts and outputs are those of medusa_heads_topk.
 *  - Shapes whose scratch need (medusa_heads_workspace_size) exceeds 4 MiB
 *    are rejected with MEDUSA_ERR_UNSUPPORTED before anything is enqueued.
 *  - The first call on a device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *    The address is kept until the process exits: do not use this call on a
 *    device after resetting it (cudaDeviceReset).
 *  - Invalid arguments are refused before anything is enqueued; a refused
 *    call leaves the array as it was.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; each call clears the part it uses on `stream` before launching.
 *    Calls whose work overlaps on the GPU (other streams, other threads)
 *    race on the array: serialise them. */
medusa_status_t medusa_heads_topk_noalloc(const void* h, const void* W1, const void* b1,
                                          const void* Wout, int B, int d, int V, int K, int topk,
                                          medusa_dtype_t dtype, float* head_logits,
                                          int32_t* topk_ids, float* topk_vals, cudaStream_t stream);

/* S3 with the vocabulary split over G ranks.  Rank g holds rows
 * [row0[g], row0[g] + n_g) of every Wout[k] (n_g = row0[g+1] - row0[g], the
 * last shard ends at V) as a [K, n_g, d] array and runs medusa_heads_topk on
 * it with V = n_g, which gives top-k lists with shard-local ids; the G lists
 * are then gathered on every rank (an all-gather of G*B*K*topk values and
 * ids, a few KB).  This call turns the gathered lists into the lists that
 * medusa_heads_topk gives on the whole Wout:
 *   vals, ids  [G, B, K, topk] device (ids shard-local, as written by
 *              medusa_heads_topk)
 *   row0       [G] HOST int32: row0[0] = 0, each shard at least topk rows
 *              (row0[g+1] - row0[g] >= topk and V - row0[G-1] >= topk)
 *   out_vals   [B, K, topk] fp32, out_ids [B, K, topk] int32 (global ids):
 *              the topk best of the G*topk candidates, value descending,
 *              lower token id first on equal values (NaN last).
 * The heads kernel computes each logit the same way whatever V is, so the
 * result equals the unsplit top-k bit for bit.  Pure selection; no
 * workspace.  1 <= G <= MEDUSA_MAX_SHARDS, 1 <= B <= MEDUSA_MAX_B,
 * 1 <= K <= MEDUSA_MAX_K, 1 <= topk <= MEDUSA_MAX_TOPK.
 * ["Medusa — 让大模型自己同时猜好几个 token", 核心要点: per-head top-k] */
medusa_status_t medusa_topk_merge(const float* vals, const int32_t* ids, const int32_t* row0, int G,
                                  int V, int B, int K, int topk, float* out_vals, int32_t* out_ids,
                                  cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* S4: candidate assembly                                                    */
/* ------------------------------------------------------------------------ */

/* flat[b] = [root_tokens[b], topk_ids[b,0,:], ..., topk_ids[b,K-1,:]]
 * tree_tokens[b,i]    = flat[b][tree_indices[i]]                [B, T]
 * candidates[b,p,j]   = tree_tokens[b, retrieve[p,j]] or -1      [B, P, D+1]
 * position_ids[b,i]   = seq_lens[b] + depth[i]                   [B, T]
 * topk_ids must be [B, K_tree, topk_tree] for the tree's own K and topk. */
medusa_status_t medusa_build_tree(const medusa_tree_t* tree, int B, const int32_t* root_tokens,
                                  const int32_t* topk_ids, const int32_t* seq_lens,
                                  int32_t* tree_tokens, int32_t* candidates,
                                  int32_t* position_ids, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* S5: tree attention                                                        */
/* ------------------------------------------------------------------------ */

size_t medusa_attention_workspace_size(const medusa_tree_t* tree, int layers, int B, int H,
                                       int hd, medusa_dtype_t dtype);

/* For every layer l, sequence b, head e and tree node i (L = seq_lens[b]):
 *   out[l,b,i,e] = sum_j softmax_j(scale * q[l,b,i,e] . k[l,b,e,j]) v[l,b,e,j]
 * over j in {0..L-1} and {L+t : t is i or an ancestor of i}.
 * q/out [layers,B,T,H,hd]; caches [layers,B,H,Lcap,hd]; dtype is that of q
 * and the caches; out is always fp32 (fp32 softmax and accumulation).  Requires seq_lens[b]+T <= Lcap (a
 * violation sets MEDUSA_ERR_DEVICE_CHECK and leaves that slice unwritten).
 * Supported: hd <= 256 and a multiple of 32 (bf16 hd = 128 takes the
 * tensor-core kernel).  Pointers 16-byte aligned. */
medusa_status_t medusa_tree_attention(const medusa_tree_t* tree, int layers, int B, int H,
                                      int hd, medusa_dtype_t dtype, const void* q,
                                      const void* k_cache, const void* v_cache, int Lcap,
                                      const int32_t* seq_lens, float scale, void* out,
                                      void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream);

/* S5 split along the cached prefix over G ranks.  Caches keep the layout of
 * medusa_tree_attention ([layers, B, H, Lcap, hd]); a rank's call uses only
 * the rows of its own window, so the other rows may hold anything (they are
 * read past a window's end only to fill a tile, and masked).  Rank `rank` attends to
 * prefix rows [lo, hi) = [floor(L r / G), floor(L (r+1) / G)) of every slice
 * (L = seq_lens[b]) and, when rank = G - 1, to the tree rows node i may see
 * (as medusa_tree_attention), and writes
 *   out [layers, B, T, H, hd] fp32: attention over that window (normalised
 *                over the window alone)
 *   lse [layers, B, T, H] fp32: ln sum exp(scale q.k) over the window.
 * medusa_attention_combine over the G ranks' (out, lse), gathered in rank
 * order, gives medusa_tree_attention's output.  Supported: bf16, hd = 128,
 * trees of at most 64 tokens (else MEDUSA_ERR_UNSUPPORTED).  Every
 * seq_lens[b] must be >= G (an empty window sets MEDUSA_ERR_DEVICE_CHECK and
 * leaves that slice unwritten), as must seq_lens[b] + T <= Lcap.
 * 1 <= G <= MEDUSA_MAX_SHARDS, 0 <= rank < G.  No workspace.
 * The pages have no counterpart: the split is this library's multi-GPU
 * option; the combine is the log-sum-exp identity. */
medusa_status_t medusa_tree_attention_split(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                            medusa_dtype_t dtype, const void* q, const void* k_cache,
                                            const void* v_cache, int Lcap, const int32_t* seq_lens,
                                            float scale, int rank, int G, float* out, float* lse,
                                            cudaStream_t stream);

/* Attention over the union of G disjoint key windows from each window's
 * normalised output and lse:
 *   outs [G, rows, hd] fp32, lses [G, rows] fp32 (rows = layers*B*T*H)
 *   out [rows, hd] = sum_g exp(lse_g - lse) outs[g],  lse = ln sum_g exp(lse_g)
 *   lse_out [rows] (may be NULL) receives lse.
 * A row whose every lse_g is -inf gets out = 0, lse = -inf.  hd a multiple
 * of 4 in [4, 1024]; outs and out 16-byte aligned; out must not overlap
 * outs.  1 <= G <= MEDUSA_MAX_SHARDS. */
medusa_status_t medusa_attention_combine(int G, int64_t rows, int hd, const float* outs, const float* lses,
                                         float* out, float* lse_out, cudaStream_t stream);

/* The combine of medusa_attention_combine split across the ranks, so that the
 * ranks exchange only their lse values and then sum their outputs (an
 * all-reduce of one output per rank instead of an all-gather of G):
 *   lses [G, rows] fp32   every rank's lse, gathered in rank order
 *   part [rows, hd] fp32  rank `rank`'s own window output, scaled in place:
 *                         part[row] *= exp(lses[rank, row] - lse[row]),
 *                         lse = ln sum_g exp(lses[g, row])
 *   lse_out [rows] (may be NULL) receives lse.
 * The sum over ranks of the scaled parts equals medusa_attention_combine's
 * out.  A row whose every lse_g is -inf gets part = 0, lse = -inf.  hd a
 * multiple of 4 in [4, 1024]; part 16-byte aligned; 1 <= G <=
 * MEDUSA_MAX_SHARDS, 0 <= rank < G.  The pages have no counterpart (this is
 * the library's multi-GPU option). */
medusa_status_t medusa_attention_rescale(int G, int rank, int64_t rows, int hd, const float* lses, float* part,
                                         float* lse_out, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* S6: posterior                                                             */
/* ------------------------------------------------------------------------ */

size_t medusa_posterior_workspace_size(const medusa_tree_t* tree, int B);

/* Per node i of sequence b: g_i = argmax_v logits[b,i,v] (lowest id on ties);
 * typical / nucleus: p_i = softmax(logits[b,i,:] / temperature),
 * H_i = -sum p ln p, thr_i = min(eps, alpha * exp(-H_i)); the nucleus N_i
 * holds the tokens, in order of p descending (lower id first on equal
 * values), whose preceding mass is below top_p.
 * Path p accepts depth j when candidates[b,p,j] == g_parent (GREEDY),
 * p_parent(candidates[b,p,j]) > thr_parent (TYPICAL), or candidates[b,p,j]
 * is in N_parent (NUCLEUS); acc_p counts leading accepted depths.
 * best_path[b] = lowest p with the largest acc_p; accept_len[b] = a = acc_best
 * (0..D); accepted_tokens[b, 0..D] = candidates[b, best, 0..a], -1 after.
 * next_token[b], at node n = retrieve[best, a]: g_n when uniforms is NULL or
 * mode is GREEDY; otherwise the first token v, in id order, whose cumulative
 * weight exceeds uniforms[b] * (total weight), the weights being p_n (TYPICAL)
 * or p_n restricted to N_n (NUCLEUS): a draw by inverse CDF with the
 * caller's uniform (uniforms [B] fp32 in [0, 1), device).
 * TYPICAL and NUCLEUS need temperature > 0; NUCLEUS needs 0 < top_p <= 1
 * (defaults of the pages: eps = 0.09, alpha = 0.3, top_p = 0.8).
 * logits [B,T,V] fp32; candidates [B,P,D+1]. */
medusa_status_t medusa_evaluate_posterior(const medusa_tree_t* tree, int B, int V,
                                          const float* logits, const int32_t* candidates,
                                          medusa_mode_t mode, float temperature, float eps,
                                          float alpha, float top_p, const float* uniforms,
                                          int32_t* best_path, int32_t* accept_len,
                                          int32_t* accepted_tokens, int32_t* next_token,
                                          void* workspace, size_t workspace_bytes,
                                          cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* S7: keep the accepted path's K/V                                          */
/* ------------------------------------------------------------------------ */

/* In place, for every layer, sequence b and head (L = seq_lens[b], a =
 * accept_len[b], n_j = retrieve[best_path[b], j]):
 *   cache row L+j  <-  cache row L+n_j,   j = 0..a   (K and V)
 * read before any write (n_j can equal a destination of a later j), then
 * seq_lens[b] = L + a + 1. */
medusa_status_t medusa_accept_kv(const medusa_tree_t* tree, int layers, int B, int H, int hd,
                                 medusa_dtype_t dtype, void* k_cache, void* v_cache, int Lcap,
                                 int32_t* seq_lens, const int32_t* best_path,
                                 const int32_t* accept_len, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* The base model's forward over the tree tokens (tree_decoding)             */
/* ------------------------------------------------------------------------ */

/* One LLaMA (Vicuna) decoder layer's weights, bf16 device pointers, hd = 128
 * (H = D / 128 heads, D <= 8192), F the feed-forward width (multiples of 128):
 *   attn_norm, mlp_norm [D]   RMSNorm weights (eps 1e-6)
 *   wqkv  [3D, D]  the rows of Wq, Wk and Wv (out x in) in that order, each
 *                  head's 128 rows packed so that row 2j is feature j and row
 *                  2j+1 feature j + 64 (the two features one rotary pair turns)
 *   wo    [D, D]   output projection
 *   wgu   [2F, D]  gate and up projections interleaved: row 2j is W_gate row
 *                  j, row 2j+1 is W_up row j
 *   wdown [D, F]   down projection
 * The packing only reorders rows; medusa_decoder_pack_rows gives the order. */
typedef struct medusa_decoder_layer {
  const void* attn_norm;
  const void* wqkv;
  const void* wo;
  const void* mlp_norm;
  const void* wgu;
  const void* wdown;
} medusa_decoder_layer_t;

typedef struct medusa_decoder {
  int layers, D, F, V;
  const void* embed;                    /* [V, D] bf16 */
  const medusa_decoder_layer_t* layer;  /* HOST array of `layers` entries (device pointers inside) */
  const void* final_norm;               /* [D] bf16 */
  const void* lm_head;                  /* [V, D] bf16, no bias */
} medusa_decoder_t;

/* Host.  The source row of every packed row: for which = 0 (wqkv, D rows of
 * one of Wq / Wk / Wv; apply it to each of the three) out[r] = the row of
 * the unpacked matrix that packed row r holds (r < D); for which = 1 (wgu,
 * 2F rows) out[r] = j for W_gate row j (r = 2j) and F + j for W_up row j
 * (r = 2j + 1), indexing the unpacked [W_gate; W_up].  INVALID_ARG unless D
 * (which 0) is a multiple of 128 and n > 0. */
medusa_status_t medusa_decoder_pack_rows(int which, int n, int32_t* out);

size_t medusa_tree_decode_workspace_size(const medusa_tree_t* tree, const medusa_decoder_t* model, int B);

/* The base model's forward over the T tree tokens of each of B sequences
 * ["Medusa API参考", 核心功能函数: tree_decoding (medusa_position_ids =
 * prefix length + depth, the tree mask, the cached K/V); "基于 Medusa 头的投机
 * 解码架构", 性能基准测试: Vicuna bases]: embedding of tree_tokens [B, T], for
 * every layer l (x the fp32 residual stream of the B*T tokens)
 *   x += Wo . tree_attention(RoPE(Wq n), RoPE(Wk n), Wv n),  n = RMSNorm(x)
 *   x += Wdown (SiLU(Wgate n) * (Wup n)),                   n = RMSNorm(x)
 * with RoPE at position seq_lens[b] + depth(node) (pair i with i + 64, base
 * 10000), the tree's own k and v written to cache rows seq_lens[b] + node of
 * layer l (caches [layers, B, H, Lcap, 128] bf16; rows below seq_lens[b]
 * hold the prefix), attention as medusa_tree_attention; then
 *   logits [B*T, V] fp32 = lm_head . RMSNorm(x),   hidden [B*T, D] fp32 = x
 * (hidden may be NULL).  The normalised activations, q/k/v, the attention
 * output and the SwiGLU activation are rounded to bf16 between the products
 * (fp32 accumulation).  Requires seq_lens[b] + T <= Lcap (a violation sets
 * MEDUSA_ERR_DEVICE_CHECK); a token outside [0, V) sets
 * MEDUSA_ERR_DEVICE_CHECK.  Every matrix product streams its weights once
 * per pass of up to 256 of the B*T tree tokens.  Pointers 16-byte aligned. */
medusa_status_t medusa_tree_decode(const medusa_tree_t* tree, const medusa_decoder_t* model, int B,
                                   const int32_t* tree_tokens, void* k_cache, void* v_cache, int Lcap,
                                   const int32_t* seq_lens, float* logits, float* hidden, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Greedy generation                                                         */
/* ------------------------------------------------------------------------ */

size_t medusa_generate_workspace_size(const medusa_tree_t* tree, const medusa_decoder_t* model);

/* Greedy Medusa decoding of one sequence ("Medusa API参考", MedusaModelABC
 * medusa_generate; "Medusa — 让大模型自己同时猜好几个 token", 实践案例 case 1
 * and 学到什么): the prompt (HOST, n_prompt tokens) goes through the base
 * model in chains of at most 17 tokens, writing cache rows 0 .. n_prompt-1;
 * the base model's arg-max after it is the first root.  Each step then runs
 * the K heads (W1 [K, D, D], b1 [K, D], Wout [K, V, D], bf16, device) on the
 * final-norm hidden state of the last accepted token, builds the candidate
 * tree rooted at the base model's next token, runs the base model over the
 * tree tokens (medusa_tree_decode), accepts greedily, compacts the accepted
 * K/V rows and emits root + accepted tokens.  Caches [layers, 1, H, Lcap,
 * 128] bf16 on the device; their content is overwritten from row 0.
 * out_tokens (HOST, n_new entries) receives the first n_new emitted tokens,
 * out_accept (HOST, max_steps entries) each step's accept length, *n_steps
 * the number of steps.  The host waits for every step (it reads the accept
 * length).  Workspace zero-filled before its first use (counters reset
 * themselves).  INVALID_ARG when the prompt plus one tree does not fit in
 * Lcap, a prompt token is outside [0, V), or the cache or max_steps ran out
 * before n_new tokens (the tokens so far are written). */
/* medusa_generate_greedy's loop with acceptance in `mode` (MEDUSA_GREEDY,
 * MEDUSA_TYPICAL or MEDUSA_NUCLEUS, with temperature, eps, alpha and top_p as
 * medusa_evaluate_posterior; "Medusa API参考", MedusaModelABC medusa_generate:
 * sampling and top_p).  uniforms (HOST, max_steps entries in [0, 1), or NULL)
 * gives step s's draw of the next token (see medusa_evaluate_posterior); the
 * first root, after the prompt, is the base model's arg-max.  Errors as
 * medusa_generate_greedy, plus medusa_evaluate_posterior's argument checks
 * and uniforms outside [0, 1). */
medusa_status_t medusa_generate(const medusa_tree_t* tree, const medusa_decoder_t* model,
                                const void* W1, const void* b1, const void* Wout, medusa_mode_t mode,
                                float temperature, float eps, float alpha, float top_p,
                                const float* uniforms, const int32_t* prompt, int n_prompt, int n_new,
                                void* k_cache, void* v_cache, int Lcap, int32_t* out_tokens,
                                int32_t* out_accept, int max_steps, int32_t* n_steps, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream);

medusa_status_t medusa_generate_greedy(const medusa_tree_t* tree, const medusa_decoder_t* model,
                                       const void* W1, const void* b1, const void* Wout,
                                       const int32_t* prompt, int n_prompt, int n_new,
                                       void* k_cache, void* v_cache, int Lcap,
                                       int32_t* out_tokens, int32_t* out_accept, int max_steps,
                                       int32_t* n_steps, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* The whole step                                                            */
/* ------------------------------------------------------------------------ */

typedef struct medusa_step_args {
  const medusa_tree_t* tree;
  int B, d, V, K, topk;           /* heads */
  int layers, H, hd, Lcap;        /* attention */
  medusa_dtype_t dtype;
  const void* h;
  const void* W1;
  const void* b1;
  const void* Wout;
  const int32_t* root_tokens;     /* [B] the base model's own next token */
  const void* q;
  void* k_cache;
  void* v_cache;
  int32_t* seq_lens;              /* [B], advanced by a+1 */
  const float* base_logits;       /* [B, T, V] */
  float scale;                    /* attention scale, usually 1/sqrt(hd) */
  medusa_mode_t mode;
  float temperature, eps, alpha;
  float* head_logits;             /* nullable */
  int32_t* topk_ids;
  float* topk_vals;
  int32_t* tree_tokens;
  int32_t* candidates;
  int32_t* position_ids;
  void* attn_out;
  int32_t* best_path;
  int32_t* accept_len;
  int32_t* accepted_tokens;
  int32_t* next_token;
  /* Optional (may be null): events the step waits for on `stream` right
   * before tree attention (q and the tree's K/V rows in the caches are ready)
   * and right before the posterior (base_logits ready), so that a caller can
   * copy those inputs on another stream while the heads run. */
  cudaEvent_t attn_inputs_ready;
  cudaEvent_t posterior_inputs_ready;
  float top_p;                    /* nucleus acceptance (MEDUSA_NUCLEUS) */
  const float* uniforms;          /* [B] or NULL: draws for the next token (see medusa_evaluate_posterior) */
} medusa_step_args_t;

size_t medusa_step_workspace_size(const medusa_step_args_t* args);

/* The computations of medusa_heads_topk, medusa_build_tree,
 * medusa_tree_attention, medusa_evaluate_posterior and medusa_accept_kv, in
 * that order, on stream, with the same outputs.  The candidate tree is built
 * by the heads' last CTA: S1-S4 take one launch at batch 1 (and per group of
 * up to four sequences for fp32), two per pass of up to 16 sequences on the
 * tensor cores (bf16, B >= 2).  Tree attention takes one launch (two for
 * trees of 129-192 tokens), and the posterior and the compaction share one (S6-S7):
 * three launches per step at batch 1.  Capturable in a CUDA graph
 * (no allocation, no synchronisation).  Validation errors are returned
 * before anything is enqueued. */
medusa_status_t medusa_step(const medusa_step_args_t* args, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/* Per-step inputs and results of medusa_step_host, in host memory.  Every
 * pointer is host memory (page-locked, for copies that overlap the step;
 * pageable memory works but the driver stages it) or NULL: a NULL input is
 * already in its device buffer of the step's args, a NULL result is not
 * read back.  A device or managed pointer here is INVALID_ARG. */
typedef struct medusa_step_host_io {
  const void* h;                  /* [B, d] dtype -> args->h */
  const int32_t* root_tokens;     /* [B] -> args->root_tokens */
  const int32_t* seq_lens;        /* [B] -> args->seq_lens; read on the host during the call to place
                                   * the tree rows; required when k_tree or v_tree is given */
  const float* uniforms;          /* [B] -> args->uniforms (which must then be non-NULL) */
  const void* q;                  /* [layers, B, T, H, hd] dtype -> args->q */
  const void* k_tree;             /* [layers, B, H, T, hd] dtype: the tree tokens' own key and value */
  const void* v_tree;             /*   rows, copied to cache rows seq_lens[b] .. seq_lens[b] + T - 1 */
  const float* base_logits;       /* [B, T, V] -> args->base_logits */
  int32_t* best_path;             /* [B] */
  int32_t* accept_len;            /* [B] */
  int32_t* accepted_tokens;       /* [B, D + 1] */
  int32_t* next_token;            /* [B] */
  int32_t* seq_lens_out;          /* [B]: the lengths after the step */
  cudaStream_t copy_stream;       /* second stream for q, the tree's K/V rows and base_logits, or NULL */
} medusa_step_host_io_t;

/* medusa_step with its per-step inputs copied in from host memory and its
 * results copied back (the end-to-end form of the step: "Medusa API参考",
 * MedusaModelABC medusa_generate calls the verification once per generated
 * block and reads the accepted tokens on the host).  Enqueued in this order:
 * h, root_tokens, seq_lens and uniforms on stream; q, k_tree / v_tree (one
 * 3-D copy per sequence into the caches) and then base_logits on
 * copy_stream, after all work enqueued earlier on stream; the step, which
 * waits for copy_stream right before tree attention and right before the
 * posterior, so the copies overlap the heads; the results on stream.  With
 * copy_stream NULL every copy goes on stream ahead of the step.  Returns
 * once all of it is enqueued: synchronise stream before reading the host
 * results or reusing the host inputs.  args->attn_inputs_ready and
 * posterior_inputs_ready must be NULL (this call supplies its own events).
 * Every check of medusa_step, and of io (host pointers, seq_lens[b] + T <=
 * Lcap on the host copy), happens before anything is enqueued.  Not
 * capturable in a CUDA graph (it reads seq_lens on the host and creates
 * events). */
medusa_status_t medusa_step_host(const medusa_step_args_t* args, const medusa_step_host_io_t* io,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MEDUSA_B200_H */
