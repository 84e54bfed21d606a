// medusa_step_host: the step with its per-step inputs in host memory.  The
// small inputs the heads need go first on the caller's stream; q, the tree's
// own K/V rows and the base logits go on a second stream while the heads
// run, and the step waits for them only before tree attention and before
// the posterior.  Every copy is one cudaMemcpyAsync / cudaMemcpy3DAsync; the
// tree rows of one sequence, scattered over its (layer, head) cache slices,
// are a single 3-D copy (rows of T*hd elements, heads as the height, layers
// as the depth).
#include "common.cuh"

namespace medusa {
namespace {

size_t dtype_bytes(medusa_dtype_t dt) { return dt == MEDUSA_BF16 ? 2 : 4; }

// Host memory (page-locked or pageable) or NULL.
bool host_or_null(const void* p) {
  if (!p) return true;
  cudaPointerAttributes at{};
  const cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

cudaError_t h2d(void* dst, const void* src, size_t n, cudaStream_t s) {
  return (src && n) ? cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s) : cudaSuccess;
}

cudaError_t d2h(void* dst, const void* src, size_t n, cudaStream_t s) {
  return (dst && n) ? cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, s) : cudaSuccess;
}

// The T tree rows of sequence b for every (layer, head): source
// [layers, B, H, T, hd], destination cache [layers, B, H, Lcap, hd] from row L.
cudaError_t scatter_tree_rows(void* cache, const void* rows, int layers, int B, int H, int T, int hd, int Lcap,
                              int b, int L, size_t esz, cudaStream_t s) {
  cudaMemcpy3DParms p{};
  const size_t row = static_cast<size_t>(T) * hd * esz;
  const size_t pitch = static_cast<size_t>(Lcap) * hd * esz;
  unsigned char* dst = static_cast<unsigned char*>(cache) + (static_cast<size_t>(b) * H * Lcap + L) * hd * esz;
  const unsigned char* src = static_cast<const unsigned char*>(rows) + static_cast<size_t>(b) * H * row;
  p.srcPtr = make_cudaPitchedPtr(const_cast<unsigned char*>(src), row, row, static_cast<size_t>(B) * H);
  p.dstPtr = make_cudaPitchedPtr(dst, pitch, row, static_cast<size_t>(B) * H);
  p.extent = make_cudaExtent(row, H, layers);
  p.kind = cudaMemcpyHostToDevice;
  return cudaMemcpy3DAsync(&p, s);
}

struct Events {
  cudaEvent_t start = nullptr, attn = nullptr, post = nullptr;
  ~Events() {   // safe while still pending: released once they complete
    if (start) cudaEventDestroy(start);
    if (attn) cudaEventDestroy(attn);
    if (post) cudaEventDestroy(post);
  }
  cudaError_t create() {
    cudaError_t e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&attn, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&post, cudaEventDisableTiming);
    return e;
  }
};

}  // namespace
}  // namespace medusa

using namespace medusa;

extern "C" medusa_status_t medusa_step_host(const medusa_step_args_t* a, const medusa_step_host_io_t* io,
                                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!io) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step_host: io is null");
  medusa_status_t st = check_step(a, workspace, workspace_bytes);
  if (st != MEDUSA_OK) return st;
  if (a->attn_inputs_ready || a->posterior_inputs_ready)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step_host: args carry input-ready events (this call sets them)");
  const void* host_ptrs[] = {io->h, io->root_tokens, io->seq_lens, io->uniforms, io->q, io->k_tree, io->v_tree,
                             io->base_logits, io->best_path, io->accept_len, io->accepted_tokens, io->next_token,
                             io->seq_lens_out};
  for (const void* p : host_ptrs)
    if (!host_or_null(p)) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step_host: a buffer in io is not host memory");
  if (io->uniforms && !a->uniforms)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step_host: io->uniforms given but args->uniforms is null");
  const int T = a->tree->T, D = a->tree->D, B = a->B;
  if ((io->k_tree || io->v_tree) && !io->seq_lens)
    return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step_host: k_tree / v_tree need the host seq_lens");
  if (io->seq_lens)
    for (int b = 0; b < B; ++b)
      if (io->seq_lens[b] < 0 || io->seq_lens[b] + T > a->Lcap)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_step_host: seq_lens[b] + T exceeds Lcap");

  const size_t esz = dtype_bytes(a->dtype);
  const size_t b4 = static_cast<size_t>(B) * 4;
  cudaStream_t cs = io->copy_stream ? io->copy_stream : stream;
  Events ev;
  cudaError_t e = ev.create();
  if (e != cudaSuccess) return cuda_fail("medusa_step_host: events", e);

  // The heads' inputs, on the step's stream.
  e = h2d(const_cast<void*>(a->h), io->h, static_cast<size_t>(B) * a->d * esz, stream);
  if (e == cudaSuccess) e = h2d(const_cast<int32_t*>(a->root_tokens), io->root_tokens, b4, stream);
  if (e == cudaSuccess) e = h2d(a->seq_lens, io->seq_lens, b4, stream);
  if (e == cudaSuccess) e = h2d(const_cast<float*>(a->uniforms), io->uniforms, b4, stream);
  if (e != cudaSuccess) return cuda_fail("medusa_step_host: copy of the heads' inputs", e);

  // Attention's and the posterior's inputs, after everything earlier on the
  // step's stream (the previous step still reads the caches and q).
  e = cudaEventRecord(ev.start, stream);
  if (e == cudaSuccess && cs != stream) e = cudaStreamWaitEvent(cs, ev.start, 0);
  const size_t q_bytes = static_cast<size_t>(a->layers) * B * T * a->H * a->hd * esz;
  if (e == cudaSuccess) e = h2d(const_cast<void*>(a->q), io->q, q_bytes, cs);
  for (int b = 0; b < B && e == cudaSuccess; ++b) {
    if (io->k_tree)
      e = scatter_tree_rows(a->k_cache, io->k_tree, a->layers, B, a->H, T, a->hd, a->Lcap, b, io->seq_lens[b], esz,
                            cs);
    if (e == cudaSuccess && io->v_tree)
      e = scatter_tree_rows(a->v_cache, io->v_tree, a->layers, B, a->H, T, a->hd, a->Lcap, b, io->seq_lens[b], esz,
                            cs);
  }
  if (e == cudaSuccess) e = cudaEventRecord(ev.attn, cs);
  if (e == cudaSuccess)
    e = h2d(const_cast<float*>(a->base_logits), io->base_logits, static_cast<size_t>(B) * T * a->V * 4, cs);
  if (e == cudaSuccess) e = cudaEventRecord(ev.post, cs);
  if (e != cudaSuccess) return cuda_fail("medusa_step_host: copy of the attention / posterior inputs", e);

  medusa_step_args_t s = *a;
  if (cs != stream) {
    s.attn_inputs_ready = ev.attn;
    s.posterior_inputs_ready = ev.post;
  }
  st = medusa_step(&s, workspace, workspace_bytes, stream);
  if (st != MEDUSA_OK) return st;

  e = d2h(io->best_path, a->best_path, b4, stream);
  if (e == cudaSuccess) e = d2h(io->accept_len, a->accept_len, b4, stream);
  if (e == cudaSuccess) e = d2h(io->accepted_tokens, a->accepted_tokens, b4 * (D + 1), stream);
  if (e == cudaSuccess) e = d2h(io->next_token, a->next_token, b4, stream);
  if (e == cudaSuccess) e = d2h(io->seq_lens_out, a->seq_lens, b4, stream);
  if (e != cudaSuccess) return cuda_fail("medusa_step_host: copy of the results", e);
  return MEDUSA_OK;
}
