// S5: tree attention ("Medusa — 让大模型自己同时猜好几个 token", 核心要点: the
// candidate tree is verified in one forward under a tree attention mask;
// 实践案例 case 3: "X after A" sees only the prefix P and A).  Node i of the
// tree attends to every cached prefix row 0..L-1 and to tree rows L+j where
// j is i or one of its ancestors; the tree's own K/V already sit at rows
// L..L+T-1 of the cache.
//
// bf16 with hd = 128 runs on the tcgen05 tensor cores in a persistent kernel:
// attention_tc64.cu for trees of up to 64 tokens, attention_tc128.cu for
// larger trees (one pass over a slice's K/V per 128 tree tokens).  Every
// other dtype / head size
// runs tree_attn_generic: one CTA per (slice, node), scores in shared memory,
// plain fp32 arithmetic.  The output is fp32 on every path.
#include <cfloat>

#include "common.cuh"

namespace medusa {
namespace {

// ------------------------------------------------------------------------
// generic kernel
// ------------------------------------------------------------------------

template <typename T>
__device__ __forceinline__ float ld_elem(const T* p);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_elem<uint16_t>(const uint16_t* p) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p))) << 16);
}

__device__ __forceinline__ bool anc_bit(const TreeDev& t, int i, int j) {
  return (t.anc[i * t.W + (j >> 6)] >> (j & 63)) & 1ull;
}

template <typename T>
__global__ void tree_attn_generic(const TreeDev t, int B, int H, int hd, const T* __restrict__ q,
                                  const T* __restrict__ kc, const T* __restrict__ vc, int Lcap,
                                  const int32_t* __restrict__ seq_lens, float scale, float* __restrict__ out,
                                  int* status) {
  extern __shared__ float sh[];  // [hd] q, then [Lcap] scores
  float* qs = sh;
  float* sc = sh + hd;
  __shared__ float red[32];
  const int i = blockIdx.x % t.T;
  const int slice = blockIdx.x / t.T;           // (l*B + b)*H + e
  const int e = slice % H;
  const int lb = slice / H;                     // l*B + b
  const int b = lb % B;
  const int L = seq_lens[b];
  if (L < 0 || L + t.T > Lcap) {
    if (threadIdx.x == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailAttnSeqLen);
    return;
  }
  const size_t qoff = ((static_cast<size_t>(lb) * t.T + i) * H + e) * hd;
  for (int c = threadIdx.x; c < hd; c += blockDim.x) qs[c] = ld_elem<T>(q + qoff + c);
  __syncthreads();
  const T* K = kc + static_cast<size_t>(slice) * Lcap * hd;
  const T* Vv = vc + static_cast<size_t>(slice) * Lcap * hd;
  const int n = L + t.T;
  float mx = -FLT_MAX;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const bool ok = j < L || anc_bit(t, i, j - L);
    float s = -FLT_MAX;
    if (ok) {
      float acc = 0.f;
      for (int c = 0; c < hd; ++c) acc = fmaf(qs[c], ld_elem<T>(K + static_cast<size_t>(j) * hd + c), acc);
      s = acc * scale;
    }
    sc[j] = s;
    mx = fmaxf(mx, s);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = -FLT_MAX;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const bool ok = j < L || anc_bit(t, i, j - L);
    const float p = ok ? expf(sc[j] - mx) : 0.f;
    sc[j] = p;
    sum += p;
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w];
  const float inv = 1.f / sum;
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < n; ++j) acc = fmaf(sc[j], ld_elem<T>(Vv + static_cast<size_t>(j) * hd + c), acc);
    out[qoff + c] = acc * inv;
  }
}

constexpr int kHd = 128;
constexpr float kLog2e = 1.4426950408889634f;


// The log-sum-exp identity: attention over a union of disjoint key sets from
// each set's normalised output O_g and lse_g = ln sum exp(scale q.k):
// out = sum_g exp(lse_g - lse) O_g with lse = ln sum_g exp(lse_g).  One thread
// per 4 output values; every O_g is read once.
__global__ void attention_combine_kernel(int G, size_t rows, int hd4, const float4* outs, const float* lses,
                                         float4* out, float* lse_out) {
  const size_t n = rows * static_cast<size_t>(hd4);
  for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = idx / hd4;
    float m = -INFINITY;
    for (int g = 0; g < G; ++g) m = fmaxf(m, lses[g * rows + row]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float tot = 0.f;
    if (m > -INFINITY) {                 // otherwise no window held a key: O = 0
      for (int g = 0; g < G; ++g) {
        const float w = expf(lses[g * rows + row] - m);
        const float4 o = outs[g * n + idx];
        tot += w;
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
      const float inv = 1.f / tot;
      acc.x *= inv;
      acc.y *= inv;
      acc.z *= inv;
      acc.w *= inv;
    }
    out[idx] = acc;
    if (lse_out != nullptr && idx % hd4 == 0) lse_out[row] = m > -INFINITY ? m + logf(tot) : -INFINITY;
  }
}

// The same identity split across ranks: rank `rank` scales its own partial
// by exp(lse_rank - lse) in place, so that the G scaled partials sum to the
// combined output (an all-reduce then replaces the gather of G outputs).
// Only the G lse values of a row are read from every rank.
__global__ void attention_rescale_kernel(int G, int rank, size_t rows, int hd4, const float* lses, float4* part,
                                         float* lse_out) {
  const size_t n = rows * static_cast<size_t>(hd4);
  for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = idx / hd4;
    float m = -INFINITY;
    for (int g = 0; g < G; ++g) m = fmaxf(m, lses[g * rows + row]);
    float w = 0.f, tot = 0.f;
    if (m > -INFINITY) {
      for (int g = 0; g < G; ++g) tot += expf(lses[g * rows + row] - m);
      w = expf(lses[rank * rows + row] - m) / tot;
    }
    float4 o = part[idx];
    o.x *= w;
    o.y *= w;
    o.z *= w;
    o.w *= w;
    part[idx] = o;
    if (lse_out != nullptr && idx % hd4 == 0) lse_out[row] = m > -INFINITY ? m + logf(tot) : -INFINITY;
  }
}

}  // namespace

medusa_status_t launch_attention_rescale(int G, int rank, size_t rows, int hd, const float* lses, float* part,
                                         float* lse_out, cudaStream_t stream) {
  const size_t n = rows * static_cast<size_t>(hd / 4);
  const size_t want = (n + 255) / 256;
  const size_t cap = static_cast<size_t>(sm_count() > 0 ? sm_count() : 1) * 16;
  const int grid = static_cast<int>(want < cap ? want : cap);
  attention_rescale_kernel<<<grid, 256, 0, stream>>>(G, rank, rows, hd / 4, lses, reinterpret_cast<float4*>(part),
                                                     lse_out);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_attention_rescale", e);
}

medusa_status_t launch_attention_split(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype,
                                       const void* q, const void* k_cache, const void* v_cache, int Lcap,
                                       const int32_t* seq_lens, float scale, int rank, int G, float* out,
                                       float* lse, cudaStream_t stream) {
  if (dtype != MEDUSA_BF16 || hd != kHd || t.T > 64)
    return fail(MEDUSA_ERR_UNSUPPORTED,
                "medusa_tree_attention_split: the split runs on the bf16, hd 128 kernel for trees of at most 64 tokens");
  return launch_attention_tc64(t, layers, B, H, q, k_cache, v_cache, Lcap, seq_lens, scale * kLog2e, out,
                               device_status_ptr(), stream, false, 0, t.T, rank, G, lse);
}

medusa_status_t launch_attention_combine(int G, size_t rows, int hd, const float* outs, const float* lses,
                                         float* out, float* lse_out, cudaStream_t stream) {
  const size_t n = rows * static_cast<size_t>(hd / 4);
  const size_t want = (n + 255) / 256;
  const size_t cap = static_cast<size_t>(sm_count() > 0 ? sm_count() : 1) * 16;
  const int grid = static_cast<int>(want < cap ? want : cap);
  attention_combine_kernel<<<grid, 256, 0, stream>>>(G, rows, hd / 4, reinterpret_cast<const float4*>(outs), lses,
                                                     reinterpret_cast<float4*>(out), lse_out);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_attention_combine", e);
}

size_t attention_workspace_bytes(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype) {
  (void)t;
  (void)layers;
  (void)B;
  (void)H;
  (void)hd;
  (void)dtype;
  return 0;
}

// Tree rows handled in groups of 128 (tree_attn_tc128): where a group would
// hold more than 64 of them; the rest (at most 64) go to one 64-row group.
int rows_in_128_groups(int T) { return T <= 64 ? 0 : (T % 128 == 0 || T % 128 > 64 ? T : T / 128 * 128); }

medusa_status_t launch_attention_bf16_out(const TreeDev& t, int B, int H, const void* q, const void* k_cache,
                                          const void* v_cache, int Lcap, const int32_t* seq_lens, float scale,
                                          uint16_t* out, cudaStream_t stream) {
  int* status = device_status_ptr();
  const float sl = scale * kLog2e;
  AttnOut dec;
  dec.bf16 = out;
  dec.wait_first = true;
  const int full = rows_in_128_groups(t.T);
  if (full > 0) {
    const medusa_status_t st = launch_attention_tc128(t, 1, B, H, q, k_cache, v_cache, Lcap, seq_lens, sl, nullptr,
                                                      status, stream, true, 0, full, dec);
    if (st != MEDUSA_OK || full == t.T) return st;
  }
  return launch_attention_tc64(t, 1, B, H, q, k_cache, v_cache, Lcap, seq_lens, sl, nullptr, status, stream, true,
                               full, t.T, 0, 1, nullptr, dec);
}

medusa_status_t launch_attention(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype,
                                 const void* q, const void* k_cache, const void* v_cache, int Lcap,
                                 const int32_t* seq_lens, float scale, void* out, void* ws,
                                 cudaStream_t stream, bool pdl) {
  (void)ws;
  const int n_slices = layers * B * H;
  int* status = device_status_ptr();
  cudaError_t e;
  if (dtype == MEDUSA_BF16 && hd == kHd) {
    float* o = static_cast<float*>(out);
    const float sl = scale * kLog2e;
    const int full = rows_in_128_groups(t.T);
    if (full > 0) {
      const medusa_status_t st =
          launch_attention_tc128(t, layers, B, H, q, k_cache, v_cache, Lcap, seq_lens, sl, o, status, stream, pdl, 0,
                                 full);
      if (st != MEDUSA_OK || full == t.T) return st;
    }
    return launch_attention_tc64(t, layers, B, H, q, k_cache, v_cache, Lcap, seq_lens, sl, o, status, stream, pdl,
                                 full, t.T);
  }
  {
    const size_t smem = static_cast<size_t>(hd + Lcap) * sizeof(float);
    if (smem > 200 * 1024) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_tree_attention: Lcap too large for this dtype/hd");
    const int threads = hd > 128 ? hd : 128;
    if (dtype == MEDUSA_BF16) {
      auto fn = tree_attn_generic<uint16_t>;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail("medusa_tree_attention: smem attribute", e);
      fn<<<n_slices * t.T, threads, smem, stream>>>(t, B, H, hd, static_cast<const uint16_t*>(q),
                                                    static_cast<const uint16_t*>(k_cache),
                                                    static_cast<const uint16_t*>(v_cache), Lcap, seq_lens, scale,
                                                    static_cast<float*>(out), status);
    } else {
      auto fn = tree_attn_generic<float>;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail("medusa_tree_attention: smem attribute", e);
      fn<<<n_slices * t.T, threads, smem, stream>>>(t, B, H, hd, static_cast<const float*>(q),
                                                    static_cast<const float*>(k_cache),
                                                    static_cast<const float*>(v_cache), Lcap, seq_lens, scale,
                                                    static_cast<float*>(out), status);
    }
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_attention: launch", e);
}

}  // namespace medusa
