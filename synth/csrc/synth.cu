// Device restatement of the seeded, counter-based input generator defined in
// synth/gen.py (splitmix64 output function over (seed, tensor id, index),
// Irwin-Hall of order 4 for normals, integer round-to-nearest-even for
// bf16).  It fills large synthetic tensors directly in device memory so
// that multi-GB inputs need no host round trip, and it plants head/base
// agreement into synthetic base logits.  It holds none of the Medusa step's
// arithmetic.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t x) {
  x ^= x >> 30;
  x *= 0xBF58476D1CE4E5B9ull;
  x ^= x >> 27;
  x *= 0x94D049BB133111EBull;
  x ^= x >> 31;
  return x;
}

__host__ __device__ __forceinline__ uint64_t stream_key(uint64_t seed, uint64_t tid) {
  return mix64(mix64(seed) + tid * kGamma);
}

__device__ __forceinline__ float normal_from(uint64_t x, float scale) {
  const int64_t c = static_cast<int64_t>((x & 0xFFFFull) + ((x >> 16) & 0xFFFFull) + ((x >> 32) & 0xFFFFull) +
                                         (x >> 48)) -
                    131070;
  return __fmul_rn(static_cast<float>(c), scale);
}

__device__ __forceinline__ uint16_t bf16_rne(float f) {
  const uint32_t b = __float_as_uint(f);
  return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

__global__ void normal_kernel(void* out, int64_t n, int bf16, uint64_t key, int64_t offset, float scale) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t x = mix64(key + static_cast<uint64_t>(offset + i + 1) * kGamma);
    const float v = normal_from(x, scale);
    if (bf16)
      static_cast<uint16_t*>(out)[i] = bf16_rne(v);
    else
      static_cast<float*>(out)[i] = v;
  }
}

// One block per (sequence, node) row of logits [B, T, V].
__global__ void plant_kernel(float* logits, int B, int T, int V, const int32_t* tree_tokens, const int32_t* parent,
                             double q, uint64_t key, float boost) {
  const int row = blockIdx.x;  // b*T + i
  const int b = row / T, i = row % T;
  __shared__ float red[32];
  __shared__ int chosen;
  if (threadIdx.x == 0) {
    int nch = 0;
    for (int c = 1; c < T; ++c) nch += parent[c] == i;
    chosen = -1;
    if (nch > 0) {
      const uint64_t x0 = mix64(key + static_cast<uint64_t>(2 * row + 1) * kGamma);
      const uint64_t x1 = mix64(key + static_cast<uint64_t>(2 * row + 2) * kGamma);
      const double u0 = static_cast<double>(x0 >> 40) * (1.0 / 16777216.0);
      const double u1 = static_cast<double>(x1 >> 40) * (1.0 / 16777216.0);
      if (u0 < q) {
        int pick = static_cast<int>(u1 * nch);
        if (pick > nch - 1) pick = nch - 1;
        for (int c = 1; c < T; ++c)
          if (parent[c] == i && pick-- == 0) {
            chosen = tree_tokens[b * T + c];
            break;
          }
      }
    }
  }
  __syncthreads();
  if (chosen < 0) return;
  float* z = logits + static_cast<size_t>(row) * V;
  float m = -3.402823466e38f;
  for (int v = threadIdx.x; v < V; v += blockDim.x) m = fmaxf(m, z[v]);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = red[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) mm = fmaxf(mm, red[w]);
    z[chosen] = __fadd_rn(mm, boost);
  }
}

}  // namespace

extern "C" int synth_normal(void* out, int64_t n, int bf16, uint64_t seed, uint64_t tensor_id, int64_t offset,
                            float scale, cudaStream_t stream) {
  if (n <= 0) return 0;
  int blocks = static_cast<int>((n + 255) / 256);
  if (blocks > 148 * 64) blocks = 148 * 64;
  normal_kernel<<<blocks, 256, 0, stream>>>(out, n, bf16, stream_key(seed, tensor_id), offset, scale);
  return static_cast<int>(cudaGetLastError());
}

extern "C" int synth_plant(float* logits, int B, int T, int V, const int32_t* tree_tokens, const int32_t* parent,
                           double q, uint64_t seed, uint64_t tensor_id, float boost, cudaStream_t stream) {
  plant_kernel<<<B * T, 256, 0, stream>>>(logits, B, T, V, tree_tokens, parent, q, stream_key(seed, tensor_id),
                                          boost);
  return static_cast<int>(cudaGetLastError());
}
