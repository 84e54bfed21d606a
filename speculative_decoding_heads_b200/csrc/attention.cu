// S5: tree attention ("Medusa — 让大模型自己同时猜好几个 token", 核心要点: the
// candidate tree is verified in one forward under a tree attention mask;
// 实践案例 case 3: "X after A" sees only the prefix P and A).  Node i of the
// tree attends to every cached prefix row 0..L-1 and to tree rows L+j where
// j is i or one of its ancestors; the tree's own K/V already sit at rows
// L..L+T-1 of the cache.
//
// Two kernels:
//  * tree_attn_mma (bf16, hd = 128): one CTA per (layer, sequence, head);
//    ceil(T/16) warps each own 16 query rows held as mma A fragments.  K/V
//    tiles of 64 keys stream through a double-buffered, XOR-swizzled shared
//    ring (cp.async, zero-fill past the last key); S = Q K^T and O += P V run
//    on the tensor cores (mma.m16n8k16 bf16, fp32 accumulate) with an online
//    softmax in registers.  Only tiles that reach row L carry the ancestor
//    mask; prefix tiles are dense.  Every K/V byte of the slice is read once
//    for all T queries.
//  * tree_attn_generic (fp32 or bf16, any hd <= 256 multiple of 32): one CTA
//    per (slice, node), scores in shared memory, plain fp32 arithmetic.
// The output is fp32 in both: P V is accumulated in fp32, and P enters the
// bf16 tensor-core product as a bf16 pair (high part + remainder), which
// keeps the result within 2e-3 of the exact value even when a few keys
// dominate the softmax.
#include <cfloat>
#include <cstdlib>

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

// ------------------------------------------------------------------------
// tensor-core kernel, bf16, hd = 128
// ------------------------------------------------------------------------

constexpr int kHd = 128;
constexpr int kKeys = 64;                                  // keys per tile
constexpr int kTileBytes = kKeys * kHd * 2;                // 16 KB per K or V tile
constexpr int kSmemBytes = 2 * 2 * kTileBytes;             // K and V, double buffered
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxWarps = 8;   // 128 query rows per CTA (register budget: 255 per thread at 256 threads)

__device__ __forceinline__ uint32_t swz(int row, int chunk) {   // byte offset in a [64][256 B] tile
  return static_cast<uint32_t>(row * 256 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_rne(lo)) | (static_cast<uint32_t>(f32_to_bf16_rne(hi)) << 16);
}

// Splits two probabilities into bf16 high parts and bf16 remainders, so that
// P V = P_hi V + P_lo V carries ~16 significant bits of P instead of 8.
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  const uint16_t ha = f32_to_bf16_rne(a), hb = f32_to_bf16_rne(b);
  hi = static_cast<uint32_t>(ha) | (static_cast<uint32_t>(hb) << 16);
  const float ra = a - __uint_as_float(static_cast<uint32_t>(ha) << 16);
  const float rb = b - __uint_as_float(static_cast<uint32_t>(hb) << 16);
  lo = pack_bf16(ra, rb);
}

// Word of a 4-word ancestor mask holding bit tj (register-only selection).
__device__ __forceinline__ uint64_t sel_word(const uint64_t (&m)[4], int tj) {
  return tj < 64 ? m[0] : tj < 128 ? m[1] : tj < 192 ? m[2] : m[3];
}

// Issues the cp.async copies of keys [j0, j0+64) of K and V into stage `buf`.
__device__ __forceinline__ void load_tile(uint32_t sbase, int buf, const unsigned char* K, const unsigned char* V,
                                          int j0, int n, int tid, int nthreads) {
  const uint32_t kb = sbase + buf * 2 * kTileBytes;
  const uint32_t vb = kb + kTileBytes;
  for (int c = tid; c < kKeys * 16; c += nthreads) {
    const int row = c >> 4, chunk = c & 15;
    const int j = j0 + row;
    const bool ok = j < n;
    const size_t off = static_cast<size_t>(ok ? j : 0) * 256 + chunk * 16;
    cp_async16(kb + swz(row, chunk), K + off, ok ? 16 : 0);
    cp_async16(vb + swz(row, chunk), V + off, ok ? 16 : 0);
  }
}

__global__ void __launch_bounds__(kMaxWarps * 32) tree_attn_mma(const TreeDev t, int B, int H, int row0_step,
                                                     const uint16_t* __restrict__ q,
                                                     const uint16_t* __restrict__ kc,
                                                     const uint16_t* __restrict__ vc, int Lcap,
                                                     const int32_t* __restrict__ seq_lens, float scale_log2,
                                                     float* __restrict__ out, int* status) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x;
  const int slice = blockIdx.x;       // (l*B + b)*H + e
  const int e = slice % H;
  const int lb = slice / H;
  const int b = lb % B;
  const int L = seq_lens[b];
  if (L < 0 || L + t.T > Lcap) {
    if (tid == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailAttnSeqLen);
    return;
  }
  const int n = L + t.T;                       // keys of this slice
  const int ntiles = (n + kKeys - 1) / kKeys;
  const unsigned char* K = reinterpret_cast<const unsigned char*>(kc) + static_cast<size_t>(slice) * Lcap * 256;
  const unsigned char* V = reinterpret_cast<const unsigned char*>(vc) + static_cast<size_t>(slice) * Lcap * 256;
  const uint32_t sbase = smem_u32(smem);

  load_tile(sbase, 0, K, V, 0, n, tid, nthreads);
  cp_commit();

  // Q fragments of this warp's 16 rows (rows >= T are zero).
  const int g = lane >> 2, tq = lane & 3;
  const int r0 = blockIdx.y * row0_step + warp * 16 + g, r1 = r0 + 8;
  uint32_t qa[8][4];
  {
    const size_t stride_row = static_cast<size_t>(H) * kHd;   // elements between consecutive tree rows
    const uint16_t* qb = q + (static_cast<size_t>(lb) * t.T * H + e) * kHd;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c0 = ks * 16 + 2 * tq;
      auto ld = [&](int r, int c) -> uint32_t {
        return r < t.T ? __ldg(reinterpret_cast<const unsigned int*>(qb + r * stride_row + c)) : 0u;
      };
      qa[ks][0] = ld(r0, c0);
      qa[ks][1] = ld(r1, c0);
      qa[ks][2] = ld(r0, c0 + 8);
      qa[ks][3] = ld(r1, c0 + 8);
    }
  }
  // Ancestor masks of rows r0 and r1 (tree nodes), up to 4 words each.
  uint64_t m0[4] = {0, 0, 0, 0}, m1[4] = {0, 0, 0, 0};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    if (w < t.W && r0 < t.T) m0[w] = t.anc[r0 * t.W + w];
    if (w < t.W && r1 < t.T) m1[w] = t.anc[r1 * t.W + w];
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow0 = -INFINITY, mrow1 = -INFINITY, lrow0 = 0.f, lrow1 = 0.f;

  for (int it = 0; it < ntiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < ntiles) {
      load_tile(sbase, buf ^ 1, K, V, (it + 1) * kKeys, n, tid, nthreads);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const uint32_t kb = sbase + buf * 2 * kTileBytes;
    const uint32_t vb = kb + kTileBytes;
    const int j0 = it * kKeys;

    // S = Q K^T for 64 keys: 8 n-tiles of 8 keys.
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {   // pairs of k-steps
        uint32_t b0, b1, b2, b3;
        const int row = nt * 8 + (lane & 7);
        const int chunk = 4 * kp + (lane >> 3);
        ldsm_x4(kb + swz(row, chunk), b0, b1, b2, b3);
        mma16816(s[nt], qa[2 * kp], b0, b1);
        mma16816(s[nt], qa[2 * kp + 1], b2, b3);
      }
    }
    // scale, mask, tile max
    const bool needs_mask = j0 + kKeys > L;
    float tmax0 = -INFINITY, tmax1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v = s[nt][c] * scale_log2;
        if (needs_mask) {
          const int j = j0 + nt * 8 + 2 * tq + (c & 1);
          bool ok = j < L;
          if (!ok && j < n) {
            const int tj = j - L;
            const uint64_t word = (c < 2) ? sel_word(m0, tj) : sel_word(m1, tj);
            ok = (word >> (tj & 63)) & 1ull;
          }
          if (!ok) v = -INFINITY;
        }
        s[nt][c] = v;
      }
      tmax0 = fmaxf(tmax0, fmaxf(s[nt][0], s[nt][1]));
      tmax1 = fmaxf(tmax1, fmaxf(s[nt][2], s[nt][3]));
    }
    tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, 1));
    tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, 2));
    tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, 1));
    tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, 2));
    const float mnew0 = fmaxf(mrow0, tmax0), mnew1 = fmaxf(mrow1, tmax1);
    const float mu0 = mnew0 == -INFINITY ? 0.f : mnew0;
    const float mu1 = mnew1 == -INFINITY ? 0.f : mnew1;
    const float corr0 = exp2f(mrow0 - mu0), corr1 = exp2f(mrow1 - mu1);
    mrow0 = mnew0;
    mrow1 = mnew1;
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - mu0);
      s[nt][1] = exp2f(s[nt][1] - mu0);
      s[nt][2] = exp2f(s[nt][2] - mu1);
      s[nt][3] = exp2f(s[nt][3] - mu1);
      ls0 += s[nt][0] + s[nt][1];
      ls1 += s[nt][2] + s[nt][3];
    }
    lrow0 = lrow0 * corr0 + ls0;
    lrow1 = lrow1 * corr1 + ls1;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= corr0;
      o[i][1] *= corr0;
      o[i][2] *= corr1;
      o[i][3] *= corr1;
    }
    // O += P V: 4 k-steps of 16 keys, 16 n-tiles of 8 dims.
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4], pl[4];
      split_bf16(s[2 * kk][0], s[2 * kk][1], pa[0], pl[0]);
      split_bf16(s[2 * kk][2], s[2 * kk][3], pa[1], pl[1]);
      split_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1], pa[2], pl[2]);
      split_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3], pa[3], pl[3]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {   // pairs of dim n-tiles
        uint32_t b0, b1, b2, b3;
        const int row = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = 2 * np + (lane >> 4);
        ldsm_x4_t(vb + swz(row, chunk), b0, b1, b2, b3);
        mma16816(o[2 * np], pa, b0, b1);
        mma16816(o[2 * np], pl, b0, b1);
        mma16816(o[2 * np + 1], pa, b2, b3);
        mma16816(o[2 * np + 1], pl, b2, b3);
      }
    }
    __syncthreads();
  }

  // Row sums across the 4 lanes of a row, normalise, store bf16.
  lrow0 += __shfl_xor_sync(0xffffffffu, lrow0, 1);
  lrow0 += __shfl_xor_sync(0xffffffffu, lrow0, 2);
  lrow1 += __shfl_xor_sync(0xffffffffu, lrow1, 1);
  lrow1 += __shfl_xor_sync(0xffffffffu, lrow1, 2);
  const float inv0 = 1.f / lrow0, inv1 = 1.f / lrow1;
  const size_t stride_row = static_cast<size_t>(H) * kHd;
  float* ob = out + (static_cast<size_t>(lb) * t.T * H + e) * kHd;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = i * 8 + 2 * tq;
    if (r0 < t.T) *reinterpret_cast<float2*>(ob + r0 * stride_row + c) = make_float2(o[i][0] * inv0, o[i][1] * inv0);
    if (r1 < t.T) *reinterpret_cast<float2*>(ob + r1 * stride_row + c) = make_float2(o[i][2] * inv1, o[i][3] * inv1);
  }
}

// MEDUSA_ATTN_MMA_SYNC=1 selects the legacy mma.sync kernel (kept for A/B
// comparison while the tcgen05 kernel is validated).
bool use_legacy_mma() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MEDUSA_ATTN_MMA_SYNC");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

}  // namespace

size_t attention_workspace_bytes(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype) {
  (void)t;
  (void)layers;
  (void)B;
  (void)H;
  (void)hd;
  (void)dtype;
  return 0;
}

medusa_status_t launch_attention(const TreeDev& t, int layers, int B, int H, int hd, medusa_dtype_t dtype,
                                 const void* q, const void* k_cache, const void* v_cache, int Lcap,
                                 const int32_t* seq_lens, float scale, void* out, void* ws,
                                 cudaStream_t stream) {
  (void)ws;
  const int n_slices = layers * B * H;
  int* status = device_status_ptr();
  cudaError_t e;
  if (dtype == MEDUSA_BF16 && hd == kHd && !use_legacy_mma()) {
    if (t.T <= 64)
      return launch_attention_tc64(t, layers, B, H, q, k_cache, v_cache, Lcap, seq_lens, scale * kLog2e,
                                   static_cast<float*>(out), status, stream);
    return launch_attention_tc(t, layers, B, H, q, k_cache, v_cache, Lcap, seq_lens, scale * kLog2e,
                               static_cast<float*>(out), status, stream);
  }
  if (dtype == MEDUSA_BF16 && hd == kHd) {
    e = cudaFuncSetAttribute(tree_attn_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return cuda_fail("medusa_tree_attention: smem attribute", e);
    // Query rows are split over gridDim.y CTAs of at most kMaxWarps warps.
    const int row_tiles = (t.T + 15) / 16;
    const int groups = (row_tiles + kMaxWarps - 1) / kMaxWarps;
    const int warps = (row_tiles + groups - 1) / groups;
    tree_attn_mma<<<dim3(n_slices, groups), warps * 32, kSmemBytes, stream>>>(
        t, B, H, warps * 16, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k_cache),
        static_cast<const uint16_t*>(v_cache), Lcap, seq_lens, scale * kLog2e, static_cast<float*>(out), status);
  } else {
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
