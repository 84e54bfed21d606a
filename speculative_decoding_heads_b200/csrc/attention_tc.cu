// S5 on the 5th-generation tensor cores: tree attention with tcgen05.mma,
// TMEM accumulators and TMA-staged K/V tiles (bf16 inputs, hd = 128).
//
// What it computes is the mask of "Medusa — 让大模型自己同时猜好几个 token"
// (核心要点: one forward of the whole candidate tree under a tree attention
// mask; 实践案例 case 3: a node sees the cached prefix, its ancestors and
// itself).  One CTA owns one (layer, sequence, head) slice and up to M query
// rows (M = 64 when T <= 64, else 128; larger trees use several row groups).
// Every K/V byte of the slice is read once for all of its tree queries.
//
// Warp roles (8 warps):
//   warp 0     TMA producer: Q once, then 64-key K and V tiles into a
//              two-stage ring (3-D tensor maps, 128-byte swizzle, no
//              multicast; rows past the cache capacity read as zero).
//   warp 1     allocates TMEM; one thread issues every tcgen05.mma:
//              S = Q K^T into TMEM (fp32), then O += P_hi V + P_lo V.
//              S of tile j+1 is issued as soon as the softmax has read S of
//              tile j, so it overlaps the softmax of tile j.
//   warps 4-7  softmax, one TMEM lane (query row) per thread: load S, apply
//              scale and the ancestor mask (only on tiles that reach row L),
//              keep a per-row reference maximum that only moves when the row
//              maximum grows by more than 2^8 (then O and the running sum are
//              rescaled in place), write P as a bf16 pair (high part and
//              remainder) into swizzled shared memory, and at the end read
//              O, divide by the running sum and store fp32 rows.
// Accumulation order differs from the plain softmax only by rounding; P
// carries ~16 significant bits, so outputs stay within 2e-3 of the exact
// value.
#include <cfloat>
#include <cudaTypedefs.h>

#include "tcgen05.cuh"

namespace medusa {
namespace {

constexpr int kHd = 128;
constexpr int kKT = 64;                        // keys per tile
constexpr int kStages = 2;
constexpr int kTileBytes = kKT * kHd * 2;      // 16 KB per K or V tile
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 256;            // S: cols [0, 64), O: cols [128, 256)
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 128;
constexpr float kRescaleLog2 = 8.0f;           // move the reference max only past 2^8

template <int M>
struct Layout {
  static constexpr int kQ = 0;                                  // M x 128 dims, two 64-dim regions
  static constexpr int kKV = M * 256;                           // stages of K then V
  static constexpr int kPhi = kKV + kStages * 2 * kTileBytes;   // M x 64 keys
  static constexpr int kPlo = kPhi + M * 128;
  static constexpr int kBars = kPlo + M * 128;
  static constexpr int kBytes = kBars + 256;
  static constexpr int kSmem = kBytes + 1024;                   // slack for 1024-byte alignment
};

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full, s_free, p_full, o_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Bars* b, int* status) {
  if (mbar_wait(bar, parity)) return true;
  set_device_status(status, MEDUSA_ERR_TIMEOUT, kDetailAttnStageWait);
  b->abort = 1;
  return false;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int M>
__global__ void __launch_bounds__(kThreads, M == 64 ? 2 : 1)
    tree_attn_tc(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                 const __grid_constant__ CUtensorMap v_map, const TreeDev t, int B, int H, int Lcap,
                 const int32_t* __restrict__ seq_lens, float scale_log2, float* __restrict__ out, int* status) {
  using Lay = Layout<M>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  Bars* bar = reinterpret_cast<Bars*>(smem + Lay::kBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.x;       // (l*B + b)*H + e
  const int e = slice % H;
  const int lb = slice / H;
  const int b = lb % B;
  const int row0 = blockIdx.y * M;
  const int L = seq_lens[b];
  if (L < 0 || L + t.T > Lcap) {
    if (tid == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailAttnSeqLen);
    return;
  }
  const int n = L + t.T;
  const int nt = (n + kKT - 1) / kKT;
  const uint32_t sbase = smem_u32(smem);

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->kv_full[s], 1);
      mbar_init(&bar->kv_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 4);
    mbar_init(&bar->p_full, 4);
    mbar_init(&bar->o_done, 1);
    bar->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bar->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tc::prefetch_tensormap(&q_map);
      tc::prefetch_tensormap(&k_map);
      tc::prefetch_tensormap(&v_map);
      mbar_arrive_expect_tx(&bar->q_full, 2 * M * 128);
      tc::tma_load_4d(smem + Lay::kQ, &q_map, 0, e, row0, lb, &bar->q_full);
      tc::tma_load_4d(smem + Lay::kQ + M * 128, &q_map, 64, e, row0, lb, &bar->q_full);
      for (int j = 0; j < nt; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !wait_or_abort(&bar->kv_empty[st], ((j / kStages) - 1) & 1, bar, status)) break;
        if (bar->abort) break;
        unsigned char* kd = smem + Lay::kKV + st * 2 * kTileBytes;
        unsigned char* vd = kd + kTileBytes;
        mbar_arrive_expect_tx(&bar->kv_full[st], 2 * kTileBytes);
        tc::tma_load_3d(kd, &k_map, 0, j * kKT, slice, &bar->kv_full[st]);
        tc::tma_load_3d(kd + kKT * 128, &k_map, 64, j * kKT, slice, &bar->kv_full[st]);
        tc::tma_load_3d(vd, &v_map, 0, j * kKT, slice, &bar->kv_full[st]);
        tc::tma_load_3d(vd + kKT * 128, &v_map, 64, j * kKT, slice, &bar->kv_full[st]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(M, kKT, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(M, kHd, 1);
      const uint32_t qa = sbase + Lay::kQ;
      auto issue_s = [&](int j) {
        const uint32_t kb = sbase + Lay::kKV + (j % kStages) * 2 * kTileBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = tc::smem_desc_sw128(qa + (k >> 2) * M * 128 + (k & 3) * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(kb + (k >> 2) * kKT * 128 + (k & 3) * 32, 16, 1024);
          tc::mma_ss(tmem + kColS, ad, bd, idS, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bar->s_full);
      };
      bool ok = wait_or_abort(&bar->q_full, 0, bar, status) && wait_or_abort(&bar->kv_full[0], 0, bar, status);
      if (ok) {
        tc::fence_after_sync();
        issue_s(0);
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          const int s1 = (j + 1) % kStages;
          ok = wait_or_abort(&bar->kv_full[s1], ((j + 1) / kStages) & 1, bar, status) &&
               wait_or_abort(&bar->s_free, j & 1, bar, status);
          if (!ok) break;
          tc::fence_after_sync();
          issue_s(j + 1);
        }
        if (!wait_or_abort(&bar->p_full, j & 1, bar, status)) break;
        tc::fence_after_sync();
        const uint32_t vb = sbase + Lay::kKV + (j % kStages) * 2 * kTileBytes + kTileBytes;
        const uint32_t ph = sbase + Lay::kPhi, pl = sbase + Lay::kPlo;
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk) {
          const uint64_t bd = tc::smem_desc_sw128(vb + kk * 16 * 128, kKT * 128, 1024);
          tc::mma_ss(tmem + kColO, tc::smem_desc_sw128(ph + kk * 32, 16, 1024), bd, idO,
                     (j > 0 || kk > 0) ? 1u : 0u);
          tc::mma_ss(tmem + kColO, tc::smem_desc_sw128(pl + kk * 32, 16, 1024), bd, idO, 1u);
        }
        tc::mma_commit(&bar->kv_empty[j % kStages]);
        tc::mma_commit(&bar->o_done);
      }
    }
  } else if (warp >= 4) {
    // ---------------- softmax / epilogue ----------------
    const int q = warp & 3;                                   // TMEM lane quarter of this warp
    const bool has_row = (M == 128) || lane < 16;
    const int r = (M == 128) ? 32 * q + lane : 16 * q + lane; // row within the group
    const int i = row0 + r;                                   // tree node
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    uint64_t anc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int w = 0; w < 4; ++w)
      if (has_row && i < t.T && w < t.W) anc[w] = t.anc[i * t.W + w];
    float mref = -INFINITY, lsum = 0.f;
    unsigned char* phi = smem + Lay::kPhi;
    unsigned char* plo = smem + Lay::kPlo;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (!wait_or_abort(&bar->s_full, j & 1, bar, status)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float s[kKT];
      tc::tmem_ld32(tmem + lane_addr + kColS, s);
      tc::tmem_ld32(tmem + lane_addr + kColS + 32, s + 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar->s_free);
      // scale, mask, tile max
      const int j0 = j * kKT;
      float tmax = -INFINITY;
      const bool masked_tile = j0 + kKT > L;
#pragma unroll
      for (int c = 0; c < kKT; ++c) {
        float v = s[c] * scale_log2;
        if (masked_tile) {
          const int key = j0 + c;
          bool keep = key < L;
          if (!keep && key < n) {
            const int tj = key - L;
            const uint64_t wd = tj < 64 ? anc[0] : tj < 128 ? anc[1] : tj < 192 ? anc[2] : anc[3];
            keep = (wd >> (tj & 63)) & 1ull;
          }
          if (!keep) v = -INFINITY;
        }
        s[c] = v;
        tmax = fmaxf(tmax, v);
      }
      float factor = 1.f;
      if (tmax > mref + kRescaleLog2 || (mref == -INFINITY && tmax > -INFINITY)) {
        factor = (mref == -INFINITY) ? 0.f : exp2f(mref - tmax);
        mref = tmax;
        lsum *= factor;
      }
      if (!has_row) factor = 1.f;   // lanes that hold no row (M = 64) never ask for a rescale
      const float mu = (mref == -INFINITY) ? 0.f : mref;
      float ps = 0.f;
#pragma unroll
      for (int c = 0; c < kKT; ++c) {
        s[c] = exp2f(s[c] - mu);
        ps += s[c];
      }
      lsum += ps;
      // PV of tile j-1 must be done before P is overwritten or O rescaled.
      if (j > 0) {
        if (!wait_or_abort(&bar->o_done, (j - 1) & 1, bar, status)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
      }
      if (has_row) {
        const uint32_t rb = (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int ch = 0; ch < kKT / 8; ++ch) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float a0 = s[ch * 8 + 2 * u], a1 = s[ch * 8 + 2 * u + 1];
            hi[u] = pack2_bf16(a0, a1);
            const float r0 = a0 - __uint_as_float(hi[u] << 16);
            const float r1 = a1 - __uint_as_float(hi[u] & 0xffff0000u);
            lo[u] = pack2_bf16(r0, r1);
          }
          const uint32_t off = rb + ((ch ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(phi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(plo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      if (j > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
#pragma unroll 1
        for (int c0 = 0; c0 < kHd; c0 += 32) {
          float o[32];
          tc::tmem_ld32(tmem + lane_addr + kColO + c0, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= factor;
          tc::tmem_st32(tmem + lane_addr + kColO + c0, o);
        }
        tc::tmem_wait_st();
      }
      if (j == nt - 1 && j0 + kKT > n) {
        // V rows past the slice's last key: zero them so 0 * (stale value) stays 0.
        unsigned char* vd = smem + Lay::kKV + (j % kStages) * 2 * kTileBytes + kTileBytes;
        const int first = n - j0;
        for (int x = (warp - 4) * 32 + lane; x < (kKT - first) * 8; x += 128) {
          const int rr = first + x / 8, cc = x % 8;   // 8 chunks of 16 B per 128-B row
          *reinterpret_cast<uint4*>(vd + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(vd + kKT * 128 + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar->p_full);
    }
    if (ok && wait_or_abort(&bar->o_done, (nt - 1) & 1, bar, status)) {
      tc::fence_after_sync();
      const float inv = 1.f / lsum;
      float* orow = out + ((static_cast<size_t>(lb) * t.T + i) * H + e) * kHd;
#pragma unroll
      for (int c0 = 0; c0 < kHd; c0 += 32) {
        float o[32];
        tc::tmem_ld32(tmem + lane_addr + kColO + c0, o);
        tc::tmem_wait_ld();
        if (has_row && i < t.T) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(orow + c0 + c) =
                make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side --------------------------------------------------------------

}  // namespace

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
void* tensor_map_encoder() {
  static void* fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  }
  return fn;
}

// Encodes the three tensor maps and launches the tcgen05 kernel.  Returns
// MEDUSA_ERR_UNSUPPORTED when the shape does not fit it (caller falls back).
medusa_status_t launch_attention_tc(const TreeDev& t, int layers, int B, int H, const void* q, const void* k_cache,
                                    const void* v_cache, int Lcap, const int32_t* seq_lens, float scale_log2,
                                    float* out, int* status, cudaStream_t stream) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: cuTensorMapEncodeTiled unavailable");
  const int M = t.T <= 64 ? 64 : 128;
  const int groups = (t.T + M - 1) / M;
  const unsigned long long slices = static_cast<unsigned long long>(layers) * B * H;
  CUtensorMap qm, km, vm;
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHd), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(t.T), static_cast<cuuint64_t>(layers) * B};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHd) * 2, static_cast<cuuint64_t>(H) * kHd * 2,
                                   static_cast<cuuint64_t>(t.T) * H * kHd * 2};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(M), 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: q tensor map rejected");
  }
  for (int which = 0; which < 2; ++which) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHd), static_cast<cuuint64_t>(Lcap), slices};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHd) * 2, static_cast<cuuint64_t>(Lcap) * kHd * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kKT), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(which == 0 ? &km : &vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void*>(which == 0 ? k_cache : v_cache), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: K/V tensor map rejected");
  }
  cudaError_t e;
  if (M == 64) {
    e = cudaFuncSetAttribute(tree_attn_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<64>::kSmem);
    if (e == cudaSuccess)
      tree_attn_tc<64><<<dim3(static_cast<unsigned>(slices), groups), kThreads, Layout<64>::kSmem, stream>>>(
          qm, km, vm, t, B, H, Lcap, seq_lens, scale_log2, out, status);
  } else {
    e = cudaFuncSetAttribute(tree_attn_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<128>::kSmem);
    if (e == cudaSuccess)
      tree_attn_tc<128><<<dim3(static_cast<unsigned>(slices), groups), kThreads, Layout<128>::kSmem, stream>>>(
          qm, km, vm, t, B, H, Lcap, seq_lens, scale_log2, out, status);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_attention: tcgen05 launch", e);
}

}  // namespace medusa
