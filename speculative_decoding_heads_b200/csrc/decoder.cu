// The base model's forward over the tree tokens (tree_decoding): the step
// either side of tree attention.  "Medusa API参考：核心函数与类详解", 核心功能函数:
// tree_decoding runs the base model once over every tree token at the tree's
// position ids (prefix length + depth) under the tree mask, against the
// cached K/V, and its logits feed evaluate_posterior; "基于 Medusa 头的投机解码架构",
// 性能基准测试: the base models are Vicuna (LLaMA) 7B/13B/33B.  The layer is the
// LLaMA decoder layer: RMSNorm, Q/K/V with rotary embedding (pair i with
// i + hd/2, base 10000), tree attention, output projection and residual,
// RMSNorm, SwiGLU feed-forward and residual; then a final RMSNorm and the LM
// head.
//
// Every matrix product here is weights x (a pass of at most 256 tree
// tokens): the weights stream from HBM once per pass, as the A operand of
// M = 128, N = kN, K = 16 tcgen05 products (TMA boxes of 128 rows x 64
// columns, 128-byte swizzle, no multicast), the tokens' activations are the
// B operand, and the fp32 accumulators live in tensor memory.  Passes hold
// 256 tokens, and the last one the smallest of 64, 128 and 256 that takes the
// rest; a ring stage holds 2 column blocks of 64 at 64 tokens and 1 above.  The
// ring stages of a product are split evenly over the CTAs (stream-K); a tile
// of 128 rows cut by a range boundary is summed, per quarter of its rows, by
// the last CTA to finish it, in CTA order.  The epilogue is fused per
// product:
//   QKV     rotary embedding of q and k at position L_b + depth ((cos, sin)
//           from a table the embedding kernel builds once per forward), q to
//           its buffer, k and v into the cache rows L_b + node
//   RESID   x += product (the fp32 residual stream)
//   SWIGLU  act = SiLU(gate) * up, bf16
//   LOGITS  fp32 logits
// For QKV and SWIGLU the rows of the packed weights interleave the two rows
// an output needs (q/k features i and i + hd/2; gate and up of one feature),
// so the pair sits in lanes 2j and 2j + 1 of one warp.
#include <cfloat>
#include <cudaTypedefs.h>

#include "tcgen05.cuh"

namespace medusa {
namespace {

constexpr int kTileRows = 128;
constexpr int kKStep = 64;
constexpr int kWBlock = kTileRows * 128;       // 16 KB
constexpr int kThreads = 256;                  // warps 0 producer, 1 MMA, 4-7 epilogue
constexpr int kRingBytes = 196608;             // 192 KB of ring stages
constexpr int kMaxN = 256;                     // tokens per pass, at most
constexpr float kRmsEps = 1e-6f;

// The shape of one pass of kN tokens.
template <int kN_>
struct Cfg {
  static constexpr int kKPS = kN_ >= 128 ? 1 : 2;            // column blocks per ring stage
  static constexpr int kXBlock = kN_ * 128;                  // activations of one column block
  static constexpr int kSB = kKPS * (kWBlock + kXBlock);     // bytes per stage: 48, 32, 48 KB
  static constexpr int kNS = kRingBytes / kSB;               // stages: 4, 6, 4
  static constexpr uint32_t kTmemCols = 2 * kN_;             // two accumulators of kN columns
  static constexpr int kTail = 4096;                         // barriers and the token table
  static constexpr int kSmem = 1024 + kNS * kSB + kTail;
};

enum Mode : int { kQKV = 0, kResid = 1, kSwiGLU = 2, kLogits = 3 };

struct GemmArgs {
  int rows;               // weight rows
  int kdim;               // reduction length (a multiple of 128)
  int tiles, nst, W, G;   // tiles of 128 rows, stages per tile, all stages, CTAs
  int kps;                // column blocks per ring stage
  int tok0, ntok;         // this pass: tokens tok0 .. tok0 + kN - 1 (clipped to ntok)
  float* part;            // [G, 2, kN, 128]: each CTA's parts of its first and last tile
  unsigned* tile_cnt;     // [tiles * 4]
  int* status;
  // QKV
  uint16_t* q_out;        // [ntok, H, 128]
  uint16_t* k_cache;      // this layer: [B, H, Lcap, 128]
  uint16_t* v_cache;
  const int32_t* seq_lens;
  const int32_t* depth;   // [T]
  const float2* rope;     // [ntok, 64]: (cos, sin) of each token's angle per frequency
  int T, H, Lcap;
  // RESID
  float* x;               // [ntok, rows]
  // SWIGLU
  uint16_t* act;          // [ntok, rows / 2]
  // LOGITS
  float* logits;          // [ntok, rows]
};

template <int kN, int kNS>
struct Bars {
  uint64_t full[kNS], empty[kNS];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint64_t tail[4];        // per lane quarter: the final unit's chunk split is decided
  int tail_n[4];           // per lane quarter: index of the final unit (-1: no help wanted)
  uint32_t tmem_base;
  int abort;
  // QKV: for each token c of the pass, its cache row offset
  // ((b H) Lcap + L + node) 128 (-1: no valid cache row)
  alignas(16) long long crow[kN];
};

__device__ __forceinline__ int stage_lo(int c, const GemmArgs& a) {
  return static_cast<int>(static_cast<long long>(a.W) * c / a.G);
}
__device__ __forceinline__ int stage_owner(int st, const GemmArgs& a) {
  return static_cast<int>((static_cast<long long>(st + 1) * a.G - 1) / a.W);
}

struct Unit {
  int tile, k0, k1;   // column blocks [k0, k1) of one tile
};

__device__ __forceinline__ bool next_unit(const GemmArgs& a, int& st, int st_hi, Unit& x) {
  if (st >= st_hi) return false;
  x.tile = st / a.nst;
  const int t0 = x.tile * a.nst;
  const int e = st_hi < t0 + a.nst ? st_hi : t0 + a.nst;
  x.k0 = (st - t0) * a.kps;
  x.k1 = (e - t0) * a.kps;
  st = e;
  return true;
}

template <class BarsT>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, BarsT* bs, int* status) {
  if (bs->abort) return false;
  if (mbar_wait(bar, parity)) return true;
  set_device_status(status, MEDUSA_ERR_TIMEOUT, kDetailDecoderWait);
  bs->abort = 1;
  return false;
}

// Orders this thread's earlier memory accesses before its later ones for
// every observer on the GPU (lighter than the sequentially consistent fence).
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// SiLU for a value that is rounded to bf16 next: the fast exponential and
// division (a few ulp of fp32) are far inside bf16's rounding.
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float bf(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// The epilogue of one finished tile row, for the 32 token columns c0 ..
// c0 + 31 (in acc).  Every global load comes before the stores, so the loads
// of the 32 tokens overlap.
constexpr int kHalf = 32;
constexpr int kPar = 3;   // partial sums of a shared tile loaded at once
template <int kMode, int kN, class BarsT>
__device__ __forceinline__ void epilogue_half(const GemmArgs& a, const BarsT* bs, int tile, int r, int c0,
                                              const float (&acc)[kHalf]) {
  const int nvalid = a.ntok - a.tok0 < kN ? a.ntok - a.tok0 : kN;
  if constexpr (kMode == kQKV) {
    const int which = tile / a.H, h = tile - which * a.H;   // 0 q, 1 k, 2 v; head h
    const int j = r >> 1;                                   // pair index (frequency)
    const int feat = j + (r & 1) * 64;                      // feature within the head
    uint16_t* cache = which == 1 ? a.k_cache : a.v_cache;
    // 16 tokens at a time: their cache rows (vector loads), rotations
    // (cos, sin of the token's angle for frequency j, from the forward's
    // table) and partner values first, so that the 16 rotations are
    // independent and no store sits between loads; then the stores, each
    // under its own predicate.
    uint16_t* const dst = which == 0 ? a.q_out + h * 128 + feat : cache + static_cast<long long>(h) * a.Lcap * 128 + feat;
#pragma unroll
    for (int i0 = 0; i0 < kHalf; i0 += 16) {
      long long row[16];
      float other[16];
      float2 rot[16];
      const longlong2* rp = reinterpret_cast<const longlong2*>(bs->crow + c0 + i0);
      if (which < 2) {
        const float2* tp = a.rope + static_cast<size_t>(a.tok0 + c0 + i0) * 64 + j;
#pragma unroll
        for (int i = 0; i < 16; ++i) rot[i] = c0 + i0 + i < nvalid ? tp[i * 64] : make_float2(1.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const longlong2 r2 = rp[k];
        row[2 * k] = r2.x;
        row[2 * k + 1] = r2.y;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) other[i] = __shfl_xor_sync(0xffffffffu, acc[i0 + i], 1);
      uint16_t v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float own = acc[i0 + i];
        float out = own;
        if (which < 2) {
          const float cs = rot[i].x, sn = rot[i].y;
          out = (r & 1) ? other[i] * sn + own * cs : own * cs - other[i] * sn;
        }
        v[i] = f32_to_bf16_rne(out);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = c0 + i0 + i;
        const long long o = which == 0 ? static_cast<long long>(a.tok0 + c) * a.H * 128 : row[i];
        if (c < nvalid && row[i] >= 0) dst[o] = v[i];
      }
    }
  } else if constexpr (kMode == kSwiGLU) {
    // Lanes 2j' (gate) and 2j' + 1 (up) of feature j share the 32 tokens:
    // the even lane finishes tokens 0-15, the odd lane tokens 16-31, each
    // with the other's value for its token.
    const int j = tile * 64 + (r >> 1);   // output feature
    const int odd = r & 1;
    const int hi = odd * (kHalf / 2);
    uint16_t* dst = a.act + static_cast<size_t>(a.tok0 + c0 + hi) * (a.rows / 2) + j;
#pragma unroll
    for (int i = 0; i < kHalf / 2; ++i) {
      const float mine = acc[i + hi];                                       // gate (even) or up (odd)
      const float theirs = __shfl_xor_sync(0xffffffffu, odd ? acc[i] : acc[i + kHalf / 2], 1);
      const float gate = odd ? theirs : mine, up = odd ? mine : theirs;
      if (c0 + hi + i < nvalid && 2 * j < a.rows)
        dst[static_cast<size_t>(i) * (a.rows / 2)] = f32_to_bf16_rne(silu(gate) * up);
    }
  } else if constexpr (kMode == kResid) {
    const int f = tile * kTileRows + r;
    if (f >= a.rows) return;
    // One finishing CTA per element: x + product, added in L2 (a single
    // fp32 addition, as a load, add and store would give), with no load.
    float* xr = a.x + static_cast<size_t>(a.tok0 + c0) * a.rows + f;
#pragma unroll
    for (int i = 0; i < kHalf; ++i)
      if (c0 + i < nvalid) atomicAdd(xr + static_cast<size_t>(i) * a.rows, acc[i]);
  } else {
    const int f = tile * kTileRows + r;
    if (f >= a.rows) return;
    float* lr = a.logits + static_cast<size_t>(a.tok0 + c0) * a.rows + f;
#pragma unroll
    for (int i = 0; i < kHalf; ++i)
      if (c0 + i < nvalid) lr[static_cast<size_t>(i) * a.rows] = acc[i];
  }
}

// The partial sums of a shared tile: CTA cc's slot sl (its first or its last
// tile) holds [kN tokens][128 rows] fp32, token-major, so that a warp's 32
// rows of one token are one 128-byte line.  This returns token c's row 0.
__device__ __forceinline__ float* part_at(const GemmArgs& a, int cc, int sl, int c, int kN) {
  return a.part + ((static_cast<size_t>(cc) * 2 + sl) * kN + c) * kTileRows;
}

// One 32-column chunk of a finished tile row: the accumulator from tensor
// memory, for a shared tile plus the other CTAs' parts (summed in CTA order,
// kPar CTAs' loads in flight at a time), then the epilogue.
template <int kMode, int kN, class BarsT>
__device__ __forceinline__ void finish_chunk(const GemmArgs& a, const BarsT* bs, int tile, int r, uint32_t tacc,
                                             int hh, bool split, int c_first, int c_last, int cta) {
  float acc[kHalf];
  if (!split) {
    tc::tmem_ld32(tacc + hh * kHalf, acc);
    tc::tmem_wait_ld();
  } else {
    // This CTA's own part is read again from tensor memory at its place in
    // the order, so that it holds no registers across the loads.
#pragma unroll
    for (int c = 0; c < kHalf; ++c) acc[c] = 0.f;
#pragma unroll 1
    for (int cc0 = c_first; cc0 <= c_last; cc0 += kPar) {
      float pv[kPar][kHalf];
#pragma unroll
      for (int u = 0; u < kPar; ++u) {
        const int cc = cc0 + u;
        if (cc == cta) {
          tc::tmem_ld32(tacc + hh * kHalf, pv[u]);
        } else if (cc <= c_last) {
          const int sl = tile == stage_lo(cc, a) / a.nst ? 0 : 1;
          const float* pc = part_at(a, cc, sl, hh * kHalf, kN) + r;
#pragma unroll
          for (int i = 0; i < kHalf; ++i) pv[u][i] = __ldcg(pc + i * kTileRows);
        }
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < kPar; ++u)
        if (cc0 + u <= c_last) {
#pragma unroll
          for (int i = 0; i < kHalf; ++i) acc[i] += pv[u][i];
        }
    }
  }
  epilogue_half<kMode, kN>(a, bs, tile, r, hh * kHalf, acc);
}

template <int kMode, int kN>
__global__ void __launch_bounds__(kThreads, 1)
    wgemm_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_map,
                 const GemmArgs a) {
  using C = Cfg<kN>;
  constexpr int kKPS = C::kKPS, kXBlock = C::kXBlock, kSB = C::kSB, kNS = C::kNS;
  constexpr uint32_t kTmemCols = C::kTmemCols;
  using BarsT = Bars<kN, kNS>;
  static_assert(sizeof(BarsT) <= C::kTail, "barrier block too large");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BarsT* bs = reinterpret_cast<BarsT*>(smem + kNS * kSB);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int st_lo = stage_lo(cta, a), st_hi = stage_lo(cta + 1, a);

  if (tid == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&bs->full[s], 1);
      mbar_init(&bs->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bs->acc_full[b], 1);
      mbar_init(&bs->acc_empty[b], 4);
    }
    mbar_init(&bs->mma_done, 1);
    for (int qq = 0; qq < 4; ++qq) mbar_init(&bs->tail[qq], 1);
    bs->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bs->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if constexpr (kMode == kQKV) {
    for (int c = tid; c < kN; c += kThreads) {
      const int n = a.tok0 + c;
      long long row = -1;
      if (n < a.ntok) {
        const int b = n / a.T, node = n - b * a.T;
        const int L = a.seq_lens[b];
        if (L < 0 || L + a.T > a.Lcap)   // the tree's rows would not fit in the cache
          set_device_status(a.status, MEDUSA_ERR_DEVICE_CHECK, kDetailDecoderSeqLen);
        else
          row = (static_cast<long long>(b) * a.H * a.Lcap + L + node) * 128;
      }
      bs->crow[c] = row;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bs->tmem_base;
  allow_dependents();

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tensormap(&w_map);
      tc::prefetch_tensormap(&x_map);
      const uint64_t pol = l2_evict_first_policy();
      // The weights do not depend on the previous kernel: the first stages'
      // weight tiles load before waiting for it, their activations after.
      bool x_ready = false;
      int pend_slot[kNS], pend_k[kNS];
      int npend = 0;
      auto flush = [&]() {
        wait_prior_grids();
        for (int i = 0; i < npend; ++i)
          tc::tma_load_4d(smem + pend_slot[i] * kSB + kKPS * kWBlock, &x_map, 0, a.tok0, pend_k[i], 0,
                          &bs->full[pend_slot[i]]);
        npend = 0;
        x_ready = true;
      };
      int g = 0;
      Unit x;
      for (int st = st_lo; !bs->abort && next_unit(a, st, st_hi, x);) {
        for (int j = x.k0; j < x.k1; j += kKPS, ++g) {
          const int slot = g % kNS;
          if (!x_ready && npend == kNS) flush();
          if (g >= kNS && !wait_or_abort(&bs->empty[slot], ((g / kNS) - 1) & 1, bs, a.status)) break;
          mbar_arrive_expect_tx(&bs->full[slot], kSB);
          unsigned char* sd = smem + slot * kSB;
          tc::tma_load_4d_hint(sd, &w_map, 0, x.tile * kTileRows, j, 0, &bs->full[slot], pol);
          if (x_ready) {
            tc::tma_load_4d(sd + kKPS * kWBlock, &x_map, 0, a.tok0, j, 0, &bs->full[slot]);
          } else {
            pend_slot[npend] = slot;
            pend_k[npend] = j;
            ++npend;
          }
        }
      }
      if (!x_ready) flush();
      for (int t = g - kNS < 0 ? 0 : g - kNS; t < g; ++t) mbar_wait(&bs->full[t % kNS], (t / kNS) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kTileRows, kN, 0);
      const uint32_t sbase = smem_u32(smem);
      int g = 0, n = 0;
      Unit x;
      for (int st = st_lo; !bs->abort && next_unit(a, st, st_hi, x); ++n) {
        const int buf = n & 1;
        if (n >= 2 && !wait_or_abort(&bs->acc_empty[buf], ((n >> 1) - 1) & 1, bs, a.status)) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + buf * kN;
        bool ok = true;
        for (int j = x.k0; j < x.k1; j += kKPS, ++g) {
          const int slot = g % kNS;
          if (!wait_or_abort(&bs->full[slot], (g / kNS) & 1, bs, a.status)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t wa = sbase + slot * kSB, xa = wa + kKPS * kWBlock;
#pragma unroll
          for (int c = 0; c < kKPS; ++c)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = tc::smem_desc_sw128(wa + c * kWBlock + kk * 32, 16, 1024);
              const uint64_t bd = tc::smem_desc_sw128(xa + c * kXBlock + kk * 32, 16, 1024);
              tc::mma_ss(d, ad, bd, idesc, (j > x.k0 || c > 0 || kk > 0) ? 1u : 0u);
            }
          tc::mma_commit(&bs->empty[slot]);
        }
        if (!ok) break;
        tc::mma_commit(&bs->acc_full[buf]);
      }
      tc::mma_commit(&bs->mma_done);
      mbar_wait(&bs->mma_done, 0);
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;
    wait_prior_grids();   // the residual stream and the outputs of the kernels before
    int n = 0;
    bool signalled = false;
    Unit x;
    for (int st = st_lo; next_unit(a, st, st_hi, x); ++n) {
      const int buf = n & 1;
      if (!wait_or_abort(&bs->acc_full[buf], (n >> 1) & 1, bs, a.status)) break;
      tc::fence_after_sync();
      const uint32_t tacc = tmem + lane_off + buf * kN;
      const int t0 = x.tile * a.nst;
      const int c_first = stage_owner(t0, a), c_last = stage_owner(t0 + a.nst - 1, a);
      const bool split = c_first != c_last;
      bool mine_last = true;
      if (split) {
        // A tile shared with other CTAs: store this part; the last to finish
        // sums the parts in CTA order.
        const int slot = x.tile == st_lo / a.nst ? 0 : 1;
        float* mine = part_at(a, cta, slot, 0, kN) + r;
#pragma unroll 1
        for (int hh = 0; hh < kN / kHalf; ++hh) {
          float acc[kHalf];
          tc::tmem_ld32(tacc + hh * kHalf, acc);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kHalf; ++c) mine[(hh * kHalf + c) * kTileRows] = acc[c];
        }
        fence_acq_rel_gpu();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          unsigned* cnt = &a.tile_cnt[x.tile * 4 + q];
          last = atom_add_acq_rel_gpu(cnt, 1u) == static_cast<unsigned>(c_last - c_first);
          if (last) *cnt = 0u;
        }
        mine_last = __shfl_sync(0xffffffffu, last, 0) != 0;
        if (mine_last) fence_acq_rel_gpu();
      }
      // This CTA's final unit ends the kernel for it: when it finishes the
      // tile, warp q of warps 0-3 (idle by now) takes the odd chunks.
      const bool final_unit = st >= st_hi;
      const bool help = final_unit && mine_last && kN / kHalf >= 2;
      if (final_unit) {
        if (lane == 0) {
          bs->tail_n[q] = help ? n : -1;
          tc::mbar_arrive(&bs->tail[q]);
        }
        signalled = true;
      }
      if (mine_last) {
#pragma unroll 1
        for (int hh = 0; hh < kN / kHalf; hh += help ? 2 : 1)
          finish_chunk<kMode, kN>(a, bs, x.tile, r, tacc, hh, split, c_first, c_last, cta);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bs->acc_empty[buf]);
    }
    if (!signalled && lane == 0) {   // no final unit reached (an abort): release the helper
      bs->tail_n[q] = -1;
      tc::mbar_arrive(&bs->tail[q]);
    }
  }
  if (warp < 4) {
    // Warps 0-3, done with their roles: warp q takes the odd chunks of the
    // final unit of lane quarter q when the epilogue warp asks for help.
    __syncwarp();
    const int q = warp;
    if (!mbar_wait(&bs->tail[q], 0)) {
      set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailDecoderWait);
      bs->abort = 1;
    } else if (bs->tail_n[q] >= 0) {
      const int nf = bs->tail_n[q];
      wait_prior_grids();
      tc::fence_after_sync();
      const int tile = (st_hi - 1) / a.nst;
      const int t0 = tile * a.nst;
      const int c_first = stage_owner(t0, a), c_last = stage_owner(t0 + a.nst - 1, a);
      const uint32_t tacc = tmem + (static_cast<uint32_t>(32 * q) << 16) + (nf & 1) * kN;
#pragma unroll 1
      for (int hh = 1; hh < kN / kHalf; hh += 2)
        finish_chunk<kMode, kN>(a, bs, tile, 32 * q + lane, tacc, hh, c_first != c_last, c_first, c_last, cta);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- small kernels ------------------------------------------------------------

// x[n] = embed[tokens[n]] (bf16 -> fp32), n over the B*T tree tokens; and the
// token's rotation table: rope[n][j] = (cos, sin)(p base^(-2j/128)), base
// 10000, at its position p = L_b + depth, the angle reduced in double.
__global__ void embed_kernel(const int32_t* tokens, const uint16_t* embed, int D, int V, float* x,
                             const int32_t* seq_lens, const int32_t* depth, int T, float2* rope, int* status) {
  allow_dependents();
  const int n = blockIdx.x;
  if (threadIdx.x < 64) {
    const int j = threadIdx.x, b = n / T;
    const int p = seq_lens[b] + depth[n - b * T];   // a bad length is reported by the QKV products
    const double ang = static_cast<double>(p) * exp2(-static_cast<double>(2 * j) / 128.0 * 13.287712379549449);
    double sn, cs;
    sincos(ang, &sn, &cs);
    rope[static_cast<size_t>(n) * 64 + j] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
  const int tok = tokens[n];
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) set_device_status(status, MEDUSA_ERR_DEVICE_CHECK, kDetailDecoderToken);
    for (int i = threadIdx.x; i < D; i += blockDim.x) x[static_cast<size_t>(n) * D + i] = 0.f;
    return;
  }
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    x[static_cast<size_t>(n) * D + i] = bf(embed[static_cast<size_t>(tok) * D + i]);
}

// y[n] = bf16(x[n] / sqrt(mean(x[n]^2) + eps) * w), one CTA per token: the
// row is loaded once (16-byte loads, kept in registers), reduced, scaled.
constexpr int kNormThreads = 256;
constexpr int kNormVec = 8;   // float4 per thread: rows of up to 8192 values
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const float* x, const uint16_t* w, int D, uint16_t* y) {
  __shared__ float red[kNormThreads / 32];
  wait_prior_grids();
  allow_dependents();
  const int n = blockIdx.x, tid = threadIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(n) * D);
  const int nv = D / 4;
  float4 v[kNormVec];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kNormVec; ++i) {
    const int k = tid + i * kNormThreads;
    v[i] = k < nv ? xr[k] : make_float4(0.f, 0.f, 0.f, 0.f);
    s = fmaf(v[i].x, v[i].x, fmaf(v[i].y, v[i].y, fmaf(v[i].z, v[i].z, fmaf(v[i].w, v[i].w, s))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((tid & 31) == 0) red[tid >> 5] = s;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < kNormThreads / 32; ++i) t += red[i];
  const float inv = rsqrtf(t / static_cast<float>(D) + kRmsEps);
  uint2* yr = reinterpret_cast<uint2*>(y + static_cast<size_t>(n) * D);
  const uint2* wr = reinterpret_cast<const uint2*>(w);
#pragma unroll
  for (int i = 0; i < kNormVec; ++i) {
    const int k = tid + i * kNormThreads;
    if (k < nv) {
      const uint2 ww = wr[k];
      const float w0 = __uint_as_float(ww.x << 16), w1 = __uint_as_float(ww.x & 0xffff0000u);
      const float w2 = __uint_as_float(ww.y << 16), w3 = __uint_as_float(ww.y & 0xffff0000u);
      uint2 o;
      o.x = static_cast<uint32_t>(f32_to_bf16_rne(v[i].x * inv * w0)) |
            (static_cast<uint32_t>(f32_to_bf16_rne(v[i].y * inv * w1)) << 16);
      o.y = static_cast<uint32_t>(f32_to_bf16_rne(v[i].z * inv * w2)) |
            (static_cast<uint32_t>(f32_to_bf16_rne(v[i].w * inv * w3)) << 16);
      yr[k] = o;
    }
  }
}

bool encode_w(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, uint64_t kdim,
              uint64_t rows, uint32_t box_rows, uint32_t kps) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kKStep), rows, kdim / kKStep, 1};
  const cuuint64_t strides[3] = {kdim * 2, kKStep * 2, kdim * rows * 2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(kKStep), box_rows, kps, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tokens in a pass over ntok remaining tokens: the smallest of 64, 128 and
// 256 that takes all of them, else 256.
int tokens_per_pass(int ntok) { return ntok <= 64 ? 64 : (ntok <= 128 ? 128 : kMaxN); }

// Scratch of the matrix products: tile counters, then [G, 2, kN, 128] partials.
size_t gemm_scratch_bytes(int D, int F, int V, int ntok) {
  int rows = 3 * D;
  if (2 * F > rows) rows = 2 * F;
  if (V > rows) rows = V;
  const int tiles = (rows + kTileRows - 1) / kTileRows;
  const int G = sm_count() > 0 ? sm_count() : 1;
  return align_up(static_cast<size_t>(tiles) * 16, 256) +
         align_up(static_cast<size_t>(G) * 2 * kTileRows * tokens_per_pass(ntok) * 4, 256);
}

template <int kMode, int kN>
medusa_status_t gemm_n(const void* Wt, const uint16_t* X, GemmArgs a, void* ws, cudaStream_t stream) {
  using C = Cfg<kN>;
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_tree_decode: cuTensorMapEncodeTiled unavailable");
  const int G = sm_count();
  a.kps = C::kKPS;
  a.tiles = (a.rows + kTileRows - 1) / kTileRows;
  a.nst = a.kdim / kKStep / C::kKPS;
  a.W = a.tiles * a.nst;
  a.G = a.W < G ? a.W : G;
  unsigned char* w = static_cast<unsigned char*>(ws);
  a.tile_cnt = reinterpret_cast<unsigned*>(w);
  a.part = reinterpret_cast<float*>(w + align_up(static_cast<size_t>(a.tiles) * 4 * 4, 256));
  a.status = device_status_ptr();
  CUtensorMap wm, xm;
  if (!encode_w(enc, &wm, Wt, a.kdim, a.rows, kTileRows, C::kKPS) ||
      !encode_w(enc, &xm, X, a.kdim, a.ntok, kN, C::kKPS))
    return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_tree_decode: tensor map rejected");
  auto fn = wgemm_kernel<kMode, kN>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e == cudaSuccess)
    e = launch_kernel(fn, dim3(a.G), dim3(kThreads), static_cast<size_t>(C::kSmem), stream, true, wm, xm, a);
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_decode: matrix-product launch", e);
}

// Passes of 256 tokens, then one pass for the rest in the smallest of 64,
// 128 and 256 tokens that holds it (a pass costs roughly in proportion to its
// width from 128 tokens up, so a narrow last pass saves most of a wide one).
template <int kMode>
medusa_status_t gemm(const void* Wt, const uint16_t* X, GemmArgs a, void* ws, cudaStream_t stream) {
  for (int tok0 = 0; tok0 < a.ntok;) {
    const int n = tokens_per_pass(a.ntok - tok0);
    a.tok0 = tok0;
    const medusa_status_t st = n == 64    ? gemm_n<kMode, 64>(Wt, X, a, ws, stream)
                               : n == 128 ? gemm_n<kMode, 128>(Wt, X, a, ws, stream)
                                          : gemm_n<kMode, kMaxN>(Wt, X, a, ws, stream);
    if (st != MEDUSA_OK) return st;
    tok0 += n;
  }
  return MEDUSA_OK;
}

}  // namespace

uint16_t* decoder_final_rows(void* ws, int ntok, int D, int F, int V) {
  // the layout of launch_tree_decode: the products' scratch, x, then xn (which
  // holds the final RMSNorm's output once the forward is done)
  const size_t o = gemm_scratch_bytes(D, F, V, ntok) + align_up(static_cast<size_t>(ntok) * D * 4, 256);
  return reinterpret_cast<uint16_t*>(static_cast<unsigned char*>(ws) + o);
}

size_t decoder_workspace_bytes(int ntok, int D, int F, int V) {
  // The products' scratch; then x fp32, xn bf16, q bf16, attention output bf16, act bf16.
  size_t o = gemm_scratch_bytes(D, F, V, ntok);
  o += align_up(static_cast<size_t>(ntok) * D * 4, 256);       // x
  o += align_up(static_cast<size_t>(ntok) * D * 2, 256);       // xn
  o += align_up(static_cast<size_t>(ntok) * D * 2, 256);       // q (bf16, [ntok, H, 128])
  o += align_up(static_cast<size_t>(ntok) * D * 2, 256);       // attention output bf16
  o += align_up(static_cast<size_t>(ntok) * F * 2, 256);       // act
  o += align_up(static_cast<size_t>(ntok) * 64 * 8, 256);      // rotation table
  return o;
}

medusa_status_t launch_tree_decode(const TreeDev& t, const medusa_decoder_t* m, int B, const int32_t* tree_tokens,
                                   void* k_cache, void* v_cache, int Lcap, const int32_t* seq_lens,
                                   float* logits, float* hidden, void* ws, cudaStream_t stream) {
  const int D = m->D, F = m->F, V = m->V, H = D / 128;
  const int ntok = B * t.T;
  unsigned char* w = static_cast<unsigned char*>(ws);
  size_t o = gemm_scratch_bytes(D, F, V, ntok);
  void* gws = w;
  float* x = reinterpret_cast<float*>(w + o);
  o += align_up(static_cast<size_t>(ntok) * D * 4, 256);
  uint16_t* xn = reinterpret_cast<uint16_t*>(w + o);
  o += align_up(static_cast<size_t>(ntok) * D * 2, 256);
  uint16_t* qb = reinterpret_cast<uint16_t*>(w + o);
  o += align_up(static_cast<size_t>(ntok) * D * 2, 256);
  uint16_t* attb = reinterpret_cast<uint16_t*>(w + o);
  o += align_up(static_cast<size_t>(ntok) * D * 2, 256);
  uint16_t* act = reinterpret_cast<uint16_t*>(w + o);
  o += align_up(static_cast<size_t>(ntok) * F * 2, 256);
  float2* rope = reinterpret_cast<float2*>(w + o);
  int* status = device_status_ptr();
  const size_t slab = static_cast<size_t>(B) * H * Lcap * 128;   // one layer of one cache, elements
  const float scale = 1.0f / sqrtf(128.0f);

  embed_kernel<<<ntok, 256, 0, stream>>>(tree_tokens, static_cast<const uint16_t*>(m->embed), D, V, x, seq_lens,
                                         t.depth, t.T, rope, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("medusa_tree_decode: embedding launch", e);
  for (int l = 0; l < m->layers; ++l) {
    const medusa_decoder_layer_t& ly = m->layer[l];
    uint16_t* kc = static_cast<uint16_t*>(k_cache) + static_cast<size_t>(l) * slab;
    uint16_t* vc = static_cast<uint16_t*>(v_cache) + static_cast<size_t>(l) * slab;
    e = launch_kernel(rmsnorm_kernel, dim3(ntok), dim3(kNormThreads), 0, stream, true, static_cast<const float*>(x),
                      static_cast<const uint16_t*>(ly.attn_norm), D, xn);
    if (e != cudaSuccess) return cuda_fail("medusa_tree_decode: RMSNorm launch", e);
    GemmArgs g{};
    g.ntok = ntok;
    g.rows = 3 * D;
    g.kdim = D;
    g.q_out = qb;
    g.k_cache = kc;
    g.v_cache = vc;
    g.seq_lens = seq_lens;
    g.depth = t.depth;
    g.rope = rope;
    g.T = t.T;
    g.H = H;
    g.Lcap = Lcap;
    medusa_status_t st = gemm<kQKV>(ly.wqkv, xn, g, gws, stream);
    if (st != MEDUSA_OK) return st;
    st = launch_attention_bf16_out(t, B, H, qb, kc, vc, Lcap, seq_lens, scale, attb, stream);
    if (st != MEDUSA_OK) return st;
    g = GemmArgs{};
    g.ntok = ntok;
    g.rows = D;
    g.kdim = D;
    g.x = x;
    st = gemm<kResid>(ly.wo, attb, g, gws, stream);
    if (st != MEDUSA_OK) return st;
    e = launch_kernel(rmsnorm_kernel, dim3(ntok), dim3(kNormThreads), 0, stream, true, static_cast<const float*>(x),
                      static_cast<const uint16_t*>(ly.mlp_norm), D, xn);
    if (e != cudaSuccess) return cuda_fail("medusa_tree_decode: RMSNorm launch", e);
    g = GemmArgs{};
    g.ntok = ntok;
    g.rows = 2 * F;
    g.kdim = D;
    g.act = act;
    st = gemm<kSwiGLU>(ly.wgu, xn, g, gws, stream);
    if (st != MEDUSA_OK) return st;
    g = GemmArgs{};
    g.ntok = ntok;
    g.rows = D;
    g.kdim = F;
    g.x = x;
    st = gemm<kResid>(ly.wdown, act, g, gws, stream);
    if (st != MEDUSA_OK) return st;
  }
  if (hidden) {
    e = cudaMemcpyAsync(hidden, x, static_cast<size_t>(ntok) * D * 4, cudaMemcpyDeviceToDevice, stream);
    if (e != cudaSuccess) return cuda_fail("medusa_tree_decode: hidden copy", e);
  }
  e = launch_kernel(rmsnorm_kernel, dim3(ntok), dim3(kNormThreads), 0, stream, true, static_cast<const float*>(x),
                    static_cast<const uint16_t*>(m->final_norm), D, xn);
  if (e != cudaSuccess) return cuda_fail("medusa_tree_decode: RMSNorm launch", e);
  GemmArgs g{};
  g.ntok = ntok;
  g.rows = V;
  g.kdim = D;
  g.logits = logits;
  medusa_status_t st = gemm<kLogits>(m->lm_head, xn, g, gws, stream);
  if (st != MEDUSA_OK) return st;
  e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_decode: launch", e);
}

}  // namespace medusa
