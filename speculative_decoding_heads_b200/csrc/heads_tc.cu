// S1-S3 for 2..16 sequences per pass on the tcgen05 tensor cores.
//
// The heads ("Medusa API参考：核心函数与类详解", MedusaModelABC: medusa_head is
// residual blocks plus a linear layer; "Medusa — 让大模型自己同时猜好几个
// token", 是什么 and 核心要点):
//     u[b,k] = h[b] + SiLU(W1[k] h[b] + b1[k])      z[b,k] = Wout[k] u[b,k]
// and the top-k of every z[b,k].  With several sequences each streamed weight
// row meets B activation vectors: a small matrix product whose A operand is
// the weights and whose B operand is the activations, so the weights are read
// from HBM once per pass whatever B is.
//
// Two persistent launches, one CTA per SM:
//  * phase 1 multiplies W1 (K heads of d x d) by h.  h is bf16, so its B
//    operand is exact (N = B, padded to 16 columns); the epilogue applies the
//    residual block and writes u as a bf16 pair (high part, and the remainder
//    rounded to bf16: about 16 significant bits of the fp32 u) for phase 2.
//  * phase 2 multiplies Wout (K heads of V x d) by those pairs (N = 2B: the
//    products of the high parts and of the remainders accumulate in separate
//    fp32 columns and are added in the epilogue); each epilogue warp keeps a
//    running top-k per sequence; when the head changes the four warps' lists
//    are merged into the CTA's list for that head; the last CTA to finish
//    merges the CTAs' lists and (inside medusa_step) builds the tree.
//  Work split: a phase is a sequence of tiles (128 rows of one head) of
//  d/64/kKPS ring stages each.  In phase 1 every CTA takes an equal
//  contiguous range of stages, so the HBM stream is balanced to one stage; a
//  tile cut by a range boundary is shared by two or three CTAs: each stores
//  its fp32 partial accumulator, and for each quarter of the tile's rows the
//  last CTA to finish (a counter per tile quarter) sums the partials in CTA
//  order and runs the epilogue.  Phase 2 splits at whole tiles (balanced to
//  one tile), so each logit is a single accumulation whose order does not
//  depend on V or on the split.
//    Phase 2 is launched with programmatic dependent launch: its producer
//    streams the first weight tiles before it waits for phase 1's pairs.
//
// Within a CTA: warp 0 issues the TMA loads (2-D tiles of 128 rows x 64
// columns of the weights, 128-byte swizzle, L2 evict-first, no multicast, and
// the matching 64 columns of the activations) into a ring of stages; warp 1
// allocates tensor memory and one thread issues the M = 128, N = 16/32, K = 16
// products (four per stage) into one of two accumulators; warps 4-7 (one per
// tensor-memory lane quarter, a row of the tile per thread) run the epilogue.
// Every wait is bounded and ends in the device status word.
#include <cfloat>
#include <cudaTypedefs.h>

#include "heads_common.cuh"
#include "tcgen05.cuh"

namespace medusa {
namespace {

constexpr int kTileRows = 128;               // weight rows per tile (MMA M)
constexpr int kKStep = 64;                   // weight columns per block (one 128-byte swizzle row)
constexpr int kKPS = 4;                       // blocks per ring stage (one TMA box per operand)
constexpr int kWBlock = kTileRows * 128;     // 16 KB of weights per block
constexpr int kWBytes = kKPS * kWBlock;      // weights per stage
constexpr int kThreads = 256;                // warps 0 producer, 1 MMA, 2-3 idle, 4-7 epilogue
constexpr int kMaxB = 16;                    // sequences per pass (N = 2B <= 32)
constexpr int kMaxStages = 12;
constexpr int kSmemMax = 232448;             // dynamic shared memory per CTA
constexpr int kEpiWarps = 4;
constexpr uint32_t kTmemCols = 64;           // two accumulators of up to 32 columns

struct HTArgs {
  int B, b0, Btot;        // sequences of this pass, the first one, all of them
  int d, V, K, topk;
  int rows;               // rows per head of this phase's matrix (d or V)
  int tph;                // tiles per head: ceil(rows / 128)
  int nst;                // ring stages per tile: d / 64 / kKPS
  int W;                  // stages of the phase: K * tph * nst
  int gran;               // stages per unit of the split (1, or nst: whole tiles)
  int ksteps;             // d / 64 (a multiple of kKPS)
  int G;                  // CTAs
  int NS;                 // ring stages
  const uint16_t* h;      // [Btot, d]
  const uint16_t* b1;     // [K, d]
  uint16_t* X2;           // [K, 2B, d]: row 2b the high parts of u[b], row 2b+1 the remainders
  float* part;            // [G, 2, 128, N] partial accumulators of the first / last tile of each CTA
  unsigned* tile_cnt;     // [K * tph * 4] partials finished per tile quarter (self-resetting)
  float* head_logits;     // nullable [Btot, K, V]
  int32_t* topk_ids;      // [Btot, K, topk]
  float* topk_vals;
  float* cand_vals;       // [B, K, G, topk] lists published by each CTA
  int32_t* cand_ids;
  unsigned* done;         // [1] CTAs finished with phase 2 (self-resetting)
  int do_build;
  TreeBuild build;
  int* status;
};

struct Bars {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int flag;
};

// Dynamic shared memory: the ring (per stage 16 KB of weights, then the
// activation box), the barrier block, then the epilogue's top-k lists.
__host__ __device__ inline int x_bytes(int npad) { return kKPS * npad * 128; }
__host__ __device__ inline int stage_bytes(int npad) { return kWBytes + x_bytes(npad); }
__host__ __device__ inline int lists_bytes(int B, int topk) { return kEpiWarps * B * (2 * topk + 1) * 4; }
__host__ __device__ inline int smem_bytes(int NS, int npad, int B, int topk) {
  return 1024 + NS * stage_bytes(npad) + 1024 + lists_bytes(B, topk);
}

// First stage of CTA c's range, and the CTA whose range holds stage st
// (ranges are equal shares of the W / gran units of gran stages each).
__device__ __forceinline__ int stage_lo(int c, const HTArgs& a) {
  return a.gran * static_cast<int>(static_cast<long long>(a.W / a.gran) * c / a.G);
}
__device__ __forceinline__ int stage_owner(int st, const HTArgs& a) {
  return static_cast<int>((static_cast<long long>(st / a.gran + 1) * a.G - 1) / (a.W / a.gran));
}

struct Unit {
  int tile, head, row0, k0, k1;   // column blocks [k0, k1) of one tile, whole stages
};

// The next unit of a CTA's stage range: the stages from `st` to the end of
// the range or of the tile, whichever comes first.
__device__ __forceinline__ bool next_unit(const HTArgs& a, int& st, int st_hi, Unit& x) {
  if (st >= st_hi) return false;
  x.tile = st / a.nst;
  const int t0 = x.tile * a.nst;
  const int e = st_hi < t0 + a.nst ? st_hi : t0 + a.nst;
  x.head = x.tile / a.tph;
  x.row0 = (x.tile - x.head * a.tph) * kTileRows;
  x.k0 = (st - t0) * kKPS;
  x.k1 = (e - t0) * kKPS;
  st = e;
  return true;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Bars* bs, int* status) {
  if (bs->abort) return false;
  if (mbar_wait(bar, parity)) return true;
  set_device_status(status, MEDUSA_ERR_TIMEOUT, kDetailHeadsStageWait);
  bs->abort = 1;
  return false;
}

__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int kPhase, int kNpad>
__global__ void __launch_bounds__(kThreads, 1)
    heads_tc_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap x_map,
                    const HTArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NS = a.NS;
  constexpr int kSB = kWBytes + kKPS * kNpad * 128;
  Bars* bs = reinterpret_cast<Bars*>(smem + NS * kSB);
  float* lv_all = reinterpret_cast<float*>(smem + NS * kSB + 1024);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int st_lo = stage_lo(cta, a), st_hi = stage_lo(cta + 1, a);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bs->full[s], 1);
      mbar_init(&bs->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bs->acc_full[b], 1);
      mbar_init(&bs->acc_empty[b], kEpiWarps);
    }
    mbar_init(&bs->mma_done, 1);
    bs->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bs->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bs->tmem_base;
  allow_dependents();

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      tc::prefetch_tensormap(&w_map);
      tc::prefetch_tensormap(&x_map);
      const uint64_t pol = l2_evict_first_policy();
      // Phase 2's activations come from phase 1: until the previous grid is
      // done only the weights of the first stages are loaded.
      bool x_ready = kPhase == 1;
      int pend_slot[kMaxStages], pend_k[kMaxStages], pend_head[kMaxStages];
      int npend = 0;
      auto flush = [&]() {
        wait_prior_grids();
        for (int i = 0; i < npend; ++i)
          tc::tma_load_4d(smem + pend_slot[i] * kSB + kWBytes, &x_map, 0, 0, pend_k[i], pend_head[i],
                          &bs->full[pend_slot[i]]);
        npend = 0;
        x_ready = true;
      };
      int g = 0;
      Unit x;
      for (int st = st_lo; !bs->abort && next_unit(a, st, st_hi, x);) {
        for (int j = x.k0; j < x.k1; j += kKPS, ++g) {
          const int slot = g % NS;
          if (!x_ready && npend == NS) flush();
          if (g >= NS && !wait_or_abort(&bs->empty[slot], ((g / NS) - 1) & 1, bs, a.status)) break;
          mbar_arrive_expect_tx(&bs->full[slot], kSB);
          tc::tma_load_4d_hint(smem + slot * kSB, &w_map, 0, x.row0, j, x.head, &bs->full[slot], pol);
          const int xh = kPhase == 1 ? 0 : x.head;
          if (x_ready) {
            tc::tma_load_4d(smem + slot * kSB + kWBytes, &x_map, 0, 0, j, xh, &bs->full[slot]);
          } else {
            pend_slot[npend] = slot;
            pend_k[npend] = j;
            pend_head[npend] = xh;
            ++npend;
          }
        }
      }
      if (!x_ready) flush();
      // Every copy issued lands before the CTA exits (after an abort the
      // consumer may not have waited for the last ones).
      for (int t = g - NS < 0 ? 0 : g - NS; t < g; ++t) mbar_wait(&bs->full[t % NS], (t / NS) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kTileRows, kNpad, 0);
      const uint32_t sbase = smem_u32(smem);
      int g = 0, n = 0;
      Unit x;
      for (int st = st_lo; !bs->abort && next_unit(a, st, st_hi, x); ++n) {
        const int buf = n & 1;
        if (n >= 2 && !wait_or_abort(&bs->acc_empty[buf], ((n >> 1) - 1) & 1, bs, a.status)) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + buf * kNpad;
        bool ok = true;
        for (int j = x.k0; j < x.k1; j += kKPS, ++g) {
          const int slot = g % NS;
          if (!wait_or_abort(&bs->full[slot], (g / NS) & 1, bs, a.status)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t wa = sbase + slot * kSB, xa = wa + kWBytes;
#pragma unroll
          for (int c = 0; c < kKPS; ++c)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = tc::smem_desc_sw128(wa + c * kWBlock + kk * 32, 16, 1024);
              const uint64_t bd = tc::smem_desc_sw128(xa + c * kNpad * 128 + kk * 32, 16, 1024);
              tc::mma_ss(d, ad, bd, idesc, (j > x.k0 || c > 0 || kk > 0) ? 1u : 0u);
            }
          tc::mma_commit(&bs->empty[slot]);
        }
        if (!ok) break;
        tc::mma_commit(&bs->acc_full[buf]);
      }
      // Every product issued is done before the CTA leaves.
      tc::mma_commit(&bs->mma_done);
      mbar_wait(&bs->mma_done, 0);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: row 32q + lane of each tile ----------------
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int r = 32 * q + lane;
    const int B = a.B, topk = a.topk;
    // Phase 2: each warp's running lists, one per sequence, for the current head.
    const int lstride = B * (2 * topk + 1);
    float* lv = lv_all + static_cast<size_t>(q) * lstride;
    int* li = reinterpret_cast<int*>(lv + B * topk);
    int* ln = li + B * topk;
    int cur_head = -1;
    auto reset_lists = [&]() {
      for (int i = lane; i < B * topk; i += 32) {
        lv[i] = -FLT_MAX;
        li[i] = -1;
      }
      for (int i = lane; i < B; i += 32) ln[i] = 0;
      __syncwarp();
    };
    // The four warps' lists of head k become this CTA's list for k.  Called by
    // all four warps at the same units whether or not the CTA has aborted, so
    // the named barriers always match.
    auto flush = [&](int k) {
      epi_sync();
      if (q == 0) {
        for (int b = 0; b < B; ++b) {
          float cv[4];
          int ci[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int c = lane + 32 * m, w = c / topk, j = c - w * topk;
            const bool in = c < kEpiWarps * topk;
            const float* wl = lv_all + static_cast<size_t>(w) * lstride;
            cv[m] = in ? wl[b * topk + j] : -FLT_MAX;
            ci[m] = in ? reinterpret_cast<const int*>(wl + B * topk)[b * topk + j] : -1;
          }
          float pv = FLT_MAX;
          int pi = -1;
          for (int rr = 0; rr < topk; ++rr) {
            float bv = -FLT_MAX;
            int bi = 0x7fffffff;
#pragma unroll
            for (int m = 0; m < 4; ++m)
              if (ci[m] >= 0 && ranks_before(pv, pi, cv[m], ci[m]) && ranks_before(cv[m], ci[m], bv, bi)) {
                bv = cv[m];
                bi = ci[m];
              }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
              const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
              if (ranks_before(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
              }
            }
            if (lane == 0) {
              const size_t o = ((static_cast<size_t>(b) * a.K + k) * a.G + cta) * topk + rr;
              a.cand_vals[o] = bi == 0x7fffffff ? -FLT_MAX : bv;
              a.cand_ids[o] = bi == 0x7fffffff ? -1 : bi;
            }
            pv = bv;
            pi = bi;
          }
        }
      }
      epi_sync();
      reset_lists();
    };
    if (kPhase == 2) reset_lists();
    int n = 0;
    Unit x;
    for (int st = st_lo; next_unit(a, st, st_hi, x); ++n) {
      if constexpr (kPhase == 2) {
        if (x.head != cur_head) {
          if (cur_head >= 0) flush(cur_head);
          cur_head = x.head;
        }
      }
      const int buf = n & 1;
      if (!wait_or_abort(&bs->acc_full[buf], (n >> 1) & 1, bs, a.status)) {
        if (kPhase == 1) break;
        continue;   // phase 2 keeps the flush schedule
      }
      tc::fence_after_sync();
      float acc[kNpad];
      if constexpr (kNpad == 16) {
        tc::tmem_ld16(tmem + lane_off + buf * kNpad, acc);
      } else {
        tc::tmem_ld32(tmem + lane_off + buf * kNpad, acc);
      }
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bs->acc_empty[buf]);

      // A tile shared with other CTAs: store this CTA's partial accumulator;
      // for each quarter of the rows the last CTA to finish sums the partials
      // in CTA order and runs the epilogue.
      const int ncol = kPhase == 1 ? B : 2 * B;
      const int t0 = x.tile * a.nst;
      const int c_first = stage_owner(t0, a), c_last = stage_owner(t0 + a.nst - 1, a);
      if (c_first != c_last) {
        const int slot = x.tile == st_lo / a.nst ? 0 : 1;
        float* mine = a.part + ((static_cast<size_t>(cta) * 2 + slot) * kTileRows + r) * ncol;
#pragma unroll
        for (int b = 0; b < kNpad; ++b)
          if (b < ncol) mine[b] = acc[b];
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          unsigned* cnt = &a.tile_cnt[x.tile * kEpiWarps + q];
          last = atom_add_acq_rel_gpu(cnt, 1u) == static_cast<unsigned>(c_last - c_first);
          if (last) *cnt = 0u;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
        float sum[kNpad];
#pragma unroll
        for (int b = 0; b < kNpad; ++b) sum[b] = 0.f;
        for (int c = c_first; c <= c_last; ++c) {
          const int sl = x.tile == stage_lo(c, a) / a.nst ? 0 : 1;
          const float* pc = a.part + ((static_cast<size_t>(c) * 2 + sl) * kTileRows + r) * ncol;
#pragma unroll
          for (int b = 0; b < kNpad; ++b)
            if (b < ncol) sum[b] += (c == cta) ? acc[b] : __ldcg(pc + b);
        }
#pragma unroll
        for (int b = 0; b < kNpad; ++b) acc[b] = sum[b];
      }
      if constexpr (kPhase == 1) {
        const int i = x.row0 + r;   // output feature of head x.head (d is a multiple of 128)
        const float bias = __uint_as_float(static_cast<uint32_t>(a.b1[static_cast<size_t>(x.head) * a.d + i]) << 16);
        uint16_t* x2 = a.X2 + static_cast<size_t>(x.head) * 2 * B * a.d + i;
#pragma unroll
        for (int b = 0; b < kNpad; ++b) {
          if (b < B) {
            const float hb = __uint_as_float(static_cast<uint32_t>(a.h[static_cast<size_t>(a.b0 + b) * a.d + i]) << 16);
            const float uu = hb + silu(acc[b] + bias);
            const uint16_t hi = f32_to_bf16_rne(uu);
            const uint16_t lo = f32_to_bf16_rne(uu - __uint_as_float(static_cast<uint32_t>(hi) << 16));
            x2[static_cast<size_t>(2 * b) * a.d] = hi;
            x2[static_cast<size_t>(2 * b + 1) * a.d] = lo;
          }
        }
      } else {
        const int v = x.row0 + r;
        const bool valid = v < a.V;
#pragma unroll
        for (int b = 0; b < kNpad / 2; ++b) {
          if (b < B) {
            const float z = acc[2 * b] + acc[2 * b + 1];
            if (valid && a.head_logits)
              a.head_logits[(static_cast<size_t>(a.b0 + b) * a.K + x.head) * a.V + v] = z;
            float* l_v = lv + b * topk;
            int* l_i = li + b * topk;
            const bool cand = valid && (ln[b] < topk || ranks_before(z, v, l_v[topk - 1], l_i[topk - 1]));
            unsigned m = __ballot_sync(0xffffffffu, cand);
            while (m) {
              const int src = __ffs(m) - 1;
              m &= m - 1;
              const float nv = __shfl_sync(0xffffffffu, z, src);
              const int nid = __shfl_sync(0xffffffffu, v, src);
              // a later candidate of the same ballot may no longer qualify
              if (ln[b] < topk || ranks_before(nv, nid, l_v[topk - 1], l_i[topk - 1]))
                list_insert(l_v, l_i, ln + b, topk, nv, nid, lane);
            }
          }
        }
      }
    }
    if (kPhase == 2 && cur_head >= 0) flush(cur_head);
  }

  // ---------------- end: the last CTA merges the lists ----------------
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  if (kPhase == 1 || bs->abort) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned done = atom_add_acq_rel_gpu(a.done, 1u);
    bs->flag = done == static_cast<unsigned>(a.G - 1);
    if (bs->flag) *a.done = 0u;
  }
  __syncthreads();
  if (!bs->flag) return;
  __threadfence();
  const int per_head = a.tph * a.nst;
  for (int lidx = warp; lidx < a.B * a.K; lidx += kThreads / 32) {
    const int b = lidx / a.K, k = lidx - b * a.K;
    const int c_lo = stage_owner(k * per_head, a);
    const int c_hi = stage_owner((k + 1) * per_head - 1, a);
    const size_t base = ((static_cast<size_t>(b) * a.K + k) * a.G + c_lo) * a.topk;
    const size_t o = (static_cast<size_t>(a.b0 + b) * a.K + k) * a.topk;
    merge_candidates(a.cand_vals + base, a.cand_ids + base, (c_hi - c_lo + 1) * a.topk, a.topk, a.topk_ids + o,
                     a.topk_vals + o, lane);
  }
  if (a.do_build) {
    __syncthreads();
    build_tree_block(a.build, a.Btot, a.topk_ids);
  }
}

struct Layout {
  size_t x2, part, tile_cnt, cand_v, cand_i, done, total;
};

Layout make_layout(int B, int d, int V, int K, int topk, int G) {
  const int nb = B < kMaxB ? B : kMaxB;
  const size_t tiles1 = static_cast<size_t>(K) * (d / kTileRows);
  const size_t tiles2 = static_cast<size_t>(K) * ((V + kTileRows - 1) / kTileRows);
  Layout l{};
  size_t o = 0;
  l.x2 = o;
  o += align_up(static_cast<size_t>(K) * 2 * nb * d * 2, 256);
  l.part = o;
  o += align_up(static_cast<size_t>(G) * 2 * kTileRows * 2 * nb * 4, 256);
  l.tile_cnt = o;
  o += align_up((tiles1 > tiles2 ? tiles1 : tiles2) * kEpiWarps * 4, 256);
  const size_t nc = static_cast<size_t>(nb) * K * G * topk;
  l.cand_v = o;
  o += align_up(nc * 4, 256);
  l.cand_i = o;
  o += align_up(nc * 4, 256);
  l.done = o;
  o += 256;
  l.total = o;
  return l;
}

template <int kPhase, int kNpad>
cudaError_t launch_phase(const CUtensorMap& wm, const CUtensorMap& xm, const HTArgs& a, int grid, cudaStream_t stream,
                         bool pdl) {
  auto fn = heads_tc_kernel<kPhase, kNpad>;
  const int smem = smem_bytes(a.NS, kNpad, kPhase == 2 ? a.B : 0, a.topk);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(fn, dim3(grid), dim3(kThreads), static_cast<size_t>(smem), stream, pdl, wm, xm, a);
}

// A [outer][mid][inner] bf16 array as a 4-D map {64 columns, mid rows, inner/64
// blocks, outer} (the block dimension has the 128-byte stride, so one box of
// {64, box_mid, kKPS, 1} lands as kKPS consecutive canonical 128-byte-swizzled
// tiles of box_mid rows each).
bool encode4(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid,
             uint64_t outer, uint32_t box_mid) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kKStep), mid, inner / kKStep, outer};
  const cuuint64_t strides[3] = {inner * 2, kKStep * 2, inner * mid * 2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(kKStep), box_mid, static_cast<cuuint32_t>(kKPS), 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool heads_tc_supported(int B, int d, medusa_dtype_t dtype) {
  return dtype == MEDUSA_BF16 && B >= 2 && d % kTileRows == 0;
}

size_t heads_tc_workspace_bytes(int B, int d, int V, int K, int topk) {
  (void)V;
  return make_layout(B, d, V, K, topk, sm_count()).total;
}

medusa_status_t launch_heads_tc(const void* h, const void* W1, const void* b1, const void* Wout, int B, int d, int V,
                                int K, int topk, float* head_logits, int32_t* topk_ids, float* topk_vals, void* ws,
                                cudaStream_t stream, const TreeBuild* build) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_heads_topk: cuTensorMapEncodeTiled unavailable");
  const int G = sm_count();
  const Layout l = make_layout(B, d, V, K, topk, G);
  unsigned char* w = static_cast<unsigned char*>(ws);
  HTArgs a{};
  a.Btot = B;
  a.d = d;
  a.V = V;
  a.K = K;
  a.topk = topk;
  a.ksteps = d / kKStep;
  a.h = static_cast<const uint16_t*>(h);
  a.b1 = static_cast<const uint16_t*>(b1);
  a.X2 = reinterpret_cast<uint16_t*>(w + l.x2);
  a.part = reinterpret_cast<float*>(w + l.part);
  a.tile_cnt = reinterpret_cast<unsigned*>(w + l.tile_cnt);
  a.cand_vals = reinterpret_cast<float*>(w + l.cand_v);
  a.cand_ids = reinterpret_cast<int32_t*>(w + l.cand_i);
  a.done = reinterpret_cast<unsigned*>(w + l.done);
  a.head_logits = head_logits;
  a.topk_ids = topk_ids;
  a.topk_vals = topk_vals;
  a.status = device_status_ptr();
  for (int b0 = 0; b0 < B; b0 += kMaxB) {
    const int nb = B - b0 < kMaxB ? B - b0 : kMaxB;
    a.b0 = b0;
    a.B = nb;
    a.do_build = (build != nullptr && b0 + nb == B) ? 1 : 0;
    if (build) a.build = *build;
    // ---- phase 1: W1 x h -> u pairs
    {
      HTArgs p = a;
      p.rows = d;
      p.tph = d / kTileRows;
      p.nst = d / kKStep / kKPS;
      p.W = K * p.tph * p.nst;
      p.gran = 1;
      const int npad = 16;   // B <= 16 columns of h
      p.NS = (kSmemMax - smem_bytes(0, npad, 0, topk)) / stage_bytes(npad);
      if (p.NS > kMaxStages) p.NS = kMaxStages;
      p.G = p.W < G ? p.W : G;
      CUtensorMap wm, xm;
      if (!encode4(enc, &wm, W1, d, d, K, kTileRows) ||
          !encode4(enc, &xm, static_cast<const uint16_t*>(h) + static_cast<size_t>(b0) * d, d, nb, 1, npad))
        return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_heads_topk: phase-1 tensor map rejected");
      const cudaError_t e = launch_phase<1, 16>(wm, xm, p, p.G, stream, false);
      if (e != cudaSuccess) return cuda_fail("medusa_heads_topk: tensor-core phase 1 launch", e);
    }
    // ---- phase 2: Wout x u pairs -> logits, top-k
    {
      HTArgs p = a;
      p.rows = V;
      p.tph = (V + kTileRows - 1) / kTileRows;
      p.nst = d / kKStep / kKPS;
      p.W = K * p.tph * p.nst;
      // Whole tiles: every logit is one accumulation over d in the same order
      // whatever V is, so vocabulary shards reproduce the unsplit logits.
      p.gran = p.nst;
      const int npad = 2 * nb <= 16 ? 16 : 32;
      p.NS = (kSmemMax - smem_bytes(0, npad, nb, topk)) / stage_bytes(npad);
      if (p.NS > kMaxStages) p.NS = kMaxStages;
      p.G = K * p.tph < G ? K * p.tph : G;
      CUtensorMap wm, xm;
      if (!encode4(enc, &wm, Wout, d, V, K, kTileRows) || !encode4(enc, &xm, a.X2, d, 2 * nb, K, npad))
        return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_heads_topk: phase-2 tensor map rejected");
      const cudaError_t e = npad == 16 ? launch_phase<2, 16>(wm, xm, p, p.G, stream, true)
                                       : launch_phase<2, 32>(wm, xm, p, p.G, stream, true);
      if (e != cudaSuccess) return cuda_fail("medusa_heads_topk: tensor-core phase 2 launch", e);
    }
  }
  return MEDUSA_OK;
}

}  // namespace medusa
