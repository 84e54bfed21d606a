// S5 (bf16, hd = 128): a persistent tcgen05 kernel that streams the K/V of
// every (layer, sequence, head) slice through shared memory and keeps the
// memory pipeline full across slice boundaries.  A work item is one slice and
// one group of 64 tree tokens (query rows); trees of up to 64 tokens have one
// group, so every K/V byte is read once; larger trees (up to 256 tokens)
// stream a slice's K/V once per group.
//
// The mask is that of "Medusa — 让大模型自己同时猜好几个 token" (核心要点:
// the candidate tree is verified in one forward under a tree mask; 实践案例
// case 3: a node sees the cached prefix, its ancestors and itself).
//
// Layout of the work.  One CTA per SM walks the items w = cta, cta + grid, ...
// (item w: slice w / groups, row group w % groups).  Each item is cut into
// steps of 128 keys.  K and V tiles (32 KB each, two
// 64-dim halves in 128-byte swizzle) arrive by TMA (no multicast) into two
// three-stage rings: a K stage is released as soon as S of its step is done,
// a V stage once P V of its step is done.  The 64 query rows of a slice sit
// in one of two Q buffers, so the next slice's Q loads while the current one
// finishes.
//
// Tensor memory (512 columns):
//   S  cols [0, 128)   M = 64 product: query 16q + i of step g in lane
//                      32q + 16 (g & 1) + i, so two consecutive steps use the
//                      two lane halves of the same columns
//   P  cols [128, 192) and [192, 256), alternating by step; an M = 128
//                      operand: lane 32q + i holds the bf16 high parts of
//                      query 16q + i, lane 32q + 16 + i the remainders, two
//                      keys per column
//   O  cols [256, 384) and [384, 512), one per slice parity; lanes as P, so
//                      O(query) = O(lane 32q + i) + O(lane 32q + 16 + i).
// A softmax thread pair (i, 16 + i) of warp quarter q owns query 16q + i:
// thread i keys 0-63 of each step, thread 16 + i keys 64-127 (16x32bx2 TMEM
// accesses put both halves of a row in one warp without any exchange).
//
// Warp roles: warp 0 TMA producer; warp 1 TMEM allocation and the single MMA
// issuer; warps 4-7 softmax (one per TMEM lane quarter); warps 2, 3, 8, 9
// epilogue (lane quarters 2, 3, 0, 1), so writing a slice's output overlaps
// the next slice.  Every wait is bounded.
#include <cfloat>
#include <cudaTypedefs.h>

#include "tcgen05.cuh"

namespace medusa {
namespace {

constexpr int kHd = 128;
constexpr int kStep = 128;                     // keys per step
constexpr int kRows = 64;                      // query rows (tree tokens) per slice
constexpr int kStages = 3;
constexpr int kHalfTile = kStep * 128;         // 128 keys x 64 dims x 2 B = 16 KB
constexpr int kTile = 2 * kHalfTile;           // one K or V tile: 32 KB
constexpr int kQHalf = kRows * 128;            // 64 rows x 64 dims x 2 B = 8 KB
constexpr int kQBuf = 2 * kQHalf;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
__device__ __forceinline__ uint32_t col_p(int buf) { return 128u + 64u * buf; }   // 64 packed columns
__device__ __forceinline__ uint32_t col_o(int buf) { return 256u + 128u * buf; }  // 128 fp32 columns
constexpr uint32_t kLaneHalf = 16u << 16;      // TMEM address offset of lane 16
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kLenTab = 160;                   // prefix lengths of a CTA's first slices, in shared memory
// The polling loops of the producer and the MMA issuer give up after this
// many SM cycles without progress (about 2 s at 2 GHz); the SM cycle counter
// is read on every pass, the global timer is too slow for that.
constexpr long long kSpinLimitCycles = 4000000000LL;

struct Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_free[2];     // by S lane half (step parity)
  uint64_t p_full[2], pv_done[2];    // by P buffer (step parity)
  uint64_t o_full[2], o_free[2], l_ready[2];   // by O buffer (slice parity)
  uint32_t tmem_base;
  int abort;
  float lsum[2][kRows];              // row sums handed to the epilogue warps
  int lens[kLenTab];                 // lens[k]: prefix length of this CTA's slice k
};

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;                               // 2 x 16 KB
constexpr int kOffK = 2 * kQBuf;                       // 3 x 32 KB
constexpr int kOffV = kOffK + kStages * kTile;         // 3 x 32 KB
constexpr int kOffBars = kOffV + kStages * kTile;
constexpr int kBarsBytes = 1664;
constexpr int kSmemBytes = kOffBars + kBarsBytes + 1024;
static_assert(sizeof(Bars) <= kBarsBytes, "barrier block too large");
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Slice {
  int slice, lb, e, L, n, steps;
  int item, grp;   // work item index; query rows 64 grp .. 64 grp + 63
  int k0;          // first key row of this launch's window (0 unless split along L)
  int plim;        // prefix keys below plim are visible
  int last;        // the window holds the tree's own rows (the last rank of a split)
};

struct Params {
  TreeDev t;
  int B, H, Lcap, total;   // total: work items = slices x groups
  int groups;              // ceil(T / 64)
  int row_lo, row_hi;      // tree tokens (query rows) handled by this launch
  const int32_t* seq_lens;
  float scale_log2;
  float* out;
  uint16_t* out_bf16;      // if set, the output goes here as bf16 instead of `out`
  int wait_first;          // wait for the preceding kernel before the first load
  int* status;
  int kv_one_box;   // 1: one 32 KB TMA box per tile (4-D map), 0: two 16 KB boxes
  int split_r, split_G;   // this launch is window split_r of split_G along the prefix (0, 1: all of it)
  float* lse;             // [layers, B, T, H] natural-log sum of exp(scale q.k) over the window, or null
};

// Work item kk of this CTA; steps = 0 when it does not exist or fails its
// check (slice >= total marks the end).  The prefix length comes from the
// shared table for the first kLenTab items (no global load on any role's
// critical path at an item boundary).
template <bool kSplit>
__device__ __forceinline__ Slice slice_info(int kk, const Params& p, const int* lens) {
  Slice s{};
  s.item = blockIdx.x + kk * gridDim.x;
  if (s.item >= p.total) {
    s.slice = p.total;
    return s;
  }
  s.slice = s.item / p.groups;
  s.grp = s.item - s.slice * p.groups;
  s.e = s.slice % p.H;
  s.lb = s.slice / p.H;
  s.L = kk < kLenTab ? lens[kk] : p.seq_lens[s.lb % p.B];
  if constexpr (kSplit) {
    // Window split_r of split_G: prefix rows [L r / G, L (r+1) / G), and the
    // tree's own rows with the last window (contiguous with its prefix rows).
    const int r = p.split_r, G = p.split_G;
    const long long L = s.L;
    s.last = r == G - 1;
    s.k0 = static_cast<int>(L * r / G);
    const int hi = static_cast<int>(L * (r + 1) / G);
    s.plim = s.last ? s.L : hi;
    s.n = s.last ? s.L + p.t.T - s.k0 : hi - s.k0;
  } else {
    s.last = 1;
    s.k0 = 0;
    s.plim = s.L;
    s.n = s.L + p.t.T;
  }
  s.steps = (s.L >= 0 && s.L + p.t.T <= p.Lcap && s.n > 0) ? (s.n + kStep - 1) / kStep : 0;
  return s;
}

// First slice at or after kk that passes its check (kk is advanced to it).
template <bool kSplit>
__device__ __forceinline__ Slice seek(int& kk, const Params& p, const int* lens) {
  Slice s = slice_info<kSplit>(kk, p, lens);
  while (s.slice < p.total && s.steps == 0) s = slice_info<kSplit>(++kk, p, lens);
  return s;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* b, int* status) {
  if (b->abort) return false;
  if (mbar_wait(bar, parity)) return true;
  set_device_status(status, MEDUSA_ERR_TIMEOUT, kDetailAttnStageWait);
  b->abort = 1;
  return false;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values in one register pair, and the packed fp32 FMA of sm_100
// (two independent IEEE fmas per instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Keys of step t that belong to the slice (1..128).
__device__ __forceinline__ int step_keys(const Slice& s, int t) {
  const int first = s.n - t * kStep;
  return first < kStep ? first : kStep;
}

// ---- TMA producer (one thread) ----------------------------------------------
// Three streams, each issued as soon as its buffer is free: Q rows of every
// slice, K tiles and V tiles of every step.
template <bool kSplit>
__device__ void run_producer(const CUtensorMap* q_map, const CUtensorMap* k_map, const CUtensorMap* v_map,
                             const Params& p, unsigned char* smem, Bars* bar) {
  tc::prefetch_tensormap(q_map);
  tc::prefetch_tensormap(k_map);
  tc::prefetch_tensormap(v_map);
  if (p.wait_first) wait_prior_grids();   // q and the tree's K/V rows come from it
  int kkq = 0, kkk = 0, kkv = 0;
  Slice sq = seek<kSplit>(kkq, p, bar->lens), sk = seek<kSplit>(kkk, p, bar->lens), sv = seek<kSplit>(kkv, p, bar->lens);
  int nq = 0, gk = 0, gv = 0, tk = 0, tv = 0;     // loads issued; step within slice
  long long last = clock64();
  while ((sq.slice < p.total || sk.slice < p.total || sv.slice < p.total) && !bar->abort) {
    bool progressed = false;
    if (sq.slice < p.total && (nq < 2 || mbar_test(&bar->q_empty[nq & 1], ((nq >> 1) - 1) & 1))) {
      unsigned char* qd = smem + kOffQ + (nq & 1) * kQBuf;
      uint64_t* fb = &bar->q_full[nq & 1];
      mbar_arrive_expect_tx(fb, kQBuf);
      tc::tma_load_4d(qd, q_map, 0, sq.e, p.row_lo + kRows * sq.grp, sq.lb, fb);
      tc::tma_load_4d(qd + kQHalf, q_map, 64, sq.e, p.row_lo + kRows * sq.grp, sq.lb, fb);
      ++nq;
      ++kkq;
      sq = seek<kSplit>(kkq, p, bar->lens);
      progressed = true;
    }
    for (int which = 0; which < 2; ++which) {
      Slice& s = which == 0 ? sk : sv;
      int& g = which == 0 ? gk : gv;
      int& t = which == 0 ? tk : tv;
      int& kk = which == 0 ? kkk : kkv;
      if (s.slice >= p.total) continue;
      const int st = g % kStages;
      uint64_t* eb = which == 0 ? &bar->k_empty[st] : &bar->v_empty[st];
      if (g >= kStages && !mbar_test(eb, ((g / kStages) - 1) & 1)) continue;
      uint64_t* fb = which == 0 ? &bar->k_full[st] : &bar->v_full[st];
      unsigned char* d = smem + (which == 0 ? kOffK : kOffV) + st * kTile;
      const CUtensorMap* m = which == 0 ? k_map : v_map;
      mbar_arrive_expect_tx(fb, kTile);
      if (p.kv_one_box) {
        tc::tma_load_4d(d, m, 0, s.k0 + t * kStep, 0, s.slice, fb);
      } else {
        tc::tma_load_3d(d, m, 0, s.k0 + t * kStep, s.slice, fb);
        tc::tma_load_3d(d + kHalfTile, m, 64, s.k0 + t * kStep, s.slice, fb);
      }
      ++g;
      if (++t == s.steps) {
        t = 0;
        ++kk;
        s = seek<kSplit>(kk, p, bar->lens);
      }
      progressed = true;
    }
    if (progressed) {
      last = clock64();
    } else {
      if (clock64() - last > kSpinLimitCycles) {
        set_device_status(p.status, MEDUSA_ERR_TIMEOUT, kDetailAttnStageWait);
        bar->abort = 1;
        break;
      }
      __nanosleep(32);
    }
  }
  // Every copy issued must have landed before the CTA exits (on the normal
  // path they all have; after an abort this waits, bounded, for the rest).
  for (int b = 0; b < 2; ++b) {
    const int j = nq - 1 - ((nq - 1 - b) & 1);   // last Q load into buffer b
    if (j >= 0 && (j & 1) == b) mbar_wait(&bar->q_full[b], (j >> 1) & 1);
  }
  for (int st = 0; st < kStages; ++st) {
    for (int which = 0; which < 2; ++which) {
      const int g = which == 0 ? gk : gv;
      if (g <= st) continue;
      const int j = st + ((g - 1 - st) / kStages) * kStages;   // last load into stage st
      mbar_wait(which == 0 ? &bar->k_full[st] : &bar->v_full[st], (j / kStages) & 1);
    }
  }
}

// ---- MMA issuer (one thread) ------------------------------------------------
// S(g) = Q K^T of step g (M = 64, N = 128, 8 products over the head dim) and
// O += P(g) V (M = 128, N = 128, one product per 16 valid keys).  Both are
// issued as soon as their inputs are ready: S(g) needs K(g) and its TMEM lane
// half back from the softmax of step g - 2, not P V(g - 1), so the products
// of later steps run while the softmax of this one computes.
template <bool kSplit>
__device__ void run_mma(const Params& p, uint32_t sbase, uint32_t tmem, Bars* bar) {
  constexpr uint32_t idS = tc::idesc_bf16_f32(64, kStep, 0);
  constexpr uint32_t idO = tc::idesc_bf16_f32(128, kHd, 1);
  int kks = 0, kkp = 0;
  Slice ss = seek<kSplit>(kks, p, bar->lens), sp = seek<kSplit>(kkp, p, bar->lens);
  int gs = 0, ts = 0, ks = 0;     // S cursor: global step, step in slice, slice count
  int gp = 0, tp = 0, kp = 0;     // P V cursor
  long long last = clock64();
  while ((ss.slice < p.total || sp.slice < p.total) && !bar->abort) {
    bool progressed = false;
    if (ss.slice < p.total && (ts != 0 || mbar_test(&bar->q_full[ks & 1], (ks >> 1) & 1)) &&
        mbar_test(&bar->k_full[gs % kStages], (gs / kStages) & 1) &&
        (gs < 2 || mbar_test(&bar->s_free[gs & 1], ((gs >> 1) - 1) & 1))) {
      tc::fence_after_sync();
      const uint32_t qa = sbase + kOffQ + (ks & 1) * kQBuf;
      const uint32_t kb = sbase + kOffK + (gs % kStages) * kTile;
      const uint32_t d = tmem + (gs & 1) * kLaneHalf + kColS;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint64_t ad = tc::smem_desc_sw128(qa + (c >> 2) * kQHalf + (c & 3) * 32, 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(kb + (c >> 2) * kHalfTile + (c & 3) * 32, 16, 1024);
        tc::mma_ss(d, ad, bd, idS, c > 0 ? 1u : 0u);
      }
      tc::mma_commit(&bar->s_full[gs & 1]);
      tc::mma_commit(&bar->k_empty[gs % kStages]);
      if (ts == ss.steps - 1) tc::mma_commit(&bar->q_empty[ks & 1]);
      ++gs;
      if (++ts == ss.steps) {
        ts = 0;
        ++ks;
        ++kks;
        ss = seek<kSplit>(kks, p, bar->lens);
      }
      progressed = true;
    }
    if (sp.slice < p.total && gp < gs && mbar_test(&bar->p_full[gp & 1], (gp >> 1) & 1) &&
        mbar_test(&bar->v_full[gp % kStages], (gp / kStages) & 1) &&
        (tp != 0 || kp < 2 || mbar_test(&bar->o_free[kp & 1], ((kp >> 1) - 1) & 1))) {
      tc::fence_after_sync();
      const uint32_t vb = sbase + kOffV + (gp % kStages) * kTile;
      const uint32_t o = tmem + col_o(kp & 1);
      const uint32_t pa = tmem + col_p(gp & 1);
      const int chunks = (step_keys(sp, tp) + 15) >> 4;
      // Lanes holding the high part of P and lanes holding the remainder
      // accumulate into their own rows of O; 16 keys per product.
      for (int c = 0; c < chunks; ++c) {
        const uint64_t bd = tc::smem_desc_sw128(vb + c * 16 * 128, kHalfTile, 1024);
        tc::mma_ts(o, pa + c * 8, bd, idO, (tp > 0 || c > 0) ? 1u : 0u);
      }
      tc::mma_commit(&bar->v_empty[gp % kStages]);
      tc::mma_commit(&bar->pv_done[gp & 1]);
      if (tp == sp.steps - 1) tc::mma_commit(&bar->o_full[kp & 1]);
      ++gp;
      if (++tp == sp.steps) {
        tp = 0;
        ++kp;
        ++kkp;
        sp = seek<kSplit>(kkp, p, bar->lens);
      }
      progressed = true;
    }
    if (progressed) {
      last = clock64();
    } else {
      if (clock64() - last > kSpinLimitCycles) {
        set_device_status(p.status, MEDUSA_ERR_TIMEOUT, kDetailAttnStageWait);
        bar->abort = 1;
        break;
      }
      __nanosleep(20);
    }
  }
}

// Bits o .. o + 63 (o >= 0) of a row of the ancestor mask held in four
// words; zero past the last word.
__device__ __forceinline__ uint64_t anc_window(const uint64_t (&a)[4], int o) {
  if (o >= 256) return 0ull;
  const int wi = o >> 6, sh = o & 63;
  const uint64_t w0 = wi == 0 ? a[0] : wi == 1 ? a[1] : wi == 2 ? a[2] : a[3];
  const uint64_t w1 = wi == 0 ? a[1] : wi == 1 ? a[2] : wi == 2 ? a[3] : 0ull;
  return sh == 0 ? w0 : (w0 >> sh) | (w1 << (64 - sh));
}

// ---- softmax (warps 4-7) ------------------------------------------------------
// Online softmax in the log2 domain with a lazy reference: the running
// maximum moves (and O is rescaled) only when a step's maximum exceeds it by
// more than 2^8, so P stays below 2^8 and O is rarely touched.
template <bool kSplit>
__device__ void run_softmax(const Params& p, unsigned char* smem, uint32_t tmem, Bars* bar, int warp, int lane) {
  const int q = warp & 3, h = lane >> 4, i = lane & 15;
  const uint32_t la = static_cast<uint32_t>(32 * q) << 16;
  int g = 0, k = 0;
  for (int kk = 0;; ++kk) {
    const Slice s = slice_info<kSplit>(kk, p, bar->lens);
    if (s.slice >= p.total) break;
    if (s.steps == 0) {
      if (lane == 0 && q == 0) set_device_status(p.status, MEDUSA_ERR_DEVICE_CHECK, kDetailAttnSeqLen);
      continue;
    }
    // This thread's tree token (query row) in the item's row group and its
    // ancestor mask (up to four words; loaded now, first used at the item's
    // last steps).
    const int r = p.row_lo + kRows * s.grp + 16 * q + i;
    uint64_t anc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int wd = 0; wd < 4; ++wd)
      if (r < p.row_hi && wd < p.t.W) anc[wd] = p.t.anc[r * p.t.W + wd];
    float mref = -INFINITY, lsum = 0.f;
    for (int t = 0; t < s.steps; ++t, ++g) {
      if (!wait_bar(&bar->s_full[g & 1], (g >> 1) & 1, bar, p.status)) return;
      tc::fence_after_sync();
      float sv[64];                                  // keys 64h .. 64h + 63 of the step
      const uint32_t sa = tmem + la + (g & 1) * kLaneHalf + kColS;
      tc::tmem_ld32x2<64>(sa, sv);
      tc::tmem_ld32x2<64>(sa + 32, sv + 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar->s_free[g & 1]);

      const int key0 = s.k0 + t * kStep + h * 64;      // key row of sv[0]
      // Eight independent partial maxima (the maximum does not depend on the
      // order; the short chains keep the one warp per scheduler busy).
      float mx[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mx[j] = -INFINITY;
      if (key0 + 64 > s.plim) {
        // Allowed keys of these 64 as a bit mask: the visible prefix, then
        // (last window only) the tree tokens that are ancestors of (or equal
        // to) row r.
        const int d = s.plim - key0;                 // visible prefix keys among them (< 64)
        uint64_t m = d > 0 ? (1ull << d) - 1ull : 0ull;
        if (s.last) m |= d >= 0 ? (anc[0] << d) : anc_window(anc, -d);
        const uint32_t mlo = static_cast<uint32_t>(m), mhi = static_cast<uint32_t>(m >> 32);
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const uint32_t bit = c < 32 ? (mlo >> c) & 1u : (mhi >> (c - 32)) & 1u;
          sv[c] = bit ? sv[c] : -INFINITY;
          mx[c & 7] = fmaxf(mx[c & 7], sv[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx[c & 7] = fmaxf(mx[c & 7], sv[c]);
      }
      float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16)) * p.scale_log2;   // both halves of the row
      float factor = 1.f;
      if (tmax > mref + kRescaleLog2 || (mref == -INFINITY && tmax > -INFINITY)) {
        factor = (mref == -INFINITY) ? 0.f : tc::ex2_ftz(mref - tmax);
        mref = tmax;
      }
      const float nmu = (mref == -INFINITY) ? 0.f : -mref;
      // p = 2^(s * scale * log2(e) - m): the scaling as packed fmas, four
      // packed partial sums of p.
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(nmu, nmu), one2 = f2_pack(1.f, 1.f);
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(sv[c], sv[c + 1]), sc2, nm2), x0, x1);
        sv[c] = tc::ex2_ftz(x0);
        sv[c + 1] = tc::ex2_ftz(x1);
        acc2[(c >> 1) & 3] = f2_fma(f2_pack(sv[c], sv[c + 1]), one2, acc2[(c >> 1) & 3]);
      }
      float ps = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float a, b;
        f2_unpack(acc2[j], a, b);
        ps += a + b;
      }
      lsum = lsum * factor + ps;

      // O is rescaled only after every P V issued into it is done (rare).
      const uint32_t ocol = col_o(k & 1);
      if (t > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
        if (!wait_bar(&bar->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, bar, p.status)) return;
        tc::fence_after_sync();
#pragma unroll 1
        for (int c0 = 0; c0 < kHd; c0 += 32) {       // thread l: lane 32q + l, query 16q + (l & 15)
          float o[32];
          tc::tmem_ld32(tmem + la + ocol + c0, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= factor;
          tc::tmem_st32(tmem + la + ocol + c0, o);
        }
      }
      // P buffer g & 1 is rewritten once the P V of step g - 2 has read it.
      if (g >= 2) {
        if (!wait_bar(&bar->pv_done[g & 1], ((g - 2) >> 1) & 1, bar, p.status)) return;
        tc::fence_after_sync();
      }
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float a0 = sv[2 * c], a1 = sv[2 * c + 1];
        hi[c] = pack2(a0, a1);
        lo[c] = pack2(a0 - bf16lo(hi[c]), a1 - bf16hi(hi[c]));
      }
      const uint32_t pa = tmem + la + col_p(g & 1);
      tc::tmem_st32x2<32>(pa, hi);                   // lanes 32q + i: high parts, keys 0-63 | 64-127
      tc::tmem_st32x2<32>(pa + kLaneHalf, lo);       // lanes 32q + 16 + i: remainders
      tc::tmem_wait_st();
      if (t == s.steps - 1) {
        const int first = step_keys(s, t);
        if (first & 15) {
          // V rows between the slice's last key and the end of its 16-key
          // chunk: zero them so 0 * (stale value) stays 0.
          if (!wait_bar(&bar->v_full[g % kStages], (g / kStages) & 1, bar, p.status)) return;
          unsigned char* vd = smem + kOffV + (g % kStages) * kTile;
          const int z = ((first + 15) & ~15) - first;
          for (int x = (warp - 4) * 32 + lane; x < z * 8; x += 128) {
            const int rr = first + x / 8, cc = x % 8;   // 8 chunks of 16 B per 128-byte row
            *reinterpret_cast<uint4*>(vd + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(vd + kHalfTile + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
          }
          tc::fence_proxy_async_smem();
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar->p_full[g & 1]);

      if (t == s.steps - 1) {
        // Hand the row sum to the epilogue warps once they are done with the
        // slice two back (same buffer).
        if (k >= 2 && !wait_bar(&bar->o_free[k & 1], ((k >> 1) - 1) & 1, bar, p.status)) return;
        const float total = lsum + __shfl_xor_sync(0xffffffffu, lsum, 16);
        if (h == 0) bar->lsum[k & 1][16 * q + i] = total;
        // ln sum exp(scale q.k) = ln 2 (m + log2 total), m the log2-domain reference.
        if (kSplit && p.lse != nullptr && h == 0 && r < p.row_hi)
          p.lse[(static_cast<size_t>(s.lb) * p.t.T + r) * p.H + s.e] = (mref + log2f(total)) * kLn2;
        tc::mbar_arrive(&bar->l_ready[k & 1]);
      }
    }
    ++k;
  }
}

// ---- epilogue (warps 2, 3, 8, 9) ------------------------------------------------
// out[query] = (O(high-part lanes) + O(remainder lanes)) / row sum, in fp32
// (or rounded to bf16 into out_bf16).
template <bool kSplit>
__device__ void run_epilogue(const Params& p, uint32_t tmem, Bars* bar, int warp, int lane) {
  const int q = warp & 3, h = lane >> 4, i = lane & 15;
  const int T = p.t.T;
  const uint32_t la = static_cast<uint32_t>(32 * q) << 16;
  int k = 0;
  for (int kk = 0;; ++kk) {
    const Slice s = seek<kSplit>(kk, p, bar->lens);
    if (s.slice >= p.total) break;
    if (!wait_bar(&bar->l_ready[k & 1], (k >> 1) & 1, bar, p.status)) return;
    if (!wait_bar(&bar->o_full[k & 1], (k >> 1) & 1, bar, p.status)) return;
    tc::fence_after_sync();
    const int r = p.row_lo + kRows * s.grp + 16 * q + i;   // tree token
    const float inv = 1.f / bar->lsum[k & 1][16 * q + i];
    const uint32_t oa = tmem + la + col_o(k & 1);
    const size_t ooff = ((static_cast<size_t>(s.lb) * T + r) * p.H + s.e) * kHd + 64 * h;
#pragma unroll 1
    for (int cp = 0; cp < 2; ++cp) {
      float a[32], b[32];                        // columns 64h + 32cp + (0..31)
      tc::tmem_ld32x2<64>(oa + 32 * cp, a);
      tc::tmem_ld32x2<64>(oa + kLaneHalf + 32 * cp, b);
      tc::tmem_wait_ld();
      if (r < p.row_hi && p.out_bf16) {
        uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + ooff + 32 * cp);
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            w[u] = static_cast<uint32_t>(f32_to_bf16_rne((a[c + 2 * u] + b[c + 2 * u]) * inv)) |
                   (static_cast<uint32_t>(f32_to_bf16_rne((a[c + 2 * u + 1] + b[c + 2 * u + 1]) * inv)) << 16);
          dst[c / 8] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else if (r < p.row_hi) {
        float* dst = p.out + ooff + 32 * cp;
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(dst + c) = make_float4((a[c] + b[c]) * inv, (a[c + 1] + b[c + 1]) * inv,
                                                            (a[c + 2] + b[c + 2]) * inv, (a[c + 3] + b[c + 3]) * inv);
      }
    }
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&bar->o_free[k & 1]);
    ++k;
  }
}

template <bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc64(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                   const __grid_constant__ CUtensorMap v_map, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->q_full[b], 1);
      mbar_init(&bar->q_empty[b], 1);
      mbar_init(&bar->s_full[b], 1);
      mbar_init(&bar->s_free[b], 4);
      mbar_init(&bar->p_full[b], 4);
      mbar_init(&bar->pv_done[b], 1);
      mbar_init(&bar->o_full[b], 1);
      mbar_init(&bar->o_free[b], 4);
      mbar_init(&bar->l_ready[b], 128);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    bar->abort = 0;
    fence_barrier_init();
  }
  for (int k = tid; k < kLenTab; k += blockDim.x) {
    const int item = blockIdx.x + k * gridDim.x;
    bar->lens[k] = item < p.total ? p.seq_lens[(item / p.groups / p.H) % p.B] : 0;
  }
  if (warp == 1) {
    tc::tmem_alloc(&bar->tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bar->tmem_base;
  allow_dependents();

  if (warp == 0) {
    if (lane == 0) run_producer<kSplit>(&q_map, &k_map, &v_map, p, smem, bar);
  } else if (warp == 1) {
    if (lane == 0) run_mma<kSplit>(p, smem_u32(smem), tmem, bar);
  } else if (warp >= 4 && warp < 8) {
    run_softmax<kSplit>(p, smem, tmem, bar, warp, lane);
  } else {
    run_epilogue<kSplit>(p, tmem, bar, warp, lane);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  // Launched inside medusa_step without waiting for the heads kernel (it reads
  // none of its outputs); completing only after it keeps the stream's order
  // for the kernels that follow.
  wait_prior_grids();
}

}  // namespace

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
void* tensor_map_encoder() {
  static void* fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = ptr;
  }
  return fn;
}

// Tensor maps: Q as [layers*B][T][H][128] (box 64 dims x 64 rows starting at
// row 64 x group, rows past T read as zero), K and V as [slices][Lcap][128].  For K/V a 4-D view
// {64 dims, rows, 2 halves, slices} loads a whole 128-key tile (both 64-dim
// halves, 32 KB) with one TMA instruction; if the driver rejects that view
// the kernel falls back to two 16 KB boxes per tile.
medusa_status_t launch_attention_tc64(const TreeDev& t, int layers, int B, int H, const void* q,
                                      const void* k_cache, const void* v_cache, int Lcap, const int32_t* seq_lens,
                                      float scale_log2, float* out, int* status, cudaStream_t stream, bool pdl,
                                      int row_lo, int row_hi, int split_r, int split_G, float* lse,
                                      const AttnOut& dec) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: cuTensorMapEncodeTiled unavailable");
  if (t.T > 4 * kRows || t.W > 4) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: more than 256 tree tokens");
  const long long slices = static_cast<long long>(layers) * B * H;
  if (row_lo < 0 || row_hi > t.T || row_lo >= row_hi)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree attention: empty row range");
  const int groups = (row_hi - row_lo + kRows - 1) / kRows;
  const long long items = slices * groups;
  if (items >= (1ll << 31)) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: too many slices");
  CUtensorMap qm, km, vm;
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHd), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(t.T), static_cast<cuuint64_t>(layers) * B};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHd) * 2, static_cast<cuuint64_t>(H) * kHd * 2,
                                   static_cast<cuuint64_t>(t.T) * H * kHd * 2};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kRows), 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    if (enc(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: q tensor map rejected");
  }
  int one_box = 1;
  for (int which = 0; which < 2; ++which) {
    void* base = const_cast<void*>(which == 0 ? k_cache : v_cache);
    CUtensorMap* m = which == 0 ? &km : &vm;
    bool done = false;
    if (one_box) {
      const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(Lcap), 2, static_cast<cuuint64_t>(slices)};
      const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHd) * 2, 128, static_cast<cuuint64_t>(Lcap) * kHd * 2};
      const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kStep), 2, 1};
      const cuuint32_t es[4] = {1, 1, 1, 1};
      done = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
      if (!done && which == 1) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: V tensor map rejected");
      if (!done) one_box = 0;
    }
    if (!done) {
      const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHd), static_cast<cuuint64_t>(Lcap),
                                  static_cast<cuuint64_t>(slices)};
      const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHd) * 2, static_cast<cuuint64_t>(Lcap) * kHd * 2};
      const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kStep), 1};
      const cuuint32_t es[3] = {1, 1, 1};
      if (enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: K/V tensor map rejected");
    }
  }
  Params prm{};
  prm.t = t;
  prm.B = B;
  prm.H = H;
  prm.Lcap = Lcap;
  prm.total = static_cast<int>(items);
  prm.groups = groups;
  prm.row_lo = row_lo;
  prm.row_hi = row_hi;
  prm.seq_lens = seq_lens;
  prm.scale_log2 = scale_log2;
  prm.out = out;
  prm.out_bf16 = dec.bf16;
  prm.wait_first = dec.wait_first ? 1 : 0;
  prm.status = status;
  prm.kv_one_box = one_box;
  prm.split_r = split_r;
  prm.split_G = split_G;
  prm.lse = lse;
  const int grid = static_cast<int>(items < sm_count() ? items : sm_count());
  // The split instantiation (window bookkeeping, lse store) only when asked
  // for: the whole-prefix kernel keeps the plain bookkeeping.
  const bool split = split_G > 1 || lse != nullptr;
  auto kernel = split ? tree_attn_tc64<true> : tree_attn_tc64<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) e = launch_kernel(kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, pdl, qm, km, vm, prm);
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_attention: tcgen05 launch", e);
}

}  // namespace medusa
