// S5 for trees of 65-256 tokens (bf16, hd = 128): a persistent tcgen05
// kernel whose work item is one (layer, sequence, head) slice and one group
// of 128 tree tokens, so a tree of up to 128 tokens streams each slice's K/V
// once.
//
// The mask is that of "Medusa — 让大模型自己同时猜好几个 token" (核心要点:
// the candidate tree is verified in one forward under a tree mask; 实践案例
// case 3: a node sees the cached prefix, its ancestors and itself).
//
// Layout of the work.  One CTA per SM walks the items w = cta, cta + grid, ...
// (item w: slice w / groups, row group w % groups), each cut into steps of
// 128 keys.  K and V tiles (32 KB, two 64-dim halves in 128-byte swizzle)
// arrive by TMA (no multicast) into two three-stage rings; an item's 128
// query rows come through the K ring as one 32 KB entry ahead of its K tiles
// and are copied into tensor memory (tcgen05.cp).
//
// Tensor memory (512 columns, M = 128 products: row R of a product in lane R):
//   S     cols [0, 128)    Q K^T of the step, Q read from tensor memory
//   P_hi  cols [128, 192)  bf16 high parts of P (two keys per column)
//   P_lo  cols [192, 256)  bf16 remainders, so P V keeps ~16 bits of P
//   O     cols [256, 384)  O += P_hi V + P_lo V
//   Q     cols [384, 448) and [448, 512), one per item parity
// Softmax: row R is owned by two threads, lane R & 31 of warp 4 + R / 32
// (keys 0-63 of each step) and of warp 8 + R / 32 (keys 64-127); they trade
// their half-row maxima through shared memory once per step so that both
// halves of P share one reference, and at the item's end the same two
// threads normalise and store their 64 columns of O.
//
// Warp roles: warp 0 TMA producer; warp 1 TMEM allocation and the single MMA
// issuer; warps 4-11 softmax and epilogue.  Every wait is bounded.
#include <cfloat>
#include <cudaTypedefs.h>

#include "tcgen05.cuh"

namespace medusa {
namespace {

constexpr int kHd = 128;
constexpr int kStep = 128;                     // keys per step
constexpr int kRows = 128;                     // query rows (tree tokens) per item
constexpr int kStagesK = 3;                    // K ring (K tiles and Q entries)
constexpr int kStagesV = 3;                    // V ring
constexpr int kHalfTile = kStep * 128;         // 128 rows x 64 dims x 2 B = 16 KB
constexpr int kTile = 2 * kHalfTile;           // one K, V or Q entry: 32 KB
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColPhi = 128;
constexpr uint32_t kColPlo = 192;
constexpr uint32_t kColO = 256;
__device__ __forceinline__ uint32_t col_q(int buf) { return 384u + 64u * buf; }
constexpr float kRescaleLog2 = 8.0f;
constexpr int kLenTab = 256;                   // prefix lengths of a CTA's first items, in shared memory
// The polling loops of the producer and the MMA issuer give up after this
// many SM cycles without progress (about 2 s at 2 GHz); the SM cycle counter
// is read on every pass, the global timer is too slow for that.
constexpr long long kSpinLimitCycles = 4000000000LL;

struct Bars {
  uint64_t k_full[kStagesK], k_empty[kStagesK], v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full, s_free, p_full, pv_done, o_full, o_read;
  uint64_t xstep[4][2];              // per lane quarter, by step parity: half-row maxima exchanged
  uint64_t xend[4];                  // per lane quarter: half-row sums exchanged at an item's end
  uint32_t tmem_base;
  int abort;
  float xmax[2][2][kRows];           // [step parity][half][row]
  float xsum[2][kRows];              // [half][row]
  int lens[kLenTab];                 // lens[k]: prefix length of this CTA's item k
};

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kStagesK * kTile;
constexpr int kOffBars = kOffV + kStagesV * kTile;
constexpr int kBarsBytes = 5120;
constexpr int kSmemBytes = kOffBars + kBarsBytes + 1024;
static_assert(sizeof(Bars) <= kBarsBytes, "barrier block too large");
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Slice {
  int slice, lb, e, L, n, steps;
  int item, grp;   // work item index; query rows 128 grp .. 128 grp + 127
};

struct Params {
  TreeDev t;
  int B, H, Lcap, total;   // total: work items = slices x groups
  int groups;              // ceil(T / 128)
  int row_lo, row_hi;      // tree tokens (query rows) handled by this launch
  const int32_t* seq_lens;
  float scale_log2;
  float* out;
  uint16_t* out_bf16;      // if set, the output goes here as bf16 instead of `out`
  int wait_first;          // wait for the preceding kernel before the first load
  int* status;
  int kv_one_box;   // 1: one 32 KB TMA box per tile (4-D map), 0: two 16 KB boxes
};

// Work item kk of this CTA; steps = 0 when it fails its check; slice =
// total marks the end.
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
  s.n = s.L + p.t.T;
  s.steps = (s.L >= 0 && s.n <= p.Lcap) ? (s.n + kStep - 1) / kStep : 0;
  return s;
}

__device__ __forceinline__ Slice seek(int& kk, const Params& p, const int* lens) {
  Slice s = slice_info(kk, p, lens);
  while (s.slice < p.total && s.steps == 0) s = slice_info(++kk, p, lens);
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

// Keys of step t that belong to the slice (1..128).
__device__ __forceinline__ int step_keys(const Slice& s, int t) {
  const int first = s.n - t * kStep;
  return first < kStep ? first : kStep;
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

__device__ __forceinline__ void tmem_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// ---- TMA producer (one thread) ----------------------------------------------
// The K ring carries, per item, one Q entry (128 query rows) and then the
// item's K tiles; the V ring the V tiles of every step.  Each stream issues
// as soon as its ring has a free stage.
__device__ void run_producer(const CUtensorMap* q_map, const CUtensorMap* k_map, const CUtensorMap* v_map,
                             const Params& p, unsigned char* smem, Bars* bar) {
  tc::prefetch_tensormap(q_map);
  tc::prefetch_tensormap(k_map);
  tc::prefetch_tensormap(v_map);
  if (p.wait_first) wait_prior_grids();   // q and the tree's K/V rows come from it
  int kkk = 0, kkv = 0;
  Slice sk = seek(kkk, p, bar->lens), sv = seek(kkv, p, bar->lens);
  int ek = 0, gv = 0;     // K-ring entries and V tiles issued
  int tk = -1, tv = 0;    // step of the next K-ring entry (-1: the item's Q entry); of the next V tile
  long long last = clock64();
  while ((sk.slice < p.total || sv.slice < p.total) && !bar->abort) {
    bool progressed = false;
    if (sk.slice < p.total) {
      const int st = ek % kStagesK;
      if (ek < kStagesK || mbar_test(&bar->k_empty[st], ((ek / kStagesK) - 1) & 1)) {
        unsigned char* d = smem + kOffK + st * kTile;
        uint64_t* fb = &bar->k_full[st];
        mbar_arrive_expect_tx(fb, kTile);
        if (tk < 0) {
          tc::tma_load_4d(d, q_map, 0, sk.e, p.row_lo + kRows * sk.grp, sk.lb, fb);
          tc::tma_load_4d(d + kHalfTile, q_map, 64, sk.e, p.row_lo + kRows * sk.grp, sk.lb, fb);
        } else if (p.kv_one_box) {
          tc::tma_load_4d(d, k_map, 0, tk * kStep, 0, sk.slice, fb);
        } else {
          tc::tma_load_3d(d, k_map, 0, tk * kStep, sk.slice, fb);
          tc::tma_load_3d(d + kHalfTile, k_map, 64, tk * kStep, sk.slice, fb);
        }
        ++ek;
        if (++tk == sk.steps) {
          tk = -1;
          ++kkk;
          sk = seek(kkk, p, bar->lens);
        }
        progressed = true;
      }
    }
    if (sv.slice < p.total) {
      const int st = gv % kStagesV;
      if (gv < kStagesV || mbar_test(&bar->v_empty[st], ((gv / kStagesV) - 1) & 1)) {
        unsigned char* d = smem + kOffV + st * kTile;
        uint64_t* fb = &bar->v_full[st];
        mbar_arrive_expect_tx(fb, kTile);
        if (p.kv_one_box) {
          tc::tma_load_4d(d, v_map, 0, tv * kStep, 0, sv.slice, fb);
        } else {
          tc::tma_load_3d(d, v_map, 0, tv * kStep, sv.slice, fb);
          tc::tma_load_3d(d + kHalfTile, v_map, 64, tv * kStep, sv.slice, fb);
        }
        ++gv;
        if (++tv == sv.steps) {
          tv = 0;
          ++kkv;
          sv = seek(kkv, p, bar->lens);
        }
        progressed = true;
      }
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
  // Every copy issued lands before the CTA exits (bounded).
  for (int st = 0; st < kStagesK; ++st)
    if (ek > st) mbar_wait(&bar->k_full[st], ((st + ((ek - 1 - st) / kStagesK) * kStagesK) / kStagesK) & 1);
  for (int st = 0; st < kStagesV; ++st)
    if (gv > st) mbar_wait(&bar->v_full[st], ((st + ((gv - 1 - st) / kStagesV) * kStagesV) / kStagesV) & 1);
}

// ---- MMA issuer (one thread) ------------------------------------------------
// A Q entry is copied into the item's Q buffer (its previous user, S of the
// item two back, completed before S of the previous item could start: S has
// one buffer).  S(g) = Q K^T: eight M = 128, N = 128, K = 16 products with Q
// from tensor memory.  O += P_hi V + P_lo V: two products per 16 valid keys.
// S(g) waits for K(g) and for the softmax to have read S(g - 1), not for
// P V(g - 1), so it runs while the softmax of step g - 1 still computes.
__device__ void run_mma(const Params& p, uint32_t sbase, uint32_t tmem, Bars* bar) {
  constexpr uint32_t idS = tc::idesc_bf16_f32(128, kStep, 0);
  constexpr uint32_t idO = tc::idesc_bf16_f32(128, kHd, 1);
  int kks = 0, kkp = 0;
  Slice ss = seek(kks, p, bar->lens), sp = seek(kkp, p, bar->lens);
  int ek = 0;
  int gs = 0, ts = -1, ks = 0;     // S cursor (ts = -1: Q entry next)
  int gp = 0, tp = 0, kp = 0;      // P V cursor
  long long last = clock64();
  while ((ss.slice < p.total || sp.slice < p.total) && !bar->abort) {
    bool progressed = false;
    const int st = ek % kStagesK;
    if (ss.slice < p.total && mbar_test(&bar->k_full[st], (ek / kStagesK) & 1)) {
      const uint32_t kb = sbase + kOffK + st * kTile;
      if (ts < 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          tmem_cp_128x256b(tmem + col_q(ks & 1) + c * 8,
                           tc::smem_desc_sw128(kb + (c >> 2) * kHalfTile + (c & 3) * 32, 16, 1024));
        tc::mma_commit(&bar->k_empty[st]);
        ++ek;
        ts = 0;
        progressed = true;
      } else if (gs == 0 || mbar_test(&bar->s_free, (gs - 1) & 1)) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint64_t bd = tc::smem_desc_sw128(kb + (c >> 2) * kHalfTile + (c & 3) * 32, 16, 1024);
          tc::mma_ts(tmem + kColS, tmem + col_q(ks & 1) + c * 8, bd, idS, c > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bar->s_full);
        tc::mma_commit(&bar->k_empty[st]);
        ++ek;
        ++gs;
        if (++ts == ss.steps) {
          ts = -1;
          ++ks;
          ++kks;
          ss = seek(kks, p, bar->lens);
        }
        progressed = true;
      }
    }
    if (sp.slice < p.total && gp < gs && mbar_test(&bar->p_full, gp & 1) &&
        mbar_test(&bar->v_full[gp % kStagesV], (gp / kStagesV) & 1) &&
        (tp != 0 || kp == 0 || mbar_test(&bar->o_read, (kp - 1) & 1))) {
      tc::fence_after_sync();
      const uint32_t vb = sbase + kOffV + (gp % kStagesV) * kTile;
      const int chunks = (step_keys(sp, tp) + 15) >> 4;
      for (int c = 0; c < chunks; ++c) {
        const uint64_t bd = tc::smem_desc_sw128(vb + c * 16 * 128, kHalfTile, 1024);
        tc::mma_ts(tmem + kColO, tmem + kColPhi + c * 8, bd, idO, (tp > 0 || c > 0) ? 1u : 0u);
      }
      for (int c = 0; c < chunks; ++c) {
        const uint64_t bd = tc::smem_desc_sw128(vb + c * 16 * 128, kHalfTile, 1024);
        tc::mma_ts(tmem + kColO, tmem + kColPlo + c * 8, bd, idO, 1u);
      }
      tc::mma_commit(&bar->v_empty[gp % kStagesV]);
      tc::mma_commit(&bar->pv_done);
      if (tp == sp.steps - 1) tc::mma_commit(&bar->o_full);
      ++gp;
      if (++tp == sp.steps) {
        tp = 0;
        ++kp;
        ++kkp;
        sp = seek(kkp, p, bar->lens);
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

// ---- softmax and epilogue (warps 4-11) ---------------------------------------
// Online softmax in the log2 domain with a lazy reference (moved, and O
// rescaled, only when a step's row maximum exceeds it by more than 2^8).
__device__ void run_softmax(const Params& p, unsigned char* smem, uint32_t tmem, Bars* bar, int warp, int lane) {
  const int q = warp & 3;                 // TMEM lane quarter
  const int hf = (warp - 4) >> 2;         // key half of every step: 0 (keys 0-63) or 1 (keys 64-127)
  const int R = 32 * q + lane;            // row of the products
  const int T = p.t.T;
  const uint32_t la = static_cast<uint32_t>(32 * q) << 16;
  int g = 0, k = 0;
  for (int kk = 0;; ++kk) {
    const Slice s = slice_info(kk, p, bar->lens);
    if (s.slice >= p.total) break;
    if (s.steps == 0) {
      if (lane == 0 && warp == 4) set_device_status(p.status, MEDUSA_ERR_DEVICE_CHECK, kDetailAttnSeqLen);
      continue;
    }
    const int r = p.row_lo + kRows * s.grp + R;   // tree token of this row
    uint64_t anc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int wd = 0; wd < 4; ++wd)
      if (r < p.row_hi && wd < p.t.W) anc[wd] = p.t.anc[r * p.t.W + wd];
    float mref = -INFINITY, lsum = 0.f;   // lsum: this half's keys
    for (int t = 0; t < s.steps; ++t, ++g) {
      if (!wait_bar(&bar->s_full, g & 1, bar, p.status)) return;
      tc::fence_after_sync();
      float sv[64];                        // keys 64 hf .. 64 hf + 63 of the step
      tc::tmem_ld32(tmem + la + kColS + 64 * hf, sv);
      tc::tmem_ld32(tmem + la + kColS + 64 * hf + 32, sv + 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar->s_free);

      const int key0 = t * kStep + hf * 64;
      float hm = -INFINITY;
      if (key0 + 64 > s.L) {
        // Allowed keys of this window: the cached prefix, then the tree
        // tokens that are ancestors of (or equal to) row r.
        const int d = s.L - key0;
        uint64_t m = d > 0 ? (1ull << d) - 1ull : 0ull;
        m |= d >= 0 ? (anc[0] << d) : anc_window(anc, -d);
        const uint32_t mlo = static_cast<uint32_t>(m), mhi = static_cast<uint32_t>(m >> 32);
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const uint32_t bit = c < 32 ? (mlo >> c) & 1u : (mhi >> (c - 32)) & 1u;
          sv[c] = bit ? sv[c] : -INFINITY;
          hm = fmaxf(hm, sv[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) hm = fmaxf(hm, sv[c]);
      }
      // Trade half-row maxima with the other half's thread (same lane of
      // warp 4 + q / 8 + q), so both halves of P share one reference.
      bar->xmax[g & 1][hf][R] = hm;
      tc::mbar_arrive(&bar->xstep[q][g & 1]);
      if (!wait_bar(&bar->xstep[q][g & 1], (g >> 1) & 1, bar, p.status)) return;
      const float tmax = fmaxf(hm, bar->xmax[g & 1][hf ^ 1][R]) * p.scale_log2;
      float factor = 1.f;
      if (tmax > mref + kRescaleLog2 || (mref == -INFINITY && tmax > -INFINITY)) {
        factor = (mref == -INFINITY) ? 0.f : tc::ex2_ftz(mref - tmax);
        mref = tmax;
      }
      const float nmu = (mref == -INFINITY) ? 0.f : -mref;
      float ps = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        sv[c] = tc::ex2_ftz(fmaf(sv[c], p.scale_log2, nmu));
        ps += sv[c];
      }
      lsum = lsum * factor + ps;

      // P (one buffer) is rewritten, and O rescaled, once P V of step g - 1
      // is done; each half rescales its own 64 columns of O.
      const bool rescale = t > 0 && __any_sync(0xffffffffu, factor != 1.f);
      if (g >= 1) {
        if (!wait_bar(&bar->pv_done, (g - 1) & 1, bar, p.status)) return;
        tc::fence_after_sync();
      }
      if (rescale) {
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float o[32];
          tc::tmem_ld32(tmem + la + kColO + 64 * hf + c0, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= factor;
          tc::tmem_st32(tmem + la + kColO + 64 * hf + c0, o);
        }
      }
      float hi[32], lo[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float a0 = sv[2 * c], a1 = sv[2 * c + 1];
        const uint32_t ph = pack2(a0, a1);
        hi[c] = __uint_as_float(ph);
        lo[c] = __uint_as_float(pack2(a0 - bf16lo(ph), a1 - bf16hi(ph)));
      }
      tc::tmem_st32(tmem + la + kColPhi + 32 * hf, hi);
      tc::tmem_st32(tmem + la + kColPlo + 32 * hf, lo);
      tc::tmem_wait_st();
      if (t == s.steps - 1 && hf == 0) {
        const int first = step_keys(s, t);
        if (first & 15) {
          // V rows between the slice's last key and the end of its 16-key
          // chunk: zero them so 0 * (stale value) stays 0.
          if (!wait_bar(&bar->v_full[g % kStagesV], (g / kStagesV) & 1, bar, p.status)) return;
          unsigned char* vd = smem + kOffV + (g % kStagesV) * kTile;
          const int z = ((first + 15) & ~15) - first;
          for (int x = (warp - 4) * 32 + lane; x < z * 8; x += 128) {
            const int rr = first + x / 8, cc = x % 8;
            *reinterpret_cast<uint4*>(vd + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(vd + kHalfTile + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
          }
          tc::fence_proxy_async_smem();
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bar->p_full);

      if (t == s.steps - 1) {
        // Item end: the row's sum over both halves, then this half's 64
        // columns of O divided by it.  O goes back to the MMA issuer (the next
        // item's first P V overwrites it) before the stores.
        bar->xsum[hf][R] = lsum;
        tc::mbar_arrive(&bar->xend[q]);
        if (!wait_bar(&bar->xend[q], k & 1, bar, p.status)) return;
        const float inv = 1.f / (lsum + bar->xsum[hf ^ 1][R]);
        if (!wait_bar(&bar->o_full, k & 1, bar, p.status)) return;
        tc::fence_after_sync();
        float o[64];
        tc::tmem_ld32(tmem + la + kColO + 64 * hf, o);
        tc::tmem_ld32(tmem + la + kColO + 64 * hf + 32, o + 32);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bar->o_read);
        const size_t ooff = ((static_cast<size_t>(s.lb) * T + r) * p.H + s.e) * kHd + 64 * hf;
        if (r < p.row_hi && p.out_bf16) {
          uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + ooff);
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              w[u] = static_cast<uint32_t>(f32_to_bf16_rne(o[c + 2 * u] * inv)) |
                     (static_cast<uint32_t>(f32_to_bf16_rne(o[c + 2 * u + 1] * inv)) << 16);
            dst[c / 8] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else if (r < p.row_hi) {
          float* dst = p.out + ooff;
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
        }
      }
    }
    ++k;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc128(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                    const __grid_constant__ CUtensorMap v_map, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int st = 0; st < kStagesK; ++st) {
      mbar_init(&bar->k_full[st], 1);
      mbar_init(&bar->k_empty[st], 1);
    }
    for (int st = 0; st < kStagesV; ++st) {
      mbar_init(&bar->v_full[st], 1);
      mbar_init(&bar->v_empty[st], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 8);
    mbar_init(&bar->p_full, 8);
    mbar_init(&bar->pv_done, 1);
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->o_read, 8);
    for (int qq = 0; qq < 4; ++qq) {
      mbar_init(&bar->xstep[qq][0], 64);
      mbar_init(&bar->xstep[qq][1], 64);
      mbar_init(&bar->xend[qq], 64);
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
    if (lane == 0) run_producer(&q_map, &k_map, &v_map, p, smem, bar);
  } else if (warp == 1) {
    if (lane == 0) run_mma(p, smem_u32(smem), tmem, bar);
  } else if (warp >= 4) {
    run_softmax(p, smem, tmem, bar, warp, lane);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  wait_prior_grids();   // see tree_attn_tc64: complete only after the preceding kernel
}

}  // namespace

// Tensor maps as for tree_attn_tc64, with Q boxes of 64 dims x 128 rows.
medusa_status_t launch_attention_tc128(const TreeDev& t, int layers, int B, int H, const void* q,
                                       const void* k_cache, const void* v_cache, int Lcap, const int32_t* seq_lens,
                                       float scale_log2, float* out, int* status, cudaStream_t stream, bool pdl,
                                       int row_lo, int row_hi, const AttnOut& dec) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: cuTensorMapEncodeTiled unavailable");
  if (t.T > 2 * kRows || t.W > 4) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: more than 256 tree tokens");
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
  const int grid = static_cast<int>(items < sm_count() ? items : sm_count());
  cudaError_t e = cudaFuncSetAttribute(tree_attn_tc128, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) e = launch_kernel(tree_attn_tc128, dim3(grid), dim3(kThreads), kSmemBytes, stream, pdl, qm, km, vm, prm);
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_attention: tcgen05 launch (128-row groups)", e);
}

}  // namespace medusa
