// S5 for trees of up to 64 tokens (bf16, hd = 128): a persistent tcgen05
// kernel that streams every (layer, sequence, head) slice of K/V through
// shared memory exactly once and keeps the memory pipeline full across
// slice boundaries.
//
// The mask is that of "Medusa — 让大模型自己同时猜好几个 token" (核心要点:
// the candidate tree is verified in one forward under a tree mask; 实践案例
// case 3: a node sees the cached prefix, its ancestors and itself).
//
// Layout of the work.  One CTA per SM walks the slices s = cta, cta + G, ...
// Each slice is cut into steps of 128 keys.  A step's K and V tiles (64 KB)
// arrive by TMA into a three-stage ring (128-byte swizzle, no multicast).
// The queries of a slice (64 rows) live in one of two Q buffers so that the
// next slice's Q loads while the current one finishes.
//
// Tensor memory (512 columns, M = 64 accumulators use lanes 0-15 of each
// lane quarter; a second M = 64 accumulator can sit at lane offset 16):
//   S     cols [0, 64)    lanes 0-15: keys 0-63 of the step, lanes 16-31: keys 64-127
//   P     cols [64, 128) and [384, 448), alternating by step: the same lanes,
//                         P as bf16 pairs (high part, then remainder; two keys
//                         per column), so the softmax of step g+1 never waits
//                         for the P V of step g
//   O     cols [128, 256) and [256, 384), one per slice parity; lanes 0-15
//                         accumulate keys 0-63 of every step, lanes 16-31
//                         keys 64-127; the two are summed once per slice.
// So every lane of every softmax warp holds one (row, half-step) and the two
// halves of a row meet in one shuffle (row maximum, running sum, final O).
//
// Warp roles: warp 0 TMA producer; warp 1 TMEM allocation and the single MMA
// issuer (S of step g+1 goes out as soon as the softmax has read S of step
// g); warps 4-7 softmax and epilogue.  Every wait is bounded.
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
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                                             // 128 fp32 columns
__device__ __forceinline__ uint32_t col_p(int buf) { return 128u + 64u * buf; }   // 64 packed columns
__device__ __forceinline__ uint32_t col_o(int buf) { return 256u + 128u * buf; }  // 128 fp32 columns
constexpr float kRescaleLog2 = 8.0f;

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;                                 // 128 rows (each query twice) x 256 B
constexpr int kOffKV = 128 * 256;                        // 3 stages x (K 32 KB + V 32 KB)
constexpr int kOffBars = kOffKV + kStages * 2 * kTile;
constexpr int kSmemBytes = kOffBars + 512 + 1024;

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, s_free, p_full, pv_done[2];   // pv_done[b]: the P V that read P buffer b
  uint64_t o_full[2], o_free[2];
  uint32_t tmem_base;
  int abort;
};

struct Slice {
  int slice, lb, e, L, n, steps;
};

// Slice k of this CTA; steps = 0 when it does not exist or fails its check.
__device__ __forceinline__ Slice slice_info(int k, int total, int B, int H, int T, int Lcap,
                                            const int32_t* seq_lens) {
  Slice s{};
  s.slice = blockIdx.x + k * gridDim.x;
  if (s.slice >= total) return s;
  s.e = s.slice % H;
  s.lb = s.slice / H;
  s.L = seq_lens[s.lb % B];
  s.n = s.L + T;
  s.steps = (s.L >= 0 && s.n <= Lcap) ? (s.n + kStep - 1) / kStep : 0;
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

struct Params {
  TreeDev t;
  int B, H, Lcap, total;
  const int32_t* seq_lens;
  float scale_log2;
  float* out;
  int* status;
  int kv_one_box;   // 1: one 32 KB TMA box per tile (4-D map), 0: two 16 KB boxes
};

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc64(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                   const __grid_constant__ CUtensorMap v_map, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  const int T = p.t.T;

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->o_full[i], 1);
      mbar_init(&bar->o_free[i], 4);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->kv_full[s], 1);
      mbar_init(&bar->kv_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 4);
    mbar_init(&bar->p_full, 4);
    mbar_init(&bar->pv_done[0], 1);
    mbar_init(&bar->pv_done[1], 1);
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

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    // Two streams, each issued as soon as its buffer is free: K/V tiles of
    // every step, and the Q rows of every slice (Q waits for the last S of
    // the previous slice; K/V of the next slice keep flowing meanwhile).
    tc::prefetch_tensormap(&q_map);
    tc::prefetch_tensormap(&k_map);
    tc::prefetch_tensormap(&v_map);
    int g = 0, kv_kk = 0, kv_t = 0;            // K/V cursor: global step, slice, step within slice
    int qk = 0, q_kk = 0;                      // Q cursor: slice count, slice index
    Slice kvs = slice_info(0, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
    while (kvs.slice < p.total && kvs.steps == 0) kvs = slice_info(++kv_kk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
    Slice qs = kvs;
    q_kk = kv_kk;
    const uint64_t t0 = globaltimer_ns();
    uint64_t last = t0;
    while ((kvs.slice < p.total || qs.slice < p.total) && !bar->abort) {
      bool progressed = false;
      if (qs.slice < p.total && (qk == 0 || mbar_test(&bar->q_empty, (qk - 1) & 1))) {
        // Q rows 32q + 16c + i (c = 0, 1) both hold query 16q + i: one M = 128
        // product then gives each lane pair the full 128-key row.
        unsigned char* qd = smem + kOffQ;
        mbar_arrive_expect_tx(&bar->q_full, 128 * 256);
        for (int qq = 0; qq < 4; ++qq)
          for (int c = 0; c < 2; ++c)
            for (int rg = 0; rg < 2; ++rg)
              tc::tma_load_4d(qd + rg * 128 * 128 + (32 * qq + 16 * c) * 128, &q_map, 64 * rg, qs.e, 16 * qq, qs.lb,
                              &bar->q_full);
        ++qk;
        do {
          qs = slice_info(++q_kk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
        } while (qs.slice < p.total && qs.steps == 0);
        progressed = true;
      }
      if (kvs.slice < p.total) {
        const int st = g % kStages;
        if (g < kStages || mbar_test(&bar->kv_empty[st], ((g / kStages) - 1) & 1)) {
          unsigned char* kd = smem + kOffKV + st * 2 * kTile;
          unsigned char* vd = kd + kTile;
          mbar_arrive_expect_tx(&bar->kv_full[st], 2 * kTile);
          if (p.kv_one_box) {
            tc::tma_load_4d(kd, &k_map, 0, kv_t * kStep, 0, kvs.slice, &bar->kv_full[st]);
            tc::tma_load_4d(vd, &v_map, 0, kv_t * kStep, 0, kvs.slice, &bar->kv_full[st]);
          } else {
            tc::tma_load_3d(kd, &k_map, 0, kv_t * kStep, kvs.slice, &bar->kv_full[st]);
            tc::tma_load_3d(kd + kHalfTile, &k_map, 64, kv_t * kStep, kvs.slice, &bar->kv_full[st]);
            tc::tma_load_3d(vd, &v_map, 0, kv_t * kStep, kvs.slice, &bar->kv_full[st]);
            tc::tma_load_3d(vd + kHalfTile, &v_map, 64, kv_t * kStep, kvs.slice, &bar->kv_full[st]);
          }
          ++g;
          if (++kv_t == kvs.steps) {
            kv_t = 0;
            do {
              kvs = slice_info(++kv_kk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
            } while (kvs.slice < p.total && kvs.steps == 0);
          }
          progressed = true;
        }
      }
      if (progressed) {
        last = globaltimer_ns();
      } else {
        if (globaltimer_ns() - last > kSpinLimitNs) {
          set_device_status(p.status, MEDUSA_ERR_TIMEOUT, kDetailAttnStageWait);
          bar->abort = 1;
          break;
        }
        __nanosleep(64);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idS = tc::idesc_bf16_f32(128, kStep, 0);
    constexpr uint32_t idO = tc::idesc_bf16_f32(128, kHd, 1);
    // S of global step g: one M = 128, N = 128 product per 16 dims (8 in all);
    // lane R gets all 128 keys of the query in Q row R.
    auto issue_s = [&](int g) {
      const uint32_t qa = sbase + kOffQ;
      const uint32_t kb = sbase + kOffKV + (g % kStages) * 2 * kTile;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint64_t ad = tc::smem_desc_sw128(qa + (c >> 2) * 128 * 128 + (c & 3) * 32, 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(kb + (c >> 2) * kHalfTile + (c & 3) * 32, 16, 1024);
        tc::mma_ss(tmem + kColS, ad, bd, idS, c > 0 ? 1u : 0u);
      }
      tc::mma_commit(&bar->s_full);
    };
    // Walk the same (slice, step) sequence as the producer, one step ahead for S.
    int k = 0, kk = 0, g = 0;
    Slice cur = slice_info(0, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
    while (cur.slice < p.total && cur.steps == 0) cur = slice_info(++kk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
    bool ok = cur.slice < p.total;
    if (ok) ok = wait_bar(&bar->q_full, 0, bar, p.status) && wait_bar(&bar->kv_full[0], 0, bar, p.status);
    if (ok) {
      tc::fence_after_sync();
      issue_s(0);
      if (cur.steps == 1) tc::mma_commit(&bar->q_empty);
    }
    while (ok) {
      for (int t = 0; ok && t < cur.steps; ++t, ++g) {
        // next step: same slice, or the first step of the next existing slice
        int nk = k, nt = t + 1;
        Slice nxt = cur;
        int nkk = kk;
        if (nt == cur.steps) {
          nt = 0;
          nk = k + 1;
          do {
            nxt = slice_info(++nkk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
          } while (nxt.slice < p.total && nxt.steps == 0);
        }
        // Issue S of the next step and P V of this step in whichever order
        // their inputs become ready (non-blocking tests, bounded overall).
        bool need_s = nxt.slice < p.total;
        bool need_pv = true;
        const uint64_t t0 = globaltimer_ns();
        while (need_s || need_pv) {
          bool progressed = false;
          if (need_s && (nt != 0 || mbar_test(&bar->q_full, nk & 1)) &&
              mbar_test(&bar->kv_full[(g + 1) % kStages], ((g + 1) / kStages) & 1) && mbar_test(&bar->s_free, g & 1)) {
            tc::fence_after_sync();
            issue_s(g + 1);
            if (nt == nxt.steps - 1) tc::mma_commit(&bar->q_empty);
            need_s = false;
            progressed = true;
          }
          if (need_pv && mbar_test(&bar->p_full, g & 1) &&
              (t != 0 || k < 2 || mbar_test(&bar->o_free[k & 1], ((k >> 1) - 1) & 1))) {
            tc::fence_after_sync();
            const uint32_t vb = sbase + kOffKV + (g % kStages) * 2 * kTile + kTile;
            // O (lanes with the high part of P) and O' (lanes with the
            // remainder) += P V over the step's 128 keys, 16 keys per product.
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint64_t bd = tc::smem_desc_sw128(vb + c * 16 * 128, kHalfTile, 1024);
              tc::mma_ts(tmem + col_o(k & 1), tmem + col_p(g & 1) + c * 8, bd, idO, (t > 0 || c > 0) ? 1u : 0u);
            }
            need_pv = false;
            progressed = true;
          }
          if (!progressed) {
            if (bar->abort || globaltimer_ns() - t0 > kSpinLimitNs) {
              set_device_status(p.status, MEDUSA_ERR_TIMEOUT, kDetailAttnStageWait);
              bar->abort = 1;
              ok = false;
              break;
            }
            __nanosleep(20);
          }
        }
        if (!ok) break;
        tc::mma_commit(&bar->kv_empty[g % kStages]);
        tc::mma_commit(&bar->pv_done[g & 1]);
        if (t == cur.steps - 1) tc::mma_commit(&bar->o_full[k & 1]);
      }
      if (!ok) break;
      // advance to the next existing slice
      do {
        cur = slice_info(++kk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
      } while (cur.slice < p.total && cur.steps == 0);
      ++k;
      if (cur.slice >= p.total) break;
    }
  } else if (warp >= 4) {
    // ---------------- softmax and epilogue ----------------
    // Lane l of warp quarter q: query row 16q + (l & 15), key half l >> 4.
    const int q = warp & 3, h = lane >> 4;
    const int r = 16 * q + (lane & 15);
    const uint32_t la = static_cast<uint32_t>(32 * q) << 16;
    uint64_t anc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int w = 0; w < 4; ++w)
      if (r < T && w < p.t.W) anc[w] = p.t.anc[r * p.t.W + w];
    int g = 0, k = 0;
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const Slice s = slice_info(kk, p.total, p.B, p.H, T, p.Lcap, p.seq_lens);
      if (s.slice >= p.total) break;
      if (s.steps == 0) {
        if (lane == 0 && q == 0) set_device_status(p.status, MEDUSA_ERR_DEVICE_CHECK, kDetailAttnSeqLen);
        continue;
      }
      float mref = -INFINITY, lsum = 0.f;
      for (int t = 0; t < s.steps; ++t, ++g) {
        if (!wait_bar(&bar->s_full, g & 1, bar, p.status)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        // tcgen05.ld addresses are warp-uniform: read both 64-key halves of
        // the row and keep this lane's half (h).
        float sv[64];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          float a[32], b[32];
          tc::tmem_ld32(tmem + la + kColS + 32 * part, a);
          tc::tmem_ld32(tmem + la + kColS + 64 + 32 * part, b);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) sv[32 * part + c] = h ? b[c] : a[c];
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bar->s_free);
        const int key0 = t * kStep + h * 64;
        float tmax = -INFINITY;
        if (key0 + 64 > s.L) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int key = key0 + c;
            bool keep = key < s.L;
            if (!keep && key < s.n) {
              const int tj = key - s.L;
              const uint64_t wd = tj < 64 ? anc[0] : tj < 128 ? anc[1] : tj < 192 ? anc[2] : anc[3];
              keep = (wd >> (tj & 63)) & 1ull;
            }
            const float v = keep ? sv[c] * p.scale_log2 : -INFINITY;
            sv[c] = v;
            tmax = fmaxf(tmax, v);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            sv[c] *= p.scale_log2;
            tmax = fmaxf(tmax, sv[c]);
          }
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));   // both halves of the row
        float factor = 1.f;
        if (tmax > mref + kRescaleLog2 || (mref == -INFINITY && tmax > -INFINITY)) {
          factor = (mref == -INFINITY) ? 0.f : exp2f(mref - tmax);
          mref = tmax;
        }
        const float mu = (mref == -INFINITY) ? 0.f : mref;
        float ps = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          sv[c] = exp2f(sv[c] - mu);
          ps += sv[c];
        }
        lsum = lsum * factor + ps;
        // O is rescaled only after every P V issued into it is done (rare);
        // P buffer g&1 is rewritten once the P V of step g-2 has read it.
        const uint32_t ocol = col_o(k & 1);
        if (t > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
          if (!wait_bar(&bar->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, bar, p.status)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
#pragma unroll 1
          for (int c0 = 0; c0 < kHd; c0 += 32) {
            float o[32];
            tc::tmem_ld32(tmem + la + ocol + c0, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= factor;
            tc::tmem_st32(tmem + la + ocol + c0, o);
          }
        }
        if (g >= 2) {
          if (!wait_bar(&bar->pv_done[g & 1], ((g - 2) >> 1) & 1, bar, p.status)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
        }
        float hi[32], lo[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float a0 = sv[2 * c], a1 = sv[2 * c + 1];
          const uint32_t ph = pack2(a0, a1);
          hi[c] = __uint_as_float(ph);
          lo[c] = __uint_as_float(pack2(a0 - __uint_as_float(ph << 16), a1 - __uint_as_float(ph & 0xffff0000u)));
        }
        // Lane pair (h = 0, 1) of a query: the h = 0 lane stores the high
        // parts of all 128 keys, the h = 1 lane the remainders, so one M = 128
        // product accumulates both; each lane hands its partner the half it
        // lacks.
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float send = h == 0 ? lo[c] : hi[c];
          const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
          if (h == 0) lo[c] = recv;   // lo[] now: high parts of keys 64-127
          else hi[c] = recv;          // hi[] now: remainders of keys 0-63
        }
        tc::tmem_st32(tmem + la + col_p(g & 1), hi);
        tc::tmem_st32(tmem + la + col_p(g & 1) + 32, lo);
        tc::tmem_wait_st();
        if (t == s.steps - 1 && t * kStep + kStep > s.n) {
          // V rows past the slice's last key: zero them so 0 * (stale value) stays 0.
          unsigned char* vd = smem + kOffKV + (g % kStages) * 2 * kTile + kTile;
          const int first = s.n - t * kStep;
          for (int x = (warp - 4) * 32 + lane; x < (kStep - first) * 8; x += 128) {
            const int rr = first + x / 8, cc = x % 8;   // 8 chunks of 16 B per 128-byte row
            *reinterpret_cast<uint4*>(vd + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(vd + kHalfTile + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
          }
          tc::fence_proxy_async_smem();
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bar->p_full);

        if (t == s.steps - 1) {
          // Epilogue: O = O(keys 0-63 of every step) + O(keys 64-127), / sum.
          if (!wait_bar(&bar->o_full[k & 1], (k >> 1) & 1, bar, p.status)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const float inv = 1.f / (lsum + __shfl_xor_sync(0xffffffffu, lsum, 16));
          float* orow = p.out + ((static_cast<size_t>(s.lb) * T + r) * p.H + s.e) * kHd;
#pragma unroll 1
          for (int cp = 0; cp < 2; ++cp) {
            float a[32], bq[32];
            tc::tmem_ld32(tmem + la + ocol + cp * 32, a);
            tc::tmem_ld32(tmem + la + ocol + 64 + cp * 32, bq);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float send = h == 0 ? bq[c] : a[c];
              const float keep = h == 0 ? a[c] : bq[c];
              a[c] = (keep + __shfl_xor_sync(0xffffffffu, send, 16)) * inv;
            }
            if (r < T) {
              float* dst = orow + h * 64 + cp * 32;
#pragma unroll
              for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(a[c], a[c + 1], a[c + 2], a[c + 3]);
            }
          }
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bar->o_free[k & 1]);
        }
      }
      ++k;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// Tensor maps: Q as [layers*B][T][H][128] (box 64 dims x 64 rows, rows past
// T read as zero), K and V as [slices][Lcap][128].  For K/V a 4-D view
// {64 dims, rows, 2 halves, slices} loads a whole 128-key tile (both 64-dim
// halves, 32 KB) with one TMA instruction; if the driver rejects that view
// the kernel falls back to two 16 KB boxes per tile.
medusa_status_t launch_attention_tc64(const TreeDev& t, int layers, int B, int H, const void* q,
                                      const void* k_cache, const void* v_cache, int Lcap, const int32_t* seq_lens,
                                      float scale_log2, float* out, int* status, cudaStream_t stream) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: cuTensorMapEncodeTiled unavailable");
  if (t.T > kRows) return fail(MEDUSA_ERR_UNSUPPORTED, "tree attention: more than 64 tree tokens");
  const long long slices = static_cast<long long>(layers) * B * H;
  CUtensorMap qm, km, vm;
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHd), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(t.T), static_cast<cuuint64_t>(layers) * B};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHd) * 2, static_cast<cuuint64_t>(H) * kHd * 2,
                                   static_cast<cuuint64_t>(t.T) * H * kHd * 2};
    const cuuint32_t box[4] = {64, 1, 16, 1};
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
  prm.total = static_cast<int>(slices);
  prm.seq_lens = seq_lens;
  prm.scale_log2 = scale_log2;
  prm.out = out;
  prm.status = status;
  prm.kv_one_box = one_box;
  const int grid = static_cast<int>(slices < sm_count() ? slices : sm_count());
  cudaError_t e = cudaFuncSetAttribute(tree_attn_tc64, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) {
    tree_attn_tc64<<<grid, kThreads, kSmemBytes, stream>>>(qm, km, vm, prm);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail("medusa_tree_attention: tcgen05 launch", e);
}

}  // namespace medusa
