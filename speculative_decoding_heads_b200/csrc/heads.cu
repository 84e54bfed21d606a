// S1-S3: the Medusa heads and their per-head top-k, as one persistent,
// HBM-streaming kernel.
//
// Each head k is one residual block followed by its own vocabulary
// projection ("Medusa API参考：核心函数与类详解", MedusaModelABC: medusa_head is
// residual blocks plus a linear layer; "Medusa — 让大模型自己同时猜好几个 token",
// 是什么: a one-layer MLP with a residual on the last hidden state):
//     u[b,k] = h[b] + SiLU(W1[k] h[b] + b1[k])        (fp32, never rounded)
//     z[b,k] = Wout[k] u[b,k]                         (fp32 head logits)
// and each head's top-k tokens become the candidates of tree depth k
// (核心要点: the heads' top-k assembled into a prefix tree).
//
// Design (batch 1..4 per launch, weights read exactly once per launch):
//  * One CTA per SM, launched cooperatively so all CTAs are resident.  The
//    W1 rows (K*d) and then the Wout rows (K*V) are split evenly over the
//    CTAs; every CTA streams its rows through a ring of shared-memory stages
//    (R rows each) filled by 1-D TMA bulk copies (cp.async.bulk + mbarrier
//    complete_tx) with an L2 evict-first hint: every weight byte is read once.
//  * Warp-specialised: warp 0 issues the copies and refills a stage as soon
//    as every consumer warp has released it; the consumer warps (thread t
//    owns the 16-byte column vectors t, t+NT, ... of every row and keeps the
//    matching slice of h or u in registers) turn a stage into R*NB partial
//    dot products per warp; warp 1 (epilogue) sums the partials of the
//    consumer warps and applies S1's residual/SiLU or S3's running top-k.
//    Stages, partial buffers and the epilogue are decoupled by mbarriers, so
//    no CTA-wide barrier sits on the weight stream.
//  * Phase 1 writes u to the workspace; once a CTA's last W1 row is done,
//    the epilogue warp bumps a release counter and waits (acquire, bounded)
//    for every CTA, then lets the consumers load u.  Wout copies keep
//    flowing meanwhile, so the stream never stops at the S1 -> S2 boundary.
//  * The epilogue warp keeps a running top-k per (sequence, head) in shared
//    memory; a new logit is inserted only when it beats the current k-th
//    entry.  At the end each CTA publishes its lists, and the last CTA to
//    finish merges them (k rounds of a warp arg-max over the published
//    candidates) and resets the counters for the next call.
#include <atomic>
#include <cfloat>
#include <cstdint>

#include "heads_common.cuh"

namespace medusa {
namespace {

constexpr int kMaxConsumers = 512;    // consumer threads, one sequence per launch
constexpr int kMaxConsumersMulti = 832;   // consumer threads with 2-4 sequences (one vector each)
constexpr int kRoleWarps = 2;         // producer + epilogue
constexpr int kMaxThreads = kMaxConsumers + 32 * kRoleWarps;
constexpr int kMaxThreadsMulti = kMaxConsumersMulti + 32 * kRoleWarps;
// With several sequences per launch a thread's work per vector grows with
// the batch; rows of 513-832 vectors (4-row stages) then get one vector per
// thread (more warps to hide the FMA chains) instead of two.
template <int NB, int VPT, int R>
constexpr int heads_threads() { return (NB > 1 && VPT == 1 && R == 4) ? kMaxThreadsMulti : kMaxThreads; }
constexpr int kMaxNB = 4;             // sequences per launch
constexpr int kStageMax = 64 * 1024;  // bytes per stage: 8 rows when they fit, else 4
constexpr int kRingTarget = 192 * 1024;
constexpr int kMaxStages = 12;

struct HeadsArgs {
  const void* h;
  const void* W1;
  const void* b1;
  const void* Wout;
  int B, d, V, K, topk;
  int b0, nb;             // sequences [b0, b0+nb) in this launch
  float* head_logits;     // nullable [B, K, V]
  int32_t* topk_ids;      // [B, K, topk]
  float* topk_vals;
  float* u;               // workspace [B, K, d]
  float* cand_vals;       // workspace [kMaxNB, K, G, topk]
  int32_t* cand_ids;
  unsigned* counters;     // workspace: [0] CTAs done with phase 1, [1] with phase 2
  int* status;
  int G;
  int NS;                 // stages in the ring
  int nvec;               // 16-byte vectors per row
  int NT;                 // consumer threads
  int p1_max;             // most phase-1 rows of any CTA
  int do_build;           // 1: the last CTA also builds the candidate tree (S4) for all B sequences
  TreeBuild build;
  unsigned s1_extra;      // arrivals the S1 -> S2 wait expects beyond the G CTAs (0; a test sets 1)
  unsigned long long s1_limit_ns;   // bound on the S1 -> S2 wait (the other waits take kSpinLimitNs)
};

template <typename TW>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int E = 4;
};
template <>
struct Elem<uint16_t> {
  static constexpr int E = 8;
};

// First row of CTA c when n rows are split evenly over G CTAs.
__device__ __forceinline__ int part_lo(int n, int c, int G) {
  return static_cast<int>(static_cast<long long>(n) * c / G);
}

// The stages of one CTA: its phase-1 rows, then its phase-2 rows, at most R
// rows each and never across a head boundary.  All 32-bit and incremental:
// the only divisions happen when the cursor enters a phase.
struct Cursor {
  int phase;      // 1, 2, or 3 (done)
  int row, n;     // stage rows [row, row + n) of the phase's matrix
  int end;        // end of this CTA's rows in the current phase
  int head;       // head of `row`
  int head_end;   // first row of the next head
  int p2_lo, p2_hi;
};

template <int R>
__device__ __forceinline__ void cursor_fix(Cursor& c, const HeadsArgs& a) {
  if (c.phase == 1 && c.row >= c.end) {
    c.phase = 2;
    c.row = c.p2_lo;
    c.end = c.p2_hi;
    c.head = c.row / a.V;
    c.head_end = (c.head + 1) * a.V;
  }
  if (c.phase == 2 && c.row >= c.end) {
    c.phase = 3;
    c.n = 0;
    return;
  }
  const int lim = c.end < c.head_end ? c.end : c.head_end;
  c.n = lim - c.row < R ? lim - c.row : R;
}

template <int R>
__device__ __forceinline__ void cursor_start(Cursor& c, const HeadsArgs& a, int p1_lo, int p1_hi, int p2_lo,
                                             int p2_hi) {
  c.phase = 1;
  c.row = p1_lo;
  c.end = p1_hi;
  c.head = p1_lo / a.d;
  c.head_end = (c.head + 1) * a.d;
  c.p2_lo = p2_lo;
  c.p2_hi = p2_hi;
  cursor_fix<R>(c, a);
}

template <int R>
__device__ __forceinline__ void cursor_next(Cursor& c, const HeadsArgs& a) {
  c.row += c.n;
  if (c.row >= c.head_end) {
    ++c.head;
    c.head_end += (c.phase == 1) ? a.d : a.V;
  }
  cursor_fix<R>(c, a);
}

template <typename TW>
__device__ __forceinline__ const char* stage_src(const HeadsArgs& a, const Cursor& c) {
  const size_t row_bytes = static_cast<size_t>(a.d) * sizeof(TW);
  const char* base = static_cast<const char*>(c.phase == 1 ? a.W1 : a.Wout);
  return base + static_cast<size_t>(c.row) * row_bytes;
}

// Loads the E elements of vector `v` of row vector x (element type TX) as fp32.
template <typename TX>
__device__ __forceinline__ void load_vec(const TX* x, int v, float* out);
template <>
__device__ __forceinline__ void load_vec<float>(const float* x, int v, float* out) {
  const float4 a = __ldcg(reinterpret_cast<const float4*>(x) + v);
  out[0] = a.x;
  out[1] = a.y;
  out[2] = a.z;
  out[3] = a.w;
}
template <>
__device__ __forceinline__ void load_vec<uint16_t>(const uint16_t* x, int v, float* out) {
  const uint4 a = __ldcg(reinterpret_cast<const uint4*>(x) + v);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = bf16lo(w[i]);
    out[2 * i + 1] = bf16hi(w[i]);
  }
}

// fp32 u (phase 2) for a bf16 model: 8 floats per 16-byte weight vector.
__device__ __forceinline__ void load_u_vec(const float* u, int v, int E, float* out) {
  const float4* p = reinterpret_cast<const float4*>(u) + static_cast<size_t>(v) * (E / 4);
  for (int i = 0; i < E / 4; ++i) {
    const float4 a = __ldcg(p + i);
    out[4 * i] = a.x;
    out[4 * i + 1] = a.y;
    out[4 * i + 2] = a.z;
    out[4 * i + 3] = a.w;
  }
}

template <typename TW>
__device__ __forceinline__ float to_f32(TW x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<uint16_t>(uint16_t x) {
  return __uint_as_float(static_cast<uint32_t>(x) << 16);
}

// Two fp32 values in one 64-bit register pair, and the packed fp32 FMA of
// sm_100 (two independent IEEE fmas per instruction).
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void fma_f2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float sum_f2(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}

// acc[b] += dot(16-byte weight vector w, x[b]) for b < NB, where x[b] holds
// the matching E activations as E/2 (even, odd) pairs and acc[b] keeps an
// even and an odd partial sum.
template <typename TW, int NB, int VPT>
__device__ __forceinline__ void dot_vec(const uint4 w, const uint64_t (&xp)[NB * VPT][Elem<TW>::E / 2], int j,
                                        uint64_t* acc) {
  constexpr int E = Elem<TW>::E;
  uint64_t wp[E / 2];
  if constexpr (E == 8) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) wp[i] = pack_f2(bf16lo(ww[i]), bf16hi(ww[i]));
  } else {
    wp[0] = pack_f2(__uint_as_float(w.x), __uint_as_float(w.y));
    wp[1] = pack_f2(__uint_as_float(w.z), __uint_as_float(w.w));
  }
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int i = 0; i < E / 2; ++i) fma_f2(acc[b], wp[i], xp[b * VPT + j][i]);
}

// Packs E activations into E/2 (even, odd) pairs.
template <int E>
__device__ __forceinline__ void pack_x(const float* f, uint64_t* xp) {
#pragma unroll
  for (int i = 0; i < E / 2; ++i) xp[i] = pack_f2(f[2 * i], f[2 * i + 1]);
}

__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

// Waits for the phase with the given parity; gives up after limit_ns, or as
// soon as another role of the CTA has aborted (*abort == 1), and returns false.
__device__ __forceinline__ bool wait_or_quit(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && (*abort == 1 || globaltimer_ns() - t0 > limit_ns)) return false;
  }
}

// CTA of row r when n rows are split evenly over G CTAs (inverse of part_lo).
__device__ __forceinline__ int part_of(int r, int n, int G) {
  return static_cast<int>((static_cast<long long>(r + 1) * G - 1) / n);
}

// Sums C values over the 32 lanes of a warp by repeated halving: at each
// step a lane keeps half of its values and trades the other half with its
// partner, so C values need C-1 + log2(32/C) shuffles instead of 5*C.  On
// return v[0] holds the full sum of value `idx`; lanes whose low
// log2(32/C) bits are zero hold each value exactly once.
template <int C, int O>
struct WarpFold {
  static __device__ __forceinline__ void run(float* v, int lane, int& idx) {
    if constexpr (O == 0) {
      return;
    } else if constexpr (C > 1) {
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < C / 2; ++i) {
        const float send = up ? v[i] : v[i + C / 2];
        const float keep = up ? v[i + C / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      if (up) idx += C / 2;
      WarpFold<C / 2, O / 2>::run(v, lane, idx);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      WarpFold<1, O / 2>::run(v, lane, idx);
    }
  }
};

// Shared-memory carve-up of one CTA (offsets in bytes; stages first, 128-byte aligned).
struct Layout {
  size_t stages, partial, pre_h, pre_b, list_v, list_i, list_n, bars, flags, total;
};

__host__ __device__ inline Layout make_layout(size_t stage_bytes, int NS, int NWC, int RNB, int NB, int K, int topk,
                                              int p1_max) {
  Layout l{};
  size_t o = 0;
  l.stages = o;
  o += stage_bytes * NS;
  l.partial = o;                                   // [NS][NWC][RNB] fp32
  o += static_cast<size_t>(NS) * NWC * RNB * 4;
  l.pre_h = o;                                     // [p1_max][NB] fp32: h[b][row within head]
  o += static_cast<size_t>(p1_max) * NB * 4;
  l.pre_b = o;                                     // [p1_max] fp32: b1[head][row within head]
  o += static_cast<size_t>(p1_max) * 4;
  l.list_v = o;                                    // [NB][K][topk]
  o += static_cast<size_t>(NB) * K * topk * 4;
  l.list_i = o;
  o += static_cast<size_t>(NB) * K * topk * 4;
  l.list_n = o;                                    // [NB][K]
  o += static_cast<size_t>(NB) * K * 4;
  o = (o + 15) & ~size_t(15);
  l.bars = o;                                      // full, empty, pready, pfree [NS] each; u_ready
  o += (4 * static_cast<size_t>(NS) + 1) * 8;
  l.flags = o;                                     // [0] abort, [1] last-CTA flag
  o += 16;
  l.total = o;
  return l;
}

template <typename TW, int NB, int VPT, int R>
__global__ void __launch_bounds__(heads_threads<NB, VPT, R>(), 1) heads_kernel(const HeadsArgs a) {
  constexpr int E = Elem<TW>::E;
  constexpr int RNB = R * NB;
  static_assert(RNB <= 32 && (32 % RNB) == 0, "partials use one lane per (row, sequence)");
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int NWC = a.NT >> 5;                      // consumer warps
  const int cta = blockIdx.x;
  const int G = a.G;
  const int NS = a.NS;
  const size_t row_bytes = static_cast<size_t>(a.d) * sizeof(TW);
  const size_t stage_bytes = row_bytes * R;
  const Layout lay = make_layout(stage_bytes, NS, NWC, RNB, NB, a.K, a.topk, a.p1_max);

  unsigned char* stages = smem + lay.stages;
  float* partial = reinterpret_cast<float*>(smem + lay.partial);
  float* pre_h = reinterpret_cast<float*>(smem + lay.pre_h);
  float* pre_b = reinterpret_cast<float*>(smem + lay.pre_b);
  float* list_v = reinterpret_cast<float*>(smem + lay.list_v);
  int* list_i = reinterpret_cast<int*>(smem + lay.list_i);
  int* list_n = reinterpret_cast<int*>(smem + lay.list_n);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + NS;
  uint64_t* pready = empty + NS;
  uint64_t* pfree = pready + NS;
  uint64_t* u_ready = pfree + NS;
  volatile int* flag = reinterpret_cast<volatile int*>(smem + lay.flags);

  const int n1 = a.K * a.d;
  const int n2 = a.K * a.V;
  const int p1_lo = part_lo(n1, cta, G), p1_hi = part_lo(n1, cta + 1, G);
  const int p2_lo = part_lo(n2, cta, G), p2_hi = part_lo(n2, cta + 1, G);

  for (int i = tid; i < NB * a.K * a.topk; i += blockDim.x) {
    list_v[i] = -FLT_MAX;
    list_i[i] = -1;
  }
  for (int i = tid; i < NB * a.K; i += blockDim.x) list_n[i] = 0;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NWC);
      mbar_init(&pready[s], NWC * RNB);
      mbar_init(&pfree[s], 1);
    }
    mbar_init(u_ready, 1);
    fence_barrier_init();
    flag[0] = 0;
    flag[1] = 0;
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const uint64_t policy = l2_evict_first_policy();
      Cursor pc;
      cursor_start<R>(pc, a, p1_lo, p1_hi, p2_lo, p2_hi);
      int s = 0;
      for (; pc.phase != 3; ++s) {
        const int slot = s % NS;
        if (s >= NS && !wait_or_quit(&empty[slot], static_cast<uint32_t>(((s / NS) - 1) & 1), flag, kSpinLimitNs)) {
          set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailHeadsStageWait);
          flag[0] = 1;
          break;
        }
        if (flag[0]) break;
        const uint32_t bytes = static_cast<uint32_t>(pc.n * row_bytes);
        mbar_arrive_expect_tx(&full[slot], bytes);
        tma_load_1d(stages + slot * stage_bytes, stage_src<TW>(a, pc), bytes, &full[slot], policy);
        cursor_next<R>(pc, a);
      }
      // Every copy issued lands before the CTA exits (after an abort the
      // consumers may not have waited for the last ones).
      for (int t = s - NS < 0 ? 0 : s - NS; t < s; ++t)
        mbar_wait(&full[t % NS], static_cast<uint32_t>((t / NS) & 1));
    }
  }
  else if (warp >= kRoleWarps) {
    // ---------------- consumers ----------------
    const int ct = tid - 32 * kRoleWarps;
    const int cw = warp - kRoleWarps;
    // x[b*VPT+j][e]: h (phase 1) or u of the current head (phase 2), for the
    // thread's column vectors ct + j*NT.
    uint64_t xp[NB * VPT][E / 2];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = ct + j * a.NT;
        float f[E];
        if (b < a.nb && v < a.nvec) {
          load_vec<TW>(static_cast<const TW*>(a.h) + static_cast<size_t>(a.b0 + b) * a.d, v, f);
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e) f[e] = 0.f;
        }
        pack_x<E>(f, xp[b * VPT + j]);
      }
    Cursor cc;
    cursor_start<R>(cc, a, p1_lo, p1_hi, p2_lo, p2_hi);
    int cur_head2 = -1;   // head whose u sits in x during phase 2
    bool u_ok = false;
    for (int s = 0; cc.phase != 3; ++s) {
      const int slot = s % NS;
      const int khead = cc.head;   // uniform per stage
      if (cc.phase == 2 && khead != cur_head2) {
        if (!u_ok) {
          if (!wait_or_quit(u_ready, 0u, flag, kSpinLimitNs)) {
            set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailHeadsS1Wait);
            flag[0] = 1;
          }
          if (flag[0]) break;
          u_ok = true;
        }
        cur_head2 = khead;
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            const int v = ct + j * a.NT;
            if (b < a.nb && v < a.nvec) {
              float f[E];
              load_u_vec(a.u + (static_cast<size_t>(a.b0 + b) * a.K + khead) * a.d, v, E, f);
              pack_x<E>(f, xp[b * VPT + j]);
            }
          }
      }
      if (!wait_or_quit(&full[slot], static_cast<uint32_t>((s / NS) & 1), flag, kSpinLimitNs)) {
        set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailHeadsStageWait);
        flag[0] = 1;
      }
      if (flag[0]) break;

      // Per row: an (even, odd) pair of partial sums per sequence, folded
      // into one fp32 partial sum once the row is done.
      float acc[RNB];
      const unsigned char* st = stages + slot * stage_bytes;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint64_t acc2[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc2[b] = 0ull;   // (+0.0f, +0.0f)
        if (r < cc.n) {
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            const int v = ct + j * a.NT;
            if (v < a.nvec) {
              const uint4 w = *reinterpret_cast<const uint4*>(st + r * row_bytes + static_cast<size_t>(v) * 16);
              dot_vec<TW, NB, VPT>(w, xp, j, acc2);
            }
          }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[r * NB + b] = sum_f2(acc2[b]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cta(&empty[slot]);   // this warp is done with the stage's bytes
      int idx = 0;
      WarpFold<RNB, 16>::run(acc, lane, idx);
      if (s >= NS && !wait_or_quit(&pfree[slot], static_cast<uint32_t>(((s / NS) - 1) & 1), flag, kSpinLimitNs)) {
        set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailHeadsStageWait);
        flag[0] = 1;
        break;
      }
      if ((lane & (32 / RNB - 1)) == 0) {
        partial[(slot * NWC + cw) * RNB + idx] = acc[0];
        mbar_arrive_cta(&pready[slot]);
      }
      cursor_next<R>(cc, a);
    }
  } else {
    // ---------------- epilogue (warp 1) ----------------
    for (int i = lane; i < p1_hi - p1_lo; i += 32) {
      const int row = p1_lo + i;
      const int head = row / a.d;
      const int local = row - head * a.d;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        pre_h[i * NB + b] =
            b < a.nb ? to_f32<TW>(static_cast<const TW*>(a.h)[static_cast<size_t>(a.b0 + b) * a.d + local]) : 0.f;
      pre_b[i] = to_f32<TW>(static_cast<const TW*>(a.b1)[static_cast<size_t>(head) * a.d + local]);
    }
    __syncwarp();
    // This CTA's u rows are written: count it, wait (bounded) for every CTA,
    // then let the consumers read u.
    auto publish = [&]() {
      __threadfence();   // every lane's u rows, once
      __syncwarp();
      if (lane == 0) {
        atom_add_release_gpu(&a.counters[0], 1u);
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(&a.counters[0]) < static_cast<unsigned>(G) + a.s1_extra) {
          if (globaltimer_ns() - t0 > a.s1_limit_ns) {
            set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailHeadsS1Wait);
            flag[0] = 1;
            break;
          }
          __nanosleep(64);
        }
        mbar_arrive_cta(u_ready);
      }
      __syncwarp();
    };
    if (p1_hi == p1_lo) publish();
    Cursor cc;
    cursor_start<R>(cc, a, p1_lo, p1_hi, p2_lo, p2_hi);
    for (int s = 0; cc.phase != 3; ++s) {
      const int slot = s % NS;
      if (!wait_or_quit(&pready[slot], static_cast<uint32_t>((s / NS) & 1), flag, kSpinLimitNs)) {
        set_device_status(a.status, MEDUSA_ERR_TIMEOUT, kDetailHeadsStageWait);
        flag[0] = 1;
      }
      if (flag[0]) break;
      // Cross-warp sum: lane l adds entries l, l+32, ... (all of value
      // l % RNB), then lanes with equal l % RNB combine.
      float val = 0.f;
      const float* pb = partial + slot * NWC * RNB;
      for (int e = lane; e < NWC * RNB; e += 32) val += pb[e];
#pragma unroll
      for (int o = RNB; o < 32; o <<= 1) val += __shfl_xor_sync(0xffffffffu, val, o);
      __syncwarp();
      if (lane == 0) mbar_arrive_cta(&pfree[slot]);
      // Lane t < RNB owns row t / NB and sequence t % NB of the stage.
      const int khead = cc.head;
      const int r = lane / NB, b = lane % NB;
      const bool live = lane < RNB && r < cc.n && b < a.nb;
      const int local = cc.row - khead * (cc.phase == 1 ? a.d : a.V) + r;   // row within the head
      if (cc.phase == 1) {
        if (live) {
          const int i = cc.row - p1_lo + r;
          a.u[(static_cast<size_t>(a.b0 + b) * a.K + khead) * a.d + local] = pre_h[i * NB + b] + silu(val + pre_b[i]);
        }
        if (cc.row + cc.n >= cc.end) publish();   // the CTA's last W1 stage
      } else {
        if (live && a.head_logits)
          a.head_logits[(static_cast<size_t>(a.b0 + b) * a.K + khead) * a.V + local] = val;
        bool cand = false;
        if (live) {
          const int li = b * a.K + khead;
          cand = list_n[li] < a.topk ||
                 ranks_before(val, local, list_v[li * a.topk + a.topk - 1], list_i[li * a.topk + a.topk - 1]);
        }
        unsigned m = __ballot_sync(0xffffffffu, cand);
        while (m) {
          const int src = __ffs(m) - 1;
          m &= m - 1;
          const float nv = __shfl_sync(0xffffffffu, val, src);
          const int nid = __shfl_sync(0xffffffffu, local, src);
          const int li = (src % NB) * a.K + khead;
          list_insert(list_v + li * a.topk, list_i + li * a.topk, list_n + li, a.topk, nv, nid, lane);
        }
      }
      cursor_next<R>(cc, a);
    }
  }
  allow_dependents();   // the next kernel of medusa_step may take SMs as CTAs finish
  __syncthreads();
  if (flag[0]) return;   // aborted: the producer has drained its copies

  // Publish the local lists of every head this CTA's phase-2 rows touched.
  if (p2_hi > p2_lo) {
    const int k_lo = p2_lo / a.V;
    const int k_hi = (p2_hi - 1) / a.V;
    for (int k = k_lo; k <= k_hi; ++k)
      for (int i = tid; i < NB * a.topk; i += blockDim.x) {
        const int b = i / a.topk, j = i % a.topk;
        const int li = b * a.K + k;
        const size_t o = ((static_cast<size_t>(b) * a.K + k) * G + cta) * a.topk + j;
        a.cand_vals[o] = list_v[li * a.topk + j];
        a.cand_ids[o] = list_i[li * a.topk + j];
      }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned done = atom_add_acq_rel_gpu(&a.counters[1], 1u);
    flag[0] = (done == static_cast<unsigned>(G - 1)) ? 2 : 0;
  }
  __syncthreads();
  if (flag[0] != 2) return;

  // Last CTA: merge the published lists of every (sequence, head).
  __threadfence();
  const int NW = blockDim.x >> 5;
  for (int li = warp; li < a.nb * a.K; li += NW) {
    const int b = li / a.K, k = li % a.K;
    const int hk_lo = k * a.V;
    const int c_lo = part_of(hk_lo, n2, G);
    const int c_hi = part_of(hk_lo + a.V - 1, n2, G);
    const size_t base = ((static_cast<size_t>(b) * a.K + k) * G + c_lo) * a.topk;
    const size_t o = (static_cast<size_t>(a.b0 + b) * a.K + k) * a.topk;
    merge_candidates(a.cand_vals + base, a.cand_ids + base, (c_hi - c_lo + 1) * a.topk, a.topk, a.topk_ids + o,
                     a.topk_vals + o, lane);
  }
  __syncthreads();
  if (tid == 0) {
    a.counters[0] = 0u;
    a.counters[1] = 0u;
    __threadfence();
  }
  if (a.do_build) {
    // S4 from the final top-k (this CTA's merge above and the earlier batch
    // groups' launches).
    __syncthreads();
    build_tree_block(a.build, a.B, a.topk_ids);
  }
}

struct Plan {
  int NT, VPT, NS, R;
  size_t smem;
};

// Consumer threads: one per 16-byte column vector up to 512.  Stages of 8
// rows when 8 rows fit in 64 KB, else 4: one bulk copy per stage, and on
// this hardware a few large copies in flight stream HBM far better than
// many small ones (64 KB stages reach ~94% of the copy bandwidth, 32 KB
// ~68%).  As many stages as fit in ~192 KB (at least 2, at most 12).
template <typename TW>
Plan make_plan(int d, int nb, int K, int topk, int p1_max) {
  constexpr int E = Elem<TW>::E;
  Plan p{};
  const int nvec = d / E;
  const size_t row = static_cast<size_t>(d) * sizeof(TW);
  p.R = row * 8 <= static_cast<size_t>(kStageMax) ? 8 : 4;
  const int max_nt = (nb > 1 && p.R == 4 && nvec <= kMaxConsumersMulti) ? kMaxConsumersMulti : kMaxConsumers;
  p.NT = nvec >= max_nt ? max_nt : ((nvec + 31) / 32) * 32;
  p.VPT = (nvec + p.NT - 1) / p.NT;
  const size_t stage = row * p.R;
  const int ns = static_cast<int>(kRingTarget / stage);
  p.NS = ns < 2 ? 2 : (ns > kMaxStages ? kMaxStages : ns);
  p.smem = make_layout(stage, p.NS, p.NT / 32, p.R * nb, nb, K, topk, p1_max).total;
  return p;
}

template <typename TW, int NB, int VPT, int R>
cudaError_t launch_one(const HeadsArgs& a, const Plan& p, cudaStream_t stream) {
  auto fn = heads_kernel<TW, NB, VPT, R>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(p.smem));
  if (e != cudaSuccess) return e;
  const int threads = p.NT + 32 * kRoleWarps;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, p.smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  void* args[] = {const_cast<HeadsArgs*>(&a)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fn), dim3(a.G), dim3(threads), args,
                                     p.smem, stream);
}

// Two vectors per thread means rows of at least 16 KB, hence 4-row stages.
template <typename TW, int NB, int VPT>
cudaError_t dispatch_r(const HeadsArgs& a, const Plan& p, cudaStream_t stream) {
  if constexpr (VPT == 1) {
    if (p.R == 8) return launch_one<TW, NB, VPT, 8>(a, p, stream);
  }
  return launch_one<TW, NB, VPT, 4>(a, p, stream);
}

template <typename TW, int NB>
cudaError_t dispatch_vpt(const HeadsArgs& a, const Plan& p, cudaStream_t stream) {
  if (p.VPT == 1) return dispatch_r<TW, NB, 1>(a, p, stream);
  return dispatch_r<TW, NB, 2>(a, p, stream);
}

template <typename TW>
cudaError_t dispatch_nb(const HeadsArgs& a, const Plan& p, cudaStream_t stream) {
  if (a.nb == 1) return dispatch_vpt<TW, 1>(a, p, stream);
  if (a.nb == 2) return dispatch_vpt<TW, 2>(a, p, stream);
  return dispatch_vpt<TW, 4>(a, p, stream);
}

// Test hook of the failure-detection path (medusa_test_heads_wait).
std::atomic<unsigned> g_test_s1_extra{0};
std::atomic<unsigned long long> g_test_limit_ns{0};

}  // namespace

size_t heads_workspace_bytes(int B, int d, int V, int K, int topk) {
  const int G = sm_count();
  size_t off = align_up(static_cast<size_t>(B) * K * d * sizeof(float), 256);
  off += align_up(static_cast<size_t>(kMaxNB) * K * G * topk * sizeof(float), 256);
  off += align_up(static_cast<size_t>(kMaxNB) * K * G * topk * sizeof(int32_t), 256);
  off += 256;  // counters
  // Batches the tensor-core kernel may take (bf16 with d a multiple of 128;
  // the size does not depend on the dtype, so it is reserved either way).
  if (heads_tc_supported(B, d, MEDUSA_BF16)) {
    const size_t tc = heads_tc_workspace_bytes(B, d, V, K, topk);
    if (tc > off) off = tc;
  }
  return off;
}

medusa_status_t launch_heads(const void* h, const void* W1, const void* b1, const void* Wout,
                             int B, int d, int V, int K, int topk, medusa_dtype_t dtype,
                             float* head_logits, int32_t* topk_ids, float* topk_vals, void* ws,
                             cudaStream_t stream, const TreeBuild* build) {
  // Two or more sequences: the tensor cores, weights read once per 16 sequences.
  if (heads_tc_supported(B, d, dtype))
    return launch_heads_tc(h, W1, b1, Wout, B, d, V, K, topk, head_logits, topk_ids, topk_vals, ws, stream, build);
  const int G = sm_count();
  HeadsArgs a{};
  a.h = h;
  a.W1 = W1;
  a.b1 = b1;
  a.Wout = Wout;
  a.B = B;
  a.d = d;
  a.V = V;
  a.K = K;
  a.topk = topk;
  a.head_logits = head_logits;
  a.topk_ids = topk_ids;
  a.topk_vals = topk_vals;
  unsigned char* w = static_cast<unsigned char*>(ws);
  size_t off = 0;
  a.u = reinterpret_cast<float*>(w + off);
  off += align_up(static_cast<size_t>(B) * K * d * sizeof(float), 256);
  a.cand_vals = reinterpret_cast<float*>(w + off);
  off += align_up(static_cast<size_t>(kMaxNB) * K * G * topk * sizeof(float), 256);
  a.cand_ids = reinterpret_cast<int32_t*>(w + off);
  off += align_up(static_cast<size_t>(kMaxNB) * K * G * topk * sizeof(int32_t), 256);
  a.counters = reinterpret_cast<unsigned*>(w + off);
  a.status = device_status_ptr();
  a.G = G;
  a.nvec = (dtype == MEDUSA_BF16) ? d / 8 : d / 4;
  a.p1_max = static_cast<int>((static_cast<long long>(K) * d + G - 1) / G) + 1;
  a.s1_extra = g_test_s1_extra.load();
  const unsigned long long lim = g_test_limit_ns.load();
  a.s1_limit_ns = lim ? lim : kSpinLimitNs;
  for (int b0 = 0; b0 < B; b0 += kMaxNB) {
    a.b0 = b0;
    a.nb = (B - b0) < kMaxNB ? (B - b0) : kMaxNB;
    const int nbt = a.nb == 1 ? 1 : (a.nb == 2 ? 2 : 4);
    const Plan p = (dtype == MEDUSA_BF16) ? make_plan<uint16_t>(d, nbt, K, topk, a.p1_max)
                                          : make_plan<float>(d, nbt, K, topk, a.p1_max);
    a.NS = p.NS;
    a.NT = p.NT;
    a.do_build = (build != nullptr && b0 + a.nb == B) ? 1 : 0;   // after the last batch group
    if (build) a.build = *build;
    cudaError_t e = (dtype == MEDUSA_BF16) ? dispatch_nb<uint16_t>(a, p, stream) : dispatch_nb<float>(a, p, stream);
    if (e != cudaSuccess) return cuda_fail("medusa_heads_topk: launch", e);
  }
  return MEDUSA_OK;
}

}  // namespace medusa

extern "C" medusa_status_t medusa_test_heads_wait(int extra_arrivals, long long limit_ns) {
  if (extra_arrivals < 0 || extra_arrivals > 1024 || limit_ns < 0)
    return medusa::fail(MEDUSA_ERR_INVALID_ARG, "medusa_test_heads_wait: extra_arrivals in [0, 1024], limit_ns >= 0");
  medusa::g_test_s1_extra.store(static_cast<unsigned>(extra_arrivals));
  medusa::g_test_limit_ns.store(static_cast<unsigned long long>(limit_ns));
  return MEDUSA_OK;
}
