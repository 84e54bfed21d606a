// Device helpers shared by the kernels of libmedusa_b200 (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "internal.h"

namespace medusa {

// Device status codes written into the per-device status word.
enum DeviceDetail : int {
  kDetailNone = 0,
  kDetailHeadsS1Wait = 1,     // heads: waiting for every CTA's residual-block rows
  kDetailHeadsStageWait = 2,  // heads: a TMA stage never completed
  kDetailAttnSeqLen = 3,      // attention: seq_lens[b] + T > Lcap
  kDetailAttnStageWait = 4,   // attention: a tile copy never completed
  kDetailAcceptSeqLen = 5,    // accept_kv: seq_lens[b] + T > Lcap or bad accept_len
  kDetailPosteriorArgs = 6,   // posterior: a candidate token outside [0, V)
  kDetailPosteriorWait = 7,   // step: the compaction waited for a sequence's walk in vain
  kDetailDecoderWait = 8,     // tree decode: a matrix product's copy or product never completed
  kDetailDecoderToken = 9,    // tree decode: a tree token outside [0, V)
  kDetailDecoderSeqLen = 10,  // tree decode: seq_lens[b] + T > Lcap
};

// Address of the current device's status word ([0] status, [1] detail).
int* device_status_ptr();

__device__ __forceinline__ void set_device_status(int* st, int code, int detail) {
  if (st && atomicCAS(st, 0, code) == 0) atomicExch(st + 1, detail);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Upper bound on any spin in this library: two seconds of wall time.
constexpr uint64_t kSpinLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- programmatic dependent launch ------------------------------------------
// In a kernel launched with programmatic stream serialisation, wait_prior_grids()
// returns once the preceding kernel of the stream has completed and its memory
// is visible; allow_dependents() lets the next such kernel be scheduled early.
// Both are no-ops in a kernel launched the ordinary way.
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- mbarrier -------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase completion.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Waits for the phase with the given parity to complete; gives up after
// kSpinLimitNs and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && globaltimer_ns() - t0 > kSpinLimitNs) return false;
  }
}

// ---- TMA bulk copies (1-D, no tensor map, no multicast) -------------------

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both ends 16-byte
// aligned) that signals `bar` with complete_tx.
__device__ __forceinline__ void tma_load_1d(void* dst_smem, const void* src, uint32_t bytes,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---- element conversion ---------------------------------------------------

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// fp32 -> bf16, round to nearest even: one conversion instruction, no branch
// (a data-dependent branch per value serialised the epilogues' unrolled loops).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

// ---- acquire / release on global counters ---------------------------------

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned atom_add_release_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Order of candidates in every top-k / argmax of the library: larger value
// first, lower token id first among equal values.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

}  // namespace medusa
