// sm100_sync.cuh -- bounded mbarrier waits shared by the tcgen05 kernels, and
// the TMA tensor-map encoder for [B, N, heads, 64] bf16 tensors.
//
// Every wait gives up after a time limit (globaltimer): it then sets
// LC_DEVSTAT_TIMEOUT in the device status word and the CTA's abort flag, so
// that every role of the CTA stops, drains what it has in flight and returns.
#pragma once

#include <cuda.h>

#include "lc_internal.cuh"
#include "sm100_ptx.cuh"

namespace lcsm100 {

struct Ctx {
  uint32_t bar0;                 // smem address of barrier 0
  volatile int *abort_flag;      // smem
  int *status;
  long long timeout_ns;
  __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
};

// Bounded wait: true when the phase of `parity` completed; false when the CTA
// aborted or this wait timed out (which sets the abort flag and the status).
// (Everything is inlined: register-split regions must not contain calls.)
__device__ __forceinline__ bool wait_bar_slow(const Ctx &c, uint32_t bar, uint32_t parity) {
  uint64_t t0 = lcptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (lcptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*c.abort_flag) return false;
      if ((long long)(lcptx::globaltimer_ns() - t0) > c.timeout_ns) {
        atomicOr(c.status, LC_DEVSTAT_TIMEOUT);
        *c.abort_flag = 1;
        __threadfence_block();
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_bar(const Ctx &c, uint32_t bar, uint32_t parity) {
  if (lcptx::mbar_try_wait(bar, parity)) return true;
  return wait_bar_slow(c, bar, parity);
}

// Warp-uniform form for warps whose lanes then run .sync.aligned tcgen05 ops
// together: every lane waits, and the warp fails as one if any lane failed.
__device__ __forceinline__ bool wait_warp(const Ctx &c, uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, wait_bar(c, bar, parity)) != 0;
}

// Wait for the phase of `parity` with a time limit and no side effects: for
// draining one's own copies or MMAs before exit.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, long long timeout_ns) {
  const uint64_t t0 = lcptx::globaltimer_ns();
  while (!lcptx::mbar_try_wait(bar, parity) &&
         (long long)(lcptx::globaltimer_ns() - t0) < timeout_ns) {
  }
}

}  // namespace lcsm100

// Tensor map over one segment of a [B, ntot, heads, 64] bf16 tensor: tokens
// [tok0, tok0 + nseg) of every batch entry; boxes of 64 tokens x 1 head,
// 128-byte swizzle, zero fill out of range (attn_sm100.cu).
lc_status lc_encode_segment(CUtensorMap *m, const void *base, int batch, long long ntot,
                            long long tok0, long long nseg, int heads);
// Tensor map over an fp32 [B, ntot, heads, 64] tensor: boxes of 64 tokens x
// 1 head x 32 channels (128 bytes, 128-byte swizzle), for TMA reduce-adds of
// half rows (attn_sm100.cu).
lc_status lc_encode_f32_halfrows(CUtensorMap *m, const float *base, int batch, long long ntot,
                                 int heads);
