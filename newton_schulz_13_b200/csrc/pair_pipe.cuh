// Unwinding of the CTA-pair operand pipeline after a wait gave up (shared by the bf16 and the
// 3xTF32 product kernels).
//
// In a pair, both CTAs' TMA producers fill the same ring stages: each copies its half of a stage
// into its own shared memory and counts the bytes on the even CTA's `full` barrier, which the
// even CTA's producer arms (one arrival, both halves' bytes). In normal operation the two
// producers issue the same number of fills. When a wait gives up, they can stop at different
// fills, at most one ring length apart (a producer refills a stage only after the MMAs have
// consumed its previous fill, which needed both halves):
//   - fills the odd CTA issued but the even CTA never armed: the odd half's copies still land
//     and count on a barrier phase that nobody will complete;
//   - fills the even CTA armed and issued alone: that phase waits for bytes that never come.
// Either way some copy may still be in flight when the CTAs want to exit, and a copy must not
// land in the shared memory of a CTA that has exited. So at exit, after a cluster barrier that
// makes both fill counts visible, the even CTA's producer settles the difference (arms the odd
// half's bytes, or removes the missing half's bytes) and waits for the last phase of every
// stage; a second cluster barrier then keeps both CTAs resident until that has happened.
#pragma once
#include <stdint.h>

#include "ptx.cuh"

namespace muon {

// Marks this CTA, and its partner in the pair, as giving up: every bounded pipeline wait of
// either CTA then returns at its next poll.
__device__ __forceinline__ void raise_abort(volatile int* abort_flag, bool pair, uint32_t rank) {
  *abort_flag = 1;
  if (pair) st_shared_cluster(mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u), 1u);
}

// Run by the even CTA's producer thread at exit. `mine` and `peer` are the fills the two producers
// issued; stage f % STAGES of fill f completes phase (f / STAGES) & 1 of its barrier; each CTA's
// half of a stage is `half_bytes`. Waits (bounded by timeout_ns; `never` is a flag nobody sets)
// until the last fill of every stage has landed.
template <int STAGES>
__device__ __forceinline__ void settle_pair_fills(uint64_t* full, uint32_t mine, uint32_t peer, uint32_t half_bytes,
                                                  volatile int* never, uint64_t timeout_ns) {
  const uint32_t lo = mine < peer ? mine : peer;
  const uint32_t hi = mine < peer ? peer : mine;
  for (uint32_t f = lo; f < hi; ++f) {
    uint64_t* bar = &full[f % STAGES];
    if (f >= mine)
      mbar_arrive_expect_tx(bar, half_bytes);   // the odd half alone: arm it
    else
      mbar_complete_tx(bar, half_bytes);        // the even half alone: the odd half never comes
  }
  for (uint32_t s = 0; s < (uint32_t)STAGES && s < hi; ++s) {
    const uint32_t last = s + ((hi - 1u - s) / STAGES) * STAGES;
    mbar_wait_bounded(&full[s], (last / STAGES) & 1u, never, timeout_ns);
  }
}

}  // namespace muon
