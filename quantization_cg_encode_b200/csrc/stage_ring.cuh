// Stage ring shared by the persistent codec kernels: a CTA consumes its work
// units in order from an NST-stage shared-memory ring filled by bulk / TMA
// copies; the last warp to release a stage refills it.  Every wait is bounded,
// and after one wait in the CTA has given up the others are skipped and no
// stage is refilled; before exit the last copy issued into every stage is
// drained (bounded), so nothing is in flight when the CTA ends.
#pragma once
#include "cg_kernels.cuh"

namespace cg {

// Release of a ring stage by one warp (returns how many warps had released it
// before); acq_rel orders every warp's reads of the stage before the refill.
__device__ __forceinline__ uint32_t stage_release(uint32_t* cnt) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(smem_u32(cnt)) : "memory");
  return old;
}
// Wait for a stage; after one wait in the CTA has given up, the others are
// skipped (one time limit per CTA).  The flag is read only when the stage is
// not ready at the first test.
__device__ __forceinline__ void stage_wait(uint64_t* bar, uint32_t phase, volatile uint32_t* abort_v,
                                           unsigned int* status) {
  if (mbar_try_wait(smem_u32(bar), phase)) return;
  if (*abort_v) return;
  if (!mbar_wait(bar, phase, status)) *abort_v = 1u;
}
// Before the CTA exits, the last load issued into every stage has landed
// (immediate unless a wait gave up and its stage was skipped).
__device__ __forceinline__ void drain_stages(uint64_t* full, const uint32_t* ctl, int nst, unsigned int* status) {
  __syncthreads();
  if (threadIdx.x != 0) return;
  const int n_iss = (int)ctl[1];
  for (int st = 0; st < nst && st < n_iss; ++st) {
    const int u = st + nst * ((n_iss - 1 - st) / nst);  // last unit loaded into stage st
    mbar_wait(&full[st], (uint32_t)(u / nst) & 1u, status);
  }
}

// Position of a CTA's work unit (head slice, stage within the slice), advanced
// one unit at a time.
struct Cursor {
  long long slice;
  int bq;
  __device__ __forceinline__ void next(int per_slice) {
    if (++bq == per_slice) {
      bq = 0;
      ++slice;
    }
  }
};

}  // namespace cg
