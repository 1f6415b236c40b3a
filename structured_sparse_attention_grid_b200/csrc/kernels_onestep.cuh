// One refinement step (the regime of finetuned models: MonarchRT explainers,
// gist.science §2.C "Finetuning and Efficient Implementation") as a single
// kernel: the R step and the output pass y = L z of the same call run in one
// grid, so the output pass of the first heads overlaps the R step of the last
// ones and no launch boundary separates them.
//
// Scheduling.  Each CTA takes one ticket from a counter (atomicAdd) when it
// starts; tickets are handed out in the order CTAs actually start.  The first
// tickets are pairs of R-step items (head-major): the CTA's two 9-warp groups
// each run one item of G key tiles on half of its shared memory and TMEM,
// which is what two R-step CTAs per SM do in the two-kernel form.  The
// remaining tickets are output-pass items (head-major), run by all 18 warps.
// An output item of head bh needs the k~, z, h and block-major q of every key
// tile of that head: its load warp waits (bounded) until the head's count of
// finished R items reaches the number of R items per head.
//
// Every wait ends: a CTA holds a ticket only once it runs, every R ticket is
// handed out before the first output ticket, and an R item waits on nothing
// outside its CTA, so every R item an output item waits for is held by a
// running CTA (or is done).  This holds whatever the number of co-resident
// CTAs.  The wait is still bounded: on expiry it records kErrMbarTimeout and
// the item's remaining waits expire in turn, so the kernel always returns.
//
// Hand-off: an R item's TMA stores are waited to completion by the threads
// that issued them, its h stores are fenced, and one thread adds to the count
// with release semantics after a proxy fence; the consumer's load thread
// acquires the count and issues a proxy fence before its TMA loads.
#pragma once

#include "kernels_rtc.cuh"
#include "kernels_l.cuh"

namespace monarch {

// Shared memory of one R-item group (1024-byte aligned for the swizzled boxes).
template <int D>
constexpr uint32_t onestep_group_bytes() { return (rtc_item_bytes<D>() + 1023u) & ~1023u; }

template <int D>
constexpr size_t onestep_smem() {
  constexpr size_t r = 2 * (size_t)onestep_group_bytes<D>();
  constexpr size_t l = tc::row_smem<D, true>();
  return r > l ? r : l;
}

// Counters of one call (int, zeroed before the launch): [0] the ticket
// counter, [1 + bh] the R items of head bh that are done.
template <typename TQ, typename TO, int D>
__global__ void __launch_bounds__(tc::kThreads, 1)
onestep_tc(const __grid_constant__ RtcMaps rmaps, const __grid_constant__ tc::Maps maps, const TQ* __restrict__ q,
           Work w, TcPlanes<TQ> planes, TO* __restrict__ out, Geo g, int mode, int G, int* __restrict__ counters) {
  static_assert(2 * kRtcThreads == tc::kThreads, "two R-item groups fill the CTA");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (tc::smem_misaligned(smem_raw)) return;
  const int tid = threadIdx.x;
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem_raw);   // read before any item writes these bytes
  if (tid < 32) {
    ptx::tmem_alloc(slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::griddep_wait();   // the counters and the inputs are ready from here on
  if (tid == 32) slot[1] = (uint32_t)atomicAdd(counters, 1);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // dependents may start once every CTA of this grid holds its TMEM, so none
  // of theirs can take the columns a CTA of this grid still has to allocate
  ptx::griddep_launch();
  const uint32_t tmem = slot[0];
  const int ticket = (int)slot[1];
  __syncthreads();

  const int n_rg = (g.b1k + G - 1) / G;   // R items per head
  const int n_r = n_rg * g.BH;
  const int n_rpairs = (n_r + 1) / 2;
  if (ticket < n_rpairs) {
    const int grp = tid >= kRtcThreads ? 1 : 0;
    const int item = 2 * ticket + grp;
    if (item < n_r) {
      const int bh = item / n_rg;
      r_step_item<TQ, D>(rmaps, q, w, planes, g, mode, 1, G, (item - bh * n_rg) * G, bh,
                         smem_raw + grp * onestep_group_bytes<D>(), tmem + 256 * grp, tid - grp * kRtcThreads,
                         grp * (kRtcThreads / 32), 1 + 2 * grp, 2 + 2 * grp, nullptr, 0, counters + 1 + bh);
    }
  } else {
    const int nqb = (g.b1q + 2 * kTile - 1) / (2 * kTile);
    const int l = ticket - n_rpairs;
    const int bh = l / (nqb * g.b2), rem = l - bh * nqb * g.b2;
    const int a2 = rem / nqb;
    tc::l_row_item<__half, TO, D, true, false>(out, maps, w.lse, g, (rem - a2 * nqb) * 2 * kTile, a2, bh, smem_raw,
                                              tmem, counters + 1 + bh, n_rg);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (tid < 32) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace monarch
