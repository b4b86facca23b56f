// det_order.cuh -- sequencing of the dQ reduce-adds for the deterministic backward.
//
// dQ is the one output that many CTAs add into (every key tile that a query tile
// attends to contributes a partial dQ for it, as fp32 bulk reduce-adds into the
// accumulator).  Floating-point addition is not associative, so the default backward's
// dQ depends on the order in which those CTAs happen to finish.  In deterministic mode
// the contributions to each (batch, query head, query tile, dQ column part) are added
// in descending key-tile order: a CTA waits until a counter equals the number of the
// query tile's active key tiles above its own, adds both 64-row halves, waits for its
// adds to complete and increments the counter.  The grid is launched from the last key
// tile down in this mode, so a CTA only waits for CTAs launched before it (the waits
// cannot form a cycle).  In this mode every CTA also walks its query tiles in
// ascending order (the full and partial lists merged), so the CTA of key tile n reaches
// a query tile about one step after the CTA of key tile n+1 and the turns mostly arrive
// on time.  Every wait is bounded all the same.
#pragma once

#include "sa_device.cuh"
#include "sa_kernels.h"

namespace sa {

// Turn of key tile nt on query tile mt of (b, kv head) row bg: the number of the query
// tile's active key tiles above nt, from the forward lists (full tiles ascending, then
// partial tiles ascending): two binary searches.
__device__ __forceinline__ int key_tile_rank(const AttnArgs& a, int64_t bg, int mt, int nt) {
  const int64_t row = bg * a.Tm + mt;
  const int nf = __ldg(a.cnt + 2 * row), np = __ldg(a.cnt + 2 * row + 1);
  const int32_t* lst = a.idx + row * a.Tn;
  auto lower = [&](const int32_t* v, int n) {
    int lo = 0, hi = n;
    while (lo < hi) {  // first entry above nt
      const int mid = (lo + hi) >> 1;
      if (__ldg(v + mid) <= nt) lo = mid + 1; else hi = mid;
    }
    return lo;
  };
  return (nf - lower(lst, nf)) + (np - lower(lst + nf, np));
}

// The k-th smallest query tile of a key tile's lists (full tiles L[0, nf) ascending,
// partial tiles L[nf, nf + np) ascending, disjoint): a merge-path binary search for the
// number i of full tiles among the k smallest.
__device__ __forceinline__ void merged_tile(const int32_t* L, int nf, int np, int k, int& tile,
                                            bool& partial) {
  int lo = max(0, k - np), hi = min(k, nf);
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(L + mid) < __ldg(L + nf + k - mid - 1)) lo = mid + 1; else hi = mid;
  }
  const int j = k - lo;
  const bool from_full = lo < nf && (j >= np || __ldg(L + lo) < __ldg(L + nf + j));
  tile = from_full ? __ldg(L + lo) : __ldg(L + nf + j);
  partial = !from_full;
}

__device__ __forceinline__ int32_t* det_slot(const AttnArgs& a, int b, int h, int mt, int part) {
  return a.sem + ((static_cast<int64_t>(b) * a.HQ + h) * a.Tm + mt) * 2 + part;
}

// Waits until the counter equals `rank` (bounded); then orders the caller's following
// TMA reduce-adds after the acquire.  False on a timeout or an abort.
__device__ __forceinline__ bool det_wait_turn(const int32_t* slot, int rank, volatile WaitCtl* ctl,
                                              int32_t* status, uint64_t limit) {
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(slot) != rank) {
    if (ctl->abort) return false;
    if (limit < kShortLimitNs || globaltimer_ns() - t0 > limit) {
      wait_timed_out(ctl, status);
      return false;
    }
    __nanosleep(128);
  }
  fence_proxy_async_global();
  return true;
}

// After the caller's last reduce-add of its turn: wait for the adds to complete, then
// pass the turn on.
__device__ __forceinline__ void det_pass_turn(int32_t* slot) {
  bulk_wait_group0();
  fence_proxy_async_global();
  red_release_gpu_add(slot, 1);
}

}  // namespace sa
