// Cluster-wide radix select over 64-bit keys, shared by the anchor selection
// and the top-R residual selection.
//
// The `want` smallest keys of a set spread over the C CTAs of a thread-block
// cluster are found digit by digit (8 bits from the top): every CTA builds a
// histogram of its keys that match the prefix found so far (one shared-memory
// atomic per distinct bin of a warp), every CTA sums the C histograms through
// distributed shared memory and picks the same digit.  The select stops as
// soon as the threshold bin holds exactly the keys still needed.  The caller
// then takes the keys below the threshold prefix and, at the threshold, all
// of them or the first `need` in its own tie order.
#pragma once

#include "common.cuh"

namespace akv {

// Hardware cluster barrier with release/acquire ordering of shared memory.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Generic pointer to the same shared-memory object in CTA `rank` of the cluster.
template <typename U>
__device__ __forceinline__ U* cluster_peer(U* p, unsigned rank) {
  return static_cast<U*>(__cluster_map_shared_rank(p, rank));
}

struct RadixSmem {
  unsigned int hist[2][256];   // double-buffered local digit histograms
  unsigned int tot[256];       // cluster totals of the current digit
  int scal[4];
};

// Keys whose top `bits` bits are below `prefix` are selected; keys equal to
// it are all selected if `all_ties`, else the first `need` in tie order.
struct RadixResult {
  uint64_t prefix;
  int bits;
  int need;
  bool all_ties;
};

__device__ __forceinline__ uint64_t radix_top(uint64_t key, int bits) {
  return bits >= 64 ? key : (bits ? key & (~0ull << (64 - bits)) : 0ull);
}

// key(j, kk) is called for j in [0, iters) with the same `iters` in every
// thread of the CTA; it returns false for items that take no part.  Keys have
// `key_bits` significant bits from the top.  Every thread of every CTA
// returns the same result.  Requires kThreads >= 256.
template <int kThreads, int C, typename KeyF>
__device__ RadixResult cluster_radix_select(RadixSmem& sm, int iters, int want, int key_bits, KeyF key) {
  static_assert(kThreads >= 256 && kThreads % 32 == 0, "one thread per bin");
  RadixResult res;
  res.prefix = 0;
  res.need = want;
  res.all_ties = false;
  int buf = 0;
  int depth = 0;
  for (; depth < key_bits; depth += 8) {
    const int shift = 64 - depth - 8;
    for (int i = threadIdx.x; i < 256; i += kThreads) sm.hist[buf][i] = 0u;
    __syncthreads();
    for (int j = 0; j < iters; ++j) {
      uint64_t kk = 0;
      const bool take = key(j, kk) && radix_top(kk, depth) == res.prefix;
      const unsigned bin = take ? (unsigned)((kk >> shift) & 255u) : 256u;
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (take && (int)(threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&sm.hist[buf][bin], (unsigned)__popc(same));
    }
    __syncthreads();
    cluster_barrier();
    if (threadIdx.x < 256) {
      unsigned t = 0;
      for (unsigned rr = 0; rr < (unsigned)C; ++rr) t += cluster_peer(&sm.hist[buf][0], rr)[threadIdx.x];
      sm.tot[threadIdx.x] = t;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // digit: the smallest d with sum_{b <= d} tot[b] >= need (8 bins per lane)
      const int lane = threadIdx.x;
      unsigned part = 0;
      for (int b = 0; b < 8; ++b) part += sm.tot[lane * 8 + b];
      unsigned incl = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned excl = incl - part;
      if (excl < (unsigned)res.need && incl >= (unsigned)res.need) {
        unsigned below = excl;
        int d = lane * 8;
        while (below + sm.tot[d] < (unsigned)res.need) { below += sm.tot[d]; ++d; }
        sm.scal[0] = d;
        sm.scal[1] = (int)below;
        sm.scal[2] = (int)sm.tot[d];
      }
    }
    __syncthreads();
    const int d = sm.scal[0], below = sm.scal[1], cnt = sm.scal[2];
    res.prefix |= (uint64_t)d << shift;
    res.need -= below;
    __syncthreads();
    buf ^= 1;
    if (cnt == res.need) { res.all_ties = true; depth += 8; break; }
  }
  res.bits = depth;
  return res;
}

}  // namespace akv
