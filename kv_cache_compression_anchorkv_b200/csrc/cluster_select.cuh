// Cluster-wide radix select, shared by the anchor selection and the top-R
// residual selection.
//
// The `want` smallest keys of a set spread over the C CTAs of a thread-block
// cluster are found digit by digit (8 bits from the top): every warp counts
// its keys that match the prefix found so far in a private histogram (native
// shared-memory integer atomics; with at most 8 keys per thread, straight
// into the CTA histogram), the CTA sums its warps' histograms, every
// CTA sums the C CTA histograms through distributed shared memory and picks
// the same digit.  The select stops as soon as the threshold bin holds
// exactly the keys still needed.  The caller then takes the keys below the
// threshold prefix and, at the threshold, all of them or the first `need` in
// its own tie order.
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

// Sum over the CTAs of the cluster of the int at `p` in each, and the sum over
// the CTAs ranked below this one: one warp reads the peers (lane rr reads CTA
// rr), the results go through `out` ([2]) to the whole CTA.  Call between
// cluster barriers that order the peers' writes of *p before the reads.
template <int C>
__device__ __forceinline__ void cluster_sums(int* p, int* out, unsigned rank, int& before, int& all) {
  static_assert(C <= 32, "one lane per CTA");
  if (threadIdx.x < 32) {
    const unsigned lane = threadIdx.x;
    const int v = lane < (unsigned)C ? *cluster_peer(p, lane) : 0;
    int b = lane < rank ? v : 0, a = v;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      b += __shfl_xor_sync(0xffffffffu, b, o);
      a += __shfl_xor_sync(0xffffffffu, a, o);
    }
    if (lane == 0) { out[0] = b; out[1] = a; }
  }
  __syncthreads();
  before = out[0];
  all = out[1];
}

template <int kThreads>
struct RadixSmem {
  unsigned int whist[kThreads / 32][256];   // per-warp histograms of the current digit
  unsigned int hist[2][256];                // CTA histograms, double-buffered (read by peers)
  unsigned int tot[256];                    // cluster totals of the current digit
  int scal[4];
};

// Keys whose top `bits` bits are below `prefix` are selected; keys equal to
// it are all selected if `all_ties`, else the first `need` in tie order.
template <typename K>
struct RadixResult {
  K prefix;
  int bits;
  int need;
  bool all_ties;
};

template <typename K>
__device__ __forceinline__ K radix_top(K key, int bits) {
  constexpr int kB = 8 * (int)sizeof(K);
  return bits >= kB ? key : (bits ? (K)(key & (~(K)0 << (kB - bits))) : (K)0);
}

// key(j, kk) is called for j in [0, iters) with the same `iters` in every
// thread of the CTA; it returns false for items that take no part.  K is
// uint32_t or uint64_t (all bits significant).  Every thread of every CTA
// returns the same result.  Requires kThreads >= 256.
template <int kThreads, int C, typename K, typename KeyF>
__device__ RadixResult<K> cluster_radix_select(RadixSmem<kThreads>& sm, int iters, int want, KeyF key) {
  static_assert(kThreads >= 256 && kThreads % 32 == 0, "one thread per bin");
  constexpr int kB = 8 * (int)sizeof(K);
  constexpr int kWarps = kThreads / 32;
  const int warp = threadIdx.x >> 5;
  RadixResult<K> res;
  res.prefix = 0;
  res.need = want;
  res.all_ties = false;
  int buf = 0;
  int depth = 0;
  // few keys per thread: count straight into the CTA histogram (no per-warp
  // histograms to clear and add up)
  const bool direct = iters <= 8;
  for (; depth < kB; depth += 8) {
    const int shift = kB - depth - 8;
    if (direct) {
      if (threadIdx.x < 256) sm.hist[buf][threadIdx.x] = 0u;
    } else {
      for (int i = threadIdx.x; i < kWarps * 256; i += kThreads) (&sm.whist[0][0])[i] = 0u;
    }
    __syncthreads();
    unsigned* wh = direct ? sm.hist[buf] : sm.whist[warp];
    for (int j = 0; j < iters; ++j) {
      K kk = 0;
      if (key(j, kk) && radix_top(kk, depth) == res.prefix) atomicAdd(&wh[(unsigned)(kk >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (!direct) {
      if (threadIdx.x < 256) {
        unsigned t = 0;
#pragma unroll 8
        for (int w = 0; w < kWarps; ++w) t += sm.whist[w][threadIdx.x];
        sm.hist[buf][threadIdx.x] = t;
      }
      __syncthreads();
    }
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
    res.prefix |= (K)d << shift;
    res.need -= below;
    __syncthreads();
    buf ^= 1;
    if (cnt == res.need) { res.all_ties = true; depth += 8; break; }
  }
  res.bits = depth;
  return res;
}

}  // namespace akv
