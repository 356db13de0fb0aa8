// Per-layer residual budget: the R largest utilities over all token-sides of
// the layer, as the residual bitmap and per-tile record prefix counts.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary" and minor comment 3: the byte budget left after anchors,
// indices and coefficients buys residuals for the top-ranked token-sides,
// pooled over the heads and both sides of the layer (Eq. 13 reading).
// Readings: eligible token-sides carry utility >= 0 (anchors -1); ties go to
// the lower flat index f = (side * H + head) * N + t.
//
// One launch: a cluster of C CTAs owns contiguous ranges of 128-token tiles
// (tiles of one (side, head) are consecutive, so tile order is flat order).
//  1. cluster radix select of the R largest utilities (keys ~bits(u), read
//     coalesced from L2 on every digit);
//  2. one warp per tile: ballots of "above the threshold" and "at the
//     threshold" per 32-token word, tie counts per tile;
//  3. tie ranks: exclusive scan of the tile tie counts in the CTA plus the
//     ties of the CTAs before it; bitmap words, record counts per tile;
//  4. tile prefixes: exclusive scan of the record counts in the CTA plus the
//     records of the CTAs before it.
#include "cluster_select.cuh"
#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

struct SelectSmem {
  RadixSmem<kThreads> rs;
  int warp_tot[kWarps];
  int scal[4];
  int cta_ties, cta_recs;            // exposed to the cluster
};

// Exclusive scan, in place, of n ints in shared memory (block-wide); returns
// the total.
__device__ int block_scan_inplace(int* v, int n, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + threadIdx.x;
    const int x0 = (i < n) ? v[i] : 0;
    int x = x0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    if (i < n) v[i] = carry + (warp ? warp_tot[warp - 1] : 0) + x - x0;
    carry += warp_tot[kWarps - 1];
    __syncthreads();
  }
  return carry;
}

template <int C>
__global__ void __launch_bounds__(kThreads, 1)
select_kernel(const float* __restrict__ util, int N, int n_t, int n_sh, int R, int take_all, int resident,
              uint32_t* __restrict__ bitmap, int* __restrict__ prefix, int* __restrict__ counters) {
  extern __shared__ __align__(16) unsigned char dsm[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(dsm);
  const unsigned r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_all = n_sh * n_t;
  const int tb = (int)((int64_t)n_all * r / C), te = (int)((int64_t)n_all * (r + 1) / C), nt = te - tb;
  int* tcount = reinterpret_cast<int*>(dsm + sizeof(SelectSmem));    // per tile of this CTA
  // keys of this CTA's slots (slot q: tile tb + q / 128, token q % 128), kept
  // in shared memory when the plan has room for them.  An eligible utility
  // u >= 0 maps to ~bits(u) - 2^31 in [0, 2^31) (smallest first = largest
  // utility), everything else to kNone.
  constexpr uint32_t kNone = 0xFFFFFFFFu;
  // per 32-token word, ballots of the slots at the threshold and above it
  uint32_t* eqw = reinterpret_cast<uint32_t*>(tcount + ((nt + 3) & ~3));   // [4 nt]
  uint32_t* abw = eqw + 4 * nt;                                            // [4 nt]
  uint32_t* keys = resident ? abw + 4 * nt : nullptr;
  auto key_of_u = [](float u) -> uint32_t { return (u >= 0.f) ? (~__float_as_uint(u)) & 0x7FFFFFFFu : kNone; };
  // when N is a multiple of the tile, slot q of this CTA is utility
  // tb * 128 + q (no per-slot division)
  const bool dense = (N % kTile) == 0;
  const float* ub = util + (int64_t)tb * kTile;
  auto key_from_global = [&](int q) -> uint32_t {
    if (dense) return key_of_u(ub[q]);
    const int tile = tb + (q >> 7);
    if (tile >= te) return kNone;
    const int sh = tile / n_t, t = (tile % n_t) * kTile + (q & 127);
    if (t >= N) return kNone;
    return key_of_u(util[(int64_t)sh * N + t]);
  };
  if (resident) {
    const int n = nt * kTile;
    int q = tid;
    if (dense) {
      // four independent loads per thread in flight
      for (; q + 3 * kThreads < n; q += 4 * kThreads) {
        const float u0 = ub[q], u1 = ub[q + kThreads], u2 = ub[q + 2 * kThreads], u3 = ub[q + 3 * kThreads];
        keys[q] = key_of_u(u0);
        keys[q + kThreads] = key_of_u(u1);
        keys[q + 2 * kThreads] = key_of_u(u2);
        keys[q + 3 * kThreads] = key_of_u(u3);
      }
    }
    for (; q < n; q += kThreads) keys[q] = key_from_global(q);
  }
  auto key_of = [&](int q) -> uint32_t { return resident ? keys[q] : key_from_global(q); };
  auto eligible = [&](int, uint32_t k32) -> bool { return k32 != kNone; };
  __syncthreads();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");

  // 1. threshold
  RadixResult<uint32_t> sr;
  sr.prefix = 0; sr.bits = 0; sr.need = 0; sr.all_ties = true;
  if (!take_all) {
    const int iters = (nt * kTile + kThreads - 1) / kThreads;
    auto key = [&](int j, uint32_t& kk) -> bool {
      const int q = j * kThreads + tid;
      if (q >= nt * kTile) return false;
      kk = key_of(q);
      return eligible(q, kk);
    };
    sr = cluster_radix_select<kThreads, C, uint32_t>(sm.rs, iters, R, key);
  }
  // classification of slot q: 2 = above the threshold, 1 = at it
  auto cls = [&](int q) -> int {
    const uint32_t k32 = key_of(q);
    if (!eligible(q, k32)) return 0;
    if (take_all) return 2;
    const uint32_t top = radix_top(k32, sr.bits);
    return top < sr.prefix ? 2 : (top == sr.prefix ? 1 : 0);
  };

  // 2. one warp per tile: ballots of "at the threshold" and "above it" per
  //    32-token word, kept in shared memory; tie counts per tile
  uint32_t eqv[4], abv[4];
  for (int i = warp; i < nt; i += kWarps) {
    int eq = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int c = cls(i * kTile + w * 32 + lane);
      eqv[w] = __ballot_sync(0xffffffffu, c == 1);
      abv[w] = __ballot_sync(0xffffffffu, c == 2);
      eq += __popc(eqv[w]);
    }
    __syncwarp();
    if (lane == 0) {
      tcount[i] = eq;
#pragma unroll
      for (int w = 0; w < 4; ++w) { eqw[4 * i + w] = eqv[w]; abw[4 * i + w] = abv[w]; }
    }
  }
  __syncthreads();
  const int ties = block_scan_inplace(tcount, nt, sm.warp_tot);
  if (tid == 0) sm.cta_ties = ties;
  cluster_barrier();
  int ties_before = 0, ties_all = 0;
  cluster_sums<C>(&sm.cta_ties, sm.scal, r, ties_before, ties_all);
  if (r == 0 && tid == 0 && !take_all && !sr.all_ties && ties_all > 0) atomicAdd(&counters[kSelectTies], ties_all);

  // 3. one thread per bitmap word: the words above the threshold, and of the
  //    words at it the first `need` bits over the cluster in flat order
  //    (lowest bit = lowest token); record counts per tile
  for (int x = tid; x < 4 * nt; x += kThreads) {
    const int i = x >> 2, w = x & 3;
    const uint32_t eq = eqw[x];
    uint32_t sel = eq;
    if (!sr.all_ties && eq) {
      int rank = ties_before + tcount[i];
      for (int v = 0; v < w; ++v) rank += __popc(eqw[4 * i + v]);
      const int n = min(max(sr.need - rank, 0), __popc(eq));
      if (n < __popc(eq)) {
        const int pos = n ? (int)__fns(eq, 0, n) : -1;     // the n-th set bit
        sel = pos < 0 ? 0u : (pos == 31 ? eq : eq & ((2u << pos) - 1u));
      }
    }
    const uint32_t sb = abw[x] | sel;
    bitmap[(int64_t)(tb + i) * 4 + w] = sb;
    abw[x] = (uint32_t)__popc(sb);     // only this thread reads abw[x]
  }
  __syncthreads();
  for (int i = tid; i < nt; i += kThreads) tcount[i] = (int)(abw[4 * i] + abw[4 * i + 1] + abw[4 * i + 2] + abw[4 * i + 3]);
  __syncthreads();

  // 4. tile prefixes [n_sh][n_t + 1]; entry n_t of (side, head) sh is the
  //    start of sh + 1, the last one the layer's total
  const int recs = block_scan_inplace(tcount, nt, sm.warp_tot);
  if (tid == 0) sm.cta_recs = recs;
  cluster_barrier();
  int recs_before = 0, recs_all = 0;
  cluster_sums<C>(&sm.cta_recs, sm.scal + 2, r, recs_before, recs_all);
  for (int i = tid; i < nt; i += kThreads) {
    const int tile = tb + i, sh = tile / n_t, j = tile % n_t;
    const int v = recs_before + tcount[i];
    prefix[sh * (n_t + 1) + j] = v;
    if (j == 0 && sh > 0) prefix[(sh - 1) * (n_t + 1) + n_t] = v;
  }
  if (r == C - 1 && tid == 0) prefix[(n_sh - 1) * (n_t + 1) + n_t] = recs_before + recs;
  cluster_barrier();   // no CTA leaves while a peer may still read its shared memory
}

template <int C>
cudaError_t launch_c(const Plan& pl, uint32_t* bitmap, int* prefix, const float* util, int* cnt, cudaStream_t s,
                     size_t smem, int resident) {
  auto kern = select_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return cudaErrorNotSupported;
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(C);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (C > 8) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &lc) != cudaSuccess || n < 1) {
      cudaGetLastError();
      return cudaErrorNotSupported;
    }
  }
  return cudaLaunchKernelEx(&lc, kern, util, pl.N, pl.n_tiles, 2 * pl.H, (int)pl.R, pl.R == pl.cap ? 1 : 0,
                            resident, bitmap, prefix, cnt);
}

}  // namespace

cudaError_t launch_select(const Plan& pl, char* out, char* ws, cudaStream_t s) {
  const int n_sh = 2 * pl.H, n_t = pl.n_tiles;
  auto* util = reinterpret_cast<const float*>(ws + pl.o_util);
  auto* cnt = reinterpret_cast<int*>(ws + pl.o_counters);
  auto* bitmap = reinterpret_cast<uint32_t*>(out + pl.L.off_bitmap);
  auto* prefix = reinterpret_cast<int*>(out + pl.L.off_tile_prefix);
  if (pl.R == 0) {
    cudaError_t e = cudaMemsetAsync(bitmap, 0, (size_t)n_sh * n_t * 16, s);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(prefix, 0, (size_t)n_sh * (n_t + 1) * 4, s);
  }
  // a 16-CTA cluster where the device schedules one, else 8; the keys stay in
  // shared memory when they fit
  static int use16 = -1;
  const int n_all = n_sh * n_t;
  auto plan = [&](int C, int* resident) -> size_t {
    const int tiles = (n_all + C - 1) / C;
    const size_t base = sizeof(SelectSmem) + 4 * (size_t)((tiles + 3) & ~3) + 32 * (size_t)tiles;
    const size_t with_keys = base + 4 * (size_t)tiles * kTile;
    *resident = with_keys <= 227 * 1024 ? 1 : 0;
    return *resident ? with_keys : base;
  };
  int res16 = 0, res8 = 0;
  const size_t smem16 = plan(16, &res16), smem8 = plan(8, &res8);
  if (use16 != 0 && smem16 <= 227 * 1024) {
    const cudaError_t e = launch_c<16>(pl, bitmap, prefix, util, cnt, s, smem16, res16);
    if (e == cudaSuccess) { use16 = 1; return e; }
    if (e != cudaErrorNotSupported) return e;
    use16 = 0;
  }
  if (smem8 > 227 * 1024) return cudaErrorNotSupported;
  return launch_c<8>(pl, bitmap, prefix, util, cnt, s, smem8, res8);
}

}  // namespace akv
