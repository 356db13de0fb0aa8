// Anchor selection: positional pooling, top-n_s by pooled score, uniform
// sample, trailing window, slot order, and the anchor rows copied into the
// compressed layout.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// "Assumptions & free parameters": the final W positions are always anchors;
// a fraction rho = 0.7 of the remaining anchor slots goes to the best pooled
// observation scores (pooling width kappa = 7, Eq. 14), the rest is sampled
// uniformly; k = S/128.  Readings: m = ceil(N/128) non-window slots,
// n_s = floor(7m/10) by score with ties to the lower position, n_u = m - n_s
// as the smallest SplitMix64 keys (seed ^ layer<<48 ^ head<<32 ^ t) among the
// other non-window positions, ties to the lower position; pooling is an
// average with zero padding outside [0, N-W), divided by kappa.
//
// One cluster of kC CTAs per KV head; CTA r owns a contiguous run of
// positions and each thread a contiguous run inside it.  Both selections are
// one cluster-wide radix select over 64-bit keys (smallest first, ties to the
// lower position): per 8-bit digit every CTA builds a warp-aggregated
// histogram of its keys, every CTA sums the kC histograms through
// distributed shared memory and takes the same digit; the select stops as
// soon as the threshold bin holds exactly the keys still needed (uniform
// hash keys need two or three digits).  Ties at the full key are ranked by
// position across the cluster.
#include "cluster_select.cuh"
#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kC = 8;                 // CTAs per head (portable cluster size)
constexpr int kSeg = 4096;            // pooling staging segment

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ void cl_sync() { cluster_barrier(); }

// Exclusive block-wide prefix sum of v (one value per thread); returns the
// thread's prefix and writes the block total to *total.
__device__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kWarps) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) warp_tot[lane] = w;          // inclusive
  }
  __syncthreads();
  const int before = (warp ? warp_tot[warp - 1] : 0) + x - v;
  *total = warp_tot[kWarps - 1];
  __syncthreads();
  return before;
}

struct PadList {
  static constexpr int kMax = 6;
  unsigned char* base;
  int64_t off[kMax];
  int len[kMax];
};

struct SelSmem {
  RadixSmem<kThreads> rs;
  int warp_tot[kWarps];
  int cta_count;                     // this CTA's count exposed to the cluster
  int csum[2];                       // cluster sums of the counts (before this CTA, all)
  float stage[kSeg + 256];           // raw scores of one pooling segment (kappa <= 255)
};

// Flags the selected positions of this thread's run [lo, hi): keys below the
// threshold prefix, and keys equal to it either all or the first `need` in
// position order across the cluster.
template <typename K, typename KeyF>
__device__ void mark_selected(SelSmem& sm, const RadixResult<K>& sr, int lo, int hi, uint8_t* flag, KeyF key) {
  int ties = 0;
  for (int i = lo; i < hi; ++i) {
    K kk;
    if (key(i - lo, kk) && radix_top(kk, sr.bits) == sr.prefix) ++ties;
  }
  int rank0 = 0;
  if (!sr.all_ties) {
    int local_total;
    const int before = block_exclusive_scan(ties, sm.warp_tot, &local_total);
    if (threadIdx.x == 0) sm.cta_count = local_total;
    cl_sync();
    int cta_before = 0, cta_all = 0;
    cluster_sums<kC>(&sm.cta_count, sm.csum, blockIdx.x % kC, cta_before, cta_all);
    rank0 = cta_before + before;
  }
  // keys are read before any flag of this thread changes (the value-sample
  // key excludes flagged positions)
  for (int i = lo; i < hi; ++i) {
    K kk;
    if (!key(i - lo, kk)) continue;
    const K top = radix_top(kk, sr.bits);
    if (top < sr.prefix) {
      flag[i] = 1;
    } else if (top == sr.prefix) {
      if (sr.all_ties || rank0 < sr.need) flag[i] = 1;
      ++rank0;
    }
  }
  __syncthreads();
  cl_sync();   // peers are done reading sm.cta_count / histograms of this select
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
anchor_select_kernel(const float* __restrict__ score, float* __restrict__ pooled, int N, int W, int kappa,
                     int n_s, int n_u, int k, int all_anchors, unsigned long long seed, int layer,
                     const T* __restrict__ K, const T* __restrict__ V, T* __restrict__ anc_k,
                     T* __restrict__ anc_v, int* __restrict__ anchor_pos, int* __restrict__ slot_of,
                     double* __restrict__ anc_n2, double* __restrict__ anc_sqrt, float* __restrict__ anc_inv,
                     int* __restrict__ counters,
                     int H, int kp16, int obs_rb, PadList pads) {
  extern __shared__ __align__(16) unsigned char dsm[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(dsm);
  uint32_t* keys = reinterpret_cast<uint32_t*>(dsm + sizeof(SelSmem));   // pooled order keys of the run
  const unsigned r = blockIdx.x % kC;
  const int h = blockIdx.x / kC;
  const int tid = threadIdx.x;
  // alignment gaps between layout sections are part of the output: zero them
  if (h == 0 && r == 0 && tid < PadList::kMax * 16) {
    const int i = tid / 16, b = tid % 16;
    if (b < pads.len[i]) pads.base[pads.off[i] + b] = 0;
  }
  const int NW = N - W;
  const int per_cta = (N + kC - 1) / kC;
  const int c0 = min(N, (int)r * per_cta), c1 = min(N, c0 + per_cta), np = c1 - c0;
  const int ppt = (np + kThreads - 1) / kThreads;
  const int lo = min(np, tid * ppt), hi = min(np, lo + ppt);         // this thread's run (local)
  float* pl = pooled + (int64_t)h * N;
  uint8_t* flag = reinterpret_cast<uint8_t*>(keys + np);               // [np] anchor flags

  // 1. pooling of [c0, min(c1, NW)) in segments (zero padding outside
  //    [0, N-W), divide by kappa); a position's score is the sum of its
  //    observation-row-block partials, in order
  const int half = kappa / 2;
  const int pend = min(c1, NW);
  for (int sb = c0; sb < pend; sb += kSeg) {
    const int se = min(pend, sb + kSeg);
    // a thread's staging entries u = sb - half + tid + i kThreads, their
    // partials loaded kRB row blocks at a time (all in flight together) and
    // summed in row-block order
    constexpr int kE = (kSeg + 256 + kThreads - 1) / kThreads;
    constexpr int kRB = 4;
    const int ub = sb - half + tid, ue = se + half;
    float acc[kE];
#pragma unroll
    for (int i = 0; i < kE; ++i) acc[i] = 0.f;
    for (int rb0 = 0; rb0 < obs_rb; rb0 += kRB) {
      float part[kE][kRB];
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        const int u = ub + i * kThreads;
        const bool in = u < ue && u >= 0 && u < NW;
#pragma unroll
        for (int q = 0; q < kRB; ++q)
          part[i][q] = (in && rb0 + q < obs_rb) ? score[((int64_t)(rb0 + q) * H + h) * N + u] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kE; ++i)
#pragma unroll
        for (int q = 0; q < kRB; ++q)
          if (rb0 + q < obs_rb) acc[i] = (rb0 + q == 0) ? part[i][q] : acc[i] + part[i][q];
    }
#pragma unroll
    for (int i = 0; i < kE; ++i) {
      const int u = ub + i * kThreads;
      if (u < ue) sm.stage[u - (sb - half)] = (u >= 0 && u < NW) ? acc[i] : 0.f;
    }
    __syncthreads();
    for (int t = sb + tid; t < se; t += kThreads) {
      float acc = 0.f;
      for (int d = -half; d <= half; ++d) {
        const int u = t + d;
        if (u >= 0 && u < NW) acc += sm.stage[u - (sb - half)];
      }
      const float pv = acc / (float)kappa;
      pl[t] = pv;
      keys[t - c0] = ~order_key(pv);                 // smallest key = largest score
    }
    __syncthreads();
  }
  for (int i = tid; i < np; i += kThreads) flag[i] = (all_anchors || c0 + i >= NW) ? 1 : 0;
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
  __syncthreads();

  // 2. the n_s largest pooled scores, ties to the lower position
  if (!all_anchors && n_s > 0) {
    auto key = [&](int j, uint32_t& kk) -> bool {
      const int i = lo + j;
      if (i >= hi || c0 + i >= NW) return false;
      kk = keys[i];
      return true;
    };
    const RadixResult<uint32_t> sr = cluster_radix_select<kThreads, kC, uint32_t>(sm.rs, ppt, n_s, key);
    mark_selected(sm, sr, lo, hi, flag, key);
  }
  // 3. the n_u smallest hash keys among the other non-window positions
  if (!all_anchors && n_u > 0) {
    auto key = [&](int j, uint64_t& kk) -> bool {
      const int i = lo + j;
      if (i >= hi || c0 + i >= NW || flag[i]) return false;
      kk = anchor_key(seed, layer, h, c0 + i);
      return true;
    };
    const RadixResult<uint64_t> sr = cluster_radix_select<kThreads, kC, uint64_t>(sm.rs, ppt, n_u, key);
    mark_selected(sm, sr, lo, hi, flag, key);
  }

  // 4. compaction in position order: slot s <-> anchor_pos[s]
  int cnt = 0;
  for (int i = lo; i < hi; ++i) cnt += flag[i];
  int local_total;
  const int before = block_exclusive_scan(cnt, sm.warp_tot, &local_total);
  if (tid == 0) sm.cta_count = local_total;
  cl_sync();
  int cta_before = 0, all = 0;
  cluster_sums<kC>(&sm.cta_count, sm.csum, r, cta_before, all);
  int* apos = anchor_pos + (int64_t)h * k;
  int* sof = slot_of + (int64_t)h * N;
  int* spos = reinterpret_cast<int*>(keys);   // this CTA's anchor positions (the keys are spent)
  {
    int s = cta_before + before;
    for (int i = lo; i < hi; ++i) {
      if (flag[i]) {
        if (s < k) apos[s] = c0 + i;
        spos[s - cta_before] = c0 + i;
        sof[c0 + i] = s;
        ++s;
      } else {
        sof[c0 + i] = -1;
      }
    }
  }
  if (all != k) {
    if (r == 0 && tid == 0) latch_error(counters, kDevErrBounds);
    cl_sync();
    return;
  }
  __syncthreads();

  // 5. this CTA's anchor rows into the layout; exact fp64 squared norms
  const int warp = tid >> 5, lane = tid & 31;
  const int s_lo = cta_before, s_hi = cta_before + local_total;
  for (int s = s_lo + warp; s < s_hi; s += kWarps) {
    const int t = spos[s - s_lo];
    // both sides' rows in flight together
    T raw[2][4];
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      const T* src = (side ? V : K) + ((int64_t)h * N + t) * kD;
#pragma unroll
      for (int e = 0; e < 4; ++e) raw[side][e] = src[lane * 4 + e];
    }
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      T* dst = (side ? anc_v : anc_k) + ((int64_t)h * k + s) * kD;
      float f[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dst[lane * 4 + e] = raw[side][e];
        f[e] = to_f(raw[side][e]);
      }
      double n2 = 0.0;
      for (int e = 0; e < 4; ++e) n2 += (double)f[e] * (double)f[e];
      n2 = warp_sum_d(n2);
      if (lane == 0) {
        const int64_t ai = ((int64_t)side * H + h) * k + s;
        anc_n2[ai] = n2;
        anc_sqrt[ai] = sqrt(n2);
        anc_inv[((int64_t)side * H + h) * kp16 + s] = (n2 > 0.0) ? (float)(1.0 / sqrt(n2)) : 0.f;
      }
    }
  }
  // 1/||a|| rows are padded to a multiple of 16 slots with zeros
  if (r == 0) {
    for (int i = tid; i < 2 * (kp16 - k); i += kThreads) {
      const int side = i / (kp16 - k), s = k + i % (kp16 - k);
      anc_inv[((int64_t)side * H + h) * kp16 + s] = 0.f;
    }
  }
  cl_sync();   // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

cudaError_t launch_anchor_select(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  auto* score = reinterpret_cast<const float*>(ws + pl.o_score);
  auto* pooled = reinterpret_cast<float*>(ws + pl.o_pooled);
  auto* apos = reinterpret_cast<int*>(out + pl.L.off_anchor_pos);
  auto* slot_of = reinterpret_cast<int*>(ws + pl.o_slot_of);
  auto* n2 = reinterpret_cast<double*>(ws + pl.o_anc_n2);
  auto* inv = reinterpret_cast<float*>(ws + pl.o_anc_inv);
  auto* sq = reinterpret_cast<double*>(ws + pl.o_anc_sqrt);
  auto* cnt = reinterpret_cast<int*>(ws + pl.o_counters);
  // section ends and the next 16-byte boundary
  const int64_t H = pl.H, N = pl.N, k = pl.k, D = kD;
  const int64_t ends[PadList::kMax] = {
      pl.L.off_anchors_k + H * k * D * pl.elem, pl.L.off_anchors_v + H * k * D * pl.elem,
      pl.L.off_anchor_pos + 4 * H * k, pl.L.off_tok + 8 * H * N,
      pl.L.off_bitmap + 2 * H * pl.n_tiles * 16, pl.L.off_tile_prefix + 8 * H * (pl.n_tiles + 1)};
  PadList pads;
  pads.base = reinterpret_cast<unsigned char*>(out);
  for (int i = 0; i < PadList::kMax; ++i) {
    pads.off[i] = ends[i];
    pads.len[i] = (int)((16 - ends[i] % 16) % 16);
  }
  const int per_cta = (int)((N + kC - 1) / kC);
  const size_t smem = sizeof(SelSmem) + (size_t)per_cta * 5;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(pl.H * kC);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  cudaError_t e;
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    auto kern = anchor_select_kernel<T>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&lc, kern, score, pooled, pl.N, pl.W, pl.p.pool_kernel, pl.n_s, pl.n_u, pl.k,
                           pl.all_anchors ? 1 : 0, (unsigned long long)pl.p.seed, pl.p.layer, (const T*)K,
                           (const T*)V, reinterpret_cast<T*>(out + pl.L.off_anchors_k),
                           reinterpret_cast<T*>(out + pl.L.off_anchors_v), apos, slot_of, n2, sq, inv, cnt, pl.H,
                           pl.kp16, pl.obs_rb, pads);
  } else {
    using T = float;
    auto kern = anchor_select_kernel<T>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&lc, kern, score, pooled, pl.N, pl.W, pl.p.pool_kernel, pl.n_s, pl.n_u, pl.k,
                           pl.all_anchors ? 1 : 0, (unsigned long long)pl.p.seed, pl.p.layer, (const T*)K,
                           (const T*)V, reinterpret_cast<T*>(out + pl.L.off_anchors_k),
                           reinterpret_cast<T*>(out + pl.L.off_anchors_v), apos, slot_of, n2, sq, inv, cnt, pl.H,
                           pl.kp16, pl.obs_rb, pads);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace akv
