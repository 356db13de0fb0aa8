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
// One CTA of 1024 threads per KV head; the per-head work is a few hundred
// KB of L2-resident scores, so a single SM per head keeps every selection
// exact and deterministic without grid-wide synchronisation.
#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kThreads = 1024;
constexpr int kCandCap = 2048;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide prefix sum of v (one value per thread); returns the
// thread's prefix and writes the block total to *total.
__device__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nw) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) warp_tot[lane] = w;          // inclusive
  }
  __syncthreads();
  const int before = (warp ? warp_tot[warp - 1] : 0) + x - v;
  *total = warp_tot[nw - 1];
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
  unsigned int hist[256];
  int warp_tot[32];
  int scalar[8];
  unsigned long long cand_key[kCandCap];
  int cand_t[kCandCap];
};

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
anchor_select_kernel(const float* __restrict__ score, float* __restrict__ pooled, int N, int W, int kappa,
                     int n_s, int n_u, int k, int all_anchors, unsigned long long seed, int layer,
                     const T* __restrict__ K, const T* __restrict__ V, T* __restrict__ anc_k,
                     T* __restrict__ anc_v, int* __restrict__ anchor_pos, int* __restrict__ slot_of,
                     double* __restrict__ anc_n2, double* __restrict__ anc_sqrt, float* __restrict__ anc_inv,
                     int* __restrict__ counters,
                     int H, int kp16, int obs_rb, PadList pads) {
  __shared__ SelSmem sm;
  const int h = blockIdx.x;
  const int tid = threadIdx.x;
  // alignment gaps between layout sections are part of the output: zero them
  if (h == 0 && tid < PadList::kMax * 16) {
    const int i = tid / 16, b = tid % 16;
    if (b < pads.len[i]) pads.base[pads.off[i] + b] = 0;
  }
  const int NW = N - W;
  float* pl = pooled + (int64_t)h * N;
  int* flag = slot_of + (int64_t)h * N;       // flags first, slots after compaction

  // 1. pooling (zero padding outside [0, N-W), divide by kappa); the score of
  //    a position is the sum of its observation-row-block partials, in order
  const int half = kappa / 2;
  for (int t = tid; t < N; t += kThreads) {
    if (t < NW) {
      float acc = 0.f;
      for (int d = -half; d <= half; ++d) {
        const int u = t + d;
        if (u >= 0 && u < NW) {
          float s = score[(int64_t)h * N + u];
          for (int rb = 1; rb < obs_rb; ++rb) s += score[((int64_t)rb * H + h) * N + u];
          acc += s;
        }
      }
      pl[t] = acc / (float)kappa;
    }
    flag[t] = (all_anchors || t >= NW) ? 1 : 0;
  }
  __syncthreads();

  if (!all_anchors && n_s > 0) {
    // 2. radix select of the n_s largest pooled scores (32-bit order keys)
    uint32_t prefix = 0;
    int need = n_s;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kThreads) sm.hist[i] = 0;
      __syncthreads();
      const uint32_t mask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
      for (int t = tid; t < NW; t += kThreads) {
        const uint32_t key = order_key(pl[t]);
        if ((key & mask) == (prefix & mask)) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0, digit = 0;
        for (int d = 255; d >= 0; --d) {
          if (cum + (int)sm.hist[d] >= need) { digit = d; break; }
          cum += sm.hist[d];
        }
        sm.scalar[0] = digit;
        sm.scalar[1] = need - cum;
      }
      __syncthreads();
      prefix |= (uint32_t)sm.scalar[0] << shift;
      need = sm.scalar[1];
      __syncthreads();
    }
    // mark keys above the threshold and the first `need` ties in position order
    int taken = 0;
    for (int base = 0; base < NW; base += kThreads) {
      const int t = base + tid;
      uint32_t key = (t < NW) ? order_key(pl[t]) : 0u;
      const int tie = (t < NW && key == prefix) ? 1 : 0;
      int tot;
      const int rank = taken + block_exclusive_scan(tie, sm.warp_tot, &tot);
      if (t < NW && (key > prefix || (tie && rank < need))) flag[t] = 1;
      taken += tot;
    }
    __syncthreads();
  }

  if (!all_anchors && n_u > 0) {
    // 3. uniform sample: the n_u smallest hash keys among unflagged non-window
    //    positions.  A key threshold is chosen so that between n_u and
    //    kCandCap candidates fall below it (bisection on the threshold); the
    //    candidates are then sorted exactly by (key, position).
    const int n_rest = NW - n_s;
    double lo = 0.0, hi = 1.0;
    double frac = fmin(1.0, (n_u + 4.0 * sqrt((double)n_u) + 32.0) / (double)n_rest);
    unsigned long long thr = 0;
    int count = -1, iter = 0;
    for (; iter < 80; ++iter) {
      thr = (frac >= 1.0) ? ~0ull : (unsigned long long)(frac * 18446744073709551616.0);
      if (tid == 0) sm.scalar[2] = 0;
      __syncthreads();
      int local = 0;
      for (int t = tid; t < NW; t += kThreads)
        if (!flag[t] && (frac >= 1.0 || anchor_key(seed, layer, h, t) < thr)) ++local;
      local = __reduce_add_sync(0xffffffffu, local);
      if ((tid & 31) == 0) atomicAdd(&sm.scalar[2], local);
      __syncthreads();
      count = sm.scalar[2];
      __syncthreads();
      if (count >= n_u && count <= kCandCap) break;
      if (count < n_u) lo = frac; else hi = frac;
      frac = 0.5 * (lo + hi);
    }
    if (count < n_u || count > kCandCap) {
      if (tid == 0) latch_error(counters, kDevErrUniform);
      return;
    }
    if (tid == 0 && iter > 0) atomicAdd(&counters[kUniformRetries], iter);
    if (tid == 0) sm.scalar[3] = 0;
    __syncthreads();
    for (int t = tid; t < NW; t += kThreads) {
      if (flag[t]) continue;
      const unsigned long long key = anchor_key(seed, layer, h, t);
      if (frac >= 1.0 || key < thr) {
        const int slot = atomicAdd(&sm.scalar[3], 1);
        sm.cand_key[slot] = key;
        sm.cand_t[slot] = t;
      }
    }
    __syncthreads();
    int P = 1;
    while (P < count) P <<= 1;
    for (int i = count + tid; i < P; i += kThreads) { sm.cand_key[i] = ~0ull; sm.cand_t[i] = 0x7fffffff; }
    __syncthreads();
    // bitonic sort by (key, t)
    for (int size = 2; size <= P; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < P; i += kThreads) {
          const int j = i ^ stride;
          if (j > i) {
            const bool up = ((i & size) == 0);
            const unsigned long long ki = sm.cand_key[i], kj = sm.cand_key[j];
            const int ti = sm.cand_t[i], tj = sm.cand_t[j];
            const bool gt = (ki > kj) || (ki == kj && ti > tj);
            if (gt == up) {
              sm.cand_key[i] = kj; sm.cand_key[j] = ki;
              sm.cand_t[i] = tj; sm.cand_t[j] = ti;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int i = tid; i < n_u; i += kThreads) flag[sm.cand_t[i]] = 1;
    __syncthreads();
  }

  // 4. compaction in position order: slot s <-> anchor_pos[s]
  int taken = 0;
  int* apos = anchor_pos + (int64_t)h * k;
  for (int base = 0; base < N; base += kThreads) {
    const int t = base + tid;
    const int f = (t < N) ? flag[t] : 0;
    int tot;
    const int s = taken + block_exclusive_scan(f, sm.warp_tot, &tot);
    if (t < N) {
      if (f && s < k) apos[s] = t;
      flag[t] = f ? s : -1;
    }
    taken += tot;
  }
  if (tid == 0 && taken != k) latch_error(counters, kDevErrBounds);
  __syncthreads();
  if (taken != k) return;

  // 5. copy anchor rows into the layout; exact fp64 squared norms
  const int warp = tid >> 5, lane = tid & 31;
  for (int s = warp; s < k; s += kThreads / 32) {
    const int t = apos[s];
    for (int side = 0; side < 2; ++side) {
      const T* src = (side ? V : K) + ((int64_t)h * N + t) * kD;
      T* dst = (side ? anc_v : anc_k) + ((int64_t)h * k + s) * kD;
      float f[4];
      load4<T>(src + lane * 4, f);
      for (int e = 0; e < 4; ++e) dst[lane * 4 + e] = src[lane * 4 + e];
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
  for (int i = tid; i < 2 * (kp16 - k); i += kThreads) {
    const int side = i / (kp16 - k), s = k + i % (kp16 - k);
    anc_inv[((int64_t)side * H + h) * kp16 + s] = 0.f;
  }
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
  if (pl.p.dtype == ANCHORKV_BF16) {
    anchor_select_kernel<__nv_bfloat16><<<pl.H, kThreads, 0, s>>>(
        score, pooled, pl.N, pl.W, pl.p.pool_kernel, pl.n_s, pl.n_u, pl.k, pl.all_anchors ? 1 : 0,
        pl.p.seed, pl.p.layer, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
        reinterpret_cast<__nv_bfloat16*>(out + pl.L.off_anchors_k),
        reinterpret_cast<__nv_bfloat16*>(out + pl.L.off_anchors_v), apos, slot_of, n2, sq, inv, cnt, pl.H, pl.kp16, pl.obs_rb, pads);
  } else {
    anchor_select_kernel<float><<<pl.H, kThreads, 0, s>>>(
        score, pooled, pl.N, pl.W, pl.p.pool_kernel, pl.n_s, pl.n_u, pl.k, pl.all_anchors ? 1 : 0,
        pl.p.seed, pl.p.layer, (const float*)K, (const float*)V,
        reinterpret_cast<float*>(out + pl.L.off_anchors_k), reinterpret_cast<float*>(out + pl.L.off_anchors_v),
        apos, slot_of, n2, sq, inv, cnt, pl.H, pl.kp16, pl.obs_rb, pads);
  }
  return cudaGetLastError();
}

}  // namespace akv
