// Observation-window statistics on the 5th-generation tensor cores (bf16).
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// "What carries the argument" / "Assumptions & free parameters": the last W
// queries of every query head of a KV head attend over the prefill; their
// attention scores positions (SnapKV-style, Eq. 14) and, with the exact
// attention outputs ybar_r, gives the first-order residual utilities (Eq. 6
// reading).  Per KV head h and block of 128 observation rows:
//
//   pass A  S  = Q K^T  (rows x tokens)   -> per row max and sum of exp2
//   rows       M_r, 1/Z_r, ||q_r||^2 from the pass-A partials (fixed order)
//   pass B  S^T = K Q^T (tokens x rows)   -> alpha = e^(s - M_r)/Z_r per token
//           (sum_r alpha, sum_r alpha^2 in registers), alpha stored as bf16
//           hi + lo in shared memory, ybar^T += V^T alpha on the tensor cores
//   ybar       ybar = sum of the pass-B partials (fixed order), hi/lo bf16
//   pass C  S^T = K Q^T and VY^T = V (ybar_hi + ybar_lo)^T -> per token
//           sum_r alpha^2 ||q_r||^2 (||V_t||^2 - 2 V_t.ybar_r + ||ybar_r||^2)
//
// Row constants are global before passes B and C, so no online rescaling is
// needed.  All operands are bf16 (K, V, Q exact; alpha and ybar split into
// two bf16 terms, error 2^-17 relative), accumulators fp32 in TMEM, exp via
// ex2.approx in the log2 domain.  Warp roles: warp 0 TMA, warp 1 TMEM owner
// + MMA issuer, warps 2..17 epilogue in four column groups of four warps (one
// TMEM lane = one row or token per thread, each group a quarter of the
// accumulator's 128 columns, so 32 values per thread and tile and four warps
// per scheduler to hide the latency of the exp2 chains).  Pass A's groups
// split the tokens of a tile and leave separate (max, sum) partials; passes B
// and C's groups split the observation rows, so their per-token sums are
// written as four row blocks per 128-row block.  Per-row constants are folded
// into the exp2 argument (log2 of the scale factors), the arithmetic runs on
// packed fp32 pairs, and the window mask is applied only on the tiles that
// reach into the window.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace akv {

namespace {

constexpr int kOp = 128 * 256;                 // one [128][128] bf16 operand tile
constexpr int kHalf = kOp / 2;                 // its 64-column swizzled half
constexpr int kGroups = kObsGroups;            // epilogue column groups (32 columns each)
constexpr int kEpi = 128 * kGroups;            // epilogue threads
constexpr int kThr = 64 + kEpi;
constexpr float kLog2e = 1.4426950408889634f;

struct ObsTc {
  int N, H, G, W, GW, n_rb, n_split, tps, row_tiles;   // part_m2/part_l hold kGroups * n_split partials per unit
  float c2;                                     // log2(e) / sqrt(D)
  float* part_m2;                               // [U][n_split][128]
  float* part_l;
  const float* row_m2;                          // [U][128]
  const float* row_iz;
  const float* row_q2;
  const float* row_y2;
  float* score;                                 // [kGroups n_rb][H][N] (row block rb, group g at kGroups rb + g)
  float* a2s;
  float* kus;
  float* part_y;                                // [U][n_split][128 rows][128 d]
  float* xnorm;                                 // [2][H][N]
  int* counters;
};

struct Item {
  int u, h, rb, s, tile0, n;
};

__device__ __forceinline__ Item item_of(const ObsTc& a) {
  Item it;
  it.u = blockIdx.x / a.n_split;
  it.s = blockIdx.x % a.n_split;
  it.h = it.u / a.n_rb;
  it.rb = it.u % a.n_rb;
  it.tile0 = it.s * a.tps;
  it.n = max(0, min(a.row_tiles, it.tile0 + a.tps) - it.tile0);
  return it;
}

// last position observation row rr may see (-1 for padding rows)
__device__ __forceinline__ int row_limit(const ObsTc& a, int rr) {
  return rr < a.GW ? a.N - a.W + rr % a.W : -1;
}

__device__ __forceinline__ uint64_t kdesc(const unsigned char* tile, int kk) {
  return tc::sw128_desc(tc::smem_u32(tile) + (uint32_t)((kk >> 2) * kHalf + (kk & 3) * 32));
}

__device__ __forceinline__ void load_op(unsigned char* dst, const CUtensorMap* m, int row, uint64_t* bar) {
  tc::tma_load_2d(dst, m, 0, row, bar);
  tc::tma_load_2d(dst + kHalf, m, 64, row, bar);
}

__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t (&v)[2][16]) {
  tc::tmem_ld16(taddr + 0, v[0]);
  tc::tmem_ld16(taddr + 16, v[1]);
  tc::tmem_wait_ld_dep2(v[0], v[1]);
}

__device__ __forceinline__ float2 f2(uint32_t x, uint32_t y) { return make_float2(__uint_as_float(x), __uint_as_float(y)); }
__device__ __forceinline__ float2 ex2x2(float2 x) { return make_float2(tc::ex2_approx(x.x), tc::ex2_approx(x.y)); }
constexpr uint32_t kNegInf = 0xFF800000u;

template <typename U>
__device__ __forceinline__ float* align16f(U* p) {
  return reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(p) + 15) & ~static_cast<uintptr_t>(15));
}

__device__ __forceinline__ unsigned char* aligned_base(unsigned char* raw) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Sum of squares of the 64 columns of half `part` of token row r of a
// swizzled [128][128] bf16 tile.  The chunk order inside the row does not
// matter for a norm, so the row reads its 16-byte chunks in the order
// c ^ (r & 7) ^ 4 part: the quarter-warp (4 rows x 2 halves, the rows 4-aligned)
// then hits 8 different bank groups.
__device__ __forceinline__ float half_sumsq(const unsigned char* tile, int r, int part) {
  float2 s = make_float2(0.f, 0.f);
  const uint4* p = reinterpret_cast<const uint4*>(tile + part * kHalf + r * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 q = p[c ^ (r & 7) ^ (part << 2)];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = f2(w[e] << 16, w[e] & 0xFFFF0000u);
      s = __ffma2_rn(x, x, s);
    }
  }
  return s.x + s.y;
}

// ============================================================== pass A

struct CtlA {
  uint64_t q_full, x_full[4], x_empty[4], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int err;
};

__global__ void __launch_bounds__(kThr, 1)
obs_a_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK, ObsTc a) {
  extern __shared__ unsigned char smem_raw[];
  constexpr int S = 4;
  unsigned char* q = aligned_base(smem_raw);
  unsigned char* xs = q + kOp;
  CtlA& ctl = *reinterpret_cast<CtlA*>(xs + S * kOp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Item it = item_of(a);
  if (threadIdx.x == 0) {
    tc::mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < S; ++s) { tc::mbar_init(&ctl.x_full[s], 1); tc::mbar_init(&ctl.x_empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&ctl.acc_full[b], 1); tc::mbar_init(&ctl.acc_empty[b], kEpi); }
    tc::mbar_init(&ctl.drain, 1);
    ctl.err = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) { tc::tmem_alloc(&ctl.tmem_base, 256); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tc::mbar_expect_tx(&ctl.q_full, kOp);
      load_op(q, &mapQ, it.h * a.GW + it.rb * 128, &ctl.q_full);
      int issued = 0;
      for (int i = 0; i < it.n && !ctl.err; ++i) {
        const int s = i % S, use = i / S;
        if (use > 0 && !tc::wait_or_fail(&ctl.x_empty[s], (use - 1) & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
        tc::mbar_expect_tx(&ctl.x_full[s], kOp);
        load_op(xs + s * kOp, &mapK, it.h * a.N + (it.tile0 + i) * 128, &ctl.x_full[s]);
        ++issued;
      }
      for (int s = 0; s < S && s < issued; ++s) tc::mbar_wait(&ctl.x_full[s], ((issued - 1 - s) / S) & 1);
      tc::mbar_wait(&ctl.q_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, 128);
      if (tc::wait_or_fail(&ctl.q_full, 0, &ctl.err, a.counters, kDevErrTimeout)) {
        for (int i = 0; i < it.n; ++i) {
          const int s = i % S, use = i / S, b = i & 1, ub = i >> 1;
          if (!tc::wait_or_fail(&ctl.x_full[s], use & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
          if (ub > 0 && !tc::wait_or_fail(&ctl.acc_empty[b], (ub - 1) & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_bf16(tmem + b * 128, kdesc(q, kk), kdesc(xs + s * kOp, kk), idesc, kk > 0);
          tc::mma_commit(&ctl.acc_full[b]);
          tc::mma_commit(&ctl.x_empty[s]);
        }
      }
      tc::mma_commit(&ctl.drain);
      tc::mbar_wait(&ctl.drain, 0);
    }
  } else {
    // group g takes tokens 32 g .. 32 g + 31 of every tile
    const int qd = warp & 3, g = (warp - 2) >> 2, r = qd * 32 + lane;
    const int lim = row_limit(a, it.rb * 128 + r);
    const float2 cc = make_float2(a.c2, a.c2);
    float m = -INFINITY, l = 0.f;
    for (int i = 0; i < it.n; ++i) {
      const int b = i & 1, ub = i >> 1;
      if (!tc::wait_or_fail(&ctl.acc_full[b], ub & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
      tc::fence_after_sync();
      uint32_t v[2][16];
      ld32(tmem + ((uint32_t)(qd * 32) << 16) + b * 128 + g * 32, v);
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl.acc_empty[b]);
      const int t0 = (it.tile0 + i) * 128 + g * 32;
      if (lim < t0) continue;                       // nothing visible (or padding row)
      if (t0 + 31 > lim) {                          // the window's edge: hidden scores -> -inf
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (t0 + e > lim) v[e >> 4][e & 15] = kNegInf;
      }
      // the maximum of the raw scores (c2 > 0 commutes with it)
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 32; ++e) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(v[e >> 4][e & 15]));
      const float mn = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * a.c2);
      const float2 nm = make_float2(-mn, -mn);
      float2 sum0 = make_float2(0.f, 0.f), sum1 = sum0;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const uint32_t* w = &v[e >> 4][e & 15];
        sum0 = __fadd2_rn(sum0, ex2x2(__ffma2_rn(f2(w[0], w[1]), cc, nm)));
        sum1 = __fadd2_rn(sum1, ex2x2(__ffma2_rn(f2(w[2], w[3]), cc, nm)));
      }
      l = l * tc::ex2_approx(m - mn) + ((sum0.x + sum0.y) + (sum1.x + sum1.y));
      m = mn;
    }
    const int64_t pi = ((int64_t)it.u * kGroups * a.n_split + kGroups * it.s + g) * 128 + r;
    a.part_m2[pi] = m;
    a.part_l[pi] = l;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) { tc::fence_after_sync(); tc::tmem_dealloc(tmem, 256); }
}

// Row constants: M_r (log2 domain), 1/Z_r and ||q_r||^2.  grid (U, 16),
// 256 threads: one warp per row, the lanes striding over the row's pass-A
// partials (merged in a fixed order: lane-strided, then a fixed butterfly)
// and over its 128 query coordinates.
__global__ void __launch_bounds__(256) obs_rows_kernel(const __nv_bfloat16* __restrict__ Q, ObsTc a,
                                                       float* __restrict__ row_m2, float* __restrict__ row_iz,
                                                       float* __restrict__ row_q2) {
  const int u = blockIdx.x, lane = threadIdx.x & 31, r = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int h = u / a.n_rb, rb = u % a.n_rb, rr = rb * 128 + r;
  const int np = kGroups * a.n_split;
  float M = -INFINITY;
  for (int s = lane; s < np; s += 32) M = fmaxf(M, a.part_m2[((int64_t)u * np + s) * 128 + r]);
  M = warp_max(M);
  float Z = 0.f;
  for (int s = lane; s < np; s += 32) {
    const int64_t pi = ((int64_t)u * np + s) * 128 + r;
    if (a.part_m2[pi] > -INFINITY) Z = fmaf(a.part_l[pi], exp2f(a.part_m2[pi] - M), Z);
  }
  Z = warp_sum(Z);
  float q2 = 0.f;
  if (rr < a.GW) {
    float f[4];
    load4<__nv_bfloat16>(Q + ((int64_t)h * a.GW + rr) * kD + lane * 4, f);
    q2 = f[0] * f[0] + f[1] * f[1] + f[2] * f[2] + f[3] * f[3];
  }
  q2 = warp_sum(q2);
  if (lane == 0) {
    const int64_t o = (int64_t)u * 128 + r;
    const bool live = rr < a.GW && Z > 0.f;
    row_m2[o] = live ? M : 0.f;
    row_iz[o] = live ? 1.f / Z : 0.f;
    row_q2[o] = q2;
  }
}

// ============================================================== pass B

struct CtlB {
  uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], s_empty[2], al_full, al_empty, y_full,
      drain;
  uint32_t tmem_base;
  int err;
};

__global__ void __launch_bounds__(kThr, 1)
obs_b_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
             const __grid_constant__ CUtensorMap mapV, ObsTc a) {
  extern __shared__ unsigned char smem_raw[];
  constexpr int S = 2;
  unsigned char* q = aligned_base(smem_raw);
  unsigned char* xs = q + kOp;                   // stage s: K at xs + 2s kOp, V at + kOp
  unsigned char* al = xs + S * 2 * kOp;          // alpha hi at al, lo at al + kOp (MN-major)
  CtlB& ctl = *reinterpret_cast<CtlB*>(al + 2 * kOp);
  float* cb = align16f(&ctl + 1);                // log2(1/Z_r) - M_r, 16-byte aligned for float4 reads
  int* clim = reinterpret_cast<int*>(cb + 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Item it = item_of(a);
  if (threadIdx.x == 0) {
    tc::mbar_init(&ctl.q_full, 1);
    // a K stage is free once its S MMA is done and the epilogue has read the
    // tile's norms (kEpi arrivals + the MMA's commit); a V stage once its Y MMA is
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&ctl.k_full[s], 1); tc::mbar_init(&ctl.k_empty[s], kEpi + 1);
      tc::mbar_init(&ctl.v_full[s], 1); tc::mbar_init(&ctl.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&ctl.s_full[b], 1); tc::mbar_init(&ctl.s_empty[b], kEpi); }
    tc::mbar_init(&ctl.al_full, kEpi);
    tc::mbar_init(&ctl.al_empty, 1);
    tc::mbar_init(&ctl.y_full, 1);
    tc::mbar_init(&ctl.drain, 1);
    ctl.err = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) { tc::tmem_alloc(&ctl.tmem_base, 512); tc::tmem_relinquish(); }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + 128) {
    // alpha = 2^(s c2 - M_r) / Z_r = 2^(s c2 + cb_r); padding rows (1/Z = 0) get -inf
    const int r = threadIdx.x - 64;
    cb[r] = log2f(a.row_iz[(int64_t)it.u * 128 + r]) - a.row_m2[(int64_t)it.u * 128 + r];
    clim[r] = row_limit(a, it.rb * 128 + r);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;
  const uint32_t ycol = 256;

  if (warp == 0) {
    if (lane == 0) {
      tc::mbar_expect_tx(&ctl.q_full, kOp);
      load_op(q, &mapQ, it.h * a.GW + it.rb * 128, &ctl.q_full);
      // K and V in separate rings, K one tile ahead: tile i + 1's K goes out
      // before tile i's V, so the S MMA of the next tile never waits behind
      // the Y MMA of the current one
      int kissued = 0, vissued = 0;
      for (int i = 0; i <= it.n && !ctl.err; ++i) {
        if (i < it.n) {
          const int s = i % S, use = i / S;
          if (use > 0 && !tc::wait_or_fail(&ctl.k_empty[s], (use - 1) & 1, &ctl.err, a.counters, kDevErrTimeout))
            break;
          tc::mbar_expect_tx(&ctl.k_full[s], kOp);
          load_op(xs + 2 * s * kOp, &mapK, it.h * a.N + (it.tile0 + i) * 128, &ctl.k_full[s]);
          ++kissued;
        }
        if (i >= 1) {
          const int j = i - 1, s = j % S, use = j / S;
          if (use > 0 && !tc::wait_or_fail(&ctl.v_empty[s], (use - 1) & 1, &ctl.err, a.counters, kDevErrTimeout))
            break;
          tc::mbar_expect_tx(&ctl.v_full[s], kOp);
          load_op(xs + 2 * s * kOp + kOp, &mapV, it.h * a.N + (it.tile0 + j) * 128, &ctl.v_full[s]);
          ++vissued;
        }
      }
      for (int s = 0; s < S && s < kissued; ++s) tc::mbar_wait(&ctl.k_full[s], ((kissued - 1 - s) / S) & 1);
      for (int s = 0; s < S && s < vissued; ++s) tc::mbar_wait(&ctl.v_full[s], ((vissued - 1 - s) / S) & 1);
      tc::mbar_wait(&ctl.q_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16_f32(128, 128);
      const uint32_t id2 = tc::idesc_bf16_f32_major(128, 128, 1, 1);
      bool ok = tc::wait_or_fail(&ctl.q_full, 0, &ctl.err, a.counters, kDevErrTimeout);
      auto mma1 = [&](int i) -> bool {
        const int s = i % S, use = i / S, b = i & 1, ub = i >> 1;
        if (!tc::wait_or_fail(&ctl.k_full[s], use & 1, &ctl.err, a.counters, kDevErrTimeout)) return false;
        if (ub > 0 && !tc::wait_or_fail(&ctl.s_empty[b], (ub - 1) & 1, &ctl.err, a.counters, kDevErrTimeout))
          return false;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + b * 128, kdesc(xs + 2 * s * kOp, kk), kdesc(q, kk), id1, kk > 0);
        tc::mma_commit(&ctl.s_full[b]);
        tc::mma_commit(&ctl.k_empty[s]);      // with the epilogue's arrivals, frees the K stage
        return true;
      };
      if (ok && it.n > 0) ok = mma1(0);
      for (int i = 0; ok && i < it.n; ++i) {
        if (i + 1 < it.n && !mma1(i + 1)) break;
        if (!tc::wait_or_fail(&ctl.al_full, i & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
        if (!tc::wait_or_fail(&ctl.v_full[i % S], (i / S) & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
        tc::fence_after_sync();
        const uint32_t vaddr = tc::smem_u32(xs + 2 * (i % S) * kOp + kOp);
        const uint32_t hi = tc::smem_u32(al), lo = tc::smem_u32(al + kOp);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da = tc::sw128_mn_desc(vaddr + kk * 2048, kHalf);
          tc::mma_bf16(tmem + ycol, da, tc::sw128_mn_desc(hi + kk * 2048, kHalf), id2, (i > 0 || kk > 0) ? 1u : 0u);
          tc::mma_bf16(tmem + ycol, da, tc::sw128_mn_desc(lo + kk * 2048, kHalf), id2, 1u);
        }
        tc::mma_commit(&ctl.al_empty);
        tc::mma_commit(&ctl.v_empty[i % S]);
      }
      tc::mma_commit(&ctl.y_full);
      tc::mma_commit(&ctl.drain);
      tc::mbar_wait(&ctl.drain, 0);
    }
  } else {
    // group g takes observation rows 32 g .. 32 g + 31 of every token
    const int qd = warp & 3, g = (warp - 2) >> 2, tl = qd * 32 + lane;
    const int rb4 = kGroups * it.rb + g;
    // norm work: epilogue thread e takes half (e & 1) of row (e >> 1) & 127 of
    // the K (e < 256) or V tile
    const int ne = threadIdx.x - 64, nrow = (ne >> 1) & 127, nside = ne >> 8, npart = ne & 1;
    const float2 cc = make_float2(a.c2, a.c2);
    bool ok = true;
    for (int i = 0; i < it.n; ++i) {
      const int b = i & 1, ub = i >> 1, s = i % S;
      if (!tc::wait_or_fail(&ctl.s_full[b], ub & 1, &ctl.err, a.counters, kDevErrTimeout)) { ok = false; break; }
      tc::fence_after_sync();
      uint32_t v[2][16];
      ld32(tmem + ((uint32_t)(qd * 32) << 16) + b * 128 + g * 32, v);
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl.s_empty[b]);
      const int t = (it.tile0 + i) * 128 + tl;
      if ((it.tile0 + i) * 128 + 127 > a.N - a.W) {   // the window's edge: hidden scores -> -inf
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (t > clim[g * 32 + e]) v[e >> 4][e & 15] = kNegInf;
      }
      float2 sc0 = make_float2(0.f, 0.f), sc1 = sc0, aa0 = sc0, aa1 = sc0;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 b4 = *reinterpret_cast<const float4*>(&cb[g * 32 + e]);
        uint32_t* w = &v[e >> 4][e & 15];
        const float2 al0 = ex2x2(__ffma2_rn(f2(w[0], w[1]), cc, make_float2(b4.x, b4.y)));
        const float2 al1 = ex2x2(__ffma2_rn(f2(w[2], w[3]), cc, make_float2(b4.z, b4.w)));
        w[0] = __float_as_uint(al0.x); w[1] = __float_as_uint(al0.y);
        w[2] = __float_as_uint(al1.x); w[3] = __float_as_uint(al1.y);
        sc0 = __fadd2_rn(sc0, al0);
        sc1 = __fadd2_rn(sc1, al1);
        aa0 = __ffma2_rn(al0, al0, aa0);
        aa1 = __ffma2_rn(al1, al1, aa1);
      }
      if (it.rb == 0) {
        // the K tile has landed (its S MMA is done); the V side's norm
        // threads wait for the V tile
        if (nside == 1 && !tc::wait_or_fail(&ctl.v_full[s], (i / S) & 1, &ctl.err, a.counters, kDevErrTimeout)) {
          ok = false;
          break;
        }
        float ss = half_sumsq(xs + (2 * s + nside) * kOp, nrow, npart);
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        const int tn = (it.tile0 + i) * 128 + nrow;
        if (npart == 0 && tn < a.N) a.xnorm[((int64_t)nside * a.H + it.h) * a.N + tn] = sqrtf(ss);
      }
      tc::mbar_arrive(&ctl.k_empty[s]);      // this thread is done with the K tile
      if (i > 0 && !tc::wait_or_fail(&ctl.al_empty, (i - 1) & 1, &ctl.err, a.counters, kDevErrTimeout)) {
        ok = false;
        break;
      }
      // alpha[t][r] as bf16 hi + lo, MN-major (r contiguous), 128-byte
      // swizzle; this group's rows are chunks 4 (g & 1) .. + 3 of half g / 2
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int r = ch * 8 + 2 * p;                 // within the group's 32 rows
          const float2 x = f2(v[r >> 4][r & 15], v[r >> 4][(r & 15) + 1]);
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x.x, x.y);
          const float2 lo = __fadd2_rn(x, make_float2(-__low2float(h2), -__high2float(h2)));
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(lo.x, lo.y);
          hw[p] = *reinterpret_cast<const uint32_t*>(&h2);
          lw[p] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        const int cg = ((g & 1) << 2) + ch;
        const int off = (g >> 1) * kHalf + tl * 128 + ((cg ^ (tl & 7)) << 4);
        *reinterpret_cast<uint4*>(al + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(al + kOp + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&ctl.al_full);
      if (t < a.N) {
        const int64_t o = ((int64_t)rb4 * a.H + it.h) * a.N + t;
        a.score[o] = (sc0.x + sc0.y) + (sc1.x + sc1.y);
        a.a2s[o] = (aa0.x + aa0.y) + (aa1.x + aa1.y);
      }
    }
    // partial ybar^T: TMEM lane = d, column = row r (this group's 32 rows)
    float* py = a.part_y + ((int64_t)it.u * a.n_split + it.s) * 128 * 128;
    if (ok && it.n > 0 && tc::wait_or_fail(&ctl.y_full, 0, &ctl.err, a.counters, kDevErrTimeout)) {
      tc::fence_after_sync();
      uint32_t v[2][16];
      ld32(tmem + ((uint32_t)(qd * 32) << 16) + ycol + g * 32, v);
      const int d = tl;
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 16; ++e) py[(g * 32 + c * 16 + e) * 128 + d] = __uint_as_float(v[c][e]);
    } else if (it.n == 0) {
      for (int r = g * 32; r < g * 32 + 32; ++r) py[r * 128 + tl] = 0.f;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) { tc::fence_after_sync(); tc::tmem_dealloc(tmem, 512); }
}

// ybar = sum of partials (split order); bf16 hi/lo copies and ||ybar_r||^2.
// grid (U, 128 / kYbarRows), 128 threads: thread d sums coordinate d of
// kYbarRows rows, all partial loads of a row in flight together.
constexpr int kYbarRows = 4;
__global__ void __launch_bounds__(128) obs_ybar_kernel(ObsTc a, __nv_bfloat16* __restrict__ yh,
                                                       __nv_bfloat16* __restrict__ yl, float* __restrict__ row_y2) {
  __shared__ float red[kYbarRows][4];
  const int u = blockIdx.x, r0 = blockIdx.y * kYbarRows, d = threadIdx.x, warp = d >> 5, lane = d & 31;
  const float* src = a.part_y + (int64_t)u * a.n_split * 128 * 128 + (int64_t)r0 * 128 + d;
  float y[kYbarRows];
#pragma unroll
  for (int i = 0; i < kYbarRows; ++i) y[i] = 0.f;
#pragma unroll 4
  for (int sp = 0; sp < a.n_split; ++sp) {
#pragma unroll
    for (int i = 0; i < kYbarRows; ++i) y[i] += src[(int64_t)sp * 128 * 128 + i * 128];
  }
#pragma unroll
  for (int i = 0; i < kYbarRows; ++i) {
    const int64_t o = ((int64_t)u * 128 + r0 + i) * 128 + d;
    const __nv_bfloat16 hi = __float2bfloat16_rn(y[i]);
    yh[o] = hi;
    yl[o] = __float2bfloat16_rn(y[i] - __bfloat162float(hi));
    const float w = warp_sum(y[i] * y[i]);
    if (lane == 0) red[i][warp] = w;
  }
  __syncthreads();
  if (d < kYbarRows) row_y2[(int64_t)u * 128 + r0 + d] = red[d][0] + red[d][1] + red[d][2] + red[d][3];
}

// ============================================================== pass C

struct CtlC {
  uint64_t b_full, x_full[2], x_empty[2], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int err;
};

__global__ void __launch_bounds__(kThr, 1)
obs_c_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
             const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapYH,
             const __grid_constant__ CUtensorMap mapYL, ObsTc a) {
  extern __shared__ unsigned char smem_raw[];
  constexpr int S = 2;
  unsigned char* q = aligned_base(smem_raw);
  unsigned char* yh = q + kOp;
  unsigned char* yl = yh + kOp;
  unsigned char* xs = yl + kOp;                  // stage s: K at xs + 2s kOp, V at + kOp
  CtlC& ctl = *reinterpret_cast<CtlC*>(xs + S * 2 * kOp);
  // per row pair (r, r + 1): {cw_r, cw_r+1, ||ybar_r||^2, ||ybar_r+1||^2}, where
  // alpha_r^2 ||q_r||^2 = 2^(2 s c2 + cw_r); 16-byte aligned for float4 reads
  float* cpk = align16f(&ctl + 1);
  int* clim = reinterpret_cast<int*>(cpk + 256);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Item it = item_of(a);
  if (threadIdx.x == 0) {
    tc::mbar_init(&ctl.b_full, 1);
    for (int s = 0; s < S; ++s) { tc::mbar_init(&ctl.x_full[s], 1); tc::mbar_init(&ctl.x_empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&ctl.acc_full[b], 1); tc::mbar_init(&ctl.acc_empty[b], kEpi); }
    tc::mbar_init(&ctl.drain, 1);
    ctl.err = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) { tc::tmem_alloc(&ctl.tmem_base, 512); tc::tmem_relinquish(); }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + 128) {
    // cw_r = 2 log2(1/Z_r) + log2 ||q_r||^2 - 2 M_r (-inf for padding rows)
    const int r = threadIdx.x - 64;
    const int64_t o = (int64_t)it.u * 128 + r;
    cpk[(r >> 1) * 4 + (r & 1)] = 2.f * log2f(a.row_iz[o]) + log2f(a.row_q2[o]) - 2.f * a.row_m2[o];
    cpk[(r >> 1) * 4 + 2 + (r & 1)] = a.row_y2[o];
    clim[r] = row_limit(a, it.rb * 128 + r);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tc::mbar_expect_tx(&ctl.b_full, 3 * kOp);
      load_op(q, &mapQ, it.h * a.GW + it.rb * 128, &ctl.b_full);
      load_op(yh, &mapYH, it.u * 128, &ctl.b_full);
      load_op(yl, &mapYL, it.u * 128, &ctl.b_full);
      int issued = 0;
      for (int i = 0; i < it.n && !ctl.err; ++i) {
        const int s = i % S, use = i / S;
        if (use > 0 && !tc::wait_or_fail(&ctl.x_empty[s], (use - 1) & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
        tc::mbar_expect_tx(&ctl.x_full[s], 2 * kOp);
        const int row = it.h * a.N + (it.tile0 + i) * 128;
        load_op(xs + 2 * s * kOp, &mapK, row, &ctl.x_full[s]);
        load_op(xs + 2 * s * kOp + kOp, &mapV, row, &ctl.x_full[s]);
        ++issued;
      }
      for (int s = 0; s < S && s < issued; ++s) tc::mbar_wait(&ctl.x_full[s], ((issued - 1 - s) / S) & 1);
      tc::mbar_wait(&ctl.b_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = tc::idesc_bf16_f32(128, 128);
      if (tc::wait_or_fail(&ctl.b_full, 0, &ctl.err, a.counters, kDevErrTimeout)) {
        for (int i = 0; i < it.n; ++i) {
          const int s = i % S, use = i / S, b = i & 1, ub = i >> 1;
          if (!tc::wait_or_fail(&ctl.x_full[s], use & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
          if (ub > 0 && !tc::wait_or_fail(&ctl.acc_empty[b], (ub - 1) & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
          tc::fence_after_sync();
          const unsigned char* kt = xs + 2 * s * kOp;
          const unsigned char* vt = kt + kOp;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + b * 256, kdesc(kt, kk), kdesc(q, kk), id, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + b * 256 + 128, kdesc(vt, kk), kdesc(yh, kk), id, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + b * 256 + 128, kdesc(vt, kk), kdesc(yl, kk), id, 1u);
          tc::mma_commit(&ctl.acc_full[b]);
          tc::mma_commit(&ctl.x_empty[s]);
        }
      }
      tc::mma_commit(&ctl.drain);
      tc::mbar_wait(&ctl.drain, 0);
    }
  } else {
    // group g takes observation rows 32 g .. 32 g + 31 of every token
    const int qd = warp & 3, g = (warp - 2) >> 2, tl = qd * 32 + lane;
    const int rb4 = kGroups * it.rb + g;
    const float2 cc = make_float2(2.f * a.c2, 2.f * a.c2), m2 = make_float2(-2.f, -2.f);
    const float4* pk = reinterpret_cast<const float4*>(cpk) + g * 16;
    // ||V_t||^2 of this thread's token, one tile ahead
    auto vnorm2 = [&](int i) -> float {
      const int t = (it.tile0 + i) * 128 + tl;
      const float vn = (i < it.n && t < a.N) ? a.xnorm[((int64_t)a.H + it.h) * a.N + t] : 0.f;
      return vn * vn;
    };
    float v2n = vnorm2(0);
    for (int i = 0; i < it.n; ++i) {
      const int b = i & 1, ub = i >> 1;
      const float v2 = v2n;
      v2n = vnorm2(i + 1);
      if (!tc::wait_or_fail(&ctl.acc_full[b], ub & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
      tc::fence_after_sync();
      const uint32_t base = tmem + ((uint32_t)(qd * 32) << 16) + b * 256 + g * 32;
      const int t = (it.tile0 + i) * 128 + tl;
      const bool edge = (it.tile0 + i) * 128 + 127 > a.N - a.W;
      // sum_r w_r (||V_t||^2 - 2 V_t.ybar_r + ||ybar_r||^2), w_r = alpha_r^2 ||q_r||^2,
      // in two rounds of 16 rows (the accumulator is released after the second load)
      const float2 vv = make_float2(v2, v2);
      float2 ku0 = make_float2(0.f, 0.f), ku1 = ku0;
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        uint32_t sv[16], vy[16];
        tc::tmem_ld16(base + hr * 16, sv);
        tc::tmem_ld16(base + 128 + hr * 16, vy);
        tc::tmem_wait_ld_dep2(sv, vy);
        if (hr == 1) {
          tc::fence_before_sync();
          tc::mbar_arrive(&ctl.acc_empty[b]);
        }
        if (edge) {                                    // the window's edge: hidden scores -> -inf
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (t > clim[g * 32 + hr * 16 + e]) sv[e] = kNegInf;
        }
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 p0 = pk[hr * 8 + (e >> 1)], p1 = pk[hr * 8 + (e >> 1) + 1];
          const float2 w0 = ex2x2(__ffma2_rn(f2(sv[e], sv[e + 1]), cc, make_float2(p0.x, p0.y)));
          const float2 w1 = ex2x2(__ffma2_rn(f2(sv[e + 2], sv[e + 3]), cc, make_float2(p1.x, p1.y)));
          const float2 d0 = __ffma2_rn(f2(vy[e], vy[e + 1]), m2, __fadd2_rn(vv, make_float2(p0.z, p0.w)));
          const float2 d1 = __ffma2_rn(f2(vy[e + 2], vy[e + 3]), m2, __fadd2_rn(vv, make_float2(p1.z, p1.w)));
          ku0 = __ffma2_rn(w0, d0, ku0);
          ku1 = __ffma2_rn(w1, d1, ku1);
        }
      }
      if (t < a.N) a.kus[((int64_t)rb4 * a.H + it.h) * a.N + t] = (ku0.x + ku0.y) + (ku1.x + ku1.y);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) { tc::fence_after_sync(); tc::tmem_dealloc(tmem, 512); }
}

PFN_cuTensorMapEncodeTiled_v12000 encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool map128(CUtensorMap* m, const void* base, int64_t rows) {
  auto fn = encode();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kSmemA = 1024 + kOp + 4 * kOp + (int)sizeof(CtlA) + 64;
constexpr int kSmemB = 1024 + kOp + 4 * kOp + 2 * kOp + (int)sizeof(CtlB) + 2 * 128 * 4 + 64;
constexpr int kSmemC = 1024 + 3 * kOp + 4 * kOp + (int)sizeof(CtlC) + 3 * 128 * 4 + 64;
static_assert(kSmemB <= 227 * 1024 && kSmemC <= 227 * 1024, "shared memory budget");

ObsTc make_args(const Plan& pl, char* ws) {
  ObsTc a;
  a.N = pl.N; a.H = pl.H; a.G = pl.G; a.W = pl.W; a.GW = pl.GW;
  a.n_rb = pl.tc_rb; a.n_split = pl.tc_split; a.tps = pl.tc_tps; a.row_tiles = (pl.N + 127) / 128;
  a.c2 = kLog2e / sqrtf((float)kD);
  a.part_m2 = reinterpret_cast<float*>(ws + pl.o_tc_pm2);
  a.part_l = reinterpret_cast<float*>(ws + pl.o_tc_pl);
  a.row_m2 = reinterpret_cast<const float*>(ws + pl.o_tc_rm2);
  a.row_iz = reinterpret_cast<const float*>(ws + pl.o_tc_riz);
  a.row_q2 = reinterpret_cast<const float*>(ws + pl.o_tc_rq2);
  a.row_y2 = reinterpret_cast<const float*>(ws + pl.o_tc_ry2);
  a.score = reinterpret_cast<float*>(ws + pl.o_score);
  a.a2s = reinterpret_cast<float*>(ws + pl.o_a2);
  a.kus = reinterpret_cast<float*>(ws + pl.o_ku);
  a.part_y = reinterpret_cast<float*>(ws + pl.o_tc_py);
  a.xnorm = reinterpret_cast<float*>(ws + pl.o_xnorm);
  a.counters = reinterpret_cast<int*>(ws + pl.o_counters);
  return a;
}

}  // namespace

bool obs_tc_supported(const Plan& pl) { return pl.p.dtype == ANCHORKV_BF16 && encode() != nullptr; }

// Passes A..C; reports the launches it made through `stage` callbacks.
cudaError_t launch_obs_tc(const Plan& pl, const void* K, const void* V, const void* Q, char* ws, cudaStream_t s) {
  const ObsTc a = make_args(pl, ws);
  CUtensorMap mQ, mK, mV, mYH, mYL;
  const int U = pl.H * pl.tc_rb;
  if (!map128(&mQ, Q, (int64_t)pl.Hq * pl.W) || !map128(&mK, K, (int64_t)pl.H * pl.N) ||
      !map128(&mV, V, (int64_t)pl.H * pl.N) || !map128(&mYH, ws + pl.o_tc_yh, (int64_t)U * 128) ||
      !map128(&mYL, ws + pl.o_tc_yl, (int64_t)U * 128))
    return cudaErrorInvalidValue;
  const int items = U * pl.tc_split;
  cudaFuncSetAttribute(obs_a_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemA);
  cudaFuncSetAttribute(obs_b_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemB);
  cudaFuncSetAttribute(obs_c_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemC);
  stage_begin(kStObsPass1, s);
  obs_a_kernel<<<items, kThr, kSmemA, s>>>(mQ, mK, a);
  obs_rows_kernel<<<dim3(U, 16), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Q), a,
                                   reinterpret_cast<float*>(ws + pl.o_tc_rm2), reinterpret_cast<float*>(ws + pl.o_tc_riz),
                                   reinterpret_cast<float*>(ws + pl.o_tc_rq2));
  stage_end(kStObsPass1, s, 2);
  stage_begin(kStObsAlpha, s);
  obs_b_kernel<<<items, kThr, kSmemB, s>>>(mQ, mK, mV, a);
  stage_end(kStObsAlpha, s, 1);
  stage_begin(kStObsCombine, s);
  obs_ybar_kernel<<<dim3(U, 128 / kYbarRows), 128, 0, s>>>(a, reinterpret_cast<__nv_bfloat16*>(ws + pl.o_tc_yh),
                                   reinterpret_cast<__nv_bfloat16*>(ws + pl.o_tc_yl),
                                   reinterpret_cast<float*>(ws + pl.o_tc_ry2));
  stage_end(kStObsCombine, s, 1);
  stage_begin(kStObsKu, s);
  obs_c_kernel<<<items, kThr, kSmemC, s>>>(mQ, mK, mV, mYH, mYL, a);
  stage_end(kStObsKu, s, 1);
  return cudaGetLastError();
}

}  // namespace akv
