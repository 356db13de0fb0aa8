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
// ex2.approx in the log2 domain.  Warp roles as in the assignment kernel:
// warp 0 TMA, warp 1 TMEM owner + MMA issuer, warps 2..9 epilogue in two
// column groups (warps 2..5 and 6..9; one TMEM lane = one row or token per
// thread, each group half of the accumulator's columns).  Pass A's groups
// split the tokens of a tile and leave separate (max, sum) partials; passes B
// and C's groups split the observation rows, so their per-token sums are
// written as two row blocks per 128-row block.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace akv {

namespace {

constexpr int kOp = 128 * 256;                 // one [128][128] bf16 operand tile
constexpr int kHalf = kOp / 2;                 // its 64-column swizzled half
constexpr int kThr = 320;
constexpr int kEpi = 256;                      // epilogue threads (8 warps, 2 column groups)
constexpr float kLog2e = 1.4426950408889634f;

struct ObsTc {
  int N, H, G, W, GW, n_rb, n_split, tps, row_tiles;   // part_m2/part_l hold 2 * n_split partials per unit
  float c2;                                     // log2(e) / sqrt(D)
  float* part_m2;                               // [U][n_split][128]
  float* part_l;
  const float* row_m2;                          // [U][128]
  const float* row_iz;
  const float* row_q2;
  const float* row_y2;
  float* score;                                 // [2 n_rb][H][N] (row block rb, column group g at 2 rb + g)
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

__device__ __forceinline__ void ld128(uint32_t taddr, uint32_t (&v)[8][16]) {
  tc::tmem_ld16(taddr + 0, v[0]);
  tc::tmem_ld16(taddr + 16, v[1]);
  tc::tmem_ld16(taddr + 32, v[2]);
  tc::tmem_ld16(taddr + 48, v[3]);
  tc::tmem_wait_ld_dep4(v[0], v[1], v[2], v[3]);
  tc::tmem_ld16(taddr + 64, v[4]);
  tc::tmem_ld16(taddr + 80, v[5]);
  tc::tmem_ld16(taddr + 96, v[6]);
  tc::tmem_ld16(taddr + 112, v[7]);
  tc::tmem_wait_ld_dep4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ void ld64(uint32_t taddr, uint32_t (&v)[4][16]) {
  tc::tmem_ld16(taddr + 0, v[0]);
  tc::tmem_ld16(taddr + 16, v[1]);
  tc::tmem_ld16(taddr + 32, v[2]);
  tc::tmem_ld16(taddr + 48, v[3]);
  tc::tmem_wait_ld_dep4(v[0], v[1], v[2], v[3]);
}

template <typename U>
__device__ __forceinline__ float* align16f(U* p) {
  return reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(p) + 15) & ~static_cast<uintptr_t>(15));
}

__device__ __forceinline__ unsigned char* aligned_base(unsigned char* raw) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Sum of squares of one token row of a swizzled [128][128] bf16 tile.  The
// chunk order inside the row does not matter for a norm, so row r reads its
// 16-byte chunks in the order c ^ (r & 7): the 8 rows of a quarter-warp then
// hit 8 different bank groups.
__device__ __forceinline__ float row_sumsq(const unsigned char* tile, int r) {
  float s = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint4* p = reinterpret_cast<const uint4*>(tile + half * kHalf + r * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 q = p[c ^ (r & 7)];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
      }
    }
  }
  return s;
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
    // group g takes tokens 64 g .. 64 g + 63 of every tile
    const int qd = warp & 3, g = (warp - 2) >> 2, r = qd * 32 + lane;
    const int lim = row_limit(a, it.rb * 128 + r);
    float m = -INFINITY, l = 0.f;
    for (int i = 0; i < it.n; ++i) {
      const int b = i & 1, ub = i >> 1;
      if (!tc::wait_or_fail(&ctl.acc_full[b], ub & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
      tc::fence_after_sync();
      uint32_t v[4][16];
      ld64(tmem + ((uint32_t)(qd * 32) << 16) + b * 128 + g * 64, v);
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl.acc_empty[b]);
      const int t0 = (it.tile0 + i) * 128 + g * 64;
      if (lim < t0) continue;                       // nothing visible (or padding row)
      const bool full = t0 + 63 <= lim;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float y = __uint_as_float(v[c][e]) * a.c2;
          v[c][e] = __float_as_uint(y);
          if (full || t0 + c * 16 + e <= lim) mx = fmaxf(mx, y);
        }
      const float mn = fmaxf(m, mx);
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p = tc::ex2_approx(__uint_as_float(v[c][e]) - mn);
          const float q = (full || t0 + c * 16 + e <= lim) ? p : 0.f;
          if (e & 1) sum1 += q; else sum0 += q;
        }
      l = l * tc::ex2_approx(m - mn) + (sum0 + sum1);
      m = mn;
    }
    const int64_t pi = ((int64_t)it.u * 2 * a.n_split + 2 * it.s + g) * 128 + r;
    a.part_m2[pi] = m;
    a.part_l[pi] = l;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) { tc::fence_after_sync(); tc::tmem_dealloc(tmem, 256); }
}

// Row constants: M_r (log2 domain), 1/Z_r and ||q_r||^2; one thread per row.
__global__ void obs_rows_kernel(const __nv_bfloat16* __restrict__ Q, ObsTc a, float* __restrict__ row_m2,
                                float* __restrict__ row_iz, float* __restrict__ row_q2) {
  const int u = blockIdx.x, r = threadIdx.x;
  const int h = u / a.n_rb, rb = u % a.n_rb, rr = rb * 128 + r;
  const int np = 2 * a.n_split;
  float M = -INFINITY;
  for (int s = 0; s < np; ++s) M = fmaxf(M, a.part_m2[((int64_t)u * np + s) * 128 + r]);
  float Z = 0.f;
  for (int s = 0; s < np; ++s) {
    const int64_t pi = ((int64_t)u * np + s) * 128 + r;
    if (a.part_m2[pi] > -INFINITY) Z = fmaf(a.part_l[pi], exp2f(a.part_m2[pi] - M), Z);
  }
  float q2 = 0.f;
  if (rr < a.GW) {
    const __nv_bfloat16* qr = Q + ((int64_t)h * a.GW + rr) * kD;
    for (int d = 0; d < kD; ++d) {
      const float x = __bfloat162float(qr[d]);
      q2 = fmaf(x, x, q2);
    }
  }
  const int64_t o = (int64_t)u * 128 + r;
  const bool live = rr < a.GW && Z > 0.f;
  row_m2[o] = live ? M : 0.f;
  row_iz[o] = live ? 1.f / Z : 0.f;
  row_q2[o] = q2;
}

// ============================================================== pass B

struct CtlB {
  uint64_t q_full, x_full[2], x_empty[2], s_full[2], s_empty[2], al_full, al_empty, y_full, drain;
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
  float* cm2 = align16f(&ctl + 1);               // 16-byte aligned for float4 reads
  float* ciz = cm2 + 128;
  int* clim = reinterpret_cast<int*>(ciz + 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Item it = item_of(a);
  if (threadIdx.x == 0) {
    tc::mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < S; ++s) { tc::mbar_init(&ctl.x_full[s], 1); tc::mbar_init(&ctl.x_empty[s], 1); }
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
    const int r = threadIdx.x - 64;
    cm2[r] = a.row_m2[(int64_t)it.u * 128 + r];
    ciz[r] = a.row_iz[(int64_t)it.u * 128 + r];
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
      tc::mbar_wait(&ctl.q_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16_f32(128, 128);
      const uint32_t id2 = tc::idesc_bf16_f32_major(128, 128, 1, 1);
      bool ok = tc::wait_or_fail(&ctl.q_full, 0, &ctl.err, a.counters, kDevErrTimeout);
      auto mma1 = [&](int i) -> bool {
        const int s = i % S, use = i / S, b = i & 1, ub = i >> 1;
        if (!tc::wait_or_fail(&ctl.x_full[s], use & 1, &ctl.err, a.counters, kDevErrTimeout)) return false;
        if (ub > 0 && !tc::wait_or_fail(&ctl.s_empty[b], (ub - 1) & 1, &ctl.err, a.counters, kDevErrTimeout))
          return false;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + b * 128, kdesc(xs + 2 * s * kOp, kk), kdesc(q, kk), id1, kk > 0);
        tc::mma_commit(&ctl.s_full[b]);
        return true;
      };
      if (ok && it.n > 0) ok = mma1(0);
      for (int i = 0; ok && i < it.n; ++i) {
        if (i + 1 < it.n && !mma1(i + 1)) break;
        if (!tc::wait_or_fail(&ctl.al_full, i & 1, &ctl.err, a.counters, kDevErrTimeout)) break;
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
        tc::mma_commit(&ctl.x_empty[i % S]);
      }
      tc::mma_commit(&ctl.y_full);
      tc::mma_commit(&ctl.drain);
      tc::mbar_wait(&ctl.drain, 0);
    }
  } else {
    // group g takes observation rows 64 g .. 64 g + 63 of every token
    const int qd = warp & 3, g = (warp - 2) >> 2, tl = qd * 32 + lane;
    const int rb2 = 2 * it.rb + g;
    bool ok = true;
    for (int i = 0; i < it.n; ++i) {
      const int b = i & 1, ub = i >> 1, s = i % S;
      if (!tc::wait_or_fail(&ctl.s_full[b], ub & 1, &ctl.err, a.counters, kDevErrTimeout)) { ok = false; break; }
      tc::fence_after_sync();
      uint32_t v[4][16];
      ld64(tmem + ((uint32_t)(qd * 32) << 16) + b * 128 + g * 64, v);
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl.s_empty[b]);
      const int t = (it.tile0 + i) * 128 + tl;
      float sc = 0.f, a2 = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e4 = 0; e4 < 16; e4 += 4) {
          const int r0 = g * 64 + c * 16 + e4;
          const float4 m4 = *reinterpret_cast<const float4*>(&cm2[r0]);
          const float4 z4 = *reinterpret_cast<const float4*>(&ciz[r0]);
          const int4 l4 = *reinterpret_cast<const int4*>(&clim[r0]);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w}, zz[4] = {z4.x, z4.y, z4.z, z4.w};
          const int ll[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float al_ = tc::ex2_approx(fmaf(__uint_as_float(v[c][e4 + q]), a.c2, -mm[q])) * zz[q];
            al_ = (t <= ll[q]) ? al_ : 0.f;
            v[c][e4 + q] = __float_as_uint(al_);
            sc += al_;
            a2 = fmaf(al_, al_, a2);
          }
        }
      }
      if (it.rb == 0 && t < a.N) {
        const unsigned char* xt = xs + 2 * s * kOp + g * kOp;    // group 0: K, group 1: V
        a.xnorm[((int64_t)g * a.H + it.h) * a.N + t] = sqrtf(row_sumsq(xt, tl));
      }
      if (i > 0 && !tc::wait_or_fail(&ctl.al_empty, (i - 1) & 1, &ctl.err, a.counters, kDevErrTimeout)) {
        ok = false;
        break;
      }
      // alpha[t][r] as bf16 hi + lo, MN-major (r contiguous), 128-byte
      // swizzle; this group's rows are the 64-row half g of the tile
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int r = ch * 8 + 2 * p;                 // within the group's 64 rows
          const float x0 = __uint_as_float(v[r >> 4][r & 15]), x1 = __uint_as_float(v[(r + 1) >> 4][(r + 1) & 15]);
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
          const float2 hf = __bfloat1622float2(h2);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
          hw[p] = *reinterpret_cast<const uint32_t*>(&h2);
          lw[p] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        const int off = g * kHalf + tl * 128 + ((ch ^ (tl & 7)) << 4);
        *reinterpret_cast<uint4*>(al + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(al + kOp + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&ctl.al_full);
      if (t < a.N) {
        const int64_t o = ((int64_t)rb2 * a.H + it.h) * a.N + t;
        a.score[o] = sc;
        a.a2s[o] = a2;
      }
    }
    // partial ybar^T: TMEM lane = d, column = row r (this group's 64 rows)
    float* py = a.part_y + ((int64_t)it.u * a.n_split + it.s) * 128 * 128;
    if (ok && it.n > 0 && tc::wait_or_fail(&ctl.y_full, 0, &ctl.err, a.counters, kDevErrTimeout)) {
      tc::fence_after_sync();
      uint32_t v[4][16];
      ld64(tmem + ((uint32_t)(qd * 32) << 16) + ycol + g * 64, v);
      const int d = tl;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 16; ++e) py[(g * 64 + c * 16 + e) * 128 + d] = __uint_as_float(v[c][e]);
    } else if (it.n == 0) {
      for (int r = g * 64; r < g * 64 + 64; ++r) py[r * 128 + tl] = 0.f;
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
  float* cm2 = align16f(&ctl + 1);               // 16-byte aligned for float4 reads
  float* ciq = cm2 + 128;                       // ||q_r||^2 / Z_r^2
  float* cy2 = ciq + 128;
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
    const int r = threadIdx.x - 64;
    const int64_t o = (int64_t)it.u * 128 + r;
    cm2[r] = a.row_m2[o];
    ciq[r] = a.row_iz[o] * a.row_iz[o] * a.row_q2[o];
    cy2[r] = a.row_y2[o];
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
    // group g takes observation rows 64 g .. 64 g + 63 of every token
    const int qd = warp & 3, g = (warp - 2) >> 2, tl = qd * 32 + lane;
    const int rb2 = 2 * it.rb + g;
    const float c2x2 = 2.f * a.c2;
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
      const int t = (it.tile0 + i) * 128 + tl;
      const uint32_t base = tmem + ((uint32_t)(qd * 32) << 16) + b * 256 + g * 64;
      // every live row sees the whole tile unless it reaches into the window
      const bool full = (it.tile0 + i) * 128 + 127 <= a.N - a.W;
      float ku0 = 0.f, ku1 = 0.f;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t s0[16], s1[16], y0[16], y1[16];
        tc::tmem_ld16(base + c * 32, s0);
        tc::tmem_ld16(base + c * 32 + 16, s1);
        tc::tmem_ld16(base + 128 + c * 32, y0);
        tc::tmem_ld16(base + 128 + c * 32 + 16, y1);
        tc::tmem_wait_ld_dep4(s0, s1, y0, y1);
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          const int r0 = g * 64 + c * 32 + e4;
          const float4 m4 = *reinterpret_cast<const float4*>(&cm2[r0]);
          const float4 q4 = *reinterpret_cast<const float4*>(&ciq[r0]);
          const float4 y4 = *reinterpret_cast<const float4*>(&cy2[r0]);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w}, qq[4] = {q4.x, q4.y, q4.z, q4.w};
          const float yy[4] = {y4.x, y4.y, y4.z, y4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = e4 + q;
            const float sv = __uint_as_float(e < 16 ? s0[e] : s1[e - 16]);
            const float vy = __uint_as_float(e < 16 ? y0[e] : y1[e - 16]);
            // alpha^2 ||q||^2 = 2^(2 (s c2 - M2)) ||q||^2 / Z^2
            float w = tc::ex2_approx(fmaf(sv, c2x2, -2.f * mm[q])) * qq[q];
            if (!full && t > row_limit(a, it.rb * 128 + r0 + q)) w = 0.f;
            const float dist = fmaf(-2.f, vy, v2 + yy[q]);
            if (q & 1) ku1 = fmaf(w, dist, ku1); else ku0 = fmaf(w, dist, ku0);
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl.acc_empty[b]);
      if (t < a.N) a.kus[((int64_t)rb2 * a.H + it.h) * a.N + t] = ku0 + ku1;
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
constexpr int kSmemB = 1024 + kOp + 4 * kOp + 2 * kOp + (int)sizeof(CtlB) + 3 * 128 * 4 + 64;
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
  obs_rows_kernel<<<U, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(Q), a,
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
