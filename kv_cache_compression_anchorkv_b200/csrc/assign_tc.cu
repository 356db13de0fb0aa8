// Nearest-anchor assignment on the 5th-generation tensor cores (bf16).
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary": every key and value is assigned to its nearest anchor.
// Reading: argmax over slots of <x, a_s>/||a_s|| (signed cosine), ties to the
// lowest slot, a zero anchor scores 0, an anchor token keeps its own slot.
//
// The contraction S = X A^T (X: 128 token rows, A: all k anchors of the
// KV head and side, D = 128) runs as tcgen05.mma (M = 128, N = chunk of
// anchors, K = 16 per instruction) from 128-byte-swizzled shared-memory
// tiles that TMA fills; accumulators live in a ring of TMEM chunk buffers
// (as many as fit in 512 columns).  Chunks are at most 96 anchors wide: the
// epilogue and the MMA wait on each other through the ring, and a deeper ring
// of narrower chunks (five buffers of 96 for 288 anchors) measured faster than
// fewer wide ones (three of 144, or of 128 at most), although wide N issues
// MMAs at a better rate per FLOP.  The ring is shared by the epilogue groups, so a group may reach
// chunk q while the buffer still waits for chunk q - nbuf; since a parity
// wait cannot tell phase p from p + 2, a group first waits until the MMA warp
// has published that it issued chunk q (which it does only after chunk
// q - nbuf was released) and only then waits on the buffer's barrier.  The
// epilogue never writes S: each thread reads its TMEM lane, scales each column by 1/||a_s|| and
// keeps the best and second-best score of its row over all chunks.  Rows
// whose fp32 margin between best and second best is not above the
// accumulation error bound are listed for the fp64 re-decision shared with
// the SIMT path.
//
// More anchors than fit in shared memory (k > kMaxKpad) are taken in groups
// of at most kMaxKpad, one launch per group: each group's best two keys of a
// row are widened to 64 bits (score grid index, then the inverted global
// slot, so the order is still (score, -slot)) and merged with the previous
// groups' through the workspace; the last group decides.  Every group uses
// the row's same key grid, so keys of different groups compare exactly.
//
// Warp roles (one CTA per SM, persistent over (side, head, 128-row tile)
// work items): warp 0 issues TMA, warp 1 owns TMEM and issues MMAs, the
// other warps run the epilogue as kGroups groups of four warps that take
// items in turn, each whole (every column of its 128 rows), so the groups
// never wait on each other and need no merge.  Anchors of the current
// (side, head) stay resident in shared memory; token tiles stream through a
// ring.
// Every mbarrier wait is bounded: on timeout the kernel latches an error,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace akv {

// Margin below which a row's decision is re-taken in fp64, relative to ||x||.
// Per key, the error against the exact cosine score (plus a row-constant
// offset) is at most: fp32 accumulation of 128 exact products <= 2^-16 ||x||
// (a conservative bound for the tensor-core adder), rounding of 1/||a||
// <= 2^-24 ||x||, and the FMA's rounding onto the key grid <= 2^-15 ||x||; two
// keys therefore differ from the exact difference by < 2^-13.4 ||x||.
constexpr float kRefineRelTC = 1.0f / 8192.0f;

namespace {

#ifndef AKV_ASSIGN_COL_GROUPS
#define AKV_ASSIGN_COL_GROUPS 1
#endif
#ifndef AKV_ASSIGN_ITEM_GROUPS
#define AKV_ASSIGN_ITEM_GROUPS 2
#endif
#ifndef AKV_ASSIGN_CHUNK
#define AKV_ASSIGN_CHUNK 96
#endif
constexpr int kGroups = AKV_ASSIGN_ITEM_GROUPS;   // item groups: epilogue groups that take whole items in turn
constexpr int kColGroups = AKV_ASSIGN_COL_GROUPS;   // groups of four warps sharing an item's columns
constexpr int kEpiWarps = 4 * kGroups * kColGroups;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kChunkMax = AKV_ASSIGN_CHUNK;   // anchors per MMA chunk (N of one instruction)
constexpr int kMaxBuf = 8;                    // accumulator buffers in the TMEM ring
constexpr int kXStageBytes = 128 * 256;       // 128 rows x 128 bf16
constexpr int kMaxKpad = 480;

struct TcArgs {
  int N, H, k, kp16, cw, n_chunks, kpad, stages, row_tiles, nbuf;
  int g0, gk, first, last;      // this launch's anchor group: slots [g0, g0 + gk)
  ulonglong2* keys;             // [2][H][N] best two 64-bit keys after earlier groups
  int total_items;
  float* probe;                 // [512][kpad] raw accumulators of the probe rows, or null
  const float* anc_inv;
  const int* slot_of;
  const float* xnorm;
  uint32_t* tok;
  int* refine;
  int* counters;
};

// Best two packed keys of a row (see the epilogue).  Keys of distinct slots
// never compare equal, so the max/min updates keep them ordered; 0 = none.
struct Keys2 {
  uint32_t b1, b2;
};

__device__ __forceinline__ void key2_push(Keys2& s, uint32_t key) {
  const uint32_t n1 = max(s.b1, key);
  const uint32_t n2 = max(s.b2, min(key, s.b1));
  s.b1 = n1; s.b2 = n2;
}

// Slot of a key: the low 9 bits hold 511 - slot.
__device__ __forceinline__ uint32_t key_slot(uint32_t key) { return 511u - (key & 511u); }

// Per-row constants of the key: C = 2^(floor(log2 ||x||) + 9) makes
// fmaf(acc, 1/||a||, ||x||(1 + 2^-7) + C) land in [C, 2C), i.e. rounded to a
// grid step of 2^(floor(log2 ||x||) - 14) <= 2^-14 ||x||, and since C's
// mantissa is zero, bits(result) * 512 (mod 2^32) = q * 512 with q the grid
// index: key = bits * 512 + (511 - column) orders by (score, -column) exactly.
struct RowKey {
  float add;      // ||x|| (1 + 2^-7) + C
  float step;     // grid step
};
__device__ __forceinline__ RowKey row_key(float xn) {
  const float x = fmaxf(xn, 1e-30f);
  const int e = (int)((__float_as_uint(x) >> 23) & 255u) - 127;
  RowKey r;
  r.add = x * (1.0f + 1.0f / 128.0f) + __uint_as_float((uint32_t)(e + 9 + 127) << 23);
  r.step = __uint_as_float((uint32_t)(e - 14 + 127) << 23);
  return r;
}

// One 16-column block of a chunk (block BLK, columns 16 BLK ..): the block
// and column indices are compile-time after unrolling, so a key costs one
// FFMA and one shift-add, and the best-two update three integer min/max.
// Keys carry 511 - (column in chunk); the chunk offset is applied to the
// chunk's best two afterwards.
template <int BLK>
__device__ __forceinline__ void scan_block(const uint32_t (&w)[16], const float* ivc, float bias, int kc, Keys2& ka,
                                           Keys2& kb) {
  asm volatile("" ::: "memory");   // keep this block's loads from being hoisted into earlier blocks
  const float4* iv4 = reinterpret_cast<const float4*>(ivc + BLK * 16);
  const float4 i0 = iv4[0], i1 = iv4[1], i2 = iv4[2], i3 = iv4[3];
  const float ivs[16] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w,
                         i2.x, i2.y, i2.z, i2.w, i3.x, i3.y, i3.z, i3.w};
  if (BLK * 16 + 16 <= kc) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t key = __float_as_uint(fmaf(__uint_as_float(w[e]), ivs[e], bias)) * 512u +
                           (uint32_t)(511 - (BLK * 16 + e));
      if (e & 1) key2_push(kb, key);
      else key2_push(ka, key);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      uint32_t key = __float_as_uint(fmaf(__uint_as_float(w[e]), ivs[e], bias)) * 512u +
                     (uint32_t)(511 - (BLK * 16 + e));
      if (BLK * 16 + e >= kc) key = 0u;
      key2_push(ka, key);
    }
  }
}

// Blocks J and J + 1 are in c0/c1; the loads of blocks J + 2 and J + 3 go
// out before c0/c1 are scanned, so the TMEM latency hides behind the scan.
// nv = valid blocks of the chunk (at most kChunkMax / 16).
template <int J>
__device__ __forceinline__ void scan_pipe(uint32_t tbase, const float* ivc, float bias, int kc, int nv,
                                          uint32_t (&c0)[16], uint32_t (&c1)[16], uint32_t (&n0)[16],
                                          uint32_t (&n1)[16], Keys2& ka, Keys2& kb) {
  constexpr int kB = kChunkMax / 16;
  if constexpr (J < kB) {
    if (J >= nv) return;
    const bool l2 = J + 2 < nv, l3 = J + 3 < nv;
    if constexpr (J + 2 < kB) { if (l2) tc::tmem_ld16(tbase + (uint32_t)((J + 2) * 16), n0); }
    if constexpr (J + 3 < kB) { if (l3) tc::tmem_ld16(tbase + (uint32_t)((J + 3) * 16), n1); }
    scan_block<J>(c0, ivc, bias, kc, ka, kb);
    if constexpr (J + 1 < kB) { if (J + 1 < nv) scan_block<J + 1>(c1, ivc, bias, kc, ka, kb); }
    if (l2) tc::tmem_wait_ld_dep2(n0, n1);
    scan_pipe<J + 2>(tbase, ivc, bias, kc, nv, n0, n1, c0, c1, ka, kb);
  }
}

// Blocks P, P + 2, ... of a chunk (one of two column groups sharing it): the
// load of block J + 2 goes out before block J is scanned.
template <int J>
__device__ __forceinline__ void scan_alt(uint32_t tbase, const float* ivc, float bias, int kc, int nv,
                                         uint32_t (&c0)[16], uint32_t (&n0)[16], Keys2& ka, Keys2& kb) {
  constexpr int kB = kChunkMax / 16;
  if constexpr (J < kB) {
    if (J >= nv) return;
    const bool l2 = J + 2 < nv;
    if constexpr (J + 2 < kB) { if (l2) tc::tmem_ld16(tbase + (uint32_t)((J + 2) * 16), n0); }
    scan_block<J>(c0, ivc, bias, kc, ka, kb);
    if (l2) tc::tmem_wait_ld_dep(n0);
    scan_alt<J + 2>(tbase, ivc, bias, kc, nv, n0, c0, ka, kb);
  }
}

template <int P>
__device__ __forceinline__ Keys2 scan_chunk_alt(uint32_t tbase, const float* ivc, float bias, int kc) {
  Keys2 ka{0u, 0u}, kb{0u, 0u};
  const int nv = (kc + 15) >> 4;
  if (P < nv) {
    uint32_t c0[16], n0[16];
    tc::tmem_ld16(tbase + (uint32_t)(P * 16), c0);
    tc::tmem_wait_ld_dep(c0);
    scan_alt<P>(tbase, ivc, bias, kc, nv, c0, n0, ka, kb);
  }
  key2_push(ka, kb.b1);
  key2_push(ka, kb.b2);
  return ka;
}

// Best two keys of one chunk (kc valid columns of its TMEM buffer).
__device__ __forceinline__ Keys2 scan_chunk(uint32_t tbase, const float* ivc, float bias, int kc) {
  Keys2 ka{0u, 0u}, kb{0u, 0u};
  const int nv = (kc + 15) >> 4;
  uint32_t c0[16], c1[16], n0[16], n1[16];
  tc::tmem_ld16(tbase, c0);
  if (nv > 1) tc::tmem_ld16(tbase + 16u, c1);
  tc::tmem_wait_ld_dep2(c0, c1);
  scan_pipe<0>(tbase, ivc, bias, kc, nv, c0, c1, n0, n1, ka, kb);
  key2_push(ka, kb.b1);
  key2_push(ka, kb.b2);
  return ka;
}

struct Ctl {
  uint64_t x_full[4], x_empty[4], acc_full[kMaxBuf], acc_empty[kMaxBuf], anc_full, anc_empty, drain;
  uint32_t tmem_base;
  int err;
  int issued;          // chunks the MMA warp has issued (store-release)
  // column groups of one item group: the second group's best two keys per
  // row (by item parity) and a failure flag both read after their barrier
  uint2 xchg[kGroups][2][128];
  int pair_fail[kGroups];
};

__device__ __forceinline__ void publish_issued(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(tc::smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int read_issued(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(tc::smem_u32(p)) : "memory");
  return v;
}

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, Ctl& ctl, int* counters) {
  uint64_t t0 = 0;
  for (uint32_t i = 0; i < tc::kWaitLimit; ++i) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u) {
      if (*(volatile int*)&ctl.err) return false;
      const uint64_t now = tc::globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > tc::kWaitNs) break;
    }
  }
  *(volatile int*)&ctl.err = 1;
  latch_error(counters, kDevErrTimeout);
  return false;
}

// Bounded wait until the MMA warp has issued chunk q.
__device__ __forceinline__ bool wait_issued(Ctl* ctl, int q, int* counters) {
  uint64_t t0 = 0;
  for (uint32_t i = 0; i < tc::kWaitLimit; ++i) {
    if (read_issued(&ctl->issued) > q) return true;
    if ((i & 255u) == 255u) {
      if (*(volatile int*)&ctl->err) return false;
      const uint64_t now = tc::globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > tc::kWaitNs) break;
    }
  }
  *(volatile int*)&ctl->err = 1;
  latch_error(counters, kDevErrTimeout);
  return false;
}

__global__ void __launch_bounds__(kThreads, 1)
assign_tc_kernel(const __grid_constant__ CUtensorMap mapXK, const __grid_constant__ CUtensorMap mapXV,
                 const __grid_constant__ CUtensorMap mapAK, const __grid_constant__ CUtensorMap mapAV, TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned base for the swizzled operand tiles
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* anc = base;                                   // kpad x 256 B
  unsigned char* xs = anc + (size_t)a.kpad * 256;              // stages x 32 KB
  Ctl& ctl = *reinterpret_cast<Ctl*>(xs + (size_t)a.stages * kXStageBytes);
  float* winv = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(&ctl + 1) + 15) & ~static_cast<uintptr_t>(15));   // [kEpiWarps][kpad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int beg = (int)((int64_t)blockIdx.x * a.total_items / G);
  const int end = (int)((int64_t)(blockIdx.x + 1) * a.total_items / G);
  const int S = a.stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { tc::mbar_init(&ctl.x_full[s], 1); tc::mbar_init(&ctl.x_empty[s], 1); }
    for (int b = 0; b < a.nbuf; ++b) {
      tc::mbar_init(&ctl.acc_full[b], 1);
      tc::mbar_init(&ctl.acc_empty[b], 128 * kColGroups);
    }
    ctl.issued = 0;
    for (int i = 0; i < kGroups; ++i) ctl.pair_fail[i] = 0;
    tc::mbar_init(&ctl.anc_full, 1);
    tc::mbar_init(&ctl.anc_empty, 1);
    tc::mbar_init(&ctl.drain, 1);
    ctl.err = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&ctl.tmem_base, 512);
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&mapXK); tc::prefetch_tensormap(&mapXV);
    tc::prefetch_tensormap(&mapAK); tc::prefetch_tensormap(&mapAV);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int cur_u = -1, anc_loads = 0, issued = 0;
      for (int it = beg; it < end && !ctl.err; ++it) {
        const int u = it / a.row_tiles, j = it % a.row_tiles;
        const int side = u / a.H, h = u % a.H;
        if (u != cur_u) {
          if (anc_loads > 0 && !wait_or_fail(&ctl.anc_empty, (anc_loads - 1) & 1, ctl, a.counters)) break;
          tc::mbar_expect_tx(&ctl.anc_full, (uint32_t)a.kpad * 256u);
          const CUtensorMap* mA = side ? &mapAV : &mapAK;
          for (int c = 0; c < a.n_chunks; ++c)
            for (int kh = 0; kh < 2; ++kh)
              tc::tma_load_2d(anc + (size_t)(c * 2 + kh) * a.cw * 128, mA, kh * 64, h * a.k + a.g0 + c * a.cw,
                              &ctl.anc_full);
          cur_u = u;
          ++anc_loads;
        }
        const int n = it - beg, s = n % S, use = n / S;
        if (use > 0 && !wait_or_fail(&ctl.x_empty[s], (use - 1) & 1, ctl, a.counters)) break;
        tc::mbar_expect_tx(&ctl.x_full[s], kXStageBytes);
        const CUtensorMap* mX = side ? &mapXV : &mapXK;
        const int row = h * a.N + j * 128;
        tc::tma_load_2d(xs + (size_t)s * kXStageBytes, mX, 0, row, &ctl.x_full[s]);
        tc::tma_load_2d(xs + (size_t)s * kXStageBytes + kXStageBytes / 2, mX, 64, row, &ctl.x_full[s]);
        ++issued;
      }
      // drain: every copy issued must have landed before the CTA exits
      for (int s = 0; s < S && s < issued; ++s) {
        const int last_use = (issued - 1 - s) / S;
        tc::mbar_wait(&ctl.x_full[s], last_use & 1);
      }
      if (anc_loads > 0) tc::mbar_wait(&ctl.anc_full, (anc_loads - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, a.cw);
      int cur_u = -1, anc_loads = 0, q = 0;
      for (int it = beg; it < end && !ctl.err; ++it) {
        const int u = it / a.row_tiles;
        if (u != cur_u) {
          if (anc_loads > 0) tc::mma_commit(&ctl.anc_empty);     // old anchors free once MMAs finish
          if (!wait_or_fail(&ctl.anc_full, anc_loads & 1, ctl, a.counters)) break;
          cur_u = u;
          ++anc_loads;
        }
        const int n = it - beg, s = n % S, use = n / S;
        if (!wait_or_fail(&ctl.x_full[s], use & 1, ctl, a.counters)) break;
        tc::fence_after_sync();
        const uint32_t xa = tc::smem_u32(xs + (size_t)s * kXStageBytes);
        bool ok = true;
        for (int c = 0; c < a.n_chunks; ++c, ++q) {
          const int b = q % a.nbuf, uq = q / a.nbuf;
          if (uq > 0 && !wait_or_fail(&ctl.acc_empty[b], (uq - 1) & 1, ctl, a.counters)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t d = tmem + (uint32_t)(b * a.cw);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (uint32_t)((kk >> 2) * (kXStageBytes / 2) + (kk & 3) * 32);
            const uint32_t boff = (uint32_t)(((c * 2 + (kk >> 2)) * a.cw) * 128 + (kk & 3) * 32);
            tc::mma_bf16(d, tc::sw128_desc(xa + aoff), tc::sw128_desc(tc::smem_u32(anc) + boff), idesc,
                         kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&ctl.acc_full[b]);
          publish_issued(&ctl.issued, q + 1);
        }
        if (!ok) break;
        tc::mma_commit(&ctl.x_empty[s]);
      }
      tc::mma_commit(&ctl.drain);
      tc::mbar_wait(&ctl.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (kEpiWarps warps)
    // Each column score s = acc / ||a|| becomes one positive integer key
    //   key = bits(s + ||x|| (1 + 2^-7) + C) * 512 + 511 - slot,
    // so the largest key is the best score and, among equal keys, the lowest
    // slot.  Item group g takes the items beg + g, beg + g + kGroups, ...;
    // with two column groups per item group, column group cg scans the
    // 16-column blocks cg, cg + 2, ... of every chunk and the pair merges its
    // rows' best two keys through shared memory after each item.
    const int g = (warp - 2) / (4 * kColGroups);
    const int cg = ((warp - 2) >> 2) % kColGroups;
    const int qd = warp & 3;                // TMEM lane quarter this warp may access
    const int row = qd * 32 + lane;
    float* inv = winv + (size_t)(warp - 2) * a.kpad;   // this warp's copy of 1/||a||
    int cur_u = -1;
    // this thread's row norm and own-slot flag, one item ahead
    auto row_info = [&](int it2, float& xn2, int& own2) {
      xn2 = 0.f;
      own2 = -1;
      if (it2 >= end) return;
      const int u2 = it2 / a.row_tiles, j2 = it2 % a.row_tiles;
      const int t2 = j2 * 128 + row;
      if (t2 >= a.N) return;
      const int side2 = u2 / a.H, h2 = u2 % a.H;
      xn2 = a.xnorm[((int64_t)side2 * a.H + h2) * a.N + t2];
      own2 = a.slot_of[(int64_t)h2 * a.N + t2];
    };
    float xn_next;
    int own_next;
    row_info(beg + g, xn_next, own_next);
    for (int it = beg + g; it < end; it += kGroups) {
      const int u = it / a.row_tiles, j = it % a.row_tiles;
      const int side = u / a.H, h = u % a.H;
      const float xn = xn_next;
      const int own = own_next;
      row_info(it + kGroups, xn_next, own_next);
      if (u != cur_u) {
        __syncwarp();
        const float* src = a.anc_inv + (int64_t)u * a.kp16;
        for (int i = lane; i < a.kpad; i += 32) inv[i] = (i < a.gk) ? src[a.g0 + i] : 0.f;
        __syncwarp();
        cur_u = u;
      }
      const int t = j * 128 + row;
      const int64_t f = ((int64_t)side * a.H + h) * a.N + t;
      const RowKey rk = row_key(xn);
      Keys2 ka{0u, 0u};
      bool ok = true;
      int q = (it - beg) * a.n_chunks;      // ring index of this item's first chunk
      for (int c = 0; c < a.n_chunks; ++c, ++q) {
        const int b = q % a.nbuf, uq = q / a.nbuf;
        // chunk q issued => chunk q - nbuf released => the barrier is at phase uq
        if (!wait_issued(&ctl, q, a.counters) || !wait_or_fail(&ctl.acc_full[b], uq & 1, ctl, a.counters)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t tbase = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(b * a.cw);
        const int kc = min(a.cw, a.gk - c * a.cw);
        Keys2 ca;
        if constexpr (kColGroups == 1) ca = scan_chunk(tbase, inv + c * a.cw, rk.add, kc);
        else ca = cg == 0 ? scan_chunk_alt<0>(tbase, inv + c * a.cw, rk.add, kc)
                          : scan_chunk_alt<1>(tbase, inv + c * a.cw, rk.add, kc);
        if (a.probe && a.first && u == 0 && j < 4 && cg == 0) {
          // diagnostic: the raw fp32 accumulators <x_t, a_s> of tokens
          // 0..511 of the key side of head 0 (first anchor group), so a test
          // can measure the tensor-core accumulation error directly
          for (int blk = 0; blk < (kc + 15) / 16; ++blk) {
            uint32_t w[16];
            tc::tmem_ld16(tbase + (uint32_t)(blk * 16), w);
            tc::tmem_wait_ld_dep(w);
            float* dst = a.probe + (int64_t)(j * 128 + row) * a.kpad + c * a.cw + blk * 16;
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2)
              if (blk * 16 + e2 < kc) dst[e2] = __uint_as_float(w[e2]);
          }
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&ctl.acc_empty[b]);
        // column in chunk -> slot: the low 9 bits drop by c cw (no borrow, slot < 512)
        const uint32_t off = (uint32_t)(c * a.cw);
        if (ca.b1) ca.b1 -= off;
        if (ca.b2) ca.b2 -= off;
        key2_push(ka, ca.b1);
        key2_push(ka, ca.b2);
      }
      if constexpr (kColGroups > 1) {
        // both column groups reach this barrier once per item, failed or
        // not, and decide together whether to go on
        const int par = ((it - beg) / kGroups) & 1;
        if (cg == 1) ctl.xchg[g][par][row] = make_uint2(ka.b1, ka.b2);
        if (!ok) ctl.pair_fail[g] = 1;
        tc::named_bar(1 + g, 32 * 4 * kColGroups);
        if (*(volatile int*)&ctl.pair_fail[g]) break;
        if (cg == 1) continue;
        const uint2 o2 = ctl.xchg[g][par][row];
        key2_push(ka, o2.x);
        key2_push(ka, o2.y);
      }
      if (!ok) break;
      if (t < a.N) {
        // 64-bit keys: grid index, then ~(global slot); 0 = none
        auto wide = [&](uint32_t k32) -> uint64_t {
          return k32 ? ((uint64_t)(k32 >> 9) << 32) | (uint32_t)~(uint32_t)(a.g0 + key_slot(k32)) : 0ull;
        };
        uint64_t b1 = wide(ka.b1), b2 = wide(ka.b2);
        if (!a.first) {
          const ulonglong2 pv = a.keys[f];
          const uint64_t p1 = pv.x, p2 = pv.y;
          auto mx = [](uint64_t x, uint64_t y) { return x > y ? x : y; };
          const uint64_t n1 = mx(b1, p1), n2 = mx(mx(b2, p2), b1 < p1 ? b1 : p1);
          b1 = n1;
          b2 = n2;
        }
        if (!a.last) {
          a.keys[f] = make_ulonglong2((unsigned long long)b1, (unsigned long long)b2);
        } else {
          uint32_t slot;
          if (own >= 0) {
            slot = (uint32_t)own;
          } else {
            slot = ~(uint32_t)b1;
            const float gap = (float)((uint32_t)(b1 >> 32) - (uint32_t)(b2 >> 32)) * rk.step;
            if (!(gap > kRefineRelTC * xn)) list_for_refine(a.refine, a.counters, u, a.N, t);
          }
          a.tok[f] = slot;
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Row-major bf16 matrix [rows][128] as a tiled map with boxes of 64 x box_rows
// (128-byte rows, 128-byte swizzle).
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

static_assert(kAssignGroupMax == kMaxKpad, "the plan's anchor groups are the kernel's resident anchor limit");

bool assign_tc_supported(const Plan& pl) { return pl.p.dtype == ANCHORKV_BF16 && encode_fn() != nullptr; }

// One launch per anchor group (a single one when k <= kMaxKpad); groups of
// equal size, each split into chunks of at most kChunkMax anchors.
cudaError_t launch_assign_tc(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  const int n_groups = (pl.k + kMaxKpad - 1) / kMaxKpad;
  const int gsize = ((pl.k + n_groups - 1) / n_groups + 15) / 16 * 16;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  CUtensorMap mXK, mXV;
  const int64_t HN = (int64_t)pl.H * pl.N, Hk = (int64_t)pl.H * pl.k;
  if (!make_map(&mXK, K, HN, 128) || !make_map(&mXV, V, HN, 128)) return cudaErrorInvalidValue;
  for (int g = 0; g < n_groups; ++g) {
    TcArgs a;
    a.N = pl.N; a.H = pl.H; a.k = pl.k; a.kp16 = pl.kp16;
    a.g0 = g * gsize;
    a.gk = std::min(gsize, pl.k - a.g0);
    a.first = g == 0;
    a.last = g == n_groups - 1;
    a.keys = n_groups > 1 ? reinterpret_cast<ulonglong2*>(ws + pl.o_asg_keys) : nullptr;
    a.n_chunks = (a.gk + kChunkMax - 1) / kChunkMax;
    a.cw = ((a.gk + a.n_chunks - 1) / a.n_chunks + 15) / 16 * 16;
    a.kpad = a.n_chunks * a.cw;
    if (a.kpad > kMaxKpad) return cudaErrorInvalidValue;
    a.nbuf = std::min(kMaxBuf, 512 / a.cw);
    a.row_tiles = (pl.N + 127) / 128;
    a.total_items = 2 * pl.H * a.row_tiles;
    const int fixed = 1024 + (int)sizeof(Ctl) + 16 + kEpiWarps * a.kpad * 4 + a.kpad * 256;
    a.stages = std::min(4, (227 * 1024 - fixed) / kXStageBytes);
    if (a.stages < 2) return cudaErrorInvalidValue;
    // the accumulator probe is a test hook (ANCHORKV_ASSIGN_PROBE=1): its
    // scattered stores would hold up the CTA that owns the probe rows
    {
      const char* e = getenv("ANCHORKV_ASSIGN_PROBE");
      a.probe = (e && e[0] == '1') ? reinterpret_cast<float*>(ws + pl.o_asg_probe) : nullptr;
    }
    a.anc_inv = reinterpret_cast<const float*>(ws + pl.o_anc_inv);
    a.slot_of = reinterpret_cast<const int*>(ws + pl.o_slot_of);
    a.xnorm = reinterpret_cast<const float*>(ws + pl.o_xnorm);
    a.tok = reinterpret_cast<uint32_t*>(out + pl.L.off_tok);
    a.refine = reinterpret_cast<int*>(ws + pl.o_refine);
    a.counters = reinterpret_cast<int*>(ws + pl.o_counters);
    CUtensorMap mAK, mAV;
    if (!make_map(&mAK, out + pl.L.off_anchors_k, Hk, a.cw) || !make_map(&mAV, out + pl.L.off_anchors_v, Hk, a.cw))
      return cudaErrorInvalidValue;
    const int smem = fixed + a.stages * kXStageBytes;
    const int grid = std::min(sms, a.total_items);
    cudaFuncSetAttribute(assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    assign_tc_kernel<<<grid, kThreads, smem, s>>>(mXK, mXV, mAK, mAV, a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace akv
