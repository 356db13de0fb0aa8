// Decode attention over the compressed layout: one thread-block cluster per
// (sequence, KV head), one launch per layer, no global scratch.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary": a FlashAttention-style decoder rebuilds tiles when they
// are consumed; "AnchorKV-adapted" (VeloxQuant-MLX), "Adaptation notes":
// decode tokens are appended at full precision.
//
// The rebuild is factored so that only compressed bytes are read per token:
//   q . K^_t / sqrt(D) = g^K_t P[i(t)] + sigma~_t <H(s . q) / D, lev(c_t)>,
//   P[a] = q . a^K_a / sqrt(D)
//   sum_t p_t V^_t = sum_a W[a] a^V_a + s . H(Z) / sqrt(D),
//   W[a] = sum_{t: i(t)=a} p_t g^V_t,  Z = sum_t p_t sigma~_t lev(c_t)
// (H the unnormalised Sylvester matrix, s the shared sign vector).
//
// Work split.  The C CTAs of a cluster share one (sequence, head):
//  1. CTA r computes P for anchor slots [r kc, (r+1) kc) and stores them into
//     every CTA's shared memory (distributed shared memory);
//  2. each CTA walks its 128-token tiles in chunks of at most 1024 tokens
//     whose residual records fit the 768-record staging buffer.  A chunk's
//     token records, bitmap words, residual codes and scales are copied into
//     shared memory with cp.async; each thread owns 4 tokens (token
//     tid + 256 u, so warp w reads bitmap words w + 8 u) and keeps their
//     scores in registers:
//       a. anchor logits, and each residual's rank in the chunk (= its staged
//          record) from a prefix count over the chunk's bitmap words;
//       b. key residual logits per key record, one warp per 32/G records
//          (lane = code byte), partial dot products reduced by a transposed
//          butterfly, stored by rank;
//       c. each token adds its record's logit; the chunk maximum raises the
//          running maximum only when it exceeds it by 2^8 (rescaling is rare);
//       d. probabilities, value-anchor weights W by shared-memory atomics, and
//          each value record's weights p sigma~ stored by rank;
//       e. value residual sums Z over the value records (lane = code byte,
//          packed f32x2 FMAs);
//  3. the cluster merges (max, sum, W, Z) through distributed shared memory:
//     CTA r forms W for its slot slice and multiplies it with its slice of
//     value anchors, the CTA owning head j undoes the rotation of its Z, and
//     the partial outputs are summed into the output rows.
// Scores are kept in log2 units (q is pre-multiplied by log2 e).
#include <algorithm>
#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTT = 1024;                  // most tokens per chunk
constexpr int kTPT = kTT / kThreads;       // tokens per thread
constexpr int kTilesPC = kTT / kTile;      // most tiles per chunk
constexpr int kWordsPC = kTT / 32;         // bitmap words per chunk and side
constexpr int kRC = 768;                   // residual records staged per chunk, both sides
constexpr int kLutCopies = 8;              // lane l reads copy l % 8: conflict-free float4 lookups
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleGap = 8.0f;        // log2 units
constexpr int kMaxC = 16;
static_assert(kRC >= 2 * kTile, "one tile's records must fit a chunk");
static_assert(kWarps >= 8, "a warp per query head of a KV head (G <= 8)");
static_assert(kWordsPC == 4 * kWarps, "warp w reads bitmap words w + 8u");

struct CArgs {
  const uint8_t* comp;
  int64_t stride;
  anchorkv_layout L;
  int N, H, G, k, n_tiles;
  int64_t R;
  float lev[4];
  uint32_t sign_bits[4];
  int naive;                 // unrotated codec: residuals live in the token domain
  const void* q;
  const void* Kt;
  const void* Vt;
  int tail_len, tail_cap;
  float* out;
};

// One chunk's token records, bitmap words (with prefix counts), residual
// codes (key records, then value records) and scales.
struct Stage {
  uint8_t codes[kRC * kCodeBytes];   // 16-byte copies: first, at offset 0
  uint32_t tok[2][kTT];
  uint32_t bm[2][kWordsPC];          // 16-byte copies: offset 32 KB
  int wpre[2][kWordsPC + 1];
  uint16_t sig[2][kRC + 8];          // 4-byte copies
};
static_assert(offsetof(Stage, bm) % 16 == 0 && offsetof(Stage, sig) % 4 == 0, "cp.async alignment");

// Shared-memory carve-up (bytes), identical on host and device.
struct SmemPlan {
  int lut, stage, pf, P, W, rbuf, vsl, zred, oacc, ofin, misc, total;
};

__host__ __device__ inline int align_up(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int gp_of(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

// tpc: most tiles one CTA owns (its tile prefixes are kept for the whole
// range); kc: anchor slots per CTA; elem: bytes per anchor element.
__host__ __device__ inline SmemPlan smem_plan(int G, int k, int tpc, int kc, int elem) {
  SmemPlan s;
  int cur = 0;
  s.lut = cur; cur += 256 * kLutCopies * 16;
  s.stage = cur; cur = align_up(cur + (int)sizeof(Stage), 16);
  s.pf = cur; cur = align_up(cur + 4 * 2 * (tpc + 1), 16);
  s.P = cur; cur = align_up(cur + 4 * G * k, 16);
  s.W = cur; cur = align_up(cur + 4 * G * k, 16);
  s.rbuf = cur; cur = align_up(cur + 4 * gp_of(G) * kRC, 16);
  s.vsl = cur; cur = align_up(cur + kc * kD * elem, 16);
  s.zred = cur; cur += 4 * G * kD;
  s.oacc = cur; cur += 4 * G * kD;
  s.ofin = cur; cur += 4 * G * kD;
  s.misc = cur; cur += 4 * (8 * 4 + kMaxC * 8 * 3 + kWarps * 8);
  s.total = align_up(cur, 16);
  return s;
}

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Hardware cluster barrier with release/acquire ordering of shared memory.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// Generic pointer to the same shared-memory object in CTA `rank` of the cluster.
template <typename U>
__device__ __forceinline__ const U* peer(const U* p, uint32_t rank) {
  return static_cast<const U*>(__cluster_map_shared_rank(p, rank));
}
__device__ __forceinline__ void cp_async4(void* s, const void* g) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(s)), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async16(void* s, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(s)), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float sign_of(const CArgs& a, int d) {
  return ((a.sign_bits[d >> 5] >> (d & 31)) & 1u) ? -1.f : 1.f;
}

// Records of tiles [i0, i1) of one side (relative prefix indices), clamped
// to [0, R) and to `cap` records: [r0, r0 + n), scales staged from the even
// record w0.
struct RecRange {
  int64_t r0, w0;
  int n;
};
__device__ __forceinline__ RecRange rec_range(const int* pfs, int i0, int i1, int64_t R, int cap) {
  RecRange rr;
  int64_t lo = pfs[i0], hi = pfs[i1];
  lo = lo < 0 ? 0 : (lo > R ? R : lo);
  hi = hi > R ? R : hi;
  int64_t n = hi - lo;
  n = n < 0 ? 0 : (n > cap ? cap : n);
  rr.r0 = lo;
  rr.n = (int)n;
  rr.w0 = lo & ~(int64_t)1;
  return rr;
}

// End tile of the chunk that starts at tile t0: at most kTilesPC tiles and
// kRC records of both sides (at least one tile).
__device__ __forceinline__ int chunk_end(const int* pf, int pf_stride, int tb, int te, int t0) {
  int t1 = t0 + 1;
  while (t1 < te && t1 - t0 < kTilesPC) {
    const int64_t nk = (int64_t)pf[t1 + 1 - tb] - pf[t0 - tb];
    const int64_t nv = (int64_t)pf[pf_stride + t1 + 1 - tb] - pf[pf_stride + t0 - tb];
    if (nk + nv > kRC) break;
    ++t1;
  }
  return t1;
}

// Issues cp.async copies of the chunk of tiles [t0, t1) into st.
__device__ __forceinline__ void stage_chunk(Stage& st, const CArgs& a, const uint8_t* comp, const int* pf,
                                            int pf_stride, int h, int tb, int t0, int t1) {
  const int tok0 = t0 * kTile, tok1 = min(a.N, t1 * kTile);
  const int ntok = tok1 - tok0, nt = t1 - t0;
  const uint8_t* codes = comp + a.L.off_res_codes;
  const uint16_t* sig = reinterpret_cast<const uint16_t*>(comp + a.L.off_res_sigma);
  const RecRange rK = rec_range(pf, t0 - tb, t1 - tb, a.R, kRC);
  const RecRange rV = rec_range(pf + pf_stride, t0 - tb, t1 - tb, a.R, kRC - rK.n);
  for (int side = 0; side < 2; ++side) {
    const uint32_t* tok = reinterpret_cast<const uint32_t*>(comp + a.L.off_tok) + ((int64_t)side * a.H + h) * a.N;
    const uint32_t* bm = reinterpret_cast<const uint32_t*>(comp + a.L.off_bitmap) +
                         ((int64_t)side * a.H + h) * a.n_tiles * 4;
    for (int i = threadIdx.x; i < ntok; i += kThreads) cp_async4(&st.tok[side][i], tok + tok0 + i);
    for (int i = threadIdx.x; i < nt; i += kThreads) cp_async16(&st.bm[side][4 * i], bm + (int64_t)(t0 + i) * 4);
    const RecRange& rr = side ? rV : rK;
    uint8_t* dst = st.codes + (side ? rK.n * kCodeBytes : 0);
    for (int i = threadIdx.x; i < 2 * rr.n; i += kThreads)
      cp_async16(dst + 16 * i, codes + rr.r0 * kCodeBytes + 16 * i);
    // scales: whole 4-byte words from the even record w0; a last record that
    // ends the array on an odd count is read on its own
    const int64_t end = rr.r0 + rr.n;
    const int64_t words = (end - rr.w0) / 2;
    for (int i = threadIdx.x; i < words; i += kThreads) cp_async4(&st.sig[side][2 * i], sig + rr.w0 + 2 * i);
    if ((end - rr.w0) & 1) {
      if (threadIdx.x == 0) st.sig[side][end - 1 - rr.w0] = sig[end - 1];
    }
  }
}

// Mask of the valid tokens (index < nt) of bitmap word w.
__device__ __forceinline__ uint32_t word_mask(int w, int nt) {
  const int lo = 32 * w;
  if (nt >= lo + 32) return 0xffffffffu;
  if (nt <= lo) return 0u;
  return (1u << (nt - lo)) - 1u;
}

template <typename T, int GP>
__global__ void __launch_bounds__(kThreads, GP <= 4 ? 2 : 1) decode_cluster_kernel(CArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int G = a.G, k = a.k;
  const uint32_t C = cluster_size(), r = cluster_rank();
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kc = (k + (int)C - 1) / (int)C;
  const int tpc = (a.n_tiles + (int)C - 1) / (int)C;
  const SmemPlan sp = smem_plan(G, k, tpc, kc, (int)sizeof(T));
  float4* lut = reinterpret_cast<float4*>(smem + sp.lut);
  Stage& st = *reinterpret_cast<Stage*>(smem + sp.stage);
  int* pf = reinterpret_cast<int*>(smem + sp.pf);        // [2][tpc + 1]
  const int pf_stride = tpc + 1;
  float* P = reinterpret_cast<float*>(smem + sp.P);
  float* W = reinterpret_cast<float*>(smem + sp.W);
  float* rbuf = reinterpret_cast<float*>(smem + sp.rbuf);  // [kRC][GP] per-record values
  T* vsl = reinterpret_cast<T*>(smem + sp.vsl);
  float* zred = reinterpret_cast<float*>(smem + sp.zred);
  float* oacc = reinterpret_cast<float*>(smem + sp.oacc);
  float* ofin = reinterpret_cast<float*>(smem + sp.ofin);
  float* misc = reinterpret_cast<float*>(smem + sp.misc);
  float* mrun = misc;                   // [8]   running max (log2 units)
  float* lsum = misc + 8;               // [8]   softmax denominator of this CTA
  float* fac = misc + 16;               // [8]   rescale factor of the current chunk
  float* Lfin = misc + 24;              // [8]   merged denominator
  float* scl = misc + 32;               // [kMaxC][8] per-CTA merge scale
  float* pm = scl + kMaxC * 8;          // [kMaxC][8] peers' running max
  float* pl = pm + kMaxC * 8;           // [kMaxC][8] peers' denominators
  float* red = pl + kMaxC * 8;          // [kWarps][8] block reductions

  const uint8_t* comp = a.comp + (int64_t)b * a.stride;
  const T* qg = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.H * G + (int64_t)h * G) * kD;
  const T* ancK = reinterpret_cast<const T*>(comp + a.L.off_anchors_k) + (int64_t)h * k * kD;
  const T* ancV = reinterpret_cast<const T*>(comp + a.L.off_anchors_v) + (int64_t)h * k * kD;

  // token tiles of this CTA and anchor slots of its slice
  const int tb = (int)((int64_t)a.n_tiles * r / C), te = (int)((int64_t)a.n_tiles * (r + 1) / C);
  const int s0 = min(k, (int)r * kc), s1 = min(k, s0 + kc), nsl = s1 - s0;
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // ---- prologue: every global load first (tile prefixes and value-anchor
  // slice by cp.async, query and this warp's anchor keys into registers),
  // then tables, rotated query and P of this CTA's slots
  for (int side = 0; side < 2; ++side) {
    const int* pfg = reinterpret_cast<const int*>(comp + a.L.off_tile_prefix) + ((int64_t)side * a.H + h) * (a.n_tiles + 1);
    for (int i = tid; i <= te - tb; i += kThreads) cp_async4(&pf[side * pf_stride + i], pfg + tb + i);
  }
  {
    const int bytes = nsl * kD * (int)sizeof(T);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(ancV + (int64_t)s0 * kD);
    for (int i = tid; i < bytes / 16; i += kThreads) cp_async16(reinterpret_cast<uint8_t*>(vsl) + 16 * i, src + 16 * i);
  }
  cp_commit();
  const float isd = rsqrtf((float)kD);
  float qf[GP][4];                       // q * log2e / sqrt(D), this lane's 4 coordinates
#pragma unroll
  for (int j = 0; j < GP; ++j) {
    if (j < G) {
      load4<T>(qg + j * kD + lane * 4, qf[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) qf[j][e] *= isd * kLog2e;
    } else {
      qf[j][0] = qf[j][1] = qf[j][2] = qf[j][3] = 0.f;
    }
  }
  constexpr int kPB = 4;                 // anchor rows in flight per warp
  float af[kPB][4];
#pragma unroll
  for (int u = 0; u < kPB; ++u) {
    const int sl = s0 + warp + u * kWarps;
    if (sl < s1) load4<T>(ancK + (int64_t)sl * kD + lane * 4, af[u]);
  }
  float* qs = ofin;          // q * log2e / sqrt(D) until the merge
  float* qr = zred;          // H(s . q) * log2e / D until the merge
  float* Pown = rbuf;        // this CTA's slots of P [G][kc] until the first chunk
  for (int i = tid; i < 256 * kLutCopies; i += kThreads) {
    const int v = i / kLutCopies;
    lut[i] = make_float4(a.lev[v & 3], a.lev[(v >> 2) & 3], a.lev[(v >> 4) & 3], a.lev[(v >> 6) & 3]);
  }
  for (int i = tid; i < G * k; i += kThreads) W[i] = 0.f;
  for (int i = tid; i < G * kD; i += kThreads) oacc[i] = 0.f;
  if (tid < 8) { mrun[tid] = -INFINITY; lsum[tid] = 0.f; }
#pragma unroll
  for (int j = 0; j < GP; ++j) {          // warp j rotates head j (GP <= kWarps)
    if (j < G && j == warp) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qs[j * kD + lane * 4 + e] = qf[j][e];
        v[e] = a.naive ? qf[j][e] : qf[j][e] * sign_of(a, lane * 4 + e);
      }
      if (!a.naive) {                      // (uniform per launch)
        fwht128<float>(v);
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] *= isd;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) qr[j * kD + lane * 4 + e] = v[e];
    }
  }
  for (int base = s0 + warp; base < s1; base += kPB * kWarps) {
#pragma unroll
    for (int u = 0; u < kPB; ++u) {
      const int sl = base + u * kWarps;
      if (sl < s1) {
#pragma unroll
        for (int j = 0; j < GP; ++j) {
          if (j < G) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) d = fmaf(qf[j][e], af[u][e], d);
            d = warp_sum(d);
            if (lane == 0) Pown[j * kc + (sl - s0)] = d;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPB; ++u) {   // the next rows of this warp
      const int sl = base + kPB * kWarps + u * kWarps;
      if (sl < s1) load4<T>(ancK + (int64_t)sl * kD + lane * 4, af[u]);
    }
  }
  cp_wait<0>();
  __syncthreads();
  int t0 = tb, t1 = (te > tb) ? chunk_end(pf, pf_stride, tb, te, tb) : tb;
  if (t1 > t0) stage_chunk(st, a, comp, pf, pf_stride, h, tb, t0, t1);
  cp_commit();
  // P into every CTA of the cluster, once all of them have started (the
  // arrive is at kernel entry)
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  for (int i = tid; i < (int)C * G * nsl; i += kThreads) {
    const int rr = i / (G * nsl), jj = i % (G * nsl), j = jj / nsl, s = jj % nsl;
    float* dst = static_cast<float*>(__cluster_map_shared_rank(&P[j * k + s0 + s], (unsigned)rr));
    *dst = Pown[j * kc + s];
  }
  // per-lane rotated query coordinates (lane = code byte = 4 coordinates)
  float qv[GP][4];
#pragma unroll
  for (int j = 0; j < GP; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[j][e] = (j < G) ? qr[j * kD + lane * 4 + e] : 0.f;
  float2 z[GP][2];
#pragma unroll
  for (int j = 0; j < GP; ++j) z[j][0] = z[j][1] = make_float2(0.f, 0.f);
  float lpart[GP];
#pragma unroll
  for (int j = 0; j < GP; ++j) lpart[j] = 0.f;
  __syncthreads();
  cluster_sync();   // P complete in every CTA

  // Raises the running max of each head to the chunk's if it exceeds it by
  // kRescaleGap, rescaling W, Z, the tail sums and the partial sums.  `mine`
  // holds this thread's maximum per head (-inf if it has none).
  auto update_max = [&](const float (&mine)[GP]) {
#pragma unroll
    for (int j = 0; j < GP; ++j) {
      if (j < G) {
        const float m = warp_max(mine[j]);
        if (lane == 0) red[warp * 8 + j] = m;
      }
    }
    __syncthreads();
    if (tid < G) {
      float m = -INFINITY;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w * 8 + tid]);
      const float old = mrun[tid];
      float f = 1.f;
      if (m > old + kRescaleGap || old == -INFINITY) {
        f = (old == -INFINITY) ? 0.f : exp2f(old - m);
        mrun[tid] = m;
      }
      fac[tid] = f;
    }
    __syncthreads();
    bool any = false;
    for (int j = 0; j < G; ++j) any |= fac[j] != 1.f;
    if (any) {
      for (int i = tid; i < G * k; i += kThreads) W[i] *= fac[i / k];
      for (int i = tid; i < G * kD; i += kThreads) oacc[i] *= fac[i / kD];
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        const float f = (j < G) ? fac[j] : 1.f;
        lpart[j] *= f;
        z[j][0].x *= f; z[j][0].y *= f; z[j][1].x *= f; z[j][1].y *= f;
      }
      __syncthreads();
    }
  };

  // ---- token chunks
  const uint32_t lt_mask = (1u << lane) - 1u;
  while (t1 > t0) {
    cp_wait<0>();
    __syncthreads();
    const int nt = min(a.N, t1 * kTile) - t0 * kTile;
    const RecRange rK = rec_range(pf, t0 - tb, t1 - tb, a.R, kRC);
    const RecRange rV = rec_range(pf + pf_stride, t0 - tb, t1 - tb, a.R, kRC - rK.n);
    // prefix counts of the bitmap words (warp 0: keys, warp 1: values)
    if (warp < 2) {
      const int side = warp;
      const uint32_t w0 = st.bm[side][lane] & word_mask(lane, nt);
      int incl = __popc(w0);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      st.wpre[side][lane] = incl - __popc(w0);
      if (lane == 31) st.wpre[side][kWordsPC] = incl;
    }
    __syncthreads();
    const int nK = min(rK.n, st.wpre[0][kWordsPC]);
    const int nV = min(rV.n, st.wpre[1][kWordsPC]);
    // (a) anchor logits, residual ranks
    float s[kTPT][GP];
    int rankK[kTPT], rankV[kTPT];
    uint32_t xV[kTPT];
#pragma unroll
    for (int u = 0; u < kTPT; ++u) {
      const int i = tid + u * kThreads, wd = warp + u * kWarps;
      const uint32_t wK = st.bm[0][wd] & word_mask(wd, nt);
      const uint32_t wVv = st.bm[1][wd] & word_mask(wd, nt);
      rankK[u] = ((wK >> lane) & 1u) ? st.wpre[0][wd] + __popc(wK & lt_mask) : kRC;
      rankV[u] = ((wVv >> lane) & 1u) ? st.wpre[1][wd] + __popc(wVv & lt_mask) : kRC;
      xV[u] = 0u;
#pragma unroll
      for (int j = 0; j < GP; ++j) s[u][j] = -INFINITY;
      if (i < nt) {
        const uint32_t x = st.tok[0][i];
        const int slot = min((int)(x & 0xFFFFu), k - 1);
        const float g = half_bits_to_f(x >> 16);
#pragma unroll
        for (int j = 0; j < GP; ++j)
          if (j < G) s[u][j] = g * P[j * k + slot];
        xV[u] = st.tok[1][i];
      }
    }
    // (b) key residual logits, groups of RB records per warp, stored by rank
    {
      constexpr int RB = 32 / GP;
      const int64_t sk = rK.r0 - rK.w0;
      for (int g0 = warp * RB; g0 < nK; g0 += kWarps * RB) {
        float v[32];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
          const int rho = g0 + u;
          uint32_t byte = 0u;
          float sg = 0.f;
          if (rho < nK) {
            byte = st.codes[rho * kCodeBytes + lane];
            sg = half_bits_to_f(st.sig[0][rho + sk]);
          }
          const float4 lv = lut[byte * kLutCopies + (lane & (kLutCopies - 1))];
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            float d = qv[j][0] * lv.x;
            d = fmaf(qv[j][1], lv.y, d);
            d = fmaf(qv[j][2], lv.z, d);
            d = fmaf(qv[j][3], lv.w, d);
            v[u * GP + j] = d * sg;
          }
        }
        transpose_reduce32(v, lane);
        if (g0 + lane / GP < nK) rbuf[(g0 + lane / GP) * GP + lane % GP] = v[0];
      }
    }
    __syncthreads();
    // (c) key residual logits into the scores, chunk maximum
    float mine[GP];
#pragma unroll
    for (int j = 0; j < GP; ++j) mine[j] = -INFINITY;
#pragma unroll
    for (int u = 0; u < kTPT; ++u) {
      if (rankK[u] < nK) {
#pragma unroll
        for (int j = 0; j < GP; ++j) s[u][j] += rbuf[rankK[u] * GP + j];
      }
#pragma unroll
      for (int j = 0; j < GP; ++j) mine[j] = fmaxf(mine[j], s[u][j]);
    }
    update_max(mine);
    // (d) probabilities, value-anchor weights, value-record weights by rank
    {
      const int64_t sv = rV.r0 - rV.w0;
#pragma unroll
      for (int u = 0; u < kTPT; ++u) {
        const int i = tid + u * kThreads;
        if (i < nt) {
          const int slot = min((int)(xV[u] & 0xFFFFu), k - 1);
          const float g = half_bits_to_f(xV[u] >> 16);
          const bool rec = rankV[u] < nV;
          const float sg = rec ? half_bits_to_f(st.sig[1][rankV[u] + sv]) : 0.f;
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            if (j < G) {
              const float p = exp2f(s[u][j] - mrun[j]);
              lpart[j] += p;
              atomicAdd(&W[j * k + slot], p * g);
              if (rec) rbuf[rankV[u] * GP + j] = p * sg;
            }
          }
        }
      }
    }
    __syncthreads();
    // (e) value residuals: Z += (p sigma~) lev(c), lane = code byte
    {
      const uint8_t* vcodes = st.codes + rK.n * kCodeBytes;
      int rho = warp;
      for (; rho + 3 * kWarps < nV; rho += 4 * kWarps) {
        uint32_t byte[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) byte[u] = vcodes[(rho + u * kWarps) * kCodeBytes + lane];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 lv = lut[byte[u] * kLutCopies + (lane & (kLutCopies - 1))];
          const float2 l01 = make_float2(lv.x, lv.y), l23 = make_float2(lv.z, lv.w);
          const int rr = rho + u * kWarps;
#pragma unroll
          for (int j = 0; j < GP; ++j) {
            if (j < G) {
              const float w = rbuf[rr * GP + j];
              const float2 ww = make_float2(w, w);
              z[j][0] = __ffma2_rn(l01, ww, z[j][0]);
              z[j][1] = __ffma2_rn(l23, ww, z[j][1]);
            }
          }
        }
      }
      for (; rho < nV; rho += kWarps) {
        const uint32_t byte = vcodes[rho * kCodeBytes + lane];
        const float4 lv = lut[byte * kLutCopies + (lane & (kLutCopies - 1))];
        const float2 l01 = make_float2(lv.x, lv.y), l23 = make_float2(lv.z, lv.w);
#pragma unroll
        for (int j = 0; j < GP; ++j) {
          if (j < G) {
            const float w = rbuf[rho * GP + j];
            const float2 ww = make_float2(w, w);
            z[j][0] = __ffma2_rn(l01, ww, z[j][0]);
            z[j][1] = __ffma2_rn(l23, ww, z[j][1]);
          }
        }
      }
    }
    __syncthreads();
    // next chunk
    t0 = t1;
    t1 = (t0 < te) ? chunk_end(pf, pf_stride, tb, te, t0) : t0;
    if (t1 > t0) stage_chunk(st, a, comp, pf, pf_stride, h, tb, t0, t1);
    cp_commit();
  }
  cp_wait<0>();
  __syncthreads();

  // ---- exact tail tokens, split over the cluster (scores in rbuf [G][256])
  if (a.tail_len > 0) {
    float* ts = rbuf;
    const int per = (a.tail_len + (int)C - 1) / (int)C;
    const int ta = min(a.tail_len, (int)r * per), tz = min(a.tail_len, ta + per);
    const T* Kt = reinterpret_cast<const T*>(a.Kt) + ((int64_t)b * a.H + h) * a.tail_cap * kD;
    const T* Vt = reinterpret_cast<const T*>(a.Vt) + ((int64_t)b * a.H + h) * a.tail_cap * kD;
    for (int base = ta; base < tz; base += kThreads) {
      const int nt = min(kThreads, tz - base);
      for (int i = warp; i < nt; i += kWarps) {
        float kf[4];
        load4<T>(Kt + (int64_t)(base + i) * kD + lane * 4, kf);
        for (int j = 0; j < G; ++j) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) d = fmaf(qs[j * kD + lane * 4 + e], kf[e], d);
          d = warp_sum(d);
          if (lane == 0) ts[j * kThreads + i] = d;
        }
      }
      __syncthreads();
      float mine[GP];
#pragma unroll
      for (int j = 0; j < GP; ++j) mine[j] = (tid < nt && j < G) ? ts[j * kThreads + tid] : -INFINITY;
      update_max(mine);
      if (tid < nt) {
#pragma unroll
        for (int j = 0; j < GP; ++j) {
          if (j < G) {
            const float p = exp2f(mine[j] - mrun[j]);
            ts[j * kThreads + tid] = p;
            lpart[j] += p;
          }
        }
      }
      __syncthreads();
      for (int i = warp; i < nt; i += kWarps) {
        float vf[4];
        load4<T>(Vt + (int64_t)(base + i) * kD + lane * 4, vf);
        for (int j = 0; j < G; ++j) {
          const float p = ts[j * kThreads + i];
#pragma unroll
          for (int e = 0; e < 4; ++e) atomicAdd(&oacc[j * kD + lane * 4 + e], p * vf[e]);
        }
      }
      __syncthreads();
    }
  }

  // ---- per-CTA totals: each warp's Z into the (free) stage buffer, summed
  // over the warps into zred (qr is no longer needed); l into lsum
  {
    float* zw = reinterpret_cast<float*>(&st);       // [kWarps][G][kD]
#pragma unroll
    for (int j = 0; j < GP; ++j) {
      if (j < G) {
        *reinterpret_cast<float4*>(&zw[(warp * G + j) * kD + lane * 4]) =
            make_float4(z[j][0].x, z[j][0].y, z[j][1].x, z[j][1].y);
        const float l = warp_sum(lpart[j]);
        if (lane == 0) red[warp * 8 + j] = l;
      }
    }
    __syncthreads();
    for (int i = tid; i < G * kD; i += kThreads) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) acc += zw[w * G * kD + i];
      zred[i] = acc;
    }
    if (tid < G) {
      float l = 0.f;
      for (int w = 0; w < kWarps; ++w) l += red[w * 8 + tid];
      lsum[tid] = l;
    }
  }
  __syncthreads();
  cluster_sync();   // every CTA's (mrun, lsum, W, zred, oacc) final

  // merge scales scl[r'][j] = 2^(m_r' - M_j) and the merged denominator
  for (int i = tid; i < (int)C * G; i += kThreads) {
    const int rr = i / G, j = i % G;
    pm[rr * 8 + j] = *peer(&mrun[j], (uint32_t)rr);
    pl[rr * 8 + j] = *peer(&lsum[j], (uint32_t)rr);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (uint32_t rr = 0; rr < C; ++rr) M = fmaxf(M, pm[rr * 8 + tid]);
    float Lj = 0.f;
    for (uint32_t rr = 0; rr < C; ++rr) {
      const float m = pm[rr * 8 + tid];
      const float sc = (m == -INFINITY) ? 0.f : exp2f(m - M);
      scl[rr * 8 + tid] = sc;
      Lj = fmaf(pl[rr * 8 + tid], sc, Lj);
    }
    Lfin[tid] = Lj;
  }
  __syncthreads();
  // value-anchor weights of this CTA's slot slice (into P, which nobody
  // reads any more), then W V_a
  float* wt = P;
  for (int i = tid; i < G * nsl; i += kThreads) {
    const int j = i / nsl, sl = s0 + i % nsl;
    float w = 0.f;
#pragma unroll 4
    for (uint32_t rr = 0; rr < C; ++rr) w = fmaf(*peer(&W[j * k + sl], rr), scl[rr * 8 + j], w);
    wt[j * kc + (sl - s0)] = w;
  }
  __syncthreads();
  for (int i = tid; i < G * kD; i += kThreads) {
    const int j = i / kD, d = i % kD;
    float o = 0.f;
    for (int sl = 0; sl < nsl; ++sl) o = fmaf(wt[j * kc + sl], to_f<T>(vsl[sl * kD + d]), o);
    ofin[i] = o;
  }
  // residual sums and exact tail of the heads this CTA owns (j = r mod C),
  // summed over the cluster into rbuf
  const int n_own = (G - (int)r + (int)C - 1) / (int)C;   // heads r, r + C, ...
  for (int i = tid; i < n_own * 2 * kD; i += kThreads) {
    const int jj = i / (2 * kD), kind = (i / kD) & 1, d = i % kD;
    const int j = (int)r + jj * (int)C;
    const float* src = kind ? oacc : zred;
    float acc = 0.f;
#pragma unroll 4
    for (uint32_t rr = 0; rr < C; ++rr) acc = fmaf(*peer(&src[j * kD + d], rr), scl[rr * 8 + j], acc);
    rbuf[i] = acc;
  }
  __syncthreads();
  for (int jj = warp; jj < n_own; jj += kWarps) {
    const int j = (int)r + jj * (int)C;
    float zv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) zv[e] = rbuf[jj * 2 * kD + lane * 4 + e];
    if (!a.naive) {                        // rotate the value residuals back (uniform per launch)
      fwht128<float>(zv);
#pragma unroll
      for (int e = 0; e < 4; ++e) zv[e] *= isd * sign_of(a, lane * 4 + e);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = lane * 4 + e;
      ofin[j * kD + d] += zv[e] + rbuf[jj * 2 * kD + kD + d];
    }
  }
  __syncthreads();
  cluster_sync();   // partial outputs final
  {
    const int total = G * kD, per = (total + (int)C - 1) / (int)C;
    const int i0 = (int)r * per, i1 = min(total, i0 + per);
    float* out = a.out + ((int64_t)b * a.H * G + (int64_t)h * G) * kD;
    for (int i = i0 + tid; i < i1; i += kThreads) {
      float o = 0.f;
#pragma unroll 4
      for (uint32_t rr = 0; rr < C; ++rr) o += *peer(&ofin[i], rr);
      out[i] = o / Lfin[i / kD];
    }
  }
  cluster_sync();   // no CTA leaves while a peer may still read its shared memory
}

struct ClusterCfg {
  int C = 0;
  int smem = 0;
};

template <typename T, int GP>
cudaError_t launch_t(const CArgs& a, int batch, const ClusterCfg& cfg, cudaStream_t s) {
  auto kern = decode_cluster_kernel<T, GP>;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(cfg.C, a.H, batch);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = cfg.smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cfg.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, a);
}

// Sets the kernel's attributes (the full 227 KB of dynamic shared memory,
// clusters above 8 CTAs) and returns how many clusters of C CTAs using `smem`
// bytes each the device can keep resident at once (0: cannot launch).
template <typename T, int GP>
int prepare_and_count(int C, int smem) {
  auto kern = decode_cluster_kernel<T, GP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    if (C > 8) return 0;
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(C, 1, 1);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &lc) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <typename T>
int prepare_and_count_g(int GP, int C, int smem) {
  switch (GP) {
    case 1: return prepare_and_count<T, 1>(C, smem);
    case 2: return prepare_and_count<T, 2>(C, smem);
    case 4: return prepare_and_count<T, 4>(C, smem);
    default: return prepare_and_count<T, 8>(C, smem);
  }
}


int plan_bytes(const Plan& pl, int C) {
  return smem_plan(pl.G, pl.k, (pl.n_tiles + C - 1) / C, (pl.k + C - 1) / C, pl.elem).total;
}

// Shared memory of a C-CTA cluster fits: the plan within 227 KB, and a CTA's
// slots of P fit the record buffer that holds them in the prologue.
bool fits(const Plan& pl, int C) {
  if ((pl.k + C - 1) / C > kRC) return false;
  return plan_bytes(pl, C) <= 227 * 1024;
}

// Cluster size for `units` (sequence, head) pairs: among C = 16, 8, 4, 2, 1
// whose shared-memory plan fits and that leave every CTA a tile, the one with
// the most CTAs per wave of resident clusters, C / ceil(units / resident(C));
// on a tie the smaller C (fewer waves).
// The kernel attributes are set as a side effect; cached per device and shape
// (the attributes are the same for every shape).
int choose_cluster(const Plan& pl, int units, ClusterCfg* cfg) {
  struct Entry { int dev, dtype, G, k, n_tiles, units, C, smem; };
  static std::mutex mu;
  static Entry cache[64];
  static int n_cache = 0, next = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ANCHORKV_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_cache; ++i) {
    const Entry& e = cache[i];
    if (e.dev == dev && e.dtype == pl.p.dtype && e.G == pl.G && e.k == pl.k && e.n_tiles == pl.n_tiles &&
        e.units == units) {
      cfg->C = e.C; cfg->smem = e.smem;
      return cfg->C ? ANCHORKV_OK : ANCHORKV_EUNSUPPORTED;
    }
  }
  const int GP = gp_of(pl.G);
  int best = 0, best_smem = 0;
  double best_score = 0.0;
  for (int C = kMaxC; C >= 1; C >>= 1) {
    if (C > pl.n_tiles && C > 1) continue;
    if (!fits(pl, C)) continue;
    const int smem = plan_bytes(pl, C);
    const int n = pl.p.dtype == ANCHORKV_BF16 ? prepare_and_count_g<__nv_bfloat16>(GP, C, smem)
                                              : prepare_and_count_g<float>(GP, C, smem);
    if (n < 1) continue;
    const int waves = (units + n - 1) / n;
    const double score = (double)C / waves;
    // equal scores: the smaller cluster, which runs in fewer waves
    if (score >= best_score) { best_score = score; best = C; best_smem = smem; }
  }
  Entry e{dev, pl.p.dtype, pl.G, pl.k, pl.n_tiles, units, best, best_smem};
  if (n_cache < 64) cache[n_cache++] = e;
  else cache[next++ % 64] = e;
  cfg->C = best; cfg->smem = best_smem;
  return best ? ANCHORKV_OK : ANCHORKV_EUNSUPPORTED;
}

}  // namespace

// G <= 8 query heads per KV head, and the shared-memory plan of the largest
// cluster fits one CTA.
bool decode_cluster_supported(const Plan& pl) {
  if (pl.G > 8) return false;
  return fits(pl, std::min(kMaxC, std::max(1, pl.n_tiles)));
}

int launch_decode_cluster(const Plan& pl, int batch, const char* comp, int64_t stride, const void* q,
                          const void* Kt, const void* Vt, int tail_len, int tail_cap, float* out, cudaStream_t s,
                          cudaError_t* err) {
  *err = cudaSuccess;
  ClusterCfg cfg;
  const int st = choose_cluster(pl, batch * pl.H, &cfg);
  if (st) return st;
  CArgs a;
  a.comp = reinterpret_cast<const uint8_t*>(comp);
  a.stride = stride;
  a.L = pl.L;
  a.N = pl.N; a.H = pl.H; a.G = pl.G; a.k = pl.k; a.n_tiles = pl.n_tiles;
  a.R = pl.R;
  a.lev[0] = (float)-pl.l2; a.lev[1] = (float)-pl.l1; a.lev[2] = (float)pl.l1; a.lev[3] = (float)pl.l2;
  for (int i = 0; i < 4; ++i) a.sign_bits[i] = pl.sign_bits[i];
  a.naive = naive_codec(pl);
  a.q = q; a.Kt = Kt; a.Vt = Vt; a.tail_len = tail_len; a.tail_cap = tail_cap; a.out = out;
  const int GP = gp_of(pl.G);
  stage_begin(kStDecodeCluster, s);
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    *err = GP == 1 ? launch_t<T, 1>(a, batch, cfg, s) : GP == 2 ? launch_t<T, 2>(a, batch, cfg, s)
         : GP == 4 ? launch_t<T, 4>(a, batch, cfg, s) : launch_t<T, 8>(a, batch, cfg, s);
  } else {
    using T = float;
    *err = GP == 1 ? launch_t<T, 1>(a, batch, cfg, s) : GP == 2 ? launch_t<T, 2>(a, batch, cfg, s)
         : GP == 4 ? launch_t<T, 4>(a, batch, cfg, s) : launch_t<T, 8>(a, batch, cfg, s);
  }
  stage_end(kStDecodeCluster, s, 1);
  return *err == cudaSuccess ? ANCHORKV_OK : ANCHORKV_ECUDA;
}

int decode_cluster_size(const Plan& pl, int batch, int* C, int* smem) {
  ClusterCfg cfg;
  const int st = choose_cluster(pl, batch * pl.H, &cfg);
  *C = cfg.C; *smem = cfg.smem;
  return st;
}

}  // namespace akv
