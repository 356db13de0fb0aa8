// Decode attention over compressed layouts: every (sequence, KV head) is cut
// into token slices that run on their own CTAs across the whole GPU, one
// launch per layer; the slices of a (sequence, head) are merged by whichever
// of its CTAs finishes last.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary": a FlashAttention-style decoder rebuilds tiles when they
// are consumed; "AnchorKV-adapted" (VeloxQuant-MLX), "Adaptation notes":
// tokens appended during decode stay at full precision.
//
// The rebuild is factored so that only compressed bytes are read per token
// (log2 units, q' = q log2(e) / sqrt(D)):
//   q' . K^_t = g^K_t P[i(t)] + sigma~_t <qr, lev(c_t)>,   P[a] = q' . K_a[a],
//   qr = H(s . q') / sqrt(D)      (H the unnormalised Sylvester matrix,
//                                  s the shared sign vector; qr = q' unrotated)
//   sum_t p_t V^_t = sum_a W[a] V_a[a] + s . H(Z) / sqrt(D),
//   W[a] = sum_{t: i(t)=a} p_t g^V_t,  Z = sum_t p_t sigma~_t lev(c_t).
//
// One CTA (256 threads) owns tiles [s tps, (s+1) tps) of its (sequence, head)
// and walks them in chunks of up to 512 tokens whose token words, bitmap
// words, residual codes and scales are staged into shared memory by cp.async
// (chunk c + 1 lands while chunk c is worked on).  Per chunk:
//   a. key-residual logits, one warp per 32/G records (lane = code byte,
//      levels from a 16-entry nibble table held in 16 bank-disjoint copies,
//      partial dots reduced by a transposed butterfly);
//   b. every token's logit for the G query heads (anchor term + its record's
//      residual term, the record found by a popcount in the bitmap word);
//   c. the chunk maximum; the running maximum moves only when the chunk beats
//      it by 2^8, so rescaling is rare;
//   d. probabilities, value-anchor weights W (shared-memory atomics) and the
//      weights p sigma~ of the chunk's value records;
//   e. value-residual sums Z in registers (lane = code byte, packed f32x2).
// The CTA that owns the last tile also takes the exact tail tokens.  At the
// end each CTA forms its partial output (W times the value anchors, Z turned
// back by one Hadamard transform) and, when the (sequence, head) has several
// slices, writes (max, sum, output) to the workspace; the last CTA to finish
// (an atomic ticket) merges them.
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace akv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCTMax = 512;                // most tokens per chunk
constexpr int kKT = kCTMax / kThreads;     // most tokens per thread and chunk
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleGap = 8.0f;        // log2 units
// anchor-weight terms in fixed point: below 2^kFixBits, split at 2^kSplit into
// two int32 parts whose sums over kFoldChunks chunks (at most 2^13 terms per
// slot) stay below 2^30
constexpr int kFixBits = 34;
constexpr int kSplit = 17;
constexpr float kSplitScale = (float)(1u << kSplit);
constexpr int kFoldChunks = 16;
// dynamic shared memory a CTA may plan for: the 227 KB opt-in limit less
// room for the kernel's static shared memory
constexpr int kSmemBudget = 227 * 1024 - 256;
// most slices per (sequence, head): the merge keeps 2 x S x G floats in the
// logit buffers (ct x G floats each, ct >= 128)
constexpr int kMaxSlices = 128;

struct FArgs {
  const uint8_t* comp;
  int64_t stride;
  int64_t total;                            // layout bytes of one sequence
  int64_t off_ak, off_av, off_tok, off_bm, off_pf, off_codes, off_sig;
  int N, H, G, k, kp, n_tiles;
  int64_t R;
  float lev[4];
  uint32_t sign_bits[4];
  int naive;
  const void* q;
  const void* Kt;
  const void* Vt;
  int tail_len, tail_cap;
  float* out;
  int S, tps, ct;                           // slices per (sequence, head), tiles per slice, tokens per chunk
  const float* rlg;                         // [B][R][GP] key-record logits from the pre-pass, or null
  float* part;                              // [B*H][S][GP*(2+128)] partial (max, sum, output)
  int* tickets;                             // [B*H] zeroed by the anchor-logit pre-kernel when S > 1
  float* Pw;                                // [B*H][kp][GP] anchor logits from the pre-kernel
  int rope;                                 // keys stored before the rotary map: rotate at decode
  double inv_freq[kD / 2];                  // rotary frequencies base^(-2i/D)
};

// Shared-memory carve-up (bytes), the same on host and device.
struct FPlan {
  int qs, qr, P, W, Wi, lut, pfs, wpre, red, rlog, wz, rot, rtok, stage, stage_bytes, total;
  // offsets inside one stage
  int s_codes, s_sig, s_tok, s_bm;
};

__host__ __device__ inline int fa_align(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline FPlan fplan(int GP, int kp, int ct, int tps, bool rope) {
  FPlan f;
  int cur = 0;
  // persistent small arrays first; from P on, the region is reused at the
  // end for the cross-warp sums ([2][warps][GP][128] floats)
  f.qs = cur; cur += GP * kD * 4;
  f.qr = cur; cur += GP * kD * 4;
  f.lut = cur; cur += 16 * 16 * 8;
  f.pfs = cur; cur = fa_align(cur + 2 * (tps + 1) * 4, 16);
  f.wpre = cur; cur = fa_align(cur + 2 * (ct / 32 + 1) * 4, 16);
  f.red = cur; cur = fa_align(cur + 2 * kWarps * GP * 4, 16);
  f.P = cur; cur += GP * kp * 4;
  f.W = cur; cur += GP * kp * 4;
  f.Wi = cur; cur += 2 * GP * kp * 4;
  f.rlog = cur; cur = fa_align(cur + ct * GP * 4, 16);
  f.wz = cur; cur = fa_align(cur + ct * GP * 8, 16);
  // rotary decode: (cos, sin) of b w_i (b < 32) and of the chunk's 32-token
  // blocks (T0 + 32 a) w_i, [32 + ct / 32][64] float2; the token of each
  // key record of the chunk, [ct] int
  f.rot = cur; cur += rope ? (32 + ct / 32) * (kD / 2) * 8 : 0;
  f.rtok = cur; cur += rope ? ct * 4 : 0;
  // stage: codes [2][ct][32], scales [2][ct + 8] (16-byte spans), token words
  // [2][ct + 4], bitmap words [2][ct / 32]
  int sc = 0;
  f.s_codes = sc; sc += 2 * ct * kCodeBytes;
  f.s_sig = sc; sc += 2 * (ct + 8) * 2;
  f.s_tok = sc; sc += 2 * (ct + 4) * 4;
  f.s_bm = sc; sc += 2 * (ct / 32) * 4;
  f.stage_bytes = fa_align(sc, 16);
  f.stage = fa_align(cur, 16);
  cur = f.stage + 2 * f.stage_bytes;
  if (cur < f.P + 2 * kWarps * GP * kD * 4) cur = f.P + 2 * kWarps * GP * kD * 4;
  f.total = fa_align(cur, 16);
  return f;
}

// Words of one slice's partial: (max, sum) per head padded to 16 bytes, then
// the GP x 128 outputs (16-byte aligned, for the merge's 16-byte copies).
__host__ __device__ constexpr int part_out(int GP) { return 4 * ((2 * GP + 3) / 4); }
__host__ __device__ constexpr int part_words(int GP) { return part_out(GP) + GP * kD; }

__host__ __device__ inline int gp_of(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : G <= 8 ? 8 : 16; }

// ---------------------------------------------------------------- small device helpers

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// 16-byte cp.async that copies the first `n` bytes of the source (0 < n <= 16)
// and fills the rest of the destination with zeros.
__device__ __forceinline__ void cp16(void* dst, const void* src, int n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copies layout bytes [off, off + n) of one sequence into shared memory
// starting at `dst` (16-byte aligned) from the 16-byte boundary at or below
// `off`: the first wanted byte lands at dst + (off & 15).  Units past the end
// of the layout are clamped (zero-filled).
__device__ __forceinline__ void copy_span(uint8_t* dst, const uint8_t* comp, int64_t total, int64_t off, int64_t n,
                                          int tid) {
  if (n <= 0) return;
  const int64_t a0 = off & ~(int64_t)15;
  const int units = (int)((off + n - a0 + 15) >> 4);
  for (int u = tid; u < units; u += kThreads) {
    const int64_t o = a0 + 16 * (int64_t)u;
    const int64_t left = total - o;
    if (left <= 0) continue;
    cp16(dst + 16 * u, comp + o, left >= 16 ? 16 : (int)left);
  }
}

// (cos, sin) of pos * w with the angle reduced modulo 2 pi in fp64 first.
__device__ __forceinline__ float2 rot_cs(double pos, double w) {
  const double two_pi = 6.283185307179586476925286766559, inv_two_pi = 0.15915494309189533576888376337251;
  const double ang = pos * w;
  float sn, cs;
  sincosf((float)(ang - two_pi * rint(ang * inv_two_pi)), &sn, &cs);
  return make_float2(cs, sn);
}

// The rotary map at position pos on this lane's four coordinates (lane l:
// 4l .. 4l + 3): coordinate d < D/2 pairs with d + D/2, held by lane l ^ 16,
// and turns by pos * base^(-2 (d mod D/2) / D).
__device__ __forceinline__ void rotate4(const FArgs& a, double pos, float (&x)[4], int lane) {
  const bool upper = lane >= 16;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 c = rot_cs(pos, a.inv_freq[4 * (lane & 15) + e]);
    const float other = __shfl_xor_sync(0xffffffffu, x[e], 16);
    x[e] = upper ? fmaf(other, c.y, x[e] * c.x) : fmaf(-other, c.y, x[e] * c.x);
  }
}

// Frequency of entry i of a rotary table row ([2][16] words of two (cos,
// sin) pairs: word (j, l) holds frequencies 4 l + 2 j and 4 l + 2 j + 1).
__device__ __forceinline__ int rot_freq(int i) {
  const int w = (i % (kD / 2)) >> 1;
  return 4 * (w & 15) + 2 * (w >> 4) + (i & 1);
}

// Coordinates 4 l + e and 64 + 4 l + e (e < 4) of one row, kept raw until used.
template <typename T> struct Row8;
template <> struct Row8<__nv_bfloat16> {
  uint2 lo, hi;
  __device__ __forceinline__ void load(const __nv_bfloat16* row) {
    lo = *reinterpret_cast<const uint2*>(row);
    hi = *reinterpret_cast<const uint2*>(row + kD / 2);
  }
  __device__ __forceinline__ void to_f(float (&x)[8]) const {
    x[0] = __uint_as_float(lo.x << 16); x[1] = __uint_as_float(lo.x & 0xFFFF0000u);
    x[2] = __uint_as_float(lo.y << 16); x[3] = __uint_as_float(lo.y & 0xFFFF0000u);
    x[4] = __uint_as_float(hi.x << 16); x[5] = __uint_as_float(hi.x & 0xFFFF0000u);
    x[6] = __uint_as_float(hi.y << 16); x[7] = __uint_as_float(hi.y & 0xFFFF0000u);
  }
};
template <> struct Row8<float> {
  float4 lo, hi;
  __device__ __forceinline__ void load(const float* row) {
    lo = *reinterpret_cast<const float4*>(row);
    hi = *reinterpret_cast<const float4*>(row + kD / 2);
  }
  __device__ __forceinline__ void to_f(float (&x)[8]) const {
    x[0] = lo.x; x[1] = lo.y; x[2] = lo.z; x[3] = lo.w;
    x[4] = hi.x; x[5] = hi.y; x[6] = hi.z; x[7] = hi.w;
  }
};

// Turns the pairs (x[e], x[4 + e]) of a half-warp row by the angles of one
// table row (lane l16's two words) and returns the G dot products with the
// turned query qa (coordinates in the same order) into v[g].
template <int GP>
__device__ __forceinline__ void turn_dot(const float (&x)[8], const float4 c01, const float4 c23,
                                         const float2 (&qa)[GP][4], float* v) {
  const float cb[4] = {c01.x, c01.z, c23.x, c23.z}, sb[4] = {c01.y, c01.w, c23.y, c23.w};
  float xr[4], yr[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    xr[e] = fmaf(x[e], cb[e], -x[4 + e] * sb[e]);
    yr[e] = fmaf(x[4 + e], cb[e], x[e] * sb[e]);
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    float2 d = __fmul2_rn(make_float2(xr[0], xr[1]), qa[g][0]);
    d = __ffma2_rn(make_float2(xr[2], xr[3]), qa[g][1], d);
    d = __ffma2_rn(make_float2(yr[0], yr[1]), qa[g][2], d);
    d = __ffma2_rn(make_float2(yr[2], yr[3]), qa[g][3], d);
    v[g] = d.x + d.y;
  }
}

// Unnormalised Walsh-Hadamard transform of a 128-vector spread over a
// half-warp: lane l (of 16) holds coordinates 4 l + e in x[e] and
// 64 + 4 l + e in x[4 + e] (e < 4).  Coordinate bits 0, 1 and 6 are register
// bits, bits 2 .. 5 the lane bits; both halves of the warp must call it.
__device__ __forceinline__ void fwht128_half(float (&x)[8], int lane) {
#pragma unroll
  for (int m = 1; m < 8; m <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!(e & m)) {
        const float u = x[e], v = x[e | m];
        x[e] = u + v;
        x[e | m] = u - v;
      }
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) {
    const float sg = (lane & m) ? -1.f : 1.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = fmaf(x[e], sg, __shfl_xor_sync(0xffffffffu, x[e], m));
  }
}

// GP consecutive floats of shared memory (16-byte aligned for GP >= 4).
template <int GP>
__device__ __forceinline__ void load_slot(const float* src, float (&v)[GP]) {
  if constexpr (GP >= 4) {
#pragma unroll
    for (int j = 0; j < GP / 4; ++j) {
      const float4 t = reinterpret_cast<const float4*>(src)[j];
      v[4 * j] = t.x; v[4 * j + 1] = t.y; v[4 * j + 2] = t.z; v[4 * j + 3] = t.w;
    }
  } else if constexpr (GP == 2) {
    const float2 t = *reinterpret_cast<const float2*>(src);
    v[0] = t.x; v[1] = t.y;
  } else {
    v[0] = src[0];
  }
}

// GP consecutive float2 of shared memory (16-byte aligned for GP >= 2).
template <int GP>
__device__ __forceinline__ void load_pairs(const float2* src, float2 (&v)[GP]) {
  if constexpr (GP >= 2) {
#pragma unroll
    for (int j = 0; j < GP / 2; ++j) {
      const float4 t = reinterpret_cast<const float4*>(src)[j];
      v[2 * j] = make_float2(t.x, t.y);
      v[2 * j + 1] = make_float2(t.z, t.w);
    }
  } else {
    v[0] = src[0];
  }
}

// One contiguous global -> shared copy by the bulk-copy engine (16-byte
// aligned addresses, size a multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

// Brings the 128-byte line at p into L2 (no register result, no wait).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float sign_of(const FArgs& a, int d) {
  return ((a.sign_bits[d >> 5] >> (d & 31)) & 1u) ? -1.f : 1.f;
}

// Eight consecutive elements (8 hl .. 8 hl + 7) of row `row` kept raw until
// used; rows at or past `rows` read as zeros.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  using type = uint4;
  __device__ __forceinline__ static uint4 load(const __nv_bfloat16* base, int row, int rows, int hl) {
    return row < rows ? *reinterpret_cast<const uint4*>(base + (int64_t)row * kD + 8 * hl) : make_uint4(0u, 0u, 0u, 0u);
  }
  __device__ __forceinline__ static void to_f2(const uint4 v, float2 (&o)[4]) {
    o[0] = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u));
    o[1] = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
    o[2] = make_float2(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u));
    o[3] = make_float2(__uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
  }
};
template <> struct Raw8<float> {
  struct type { float4 a, b; };
  __device__ __forceinline__ static type load(const float* base, int row, int rows, int hl) {
    type t;
    if (row < rows) {
      t.a = *reinterpret_cast<const float4*>(base + (int64_t)row * kD + 8 * hl);
      t.b = *reinterpret_cast<const float4*>(base + (int64_t)row * kD + 8 * hl + 4);
    } else {
      t.a = t.b = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return t;
  }
  __device__ __forceinline__ static void to_f2(const type& v, float2 (&o)[4]) {
    o[0] = make_float2(v.a.x, v.a.y); o[1] = make_float2(v.a.z, v.a.w);
    o[2] = make_float2(v.b.x, v.b.y); o[3] = make_float2(v.b.z, v.b.w);
  }
};

// Sums V values over the 16 lanes of each half-warp, transposed: afterwards
// lane l holds the total of value (l & 15) / (16 / V).
template <int V>
__device__ __forceinline__ void transpose_reduce16(float (&v)[V], int lane) {
  int n = V;
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) {
    if (n > 1) {
      const int hf = n / 2;
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i)
        if (i < hf) {
          const float keep = up ? v[i + hf] : v[i];
          const float send = up ? v[i] : v[i + hf];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      n = hf;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}

// ---------------------------------------------------------------- anchor logits

constexpr int kPSlots = 64;   // slots per CTA of the anchor-logit pre-kernel

// P = q . K_a (log2 units) of every slot, for each (sequence, head): CTA
// (x, bh) takes slots [64 x, 64 x + 64), heads in passes of up to 8.  A
// half-warp per slot, 8 coordinates per lane (the query's 8 x 8 values in
// registers, one 16-byte row load), and a 16-lane transposed reduction of the
// dot products.  Block x = 0 also clears the (sequence, head)'s merge ticket.
// The decode is launched as a programmatic dependent of this kernel.
template <typename T, int GP>
__global__ void __launch_bounds__(kThreads) anchor_logit_kernel(FArgs a) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ __align__(16) float qs[GP * kD];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H, G = a.G, kp = a.kp;
  if (blockIdx.x == 0 && tid == 0 && a.tickets) a.tickets[bh] = 0;
  if (a.rope) return;            // the rotary decode has no per-slot logits
  const int s0 = blockIdx.x * kPSlots, s1 = min(a.k, s0 + kPSlots);
  const uint8_t* comp = a.comp + (int64_t)b * a.stride;
  {
    const T* q = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.H * G + (int64_t)h * G) * kD;
    const float qscale = kLog2e * rsqrtf((float)kD);
    for (int i = tid; i < GP * kD; i += kThreads) {
      const int g = i / kD;
      qs[i] = g < G ? to_f(q[(int64_t)g * kD + (i % kD)]) * qscale : 0.f;
    }
  }
  __syncthreads();
  float* Pw = a.Pw + (int64_t)bh * kp * GP;
  constexpr int HG = GP < 8 ? GP : 8;
#pragma unroll 1
  for (int g0 = 0; g0 < GP; g0 += HG)
  {
    // half-warp per slot, 8 coordinates per lane: the query's 8 x GP values
    // stay in registers, the row is one 16-byte load (bf16), and the GP dot
    // products meet in a 16-lane transposed reduction
    const int half = lane >> 4, hl = lane & 15;
    float2 q2[HG][4];
#pragma unroll
    for (int g = 0; g < HG; ++g) {
      const float4 a4 = *reinterpret_cast<const float4*>(qs + (g0 + g) * kD + 8 * hl);
      const float4 b4 = *reinterpret_cast<const float4*>(qs + (g0 + g) * kD + 8 * hl + 4);
      q2[g][0] = make_float2(a4.x, a4.y); q2[g][1] = make_float2(a4.z, a4.w);
      q2[g][2] = make_float2(b4.x, b4.y); q2[g][3] = make_float2(b4.z, b4.w);
    }
    const T* Ka = reinterpret_cast<const T*>(comp + a.off_ak) + (int64_t)h * a.k * kD;
    using R8 = Raw8<T>;
    // four slot pairs per step, the next step's rows in flight meanwhile
    constexpr int kPS = 4;
    typename R8::type nx[kPS];
    const int npair = (s1 - s0 + 1) / 2;
    auto fetch = [&](int sp0) {
#pragma unroll
      for (int u = 0; u < kPS; ++u) nx[u] = R8::load(Ka, s0 + 2 * (sp0 + u * kWarps) + half, s1, hl);
    };
    if (warp < npair) fetch(warp);
    for (int sp0 = warp; sp0 < npair; sp0 += kPS * kWarps) {
      typename R8::type cx[kPS];
#pragma unroll
      for (int u = 0; u < kPS; ++u) cx[u] = nx[u];
      if (sp0 + kPS * kWarps < npair) fetch(sp0 + kPS * kWarps);
#pragma unroll
      for (int u = 0; u < kPS; ++u) {
        float2 x2[4];
        R8::to_f2(cx[u], x2);
        float v[HG];
#pragma unroll
        for (int g = 0; g < HG; ++g) {
          float2 acc = __fmul2_rn(x2[0], q2[g][0]);
          acc = __ffma2_rn(x2[1], q2[g][1], acc);
          acc = __ffma2_rn(x2[2], q2[g][2], acc);
          acc = __ffma2_rn(x2[3], q2[g][3], acc);
          v[g] = acc.x + acc.y;
        }
        transpose_reduce16<HG>(v, lane);
        const int slot = s0 + 2 * (sp0 + u * kWarps) + half;
        if (slot < s1 && (hl % (16 / HG)) == 0) Pw[slot * GP + g0 + hl / (16 / HG)] = v[0];
      }
    }
  }
}

// ---------------------------------------------------------------- the kernel

template <typename T, int GP, bool ROPE>
__global__ void __launch_bounds__(kThreads, GP <= 4 ? 2 : 1) flash_decode_kernel(FArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H, s = blockIdx.x;
  const int G = a.G, kp = a.kp, ct = a.ct;
  const FPlan F = fplan(GP, kp, ct, a.tps, ROPE);
  float* qs = reinterpret_cast<float*>(sm + F.qs);       // [GP][128] q' (log2 units)
  float* qr = reinterpret_cast<float*>(sm + F.qr);       // [GP][128] rotated q'
  float* P = reinterpret_cast<float*>(sm + F.P);         // [GP][kp]
  // [GP][kp] anchor weights W: floats, plus the latest chunks' terms in
  // fixed point (value 2^-e (hi 2^kSplit + lo), native 32-bit atomics),
  // folded into the floats every kFoldChunks chunks and before any rescale
  float* Wt = reinterpret_cast<float*>(sm + F.W);
  int* Whi = reinterpret_cast<int*>(sm + F.Wi);
  int* Wlo = Whi + GP * kp;
  float2* lut = reinterpret_cast<float2*>(sm + F.lut);   // [16 nibbles][16 copies]
  int* pfs = reinterpret_cast<int*>(sm + F.pfs);         // [2][tps + 1]
  int* wpre = reinterpret_cast<int*>(sm + F.wpre);       // [2][ct/32 + 1]
  float* red = reinterpret_cast<float*>(sm + F.red);     // [2][kWarps][GP]
  float* rlog = reinterpret_cast<float*>(sm + F.rlog);   // [ct][GP] key-record logits by rank
  // [ct][GP] value-record weights by rank, each stored twice (an f32x2 operand)
  float2* wz2 = reinterpret_cast<float2*>(sm + F.wz);
  float* wz = reinterpret_cast<float*>(sm + F.wz);         // the merge's scratch

  const uint8_t* comp = a.comp + (int64_t)b * a.stride;
  const int t_beg = s * a.tps, t_end = min(a.n_tiles, t_beg + a.tps);
  const int nt = t_end - t_beg;
  const int n_chunks = (nt * kTile + ct - 1) / ct;
  const int tiles_pc = ct / kTile;
  const bool has_tail = (s == a.S - 1) && a.tail_len > 0;
  bool copy_failed = false;         // a chunk's bulk copy never completed (bounded wait)

  // ---- 1. prefixes of the slice's tiles, the query, the nibble table; first token words
  {
    // the anchor rows are read twice later (keys for P, values at the end):
    // start their trip to L2 now
    const int64_t arow = (int64_t)kD * sizeof(T), abytes = (int64_t)a.k * arow;
    const uint8_t* ak = comp + a.off_ak + (int64_t)h * abytes;
    const uint8_t* av = comp + a.off_av + (int64_t)h * abytes;
    for (int64_t o = (int64_t)tid * 128; o < abytes; o += (int64_t)kThreads * 128) {
      prefetch_l2(ak + o);
      prefetch_l2(av + o);
    }
    if (has_tail) {
      // the exact tail's rows too, read after the last chunk
      const int64_t tb = (int64_t)a.tail_len * kD * sizeof(T), base = ((int64_t)b * a.H + h) * a.tail_cap * kD * sizeof(T);
      for (int64_t o = (int64_t)tid * 128; o < tb; o += (int64_t)kThreads * 128) {
        prefetch_l2(reinterpret_cast<const uint8_t*>(a.Kt) + base + o);
        prefetch_l2(reinterpret_cast<const uint8_t*>(a.Vt) + base + o);
      }
    }
    const int* pf = reinterpret_cast<const int*>(comp + a.off_pf);
    for (int i = tid; i < 2 * (nt + 1); i += kThreads) {
      const int side = i / (nt + 1), j = i % (nt + 1);
      int64_t v = pf[((int64_t)side * a.H + h) * (a.n_tiles + 1) + t_beg + j];
      v = v < 0 ? 0 : (v > a.R ? a.R : v);
      pfs[side * (a.tps + 1) + j] = (int)v;
    }
    const T* q = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.H * G + (int64_t)h * G) * kD;
    const float qscale = kLog2e * rsqrtf((float)kD);
    for (int i = tid; i < GP * kD; i += kThreads) {
      const int g = i / kD;
      qs[i] = g < G ? to_f(q[(int64_t)g * kD + (i % kD)]) * qscale : 0.f;
    }
    if (tid < 256) {
      const int n = tid >> 4;
      lut[tid] = make_float2(a.lev[n & 3], a.lev[n >> 2]);
    }
  }
  // token words and bitmap words of a chunk (no prefix needed); records need the prefixes
  auto stage_of = [&](int c) -> uint8_t* { return sm + F.stage + (c & 1) * F.stage_bytes; };
  auto issue_words = [&](int c) {
    uint8_t* st = stage_of(c);
    const int c0 = t_beg + c * tiles_pc, c1 = min(t_end, c0 + tiles_pc);
    const int tok0 = c0 * kTile, tok1 = min(a.N, c1 * kTile);
    for (int side = 0; side < 2; ++side) {
      const int64_t toff = a.off_tok + 4 * (((int64_t)side * a.H + h) * a.N + tok0);
      copy_span(st + F.s_tok + side * (ct + 4) * 4, comp, a.total, toff, 4 * (int64_t)(tok1 - tok0), tid);
      const int64_t boff = a.off_bm + 16 * (((int64_t)side * a.H + h) * a.n_tiles + c0);
      copy_span(st + F.s_bm + side * (ct / 32) * 4, comp, a.total, boff, 16 * (int64_t)(c1 - c0), tid);
    }
  };
  // residual codes (and the pre-pass key logits) by the bulk-copy engine, one
  // instruction per section issued by thread 0 and completing on the stage's
  // barrier; the 2-byte scales by cp.async (their spans are not 16-byte aligned)
  __shared__ __align__(8) uint64_t sbar[2];
  auto issue_records = [&](int c) {
    uint8_t* st = stage_of(c);
    const int j0 = c * tiles_pc, j1 = min(nt, j0 + tiles_pc);
    int r0s[2], ns[2];
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      r0s[side] = pfs[side * (a.tps + 1) + j0];
      const int n = pfs[side * (a.tps + 1) + j1] - r0s[side];
      ns[side] = n < 0 ? 0 : (n > ct ? ct : n);
    }
    const bool rlg_bulk = a.rlg && GP >= 4;   // 16-byte aligned rows of GP floats
    if (tid == 0) {
      tc::fence_proxy_async_smem();   // the buffer's last generic reads precede these writes
      uint32_t bytes = (uint32_t)ns[1] * kCodeBytes;
      if (!a.rlg) bytes += (uint32_t)ns[0] * kCodeBytes;
      else if (rlg_bulk) bytes += (uint32_t)ns[0] * GP * 4;
      tc::mbar_expect_tx(&sbar[c & 1], bytes);
#pragma unroll
      for (int side = 0; side < 2; ++side)
        if (ns[side] > 0 && !(side == 0 && a.rlg))
          bulk_g2s(st + F.s_codes + side * ct * kCodeBytes, comp + a.off_codes + (int64_t)kCodeBytes * r0s[side],
                   (uint32_t)ns[side] * kCodeBytes, &sbar[c & 1]);
      if (rlg_bulk && ns[0] > 0)
        bulk_g2s(st + F.s_codes, a.rlg + ((int64_t)b * a.R + r0s[0]) * GP, (uint32_t)ns[0] * GP * 4, &sbar[c & 1]);
    }
    if (a.rlg && !rlg_bulk)
      copy_span(st + F.s_codes, reinterpret_cast<const uint8_t*>(a.rlg), (int64_t)(b + 1) * a.R * GP * 4,
                ((int64_t)b * a.R + r0s[0]) * GP * 4, (int64_t)ns[0] * GP * 4, tid);
#pragma unroll
    for (int side = 0; side < 2; ++side)
      if (!(side == 0 && a.rlg))
        copy_span(st + F.s_sig + side * (ct + 8) * 2, comp, a.total, a.off_sig + 2 * (int64_t)r0s[side],
                  2 * (int64_t)ns[side], tid);
  };
  if (tid == 0) {
    tc::mbar_init(&sbar[0], 1);
    tc::mbar_init(&sbar[1], 1);
    tc::fence_barrier_init();
  }
  issue_words(0);
  __syncthreads();
  issue_records(0);
  cp_commit();

  // ---- 2. rotated query and anchor logits P (while the copies fly); the
  //    rotary decode instead turns the query to its position N + tail_len
  //    and tabulates (cos, sin)(b w_i) for b < 32
  if constexpr (ROPE) {
    for (int g = warp; g < GP; g += kWarps) {
      float v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = qs[g * kD + 4 * lane + i];
      rotate4(a, (double)a.N + a.tail_len, v, lane);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) qs[g * kD + 4 * lane + i] = v[i];
    }
    // rows of 64 entries as [2][16] 16-byte words: word (j, l16) holds the
    // pairs of frequencies 4 l16 + 2 j and 4 l16 + 2 j + 1, so a half-warp's
    // read of one word per lane is 256 contiguous bytes
    float2* tb = reinterpret_cast<float2*>(sm + F.rot);
    for (int i = tid; i < 32 * (kD / 2); i += kThreads) tb[i] = rot_cs((double)(i / (kD / 2)), a.inv_freq[rot_freq(i)]);
  }
  for (int g = warp; g < GP && !ROPE; g += kWarps) {
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = qs[g * kD + 4 * lane + i];
    if (!a.naive) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] *= sign_of(a, 4 * lane + i);
      fwht128(v);
      const float r = rsqrtf((float)kD);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] *= r;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) qr[g * kD + 4 * lane + i] = v[i];
  }
  // anchor logits P = q . K_a of this (sequence, head), computed by the
  // pre-kernel that this launch depends on (programmatic dependent launch: the
  // prologue above overlapped it); its writes, the cleared ticket included,
  // are visible past this wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!ROPE) {
    const float* src = a.Pw + (int64_t)bh * kp * GP;
    for (int u = tid; u < GP * kp / 4; u += kThreads) cp16(P + 4 * u, src + 4 * u, 16);
    cp_commit();
  }
  for (int i = tid; i < GP * kp; i += kThreads) {
    Wt[i] = 0.f;
    Whi[i] = 0;
    Wlo[i] = 0;
  }

  // running state (identical in every thread): max per head; per-thread sums
  float mrun[GP], lsum[GP];
  float2 z01[GP], z23[GP];          // value-residual sums for dims 4 lane .. 4 lane + 3
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    mrun[g] = -INFINITY;
    lsum[g] = 0.f;
    z01[g] = make_float2(0.f, 0.f);
    z23[g] = make_float2(0.f, 0.f);
  }
  // W's fixed-point scale 2^e: a term p gamma 2^e with p <= 2^gap and
  // |gamma| < 2^eg stays below 2^kFixBits; split at 2^kSplit into two int32
  // parts, kFoldChunks chunks of terms fit either part's sum
  int eg = -1000;                   // no gamma seen yet
  float gbound = 0.f;               // 2^eg: |gamma| below it needs no rescale
  float wsc = 1.f, winv = 1.f;      // 2^e, 2^-e
  bool folded_all = true;           // no term since the last fold
  float2 qr01[GP], qr23[GP];
  __syncthreads();
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float4 t4 = *reinterpret_cast<const float4*>(qr + g * kD + 4 * lane);
    qr01[g] = make_float2(t4.x, t4.y);
    qr23[g] = make_float2(t4.z, t4.w);
  }
  const float2* lutc = lut + (lane & 15);

  // Adds the fixed-point parts into the float weights (times f[g] for head g
  // afterwards) and clears them.  Each thread touches its own entries only.
  auto fold = [&](const float (&f)[GP]) {
#pragma unroll
    for (int g = 0; g < GP; ++g)
      for (int i = tid; i < kp; i += kThreads) {
        const int j = g * kp + i, jt = i * GP + g;
        const float add = fmaf((float)Whi[j], kSplitScale, (float)Wlo[j]) * winv;
        Wt[jt] = (Wt[jt] + add) * f[g];
        Whi[j] = 0;
        Wlo[j] = 0;
      }
  };
  // Raises the running maximum of head g to ceil(cm[g]) when cm[g] beats it by
  // the gap (or on the first values), and the bound on |gamma| to the power of
  // two above gm (a new fixed-point scale).  CTA-uniform; the factors (exact
  // powers of two) are left in f, 1 where the maximum stayed.
  auto update_max = [&](const float (&cm)[GP], float gm, float (&f)[GP]) {
    bool any = false;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      f[g] = 1.f;
      if (mrun[g] == -INFINITY) {
        mrun[g] = ceilf(cm[g]);
      } else if (cm[g] > mrun[g] + kRescaleGap) {
        const float nm = ceilf(cm[g]);
        f[g] = exp2f(-fminf(nm - mrun[g], 200.f));
        mrun[g] = nm;
        any = true;
      }
    }
    const bool rescale = gm >= gbound;
    if (any || rescale) {
      // the parts so far go in at the old scale; a raised maximum rescales
      // the floats as well
      if (!folded_all || any) fold(f);
      folded_all = true;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        lsum[g] *= f[g];
        z01[g].x *= f[g]; z01[g].y *= f[g]; z23[g].x *= f[g]; z23[g].y *= f[g];
      }
      __syncthreads();
    }
    if (rescale) {
      eg = max(gm > 0.f ? (int)((__float_as_uint(gm) >> 23) & 255u) - 126 : -40, -40);   // gm < 2^eg
      gbound = __uint_as_float((uint32_t)(eg + 127) << 23);
      const int e = kFixBits - (int)kRescaleGap - eg;
      wsc = __uint_as_float((uint32_t)(e + 127) << 23);
      winv = __uint_as_float((uint32_t)(127 - e) << 23);
    }
  };
  // CTA-wide maximum per head of per-thread values (all threads get it).
  auto block_max = [&](float (&v)[GP], float (&out)[GP]) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float m = warp_max(v[g]);
      if (lane == 0) red[warp * GP + g] = m;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float m = red[g];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[w * GP + g]);
      out[g] = m;
    }
  };

  // CTA-wide maxima per head of per-thread values, and of one more value.
  auto block_max2 = [&](float (&v)[GP], float x, float (&out)[GP], float& xout) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float m = warp_max(v[g]);
      if (lane == 0) red[warp * (GP + 1) + g] = m;
    }
    const float mx = warp_max(x);
    if (lane == 0) red[warp * (GP + 1) + GP] = mx;
    __syncthreads();
#pragma unroll
    for (int g = 0; g <= GP; ++g) {
      float m = red[g];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[w * (GP + 1) + g]);
      if (g < GP) out[g] = m;
      else xout = m;
    }
  };

  // ---- 3. chunks
  for (int c = 0; c < n_chunks; ++c) {
    // chunk c has landed; past this barrier every thread is done with chunk
    // c - 1, so its buffer takes chunk c + 1 while chunk c is worked on
    cp_wait<0>();
    if (!tc::mbar_wait(&sbar[c & 1], (c >> 1) & 1)) copy_failed = true;
    __syncthreads();
    if (c + 1 < n_chunks) {
      issue_words(c + 1);
      issue_records(c + 1);
      cp_commit();
    }
    const uint8_t* st = stage_of(c);
    const uint8_t* codes = st + F.s_codes;
    const int j0 = c * tiles_pc, j1 = min(nt, j0 + tiles_pc);
    const int tok0 = (t_beg + j0) * kTile, ntok = min(a.N, (t_beg + j1) * kTile) - tok0;
    int rbase[2], nrec[2], sh_sig[2], sh_tok[2];
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      rbase[side] = pfs[side * (a.tps + 1) + j0];
      int n = pfs[side * (a.tps + 1) + j1] - rbase[side];
      nrec[side] = n < 0 ? 0 : (n > ct ? ct : n);
      sh_sig[side] = (int)((a.off_sig + 2 * (int64_t)rbase[side]) & 15) / 2;
      sh_tok[side] = (int)((a.off_tok + 4 * (((int64_t)side * a.H + h) * a.N + tok0)) & 15) / 4;
    }
    const uint32_t* bm0 = reinterpret_cast<const uint32_t*>(st + F.s_bm);
    const uint16_t* sig0 = reinterpret_cast<const uint16_t*>(st + F.s_sig);
    const uint32_t* tok0p = reinterpret_cast<const uint32_t*>(st + F.s_tok);
    const int nwords = (ntok + 31) >> 5;

    // a. bitmap word prefixes (warp = side) and key-residual logits
    if (warp < 2) {
      const int side = warp;
      const uint32_t w = lane < nwords ? bm0[side * (ct / 32) + lane] : 0u;
      int x = __popc(w);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane < ct / 32) wpre[side * (ct / 32 + 1) + lane + 1] = x;
      if (lane == 0) wpre[side * (ct / 32 + 1)] = 0;
      if (ROPE && side == 0) {
        // the token of every key record (rank), for the rotary residual pass
        int* rtok = reinterpret_cast<int*>(sm + F.rtok);
        int r = x - __popc(w);
        for (uint32_t m = w; m != 0u && r < nrec[0]; m &= m - 1u, ++r) rtok[r] = 32 * lane + __ffs(m) - 1;
      }
    }
    // key-record logits by rank: staged from the tensor-core pre-pass (sigma~
    // included), or computed here into rlog
    // (the rotary decode keeps its residual terms by rank in the wz buffer,
    // free until step d)
    const float* klg = ROPE ? reinterpret_cast<const float*>(sm + F.wz)
                     : a.rlg ? reinterpret_cast<const float*>(codes) +
                                   (int)((((int64_t)b * a.R + rbase[0]) * GP * 4) & 15) / 4
                             : rlog;
    if constexpr (ROPE) {
      // (cos, sin) of the chunk's 32-token blocks (T0 + 32 a) w_i
      float2* ta = reinterpret_cast<float2*>(sm + F.rot) + 32 * (kD / 2);
      for (int i = tid; i < (ct / 32) * (kD / 2); i += kThreads)
        ta[i] = rot_cs((double)tok0 + 32.0 * (i / (kD / 2)), a.inv_freq[rot_freq(i)]);
    }
    if (!ROPE && !a.rlg) {
      constexpr int RB = 32 / GP;
      const int nK = nrec[0];
      for (int base = warp * RB; base < nK; base += kWarps * RB) {
        float v[32];
#pragma unroll
        for (int i = 0; i < RB; ++i) {
          // records past nK (up to the batch's end, inside the chunk's buffer)
          // are computed from stale codes and not stored
          const uint32_t byte = codes[(base + i) * kCodeBytes + lane];
          const float2 l01 = lutc[(byte & 15u) * 16], l23 = lutc[(byte >> 4) * 16];
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            float2 t2 = __fmul2_rn(l01, qr01[g]);
            t2 = __ffma2_rn(l23, qr23[g], t2);
            v[i * GP + g] = t2.x + t2.y;
          }
        }
        transpose_reduce32(v, lane);
        const int r = base + lane / GP;
        if (r < nK) rlog[r * GP + (lane % GP)] = v[0] * half_bits_to_f(sig0[sh_sig[0] + r]);
      }
    }
    __syncthreads();

    if constexpr (ROPE) {
      // b'. rotary logits, on half-warps whose lane l16 holds coordinates
      //     4 l16 + e and 64 + 4 l16 + e (e < 4), so that each rotary pair
      //     (d, d + 64) sits in one lane.  Each warp takes 32-token blocks; the
      //     query (at its own position) is turned back once by the block's
      //     start T0 + 32 blk, and every key of the block is then turned only
      //     by its offset b = t mod 32 (one table row):
      //     - anchor terms: gamma~ times the dot product with the token's
      //       anchor row goes to rlog by token (the rows of the next TL
      //       tokens are in flight while TL tokens are worked on);
      //     - residual terms of the block's key records: the residual is
      //       rebuilt by one half-warp Hadamard transform; sigma~ times its
      //       dot product goes to klg by rank.
      //     Anchor terms: 16 / G tokens per half-warp step, the 16 G products
      //     finished by one transposed reduction.
      constexpr int TBH = 16 / GP;
      constexpr int TL0 = sizeof(T) == 2 ? 4 : 2;
      constexpr int TL = TBH < TL0 ? TBH : TL0;   // rows per load batch
      constexpr int BPS = TBH / TL;               // load batches per step
      constexpr int NS = 16 / TBH;                // steps per 32-token block
      const int half = lane >> 4, l16 = lane & 15;
      const T* Ka = reinterpret_cast<const T*>(comp + a.off_ak) + (int64_t)h * a.k * kD + 4 * l16;
      const float4* tbB = reinterpret_cast<const float4*>(sm + F.rot) + l16;   // [32][2][16]
      const float4* tbA = tbB + 32 * 32;                                       // [ct / 32][2][16]
      const int nK = nrec[0];
      const int* rtok = reinterpret_cast<const int*>(sm + F.rtok);
      float* rres = reinterpret_cast<float*>(sm + F.wz);
      // the shared signs and 1 / sqrt(D) of the inverse rotation
      float sg[8];
      {
        const float rs = rsqrtf((float)kD);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sg[e] = a.naive ? 1.f : sign_of(a, 4 * l16 + e) * rs;
          sg[4 + e] = a.naive ? 1.f : sign_of(a, kD / 2 + 4 * l16 + e) * rs;
        }
      }
      for (int blk = warp; blk * 32 < ntok; blk += kWarps) {
        float2 qa[GP][4];
        {
          const float4 c01 = tbA[blk * 32], c23 = tbA[blk * 32 + 16];
          const float ca[4] = {c01.x, c01.z, c23.x, c23.z}, sa[4] = {c01.y, c01.w, c23.y, c23.w};
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            const float4 x4 = *reinterpret_cast<const float4*>(qs + g * kD + 4 * l16);
            const float4 y4 = *reinterpret_cast<const float4*>(qs + g * kD + kD / 2 + 4 * l16);
            const float xs[4] = {x4.x, x4.y, x4.z, x4.w}, ys[4] = {y4.x, y4.y, y4.z, y4.w};
            float xq[4], yq[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              xq[e] = fmaf(xs[e], ca[e], ys[e] * sa[e]);
              yq[e] = fmaf(ys[e], ca[e], -xs[e] * sa[e]);
            }
            qa[g][0] = make_float2(xq[0], xq[1]); qa[g][1] = make_float2(xq[2], xq[3]);
            qa[g][2] = make_float2(yq[0], yq[1]); qa[g][3] = make_float2(yq[2], yq[3]);
          }
        }
        const int bend = min(ntok, blk * 32 + 32);
        // anchor terms: this half's tokens of step st are
        // blk * 32 + st * 2 TBH + half * TBH + [0, TBH); rows past bend are
        // read from stale token words (slots clamped) and not stored
        const int tb0 = blk * 32 + half * TBH;
        auto fetch = [&](int bi, Row8<T> (&r)[TL]) {
          const int t1 = tb0 + (bi / BPS) * 2 * TBH + (bi % BPS) * TL;
#pragma unroll
          for (int w = 0; w < TL; ++w)
            r[w].load(Ka + (int64_t)min((int)(tok0p[sh_tok[0] + t1 + w] & 0xFFFFu), a.k - 1) * kD);
        };
        Row8<T> cur[TL], nxt[TL];
        fetch(0, cur);
#pragma unroll 1
        for (int st = 0; st < NS && blk * 32 + st * 2 * TBH < bend; ++st) {
          float v[16];
#pragma unroll
          for (int j = 0; j < BPS; ++j) {
            const int bi = st * BPS + j;
            if (bi + 1 < NS * BPS) fetch(bi + 1, nxt);
#pragma unroll
            for (int w = 0; w < TL; ++w) {
              const int bo = (tb0 + st * 2 * TBH + j * TL + w) & 31;
              float x[8];
              cur[w].to_f(x);
              turn_dot<GP>(x, tbB[bo * 32], tbB[bo * 32 + 16], qa, v + (j * TL + w) * GP);
            }
#pragma unroll
            for (int w = 0; w < TL; ++w) cur[w] = nxt[w];
          }
          transpose_reduce16<16>(v, lane);
          const int t = tb0 + st * 2 * TBH + l16 / GP;
          if (t < bend) rlog[t * GP + l16 % GP] = v[0] * half_bits_to_f(tok0p[sh_tok[0] + t] >> 16);
        }
        // residual terms of the block's key records, one record per
        // half-warp per step (a rolled loop: the transform is the bulk of
        // the code), its G dot products finished by a 16-lane reduction
        const int rlo = min(wpre[blk], nK), rhi = min(wpre[blk + 1], nK);
#pragma unroll 1
        for (int r0 = rlo; r0 < rhi; r0 += 2) {
          // a record past rhi repeats the last one (every lane takes part
          // in the shuffles); its terms are not stored
          const int r = min(r0 + half, rhi - 1);
          const int bo = rtok[r] & 31;
          const uint32_t b0 = codes[r * kCodeBytes + l16], b1 = codes[r * kCodeBytes + 16 + l16];
          const float2 p0 = lutc[(b0 & 15u) * 16], p1 = lutc[(b0 >> 4) * 16];
          const float2 p2 = lutc[(b1 & 15u) * 16], p3 = lutc[(b1 >> 4) * 16];
          float y[8] = {p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y};
          if (!a.naive) fwht128_half(y, lane);
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] *= sg[e];
          float d[GP];
          turn_dot<GP>(y, tbB[bo * 32], tbB[bo * 32 + 16], qa, d);
          transpose_reduce16<GP>(d, lane);
          if (r0 + half < rhi && (l16 % (16 / GP)) == 0)
            rres[r * GP + l16 / (16 / GP)] = d[0] * half_bits_to_f(sig0[sh_sig[0] + r]);
        }
      }
      __syncthreads();
    }
    // b. every token's logit for the G heads (anchor term + its record's
    //    residual term), kept in registers; the value side's slot and coefficient
    float lg[kKT][GP];
    float cmx[GP];
    int slv[kKT];
    float gmv[kKT];
    float gabs = 0.f;
#pragma unroll
    for (int g = 0; g < GP; ++g) cmx[g] = -INFINITY;
#pragma unroll
    for (int i = 0; i < kKT; ++i) {
      const int t = tid + i * kThreads;
      slv[i] = 0;
      gmv[i] = 0.f;
#pragma unroll
      for (int g = 0; g < GP; ++g) lg[i][g] = -INFINITY;
      if (t < ntok) {
        const uint32_t wv = tok0p[(ct + 4) + sh_tok[1] + t];
        slv[i] = min((int)(wv & 0xFFFFu), a.k - 1);
        gmv[i] = half_bits_to_f(wv >> 16);
        gabs = fmaxf(gabs, fabsf(gmv[i]));
        const uint32_t word = bm0[t >> 5];
        const uint32_t below = word & ((1u << (t & 31)) - 1u);
        const int rank = wpre[t >> 5] + __popc(below);
        const bool res = ((word >> (t & 31)) & 1u) && rank < nrec[0];
        float pv[GP];
        float gam = 1.f;
        if constexpr (ROPE) {
          load_slot<GP>(rlog + t * GP, pv);             // anchor terms, gamma~ included
        } else {
          const uint32_t wk = tok0p[sh_tok[0] + t];
          const int slot = min((int)(wk & 0xFFFFu), a.k - 1);
          gam = half_bits_to_f(wk >> 16);
          load_slot<GP>(P + slot * GP, pv);
        }
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float x = gam * pv[g];
          if (res) x += klg[rank * GP + g];
          lg[i][g] = x;
          cmx[g] = fmaxf(cmx[g], x);
        }
      }
    }
    // c. the running maximum and W's scale change only when a logit beats the
    //    maximum by the gap or a |gamma| reaches the scale's bound: one CTA
    //    vote, and the reductions only when it says so (rare after the first chunk)
    {
      bool up = gabs >= gbound;
#pragma unroll
      for (int g = 0; g < GP; ++g) up |= cmx[g] > mrun[g] + kRescaleGap;
      if (__syncthreads_or(up)) {
        float cm[GP], gmax, fsc[GP];
        block_max2(cmx, gabs, cm, gmax);
        update_max(cm, gmax, fsc);
      }
    }
    // d. probabilities, anchor weights (two native 32-bit integer atomics per
    //    head on the fixed point), value-record weights p sigma~
#pragma unroll
    for (int i = 0; i < kKT; ++i) {
      const int t = tid + i * kThreads;
      if (t < ntok) {
        const int slot = slv[i];
        const float gs = gmv[i] * wsc;
        const uint32_t word = bm0[ct / 32 + (t >> 5)];
        const int rank = wpre[ct / 32 + 1 + (t >> 5)] + __popc(word & ((1u << (t & 31)) - 1u));
        const bool res = ((word >> (t & 31)) & 1u) && rank < nrec[1];
        const float sg = res ? half_bits_to_f(sig0[(ct + 8) + sh_sig[1] + rank]) : 0.f;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float pr = exp2f(lg[i][g] - mrun[g]);
          lsum[g] += pr;
          const float x = pr * gs;                              // |x| < 2^kFixBits
          const float xh = floorf(x * (1.0f / kSplitScale));
          atomicAdd(&Whi[g * kp + slot], (int)xh);
          atomicAdd(&Wlo[g * kp + slot], __float2int_rn(fmaf(-xh, kSplitScale, x)));
          if (res) wz2[rank * GP + g] = make_float2(pr * sg, pr * sg);
        }
      }
    }
    // the value records up to the next multiple of 32 get zero weights, so
    // the value loop below runs whole steps (their codes are stale but in
    // the chunk's buffer)
    {
      const int nV = nrec[1], pad = (((nV + 31) & ~31) - nV) * GP;
      for (int i = tid; i < pad; i += kThreads) wz2[nV * GP + i] = make_float2(0.f, 0.f);
    }
    __syncthreads();
    folded_all = false;
    // every kFoldChunks chunks the parts go into the floats (the next chunk's
    // atomics come after its own barriers)
    if ((c + 1) % kFoldChunks == 0 && c + 1 < n_chunks) {
      float f1[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) f1[g] = 1.f;
      fold(f1);
      folded_all = true;
    }
    // e. value-residual sums
    {
      const int nV = nrec[1];
      const uint8_t* vcodes = codes + ct * kCodeBytes;
      // four records per step, their loads issued before any arithmetic; the
      // records run to a multiple of 32 (zero weights past nV)
      constexpr int kU = 4;
      const int nV32 = (nV + 31) & ~31;
      for (int r0 = warp; r0 < nV32; r0 += kU * kWarps) {
        uint32_t byte[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) byte[u] = vcodes[(r0 + u * kWarps) * kCodeBytes + lane];
        float2 l01[kU], l23[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          l01[u] = lutc[(byte[u] & 15u) * 16];
          l23[u] = lutc[(byte[u] >> 4) * 16];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          float2 ww[GP];
          load_pairs<GP>(wz2 + (r0 + u * kWarps) * GP, ww);
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            z01[g] = __ffma2_rn(l01[u], ww[g], z01[g]);
            z23[g] = __ffma2_rn(l23[u], ww[g], z23[g]);
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- 4. exact tail tokens (last slice): logits in rlog, then values
  float4 oacc[GP];                  // tail values, then anchor values, dims 4 lane ..
#pragma unroll
  for (int g = 0; g < GP; ++g) oacc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (has_tail) {
    float4 q4[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) q4[g] = *reinterpret_cast<const float4*>(qs + g * kD + 4 * lane);
    const T* Kt = reinterpret_cast<const T*>(a.Kt) + ((int64_t)b * a.H + h) * a.tail_cap * kD;
    const T* Vt = reinterpret_cast<const T*>(a.Vt) + ((int64_t)b * a.H + h) * a.tail_cap * kD;
    for (int t0 = 0; t0 < a.tail_len; t0 += ct) {
      const int n = min(ct, a.tail_len - t0);
      // logits: TB tokens per warp step, their rows loaded together and their
      // TB x GP dot products finished by one transposed reduction
      {
        constexpr int TB = GP >= 4 ? 32 / GP : 8;
        for (int base = warp * TB; base < n; base += kWarps * TB) {
          float x[TB][4];
#pragma unroll
          for (int i = 0; i < TB; ++i) {
            if (base + i < n) {
              load4(Kt + (int64_t)(t0 + base + i) * kD + 4 * lane, x[i]);
            } else {
              x[i][0] = x[i][1] = x[i][2] = x[i][3] = 0.f;
            }
          }
          if constexpr (ROPE) {
#pragma unroll
            for (int i = 0; i < TB; ++i) rotate4(a, (double)a.N + t0 + base + i, x[i], lane);
          }
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
#pragma unroll
          for (int i = 0; i < TB; ++i)
#pragma unroll
            for (int g = 0; g < GP; ++g)
              v[i * GP + g] = fmaf(q4[g].x, x[i][0], fmaf(q4[g].y, x[i][1], fmaf(q4[g].z, x[i][2], q4[g].w * x[i][3])));
          transpose_reduce32(v, lane);
          const int i = base + lane / GP;
          if (lane < TB * GP && i < n) rlog[i * GP + (lane % GP)] = v[0];
        }
      }
      __syncthreads();
      float cmx[GP], cm[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) cmx[g] = -INFINITY;
      for (int i = tid; i < n; i += kThreads)
#pragma unroll
        for (int g = 0; g < GP; ++g) cmx[g] = fmaxf(cmx[g], rlog[i * GP + g]);
      float fsc[GP];
      block_max(cmx, cm);
      update_max(cm, 0.f, fsc);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        oacc[g].x *= fsc[g]; oacc[g].y *= fsc[g]; oacc[g].z *= fsc[g]; oacc[g].w *= fsc[g];
      }
      // (heads unrolled: mrun stays in registers)
      for (int i = tid; i < n; i += kThreads)
#pragma unroll
        for (int g = 0; g < GP; ++g) rlog[i * GP + g] = exp2f(rlog[i * GP + g] - mrun[g]);
      __syncthreads();
      // probabilities were written by other threads: sum them per head here
      for (int i = tid; i < n; i += kThreads)
#pragma unroll
        for (int g = 0; g < GP; ++g) lsum[g] += rlog[i * GP + g];
      // values: four rows per warp step, loaded together
      for (int i0 = warp; i0 < n; i0 += 4 * kWarps) {
        float x[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * kWarps;
          if (i < n) {
            load4(Vt + (int64_t)(t0 + i) * kD + 4 * lane, x[u]);
          } else {
            x[u][0] = x[u][1] = x[u][2] = x[u][3] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * kWarps;
          if (i < n) {
#pragma unroll
            for (int g = 0; g < GP; ++g) {
              const float p = rlog[i * GP + g];
              oacc[g].x = fmaf(p, x[u][0], oacc[g].x); oacc[g].y = fmaf(p, x[u][1], oacc[g].y);
              oacc[g].z = fmaf(p, x[u][2], oacc[g].z); oacc[g].w = fmaf(p, x[u][3], oacc[g].w);
            }
          }
        }
      }
      __syncthreads();
    }
  }

  // ---- 5. partial output of this slice
  // sum of probabilities per head (per warp; summed where used); a slice
  // whose data never arrived poisons its heads' sums
  if (copy_failed) {
#pragma unroll
    for (int g = 0; g < GP; ++g) lsum[g] = __int_as_float(0x7fc00000);
  }
  {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float v = warp_sum(lsum[g]);
      if (lane == 0) red[kWarps * GP + warp * GP + g] = v;
    }
  }
  // the last parts into the float weights, then the value anchors weighted by W
  {
    float f1[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) f1[g] = 1.f;
    fold(f1);
  }
  __syncthreads();
  {
    const T* Va = reinterpret_cast<const T*>(comp + a.off_av) + (int64_t)h * a.k * kD;
    if constexpr (GP >= 2) {
      // heads in pairs: (o_2j, o_2j+1)[d] += (W_2j, W_2j+1) x[d], one f32x2 FMA
      float2 acc[GP / 2][4];
#pragma unroll
      for (int j = 0; j < GP / 2; ++j)
#pragma unroll
        for (int d = 0; d < 4; ++d) acc[j][d] = make_float2(0.f, 0.f);
#pragma unroll 8
      for (int slot = warp; slot < a.k; slot += kWarps) {
        float x[4];
        load4(Va + (int64_t)slot * kD + 4 * lane, x);
        float w[GP];
        load_slot<GP>(Wt + slot * GP, w);
#pragma unroll
        for (int j = 0; j < GP / 2; ++j) {
          const float2 w2 = make_float2(w[2 * j], w[2 * j + 1]);
#pragma unroll
          for (int d = 0; d < 4; ++d) acc[j][d] = __ffma2_rn(w2, make_float2(x[d], x[d]), acc[j][d]);
        }
      }
#pragma unroll
      for (int j = 0; j < GP / 2; ++j) {
        oacc[2 * j].x += acc[j][0].x; oacc[2 * j].y += acc[j][1].x;
        oacc[2 * j].z += acc[j][2].x; oacc[2 * j].w += acc[j][3].x;
        oacc[2 * j + 1].x += acc[j][0].y; oacc[2 * j + 1].y += acc[j][1].y;
        oacc[2 * j + 1].z += acc[j][2].y; oacc[2 * j + 1].w += acc[j][3].y;
      }
    } else {
#pragma unroll 16
      for (int slot = warp; slot < a.k; slot += kWarps) {
        float x[4];
        load4(Va + (int64_t)slot * kD + 4 * lane, x);
        const float w = Wt[slot];
        oacc[0].x = fmaf(w, x[0], oacc[0].x); oacc[0].y = fmaf(w, x[1], oacc[0].y);
        oacc[0].z = fmaf(w, x[2], oacc[0].z); oacc[0].w = fmaf(w, x[3], oacc[0].w);
      }
    }
  }
  // cross-warp sums of the anchor/tail values and of Z, through the stage buffers
  float* ored = reinterpret_cast<float*>(sm + F.P);              // [kWarps][GP][128]
  float* zred = ored + kWarps * GP * kD;                           // [kWarps][GP][128]
  __syncthreads();    // every chunk is consumed and no copy is in flight
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    *reinterpret_cast<float4*>(ored + (warp * GP + g) * kD + 4 * lane) = oacc[g];
    *reinterpret_cast<float4*>(zred + (warp * GP + g) * kD + 4 * lane) =
        make_float4(z01[g].x, z01[g].y, z23[g].x, z23[g].y);
  }
  __syncthreads();
  // Z turned back to the token domain: s . H(Z) / sqrt(D) (unrotated codec: Z)
  for (int g = warp; g < GP; g += kWarps) {
    float z[4] = {0.f, 0.f, 0.f, 0.f};
    for (int w = 0; w < kWarps; ++w) {
      const float4 t4 = *reinterpret_cast<const float4*>(zred + (w * GP + g) * kD + 4 * lane);
      z[0] += t4.x; z[1] += t4.y; z[2] += t4.z; z[3] += t4.w;
    }
    if (!a.naive) {
      fwht128(z);
      const float r = rsqrtf((float)kD);
#pragma unroll
      for (int i = 0; i < 4; ++i) z[i] *= sign_of(a, 4 * lane + i) * r;
    }
    // slot 0 of the warp sums takes the total (read only by this warp below)
    *reinterpret_cast<float4*>(zred + g * kD + 4 * lane) = make_float4(z[0], z[1], z[2], z[3]);
  }
  __syncthreads();
  // o[g][d] = sum over warps of the anchor/tail values + Z term, relative to mrun
  float* opart = qr;   // reuse: [GP][128]
  for (int i = tid; i < GP * kD; i += kThreads) {
    const int g = i / kD;
    float v = zred[i];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += ored[(w * GP + g) * kD + (i % kD)];
    opart[i] = v;
  }
  __syncthreads();
  const int Hq = a.H * G;
  float* out = a.out + ((int64_t)b * Hq + (int64_t)h * G) * kD;
  auto total_l = [&](int g) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += red[kWarps * GP + w * GP + g];
    return v;
  };
  if (a.S == 1) {
    for (int i = tid; i < G * kD; i += kThreads) out[i] = opart[i] / total_l(i / kD);
    return;
  }
  // several slices: publish this one, the last to finish merges
  constexpr int PW = part_words(GP), PO = part_out(GP);
  float* mine = a.part + ((int64_t)bh * a.S + s) * PW;
  for (int i = tid; i < GP * kD; i += kThreads) mine[PO + i] = opart[i];
#pragma unroll
  for (int g = 0; g < GP; ++g)
    if (tid == g) {
      mine[g] = mrun[g];
      mine[GP + g] = total_l(g);
    }
  __threadfence();
  __syncthreads();
  __shared__ int last;
  if (tid == 0) last = atomicAdd(&a.tickets[bh], 1) == a.S - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* all = a.part + (int64_t)bh * a.S * PW;
  // the slices' partials come into the (now idle) stage buffers by cp.async,
  // as many per round as fit: all of them at once for the usual slice counts
  uint8_t* mbuf = sm + F.stage;
  const int cap = max(1, 2 * F.stage_bytes / (PW * 4));
  auto issue = [&](int j0, int j1) {
    const uint8_t* src = reinterpret_cast<const uint8_t*>(all + (int64_t)j0 * PW);
    const int units = (j1 - j0) * PW / 4;
    for (int u = tid; u < units; u += kThreads) cp16(mbuf + 16 * u, src + 16 * u, 16);
    cp_commit();
  };
  issue(0, min(a.S, cap));
  // every slice's (max, sum) per head, then the weights 2^(m_s - M) / L (one
  // warp per head, lanes over slices)
  float* ms = rlog;                    // [S][GP] maxima, then weights (S <= kMaxSlices)
  float* ls = wz;                      // [S][GP] sums
  for (int i = tid; i < a.S * GP; i += kThreads) {
    const int j = i / GP, g = i % GP;
    ms[i] = __ldcg(all + (int64_t)j * PW + g);
    ls[i] = __ldcg(all + (int64_t)j * PW + GP + g);
  }
  __syncthreads();
  for (int g = warp; g < GP; g += kWarps) {
    float M = -INFINITY;
    for (int j = lane; j < a.S; j += 32) M = fmaxf(M, ms[j * GP + g]);
    M = warp_max(M);
    float lt = 0.f;
    for (int j = lane; j < a.S; j += 32) {
      const float f = exp2f(ms[j * GP + g] - M);
      ms[j * GP + g] = f;
      lt = fmaf(ls[j * GP + g], f, lt);
    }
    const float inv = 1.f / warp_sum(lt);
    for (int j = lane; j < a.S; j += 32) ms[j * GP + g] *= inv;
  }
  // thread t sums float4 column q = t mod NQ of the outputs over the slices
  // j = t / NQ (mod NG)
  constexpr int NQ = GP * kD / 4;
  constexpr int NG = NQ >= kThreads ? 1 : kThreads / NQ;
  constexpr int QPT = NQ > kThreads ? NQ / kThreads : 1;   // columns per thread
  float4 acc[QPT];
#pragma unroll
  for (int m = 0; m < QPT; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int grp = NQ >= kThreads ? 0 : tid / NQ;
  for (int j0 = 0; j0 < a.S; j0 += cap) {
    const int j1 = min(a.S, j0 + cap);
    cp_wait<0>();
    __syncthreads();
    for (int j = j0 + grp; j < j1; j += NG) {
      const float* pj = reinterpret_cast<const float*>(mbuf) + (j - j0) * PW + PO;
#pragma unroll
      for (int m = 0; m < QPT; ++m) {
        const int q = (NQ >= kThreads ? tid + m * kThreads : tid % NQ);
        const float w = ms[j * GP + (4 * q) / kD];
        const float4 v = reinterpret_cast<const float4*>(pj)[q];
        acc[m].x = fmaf(v.x, w, acc[m].x); acc[m].y = fmaf(v.y, w, acc[m].y);
        acc[m].z = fmaf(v.z, w, acc[m].z); acc[m].w = fmaf(v.w, w, acc[m].w);
      }
    }
    __syncthreads();
    if (j1 < a.S) issue(j1, min(a.S, j1 + cap));
  }
  // the groups' sums meet in the stage buffers
  float4* mred = reinterpret_cast<float4*>(mbuf);
#pragma unroll
  for (int m = 0; m < QPT; ++m) {
    const int q = (NQ >= kThreads ? tid + m * kThreads : tid % NQ);
    mred[grp * NQ + q] = acc[m];
  }
  __syncthreads();
  for (int q = tid; q < G * kD / 4; q += kThreads) {
    float4 o = mred[q];
#pragma unroll
    for (int r = 1; r < NG; ++r) {
      const float4 t = mred[r * NQ + q];
      o.x += t.x; o.y += t.y; o.z += t.z; o.w += t.w;
    }
    reinterpret_cast<float4*>(out)[q] = o;
  }
}

// ---------------------------------------------------------------- host side

// Resident CTAs per SM at `smem` bytes of dynamic shared memory (0: none).
// The kernel's dynamic shared-memory limit is raised once to the largest a
// CTA may use, so every later shape launches without touching it.
template <typename T, int GP, bool ROPE>
int max_ctas_per_sm(int smem) {
  static std::mutex mu;
  static int cache_smem[8] = {0}, cache_n[8] = {0}, n_cache = 0;
  static int dev_set = -1;
  std::lock_guard<std::mutex> lock(mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev != dev_set) {
    // the opt-in maximum per block, less the kernel's static shared memory
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, flash_decode_kernel<T, GP, ROPE>) != cudaSuccess)
      return 0;
    if (cudaFuncSetAttribute(flash_decode_kernel<T, GP, ROPE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes) != cudaSuccess)
      return 0;
    dev_set = dev;
    n_cache = 0;
  }
  for (int i = 0; i < n_cache; ++i)
    if (cache_smem[i] == smem) return cache_n[i];
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, flash_decode_kernel<T, GP, ROPE>, kThreads, smem) != cudaSuccess)
    n = 0;
  if (n_cache < 8) { cache_smem[n_cache] = smem; cache_n[n_cache] = n; ++n_cache; }
  return n;
}

}  // namespace

// Shape of the slice decode for `batch` sequences: tokens per chunk, slices
// per (sequence, head) and the workspace.  Returns false when no chunk size
// fits the shared memory (the split-token kernels take over).
bool flash_decode_plan(const Plan& pl, int batch, FlashShape* fs, bool allow_prepass, bool rope) {
  const int GP = gp_of(pl.G);
  const int kp = (pl.k + 3) & ~3;
  // CTAs resident per SM: two when the registers allow it (G <= 4) and the
  // shared memory of the largest chunk size that fits does; the slice plan
  // is sized for the whole head, which bounds every slice
  static const int kChunkSizes[4] = {512, 384, 256, 128};
  int per_sm = GP <= 4 ? 2 : 1;
  const char* env = getenv("ANCHORKV_DECODE_CTAS_PER_SM");
  if (env && env[0]) per_sm = std::max(1, std::min(per_sm, atoi(env)));
  fs->ct = 0;
  for (; per_sm >= 1 && !fs->ct; --per_sm)
    for (int ct : kChunkSizes) {
      const int need = fplan(GP, kp, ct, pl.n_tiles, rope).total;
      if (need <= kSmemBudget && (need + 1024) * per_sm <= 228 * 1024) { fs->ct = ct; break; }
    }
  if (!fs->ct) return false;
  ++per_sm;                      // the loop stepped past the count that fit
  const int units = std::max(1, batch * pl.H);
  const int target = 148 * per_sm;
  int S = std::max(1, std::min({pl.n_tiles, target / units, kMaxSlices}));
  int tps = (pl.n_tiles + S - 1) / S;
  S = (pl.n_tiles + tps - 1) / tps;
  fs->S = S;
  fs->tps = tps;
  fs->smem = fplan(GP, kp, fs->ct, tps, rope).total;
  // key-residual logits on the tensor cores ahead of the decode: worth it
  // when the launch is throughput-bound (two slices per head or fewer, i.e.
  // many sequences), not when a few heads are cut into many slices and
  // latency rules; ANCHORKV_DECODE_KLOGIT=0/1 forces it either way
  const char* kenv = getenv("ANCHORKV_DECODE_KLOGIT");
  fs->klogit = allow_prepass && !rope && klogit_tc_supported(pl) && pl.R > 0 &&
               (kenv && kenv[0] ? kenv[0] == '1' : S <= 2);
  int64_t off = 0;
  auto take = [&](int64_t bytes) { int64_t o = off; off += (bytes + 255) / 256 * 256; return o; };
  fs->o_tickets = S > 1 ? take(4 * (int64_t)units) : 0;
  fs->o_part = S > 1 ? take(4 * (int64_t)units * S * part_words(GP)) : 0;
  fs->o_rlog = fs->klogit ? take(klogit_ws_bytes(pl, batch)) : 0;
  fs->o_P = take(4 * (int64_t)units * ((pl.k + 3) & ~3) * GP);
  fs->ws_total = off;
  return true;
}

int launch_flash_decode(const Plan& pl, const FlashShape& fs, int batch, const char* comp, int64_t stride,
                        const void* q, const void* Kt, const void* Vt, int tail_len, int tail_cap, float* out,
                        char* ws, cudaStream_t s, double rope_base) {
  FArgs a;
  a.rope = rope_base > 0.0;
  for (int i = 0; i < kD / 2; ++i) a.inv_freq[i] = a.rope ? pow(rope_base, -2.0 * i / kD) : 0.0;
  a.comp = reinterpret_cast<const uint8_t*>(comp);
  a.stride = stride;
  a.total = pl.L.total_bytes;
  a.off_ak = pl.L.off_anchors_k; a.off_av = pl.L.off_anchors_v; a.off_tok = pl.L.off_tok;
  a.off_bm = pl.L.off_bitmap; a.off_pf = pl.L.off_tile_prefix; a.off_codes = pl.L.off_res_codes;
  a.off_sig = pl.L.off_res_sigma;
  a.N = pl.N; a.H = pl.H; a.G = pl.G; a.k = pl.k; a.kp = (pl.k + 3) & ~3; a.n_tiles = pl.n_tiles;
  a.R = pl.R;
  a.lev[0] = (float)-pl.l2; a.lev[1] = (float)-pl.l1; a.lev[2] = (float)pl.l1; a.lev[3] = (float)pl.l2;
  for (int i = 0; i < 4; ++i) a.sign_bits[i] = pl.sign_bits[i];
  a.naive = naive_codec(pl);
  a.q = q; a.Kt = Kt; a.Vt = Vt; a.tail_len = tail_len; a.tail_cap = tail_cap; a.out = out;
  a.S = fs.S; a.tps = fs.tps; a.ct = fs.ct;
  a.rlg = fs.klogit ? reinterpret_cast<const float*>(ws + fs.o_rlog) : nullptr;
  a.part = fs.S > 1 ? reinterpret_cast<float*>(ws + fs.o_part) : nullptr;
  a.tickets = fs.S > 1 ? reinterpret_cast<int*>(ws + fs.o_tickets) : nullptr;
  a.Pw = reinterpret_cast<float*>(ws + fs.o_P);
  stage_begin(kStDecodeCluster, s);
  if (fs.klogit) {
    const int st = launch_klogit_tc(pl, batch, comp, stride, q, reinterpret_cast<float*>(ws + fs.o_rlog), s);
    if (st) return st;
  }
  const dim3 grid(fs.S, batch * pl.H);
  const dim3 pgrid((pl.k + kPSlots - 1) / kPSlots, batch * pl.H);
  const int GP = gp_of(pl.G);
  cudaError_t e = cudaSuccess;
  // the anchor-logit pre-kernel (it also clears the merge tickets), then the
  // decode as its programmatic dependent: the decode's CTAs start once every
  // pre-kernel CTA is running and wait for its results where they need them
  auto go = [&](auto kernel, auto pkernel, int n_ok) {
    if (n_ok < 1) { e = cudaErrorNotSupported; return; }
    pkernel<<<pgrid, kThreads, 0, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = fs.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, a);
  };
  auto pick = [&](auto tag) {
    using T = decltype(tag);
    if (a.rope) {
      switch (GP) {
        case 1: go(flash_decode_kernel<T, 1, true>, anchor_logit_kernel<T, 1>, max_ctas_per_sm<T, 1, true>(fs.smem)); break;
        case 2: go(flash_decode_kernel<T, 2, true>, anchor_logit_kernel<T, 2>, max_ctas_per_sm<T, 2, true>(fs.smem)); break;
        case 4: go(flash_decode_kernel<T, 4, true>, anchor_logit_kernel<T, 4>, max_ctas_per_sm<T, 4, true>(fs.smem)); break;
        case 8: go(flash_decode_kernel<T, 8, true>, anchor_logit_kernel<T, 8>, max_ctas_per_sm<T, 8, true>(fs.smem)); break;
        default: e = cudaErrorNotSupported; break;
      }
      return;
    }
    switch (GP) {
      case 1: go(flash_decode_kernel<T, 1, false>, anchor_logit_kernel<T, 1>, max_ctas_per_sm<T, 1, false>(fs.smem)); break;
      case 2: go(flash_decode_kernel<T, 2, false>, anchor_logit_kernel<T, 2>, max_ctas_per_sm<T, 2, false>(fs.smem)); break;
      case 4: go(flash_decode_kernel<T, 4, false>, anchor_logit_kernel<T, 4>, max_ctas_per_sm<T, 4, false>(fs.smem)); break;
      case 8: go(flash_decode_kernel<T, 8, false>, anchor_logit_kernel<T, 8>, max_ctas_per_sm<T, 8, false>(fs.smem)); break;
      default: go(flash_decode_kernel<T, 16, false>, anchor_logit_kernel<T, 16>, max_ctas_per_sm<T, 16, false>(fs.smem)); break;
    }
  };
  if (pl.p.dtype == ANCHORKV_BF16) pick(__nv_bfloat16{});
  else pick(0.f);
  stage_end(kStDecodeCluster, s, fs.klogit ? 3 : 2);   // pre-pass, anchor logits, decode
  if (e == cudaErrorNotSupported) return ANCHORKV_EUNSUPPORTED;
  return e == cudaSuccess ? ANCHORKV_OK : ANCHORKV_ECUDA;
}

int flash_ctas_per_sm(const Plan& pl, const FlashShape& fs) {
  const int GP = gp_of(pl.G);
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    return GP == 1 ? max_ctas_per_sm<T, 1, false>(fs.smem) : GP == 2 ? max_ctas_per_sm<T, 2, false>(fs.smem)
         : GP == 4 ? max_ctas_per_sm<T, 4, false>(fs.smem) : GP == 8 ? max_ctas_per_sm<T, 8, false>(fs.smem)
         : max_ctas_per_sm<T, 16, false>(fs.smem);
  }
  using T = float;
  return GP == 1 ? max_ctas_per_sm<T, 1, false>(fs.smem) : GP == 2 ? max_ctas_per_sm<T, 2, false>(fs.smem)
       : GP == 4 ? max_ctas_per_sm<T, 4, false>(fs.smem) : GP == 8 ? max_ctas_per_sm<T, 8, false>(fs.smem)
       : max_ctas_per_sm<T, 16, false>(fs.smem);
}

}  // namespace akv
