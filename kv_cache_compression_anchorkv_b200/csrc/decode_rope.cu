// Decode attention with rotary positions: keys are stored before the rotary
// map and rotated at decode time.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// "Assumptions & free parameters" (standard math, Section 3.2): RoPE is a
// per-position orthogonal linear map R_t, so R_t K_t = R_t K~_t + R_t r_t and
// ||R_t r_t|| = ||r_t||, which justifies pre-RoPE storage and rotation at
// decode time.  Reading: the rotate-half pairing (coordinate i with i + D/2,
// angle p * base^(-2i/D)); cached token t at position t, tail token i at
// N + i, the decode query at N + T.
//
// The per-slot factorisation q.K_a of the plain decode does not survive the
// rotation (every token turns its anchor by a different angle, and the
// rotation does not commute with the residual codec's Hadamard transform), so
// each warp rebuilds K^_t = gamma~ K_a + r~_t for one token at a time in
// registers (lane l holds coordinates 4l .. 4l + 3; the residual through a
// warp FWHT), rotates it by its position (the partner coordinate is in lane
// l ^ 16), scores it against the G rotated queries of the KV head and
// updates an online softmax over V^_t.  Angles are reduced modulo 2 pi in
// fp64 before the fast sine/cosine.
//
// A warp walks 32-token chunks (one bitmap word each): its lanes decode the
// chunk's record words, one token per lane (slot, gamma~, residual record
// index), and the per-token loop then takes them by shuffle, with the next
// token's anchor rows and residual codes already in flight; the next chunk's
// words are loaded a chunk ahead.  Tail tokens take the same path, their raw
// row standing in for the anchor row with gamma~ = 1 and no residual.
// Splits of the tokens (multiples of 32) over CTAs fill the SMs; a second
// kernel merges the splits in order.
//
// These kernels serve 16 query heads per KV head.  Up to 8, the rotary decode
// runs on the slice decode (decode_flash.cu) with its rotary key phase, which
// the plan below picks first.
#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kRopeWarps = 8;
constexpr float kLog2eR = 1.4426950408889634f;

struct RopeArgs {
  const uint8_t* comp;
  int64_t stride;
  anchorkv_layout L;
  int N, H, G, k, n_tiles, n_split, split_tokens, tail_len, tail_cap, naive;
  int64_t R;
  float lev[4];
  uint32_t sign_bits[4];
  double inv_freq[kD / 2];      // base^(-2i/D)
  float* part;                  // [b][h][split][G][D + 2]: m, l, acc
};

__device__ __forceinline__ float sgn_of(const RopeArgs& a, int d) {
  return ((a.sign_bits[d >> 5] >> (d & 31)) & 1u) ? -1.f : 1.f;
}

template <typename T> __device__ __forceinline__ void load4r(const T* p, float (&o)[4]);
template <> __device__ __forceinline__ void load4r<float>(const float* p, float (&o)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <> __device__ __forceinline__ void load4r<__nv_bfloat16>(const __nv_bfloat16* p, float (&o)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xFFFF0000u);
  o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xFFFF0000u);
}

// R_p x for this lane's four coordinates (lane l: 4l .. 4l + 3; the pair of
// coordinate d < D/2 is d + D/2, held by lane l ^ 16).  f: this lane's four
// frequencies base^(-2i/D), i = 4 (l mod 16) + e.
__device__ __forceinline__ void rope4(const double* f, int64_t pos, float (&x)[4], int lane) {
  const bool upper = lane >= 16;
  const double two_pi = 6.283185307179586476925286766559, inv_two_pi = 0.15915494309189533576888376337251;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const double ang = (double)pos * f[e];
    const float r = (float)(ang - two_pi * rint(ang * inv_two_pi));
    float s, c;
    __sincosf(r, &s, &c);
    const float other = __shfl_xor_sync(0xffffffffu, x[e], 16);
    x[e] = upper ? fmaf(other, s, x[e] * c) : fmaf(-other, s, x[e] * c);
  }
}

// Four coordinates of a row as loaded (bf16: 8 bytes, fp32: 16 bytes).
template <typename T> struct Raw4 { using type = uint4; };
template <> struct Raw4<__nv_bfloat16> { using type = uint2; };

template <typename T>
__device__ __forceinline__ typename Raw4<T>::type load_raw4(const T* p) {
  return *reinterpret_cast<const typename Raw4<T>::type*>(p);
}
__device__ __forceinline__ void unpack4(const uint2& v, float (&o)[4]) {
  o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xFFFF0000u);
  o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xFFFF0000u);
}
__device__ __forceinline__ void unpack4(const uint4& v, float (&o)[4]) {
  o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
  o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
}

// The raw words of a 32-token chunk (tc a multiple of 32): lane l's token
// record words (both sides), and one word of the chunk's tile spread over
// lanes 0 .. 9 (lane 4s + w: bitmap word w of side s; lane 8 + s: the tile's
// first record index of side s).
struct ChunkRaw {
  uint32_t rt[2];
  uint32_t wv;
};

__device__ __forceinline__ void chunk_load(const RopeArgs& a, const uint8_t* comp, int h, int tc, int lane,
                                           ChunkRaw& cr) {
  cr.rt[0] = cr.rt[1] = 0u;
  cr.wv = 0u;
  if (tc >= a.N) return;                            // tail tokens only
  const int t = tc + lane, tile = tc / kTile;
  const uint32_t* tok = reinterpret_cast<const uint32_t*>(comp + a.L.off_tok);
#pragma unroll
  for (int side = 0; side < 2; ++side)
    if (t < a.N) cr.rt[side] = tok[(int64_t)(side * a.H + h) * a.N + t];
  if (lane < 8) {
    const int sh = (lane >> 2) * a.H + h;
    cr.wv = reinterpret_cast<const uint32_t*>(comp + a.L.off_bitmap)[((int64_t)sh * a.n_tiles + tile) * 4 + (lane & 3)];
  } else if (lane < 10) {
    const int sh = (lane - 8) * a.H + h;
    cr.wv = (uint32_t)reinterpret_cast<const int*>(comp + a.L.off_tile_prefix)[(int64_t)sh * (a.n_tiles + 1) + tile];
  }
}

// Lane l's token of the chunk: its record words and its residual record index
// per side (-1: no residual).
struct Chunk {
  uint32_t rt[2];
  int rec[2];
};

__device__ __forceinline__ void chunk_decode(const RopeArgs& a, int tc, int lane, const ChunkRaw& cr, Chunk& ck) {
  const int w = (tc % kTile) / 32;
  const bool cached = tc + lane < a.N;
#pragma unroll
  for (int side = 0; side < 2; ++side) {
    int rec = (int)__shfl_sync(0xffffffffu, cr.wv, 8 + side);
    uint32_t word = 0u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t wq = __shfl_sync(0xffffffffu, cr.wv, 4 * side + q);
      if (q < w) rec += __popc(wq);
      if (q == w) word = wq;
    }
    rec += __popc(word & ((1u << lane) - 1u));
    const bool has = cached && ((word >> lane) & 1u) && (int64_t)rec < a.R;
    ck.rec[side] = has ? rec : -1;
    ck.rt[side] = cr.rt[side];
  }
}

// One token's loads (both sides): the anchor row (a tail token: its raw row),
// the gamma~ bits, and the residual code byte and sigma when it has a record.
template <typename T>
struct TokRaw {
  typename Raw4<T>::type row[2];
  uint32_t gb[2];
  uint32_t code[2];
  uint32_t sig[2];
  bool has[2];
};

template <typename T>
__device__ __forceinline__ void tok_issue(const RopeArgs& a, const uint8_t* comp, const T* AK, const T* AV,
                                          const T* Kt, const T* Vt, int bb, int h, int t, int b, const Chunk& ck,
                                          int lane, TokRaw<T>& r) {
#pragma unroll
  for (int side = 0; side < 2; ++side) {
    const uint32_t rt = __shfl_sync(0xffffffffu, ck.rt[side], b);
    const int rec = __shfl_sync(0xffffffffu, ck.rec[side], b);
    r.has[side] = rec >= 0;                           // (uniform over the warp)
    r.code[side] = 0u;
    r.sig[side] = 0u;
    if (t < a.N) {
      const int slot = min((int)(rt & 0xFFFFu), a.k - 1);
      r.row[side] = load_raw4<T>((side ? AV : AK) + ((int64_t)h * a.k + slot) * kD + lane * 4);
      r.gb[side] = rt >> 16;
      if (rec >= 0) {
        r.code[side] = (comp + a.L.off_res_codes)[(int64_t)rec * kCodeBytes + lane];
        r.sig[side] = reinterpret_cast<const uint16_t*>(comp + a.L.off_res_sigma)[rec];
      }
    } else {
      const int64_t row = (((int64_t)bb * a.H + h) * a.tail_cap + (t - a.N)) * kD + lane * 4;
      r.row[side] = load_raw4<T>((side ? Vt : Kt) + row);
      r.gb[side] = 0x3C00u;                           // gamma~ = 1
    }
  }
}

// Both sides' reconstructed rows x^_t (this lane's four coordinates): gamma~
// times the anchor row plus the decoded residual when the bitmap has it.
template <typename T>
__device__ __forceinline__ void tok_rebuild(const RopeArgs& a, const TokRaw<T>& r, float (&kx)[4], float (&vx)[4],
                                            int lane) {
  const float isd = rsqrtf((float)kD);
#pragma unroll
  for (int side = 0; side < 2; ++side) {
    float* x = side ? vx : kx;
    float av[4];
    unpack4(r.row[side], av);
    const float g = half_bits_to_f((uint16_t)r.gb[side]);
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = g * av[e];
    if (!r.has[side]) continue;
    const float sg = half_bits_to_f((uint16_t)r.sig[side]);
    float z[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) z[e] = a.lev[(r.code[side] >> (2 * e)) & 3u] * sg;
    if (a.naive) {
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] += z[e];
    } else {
      fwht128<float>(z);
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = fmaf(z[e] * isd, sgn_of(a, lane * 4 + e), x[e]);
    }
  }
}

// Sums over the warp of GM values at once (GM a power of two <= 32): a
// transposed butterfly leaves value j's sum in lanes whose top log2(GM) bits
// are j, and one shuffle per value hands every lane all of them.
template <int GM>
__device__ __forceinline__ void warp_sums(float (&d)[GM], int lane) {
  constexpr int kBits = GM == 1 ? 0 : GM == 2 ? 1 : GM == 4 ? 2 : GM == 8 ? 3 : 4;
  float v[GM];
#pragma unroll
  for (int i = 0; i < GM; ++i) v[i] = d[i];
#pragma unroll
  for (int st = 0; st < kBits; ++st) {
    const int off = 16 >> st, half = GM >> (st + 1);
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = up ? v[i + half] : v[i];
      const float send = up ? v[i] : v[i + half];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = 16 >> kBits; off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
#pragma unroll
  for (int j = 0; j < GM; ++j) d[j] = __shfl_sync(0xffffffffu, v[0], j << (5 - kBits));
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// grid (n_split, batch * H), kRopeWarps warps; each warp takes the 32-token
// chunks t0 + 32 warp, t0 + 32 (warp + 8), ... of its split (the tail after
// the N cached ones).  GM: a power of two >= G (register arrays per query
// head).
template <typename T, int GM>
__global__ void __launch_bounds__(kRopeWarps * 32, GM <= 4 ? 2 : 1) rope_split_kernel(RopeArgs a, const T* __restrict__ q,
                                                                     const T* __restrict__ Kt,
                                                                     const T* __restrict__ Vt) {
  extern __shared__ __align__(16) float smr[];       // [8][G][D + 2]
  __shared__ double s_freq[kD / 2];
  const int split = blockIdx.x, bh = blockIdx.y, bb = bh / a.H, h = bh % a.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, G = a.G;
  const uint8_t* comp = a.comp + (int64_t)bb * a.stride;
  const T* AK = reinterpret_cast<const T*>(comp + a.L.off_anchors_k);
  const T* AV = reinterpret_cast<const T*>(comp + a.L.off_anchors_v);
  const int total = a.N + a.tail_len;
  for (int i = threadIdx.x; i < kD / 2; i += blockDim.x) s_freq[i] = a.inv_freq[i];
  __syncthreads();
  const double* fr = s_freq + (lane & 15) * 4;
  // this KV head's queries, rotated to the decode position, scaled for exp2
  const float qs = kLog2eR * rsqrtf((float)kD);
  float qr[GM][4], m[GM], l[GM], acc[GM][4];
#pragma unroll
  for (int j = 0; j < GM; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) { acc[j][e] = 0.f; qr[j][e] = 0.f; }
    if (j < G) {
      float v[4];
      load4r<T>(q + ((int64_t)bb * a.H * G + h * G + j) * kD + lane * 4, v);
      rope4(fr, (int64_t)total, v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) qr[j][e] = v[e] * qs;
    }
  }
  const int t0 = split * a.split_tokens, t1 = min(total, t0 + a.split_tokens);
  ChunkRaw cr;
  int tc = t0 + 32 * warp;
  if (tc < t1) chunk_load(a, comp, h, tc, lane, cr);
  for (; tc < t1; tc += 32 * kRopeWarps) {
    Chunk ck;
    chunk_decode(a, tc, lane, cr, ck);
    if (tc + 32 * kRopeWarps < t1) chunk_load(a, comp, h, tc + 32 * kRopeWarps, lane, cr);
    const int nb = min(32, t1 - tc);
    TokRaw<T> cur, nxt;
    tok_issue<T>(a, comp, AK, AV, Kt, Vt, bb, h, tc, 0, ck, lane, cur);
    for (int b = 0; b < nb; ++b) {
      const int t = tc + b;
      if (b + 1 < nb) tok_issue<T>(a, comp, AK, AV, Kt, Vt, bb, h, t + 1, b + 1, ck, lane, nxt);
      float kx[4], vx[4];
      tok_rebuild<T>(a, cur, kx, vx, lane);
      rope4(fr, (int64_t)t, kx, lane);
      float dl[GM];
#pragma unroll
      for (int j = 0; j < GM; ++j) {
        dl[j] = qr[j][0] * kx[0];
#pragma unroll
        for (int e = 1; e < 4; ++e) dl[j] = fmaf(qr[j][e], kx[e], dl[j]);
      }
      warp_sums<GM>(dl, lane);                       // log2-domain logits, on every lane
#pragma unroll
      for (int j = 0; j < GM; ++j) {
        if (j < G) {
          const float d = dl[j];
          const float mn = fmaxf(m[j], d);
          const float sc = ex2f(m[j] - mn), p = ex2f(d - mn);
          l[j] = fmaf(l[j], sc, p);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[j][e] = fmaf(acc[j][e], sc, p * vx[e]);
          m[j] = mn;
        }
      }
      cur = nxt;
    }
  }
  // merge the warps of the CTA (fixed order) and write this split's partial
  const int stride = kD + 2;
#pragma unroll
  for (int j = 0; j < GM; ++j) {
    if (j < G) {
      float* dst = smr + ((size_t)warp * G + j) * stride;
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[lane * 4 + e] = acc[j][e];
      if (lane == 0) { dst[kD] = m[j]; dst[kD + 1] = l[j]; }
    }
  }
  __syncthreads();
  float* out = a.part + (((int64_t)bh * a.n_split + split) * G) * stride;
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
    const int j = i / kD, d = i % kD;
    float M = -INFINITY;
    for (int w = 0; w < kRopeWarps; ++w) M = fmaxf(M, smr[((size_t)w * G + j) * stride + kD]);
    float L = 0.f, O = 0.f;
    for (int w = 0; w < kRopeWarps; ++w) {
      const float* src = smr + ((size_t)w * G + j) * stride;
      const float f = src[kD] > -INFINITY ? exp2f(src[kD] - M) : 0.f;
      L = fmaf(src[kD + 1], f, L);
      O = fmaf(src[d], f, O);
    }
    out[j * stride + d] = O;
    if (d == 0) { out[j * stride + kD] = M; out[j * stride + kD + 1] = L; }
  }
}

// grid (batch * H), 128 threads: merge the splits in order.
__global__ void __launch_bounds__(128) rope_combine_kernel(RopeArgs a, float* __restrict__ o) {
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H, d = threadIdx.x, G = a.G;
  const int stride = kD + 2;
  const float* base = a.part + (int64_t)bh * a.n_split * G * stride;
  for (int j = 0; j < G; ++j) {
    float M = -INFINITY;
    for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, base[((int64_t)s * G + j) * stride + kD]);
    float L = 0.f, O = 0.f;
    for (int s = 0; s < a.n_split; ++s) {
      const float* src = base + ((int64_t)s * G + j) * stride;
      const float f = src[kD] > -INFINITY ? exp2f(src[kD] - M) : 0.f;
      L = fmaf(src[kD + 1], f, L);
      O = fmaf(src[d], f, O);
    }
    o[((int64_t)b * a.H * G + h * G + j) * kD + d] = O / L;
  }
}

}  // namespace

// Token splits of the rotary decode: about two CTAs per SM over batch * H
// (sequence, head) pairs, at least 256 cached tokens per split.
RopePlan make_rope_plan(const Plan& pl, int batch) {
  RopePlan rp;
  rp.flash = pl.G <= 8 && flash_decode_plan(pl, batch, &rp.fs, false, true);
  if (rp.flash) {
    rp.n_split = 0;
    rp.ws_total = rp.fs.ws_total;
    return rp;
  }
  const int bh = std::max(1, batch * pl.H);
  const int want = std::max(1, (2 * 148 + bh - 1) / bh);
  rp.n_split = std::max(1, std::min(want, (pl.N + 255) / 256));
  rp.ws_total = (int64_t)batch * pl.H * rp.n_split * pl.G * (kD + 2) * 4;
  return rp;
}

cudaError_t launch_decode_rope(const Plan& pl, const RopePlan& rp, const char* comp, int64_t stride, int batch,
                               const void* q, const void* Kt, const void* Vt, int tail_len, int tail_cap,
                               double rope_base, float* out, char* ws, cudaStream_t s) {
  if (rp.flash) {
    const int st = launch_flash_decode(pl, rp.fs, batch, comp, stride, q, Kt, Vt, tail_len, tail_cap, out, ws, s,
                                       rope_base);
    return st == ANCHORKV_OK ? cudaSuccess : st == ANCHORKV_EUNSUPPORTED ? cudaErrorNotSupported : cudaErrorUnknown;
  }
  RopeArgs a;
  a.comp = reinterpret_cast<const uint8_t*>(comp);
  a.stride = stride;
  a.L = pl.L;
  a.N = pl.N; a.H = pl.H; a.G = pl.G; a.k = pl.k; a.n_tiles = pl.n_tiles;
  a.n_split = rp.n_split;
  a.split_tokens = ((pl.N + tail_len + rp.n_split - 1) / rp.n_split + 31) / 32 * 32;   // whole chunks
  a.tail_len = tail_len; a.tail_cap = tail_cap;
  a.naive = naive_codec(pl);
  a.R = pl.R;
  a.lev[0] = (float)-pl.l2; a.lev[1] = (float)-pl.l1; a.lev[2] = (float)pl.l1; a.lev[3] = (float)pl.l2;
  for (int i = 0; i < 4; ++i) a.sign_bits[i] = pl.sign_bits[i];
  for (int i = 0; i < kD / 2; ++i) a.inv_freq[i] = pow(rope_base, -2.0 * i / kD);
  a.part = reinterpret_cast<float*>(ws);
  const dim3 grid(rp.n_split, batch * pl.H);
  const size_t smem = sizeof(float) * (size_t)kRopeWarps * pl.G * (kD + 2);
  auto go = [&](auto kern, auto tag) {
    using T = decltype(tag);
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kRopeWarps * 32, smem, s>>>(a, static_cast<const T*>(q), static_cast<const T*>(Kt),
                                             static_cast<const T*>(Vt));
  };
  stage_begin(kStDecodeRope, s);
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    if (pl.G <= 4) go(rope_split_kernel<T, 4>, T{});
    else if (pl.G <= 8) go(rope_split_kernel<T, 8>, T{});
    else go(rope_split_kernel<T, 16>, T{});
  } else {
    using T = float;
    if (pl.G <= 4) go(rope_split_kernel<T, 4>, T{});
    else if (pl.G <= 8) go(rope_split_kernel<T, 8>, T{});
    else go(rope_split_kernel<T, 16>, T{});
  }
  rope_combine_kernel<<<batch * pl.H, 128, 0, s>>>(a, out);
  stage_end(kStDecodeRope, s, 2);
  return cudaGetLastError();
}

}  // namespace akv
