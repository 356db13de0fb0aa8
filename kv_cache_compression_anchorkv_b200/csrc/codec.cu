// Coefficient/residual/utility, per-layer top-R residual selection, the
// residual codec and the dense reconstruction hook.
//
// Sources ("AnchorKV: Anchor-Residual KV Cache Compression", pith.science
// review; "AnchorKV-adapted", VeloxQuant-MLX docs):
//  * gamma_i = <x_i, x_a>/||x_a||^2, x^_i = gamma_i x_a + r~_i
//    (review, "What carries the argument"); gamma is stored in 2 bytes
//    (review, "Assumptions & free parameters", codec parameters).
//  * utilities: first-order softmax expansion under the incoherence model
//    (review, "Circularity Check"; "Assumptions": Eq. 5, Eq. 6, Eq. 16).
//    Reading: u^V_t = ||r^V_t||^2 sum_r alpha_rt^2,
//             u^K_t = ||r^K_t||^2 / D^2 sum_r alpha_rt^2 ||q_r||^2 ||V_t - ybar_r||^2.
//  * the byte budget buys the R best token-sides of the layer, pooled over
//    heads and sides (VeloxQuant "Evidence": the budget pools across heads;
//    review: 17.3% of token-sides get residuals).  Ties -> lower flat index
//    (side, head, position).
//  * residuals: randomized Hadamard rotation, one fp16 scale ||r||/sqrt(D),
//    2-bit Lloyd-Max codes for a unit Gaussian (review, Referee "Summary";
//    "Assumptions": rotated coordinates ~ N(0, ||r||^2/D)).
// gamma~, ||r||^2, the scale and the code decisions are taken in fp64 from
// exact inputs (a bf16/fp32 product is exact in fp64), so each integer the
// codec stores is decided in the precision of a float64 restatement.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

// ---------------------------------------------------------------- project

// grid (ceil(N / 64), H, 2), 256 threads: 4 lanes per token (a warp takes 8
// consecutive tokens of one (side, head)).  Lane q of a token reads the
// 16-byte pieces q, q + 4, ... of the token's row and of its anchor's row,
// so every load instruction reads 64 contiguous bytes of 8 rows, and one
// pass accumulates d = <x, x_a> and n = ||x||^2 in fp64.  The 4 partial sums
// are combined by two shuffles.  With the stored g = fp16(d / a2),
// a2 = ||x_a||^2, the residual energy is r2 = n - 2 g d + g^2 a2: the sums of
// exact bf16/fp32 products are exact or within fp64 rounding, so the
// cancellation leaves an error near 1e-12 ||x||^2.
constexpr int kProjTokens = 64;
constexpr int kProjTPQ = 2;      // tokens per quad of lanes (kProjTPQ x kProjTokens per block)

template <typename T>
__device__ __forceinline__ void load16(const T* p, float (&o)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void load16<float>(const float* p, float (&o)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* p, float (&o)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// kUtility: the method's ranking (the other criteria, an ablation, share the
// second instantiation and switch on `rank`).
template <typename T, bool kUtility>
__global__ void __launch_bounds__(256)
project_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ anc_k,
               const T* __restrict__ anc_v, const double* __restrict__ anc_n2, const int* __restrict__ slot_of,
               const float* __restrict__ a2s, const float* __restrict__ kus, const float* __restrict__ score,
               uint32_t* __restrict__ tok, float* __restrict__ util, int N, int H, int k, int obs_rb, int rank,
               uint64_t seed, int layer) {
  constexpr int EPV = 16 / (int)sizeof(T);        // elements per 16-byte load
  constexpr int STEPS = kD / (4 * EPV);           // loads per lane and row
  const int q = threadIdx.x & 3;
  const int h = blockIdx.y, side = blockIdx.z;
  // each quad takes kProjTPQ tokens kProjTokens apart, all their loads in
  // flight together (record words, then rows and token-only values)
  int tq[kProjTPQ], ttq[kProjTPQ];
  int64_t fq[kProjTPQ];
  uint32_t tw[kProjTPQ];
#pragma unroll
  for (int u = 0; u < kProjTPQ; ++u) {
    tq[u] = (blockIdx.x * kProjTPQ + u) * kProjTokens + (threadIdx.x >> 2);
    ttq[u] = tq[u] < N ? tq[u] : N - 1;           // every lane takes part in the shuffles
    fq[u] = ((int64_t)side * H + h) * N + ttq[u];
    tw[u] = tok[fq[u]];
  }
  // Loads that depend only on the token go out with the row loads: the
  // anchor flag, the anchor's squared norm, and (utility ranking) lane q's observation-row-block
  // partial q, for the first npre of the obs_rb partials.
  static_assert(kObsGroups <= 4, "one partial per lane of the quad");
  const int npre = min(obs_rb, kObsGroups);
  const float* src = side ? a2s : kus;
  uint32_t slotq[kProjTPQ];
  bool anc[kProjTPQ];
  double n2q[kProjTPQ], dotq[kProjTPQ], nxq[kProjTPQ];
  float partq[kProjTPQ];
#pragma unroll
  for (int u = 0; u < kProjTPQ; ++u) {
    slotq[u] = min(tw[u] & 0xFFFFu, (uint32_t)(k - 1));
    anc[u] = slot_of[(int64_t)h * N + ttq[u]] >= 0;
    n2q[u] = anc_n2[((int64_t)side * H + h) * k + slotq[u]];
    partq[u] = (kUtility && q < npre) ? src[((int64_t)q * H + h) * N + ttq[u]] : 0.0f;
    dotq[u] = 0.0;
    nxq[u] = 0.0;
  }
#pragma unroll
  for (int u = 0; u < kProjTPQ; ++u) {
    const T* x = (side ? V : K) + ((int64_t)h * N + ttq[u]) * kD;
    const T* a = (side ? anc_v : anc_k) + ((int64_t)h * k + slotq[u]) * kD;
#pragma unroll
    for (int i = 0; i < STEPS; ++i) {
      const int d = (4 * i + q) * EPV;
      float xf[EPV], af[EPV];
      load16<T>(x + d, xf);
      load16<T>(a + d, af);
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        dotq[u] = fma((double)xf[e], (double)af[e], dotq[u]);
        nxq[u] = fma((double)xf[e], (double)xf[e], nxq[u]);
      }
    }
  }
  const int l0 = threadIdx.x & 31 & ~3;
#pragma unroll
  for (int u = 0; u < kProjTPQ; ++u) {
    double dot = dotq[u], nx = nxq[u];
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    nx += __shfl_xor_sync(0xffffffffu, nx, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    nx += __shfl_xor_sync(0xffffffffu, nx, 2);
    // partials 0 .. npre-1 to the quad's lane 0, summed in row-block order
    float m = __shfl_sync(0xffffffffu, partq[u], l0);
    for (int rb = 1; rb < npre; ++rb) m += __shfl_sync(0xffffffffu, partq[u], l0 + rb);
    const int t = tq[u];
    if (t >= N || q != 0) continue;
    const int64_t f = fq[u];
    const uint32_t slot = slotq[u];
    const double n2 = n2q[u];
    const bool is_anchor = anc[u];
    double gamma = (n2 > 0.0) ? dot / n2 : 0.0;
    if (is_anchor) gamma = 1.0;
    const uint16_t gb = half_bits_rn(gamma);
    const double g = (double)half_bits_to_f(gb);
    const double r2 = fmax(0.0, nx - 2.0 * g * dot + g * g * n2);
    tok[f] = slot | ((uint32_t)gb << 16);
    float uval;
    if (is_anchor) {
      uval = -1.0f;
    } else if (kUtility) {
      // sum of the observation-row-block partials, in order
      for (int rb = npre; rb < obs_rb; ++rb) m += src[((int64_t)rb * H + h) * N + t];
      uval = side ? (float)(r2 * (double)m) : (float)(r2 / (double)(kD * kD) * (double)m);
    } else if (rank == ANCHORKV_RANK_RESIDUAL_NORM) {
      uval = (float)r2;
    } else if (rank == ANCHORKV_RANK_ATTENTION) {
      // sum over the observation rows of alpha (row-block partials, in order)
      float sa = score[(int64_t)h * N + t];
      for (int rb = 1; rb < obs_rb; ++rb) sa += score[((int64_t)rb * H + h) * N + t];
      uval = sa;
    } else if (rank == ANCHORKV_RANK_COSINE) {
      const double den = sqrt(nx * n2);
      uval = (float)(1.0 - (den > 0.0 ? dot / den : 0.0));
    } else {
      // a seeded uniform value of the flat index: the top 24 bits of SplitMix64
      const uint64_t z = splitmix64(seed ^ kRankSalt ^ ((uint64_t)(layer & 0x7FFF) << 48) ^ (uint64_t)f);
      uval = (float)(z >> 40) * (1.0f / 16777216.0f);
    }
    util[f] = uval;
  }
}

// ---------------------------------------------------------------- key-as-query proxies

// Q[j][w] = K[j / G][N - W + w]: the trailing window keys of each KV head as
// the observation queries of its query heads (VeloxQuant "Adaptation notes",
// key-as-query proxy).  One thread per 16 bytes.
__global__ void key_query_kernel(const uint4* __restrict__ K, uint4* __restrict__ Q, int N, int W, int G,
                                 int chunks_per_row, int64_t total) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int64_t row = i / chunks_per_row;
  const int c = (int)(i % chunks_per_row);
  const int j = (int)(row / W), w = (int)(row % W);
  Q[i] = K[((int64_t)(j / G) * N + (N - W + w)) * chunks_per_row + c];
}

// ---------------------------------------------------------------- quantize

struct CodecConst {
  double tau, l1, l2;
  uint32_t sign_bits[4];
};

// 16 consecutive elements of a row (32-byte aligned for bf16, 64 for fp32).
template <typename T> __device__ __forceinline__ void load16(const T* p, float (&o)[16]);
template <> __device__ __forceinline__ void load16<float>(const float* p, float (&o)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = reinterpret_cast<const float4*>(p)[i];
    o[4 * i] = v.x; o[4 * i + 1] = v.y; o[4 * i + 2] = v.z; o[4 * i + 3] = v.w;
  }
}
template <> __device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* p, float (&o)[16]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 v = reinterpret_cast<const uint4*>(p)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
      o[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
}

// One warp per (tile, 32-token word); its residual records (flat order) go
// four at a time, eight lanes per record, lane l8 holding elements
// 16 l8 .. 16 l8 + 15.  The word's token records are gathered once (lane b
// holds token b's), so each record costs one round of independent row loads.
// The Hadamard transform runs its four low stages in registers and its three
// high stages across the record's eight lanes, all in fp64.
template <typename T>
__global__ void __launch_bounds__(256, 3) quantize_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                const T* __restrict__ anc_k, const T* __restrict__ anc_v,
                                const uint32_t* __restrict__ tok, const uint32_t* __restrict__ bitmap,
                                const int* __restrict__ tile_prefix, uint8_t* __restrict__ codes,
                                uint16_t* __restrict__ sigma, int N, int H, int k, int n_tiles, int64_t R,
                                int* __restrict__ counters, CodecConst cc, int naive) {
  const int lane = threadIdx.x & 31, grp = lane >> 3, l8 = lane & 7;
  const int n_words = 2 * H * n_tiles * 4;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= n_words) return;
  const int tile = wid >> 2, w = wid & 3;
  const int sh = tile / n_tiles, j = tile % n_tiles;
  const int side = sh / H, h = sh % H;
  const uint32_t* bw = bitmap + (int64_t)tile * 4;
  int rec0 = tile_prefix[sh * (n_tiles + 1) + j];
  for (int q = 0; q < w; ++q) rec0 += __popc(bw[q]);
  const uint32_t bits = bw[w];
  const int nrec = __popc(bits);
  if (nrec == 0) return;
  const int t0 = j * kTile + w * 32;
  // token (t0 + lane)'s record word, if selected
  uint32_t my_tok = 0;
  if (((bits >> lane) & 1u) && t0 + lane < N) my_tok = tok[(int64_t)sh * N + t0 + lane];
  const double inv_sqrt_d = 1.0 / sqrt((double)kD);
  // sign bits of elements 16 l8 .. 16 l8 + 15 (bit i set: s = -1)
  const uint32_t sw = l8 < 2 ? cc.sign_bits[0] : l8 < 4 ? cc.sign_bits[1] : l8 < 6 ? cc.sign_bits[2] : cc.sign_bits[3];
  const uint32_t sgn = (sw >> ((l8 & 1) * 16)) & 0xFFFFu;
  const T* X = (side ? V : K) + (int64_t)h * N * kD + l8 * 16;
  const T* A = (side ? anc_v : anc_k) + (int64_t)h * k * kD + l8 * 16;
  for (int base = 0; base < nrec; base += 4) {
    const int i = base + grp;
    const bool act = i < nrec;
    const int b = act ? (int)__fns(bits, 0, i + 1) : 0;
    const int t = t0 + b;
    const int64_t rec = (int64_t)rec0 + i;
    const uint32_t rec_tok = __shfl_sync(0xffffffffu, my_tok, b);
    const uint32_t slot = rec_tok & 0xFFFFu;
    const bool bad = act && (rec >= R || t >= N || slot >= (uint32_t)k);
    if (bad && l8 == 0) latch_error(counters, kDevErrBounds);   // inconsistent record: write nothing
    const bool live = act && !bad;
    const double g = (double)half_bits_to_f(rec_tok >> 16);
    float xf[16], af[16];
    if (live) {
      load16<T>(X + (int64_t)t * kD, xf);
      load16<T>(A + (int64_t)slot * kD, af);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) { xf[e] = 0.f; af[e] = 0.f; }
    }
    double y[16];
    double r2 = 0.0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const double r = (double)xf[e] - g * (double)af[e];
      r2 = fma(r, r, r2);
      y[e] = (!naive && ((sgn >> e) & 1u)) ? -r : r;
    }
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, m);
    if (!naive) {                             // (uniform per launch)
      // Hadamard transform (natural order): four stages on the element bits ...
#pragma unroll
      for (int m = 1; m < 16; m <<= 1)
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (!(e & m)) {
            const double a0 = y[e], a1 = y[e | m];
            y[e] = a0 + a1;
            y[e | m] = a0 - a1;
          }
      // ... and three on the lane bits: y + other below, other - y above,
      // both one fma with a sign of +-1 (exact: one rounding, as the add)
#pragma unroll
      for (int m = 1; m < 8; m <<= 1) {
        const double sg = (l8 & m) ? -1.0 : 1.0;
#pragma unroll
        for (int e = 0; e < 16; ++e) y[e] = fma(y[e], sg, __shfl_xor_sync(0xffffffffu, y[e], m));
      }
    }
    if (!live) continue;
    const uint16_t sb = half_bits_rn(sqrt(r2 / (double)kD));
    const double th = cc.tau * (double)half_bits_to_f(sb);
    const double ysc = naive ? 1.0 : inv_sqrt_d;
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const double v = y[e] * ysc;
      const uint32_t c = (v >= th) ? 3u : (v >= 0.0) ? 2u : (v >= -th) ? 1u : 0u;
      word |= c << (2 * e);
    }
    reinterpret_cast<uint32_t*>(codes + rec * kCodeBytes)[l8] = word;
    if (l8 == 0) sigma[rec] = sb;
  }
}

// ---------------------------------------------------------------- reconstruct

template <typename T>
__global__ void reconstruct_kernel(const uint8_t* __restrict__ comp, anchorkv_layout L, int N, int H, int k,
                                   CodecConst cc, int naive, float* __restrict__ Kh, float* __restrict__ Vh) {
  const int lane = threadIdx.x & 31;
  const int64_t total = 2LL * H * N;
  const int n_tiles = L.n_tiles;
  const uint32_t* tok = reinterpret_cast<const uint32_t*>(comp + L.off_tok);
  const uint32_t* bitmap = reinterpret_cast<const uint32_t*>(comp + L.off_bitmap);
  const int* prefix = reinterpret_cast<const int*>(comp + L.off_tile_prefix);
  const uint8_t* codes = comp + L.off_res_codes;
  const uint16_t* sigma = reinterpret_cast<const uint16_t*>(comp + L.off_res_sigma);
  const float lev[4] = {(float)-cc.l2, (float)-cc.l1, (float)cc.l1, (float)cc.l2};
  for (int64_t f = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); f < total;
       f += (int64_t)gridDim.x * (blockDim.x >> 5)) {
    const int sh = (int)(f / N), t = (int)(f % N);
    const int side = sh / H, h = sh % H;
    const uint32_t rt = tok[f];
    const T* a = reinterpret_cast<const T*>(comp + (side ? L.off_anchors_v : L.off_anchors_k)) +
                 ((int64_t)h * k + (rt & 0xFFFFu)) * kD;
    float af[4];
    load4<T>(a + lane * 4, af);
    const float g = half_bits_to_f(rt >> 16);
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = g * af[e];
    const int j = t / kTile, w = (t % kTile) / 32, b = t % 32;
    const uint32_t* bw = bitmap + ((int64_t)sh * n_tiles + j) * 4;
    if ((bw[w] >> b) & 1u) {
      int rec = prefix[sh * (n_tiles + 1) + j];
      for (int q = 0; q < w; ++q) rec += __popc(bw[q]);
      rec += __popc(bw[w] & ((1u << b) - 1u));
      if (rec >= L.n_residuals) continue;     // corrupt layout: leave the anchor part only
      const float sg = half_bits_to_f(sigma[rec]);
      const uint32_t byte = codes[(int64_t)rec * kCodeBytes + lane];
      float z[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) z[e] = lev[(byte >> (2 * e)) & 3u] * sg;
      if (naive) {                              // unrotated codec: r~ = sigma~ level(code)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] += z[e];
      } else {
        fwht128<float>(z);
        const float isd = rsqrtf((float)kD);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s = ((cc.sign_bits[(lane * 4 + e) >> 5] >> ((lane * 4 + e) & 31)) & 1u) ? -1.f : 1.f;
          o[e] += s * z[e] * isd;
        }
      }
    }
    float* dst = (side ? Vh : Kh) + ((int64_t)h * N + t) * kD + lane * 4;
    *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
  }
}

CodecConst make_cc(const Plan& pl) {
  CodecConst cc;
  cc.tau = pl.tau; cc.l1 = pl.l1; cc.l2 = pl.l2;
  for (int i = 0; i < 4; ++i) cc.sign_bits[i] = pl.sign_bits[i];
  return cc;
}

}  // namespace

cudaError_t launch_project(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  const dim3 blocks((pl.N + kProjTokens * kProjTPQ - 1) / (kProjTokens * kProjTPQ), pl.H, 2);
  auto* n2 = reinterpret_cast<const double*>(ws + pl.o_anc_n2);
  auto* slot_of = reinterpret_cast<const int*>(ws + pl.o_slot_of);
  auto* a2 = reinterpret_cast<const float*>(ws + pl.o_a2);
  auto* ku = reinterpret_cast<const float*>(ws + pl.o_ku);
  auto* sc = reinterpret_cast<const float*>(ws + pl.o_score);
  auto* tok = reinterpret_cast<uint32_t*>(out + pl.L.off_tok);
  auto* util = reinterpret_cast<float*>(ws + pl.o_util);
  const int rank = rank_of(pl);
  auto go = [&](auto kern, auto tag) {
    using T = decltype(tag);
    kern<<<blocks, 256, 0, s>>>(static_cast<const T*>(K), static_cast<const T*>(V),
                                reinterpret_cast<const T*>(out + pl.L.off_anchors_k),
                                reinterpret_cast<const T*>(out + pl.L.off_anchors_v), n2, slot_of, a2, ku, sc, tok,
                                util, pl.N, pl.H, pl.k, pl.obs_rb, rank, pl.p.seed, pl.p.layer);
  };
  if (pl.p.dtype == ANCHORKV_BF16) {
    if (rank == ANCHORKV_RANK_UTILITY) go(project_kernel<__nv_bfloat16, true>, __nv_bfloat16{});
    else go(project_kernel<__nv_bfloat16, false>, __nv_bfloat16{});
  } else {
    if (rank == ANCHORKV_RANK_UTILITY) go(project_kernel<float, true>, float{});
    else go(project_kernel<float, false>, float{});
  }
  return cudaGetLastError();
}

cudaError_t launch_key_queries(const Plan& pl, const void* K, void* Q, cudaStream_t s) {
  const int chunks = kD * pl.elem / 16;
  const int64_t total = (int64_t)pl.Hq * pl.W * chunks;
  const int blocks = (int)((total + 255) / 256);
  key_query_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(K), static_cast<uint4*>(Q), pl.N, pl.W, pl.G,
                                          chunks, total);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  if (pl.R == 0) return cudaSuccess;
  const int n_words = 2 * pl.H * pl.n_tiles * 4;
  const int blocks = (n_words + 7) / 8;
  auto* tok = reinterpret_cast<const uint32_t*>(out + pl.L.off_tok);
  auto* bitmap = reinterpret_cast<const uint32_t*>(out + pl.L.off_bitmap);
  auto* prefix = reinterpret_cast<const int*>(out + pl.L.off_tile_prefix);
  auto* codes = reinterpret_cast<uint8_t*>(out + pl.L.off_res_codes);
  auto* sigma = reinterpret_cast<uint16_t*>(out + pl.L.off_res_sigma);
  const CodecConst cc = make_cc(pl);
  if (pl.p.dtype == ANCHORKV_BF16) {
    quantize_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
        reinterpret_cast<const __nv_bfloat16*>(out + pl.L.off_anchors_k),
        reinterpret_cast<const __nv_bfloat16*>(out + pl.L.off_anchors_v), tok, bitmap, prefix, codes, sigma,
        pl.N, pl.H, pl.k, pl.n_tiles, pl.R, reinterpret_cast<int*>(ws + pl.o_counters), cc, naive_codec(pl));
  } else {
    quantize_kernel<float><<<blocks, 256, 0, s>>>(
        (const float*)K, (const float*)V, reinterpret_cast<const float*>(out + pl.L.off_anchors_k),
        reinterpret_cast<const float*>(out + pl.L.off_anchors_v), tok, bitmap, prefix, codes, sigma,
        pl.N, pl.H, pl.k, pl.n_tiles, pl.R, reinterpret_cast<int*>(ws + pl.o_counters), cc, naive_codec(pl));
  }
  return cudaGetLastError();
}

cudaError_t launch_reconstruct(const Plan& pl, const char* comp, float* Kh, float* Vh, cudaStream_t s) {
  const CodecConst cc = make_cc(pl);
  const int blocks = 148 * 8;
  if (pl.p.dtype == ANCHORKV_BF16)
    reconstruct_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>((const uint8_t*)comp, pl.L, pl.N, pl.H, pl.k, cc,
                                                             naive_codec(pl), Kh, Vh);
  else
    reconstruct_kernel<float><<<blocks, 256, 0, s>>>((const uint8_t*)comp, pl.L, pl.N, pl.H, pl.k, cc,
                                                     naive_codec(pl), Kh, Vh);
  return cudaGetLastError();
}

}  // namespace akv
