// Decode attention over the compressed layout (split over tokens).
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary": a FlashAttention-style decoder rebuilds tiles when they
// are consumed; "AnchorKV-adapted" (VeloxQuant-MLX), "Adaptation notes":
// decode tokens are appended at full precision.
//
// The rebuild is factored so that only compressed bytes are read per token:
//   K^_t = g^K_t a^K_{i(t)} + r~^K_t, r~ = s . H(sigma~ lev(c))   (H orthonormal,
//   symmetric), so
//   q . K^_t / sqrt(D) = g^K_t P[i(t)] + sigma~_t <H(s . q)/sqrt(D), lev(c_t)>
// with P[a] = q . a^K_a / sqrt(D) computed once per (sequence, KV head); and
//   sum_t p_t V^_t = sum_a W[a] a^V_a + s . H(Z),
//   W[a] = sum_{t: i(t)=a} p_t g^V_t,  Z = sum_t p_t sigma~_t lev(c_t),
// so a token costs its 8 record bytes, plus 34 bytes per residual side.
// Each split writes (max, sum, W, Z) per query head; the combine merges the
// splits in order, adds the exact tail tokens and rebuilds the output.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kMaxG = 16;

struct DecodeArgs {
  const uint8_t* comp;
  int64_t stride;
  anchorkv_layout L;
  int N, H, G, k, n_tiles, n_split, split_tokens;
  int64_t R;
  float* P;      // [b][h][G][k]
  float* qrot;   // [b][h][G][D]
  float* pm;     // [b][h][split][G]
  float* plx;    // [b][h][split][G]
  float* pw;     // [b][h][split][G][k]
  float* pz;     // [b][h][split][G][D]
  float lev[4];
  uint32_t sign_bits[4];
  int naive;     // unrotated codec: residuals live in the token domain
};

__device__ __forceinline__ float sgnf(const DecodeArgs& a, int j) {
  return ((a.sign_bits[j >> 5] >> (j & 31)) & 1u) ? -1.f : 1.f;
}

// grid (ceil(k / 32), batch * H): P for 32 anchors per CTA; CTA x == 0 also
// writes the rotated queries.
template <typename T>
__global__ void decode_prep_kernel(DecodeArgs a, const T* __restrict__ q) {
  __shared__ float qs[kMaxG][kD];
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float isd = rsqrtf((float)kD);
  for (int i = threadIdx.x; i < a.G * kD; i += blockDim.x) {
    const int j = i / kD, d = i % kD;
    qs[j][d] = to_f<T>(q[((int64_t)b * a.H * a.G + h * a.G + j) * kD + d]);
  }
  __syncthreads();
  const T* anc = reinterpret_cast<const T*>(a.comp + (int64_t)b * a.stride + a.L.off_anchors_k) +
                 (int64_t)h * a.k * kD;
  for (int s = blockIdx.x * 32 + warp; s < min(a.k, blockIdx.x * 32 + 32); s += blockDim.x >> 5) {
    float af[4];
    load4<T>(anc + (int64_t)s * kD + lane * 4, af);
    for (int j = 0; j < a.G; ++j) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) d = fmaf(qs[j][lane * 4 + e], af[e], d);
      d = warp_sum(d);
      if (lane == 0) a.P[((int64_t)bh * a.G + j) * a.k + s] = d * isd;
    }
  }
  if (blockIdx.x == 0) {
    for (int j = warp; j < a.G; j += blockDim.x >> 5) {
      float v[4];
      float* dst = a.qrot + ((int64_t)bh * a.G + j) * kD + lane * 4;
      if (a.naive) {
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = qs[j][lane * 4 + e] * isd;
        continue;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = qs[j][lane * 4 + e] * sgnf(a, lane * 4 + e);
      fwht128<float>(v);
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = v[e] * isd * isd;   // orthonormal H, then 1/sqrt(D)
    }
  }
}

// grid (n_split, batch * H), 256 threads.  Dynamic smem:
//   P [G][k], W [G][k], shat [G][split_tokens], qrot [G][D], Z [G][D]
template <typename T>
__global__ void __launch_bounds__(256) decode_split_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int split = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int G = a.G, k = a.k;
  float* Ps = sm;
  float* Ws = Ps + G * k;
  float* shat = Ws + G * k;
  float* qr = shat + G * a.split_tokens;
  float* Zs = qr + G * kD;
  __shared__ float red[kMaxG][8];
  __shared__ float mrow[kMaxG], lrow[kMaxG];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint8_t* comp = a.comp + (int64_t)b * a.stride;
  const uint32_t* tokK = reinterpret_cast<const uint32_t*>(comp + a.L.off_tok) + (int64_t)h * a.N;
  const uint32_t* tokV = reinterpret_cast<const uint32_t*>(comp + a.L.off_tok) + ((int64_t)a.H + h) * a.N;
  const uint32_t* bmK = reinterpret_cast<const uint32_t*>(comp + a.L.off_bitmap) + (int64_t)h * a.n_tiles * 4;
  const uint32_t* bmV = reinterpret_cast<const uint32_t*>(comp + a.L.off_bitmap) + ((int64_t)a.H + h) * a.n_tiles * 4;
  const int* pfK = reinterpret_cast<const int*>(comp + a.L.off_tile_prefix) + (int64_t)h * (a.n_tiles + 1);
  const int* pfV = reinterpret_cast<const int*>(comp + a.L.off_tile_prefix) + ((int64_t)a.H + h) * (a.n_tiles + 1);
  const uint8_t* codes = comp + a.L.off_res_codes;
  const uint16_t* sig = reinterpret_cast<const uint16_t*>(comp + a.L.off_res_sigma);

  for (int i = threadIdx.x; i < G * k; i += blockDim.x) {
    Ps[i] = a.P[(int64_t)bh * G * k + i];
    Ws[i] = 0.f;
  }
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
    qr[i] = a.qrot[(int64_t)bh * G * kD + i];
    Zs[i] = 0.f;
  }
  __syncthreads();
  const int t0 = split * a.split_tokens;
  const int nt = min(a.split_tokens, a.N - t0);
  // phase 1a: anchor part of every key logit
  for (int i = threadIdx.x; i < nt; i += blockDim.x) {
    const uint32_t r = tokK[t0 + i];
    const uint32_t slot = min((int)(r & 0xFFFFu), k - 1);
    const float g = half_bits_to_f(r >> 16);
    for (int j = 0; j < G; ++j) shat[j * a.split_tokens + i] = g * Ps[j * k + slot];
  }
  __syncthreads();
  // phase 1b: key residuals, one warp per 32-token bitmap word
  const int j0 = t0 / kTile, nwords = (nt + 31) / 32;
  for (int wd = warp; wd < nwords; wd += 8) {
    const int tile = j0 + wd / 4, w = wd % 4;
    const uint32_t* bw = bmK + (int64_t)tile * 4;
    uint32_t bits = bw[w];
    int rec = pfK[tile];
    for (int q = 0; q < w; ++q) rec += __popc(bw[q]);
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int i = wd * 32 + bit;
      if (rec >= a.R || i >= nt) break;      // corrupt layout: ignore the rest of the word
      const float sg = half_bits_to_f(sig[rec]);
      const uint32_t byte = codes[(int64_t)rec * kCodeBytes + lane];
      float lv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) lv[e] = a.lev[(byte >> (2 * e)) & 3u];
      for (int j = 0; j < G; ++j) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) d = fmaf(qr[j * kD + lane * 4 + e], lv[e], d);
        d = warp_sum(d);
        if (lane == 0) shat[j * a.split_tokens + i] += sg * d;
      }
      ++rec;
    }
  }
  __syncthreads();
  // phase 2: split max and sum per query head
  for (int j = 0; j < G; ++j) {
    float m = -INFINITY;
    for (int i = threadIdx.x; i < nt; i += blockDim.x) m = fmaxf(m, shat[j * a.split_tokens + i]);
    m = warp_max(m);
    if (lane == 0) red[j][warp] = m;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float m = -INFINITY;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[threadIdx.x][w]);
    mrow[threadIdx.x] = m;
  }
  __syncthreads();
  for (int j = 0; j < G; ++j) {
    float l = 0.f;
    for (int i = threadIdx.x; i < nt; i += blockDim.x) {
      const float p = expf(shat[j * a.split_tokens + i] - mrow[j]);
      shat[j * a.split_tokens + i] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) red[j][warp] = l;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float l = 0.f;
    for (int w = 0; w < 8; ++w) l += red[threadIdx.x][w];
    lrow[threadIdx.x] = l;
  }
  // phase 3a: value anchors, weights scattered to their slot
  for (int i = threadIdx.x; i < nt; i += blockDim.x) {
    const uint32_t r = tokV[t0 + i];
    const uint32_t slot = min((int)(r & 0xFFFFu), k - 1);
    const float g = half_bits_to_f(r >> 16);
    for (int j = 0; j < G; ++j) atomicAdd(&Ws[j * k + slot], shat[j * a.split_tokens + i] * g);
  }
  // phase 3b: value residuals in the rotated domain
  float zacc[kMaxG][4];
  for (int j = 0; j < kMaxG; ++j) zacc[j][0] = zacc[j][1] = zacc[j][2] = zacc[j][3] = 0.f;
  for (int wd = warp; wd < nwords; wd += 8) {
    const int tile = j0 + wd / 4, w = wd % 4;
    const uint32_t* bw = bmV + (int64_t)tile * 4;
    uint32_t bits = bw[w];
    int rec = pfV[tile];
    for (int q = 0; q < w; ++q) rec += __popc(bw[q]);
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int i = wd * 32 + bit;
      if (rec >= a.R || i >= nt) break;
      const float sg = half_bits_to_f(sig[rec]);
      const uint32_t byte = codes[(int64_t)rec * kCodeBytes + lane];
      float lv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) lv[e] = a.lev[(byte >> (2 * e)) & 3u] * sg;
#pragma unroll
      for (int j = 0; j < kMaxG; ++j) {
        if (j < G) {
          const float p = shat[j * a.split_tokens + i];
#pragma unroll
          for (int e = 0; e < 4; ++e) zacc[j][e] = fmaf(p, lv[e], zacc[j][e]);
        }
      }
      ++rec;
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxG; ++j)
    if (j < G)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (zacc[j][e] != 0.f) atomicAdd(&Zs[j * kD + lane * 4 + e], zacc[j][e]);
  __syncthreads();
  const int64_t ps = (int64_t)bh * a.n_split + split;
  if (threadIdx.x < G) {
    a.pm[ps * G + threadIdx.x] = mrow[threadIdx.x];
    a.plx[ps * G + threadIdx.x] = lrow[threadIdx.x];
  }
  for (int i = threadIdx.x; i < G * k; i += blockDim.x) a.pw[ps * G * k + i] = Ws[i];
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) a.pz[ps * G * kD + i] = Zs[i];
}

// grid (batch * H), 256 threads: merge splits in order, add the exact tail.
template <typename T>
__global__ void __launch_bounds__(256)
decode_combine_kernel(DecodeArgs a, const T* __restrict__ q, const T* __restrict__ Kt, const T* __restrict__ Vt,
                      int tail_len, int tail_cap, float* __restrict__ out) {
  extern __shared__ __align__(16) float sm[];
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int G = a.G, k = a.k;
  float* Wt = sm;                               // [G][k]
  float* ptail = Wt + G * k;                    // [G][tail_len]
  __shared__ float qs[kMaxG][kD];
  __shared__ float Mrow[kMaxG], Lrow[kMaxG], zrot[kMaxG][kD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float isd = rsqrtf((float)kD);
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x)
    qs[i / kD][i % kD] = to_f<T>(q[((int64_t)b * a.H * G + h * G) * kD + i]);
  __syncthreads();
  const T* Kth = Kt ? Kt + ((int64_t)b * a.H + h) * tail_cap * kD : nullptr;
  const T* Vth = Vt ? Vt + ((int64_t)b * a.H + h) * tail_cap * kD : nullptr;
  // tail logits (exact)
  for (int ti = warp; ti < tail_len; ti += 8) {
    float kf[4];
    load4<T>(Kth + (int64_t)ti * kD + lane * 4, kf);
    for (int j = 0; j < G; ++j) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) d = fmaf(qs[j][lane * 4 + e], kf[e], d);
      d = warp_sum(d);
      if (lane == 0) ptail[j * tail_len + ti] = d * isd;
    }
  }
  __syncthreads();
  const int64_t ps0 = (int64_t)bh * a.n_split;
  if (threadIdx.x < G) {
    const int j = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, a.pm[(ps0 + s) * G + j]);
    for (int ti = 0; ti < tail_len; ++ti) M = fmaxf(M, ptail[j * tail_len + ti]);
    float L = 0.f;
    for (int s = 0; s < a.n_split; ++s) L += a.plx[(ps0 + s) * G + j] * expf(a.pm[(ps0 + s) * G + j] - M);
    for (int ti = 0; ti < tail_len; ++ti) {
      const float p = expf(ptail[j * tail_len + ti] - M);
      ptail[j * tail_len + ti] = p;
      L += p;
    }
    Mrow[j] = M;
    Lrow[j] = L;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * k; i += blockDim.x) {
    const int j = i / k;
    float w = 0.f;
    for (int s = 0; s < a.n_split; ++s)
      w = fmaf(a.pw[(ps0 + s) * G * k + i], expf(a.pm[(ps0 + s) * G + j] - Mrow[j]), w);
    Wt[i] = w;
  }
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
    const int j = i / kD;
    float z = 0.f;
    for (int s = 0; s < a.n_split; ++s)
      z = fmaf(a.pz[(ps0 + s) * G * kD + i], expf(a.pm[(ps0 + s) * G + j] - Mrow[j]), z);
    zrot[j][i % kD] = z;
  }
  __syncthreads();
  // rotate Z back: s . H(Z), one warp per head (not for the unrotated codec)
  for (int j = warp; j < G && !a.naive; j += 8) {
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = zrot[j][lane * 4 + e];
    fwht128<float>(v);
#pragma unroll
    for (int e = 0; e < 4; ++e) zrot[j][lane * 4 + e] = v[e] * isd * sgnf(a, lane * 4 + e);
  }
  __syncthreads();
  const T* ancv = reinterpret_cast<const T*>(a.comp + (int64_t)b * a.stride + a.L.off_anchors_v) +
                  (int64_t)h * k * kD;
  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
    const int j = i / kD, d = i % kD;
    float o = zrot[j][d];
    for (int s = 0; s < k; ++s) o = fmaf(Wt[j * k + s], to_f<T>(ancv[(int64_t)s * kD + d]), o);
    for (int ti = 0; ti < tail_len; ++ti) o = fmaf(ptail[j * tail_len + ti], to_f<T>(Vth[(int64_t)ti * kD + d]), o);
    out[((int64_t)b * a.H * G + h * G + j) * kD + d] = o / Lrow[j];
  }
}

}  // namespace

int make_decode_plan(const Plan& pl, int batch, DecodePlan* dp, bool allow_prepass) {
  dp->batch = batch;
  dp->flash = flash_decode_plan(pl, batch, &dp->fs, allow_prepass);
  if (dp->flash) {
    dp->n_split = 0; dp->split_tokens = 0;
    dp->o_P = dp->o_qrot = dp->o_part_m = dp->o_part_l = dp->o_part_w = dp->o_part_z = 0;
    dp->ws_total = dp->fs.ws_total;
    return ANCHORKV_OK;
  }
  const int units = std::max(1, batch * pl.H);
  int want = std::max(1, (2 * 148 + units - 1) / units);
  int tiles_per = std::max(1, (pl.n_tiles + want - 1) / want);
  tiles_per = std::min(tiles_per, 16);                  // <= 2048 tokens per split
  dp->split_tokens = tiles_per * kTile;
  dp->n_split = (pl.N + dp->split_tokens - 1) / dp->split_tokens;
  const int64_t bh = (int64_t)batch * pl.H;
  int64_t off = 0;
  auto take = [&](int64_t bytes) { int64_t o = off; off += (bytes + 255) / 256 * 256; return o; };
  dp->o_P = take(bh * pl.G * pl.k * 4);
  dp->o_qrot = take(bh * pl.G * kD * 4);
  dp->o_part_m = take(bh * dp->n_split * pl.G * 4);
  dp->o_part_l = take(bh * dp->n_split * pl.G * 4);
  dp->o_part_w = take(bh * dp->n_split * pl.G * pl.k * 4);
  dp->o_part_z = take(bh * dp->n_split * pl.G * kD * 4);
  dp->ws_total = off;
  return ANCHORKV_OK;
}

int check_decode_shape(const Plan& pl, const DecodePlan& dp, int tail_len) {
  if ((int64_t)dp.batch * pl.H > 65535) return ANCHORKV_EUNSUPPORTED;   // (sequence, head) pairs: grid y
  if (dp.flash) return ANCHORKV_OK;
  if ((int64_t)dp.batch * pl.H > 65535) return ANCHORKV_EUNSUPPORTED;   // (sequence, head) pairs: grid y
  const size_t smem_split = sizeof(float) * ((size_t)2 * pl.G * pl.k + (size_t)pl.G * dp.split_tokens + 2 * pl.G * kD);
  const size_t smem_comb = sizeof(float) * ((size_t)pl.G * pl.k + (size_t)pl.G * std::max(tail_len, 1));
  if (smem_split > 220 * 1024 || smem_comb > 180 * 1024) return ANCHORKV_EUNSUPPORTED;
  return ANCHORKV_OK;
}

int launch_decode(const Plan& pl, const DecodePlan& dp, const char* comp, int64_t stride, const void* q,
                  const void* Kt, const void* Vt, int tail_len, int tail_cap, float* out, char* ws, cudaStream_t s) {
  if (dp.flash) return launch_flash_decode(pl, dp.fs, dp.batch, comp, stride, q, Kt, Vt, tail_len, tail_cap, out, ws, s);
  DecodeArgs a;
  a.comp = reinterpret_cast<const uint8_t*>(comp);
  a.stride = stride;
  a.L = pl.L;
  a.N = pl.N; a.H = pl.H; a.G = pl.G; a.k = pl.k; a.n_tiles = pl.n_tiles;
  a.n_split = dp.n_split; a.split_tokens = dp.split_tokens;
  a.R = pl.R;
  a.P = reinterpret_cast<float*>(ws + dp.o_P);
  a.qrot = reinterpret_cast<float*>(ws + dp.o_qrot);
  a.pm = reinterpret_cast<float*>(ws + dp.o_part_m);
  a.plx = reinterpret_cast<float*>(ws + dp.o_part_l);
  a.pw = reinterpret_cast<float*>(ws + dp.o_part_w);
  a.pz = reinterpret_cast<float*>(ws + dp.o_part_z);
  a.lev[0] = (float)-pl.l2; a.lev[1] = (float)-pl.l1; a.lev[2] = (float)pl.l1; a.lev[3] = (float)pl.l2;
  for (int i = 0; i < 4; ++i) a.sign_bits[i] = pl.sign_bits[i];
  a.naive = naive_codec(pl);
  const int bh = dp.batch * pl.H;
  dim3 gp((pl.k + 31) / 32, bh);
  const size_t smem_split = sizeof(float) * ((size_t)2 * pl.G * pl.k + (size_t)pl.G * dp.split_tokens + 2 * pl.G * kD);
  const size_t smem_comb = sizeof(float) * ((size_t)pl.G * pl.k + (size_t)pl.G * std::max(tail_len, 1));
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    stage_begin(kStDecodePrep, s);
    decode_prep_kernel<T><<<gp, 256, 0, s>>>(a, (const T*)q);
    stage_end(kStDecodePrep, s, 1);
    auto ks = decode_split_kernel<T>;
    cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_split);
    stage_begin(kStDecodeSplit, s);
    ks<<<dim3(dp.n_split, bh), 256, smem_split, s>>>(a);
    stage_end(kStDecodeSplit, s, 1);
    auto kc = decode_combine_kernel<T>;
    cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_comb);
    stage_begin(kStDecodeCombine, s);
    kc<<<bh, 256, smem_comb, s>>>(a, (const T*)q, (const T*)Kt, (const T*)Vt, tail_len, tail_cap, out);
    stage_end(kStDecodeCombine, s, 1);
  } else {
    using T = float;
    stage_begin(kStDecodePrep, s);
    decode_prep_kernel<T><<<gp, 256, 0, s>>>(a, (const T*)q);
    stage_end(kStDecodePrep, s, 1);
    auto ks = decode_split_kernel<T>;
    cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_split);
    stage_begin(kStDecodeSplit, s);
    ks<<<dim3(dp.n_split, bh), 256, smem_split, s>>>(a);
    stage_end(kStDecodeSplit, s, 1);
    auto kc = decode_combine_kernel<T>;
    cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_comb);
    stage_begin(kStDecodeCombine, s);
    kc<<<bh, 256, smem_comb, s>>>(a, (const T*)q, (const T*)Kt, (const T*)Vt, tail_len, tail_cap, out);
    stage_end(kStDecodeCombine, s, 1);
  }
  return cudaGetLastError() == cudaSuccess ? ANCHORKV_OK : ANCHORKV_ECUDA;
}

}  // namespace akv
