// Nearest-anchor assignment, SIMT fp32 path (any dtype), plus the fp64
// re-decision of close calls shared by every assignment path.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary": each key and value vector is assigned to its nearest
// anchor.  Reading: nearest = largest signed cosine, i.e. argmax over slots
// s of <x, a_s>/||a_s||; a zero anchor scores 0; ties go to the lowest slot;
// an anchor token keeps its own slot.
//
// Exactness: the fp32 dot of D = 128 exact products is within
// 2^-17 ||x|| ||a|| of the real value, and 1/||a|| is correctly rounded from
// an exact fp64 norm, so two scaled scores whose fp32 gap exceeds
// kRefineRel * ||x|| (= 2^-13 ||x||, 8x the bound) are ordered correctly.
// Rows closer than that are listed and re-decided by refine_kernel from exact
// fp64 dots (bf16 and fp32 products are exact in fp64), which takes the
// decision in the same precision as a float64 restatement of the rule.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace akv {

constexpr float kRefineRel = 1.0f / 8192.0f;

namespace {

constexpr int kTM = 64, kTN = 64, kPad = 68, kThreads = 256;

struct AsgSmem {
  float xs[kD][kPad];      // token tile, transposed
  float as[kD][kPad];      // anchor chunk, transposed
  float inv[kTN];
  float xn[kTM];
};

template <typename T>
__global__ void __launch_bounds__(kThreads)
assign_simt_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ anc_k,
                   const T* __restrict__ anc_v, const float* __restrict__ anc_inv,
                   const int* __restrict__ slot_of, uint32_t* __restrict__ tok, int* __restrict__ refine,
                   int* __restrict__ counters, int N, int H, int k, int kp16) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AsgSmem& sm = *reinterpret_cast<AsgSmem*>(smem_raw);
  const int t0 = blockIdx.x * kTM, h = blockIdx.y, side = blockIdx.z;
  const int nv = min(kTM, N - t0);
  const T* X = (side ? V : K) + (int64_t)h * N * kD;
  const T* A = (side ? anc_v : anc_k) + (int64_t)h * k * kD;
  const float* inv = anc_inv + ((int64_t)side * H + h) * kp16;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  for (int i = tid; i < kTM * (kD / 4); i += kThreads) {
    const int r = i / (kD / 4), c = (i % (kD / 4)) * 4;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < nv) load4<T>(X + (int64_t)(t0 + r) * kD + c, f);
    for (int e = 0; e < 4; ++e) sm.xs[c + e][r] = f[e];
  }
  __syncthreads();
  if (tid < kTM) {
    float s = 0.f;
    for (int d = 0; d < kD; ++d) s = fmaf(sm.xs[d][tid], sm.xs[d][tid], s);
    sm.xn[tid] = sqrtf(s);
  }
  Top3 best[4];
  for (int i = 0; i < 4; ++i) best[i] = top3_init();

  for (int a0 = 0; a0 < k; a0 += kTN) {
    const int na = min(kTN, k - a0);
    __syncthreads();
    for (int i = tid; i < kTN * (kD / 4); i += kThreads) {
      const int r = i / (kD / 4), c = (i % (kD / 4)) * 4;
      float f[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < na) load4<T>(A + (int64_t)(a0 + r) * kD + c, f);
      for (int e = 0; e < 4; ++e) sm.as[c + e][r] = f[e];
    }
    if (tid < kTN) sm.inv[tid] = (tid < na) ? inv[a0 + tid] : 0.f;
    __syncthreads();
    float acc[4][4];
    for (int i = 0; i < 4; ++i)
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int d = 0; d < kD; ++d) {
      const float4 xv = *reinterpret_cast<const float4*>(&sm.xs[d][ty * 4]);
      const float4 av = *reinterpret_cast<const float4*>(&sm.as[d][tx * 4]);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w}, aa[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], aa[j], acc[i][j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int a = tx * 4 + j;
      if (a >= na) continue;
      const float iv = sm.inv[a];
#pragma unroll
      for (int i = 0; i < 4; ++i) push(best[i], acc[i][j] * iv, a0 + a);
    }
  }
  // merge across the 16 threads (tx) that share the same 4 tokens
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    Top3 b = best[i];
#pragma unroll
    for (int o = 8; o; o >>= 1) {
      Top3 other;
      other.b1 = __shfl_xor_sync(0xffffffffu, b.b1, o);
      other.b2 = __shfl_xor_sync(0xffffffffu, b.b2, o);
      other.b3 = __shfl_xor_sync(0xffffffffu, b.b3, o);
      other.i1 = __shfl_xor_sync(0xffffffffu, b.i1, o);
      other.i2 = __shfl_xor_sync(0xffffffffu, b.i2, o);
      b = merge(b, other);
    }
    best[i] = b;
  }
  if (tx == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
      if (r >= nv) continue;
      const int t = t0 + r;
      const int own = slot_of[(int64_t)h * N + t];
      uint32_t slot;
      if (own >= 0) {
        slot = (uint32_t)own;
      } else {
        slot = (uint32_t)best[i].i1;
        if (!(best[i].b1 - best[i].b2 > kRefineRel * sm.xn[r])) list_for_refine(refine, counters, side * H + h, N, t);
      }
      tok[((int64_t)side * H + h) * N + t] = slot;
    }
  }
}

// Re-decision of the listed rows of one (side, head) per blockIdx.y.
// The block stages the head's anchors in shared memory transposed as
// (d, d+1) pairs per slot, so that lanes scoring consecutive slots read
// consecutive words.  Each warp takes one row: fp32 scores of every slot
// (sequential FMA over D = 128 exact products: error <= 2^-17 ||x|| after
// scaling), candidates within 2^-14 ||x|| of the best fp32 score, and the
// exact fp64 score dot / sqrt(||a||^2) of each candidate (correctly rounded
// sqrt and division) decides; ties go to the lowest slot.
constexpr int kRefineWarps = 8;
constexpr int kRefineMaxK = 2048;
template <typename T> struct RefineCfg;
// kChunk slots per staging round; the transposed rows are kChunk + 1 pairs
// apart so that the staging stores of consecutive pairs fall in different banks.
template <> struct RefineCfg<__nv_bfloat16> { using P = __nv_bfloat162; static constexpr int kChunk = 448; };
template <> struct RefineCfg<float> { using P = float2; static constexpr int kChunk = 192; };
template <typename T> __host__ __device__ constexpr int refine_ld() { return RefineCfg<T>::kChunk + 1; }

__device__ __forceinline__ float2 pair_f(__nv_bfloat162 p) { return __bfloat1622float2(p); }
__device__ __forceinline__ float2 pair_f(float2 p) { return p; }

template <typename T>
__global__ void __launch_bounds__(kRefineWarps * 32)
refine_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ anc_k,
              const T* __restrict__ anc_v, const float* __restrict__ anc_inv, const double* __restrict__ anc_sqrt,
              const int* __restrict__ refine, const int* __restrict__ counters, uint32_t* __restrict__ tok, int N,
              int H, int k, int kp16) {
  using P = typename RefineCfg<T>::P;
  constexpr int CH = RefineCfg<T>::kChunk;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int LD = refine_ld<T>();
  P* aT = reinterpret_cast<P*>(smem_raw);                              // [64][LD]
  float* xs = reinterpret_cast<float*>(aT + 64 * LD);                  // [8][128]
  float* sc = xs + kRefineWarps * kD;                                  // [8][kRefineMaxK]
  const int u = blockIdx.y, side = u / H, h = u % H;
  const int n = counters[kRefineListBase + u];
  if ((int)blockIdx.x * kRefineWarps >= n) return;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const T* A = (side ? anc_v : anc_k) + (int64_t)h * k * kD;
  const float* inv = anc_inv + (int64_t)u * kp16;
  const double* sq = anc_sqrt + (int64_t)u * k;
  float* xw = xs + w * kD;
  float* sw = sc + w * kRefineMaxK;
  auto stage = [&](int c0, int cn) {
    __syncthreads();
    for (int i = threadIdx.x; i < cn * 64; i += blockDim.x) {
      const int j = i / 64, dp = i % 64;
      const T* src = A + (int64_t)(c0 + j) * kD + 2 * dp;
      aT[dp * LD + j] = *reinterpret_cast<const P*>(src);
    }
    __syncthreads();
  };
  const bool one_chunk = k <= CH;
  if (one_chunk) stage(0, k);
  for (int base = blockIdx.x * kRefineWarps; base < n; base += gridDim.x * kRefineWarps) {
    const int i = base + w;
    const bool live = i < n;
    const int t = live ? refine[(int64_t)u * N + i] : 0;
    const T* x = (side ? V : K) + ((int64_t)h * N + t) * kD;
    float xf[4];
    load4<T>(x + lane * 4, xf);
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 4; ++e) xw[lane * 4 + e] = xf[e];
    const float xn = sqrtf(warp_sum(xf[0] * xf[0] + xf[1] * xf[1] + xf[2] * xf[2] + xf[3] * xf[3]));
    __syncwarp();
    float best = -INFINITY;
    for (int c0 = 0; c0 < k; c0 += CH) {
      const int cn = min(CH, k - c0);
      if (!one_chunk) stage(c0, cn);
      for (int j = lane; j < cn; j += 32) {
        float acc = 0.f;
#pragma unroll 8
        for (int dp = 0; dp < 64; ++dp) {
          const float2 av = pair_f(aT[dp * LD + j]);
          acc = fmaf(xw[2 * dp], av.x, acc);
          acc = fmaf(xw[2 * dp + 1], av.y, acc);
        }
        const float s = acc * inv[c0 + j];
        sw[c0 + j] = s;
        best = fmaxf(best, s);
      }
    }
    best = warp_max(best);
    __syncwarp();
    const float thr = best - xn * (1.0f / 16384.0f);
    double cbest = -INFINITY;
    int cbi = 0x7fffffff;
    for (int j0 = 0; j0 < k; j0 += 32) {
      const int j = j0 + lane;
      uint32_t cand = __ballot_sync(0xffffffffu, j < k && sw[j] >= thr);
      while (cand) {
        const int s = j0 + __ffs(cand) - 1;
        cand &= cand - 1;
        float af[4];
        load4<T>(A + (int64_t)s * kD + lane * 4, af);
        double d = 0.0;
#pragma unroll
        for (int e = 0; e < 4; ++e) d = fma((double)xf[e], (double)af[e], d);
        d = warp_sum_d(d);
        const double nn = sq[s];
        const double cs = (nn > 0.0) ? d / nn : 0.0;
        if (cs > cbest) { cbest = cs; cbi = s; }
      }
    }
    if (live && lane == 0 && cbi < k) tok[(int64_t)u * N + t] = (uint32_t)cbi;
  }
}

template <typename T>
constexpr int refine_smem() {
  return 64 * refine_ld<T>() * (int)sizeof(typename RefineCfg<T>::P) + kRefineWarps * kD * 4 +
         kRefineWarps * kRefineMaxK * 4;
}

}  // namespace

cudaError_t launch_assign_simt(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  dim3 grid((pl.N + kTM - 1) / kTM, pl.H, 2);
  const size_t smem = sizeof(AsgSmem);
  auto* inv = reinterpret_cast<const float*>(ws + pl.o_anc_inv);
  auto* slot_of = reinterpret_cast<const int*>(ws + pl.o_slot_of);
  auto* tok = reinterpret_cast<uint32_t*>(out + pl.L.off_tok);
  auto* ref = reinterpret_cast<int*>(ws + pl.o_refine);
  auto* cnt = reinterpret_cast<int*>(ws + pl.o_counters);
  if (pl.p.dtype == ANCHORKV_BF16) {
    auto kfn = assign_simt_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kfn<<<grid, kThreads, smem, s>>>((const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
                                     reinterpret_cast<const __nv_bfloat16*>(out + pl.L.off_anchors_k),
                                     reinterpret_cast<const __nv_bfloat16*>(out + pl.L.off_anchors_v),
                                     inv, slot_of, tok, ref, cnt, pl.N, pl.H, pl.k, pl.kp16);
  } else {
    auto kfn = assign_simt_kernel<float>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kfn<<<grid, kThreads, smem, s>>>((const float*)K, (const float*)V,
                                     reinterpret_cast<const float*>(out + pl.L.off_anchors_k),
                                     reinterpret_cast<const float*>(out + pl.L.off_anchors_v),
                                     inv, slot_of, tok, ref, cnt, pl.N, pl.H, pl.k, pl.kp16);
  }
  return cudaGetLastError();
}

cudaError_t launch_refine(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  auto* sq = reinterpret_cast<const double*>(ws + pl.o_anc_sqrt);
  auto* inv = reinterpret_cast<const float*>(ws + pl.o_anc_inv);
  auto* ref = reinterpret_cast<const int*>(ws + pl.o_refine);
  auto* cnt = reinterpret_cast<const int*>(ws + pl.o_counters);
  auto* tok = reinterpret_cast<uint32_t*>(out + pl.L.off_tok);
  // a few CTAs per (side, head) list; the lists are short (about 1% of rows)
  const dim3 grid(std::max(1, 2 * 148 / (2 * pl.H)), 2 * pl.H);
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    auto kfn = refine_kernel<T>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, refine_smem<T>());
    kfn<<<grid, kRefineWarps * 32, refine_smem<T>(), s>>>(
        (const T*)K, (const T*)V, reinterpret_cast<const T*>(out + pl.L.off_anchors_k),
        reinterpret_cast<const T*>(out + pl.L.off_anchors_v), inv, sq, ref, cnt, tok, pl.N, pl.H, pl.k, pl.kp16);
  } else {
    using T = float;
    auto kfn = refine_kernel<T>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, refine_smem<T>());
    kfn<<<grid, kRefineWarps * 32, refine_smem<T>(), s>>>(
        (const T*)K, (const T*)V, reinterpret_cast<const T*>(out + pl.L.off_anchors_k),
        reinterpret_cast<const T*>(out + pl.L.off_anchors_v), inv, sq, ref, cnt, tok, pl.N, pl.H, pl.k, pl.kp16);
  }
  return cudaGetLastError();
}

}  // namespace akv
