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

struct Best {
  float b1, b2;
  int i1;
};

__device__ __forceinline__ void best_push(Best& b, float v, int i) {
  // slots arrive in ascending order within a thread: strict > keeps the lowest
  if (v > b.b1) { b.b2 = b.b1; b.b1 = v; b.i1 = i; }
  else if (v > b.b2) { b.b2 = v; }
}

__device__ __forceinline__ Best best_merge(const Best& a, const Best& b) {
  const bool a_wins = (a.b1 > b.b1) || (a.b1 == b.b1 && a.i1 < b.i1);
  Best w = a_wins ? a : b;
  const Best& l = a_wins ? b : a;
  w.b2 = fmaxf(w.b2, l.b1);
  return w;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
assign_simt_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ anc_k,
                   const T* __restrict__ anc_v, const float* __restrict__ anc_inv,
                   const int* __restrict__ slot_of, uint32_t* __restrict__ tok, int* __restrict__ refine,
                   int* __restrict__ counters, int N, int H, int k) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AsgSmem& sm = *reinterpret_cast<AsgSmem*>(smem_raw);
  const int t0 = blockIdx.x * kTM, h = blockIdx.y, side = blockIdx.z;
  const int nv = min(kTM, N - t0);
  const T* X = (side ? V : K) + (int64_t)h * N * kD;
  const T* A = (side ? anc_v : anc_k) + (int64_t)h * k * kD;
  const float* inv = anc_inv + ((int64_t)side * H + h) * k;
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
  Best best[4];
  for (int i = 0; i < 4; ++i) best[i] = Best{-INFINITY, -INFINITY, 0x7fffffff};

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
      for (int i = 0; i < 4; ++i) best_push(best[i], acc[i][j] * iv, a0 + a);
    }
  }
  // merge across the 16 threads (tx) that share the same 4 tokens
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    Best b = best[i];
#pragma unroll
    for (int o = 8; o; o >>= 1) {
      Best other;
      other.b1 = __shfl_xor_sync(0xffffffffu, b.b1, o);
      other.b2 = __shfl_xor_sync(0xffffffffu, b.b2, o);
      other.i1 = __shfl_xor_sync(0xffffffffu, b.i1, o);
      b = best_merge(b, other);
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
        if (!(best[i].b1 - best[i].b2 > kRefineRel * sm.xn[r])) {
          const int at = atomicAdd(&counters[kRefineRows], 1);
          refine[at] = (side * H + h) * N + t;
        }
      }
      tok[((int64_t)side * H + h) * N + t] = slot;
    }
  }
}

// One warp per listed row: exact fp64 dots against every anchor.
template <typename T>
__global__ void refine_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ anc_k,
                              const T* __restrict__ anc_v, const double* __restrict__ anc_n2,
                              const int* __restrict__ refine, const int* __restrict__ counters,
                              uint32_t* __restrict__ tok, int N, int H, int k) {
  const int lane = threadIdx.x & 31;
  const int n_list = counters[kRefineRows];
  for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n_list;
       i += gridDim.x * (blockDim.x >> 5)) {
    const int f = refine[i];
    const int side = f / (H * N), h = (f / N) % H, t = f % N;
    const T* x = (side ? V : K) + ((int64_t)h * N + t) * kD;
    const T* A = (side ? anc_v : anc_k) + (int64_t)h * k * kD;
    const double* n2 = anc_n2 + ((int64_t)side * H + h) * k;
    float xf[4];
    load4<T>(x + lane * 4, xf);
    double best = -INFINITY;
    int bi = 0;
    for (int s = 0; s < k; ++s) {
      float af[4];
      load4<T>(A + (int64_t)s * kD + lane * 4, af);
      double d = 0.0;
#pragma unroll
      for (int e = 0; e < 4; ++e) d = fma((double)xf[e], (double)af[e], d);
      d = warp_sum_d(d);
      const double nn = n2[s];
      const double c = (nn > 0.0) ? d / sqrt(nn) : 0.0;
      if (c > best) { best = c; bi = s; }
    }
    if (lane == 0) tok[f] = (uint32_t)bi;
  }
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
                                     inv, slot_of, tok, ref, cnt, pl.N, pl.H, pl.k);
  } else {
    auto kfn = assign_simt_kernel<float>;
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kfn<<<grid, kThreads, smem, s>>>((const float*)K, (const float*)V,
                                     reinterpret_cast<const float*>(out + pl.L.off_anchors_k),
                                     reinterpret_cast<const float*>(out + pl.L.off_anchors_v),
                                     inv, slot_of, tok, ref, cnt, pl.N, pl.H, pl.k);
  }
  return cudaGetLastError();
}

cudaError_t launch_refine(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s) {
  auto* n2 = reinterpret_cast<const double*>(ws + pl.o_anc_n2);
  auto* ref = reinterpret_cast<const int*>(ws + pl.o_refine);
  auto* cnt = reinterpret_cast<const int*>(ws + pl.o_counters);
  auto* tok = reinterpret_cast<uint32_t*>(out + pl.L.off_tok);
  if (pl.p.dtype == ANCHORKV_BF16) {
    refine_kernel<__nv_bfloat16><<<2 * 148, 256, 0, s>>>(
        (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
        reinterpret_cast<const __nv_bfloat16*>(out + pl.L.off_anchors_k),
        reinterpret_cast<const __nv_bfloat16*>(out + pl.L.off_anchors_v), n2, ref, cnt, tok, pl.N, pl.H, pl.k);
  } else {
    refine_kernel<float><<<2 * 148, 256, 0, s>>>(
        (const float*)K, (const float*)V, reinterpret_cast<const float*>(out + pl.L.off_anchors_k),
        reinterpret_cast<const float*>(out + pl.L.off_anchors_v), n2, ref, cnt, tok, pl.N, pl.H, pl.k);
  }
  return cudaGetLastError();
}

}  // namespace akv
