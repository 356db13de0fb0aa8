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
// The (side, head) lists are walked as one flat sequence (their lengths are
// very uneven), one listed row per warp; nothing is staged: the anchors stay
// in L2 (k x 256 bytes, shared by every row of the list).  Scores go 32 slots
// at a time: lane l holds coordinates 4l .. 4l + 3 of the row and of each of
// the 32 anchors (coalesced loads, all 32 in flight together), and a transposed butterfly
// leaves slot j0 + l's dot product on lane l.  fp32 products of exact inputs
// summed in any order err by at most 127 u sum|x_d a_d| <= 2^-17 ||x|| ||a||,
// so after scaling by 1/||a|| every slot within 2^-14 ||x|| of the best fp32
// score is a candidate.  Candidates are gathered 32 at a time and each lane
// takes one: the exact fp64 score dot / sqrt(||a||^2) (correctly rounded
// sqrt and division) decides, ties to the lowest slot.
constexpr int kRefineWarps = 8;
constexpr int kRefineMaxK = 2048;

template <typename T> struct RawRow;    // 4 consecutive elements as loaded
template <> struct RawRow<__nv_bfloat16> {
  uint2 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = *reinterpret_cast<const uint2*>(p); }
  __device__ __forceinline__ float dot(const float (&x)[4]) const {
    return fmaf(x[3], __uint_as_float(v.y & 0xFFFF0000u), fmaf(x[2], __uint_as_float(v.y << 16),
           fmaf(x[1], __uint_as_float(v.x & 0xFFFF0000u), x[0] * __uint_as_float(v.x << 16))));
  }
};
template <> struct RawRow<float> {
  float4 v;
  __device__ __forceinline__ void load(const float* p) { v = *reinterpret_cast<const float4*>(p); }
  __device__ __forceinline__ float dot(const float (&x)[4]) const {
    return fmaf(x[3], v.w, fmaf(x[2], v.z, fmaf(x[1], v.y, x[0] * v.x)));
  }
};

// One lane's exact fp64 score of slot s against the row held in shared memory.
template <typename T>
__device__ __forceinline__ double exact_score(const T* A, const float* xw, const double* sq, int s) {
  const T* a = A + (int64_t)s * kD;
  double d = 0.0;
#pragma unroll 4
  for (int c = 0; c < kD; c += 4) {
    float af[4];
    load4<T>(a + c, af);
#pragma unroll
    for (int e = 0; e < 4; ++e) d = fma((double)xw[c + e], (double)af[e], d);
  }
  const double nn = sq[s];
  return nn > 0.0 ? d / nn : 0.0;
}

template <typename T>
__global__ void __launch_bounds__(kRefineWarps * 32, 3)
refine_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ anc_k,
              const T* __restrict__ anc_v, const float* __restrict__ anc_inv, const double* __restrict__ anc_sqrt,
              const int* __restrict__ refine, const int* __restrict__ counters, uint32_t* __restrict__ tok, int N,
              int H, int k, int kp16) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* sc = reinterpret_cast<float*>(smem_raw);                      // [8][kRefineMaxK]
  float* xs = sc + kRefineWarps * kRefineMaxK;                         // [8][128]
  int* cs_all = reinterpret_cast<int*>(xs + kRefineWarps * kD);        // [8][32]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* sw = sc + w * kRefineMaxK;
  float* xw = xs + w * kD;
  int* cl = cs_all + w * 32;
  int total = 0;
  for (int u = 0; u < 2 * H; ++u) total += counters[kRefineListBase + u];
  for (int g = blockIdx.x * kRefineWarps + w; g < total; g += gridDim.x * kRefineWarps) {
    int u = 0, i = g;
    while (i >= counters[kRefineListBase + u]) i -= counters[kRefineListBase + u++];
    const int side = u / H, h = u % H;
    const T* A = (side ? anc_v : anc_k) + (int64_t)h * k * kD;
    const float* inv = anc_inv + (int64_t)u * kp16;
    const double* sq = anc_sqrt + (int64_t)u * k;
    const int t = refine[(int64_t)u * N + i];
    float xf[4];
    load4<T>((side ? V : K) + ((int64_t)h * N + t) * kD + lane * 4, xf);
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 4; ++e) xw[lane * 4 + e] = xf[e];
    const float xn = sqrtf(warp_sum(xf[0] * xf[0] + xf[1] * xf[1] + xf[2] * xf[2] + xf[3] * xf[3]));
    float best = -INFINITY;
    const T* Al = A + lane * 4;
    for (int j0 = 0; j0 < k; j0 += 32) {
      RawRow<T> r[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        if (j0 + jj < k) r[jj].load(Al + (int64_t)(j0 + jj) * kD);
        else r[jj].v = {};
      }
      float v[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) v[jj] = r[jj].dot(xf);
      transpose_reduce32(v, lane);
      const int j = j0 + lane;
      if (j < k) {
        const float s = v[0] * inv[j];
        sw[j] = s;
        best = fmaxf(best, s);
      }
    }
    best = warp_max(best);
    __syncwarp();
    const float thr = best - xn * (1.0f / 16384.0f);
    double cbest = -INFINITY;
    int cbi = 0x7fffffff;
    int nb = 0;                               // candidates gathered in cl (warp-uniform)
    auto evaluate = [&]() {
      __syncwarp();
      if (lane < nb) {
        const int s = cl[lane];
        const double c = exact_score<T>(A, xw, sq, s);
        if (c > cbest || (c == cbest && s < cbi)) { cbest = c; cbi = s; }
      }
      __syncwarp();
      nb = 0;
    };
    for (int j0 = 0; j0 < k; j0 += 32) {
      const int j = j0 + lane;
      bool mine = j < k && sw[j] >= thr;
      uint32_t m = __ballot_sync(0xffffffffu, mine);
      while (m) {
        const int take = min(__popc(m), 32 - nb);
        const int rank = __popc(m & ((1u << lane) - 1u));
        if (mine && rank < take) { cl[nb + rank] = j; mine = false; }
        nb += take;
        m = __ballot_sync(0xffffffffu, mine);
        if (nb == 32) evaluate();
      }
    }
    if (nb) evaluate();
    // warp argmax over (score, -slot)
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const double oc = __shfl_xor_sync(0xffffffffu, cbest, o);
      const int oi = __shfl_xor_sync(0xffffffffu, cbi, o);
      if (oc > cbest || (oc == cbest && oi < cbi)) { cbest = oc; cbi = oi; }
    }
    if (lane == 0 && cbi < k) tok[(int64_t)u * N + t] = (uint32_t)cbi;
    __syncwarp();
  }
}

template <typename T>
constexpr int refine_smem() {
  return kRefineWarps * (kRefineMaxK + kD + 32) * 4;
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
  // the lists are short (about 1% of rows) and uneven: a flat walk over all
  // of them, a few resident CTAs per SM
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const dim3 grid(3 * sms);
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
