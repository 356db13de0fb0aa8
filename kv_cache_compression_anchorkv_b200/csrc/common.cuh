// Device helpers shared by the AnchorKV kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/anchorkv.h"

namespace akv {

constexpr int kD = 128;          // head_dim supported by every kernel
constexpr int kTile = 128;       // token tile of the residual bitmap / prefix table
constexpr int kCodeBytes = kD / 4;

// Counter slots in the compress workspace (int32 at offset 0): 16 scalar
// counters, then one re-decision list length per (side, head).
enum Counter {
  kStatus = 0,        // non-zero: a device-side check failed (code below)
  kRefineRows = 1,    // nearest-anchor rows re-decided in fp64
  kSelectTies = 2,    // token-sides whose utility equals the selection threshold
  kRefineOverflow = 3,
  kUniformRetries = 4,
  kCounterCount = 16,
  kRefineListBase = 16
};
enum DeviceError { kDevErrNone = 0, kDevErrUniform = 1, kDevErrRefine = 2, kDevErrBounds = 3, kDevErrTimeout = 4 };

__device__ __forceinline__ void latch_error(int* counters, int code) {
  atomicCAS(&counters[kStatus], 0, code);
}

// Salt of the random residual ranking ("rank_rnd"), keeping its keys apart
// from the uniform anchor sample's.
constexpr uint64_t kRankSalt = 0x72616E6B5F726E64ull;

// SplitMix64 output for state x (Steele, Lea & Flood, OOPSLA 2014).
__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t anchor_key(uint64_t seed, int layer, int head, int t) {
  return splitmix64(seed ^ ((uint64_t)layer << 48) ^ ((uint64_t)head << 32) ^ (uint64_t)(uint32_t)t);
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Four consecutive elements starting at p (16-byte aligned for float, 8 for bf16).
template <typename T> __device__ __forceinline__ void load4(const T* p, float (&o)[4]);
template <> __device__ __forceinline__ void load4<float>(const float* p, float (&o)[4]) {
  float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <> __device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&o)[4]) {
  uint2 v = *reinterpret_cast<const uint2*>(p);
  o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xFFFF0000u);
  o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xFFFF0000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Running best, second and third score of a row with the slots of the first
// two; slots are pushed in ascending order, so strict comparisons keep the
// lowest slot among equal scores.
struct Top3 {
  float b1, b2, b3;
  int i1, i2;
};

__device__ __forceinline__ Top3 top3_init() { return Top3{-INFINITY, -INFINITY, -INFINITY, 0x7fffffff, 0x7fffffff}; }

__device__ __forceinline__ void push(Top3& b, float v, int i) {
  if (v > b.b1) { b.b3 = b.b2; b.b2 = b.b1; b.i2 = b.i1; b.b1 = v; b.i1 = i; }
  else if (v > b.b2) { b.b3 = b.b2; b.b2 = v; b.i2 = i; }
  else if (v > b.b3) { b.b3 = v; }
}

__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ Top3 merge(const Top3& a, const Top3& b) {
  const bool a_wins = before(a.b1, a.i1, b.b1, b.i1);
  const Top3& w = a_wins ? a : b;
  const Top3& l = a_wins ? b : a;
  Top3 r;
  r.b1 = w.b1; r.i1 = w.i1;
  if (before(l.b1, l.i1, w.b2, w.i2)) { r.b2 = l.b1; r.i2 = l.i1; r.b3 = fmaxf(w.b2, l.b2); }
  else { r.b2 = w.b2; r.i2 = w.i2; r.b3 = fmaxf(w.b3, l.b1); }
  return r;
}

// Lists token t of (side, head) u (= side * H + head) for the fp64
// re-decision of its nearest anchor; list u holds up to N tokens.
__device__ __forceinline__ void list_for_refine(int* refine, int* counters, int u, int N, int t) {
  const int at = atomicAdd(&counters[kRefineListBase + u], 1);
  refine[(int64_t)u * N + at] = t;
  atomicAdd(&counters[kRefineRows], 1);
}

// fp16 (IEEE half) round-to-nearest-even of a double, saturating at +-65504.
__device__ __forceinline__ uint16_t half_bits_rn(double v) {
  v = fmin(fmax(v, -65504.0), 65504.0);
  return __half_as_ushort(__double2half(v));
}
__device__ __forceinline__ float half_bits_to_f(uint32_t bits16) {
  return __half2float(__ushort_as_half((unsigned short)bits16));
}

// In-warp Walsh-Hadamard transform (unnormalised: the Sylvester matrix of
// +-1 entries) of a 128-vector held as 4 consecutive coordinates per lane
// (lane l owns 4l..4l+3), natural order.
template <typename F>
__device__ __forceinline__ void fwht128(F (&v)[4]) {
  F a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2; v[2] = a0 - a2; v[1] = a1 + a3; v[3] = a1 - a3;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = lane & m;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      F other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (other - v[i]) : (v[i] + other);
    }
  }
}

// Transposed butterfly: on entry lane l holds 32 partial values v[i]; on
// exit v[0] of lane l is the sum over lanes of value l (31 shuffles).
__device__ __forceinline__ void transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float keep = up ? v[i + off] : v[i];
      const float send = up ? v[i] : v[i + off];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
}

}  // namespace akv
