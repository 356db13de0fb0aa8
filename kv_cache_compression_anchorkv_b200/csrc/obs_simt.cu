// Observation-window attention statistics (SIMT, fp32 accumulation).
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// "What carries the argument" and free parameter W: the last W queries of
// each query head attend over the prefill; their attention, pooled over the
// GQA heads of a KV head, scores every position (SnapKV-style, Eq. 14).  The
// residual utilities (Eq. 6 reading) need, per position t, sum_r alpha_rt,
// sum_r alpha_rt^2 and sum_r alpha_rt^2 ||q_r||^2 ||V_t - ybar_r||^2 with
// ybar_r the exact attention output of observation row r.
//
// Pass 1 (obs_pass1): per (KV head, 1024-token chunk, block of 128 rows), an
//   online softmax gives the chunk's row max m, sum l and unnormalised output.
// Combine (obs_combine): per row, M = max m, Z = sum l e^(m-M), ybar.
// Pass 2 (token_stats): per (KV head, 64-token tile), logits are recomputed,
//   alpha = e^(s-M)/Z, and the three per-position sums are formed in a fixed
//   order (deterministic).
// Row r = j*W + w of KV head h is query head h*G + j at window slot w; it sees
// positions t <= N - W + w.
#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

constexpr int kRowBlk = 128;     // observation rows per CTA
constexpr int kTokTile = 64;     // tokens per smem tile
constexpr int kKStride = 132;    // padded fp32 row stride of the token tiles
constexpr int kThreads = 256;    // 8 warps x 16 rows

struct ObsSmem {
  float q[kRowBlk][kD];          // observation rows (fp32)
  float x[kTokTile][kKStride];   // K tile
  float v[kTokTile][kKStride];   // V tile
  float p[8][16][kTokTile];      // per-warp softmax weights (pass 1) / scratch
};

template <typename T>
__device__ void load_rows(float (*dst)[kD], const T* src, int n_rows, int row_stride_elems) {
  for (int i = threadIdx.x; i < n_rows * (kD / 4); i += blockDim.x) {
    int r = i / (kD / 4), c = (i % (kD / 4)) * 4;
    float f[4];
    load4<T>(src + (int64_t)r * row_stride_elems + c, f);
    *reinterpret_cast<float4*>(&dst[r][c]) = make_float4(f[0], f[1], f[2], f[3]);
  }
}

template <typename T>
__device__ void load_tile(float (*dst)[kKStride], const T* src, int t0, int n_valid) {
  for (int i = threadIdx.x; i < kTokTile * (kD / 4); i += blockDim.x) {
    int r = i / (kD / 4), c = (i % (kD / 4)) * 4;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < n_valid) load4<T>(src + (int64_t)(t0 + r) * kD + c, f);
    *reinterpret_cast<float4*>(&dst[r][c]) = make_float4(f[0], f[1], f[2], f[3]);
  }
}

// Query rows of KV head h: Q_obs[h*G + j][w][:] for r = j*W + w.
template <typename T>
__device__ void load_q_block(ObsSmem& sm, const T* Q, int h, int G, int W, int r0, int nr) {
  for (int i = threadIdx.x; i < kRowBlk * (kD / 4); i += blockDim.x) {
    int r = i / (kD / 4), c = (i % (kD / 4)) * 4;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < nr) {
      int rr = r0 + r, j = rr / W, w = rr % W;
      load4<T>(Q + ((int64_t)(h * G + j) * W + w) * kD + c, f);
    }
    *reinterpret_cast<float4*>(&sm.q[r][c]) = make_float4(f[0], f[1], f[2], f[3]);
  }
}

// logits[i][u] for the warp's 16 rows and the lane's two tokens (lane, lane+32).
__device__ __forceinline__ void tile_logits(const ObsSmem& sm, int row0, float (&s)[16][2]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i][0] = s[i][1] = 0.f;
#pragma unroll 2
  for (int d = 0; d < kD; d += 4) {
    float4 k0 = *reinterpret_cast<const float4*>(&sm.x[lane][d]);
    float4 k1 = *reinterpret_cast<const float4*>(&sm.x[lane + 32][d]);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float4 q = *reinterpret_cast<const float4*>(&sm.q[row0 + i][d]);
      s[i][0] = fmaf(q.x, k0.x, fmaf(q.y, k0.y, fmaf(q.z, k0.z, fmaf(q.w, k0.w, s[i][0]))));
      s[i][1] = fmaf(q.x, k1.x, fmaf(q.y, k1.y, fmaf(q.z, k1.z, fmaf(q.w, k1.w, s[i][1]))));
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
obs_pass1_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ Q,
                 int N, int G, int W, int chunk, float* __restrict__ part_m,
                 float* __restrict__ part_l, float* __restrict__ part_y, int n_chunks) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ObsSmem& sm = *reinterpret_cast<ObsSmem*>(smem_raw);
  const int c = blockIdx.x, h = blockIdx.y, rb = blockIdx.z;
  const int GW = G * W;
  const int r0 = rb * kRowBlk, nr = min(kRowBlk, GW - r0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = warp * 16;
  const float scale = rsqrtf((float)kD);
  const T* Kh = K + (int64_t)h * N * kD;
  const T* Vh = V + (int64_t)h * N * kD;
  load_q_block<T>(sm, Q, h, G, W, r0, nr);

  float m[16], l[16], y[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    m[i] = -INFINITY; l[i] = 0.f;
    y[i][0] = y[i][1] = y[i][2] = y[i][3] = 0.f;
  }
  const int t_begin = c * chunk, t_end = min(N, t_begin + chunk);
  for (int t0 = t_begin; t0 < t_end; t0 += kTokTile) {
    const int nv = min(kTokTile, t_end - t0);
    __syncthreads();
    load_tile<T>(sm.x, Kh, t0, nv);
    load_tile<T>(sm.v, Vh, t0, nv);
    __syncthreads();
    float s[16][2];
    tile_logits(sm, row0, s);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int rr = r0 + row0 + i;
      const int limit = (rr < GW) ? (N - W + rr % W) : -1;   // last visible position
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = t0 + lane + 32 * u;
        s[i][u] = (lane + 32 * u < nv && t <= limit) ? s[i][u] * scale : -INFINITY;
      }
      float tm = warp_max(fmaxf(s[i][0], s[i][1]));
      float nm = fmaxf(m[i], tm);
      float corr = (nm == -INFINITY) ? 1.f : expf(m[i] - nm);
      float p0 = (s[i][0] == -INFINITY) ? 0.f : expf(s[i][0] - nm);
      float p1 = (s[i][1] == -INFINITY) ? 0.f : expf(s[i][1] - nm);
      l[i] = l[i] * corr + warp_sum(p0 + p1);
      m[i] = nm;
#pragma unroll
      for (int e = 0; e < 4; ++e) y[i][e] *= corr;
      sm.p[warp][i][lane] = p0;
      sm.p[warp][i][lane + 32] = p1;
    }
    __syncwarp();
    for (int t = 0; t < nv; t += 4) {
      float4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v4[u] = *reinterpret_cast<const float4*>(&sm.v[t + u][lane * 4]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float4 pp = *reinterpret_cast<const float4*>(&sm.p[warp][i][t]);
        float pv[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          y[i][0] = fmaf(pv[u], v4[u].x, y[i][0]);
          y[i][1] = fmaf(pv[u], v4[u].y, y[i][1]);
          y[i][2] = fmaf(pv[u], v4[u].z, y[i][2]);
          y[i][3] = fmaf(pv[u], v4[u].w, y[i][3]);
        }
      }
    }
    __syncwarp();
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int rr = r0 + row0 + i;
    if (rr >= GW) continue;
    const int64_t pi = ((int64_t)h * n_chunks + c) * GW + rr;
    if (lane == 0) { part_m[pi] = m[i]; part_l[pi] = l[i]; }
    *reinterpret_cast<float4*>(&part_y[pi * kD + lane * 4]) = make_float4(y[i][0], y[i][1], y[i][2], y[i][3]);
  }
}

// One warp per observation row: merge the chunk partials in chunk order.
__global__ void obs_combine_kernel(const float* __restrict__ part_m, const float* __restrict__ part_l,
                                   const float* __restrict__ part_y, int H, int GW, int n_chunks,
                                   float* __restrict__ row_m, float* __restrict__ row_z,
                                   float* __restrict__ ybar) {
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= H * GW) return;
  const int h = gw / GW, r = gw % GW;
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, part_m[((int64_t)h * n_chunks + c) * GW + r]);
  float Z = 0.f, y[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c = 0; c < n_chunks; ++c) {
    const int64_t pi = ((int64_t)h * n_chunks + c) * GW + r;
    const float mc = part_m[pi];
    if (mc == -INFINITY) continue;
    const float f = expf(mc - M);
    Z = fmaf(part_l[pi], f, Z);
    float4 py = *reinterpret_cast<const float4*>(&part_y[pi * kD + lane * 4]);
    y[0] = fmaf(py.x, f, y[0]); y[1] = fmaf(py.y, f, y[1]);
    y[2] = fmaf(py.z, f, y[2]); y[3] = fmaf(py.w, f, y[3]);
  }
  const float inv = 1.f / Z;
  if (lane == 0) { row_m[gw] = M; row_z[gw] = Z; }
  *reinterpret_cast<float4*>(&ybar[(int64_t)gw * kD + lane * 4]) =
      make_float4(y[0] * inv, y[1] * inv, y[2] * inv, y[3] * inv);
}

struct StatSmem {
  float q[kRowBlk][kD];
  float yb[kRowBlk][kD];
  float x[kTokTile][kKStride];
  float v[kTokTile][kKStride];
  float q2[kRowBlk], M[kRowBlk], invZ[kRowBlk];
  float red[8][3][kTokTile];
};

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
token_stats_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ Q,
                   int N, int G, int W, const float* __restrict__ row_m, const float* __restrict__ row_z,
                   const float* __restrict__ ybar, float* __restrict__ score, float* __restrict__ a2s,
                   float* __restrict__ kus, float* __restrict__ xnorm, int H) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  StatSmem& sm = *reinterpret_cast<StatSmem*>(smem_raw);
  const int h = blockIdx.y;
  const int t0 = blockIdx.x * kTokTile, nv = min(kTokTile, N - t0);
  const int GW = G * W;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = warp * 16;
  const float scale = rsqrtf((float)kD);
  load_tile<T>(sm.x, K + (int64_t)h * N * kD, t0, nv);
  load_tile<T>(sm.v, V + (int64_t)h * N * kD, t0, nv);
  __syncthreads();
  if (threadIdx.x < 2 * kTokTile) {
    // row norms of the keys and values (fp32), used by the assignment's
    // error bound
    const int t = threadIdx.x % kTokTile, side = threadIdx.x / kTokTile;
    const float* rowp = side ? sm.v[t] : sm.x[t];
    float s2 = 0.f;
    for (int d = 0; d < kD; ++d) s2 = fmaf(rowp[d], rowp[d], s2);
    if (t < nv) xnorm[((int64_t)side * H + h) * N + t0 + t] = sqrtf(s2);
  }
  float acc[3][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
  for (int r0 = 0; r0 < GW; r0 += kRowBlk) {
    const int nr = min(kRowBlk, GW - r0);
    __syncthreads();
    // ObsSmem-compatible view for the shared logits helper
    for (int i = threadIdx.x; i < kRowBlk * (kD / 4); i += blockDim.x) {
      int r = i / (kD / 4), cc = (i % (kD / 4)) * 4;
      float f[4] = {0.f, 0.f, 0.f, 0.f};
      float g[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < nr) {
        int rr = r0 + r, j = rr / W, w = rr % W;
        load4<T>(Q + ((int64_t)(h * G + j) * W + w) * kD + cc, f);
        float4 yy = *reinterpret_cast<const float4*>(&ybar[((int64_t)h * GW + rr) * kD + cc]);
        g[0] = yy.x; g[1] = yy.y; g[2] = yy.z; g[3] = yy.w;
      }
      *reinterpret_cast<float4*>(&sm.q[r][cc]) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4*>(&sm.yb[r][cc]) = make_float4(g[0], g[1], g[2], g[3]);
    }
    if (threadIdx.x < kRowBlk) {
      const int r = threadIdx.x;
      sm.M[r] = (r < nr) ? row_m[(int64_t)h * GW + r0 + r] : 0.f;
      sm.invZ[r] = (r < nr) ? 1.f / row_z[(int64_t)h * GW + r0 + r] : 0.f;
    }
    __syncthreads();
    if (threadIdx.x < kRowBlk) {
      float s = 0.f;
      for (int d = 0; d < kD; ++d) s = fmaf(sm.q[threadIdx.x][d], sm.q[threadIdx.x][d], s);
      sm.q2[threadIdx.x] = s;
    }
    __syncthreads();
    // logits and squared distances for 16 rows x 2 tokens
    float s[16][2], dist[16][2];
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i][0] = s[i][1] = dist[i][0] = dist[i][1] = 0.f;
#pragma unroll 1
    for (int d = 0; d < kD; d += 4) {
      float4 k0 = *reinterpret_cast<const float4*>(&sm.x[lane][d]);
      float4 k1 = *reinterpret_cast<const float4*>(&sm.x[lane + 32][d]);
      float4 v0 = *reinterpret_cast<const float4*>(&sm.v[lane][d]);
      float4 v1 = *reinterpret_cast<const float4*>(&sm.v[lane + 32][d]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float4 q = *reinterpret_cast<const float4*>(&sm.q[row0 + i][d]);
        float4 yb = *reinterpret_cast<const float4*>(&sm.yb[row0 + i][d]);
        s[i][0] = fmaf(q.x, k0.x, fmaf(q.y, k0.y, fmaf(q.z, k0.z, fmaf(q.w, k0.w, s[i][0]))));
        s[i][1] = fmaf(q.x, k1.x, fmaf(q.y, k1.y, fmaf(q.z, k1.z, fmaf(q.w, k1.w, s[i][1]))));
        float a0 = v0.x - yb.x, a1 = v0.y - yb.y, a2 = v0.z - yb.z, a3 = v0.w - yb.w;
        float b0 = v1.x - yb.x, b1 = v1.y - yb.y, b2 = v1.z - yb.z, b3 = v1.w - yb.w;
        dist[i][0] = fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, fmaf(a3, a3, dist[i][0]))));
        dist[i][1] = fmaf(b0, b0, fmaf(b1, b1, fmaf(b2, b2, fmaf(b3, b3, dist[i][1]))));
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = row0 + i;
      if (r >= nr) continue;
      const int rr = r0 + r;
      const int limit = N - W + rr % W;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = t0 + lane + 32 * u;
        float a = 0.f;
        if (lane + 32 * u < nv && t <= limit) a = expf(s[i][u] * scale - sm.M[r]) * sm.invZ[r];
        const float aa = a * a;
        acc[0][u] += a;
        acc[1][u] += aa;
        acc[2][u] = fmaf(aa * sm.q2[r], dist[i][u], acc[2][u]);
      }
    }
  }
  // reduce the 8 warps' partial sums per token in warp order
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int st = 0; st < 3; ++st) sm.red[warp][st][lane + 32 * u] = acc[st][u];
  __syncthreads();
  if (threadIdx.x < kTokTile && threadIdx.x < nv) {
    const int t = threadIdx.x;
    float o[3] = {0.f, 0.f, 0.f};
    for (int w8 = 0; w8 < 8; ++w8)
      for (int st = 0; st < 3; ++st) o[st] += sm.red[w8][st][t];
    const int64_t gi = (int64_t)h * N + t0 + t;
    score[gi] = o[0];
    a2s[gi] = o[1];
    kus[gi] = o[2];
  }
}

}  // namespace

cudaError_t launch_obs_pass1(const Plan& pl, const void* K, const void* V, const void* Q, char* ws, cudaStream_t s) {
  dim3 grid(pl.n_chunk1, pl.H, (pl.GW + kRowBlk - 1) / kRowBlk);
  const size_t smem = sizeof(ObsSmem);
  float* pm = reinterpret_cast<float*>(ws + pl.o_part_m);
  float* plx = reinterpret_cast<float*>(ws + pl.o_part_l);
  float* py = reinterpret_cast<float*>(ws + pl.o_part_y);
  if (pl.p.dtype == ANCHORKV_BF16) {
    auto k = obs_pass1_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>((const __nv_bfloat16*)K, (const __nv_bfloat16*)V, (const __nv_bfloat16*)Q,
                                   pl.N, pl.G, pl.W, pl.chunk1, pm, plx, py, pl.n_chunk1);
  } else {
    auto k = obs_pass1_kernel<float>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>((const float*)K, (const float*)V, (const float*)Q,
                                   pl.N, pl.G, pl.W, pl.chunk1, pm, plx, py, pl.n_chunk1);
  }
  return cudaGetLastError();
}

cudaError_t launch_obs_combine(const Plan& pl, char* ws, cudaStream_t s) {
  const int rows = pl.H * pl.GW;
  obs_combine_kernel<<<(rows + 7) / 8, 256, 0, s>>>(
      reinterpret_cast<const float*>(ws + pl.o_part_m), reinterpret_cast<const float*>(ws + pl.o_part_l),
      reinterpret_cast<const float*>(ws + pl.o_part_y), pl.H, pl.GW, pl.n_chunk1,
      reinterpret_cast<float*>(ws + pl.o_row_m), reinterpret_cast<float*>(ws + pl.o_row_z),
      reinterpret_cast<float*>(ws + pl.o_ybar));
  return cudaGetLastError();
}

cudaError_t launch_token_stats(const Plan& pl, const void* K, const void* V, const void* Q, char* ws, cudaStream_t s) {
  dim3 grid((pl.N + kTokTile - 1) / kTokTile, pl.H);
  const size_t smem = sizeof(StatSmem);
  auto* rm = reinterpret_cast<const float*>(ws + pl.o_row_m);
  auto* rz = reinterpret_cast<const float*>(ws + pl.o_row_z);
  auto* yb = reinterpret_cast<const float*>(ws + pl.o_ybar);
  auto* sc = reinterpret_cast<float*>(ws + pl.o_score);
  auto* a2 = reinterpret_cast<float*>(ws + pl.o_a2);
  auto* ku = reinterpret_cast<float*>(ws + pl.o_ku);
  auto* xn = reinterpret_cast<float*>(ws + pl.o_xnorm);
  if (pl.p.dtype == ANCHORKV_BF16) {
    auto k = token_stats_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>((const __nv_bfloat16*)K, (const __nv_bfloat16*)V, (const __nv_bfloat16*)Q,
                                   pl.N, pl.G, pl.W, rm, rz, yb, sc, a2, ku, xn, pl.H);
  } else {
    auto k = token_stats_kernel<float>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>((const float*)K, (const float*)V, (const float*)Q,
                                   pl.N, pl.G, pl.W, rm, rz, yb, sc, a2, ku, xn, pl.H);
  }
  return cudaGetLastError();
}

}  // namespace akv
