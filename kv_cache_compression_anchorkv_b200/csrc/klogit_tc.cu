// Key-residual logits of a batch of compressed layers on the 5th-generation
// tensor cores (kind::i8), computed ahead of the slice decode.
//
// "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science review),
// Referee "Summary": the decoder rebuilds K^ = gamma K_a + r~ when it is
// consumed.  The rebuilt key's residual enters a logit as
//   q' . r~_t = sigma~_t <qr, lev(c_t)>,   qr = H(s . q') / sqrt(D)
// (q' the query in log2 units, H the Sylvester matrix, s the shared signs;
// qr = q' for the unrotated codec).  The four Lloyd-Max levels are affine in
// the two bits of a code, u = bit 1 and v = bit 0:
//   lev(c) = -l2 + (l1 + l2) u + (l2 - l1) v,
// so <qr, lev(c)> = -l2 sum_j qr_j + (l1 + l2) <u, qr> + (l2 - l1) <v, qr>,
// and <u, qr>, <v, qr> are exact integer contractions once qr is held in
// fixed point: qr_j ~ s Q_j with Q_j in [-2^26, 2^26], written as four
// balanced base-128 digits Q_j = d0 2^21 + d1 2^14 + d2 2^7 + d3, d in
// [-64, 63] (the fixed-point error is 2^-27 of max_j |qr_j| per coordinate).
//
// One CTA of 128 threads takes 128-record tiles of one (sequence, head):
// each thread (one record = one tensor-memory lane) turns its 32 code bytes
// into the u and v bit planes (one byte 0/1 per coordinate, the coordinates
// permuted within every 16 so that one shift and one mask make four of them;
// the query digits use the same permutation) and stores them to tensor
// memory; one thread issues
//   D[record][(g, digit)] = sum_j plane[record][j] digit[(g, digit)][j]
// for both planes as tcgen05.mma kind::i8 (A = planes from tensor memory,
// B = digits from shared memory, 128-byte swizzle, int32 accumulators); the
// threads read D back, recombine the digits in fp32 and write
// sigma~ * <qr, lev(c)> per query head.  Every wait is bounded: on a timeout
// the tile's logits are written as NaN and the CTA moves on.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace akv {
namespace {

constexpr int kThr = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTmemCols = 128;     // A planes (64 columns) + D (2 x up to 32 columns)

struct KArgs {
  const uint8_t* comp;
  int64_t stride;
  int64_t off_tok_pf, off_codes, off_sig;
  int H, G, n_tiles;
  int64_t R;
  float lev[4];
  uint32_t sign_bits[4];
  int naive;
  const void* q;
  float* out;           // [batch][R][GP] logits of key records (value-record rows unused)
  int P;                // CTAs per (sequence, head)
};

__host__ __device__ constexpr int kgp_of(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

// Rows of the digit operand: (g, digit) for GP heads, at least 16 (N of one
// instruction is a multiple of 16).
__host__ __device__ constexpr int nb_of(int GP) { return GP * 4 < 16 ? 16 : GP * 4; }

// Instruction descriptor, kind::i8: A unsigned 8-bit, B signed 8-bit, both
// K-major, int32 accumulator, M x N.
__host__ __device__ constexpr uint32_t idesc_u8s8_s32(int M, int N) {
  return (2u << 4)                      // D format: s32
         | (0u << 7)                    // A format: unsigned 8-bit
         | (1u << 10)                   // B format: signed 8-bit
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit words: thread i of the warp writes its lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Coordinate of plane position p (0..127): within each group of 16 the two
// 2-bit fields swap, p = 16w + 4k + i  <->  j = 16w + 4i + k.
__host__ __device__ inline int perm16(int p) { return (p & ~15) | ((p & 3) << 2) | ((p >> 2) & 3); }

struct KSmem {
  uint8_t B[8 * 128 * 4];            // digits, [NB rows][128 bytes], 128-byte swizzle (NB <= 32)
  uint64_t bar;
  uint32_t tmem;
  float s[8], xq[8];                 // fixed-point step and sum_j s Q_j per head
  float qs[8][128];                  // query in log2 units, then rotated
  float amax[8];
};

template <typename T, int GP>
__global__ void __launch_bounds__(kThr) klogit_tc_kernel(KArgs a) {
  extern __shared__ __align__(1024) unsigned char ksm_raw[];
  KSmem& sm = *reinterpret_cast<KSmem*>(
      (reinterpret_cast<uintptr_t>(ksm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int NB = nb_of(GP);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const uint8_t* comp = a.comp + (int64_t)b * a.stride;
  const int* pf = reinterpret_cast<const int*>(comp + a.off_tok_pf);
  // key records of (b, h): [r0, r1)
  int64_t r0 = pf[(int64_t)h * (a.n_tiles + 1)], r1 = pf[(int64_t)h * (a.n_tiles + 1) + a.n_tiles];
  r0 = r0 < 0 ? 0 : (r0 > a.R ? a.R : r0);
  r1 = r1 < r0 ? r0 : (r1 > a.R ? a.R : r1);
  const int n_tiles_rec = (int)((r1 - r0 + 127) / 128);
  if ((int)blockIdx.x >= n_tiles_rec) return;      // uniform across the CTA

  // ---- query: log2 units, rotated; fixed-point digits into the B operand
  const T* q = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.H * a.G + (int64_t)h * a.G) * kD;
  const float qscale = kLog2e * rsqrtf((float)kD);
  for (int i = tid; i < GP * kD; i += kThr) {
    const int g = i / kD;
    sm.qs[g][i % kD] = g < a.G ? to_f(q[(int64_t)g * kD + (i % kD)]) * qscale : 0.f;
  }
  if (warp == 0) {
    tc::tmem_alloc(&sm.tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(&sm.bar, 1);
    tc::fence_barrier_init();
  }
  for (int i = tid; i < NB * 128; i += kThr) sm.B[i] = 0;
  __syncthreads();
  for (int g = warp; g < GP; g += kThr / 32) {
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = sm.qs[g][4 * lane + i];
    if (!a.naive) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int d = 4 * lane + i;
        if ((a.sign_bits[d >> 5] >> (d & 31)) & 1u) v[i] = -v[i];
      }
      fwht128(v);
      const float r = rsqrtf((float)kD);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] *= r;
    }
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    m = warp_max(m);
#pragma unroll
    for (int i = 0; i < 4; ++i) sm.qs[g][4 * lane + i] = v[i];
    if (lane == 0) sm.amax[g] = m;
  }
  __syncthreads();
  // digits: Q_j = rint(qr_j / s), s = max|qr| / 2^26
  for (int i = tid; i < GP * kD; i += kThr) {
    const int g = i / kD, j = i % kD;
    const float am = sm.amax[g];
    const float s = am > 0.f ? am * (1.0f / 67108864.0f) : 1.0f;
    int Q = am > 0.f ? __float2int_rn(sm.qs[g][j] / s) : 0;
    Q = max(-(1 << 26), min(1 << 26, Q));
    int d[4];
#pragma unroll
    for (int p = 3; p >= 1; --p) {
      const int lo = ((Q + 64) & 127) - 64;
      d[p] = lo;
      Q = (Q - lo) >> 7;
    }
    d[0] = Q;
    // plane position of coordinate j (the permutation is its own inverse)
    const int pos = perm16(j);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int n = g * 4 + p;
      const int off = (n >> 3) * 1024 + (n & 7) * 128 + ((((pos >> 4) ^ (n & 7)) & 7) << 4) + (pos & 15);
      sm.B[off] = (uint8_t)(int8_t)d[p];
    }
  }
  __syncthreads();
  // per-head step and sum_j s Q_j (from the digits, so both terms use the same fixed point)
  for (int g = warp; g < GP; g += kThr / 32) {
    const float am = sm.amax[g];
    const float s = am > 0.f ? am * (1.0f / 67108864.0f) : 1.0f;
    double acc = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 4 * lane + i, pos = perm16(j);
      int64_t Q = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int n = g * 4 + p;
        const int off = (n >> 3) * 1024 + (n & 7) * 128 + ((((pos >> 4) ^ (n & 7)) & 7) << 4) + (pos & 15);
        Q = Q * 128 + (int8_t)sm.B[off];
      }
      acc += (double)Q;
    }
    acc = warp_sum_d(acc);
    if (lane == 0) {
      sm.s[g] = s;
      sm.xq[g] = (float)(acc * (double)s);
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  const uint32_t tmem = sm.tmem;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t colA = 0, colD = 64;
  constexpr uint32_t idesc = idesc_u8s8_s32(128, NB);
  const uint32_t bbase = tc::smem_u32(sm.B);
  const float l1 = a.lev[2], l2 = a.lev[3];
  const float cu = l1 + l2, cv = l2 - l1;
  const uint8_t* codes = comp + a.off_codes;
  const uint16_t* sig = reinterpret_cast<const uint16_t*>(comp + a.off_sig);
  float* out = a.out + (int64_t)b * a.R * GP;
  uint32_t phase = 0;
  bool failed = false;

  for (int t = blockIdx.x; t < n_tiles_rec; t += a.P) {
    const int64_t r = r0 + (int64_t)t * 128 + tid;
    const bool valid = r < r1;
    uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + r * kCodeBytes);
      c0 = src[0];
      c1 = src[1];
    }
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    // planes: word 4w + k holds the bit of coordinates 16w + 4i + k, i = 0..3
    uint32_t pu[32], pv[32];
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pu[4 * w + k] = (cw[w] >> (2 * k + 1)) & 0x01010101u;
        pv[4 * w + k] = (cw[w] >> (2 * k)) & 0x01010101u;
      }
    tmem_st32(tmem + lane_base + colA, pu);
    tmem_st32(tmem + lane_base + colA + 32, pv);
    tmem_wait_st();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && !failed) {
      tc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bd = tc::sw128_desc(bbase + (uint32_t)ks * 32u);
        mma_i8_ts(tmem + colD, tmem + colA + (uint32_t)ks * 8u, bd, idesc, ks > 0 ? 1u : 0u);
        mma_i8_ts(tmem + colD + NB, tmem + colA + 32u + (uint32_t)ks * 8u, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(&sm.bar);
    }
    // the MMAs of a tile are issued only while nothing has failed, so after a
    // timeout no new work reaches the tensor core
    bool ok = false;
    if (!failed) {
      ok = tc::mbar_wait(&sm.bar, phase);
      phase ^= 1u;
    }
    if (!ok) failed = true;
    tc::fence_after_sync();
    // D row of this record: NB u-columns then NB v-columns
    uint32_t du[16], dv[16];
    float lg[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) lg[g] = 0.f;
#pragma unroll
    for (int c16 = 0; c16 < NB / 16; ++c16) {
      tc::tmem_ld16(tmem + lane_base + colD + (uint32_t)(c16 * 16), du);
      tc::tmem_ld16(tmem + lane_base + colD + NB + (uint32_t)(c16 * 16), dv);
      tc::tmem_wait_ld_dep2(du, dv);
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        const int g = c16 * 4 + g4;
        if (g < GP) {
          const float su = (float)(int)du[g4 * 4] * 2097152.0f + (float)(int)du[g4 * 4 + 1] * 16384.0f +
                           (float)(int)du[g4 * 4 + 2] * 128.0f + (float)(int)du[g4 * 4 + 3];
          const float sv = (float)(int)dv[g4 * 4] * 2097152.0f + (float)(int)dv[g4 * 4 + 1] * 16384.0f +
                           (float)(int)dv[g4 * 4 + 2] * 128.0f + (float)(int)dv[g4 * 4 + 3];
          lg[g] = sm.s[g] * (cu * su + cv * sv) - l2 * sm.xq[g];
        }
      }
    }
    if (valid) {
      const float sg = half_bits_to_f(sig[r]);
#pragma unroll
      for (int g = 0; g < GP; ++g) out[r * GP + g] = failed ? __int_as_float(0x7fc00000) : lg[g] * sg;
    }
    tc::fence_before_sync();
    __syncthreads();      // D and the planes are free for the next tile
  }
  // a tile whose wait timed out may still have its MMAs in flight: wait once
  // more (bounded) before the columns are freed
  if (failed) tc::mbar_wait(&sm.bar, phase);
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

template <typename T, int GP>
int launch_t(const KArgs& a, int batch, int H, cudaStream_t s) {
  static int ready_dev = -1;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ANCHORKV_ECUDA;
  // shared memory sized for at most four resident CTAs per SM, which is what
  // the 512 tensor-memory columns hold at 128 columns each
  const int smem = std::max((int)sizeof(KSmem) + 1024, 50 * 1024);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (ready_dev != dev) {
      if (cudaFuncSetAttribute(klogit_tc_kernel<T, GP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
        return ANCHORKV_ECUDA;
      ready_dev = dev;
    }
  }
  klogit_tc_kernel<T, GP><<<dim3(a.P, batch * H), kThr, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? ANCHORKV_OK : ANCHORKV_ECUDA;
}

}  // namespace

bool klogit_tc_supported(const Plan& pl) { return pl.G <= 8; }

int64_t klogit_ws_bytes(const Plan& pl, int batch) {
  return (int64_t)batch * std::max<int64_t>(pl.R, 1) * kgp_of(pl.G) * 4;
}

int launch_klogit_tc(const Plan& pl, int batch, const char* comp, int64_t stride, const void* q, float* out,
                     cudaStream_t s) {
  KArgs a;
  a.comp = reinterpret_cast<const uint8_t*>(comp);
  a.stride = stride;
  a.off_tok_pf = pl.L.off_tile_prefix;
  a.off_codes = pl.L.off_res_codes;
  a.off_sig = pl.L.off_res_sigma;
  a.H = pl.H; a.G = pl.G; a.n_tiles = pl.n_tiles;
  a.R = pl.R;
  a.lev[0] = (float)-pl.l2; a.lev[1] = (float)-pl.l1; a.lev[2] = (float)pl.l1; a.lev[3] = (float)pl.l2;
  for (int i = 0; i < 4; ++i) a.sign_bits[i] = pl.sign_bits[i];
  a.naive = naive_codec(pl);
  a.q = q;
  a.out = out;
  // about four CTAs per SM over the whole launch; a (sequence, head) has at
  // most N - k key records
  const int units = std::max(1, batch * pl.H);
  const int max_tiles = std::max(1, (pl.N + 127) / 128);
  a.P = std::max(1, std::min(max_tiles, (4 * 148 + units - 1) / units));
  const int GP = kgp_of(pl.G);
  stage_begin(kStDecodePrep, s);
  int st;
  if (pl.p.dtype == ANCHORKV_BF16) {
    using T = __nv_bfloat16;
    st = GP == 1 ? launch_t<T, 1>(a, batch, pl.H, s) : GP == 2 ? launch_t<T, 2>(a, batch, pl.H, s)
       : GP == 4 ? launch_t<T, 4>(a, batch, pl.H, s) : launch_t<T, 8>(a, batch, pl.H, s);
  } else {
    using T = float;
    st = GP == 1 ? launch_t<T, 1>(a, batch, pl.H, s) : GP == 2 ? launch_t<T, 2>(a, batch, pl.H, s)
       : GP == 4 ? launch_t<T, 4>(a, batch, pl.H, s) : launch_t<T, 8>(a, batch, pl.H, s);
  }
  stage_end(kStDecodePrep, s, 1);
  return st;
}

}  // namespace akv
