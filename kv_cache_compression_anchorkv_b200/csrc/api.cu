// C-ABI entry points: parameter checks, the byte accounting, workspace plans
// and the launch sequence of one compress / decode call.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace akv {

// Four-level Lloyd-Max quantizer for N(0,1) by Lloyd's fixed-point iteration:
// thresholds at the midpoints of neighbouring levels, levels at the
// conditional means of their cells (symmetric: cells split at 0 and +-tau).
void codebook(double* tau_out, double* l1_out, double* l2_out, double* mse_out) {
  static double c[4];
  static std::once_flag once;
  std::call_once(once, [] {
    const double inv_sqrt_2pi = 0.3989422804014327;
    auto pdf = [&](double x) { return inv_sqrt_2pi * exp(-0.5 * x * x); };
    auto upper = [](double x) { return 0.5 * erfc(x / sqrt(2.0)); };   // P(X >= x)
    double a = 0.4, b = 1.6;
    for (int it = 0; it < 100000; ++it) {
      const double t = 0.5 * (a + b);
      const double na = (pdf(0.0) - pdf(t)) / (0.5 - upper(t));
      const double nb = pdf(t) / upper(t);
      const bool done = fabs(na - a) < 1e-15 && fabs(nb - b) < 1e-15;
      a = na;
      b = nb;
      if (done) break;
    }
    const double t = 0.5 * (a + b);
    const double pin = 0.5 - upper(t), pout = upper(t);
    c[0] = t; c[1] = a; c[2] = b;
    c[3] = 1.0 - 2.0 * (pin * a * a + pout * b * b);
  });
  if (tau_out) *tau_out = c[0];
  if (l1_out) *l1_out = c[1];
  if (l2_out) *l2_out = c[2];
  if (mse_out) *mse_out = c[3];
}

static int64_t align16(int64_t x) { return (x + 15) / 16 * 16; }

static int fill_layout(const anchorkv_params* p, anchorkv_layout* L, int* n_s, int* n_u, bool* all) {
  const int64_t N = p->n_tokens, H = p->n_kv_heads, D = p->head_dim, W = p->window;
  const int64_t e = p->dtype == ANCHORKV_BF16 ? 2 : 4;
  const int64_t m = (N + p->anchor_div - 1) / p->anchor_div;
  int64_t k;
  if (N - W <= m) {
    k = N; *n_s = 0; *n_u = 0; *all = true;
  } else {
    k = W + m;
    *n_s = (int)((p->rho_num * m) / p->rho_den);
    *n_u = (int)(m - *n_s);
    *all = false;
  }
  if (k > 65535) return ANCHORKV_EINVAL;          // slots are 16-bit (b_a = 2 bytes)
  const int64_t n_t = (N + kTile - 1) / kTile;
  memset(L, 0, sizeof(*L));
  int64_t cur = 0;
  L->off_anchors_k = cur; cur = align16(cur + H * k * D * e);
  L->off_anchors_v = cur; cur = align16(cur + H * k * D * e);
  L->off_anchor_pos = cur; cur = align16(cur + 4 * H * k);
  L->off_tok = cur; cur = align16(cur + 4 * 2 * H * N);
  L->off_bitmap = cur; cur = align16(cur + 2 * H * n_t * 16);
  L->off_tile_prefix = cur; cur = align16(cur + 4 * 2 * H * (n_t + 1));
  L->base_bytes = cur;
  L->residual_bytes_each = D * 2 / 8 + 2;
  L->uncompressed_bytes = 2 * H * N * D * e;
  L->budget_bytes = (int64_t)floor(p->theta * (double)L->uncompressed_bytes);
  L->residual_cap = 2 * H * (N - k);
  int64_t r = (L->budget_bytes - L->base_bytes) / L->residual_bytes_each;
  if (L->budget_bytes < L->base_bytes) r = 0;
  L->n_residuals = std::min(L->residual_cap, std::max<int64_t>(0, r));
  L->off_res_codes = L->base_bytes;
  L->off_res_sigma = L->base_bytes + (D / 4) * L->n_residuals;
  L->total_bytes = L->base_bytes + L->residual_bytes_each * L->n_residuals;
  L->n_anchors = (int32_t)k;
  L->n_scored = *n_s;
  L->n_uniform = *n_u;
  L->n_tiles = (int32_t)n_t;
  return ANCHORKV_OK;
}

static int validate(const anchorkv_params* p) {
  if (!p) return ANCHORKV_EINVAL;
  if (p->head_dim != kD) return ANCHORKV_EUNSUPPORTED;
  if (p->dtype != ANCHORKV_FP32 && p->dtype != ANCHORKV_BF16) return ANCHORKV_EUNSUPPORTED;
  if (p->n_kv_heads < 1 || p->n_kv_heads > 65535) return ANCHORKV_EINVAL;
  if (p->n_q_heads < p->n_kv_heads || p->n_q_heads % p->n_kv_heads) return ANCHORKV_EINVAL;
  if (p->n_q_heads / p->n_kv_heads > 16) return ANCHORKV_EUNSUPPORTED;
  if (p->window < 1 || p->window > 256) return ANCHORKV_EINVAL;
  if (p->n_tokens <= p->window || p->n_tokens > (1 << 20)) return ANCHORKV_EINVAL;
  if (!(p->theta > 0.0) || !isfinite(p->theta)) return ANCHORKV_EINVAL;
  if (p->anchor_div < 1 || p->rho_den < 1 || p->rho_num < 0 || p->rho_num > p->rho_den) return ANCHORKV_EINVAL;
  if (p->pool_kernel < 1 || !(p->pool_kernel & 1) || p->pool_kernel > 255) return ANCHORKV_EINVAL;
  if (p->layer < 0 || p->layer > 32767) return ANCHORKV_EINVAL;
  if (p->mode & ~ANCHORKV_MODE_ALL) return ANCHORKV_EINVAL;
  if (((p->mode & ANCHORKV_MODE_RANK_MASK) >> ANCHORKV_MODE_RANK_SHIFT) > ANCHORKV_RANK_RANDOM) return ANCHORKV_EINVAL;
  if ((int64_t)2 * p->n_kv_heads * p->n_tokens > (int64_t)1 << 30) return ANCHORKV_EINVAL;
  return ANCHORKV_OK;
}

int make_plan(const anchorkv_params* p, Plan* pl) {
  int st = validate(p);
  if (st) return st;
  memset(pl, 0, sizeof(*pl));
  pl->p = *p;
  int n_s, n_u;
  bool all;
  st = fill_layout(p, &pl->L, &n_s, &n_u, &all);
  if (st) return st;
  if (n_u > 2048) return ANCHORKV_EUNSUPPORTED;          // uniform-sample candidate buffer
  if (pl->L.n_anchors > 2048) return ANCHORKV_EUNSUPPORTED;   // fp64 re-decision score buffer
  pl->N = p->n_tokens; pl->D = p->head_dim; pl->H = p->n_kv_heads; pl->Hq = p->n_q_heads;
  pl->G = pl->Hq / pl->H; pl->W = p->window; pl->GW = pl->G * pl->W;
  pl->k = pl->L.n_anchors; pl->n_s = n_s; pl->n_u = n_u; pl->n_tiles = pl->L.n_tiles;
  pl->elem = p->dtype == ANCHORKV_BF16 ? 2 : 4;
  pl->R = pl->L.n_residuals; pl->cap = pl->L.residual_cap;
  pl->all_anchors = all;
  pl->chunk1 = 1024;
  pl->n_chunk1 = (pl->N + pl->chunk1 - 1) / pl->chunk1;
  // tensor-core observation passes: 128-row blocks, token range split so
  // that the (head, row block, split) items fill the SMs about once
  pl->tc_rb = (pl->GW + 127) / 128;
  {
    // one CTA per SM (their shared memory allows no more): at most 148 items,
    // so every item runs in the first wave
    const int units = pl->H * pl->tc_rb, row_tiles = (pl->N + 127) / 128;
    const int want = std::max(1, 148 / units);
    pl->tc_tps = std::max(1, (row_tiles + want - 1) / want);
    pl->tc_split = (row_tiles + pl->tc_tps - 1) / pl->tc_tps;
  }
  pl->obs_rb = 1;
  const int64_t H = pl->H, N = pl->N, GW = pl->GW, k = pl->k, D = kD;
  const int64_t n_sh_t = 2 * H * pl->n_tiles;
  // the tensor-core passes leave kObsGroups row-block partials per 128-row block
  const int64_t U = H * pl->tc_rb, nrb = kObsGroups * pl->tc_rb;
  int64_t off = 0;
  auto take = [&](int64_t bytes) { int64_t o = off; off += (bytes + 255) / 256 * 256; return o; };
  pl->o_counters = take(4 * (kCounterCount + 2 * H));
  pl->o_row_m = take(4 * H * GW);
  pl->o_row_z = take(4 * H * GW);
  pl->o_ybar = take(4 * H * GW * D);
  pl->o_part_m = take(4 * H * pl->n_chunk1 * GW);
  pl->o_part_l = take(4 * H * pl->n_chunk1 * GW);
  pl->o_part_y = take(4 * H * pl->n_chunk1 * GW * D);
  pl->o_tc_pm2 = take(4 * U * kObsGroups * pl->tc_split * 128);
  pl->o_tc_pl = take(4 * U * kObsGroups * pl->tc_split * 128);
  pl->o_tc_rm2 = take(4 * U * 128);
  pl->o_tc_riz = take(4 * U * 128);
  pl->o_tc_rq2 = take(4 * U * 128);
  pl->o_tc_ry2 = take(4 * U * 128);
  pl->o_tc_py = take(4 * U * pl->tc_split * 128 * 128);
  pl->o_tc_yh = take(2 * U * 128 * 128);
  pl->o_tc_yl = take(2 * U * 128 * 128);
  pl->o_score = take(4 * nrb * H * N);
  pl->o_a2 = take(4 * nrb * H * N);
  pl->o_ku = take(4 * nrb * H * N);
  pl->o_pooled = take(4 * H * N);
  pl->o_slot_of = take(4 * H * N);
  pl->o_anc_n2 = take(8 * 2 * H * k);
  pl->kp16 = (pl->k + 15) / 16 * 16;
  pl->o_anc_inv = take(4 * 2 * H * pl->kp16);
  pl->o_anc_sqrt = take(8 * 2 * H * k);
  pl->o_xnorm = take(4 * 2 * H * N);
  pl->o_util = take(4 * 2 * H * N);
  pl->o_refine = take(4 * 2 * H * N);
  pl->o_sel_state = take(64);
  pl->o_hist = take(4 * 256);
  pl->o_tile_gt = take(4 * n_sh_t);
  pl->o_tile_eq = take(4 * n_sh_t);
  pl->o_tie_before = take(4 * (n_sh_t + 1));
  pl->o_tile_cnt = take(4 * n_sh_t);
  // proxy observation queries (key-as-query mode)
  pl->o_qproxy = (p->mode & ANCHORKV_MODE_KEY_QUERIES) ? take((int64_t)pl->Hq * pl->W * kD * pl->elem) : 0;
  pl->o_asg_keys = pl->k > kAssignGroupMax ? take(16 * 2 * H * N) : 0;
  pl->o_asg_probe = take(4 * 512 * kAssignGroupMax);
  pl->ws_total = off;
  double mse;
  codebook(&pl->tau, &pl->l1, &pl->l2, &mse);
  for (int j = 0; j < 4; ++j) pl->sign_bits[j] = 0;
  for (int j = 0; j < kD; ++j) {
    const uint64_t z = splitmix64(p->seed ^ (1ull << 63) ^ (uint64_t)j);
    if (z & 1ull) pl->sign_bits[j >> 5] |= 1u << (j & 31);
  }
  return ANCHORKV_OK;
}

// The tensor-core assignment runs for bf16 caches whose anchors fit in
// shared memory; ANCHORKV_SIMT_ASSIGN=1 forces the SIMT path (tests use it to
// compare the two).
static bool use_tc_assign(const Plan& pl) {
  const char* e = getenv("ANCHORKV_SIMT_ASSIGN");
  if (e && e[0] == '1') return false;
  return assign_tc_supported(pl);
}

// The tensor-core observation passes run for bf16 caches;
// ANCHORKV_SIMT_OBS=1 forces the SIMT passes.
static bool use_tc_obs(const Plan& pl) {
  const char* e = getenv("ANCHORKV_SIMT_OBS");
  if (e && e[0] == '1') return false;
  return obs_tc_supported(pl);
}

static int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ANCHORKV_ECUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return ANCHORKV_ECUDA;
  return major == 10 ? ANCHORKV_OK : ANCHORKV_EUNSUPPORTED;
}

#define AKV_LAUNCH(expr)                         \
  do {                                           \
    cudaError_t e_ = (expr);                     \
    if (e_ != cudaSuccess) return ANCHORKV_ECUDA; \
  } while (0)

// Device staging of anchorkv_compress_host: K, V, Q_obs and the layout, each
// section 256-byte aligned.
struct HostStaging {
  int64_t kv, q, out, o_k, o_v, o_q, o_out, total;
};
HostStaging host_staging(const Plan& pl) {
  auto al = [](int64_t x) { return (x + 255) / 256 * 256; };
  HostStaging h;
  h.kv = (int64_t)pl.H * pl.N * kD * pl.elem;
  h.q = (int64_t)pl.Hq * pl.W * kD * pl.elem;
  h.out = pl.L.total_bytes;
  h.o_k = 0;
  h.o_v = al(h.kv);
  h.o_q = h.o_v + al(h.kv);
  h.o_out = h.o_q + al(h.q);
  h.total = h.o_out + al(h.out);
  return h;
}

}  // namespace akv

using namespace akv;

extern "C" {

int anchorkv_default_params(anchorkv_params* p) {
  if (!p) return ANCHORKV_EINVAL;
  memset(p, 0, sizeof(*p));
  p->n_tokens = 0;
  p->head_dim = 128;
  p->n_kv_heads = 8;
  p->n_q_heads = 32;
  p->window = 32;
  p->dtype = ANCHORKV_BF16;
  p->theta = 0.05;
  p->seed = 0;
  p->layer = 0;
  p->anchor_div = 128;
  p->rho_num = 7;
  p->rho_den = 10;
  p->pool_kernel = 7;
  return ANCHORKV_OK;
}

int anchorkv_bytes(const anchorkv_params* p, anchorkv_layout* out) {
  if (!out) return ANCHORKV_EINVAL;
  int st = validate(p);
  if (st) return st;
  int n_s, n_u;
  bool all;
  return fill_layout(p, out, &n_s, &n_u, &all);
}

int anchorkv_compress_workspace(const anchorkv_params* p, anchorkv_workspace_view* out) {
  if (!out) return ANCHORKV_EINVAL;
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  out->total_bytes = pl.ws_total;
  out->off_pooled = pl.o_pooled;
  out->off_utility = pl.o_util;
  out->off_counters = pl.o_counters;
  out->off_assign_probe = pl.o_asg_probe;
  return ANCHORKV_OK;
}

int anchorkv_compress(const anchorkv_params* p, const void* K, const void* V, const void* Q_obs, void* out,
                      size_t out_bytes, void* ws, size_t ws_bytes, void* stream) {
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  const bool key_queries = (p->mode & ANCHORKV_MODE_KEY_QUERIES) != 0;
  if (!K || !V || (!Q_obs && !key_queries) || !out || !ws) return ANCHORKV_EINVAL;
  if ((int64_t)out_bytes < pl.L.total_bytes || (int64_t)ws_bytes < pl.ws_total) return ANCHORKV_ENOSPC;
  if (((uintptr_t)K | (uintptr_t)V | (uintptr_t)Q_obs | (uintptr_t)out | (uintptr_t)ws) & 15) return ANCHORKV_EINVAL;
  st = check_device();
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char* o = (char*)out;
  char* w = (char*)ws;
  AKV_LAUNCH(cudaMemsetAsync(w + pl.o_counters, 0, 4 * (kCounterCount + 2 * (size_t)pl.H), s));
  if (key_queries) {
    AKV_LAUNCH(launch_key_queries(pl, K, w + pl.o_qproxy, s));
    Q_obs = w + pl.o_qproxy;
  }
#define AKV_STAGE(st, nk, expr) \
  do { stage_begin(st, s); AKV_LAUNCH(expr); stage_end(st, s, nk); } while (0)
  if (use_tc_obs(pl)) {
    pl.obs_rb = kObsGroups * pl.tc_rb;
    AKV_LAUNCH(launch_obs_tc(pl, K, V, Q_obs, w, s));
  } else {
    pl.obs_rb = 1;
    AKV_STAGE(kStObsPass1, 1, launch_obs_pass1(pl, K, V, Q_obs, w, s));
    AKV_STAGE(kStObsCombine, 1, launch_obs_combine(pl, w, s));
    AKV_STAGE(kStTokenStats, 1, launch_token_stats(pl, K, V, Q_obs, w, s));
  }
  AKV_STAGE(kStAnchorSelect, 1, launch_anchor_select(pl, K, V, o, w, s));
  if (use_tc_assign(pl)) {
    AKV_STAGE(kStAssign, 1, launch_assign_tc(pl, K, V, o, w, s));
  } else {
    AKV_STAGE(kStAssign, 1, launch_assign_simt(pl, K, V, o, w, s));
  }
  AKV_STAGE(kStRefine, 1, launch_refine(pl, K, V, o, w, s));
  AKV_STAGE(kStProject, 1, launch_project(pl, K, V, o, w, s));
  const int sel_kernels = pl.R == 0 ? 0 : 1;
  AKV_STAGE(kStSelect, sel_kernels, launch_select(pl, o, w, s));
  AKV_STAGE(kStQuantize, pl.R ? 1 : 0, launch_quantize(pl, K, V, o, w, s));
#undef AKV_STAGE
  return ANCHORKV_OK;
}

int anchorkv_compress_host_staging_bytes(const anchorkv_params* p, size_t* bytes) {
  if (!bytes) return ANCHORKV_EINVAL;
  Plan pl;
  const int st = make_plan(p, &pl);
  if (st) return st;
  *bytes = (size_t)host_staging(pl).total;
  return ANCHORKV_OK;
}

int anchorkv_compress_host(const anchorkv_params* p, const void* K_host, const void* V_host, const void* Q_host,
                           void* out_host, size_t out_bytes, void* staging, size_t staging_bytes, void* ws,
                           size_t ws_bytes, void* stream) {
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  const bool key_queries = (p->mode & ANCHORKV_MODE_KEY_QUERIES) != 0;
  if (!K_host || !V_host || (!Q_host && !key_queries) || !out_host || !staging || !ws) return ANCHORKV_EINVAL;
  const HostStaging hs = host_staging(pl);
  if ((int64_t)out_bytes < pl.L.total_bytes || (int64_t)staging_bytes < hs.total) return ANCHORKV_ENOSPC;
  if (((uintptr_t)staging | (uintptr_t)ws) & 15) return ANCHORKV_EINVAL;
  st = check_device();
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char* d = (char*)staging;
  AKV_LAUNCH(cudaMemcpyAsync(d + hs.o_k, K_host, (size_t)hs.kv, cudaMemcpyHostToDevice, s));
  AKV_LAUNCH(cudaMemcpyAsync(d + hs.o_v, V_host, (size_t)hs.kv, cudaMemcpyHostToDevice, s));
  if (Q_host) AKV_LAUNCH(cudaMemcpyAsync(d + hs.o_q, Q_host, (size_t)hs.q, cudaMemcpyHostToDevice, s));
  st = anchorkv_compress(p, d + hs.o_k, d + hs.o_v, Q_host ? d + hs.o_q : nullptr, d + hs.o_out, (size_t)hs.out, ws,
                         ws_bytes, stream);
  if (st) return st;
  AKV_LAUNCH(cudaMemcpyAsync(out_host, d + hs.o_out, (size_t)hs.out, cudaMemcpyDeviceToHost, s));
  return ANCHORKV_OK;
}

int anchorkv_decode_workspace_bytes(const anchorkv_params* p, int32_t batch, size_t* ws_bytes) {
  if (!ws_bytes || batch < 0) return ANCHORKV_EINVAL;
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  DecodePlan dp;
  make_decode_plan(pl, std::max(batch, 1), &dp);
  *ws_bytes = (size_t)dp.ws_total;
  return ANCHORKV_OK;
}

int anchorkv_decode_attn(const anchorkv_params* p, const void* compressed, int64_t seq_stride_bytes, int32_t batch,
                         const void* q, const void* K_tail, const void* V_tail, int32_t tail_len, int32_t tail_cap,
                         float* out, void* ws, size_t ws_bytes, void* stream) {
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  if (batch < 0 || tail_len < 0 || tail_cap < tail_len) return ANCHORKV_EINVAL;
  if (batch == 0) return ANCHORKV_OK;
  if (batch > 65535) return ANCHORKV_EUNSUPPORTED;
  if (!compressed || !q || !out) return ANCHORKV_EINVAL;
  if (tail_len > 0 && (!K_tail || !V_tail)) return ANCHORKV_EINVAL;
  if (tail_len > 4096) return ANCHORKV_EUNSUPPORTED;
  if (seq_stride_bytes < pl.L.total_bytes && batch > 1) return ANCHORKV_EINVAL;
  if (seq_stride_bytes % 16) return ANCHORKV_EINVAL;
  if (((uintptr_t)compressed | (uintptr_t)q | (uintptr_t)out | (uintptr_t)ws | (uintptr_t)K_tail |
       (uintptr_t)V_tail) & 15)
    return ANCHORKV_EINVAL;
  DecodePlan dp;
  make_decode_plan(pl, batch, &dp);
  if ((int64_t)ws_bytes < dp.ws_total) return ANCHORKV_ENOSPC;
  if (dp.ws_total > 0 && !ws) return ANCHORKV_EINVAL;
  st = check_decode_shape(pl, dp, tail_len);
  if (st) return st;
  st = check_device();
  if (st) return st;
  return launch_decode(pl, dp, (const char*)compressed, seq_stride_bytes, q, K_tail, V_tail, tail_len, tail_cap, out,
                       (char*)ws, (cudaStream_t)stream);
}

int anchorkv_decode_rope_workspace_bytes(const anchorkv_params* p, int32_t batch, size_t* ws_bytes) {
  if (!ws_bytes || batch < 0) return ANCHORKV_EINVAL;
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  *ws_bytes = (size_t)make_rope_plan(pl, std::max(batch, 1)).ws_total;
  return ANCHORKV_OK;
}

int anchorkv_decode_attn_rope(const anchorkv_params* p, const void* compressed, int64_t seq_stride_bytes,
                              int32_t batch, const void* q, const void* K_tail, const void* V_tail, int32_t tail_len,
                              int32_t tail_cap, double rope_base, float* out, void* ws, size_t ws_bytes,
                              void* stream) {
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  if (batch < 0 || tail_len < 0 || tail_cap < tail_len) return ANCHORKV_EINVAL;
  if (!(rope_base > 1.0) || !isfinite(rope_base)) return ANCHORKV_EINVAL;
  if (batch == 0) return ANCHORKV_OK;
  if ((int64_t)batch * pl.H > 65535) return ANCHORKV_EUNSUPPORTED;     // (sequence, head) pairs: grid y
  if (!compressed || !q || !out || !ws) return ANCHORKV_EINVAL;
  if (tail_len > 0 && (!K_tail || !V_tail)) return ANCHORKV_EINVAL;
  if ((int64_t)pl.N + tail_len > (1 << 21)) return ANCHORKV_EUNSUPPORTED;
  if (seq_stride_bytes < pl.L.total_bytes && batch > 1) return ANCHORKV_EINVAL;
  if (seq_stride_bytes % 16) return ANCHORKV_EINVAL;
  if (((uintptr_t)compressed | (uintptr_t)q | (uintptr_t)out | (uintptr_t)ws | (uintptr_t)K_tail |
       (uintptr_t)V_tail) & 15)
    return ANCHORKV_EINVAL;
  const RopePlan rp = make_rope_plan(pl, batch);
  if ((int64_t)ws_bytes < rp.ws_total) return ANCHORKV_ENOSPC;
  st = check_device();
  if (st) return st;
  AKV_LAUNCH(launch_decode_rope(pl, rp, (const char*)compressed, seq_stride_bytes, batch, q, K_tail, V_tail, tail_len,
                                tail_cap, rope_base, out, (char*)ws, (cudaStream_t)stream));
  return ANCHORKV_OK;
}

int anchorkv_decode_config(const anchorkv_params* p, int32_t batch, int32_t* slices, int32_t* smem_bytes) {
  if (!slices || !smem_bytes || batch < 1) return ANCHORKV_EINVAL;
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  DecodePlan dp;
  make_decode_plan(pl, batch, &dp);
  *slices = 0;
  *smem_bytes = 0;
  if (!dp.flash) return ANCHORKV_OK;
  st = check_device();
  if (st) return st;
  if (flash_ctas_per_sm(pl, dp.fs) < 1) return ANCHORKV_EUNSUPPORTED;
  *slices = dp.fs.S;
  *smem_bytes = dp.fs.smem;
  return ANCHORKV_OK;
}

int anchorkv_reconstruct(const anchorkv_params* p, const void* compressed, float* K_hat, float* V_hat,
                         void* stream) {
  Plan pl;
  int st = make_plan(p, &pl);
  if (st) return st;
  if (!compressed || !K_hat || !V_hat) return ANCHORKV_EINVAL;
  st = check_device();
  if (st) return st;
  AKV_LAUNCH(launch_reconstruct(pl, (const char*)compressed, K_hat, V_hat, (cudaStream_t)stream));
  return ANCHORKV_OK;
}

int anchorkv_read_device_status(const void* ws, int32_t* host_counters, void* stream) {
  if (!ws || !host_counters) return ANCHORKV_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(host_counters, ws, 4 * kCounterCount, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ANCHORKV_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ANCHORKV_ECUDA;
  return host_counters[kStatus] ? ANCHORKV_EDEVICE : ANCHORKV_OK;
}

int anchorkv_codebook(double* out4) {
  if (!out4) return ANCHORKV_EINVAL;
  codebook(&out4[0], &out4[1], &out4[2], &out4[3]);
  return ANCHORKV_OK;
}

const char* anchorkv_strerror(int status) {
  switch (status) {
    case ANCHORKV_OK: return "ok";
    case ANCHORKV_EINVAL: return "invalid argument";
    case ANCHORKV_ENOSPC: return "buffer too small";
    case ANCHORKV_EUNSUPPORTED: return "unsupported configuration or device";
    case ANCHORKV_ECUDA: return "CUDA error";
    case ANCHORKV_EDEVICE: return "device-side check failed";
    default: return "unknown status";
  }
}

}  // extern "C"
