// Host-side plan shared by the C-ABI entry points and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/anchorkv.h"

namespace akv {

// Stages bracketed by the optional event timing (profile.cu).
enum Stage {
  kStObsPass1 = 0, kStObsCombine, kStTokenStats, kStAnchorSelect, kStAssign, kStRefine, kStProject,
  kStSelect, kStQuantize, kStDecodePrep, kStDecodeSplit, kStDecodeCombine, kStObsAlpha, kStObsKu, kStDecodeCluster,
  kStDecodeRope, kStageCount
};
void stage_begin(int stage, cudaStream_t s);
void stage_end(int stage, cudaStream_t s, int kernels);

// Epilogue column groups of the tensor-core observation passes: each leaves
// its own (max, sum) partials (pass A) or per-token row-block sums (B, C).
constexpr int kObsGroups = 4;

// Anchors the tensor-core assignment keeps resident in shared memory at once;
// more are taken in groups of at most this many (best keys merged through
// the workspace between groups).
constexpr int kAssignGroupMax = 480;

// Everything one compress call needs to know, derived from the parameters.
struct Plan {
  anchorkv_params p;
  anchorkv_layout L;
  int N, D, H, Hq, G, W, GW, k, kp16, n_s, n_u, n_tiles, elem;
  int64_t R, cap;
  bool all_anchors;
  // pass-1 token chunks (SIMT observation passes)
  int chunk1, n_chunk1;
  // tensor-core observation passes: row blocks, token splits, tiles per split
  int tc_rb, tc_split, tc_tps;
  // row-block partials of score / sum alpha^2 / key term the consumers sum
  int obs_rb;
  // workspace offsets (bytes from the workspace base)
  int64_t ws_total;
  int64_t o_counters, o_row_m, o_row_z, o_ybar, o_part_m, o_part_l, o_part_y;
  int64_t o_tc_pm2, o_tc_pl, o_tc_rm2, o_tc_riz, o_tc_rq2, o_tc_ry2, o_tc_py, o_tc_yh, o_tc_yl;
  int64_t o_score, o_a2, o_ku, o_pooled, o_slot_of, o_anc_n2, o_anc_inv, o_anc_sqrt, o_xnorm;
  int64_t o_util, o_refine, o_sel_state, o_hist, o_tile_gt, o_tile_eq, o_tie_before, o_tile_cnt;
  int64_t o_qproxy;          // proxy observation queries [Hq][W][D] (key-as-query mode), else 0
  int64_t o_asg_keys;        // best two 64-bit keys per token-side between anchor groups (k > kAssignGroupMax)
  int64_t o_asg_probe;       // [512][kAssignGroupMax] fp32 tensor-core accumulators of the probe rows
  // codebook and Hadamard signs (bit j set: s_j = -1)
  double tau, l1, l2;
  uint32_t sign_bits[4];
};

int make_plan(const anchorkv_params* p, Plan* out);
void codebook(double* tau, double* l1, double* l2, double* mse);

// Slice decode (decode_flash.cu): chunk size, slices per (sequence, head),
// shared memory per CTA and its workspace (tickets, slice partials).
struct FlashShape {
  int ct, S, tps, smem;
  bool klogit;            // key-residual logits from the tensor-core pre-pass
  int64_t ws_total, o_tickets, o_part, o_rlog, o_P;
};
// Tensor-core pre-pass of the slice decode: sigma~ <qr, lev(c)> of every key
// record, [batch][R][GP] floats in the workspace.
bool klogit_tc_supported(const Plan& pl);
int64_t klogit_ws_bytes(const Plan& pl, int batch);
int launch_klogit_tc(const Plan& pl, int batch, const char* comp, int64_t stride, const void* q, float* out,
                     cudaStream_t s);
struct DecodePlan {
  bool flash;             // slice decode; otherwise the split-token kernels
  FlashShape fs;
  int batch, n_split, split_tokens;
  int64_t ws_total, o_P, o_qrot, o_part_m, o_part_l, o_part_w, o_part_z;
};
// allow_prepass = false keeps the key logits inside the decode (no pre-pass
// workspace), for callers whose scratch is fixed.
int make_decode_plan(const Plan& pl, int batch, DecodePlan* out, bool allow_prepass = true);
// Shape checks of a decode call (shared-memory limits of the chosen path).
int check_decode_shape(const Plan& pl, const DecodePlan& dp, int tail_len);
// rope: the rotary decode (keys stored before the rotary map), G <= 8
bool flash_decode_plan(const Plan& pl, int batch, FlashShape* fs, bool allow_prepass = true, bool rope = false);
int launch_flash_decode(const Plan& pl, const FlashShape& fs, int batch, const char* comp, int64_t stride,
                        const void* q, const void* Kt, const void* Vt, int tail_len, int tail_cap, float* out,
                        char* ws, cudaStream_t s, double rope_base = 0.0);
int flash_ctas_per_sm(const Plan& pl, const FlashShape& fs);

// Kernel launchers (one per hot-path step), all asynchronous on `s`.
cudaError_t launch_obs_pass1(const Plan& pl, const void* K, const void* V, const void* Q, char* ws, cudaStream_t s);
cudaError_t launch_obs_combine(const Plan& pl, char* ws, cudaStream_t s);
cudaError_t launch_token_stats(const Plan& pl, const void* K, const void* V, const void* Q, char* ws, cudaStream_t s);
cudaError_t launch_anchor_select(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s);
cudaError_t launch_assign_simt(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s);
cudaError_t launch_refine(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s);
cudaError_t launch_assign_tc(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s);
bool assign_tc_supported(const Plan& pl);
cudaError_t launch_obs_tc(const Plan& pl, const void* K, const void* V, const void* Q, char* ws, cudaStream_t s);
bool obs_tc_supported(const Plan& pl);
cudaError_t launch_project(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s);
cudaError_t launch_select(const Plan& pl, char* out, char* ws, cudaStream_t s);
cudaError_t launch_quantize(const Plan& pl, const void* K, const void* V, char* out, char* ws, cudaStream_t s);
cudaError_t launch_key_queries(const Plan& pl, const void* K, void* Q, cudaStream_t s);

// Decode attention with rotary positions (keys stored before the rotary map).
struct RopePlan {
  bool flash;             // the slice decode with its rotary phase (G <= 8); else the split-token kernels
  FlashShape fs;
  int n_split;
  int64_t ws_total;
};
RopePlan make_rope_plan(const Plan& pl, int batch);
cudaError_t launch_decode_rope(const Plan& pl, const RopePlan& rp, const char* comp, int64_t stride, int batch,
                               const void* q, const void* Kt, const void* Vt, int tail_len, int tail_cap,
                               double rope_base, float* out, char* ws, cudaStream_t s);
// mode bits of the plan's parameters
inline int rank_of(const Plan& pl) { return (pl.p.mode & ANCHORKV_MODE_RANK_MASK) >> ANCHORKV_MODE_RANK_SHIFT; }
inline int naive_codec(const Plan& pl) { return (pl.p.mode & ANCHORKV_MODE_NAIVE_CODEC) ? 1 : 0; }
// Returns an ANCHORKV_* status.
int launch_decode(const Plan& pl, const DecodePlan& dp, const char* comp, int64_t stride,
                  const void* q, const void* Kt, const void* Vt, int tail_len, int tail_cap,
                  float* out, char* ws, cudaStream_t s);
cudaError_t launch_reconstruct(const Plan& pl, const char* comp, float* Kh, float* Vh, cudaStream_t s);

}  // namespace akv
