/*
 * anchorkv.h - C ABI of the AnchorKV anchor-residual KV-cache codec for
 * NVIDIA B200 (sm_100a).
 *
 * The method (arXiv 2608.02901; pages "AnchorKV: Anchor-Residual KV Cache
 * Compression" (pith.science review) and "AnchorKV-adapted - Anchor-Residual
 * Compression, No Eviction" (VeloxQuant-MLX docs)):
 *   every cached key/value x_i of a KV head is stored as an anchor index a(i),
 *   a 2-byte coefficient gamma_i = <x_i, x_a>/||x_a||^2 and, for the token-sides
 *   a per-layer byte budget can buy, a 2-bit Hadamard-rotated Lloyd-Max
 *   residual; reconstruction is x^_i = gamma_i x_a(i) + r~_i
 *   (review, "What carries the argument").  Compression runs once per layer at
 *   the end of prefill; decode tokens are appended uncompressed (VeloxQuant,
 *   "Adaptation notes").
 *
 * Conventions for every entry point:
 *   - returns ANCHORKV_OK (0) or a negative ANCHORKV_E* code; never throws,
 *     never allocates device or pinned memory, never synchronizes the device
 *     except where stated;
 *   - "device" pointers are CUDA global-memory addresses on the current
 *     device; "host" pointers are ordinary CPU memory;
 *   - the caller owns every buffer; work is enqueued on `stream`
 *     (a cudaStream_t passed as void*, NULL = legacy default stream) and is
 *     asynchronous: a 0 return means "validated and launched";
 *   - device-side checks that fail latch a status word in the workspace
 *     (read it with anchorkv_read_device_status) instead of trapping.
 * Tensors are dense and row-major; D (head_dim) is the fastest dimension.
 * Query head j belongs to KV head j / (n_q_heads / n_kv_heads).
 */
#ifndef ANCHORKV_H_
#define ANCHORKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum anchorkv_status {
  ANCHORKV_OK = 0,
  ANCHORKV_EINVAL = -1,        /* null pointer, bad size or bad parameter        */
  ANCHORKV_ENOSPC = -2,        /* an output or workspace buffer is too small     */
  ANCHORKV_EUNSUPPORTED = -3,  /* dtype/head_dim/device not supported            */
  ANCHORKV_ECUDA = -4,         /* a CUDA runtime call or launch failed           */
  ANCHORKV_EDEVICE = -5        /* a device-side check latched an error           */
};

enum anchorkv_dtype { ANCHORKV_FP32 = 0, ANCHORKV_BF16 = 1 };

/*
 * One layer's compression problem.  Defaults (anchorkv_default_params) follow
 * the review's "Assumptions & free parameters": W = 32, k = S/128,
 * rho = 0.7, kappa = 7; theta is the single user knob (VeloxQuant,
 * "The one setting worth tuning: anchorkv_theta").
 */
typedef struct anchorkv_params {
  int32_t n_tokens;     /* N, prefill length of the layer (> window)           */
  int32_t head_dim;     /* D, must be 128                                      */
  int32_t n_kv_heads;   /* H, 1..65535                                         */
  int32_t n_q_heads;    /* H_q, a multiple of H                                */
  int32_t window;       /* W, trailing positions kept exactly; 1..256          */
  int32_t dtype;        /* anchorkv_dtype of K, V, Q_obs, anchors, tails, q    */
  double theta;         /* retained fraction of the uncompressed bytes, > 0    */
  uint64_t seed;        /* uniform anchor sample + shared Hadamard signs       */
  int32_t layer;        /* layer index (0..32767), keys the uniform sample     */
  int32_t anchor_div;   /* m = ceil(N / anchor_div) non-window anchors (128)   */
  int32_t rho_num;      /* scored share of the m slots = rho_num/rho_den (7)   */
  int32_t rho_den;      /* (10)                                                */
  int32_t pool_kernel;  /* kappa, odd, positional pooling width (7)            */
  int32_t mode;         /* ANCHORKV_MODE_* bits; 0 = the method as published   */
} anchorkv_params;

/*
 * Mode bits of anchorkv_params.mode (compress and decode of one layout must
 * use the same mode):
 *   ANCHORKV_MODE_KEY_QUERIES  Q_obs may be NULL; the trailing W keys of each
 *       KV head serve as the observation queries of its query heads (VeloxQuant
 *       "Adaptation notes": key-as-query proxy, since a cache wrapper never
 *       sees queries).
 *   bits 1..3 (ANCHORKV_MODE_RANK(r)): the criterion that ranks token-sides
 *       for the residual budget; UTILITY is the method, the others are the
 *       alternatives the review's "Circularity Check" names for the Figure 5
 *       ablation: residual norm ||r||^2, attention (sum of the observation
 *       weights), cosine (1 - cos(x, x_a)), random (a seeded hash of the flat
 *       index).  Values above ANCHORKV_RANK_RANDOM are rejected (EINVAL).
 *   ANCHORKV_MODE_NAIVE_CODEC  the 2-bit codec without the sign flip and
 *       Hadamard rotation (the review's "Naive 2 bit" ablation).
 * Any other bit set: EINVAL.
 */
#define ANCHORKV_MODE_KEY_QUERIES 0x1
#define ANCHORKV_MODE_RANK_SHIFT 1
#define ANCHORKV_MODE_RANK_MASK 0xE
#define ANCHORKV_MODE_RANK(r) ((int32_t)(r) << ANCHORKV_MODE_RANK_SHIFT)
#define ANCHORKV_MODE_NAIVE_CODEC 0x10
#define ANCHORKV_MODE_ALL 0x1F
enum anchorkv_rank {
  ANCHORKV_RANK_UTILITY = 0,
  ANCHORKV_RANK_RESIDUAL_NORM = 1,
  ANCHORKV_RANK_ATTENTION = 2,
  ANCHORKV_RANK_COSINE = 3,
  ANCHORKV_RANK_RANDOM = 4
};

/*
 * Byte accounting of one compressed layer (review, Referee "Summary": an exact
 * byte accounting, Eq. 13, maps theta to a per-layer residual budget; minor
 * comment 1: b_a = b_gamma = 2).  All offsets are from the start of the
 * compressed buffer; sections start on 16-byte boundaries:
 *   anchors_k  [H][k][D]  dtype      anchor keys, exact
 *   anchors_v  [H][k][D]  dtype      anchor values, exact
 *   anchor_pos [H][k]     int32      positions, ascending (slot order)
 *   tok        [2][H][N]  uint32     side 0 = K, 1 = V; bits 0..15 anchor slot,
 *                                    bits 16..31 fp16 gamma
 *   bitmap     [2][H][n_tiles][4] uint32   bit t%32 of word (t%128)/32 of
 *                                    tile t/128: token-side t has a residual
 *   tile_prefix [2][H][n_tiles+1] int32    residual record index at each tile
 *                                    start (flat order side, head, token)
 *   res_codes  [R][D/4]   uint8      2-bit codes, coordinate j in byte j/4,
 *                                    bits 2*(j%4)
 *   res_sigma  [R]        fp16       residual scale ||r||/sqrt(D)
 * total_bytes = base_bytes + residual_bytes_each * n_residuals <= budget_bytes
 * whenever n_residuals > 0 (if theta is so small that base_bytes exceeds the
 * budget, n_residuals is 0 and total_bytes > budget_bytes; VeloxQuant
 * "The one setting worth tuning" notes the same floor to zero).
 */
typedef struct anchorkv_layout {
  int64_t total_bytes;
  int64_t base_bytes;
  int64_t budget_bytes;        /* floor(theta * uncompressed_bytes)          */
  int64_t uncompressed_bytes;  /* 2 * H * N * D * elem                       */
  int64_t n_residuals;         /* R                                          */
  int64_t residual_cap;        /* 2 * H * (N - k) eligible token-sides       */
  int64_t residual_bytes_each; /* D/4 + 2                                    */
  int32_t n_anchors;           /* k                                          */
  int32_t n_scored;            /* n_s                                        */
  int32_t n_uniform;           /* n_u                                        */
  int32_t n_tiles;             /* ceil(N / 128)                              */
  int64_t off_anchors_k, off_anchors_v, off_anchor_pos, off_tok;
  int64_t off_bitmap, off_tile_prefix, off_res_codes, off_res_sigma;
} anchorkv_layout;

/*
 * Diagnostic views into the compress workspace (device offsets from the
 * workspace base), valid after anchorkv_compress returns and its stream
 * work completes.  Counters: [0] device status (0 = ok), [1] rows whose
 * nearest-anchor decision was re-taken in fp64 because the fp32 margin was
 * inside the fp32 error bound, [2] residual ties at the selection threshold.
 */
typedef struct anchorkv_workspace_view {
  int64_t total_bytes;
  int64_t off_pooled;      /* float [H][N]: pooled score (first N-W valid)     */
  int64_t off_utility;     /* float [2][H][N]: utility, -1 for anchors         */
  int64_t off_counters;    /* int32 [16]                                       */
  /* float [512][kpad]: the tensor-core assignment's raw fp32 accumulators
   * <x_t, a_s> for tokens t < min(N, 512) of the key side of KV head 0
   * against the slots s of the first anchor group (kpad = that group's width
   * rounded up to its chunking, at most 480); written only on the bf16
   * tensor-core path and only when the environment variable
   * ANCHORKV_ASSIGN_PROBE is 1 at the call.  A diagnostic that lets a test
   * measure the accumulation error the nearest-anchor certification relies
   * on. */
  int64_t off_assign_probe;
} anchorkv_workspace_view;

/* Fills `p` with the pages' defaults (D = 128, W = 32, k = S/128, rho = 0.7,
 * kappa = 7, bf16, theta = 0.05, seed 0, layer 0).  Host, pure. */
int anchorkv_default_params(anchorkv_params* p);

/* Validates `p` and computes the compressed layout (Eq. 13 reading).
 * Host, pure, no CUDA call.  EINVAL on a bad parameter. */
int anchorkv_bytes(const anchorkv_params* p, anchorkv_layout* out);

/* Workspace bytes anchorkv_compress needs for `p`, and where its diagnostic
 * arrays live.  Host, pure. */
int anchorkv_compress_workspace(const anchorkv_params* p, anchorkv_workspace_view* out);

/*
 * Compresses one layer (review, Referee "Summary"; "What carries the
 * argument"): observation-window score and kappa pooling (Eq. 14), anchors
 * (window + rho by score + uniform sample), nearest-anchor assignment per
 * side, gamma and residual, first-order key/value utilities (Eq. 6 reading),
 * per-layer top-R residual selection pooled over heads and sides, randomized
 * Hadamard rotation + 2-bit Lloyd-Max codes.
 *   K, V   device [H][N][D] dtype     prefill keys (pre-RoPE) and values
 *   Q_obs  device [H_q][W][D] dtype   queries of the last W positions (may be
 *          NULL with ANCHORKV_MODE_KEY_QUERIES)
 *   out    device, out_bytes >= anchorkv_layout.total_bytes
 *   ws     device, ws_bytes >= anchorkv_workspace_view.total_bytes; the call
 *          overwrites it (no state is carried between calls)
 * Inputs are not modified.  Output is bit-for-bit deterministic.
 */
int anchorkv_compress(const anchorkv_params* p, const void* K, const void* V,
                      const void* Q_obs, void* out, size_t out_bytes,
                      void* ws, size_t ws_bytes, void* stream);

/* Device staging bytes anchorkv_compress_host needs for `p`: K, V, Q_obs and
 * the compressed layout of one layer, each 256-byte aligned.  Host, pure. */
int anchorkv_compress_host_staging_bytes(const anchorkv_params* p, size_t* bytes);

/*
 * anchorkv_compress from host buffers: copies K, V and Q_obs into `staging`,
 * compresses there and copies the layout back, everything queued on
 * `stream` (one cudaMemcpyAsync per buffer, so page-locked host buffers make
 * the copies asynchronous and let them overlap work on other streams).
 *   K_host, V_host  host [H][N][D] dtype
 *   Q_host          host [H_q][W][D] dtype (may be NULL with
 *                   ANCHORKV_MODE_KEY_QUERIES)
 *   out_host        host, out_bytes >= anchorkv_layout.total_bytes; valid once
 *                   `stream` has completed the call's work
 *   staging         device, 16-byte aligned, staging_bytes >=
 *                   anchorkv_compress_host_staging_bytes; owned by the caller.
 *                   It holds K, V, Q_obs and the layout in that order, each
 *                   section rounded up to 256 bytes; the layout (its last
 *                   section) stays there for the caller's device-side use
 *   ws, ws_bytes    as for anchorkv_compress
 * The host buffers must stay alive and unmodified until the stream completes.
 * Errors as anchorkv_compress; ENOSPC also for a small staging buffer.
 */
int anchorkv_compress_host(const anchorkv_params* p, const void* K_host, const void* V_host,
                           const void* Q_host, void* out_host, size_t out_bytes, void* staging,
                           size_t staging_bytes, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes anchorkv_decode_attn needs for `batch` sequences (0 when
 * every (sequence, head) is decoded by a single CTA). */
int anchorkv_decode_workspace_bytes(const anchorkv_params* p, int32_t batch, size_t* ws_bytes);

/*
 * Decode attention over compressed layers (review, Referee "Summary": a
 * FlashAttention-style decoder that rebuilds tiles when consumed):
 *   o_j = softmax_t(q_j . K^_t / sqrt(D)) V^  over the N compressed tokens of
 *   the sequence followed by the `tail_len` exact tokens appended during
 *   decode (VeloxQuant, "Adaptation notes").  K^ and V^ are never written out.
 *   compressed  device, `batch` layouts of this layer, one every
 *               `seq_stride_bytes` bytes (>= total_bytes, multiple of 16)
 *   q           device [batch][H_q][D] dtype
 *   K_tail, V_tail device [batch][H][tail_cap][D] dtype, first tail_len valid
 *               (may be NULL when tail_len == 0), 16-byte aligned
 *   out         device [batch][H_q][D] float32
 *   ws          device, ws_bytes >= anchorkv_decode_workspace_bytes; the call
 *               overwrites it (it clears its own counters on `stream` first)
 * Every device pointer must be 16-byte aligned (EINVAL otherwise, checked
 * before any launch).  Errors: EINVAL for a bad pointer, size or stride;
 * ENOSPC for a small workspace; EUNSUPPORTED when batch * H > 65535,
 * tail_len > 4096 or no launch shape fits the device.
 * Work split: each (sequence, KV head) is cut into token slices that run on
 * separate CTAs across the GPU; the last slice to finish merges the others.
 * When a head gets two slices or fewer (many sequences), a tensor-core pass
 * first computes every key record's residual logits into the workspace
 * (batch x R x G floats); ANCHORKV_DECODE_KLOGIT=0 or 1 in the environment
 * turns that pass off or on for every shape.
 */
int anchorkv_decode_attn(const anchorkv_params* p, const void* compressed,
                         int64_t seq_stride_bytes, int32_t batch, const void* q,
                         const void* K_tail, const void* V_tail, int32_t tail_len,
                         int32_t tail_cap, float* out, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * Decode attention when the cached keys were stored before the rotary
 * position map (review, "Assumptions & free parameters": RoPE is a
 * per-position orthogonal linear map, so it distributes over the
 * anchor-residual split, which justifies pre-RoPE storage and rotation at
 * decode time).  Same layouts and arguments as anchorkv_decode_attn, plus
 * rope_base (> 1, e.g. 10000 or 500000).  Rotate-half pairing: coordinate i
 * and i + D/2 turn by p * rope_base^(-2i/D); cached token t sits at
 * position t, tail token i at N + i (the tail keys are passed pre-rotary as
 * well), the query q at N + tail_len; values are not rotated.  Keys are
 * rebuilt token by token (gamma~ K_a + r~), so this path reads the anchors
 * once per token instead of once per slot.
 *   ws  device, ws_bytes >= anchorkv_decode_rope_workspace_bytes
 * Errors: EINVAL for a bad base, pointer, size or stride; EUNSUPPORTED when
 * batch * H > 65535 or N + tail_len > 2^21; ENOSPC for a small workspace.
 */
int anchorkv_decode_rope_workspace_bytes(const anchorkv_params* p, int32_t batch, size_t* ws_bytes);
int anchorkv_decode_attn_rope(const anchorkv_params* p, const void* compressed,
                              int64_t seq_stride_bytes, int32_t batch, const void* q,
                              const void* K_tail, const void* V_tail, int32_t tail_len,
                              int32_t tail_cap, double rope_base, float* out, void* ws,
                              size_t ws_bytes, void* stream);

/*
 * Launch shape of anchorkv_decode_attn for `batch` sequences on the current
 * device (a diagnostic with no counterpart in the method): token slices (one
 * CTA each) per (sequence, KV head) and dynamic shared memory per CTA.  When
 * the slice decode's shared-memory plan does not fit (many query heads per KV
 * head together with many anchors), *slices = 0 and the split-token kernels
 * run.  Host; queries the device once per shape.  EUNSUPPORTED if the slice
 * kernel cannot be resident on the device.
 */
int anchorkv_decode_config(const anchorkv_params* p, int32_t batch, int32_t* slices, int32_t* smem_bytes);

/*
 * Decode attention that allocates nothing.  The paper has no counterpart:
 * this is a library service, not part of the method.  Same operation,
 * arguments and errors as anchorkv_decode_attn, without the workspace: the
 * scratch comes from one library-owned array of
 * ANCHORKV_DECODE_NOALLOC_SCRATCH_BYTES per device, and the call makes no
 * cudaMalloc, cudaFree or other allocating call.  It is meant for callers
 * that cannot allocate device memory while decoding: a serving engine whose
 * free HBM is all handed to its KV-cache pool, a plain-C caller without a
 * device allocator, or a decode loop that must not take the device-wide
 * synchronisation cudaMalloc / cudaFree bring.
 *   - When anchorkv_decode_workspace_bytes exceeds the array, the call first
 *     drops the tensor-core key-logit pre-pass (whose batch x R x G floats
 *     dominate that workspace at large batch) and computes those logits
 *     inside the decode instead; sizes that still do not fit are rejected
 *     with ANCHORKV_ENOSPC before any launch.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - Every call on a device shares the array, which keeps the last call's
 *     contents; the words that must start at zero (per-(sequence, head)
 *     tickets of the slice merge) are cleared by the call on its stream.
 *     Calls that overlap on the GPU (different streams, or different host
 *     threads without ordering between their streams) race on it: order
 *     them on one stream.
 *   - Pointers as for anchorkv_decode_attn (16-byte aligned, tails included).
 */
#define ANCHORKV_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
int anchorkv_decode_attn_noalloc(const anchorkv_params* p, const void* compressed,
                                 int64_t seq_stride_bytes, int32_t batch, const void* q,
                                 const void* K_tail, const void* V_tail, int32_t tail_len,
                                 int32_t tail_cap, float* out, void* stream);

/*
 * Test and inspection hook: writes the dense reconstruction
 * x^_t = gamma~_t x_a(t) + r~_t of one compressed layer.
 *   K_hat, V_hat device [H][N][D] float32.
 */
int anchorkv_reconstruct(const anchorkv_params* p, const void* compressed,
                         float* K_hat, float* V_hat, void* stream);

/* Copies the device status word and counters of a compress workspace to
 * `host_counters` (16 int32) with a synchronous copy on `stream`.  Returns
 * ANCHORKV_EDEVICE if the status word is non-zero.  The first failing check
 * latches its code: 1 uniform anchor sample, 2 refine list, 3 an
 * inconsistent record or selection (a write that would leave its bounds is
 * skipped), 4 a bounded wait in a tensor-core kernel timed out (the kernel
 * drained its own work and returned). */
int anchorkv_read_device_status(const void* ws, int32_t* host_counters, void* stream);

/* The fp32 codebook the kernels use: {tau, l1, l2, mse} of the four-level
 * Lloyd-Max quantizer for N(0,1), computed by the library at load. */
int anchorkv_codebook(double* out4);

/* Optional stage timing (tracing).  anchorkv_stage_timing(1) starts
 * recording a CUDA event pair around every compress/decode stage on the
 * caller's stream and clears the accumulators; (0) stops.  Host-side state,
 * process-wide; recording adds a few microseconds per stage. */
int anchorkv_stage_timing(int enable);

/* Number of timed stages reported by anchorkv_stage_times. */
#define ANCHORKV_N_STAGES 16

/* Waits for the recorded events and returns, per stage (n >= ANCHORKV_N_STAGES entries),
 * the accumulated milliseconds and the number of timed calls since the last
 * anchorkv_stage_timing call.  Stage names: anchorkv_stage_name. */
int anchorkv_stage_times(double* ms_out, int64_t* calls_out, int32_t n);
const char* anchorkv_stage_name(int32_t stage);

/* Number of kernels this library has launched in this process (host count). */
int anchorkv_launch_count(int64_t* out);

/* Static description of a status code. */
const char* anchorkv_strerror(int status);

#ifdef __cplusplus
}
#endif
#endif /* ANCHORKV_H_ */
