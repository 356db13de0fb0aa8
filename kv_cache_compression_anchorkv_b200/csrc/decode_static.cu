// Decode attention that allocates nothing: anchorkv_decode_attn with its
// scratch taken from one library-owned array per device instead of a
// caller-provided workspace.
//
// Who needs it: a caller that cannot allocate device memory at decode time.
// A serving engine typically hands nearly all free HBM to its KV-cache pool at
// start-up and has no spare block to lend as a workspace; a caller driving
// the library from plain C may have no device allocator at all; and
// cudaMalloc / cudaFree (or a caching allocator that has to grow) synchronise
// the device, stalling every other stream of a latency-bound decode loop.
// Such a caller passes no workspace here; this entry point calls no
// cudaMalloc, cudaFree or allocating library routine.
//
// The kernels are the ones anchorkv_decode_attn launches; only the origin of
// the scratch pointer differs.

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace akv {
namespace {

// Shared scratch of every anchorkv_decode_attn_noalloc call on a device.  It
// keeps the previous call's contents; the only words that must start at zero
// (the slice decode's per-(sequence, head) tickets) are cleared on the call's
// stream before its kernel runs, and every other word is written before it
// is read.
static __device__ __align__(256) char g_decode_scratch[ANCHORKV_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
char* g_scratch_ptr[kMaxDevices];   // device address of g_decode_scratch, per device

// Device address of the scratch array on the current device, looked up once
// per device (the first call on a device does this with that device current).
int scratch_on_current_device(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ANCHORKV_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return ANCHORKV_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return ANCHORKV_ECUDA;
    g_scratch_ptr[dev] = static_cast<char*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return ANCHORKV_OK;
}

int device_is_sm100() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ANCHORKV_ECUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return ANCHORKV_ECUDA;
  return major == 10 ? ANCHORKV_OK : ANCHORKV_EUNSUPPORTED;
}

}  // namespace
}  // namespace akv

using namespace akv;

extern "C" {

int anchorkv_decode_attn_noalloc(const anchorkv_params* p, const void* compressed, int64_t seq_stride_bytes,
                                 int32_t batch, const void* q, const void* K_tail, const void* V_tail,
                                 int32_t tail_len, int32_t tail_cap, float* out, void* stream) {
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
  if (((uintptr_t)compressed | (uintptr_t)q | (uintptr_t)out | (uintptr_t)K_tail | (uintptr_t)V_tail) & 15)
    return ANCHORKV_EINVAL;
  DecodePlan dp;
  make_decode_plan(pl, batch, &dp);
  // the key-logit pre-pass needs batch x R x G floats of scratch: without it
  // if the array cannot hold them (the decode computes those logits itself)
  if (dp.ws_total > (int64_t)ANCHORKV_DECODE_NOALLOC_SCRATCH_BYTES) make_decode_plan(pl, batch, &dp, false);
  if (dp.ws_total > (int64_t)ANCHORKV_DECODE_NOALLOC_SCRATCH_BYTES) return ANCHORKV_ENOSPC;
  st = check_decode_shape(pl, dp, tail_len);
  if (st) return st;
  st = device_is_sm100();
  if (st) return st;
  char* scratch = nullptr;
  st = scratch_on_current_device(&scratch);
  if (st) return st;
  return launch_decode(pl, dp, (const char*)compressed, seq_stride_bytes, q, K_tail, V_tail, tail_len, tail_cap, out,
                       scratch, (cudaStream_t)stream);
}

}  // extern "C"
