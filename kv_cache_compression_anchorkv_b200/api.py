"""Thin PyTorch binding of the AnchorKV C ABI.

PyTorch supplies device memory and the current CUDA stream; every step of the
codec runs in libanchorkv.so.  Functions mirror the C entry points:
``anchorkv_bytes``, ``compress`` (anchorkv_compress), ``decode_attn``
(anchorkv_decode_attn), ``reconstruct`` (anchorkv_reconstruct).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import capi

_DT = {"fp32": capi.FP32, "bf16": capi.BF16}

# anchorkv_params.mode bits (include/anchorkv.h)
MODE_KEY_QUERIES = 0x1       # Q_obs may be None: the trailing W keys serve as the observation queries
MODE_RANK_SHIFT = 1
RANK_UTILITY, RANK_RESIDUAL_NORM, RANK_ATTENTION, RANK_COSINE, RANK_RANDOM = 0, 1, 2, 3, 4
MODE_NAIVE_CODEC = 0x10      # 2-bit codec without the sign flip and Hadamard rotation


def mode_bits(key_queries: bool = False, rank: int = RANK_UTILITY, naive_codec: bool = False) -> int:
    """The anchorkv_params.mode value of a combination of options."""
    return (MODE_KEY_QUERIES if key_queries else 0) | (rank << MODE_RANK_SHIFT) | (MODE_NAIVE_CODEC if naive_codec else 0)
_TORCH_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class AnchorKVParams:
    """One layer's codec parameters (defaults: the pages' hyper-parameters)."""
    n_tokens: int
    n_kv_heads: int = 8
    n_q_heads: int = 32
    theta: float = 0.05
    head_dim: int = 128
    window: int = 32
    dtype: str = "bf16"
    seed: int = 0
    layer: int = 0
    anchor_div: int = 128
    rho_num: int = 7
    rho_den: int = 10
    pool_kernel: int = 7
    mode: int = 0                # mode_bits(...); compress and decode of one layout use the same

    def c(self) -> capi.Params:
        return capi.Params(self.n_tokens, self.head_dim, self.n_kv_heads, self.n_q_heads, self.window,
                           _DT[self.dtype], float(self.theta), self.seed, self.layer, self.anchor_div,
                           self.rho_num, self.rho_den, self.pool_kernel, self.mode)

    @property
    def torch_dtype(self) -> torch.dtype:
        return _TORCH_DT[self.dtype]


def anchorkv_bytes(p: AnchorKVParams) -> dict:
    L = capi.Layout()
    capi.check("anchorkv_bytes", capi.lib().anchorkv_bytes(ctypes.byref(p.c()), ctypes.byref(L)))
    return {name: getattr(L, name) for name, _ in capi.Layout._fields_}


def compress_workspace(p: AnchorKVParams) -> dict:
    v = capi.WorkspaceView()
    capi.check("anchorkv_compress_workspace",
               capi.lib().anchorkv_compress_workspace(ctypes.byref(p.c()), ctypes.byref(v)))
    return {name: getattr(v, name) for name, _ in capi.WorkspaceView._fields_}


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _check_tensor(name, t, shape, dtype):
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def compress(p: AnchorKVParams, K: torch.Tensor, V: torch.Tensor, Q_obs: torch.Tensor | None,
             out: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Compress one layer.  K, V: [H, N, D]; Q_obs: [H_q, W, D] (CUDA, p.dtype),
    or None with the key-as-query mode.
    Returns (compressed uint8 tensor of layout.total_bytes, workspace)."""
    H, N, D, W = p.n_kv_heads, p.n_tokens, p.head_dim, p.window
    _check_tensor("K", K, (H, N, D), p.torch_dtype)
    _check_tensor("V", V, (H, N, D), p.torch_dtype)
    if Q_obs is not None or not (p.mode & MODE_KEY_QUERIES):
        _check_tensor("Q_obs", Q_obs, (p.n_q_heads, W, D), p.torch_dtype)
    L = anchorkv_bytes(p)
    ws = compress_workspace(p)
    if out is None:
        out = torch.empty(L["total_bytes"], dtype=torch.uint8, device=K.device)
    if workspace is None:
        workspace = torch.empty(ws["total_bytes"], dtype=torch.uint8, device=K.device)
    st = capi.lib().anchorkv_compress(ctypes.byref(p.c()), _ptr(K), _ptr(V), _ptr(Q_obs), _ptr(out),
                                      out.numel(), _ptr(workspace), workspace.numel(), _stream(K.device))
    capi.check("anchorkv_compress", st)
    return out, workspace


def compress_host_staging_bytes(p: AnchorKVParams) -> int:
    """Device staging bytes compress_host needs (K, V, Q_obs and the layout)."""
    n = ctypes.c_size_t()
    capi.check("anchorkv_compress_host_staging_bytes",
               capi.lib().anchorkv_compress_host_staging_bytes(ctypes.byref(p.c()), ctypes.byref(n)))
    return n.value


def _check_host(name, t, shape, dtype):
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def compress_host(p: AnchorKVParams, K: torch.Tensor, V: torch.Tensor, Q_obs: torch.Tensor | None,
                  out: torch.Tensor, staging: torch.Tensor, workspace: torch.Tensor, device="cuda") -> torch.Tensor:
    """Compress one layer from host buffers through anchorkv_compress_host: the
    library copies K, V, Q_obs (host, ideally pinned) into `staging` (device),
    compresses there and copies the layout into `out` (host uint8), all on the
    current stream of `device`.  `out` is valid once that stream has run."""
    H, N, D, W = p.n_kv_heads, p.n_tokens, p.head_dim, p.window
    _check_host("K", K, (H, N, D), p.torch_dtype)
    _check_host("V", V, (H, N, D), p.torch_dtype)
    if Q_obs is not None or not (p.mode & MODE_KEY_QUERIES):
        _check_host("Q_obs", Q_obs, (p.n_q_heads, W, D), p.torch_dtype)
    if out.device.type != "cpu" or out.dtype != torch.uint8:
        raise ValueError("out must be a host uint8 tensor")
    st = capi.lib().anchorkv_compress_host(ctypes.byref(p.c()), _ptr(K), _ptr(V), _ptr(Q_obs), _ptr(out),
                                           out.numel(), _ptr(staging), staging.numel(), _ptr(workspace),
                                           workspace.numel(), _stream(torch.device(device)))
    capi.check("anchorkv_compress_host", st)
    return out


def decode_workspace_bytes(p: AnchorKVParams, batch: int) -> int:
    n = ctypes.c_size_t()
    capi.check("anchorkv_decode_workspace_bytes",
               capi.lib().anchorkv_decode_workspace_bytes(ctypes.byref(p.c()), batch, ctypes.byref(n)))
    return n.value


def decode_attn(p: AnchorKVParams, compressed: torch.Tensor, q: torch.Tensor,
                K_tail: torch.Tensor | None = None, V_tail: torch.Tensor | None = None, tail_len: int = 0,
                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Decode attention.  compressed: uint8 [batch, stride] (one layout per
    row) or [total_bytes]; q: [batch, H_q, D]; tails [batch, H, T_cap, D].
    Returns fp32 [batch, H_q, D]."""
    if compressed.dim() == 1:
        # one layout: the stride never steps to a second sequence, it only has
        # to satisfy the ABI (>= total bytes, a multiple of 16)
        batch, stride = 1, (compressed.numel() + 15) // 16 * 16
    else:
        batch, stride = compressed.shape
    _check_tensor("q", q, (batch, p.n_q_heads, p.head_dim), p.torch_dtype)
    cap = 0
    if K_tail is not None:
        cap = K_tail.shape[2]
        _check_tensor("K_tail", K_tail, (batch, p.n_kv_heads, cap, p.head_dim), p.torch_dtype)
        _check_tensor("V_tail", V_tail, (batch, p.n_kv_heads, cap, p.head_dim), p.torch_dtype)
    if out is None:
        out = torch.empty(batch, p.n_q_heads, p.head_dim, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(p, batch), dtype=torch.uint8, device=q.device)
    st = capi.lib().anchorkv_decode_attn(ctypes.byref(p.c()), _ptr(compressed), stride, batch, _ptr(q),
                                         _ptr(K_tail), _ptr(V_tail), tail_len, cap, _ptr(out), _ptr(workspace),
                                         workspace.numel(), _stream(q.device))
    capi.check("anchorkv_decode_attn", st)
    return out


def decode_rope_workspace_bytes(p: AnchorKVParams, batch: int) -> int:
    n = ctypes.c_size_t()
    capi.check("anchorkv_decode_rope_workspace_bytes",
               capi.lib().anchorkv_decode_rope_workspace_bytes(ctypes.byref(p.c()), batch, ctypes.byref(n)))
    return n.value


def decode_attn_rope(p: AnchorKVParams, compressed: torch.Tensor, q: torch.Tensor, rope_base: float,
                     K_tail: torch.Tensor | None = None, V_tail: torch.Tensor | None = None, tail_len: int = 0,
                     out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Decode attention over layouts whose keys were stored before the rotary
    map (anchorkv_decode_attn_rope): cached token t at position t, tail token
    i at N + i, the query at N + tail_len.  Shapes as decode_attn."""
    if compressed.dim() == 1:
        batch, stride = 1, (compressed.numel() + 15) // 16 * 16
    else:
        batch, stride = compressed.shape
    _check_tensor("q", q, (batch, p.n_q_heads, p.head_dim), p.torch_dtype)
    cap = 0
    if K_tail is not None:
        cap = K_tail.shape[2]
        _check_tensor("K_tail", K_tail, (batch, p.n_kv_heads, cap, p.head_dim), p.torch_dtype)
        _check_tensor("V_tail", V_tail, (batch, p.n_kv_heads, cap, p.head_dim), p.torch_dtype)
    if out is None:
        out = torch.empty(batch, p.n_q_heads, p.head_dim, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(decode_rope_workspace_bytes(p, batch), dtype=torch.uint8, device=q.device)
    st = capi.lib().anchorkv_decode_attn_rope(ctypes.byref(p.c()), _ptr(compressed), stride, batch, _ptr(q),
                                              _ptr(K_tail), _ptr(V_tail), tail_len, cap, float(rope_base),
                                              _ptr(out), _ptr(workspace), workspace.numel(), _stream(q.device))
    capi.check("anchorkv_decode_attn_rope", st)
    return out


def decode_config(p: AnchorKVParams, batch: int) -> dict:
    """Launch shape of decode_attn on the current device: token slices (CTAs)
    per (sequence, head) of the slice decode (0: the split-token kernels run)
    and shared memory per CTA."""
    c, m = ctypes.c_int32(), ctypes.c_int32()
    capi.check("anchorkv_decode_config",
               capi.lib().anchorkv_decode_config(ctypes.byref(p.c()), batch, ctypes.byref(c), ctypes.byref(m)))
    return {"slices": c.value, "smem_bytes": m.value}


NOALLOC_SCRATCH_BYTES = 32 << 20   # ANCHORKV_DECODE_NOALLOC_SCRATCH_BYTES in include/anchorkv.h


def decode_attn_noalloc(p: AnchorKVParams, compressed: torch.Tensor, q: torch.Tensor, out: torch.Tensor,
                        K_tail: torch.Tensor | None = None, V_tail: torch.Tensor | None = None,
                        tail_len: int = 0) -> torch.Tensor:
    """Decode attention that allocates no device memory: the library's
    per-device scratch array stands in for the workspace, and `out` must be
    supplied.  For callers that cannot allocate while decoding (all free HBM
    given to a KV-cache pool, no device allocator, or no room for the
    device-wide synchronisation of cudaMalloc/cudaFree).  Calls that overlap
    on the GPU share the scratch and race; sizes whose decode workspace
    exceeds NOALLOC_SCRATCH_BYTES raise (ANCHORKV_ENOSPC)."""
    if compressed.dim() == 1:
        # one layout: the stride never steps to a second sequence, it only has
        # to satisfy the ABI (>= total bytes, a multiple of 16)
        batch, stride = 1, (compressed.numel() + 15) // 16 * 16
    else:
        batch, stride = compressed.shape
    _check_tensor("q", q, (batch, p.n_q_heads, p.head_dim), p.torch_dtype)
    _check_tensor("out", out, (batch, p.n_q_heads, p.head_dim), torch.float32)
    cap = 0
    if K_tail is not None:
        cap = K_tail.shape[2]
        _check_tensor("K_tail", K_tail, (batch, p.n_kv_heads, cap, p.head_dim), p.torch_dtype)
        _check_tensor("V_tail", V_tail, (batch, p.n_kv_heads, cap, p.head_dim), p.torch_dtype)
    st = capi.lib().anchorkv_decode_attn_noalloc(ctypes.byref(p.c()), _ptr(compressed), stride, batch, _ptr(q),
                                                 _ptr(K_tail), _ptr(V_tail), tail_len, cap, _ptr(out),
                                                 _stream(q.device))
    if st == capi.ENOSPC:
        raise capi.AnchorKVError(
            f"anchorkv_decode_attn_noalloc (decode workspace {decode_workspace_bytes(p, batch)} B exceeds the "
            f"{NOALLOC_SCRATCH_BYTES} B static scratch)", st)
    capi.check("anchorkv_decode_attn_noalloc", st)
    return out


def reconstruct(p: AnchorKVParams, compressed: torch.Tensor):
    """Dense fp32 K^, V^ [H, N, D] of one compressed layer (inspection hook)."""
    H, N, D = p.n_kv_heads, p.n_tokens, p.head_dim
    Kh = torch.empty(H, N, D, dtype=torch.float32, device=compressed.device)
    Vh = torch.empty_like(Kh)
    st = capi.lib().anchorkv_reconstruct(ctypes.byref(p.c()), _ptr(compressed), _ptr(Kh), _ptr(Vh),
                                         _stream(compressed.device))
    capi.check("anchorkv_reconstruct", st)
    return Kh, Vh


# device status word values (the first kernel to fail latches its code)
DEVICE_ERRORS = {1: "uniform anchor sample", 2: "refine list", 3: "inconsistent record or selection (bounds)",
                 4: "bounded wait timed out"}


def read_status(workspace: torch.Tensor) -> list[int]:
    """Device status word and counters of a compress workspace (synchronises
    the current stream).  Raises if a device-side check failed, naming it."""
    buf = (ctypes.c_int32 * 16)()
    st = capi.lib().anchorkv_read_device_status(_ptr(workspace), buf, _stream(workspace.device))
    vals = list(buf)
    if st == capi.EDEVICE:
        raise capi.AnchorKVError("anchorkv_read_device_status", st,
                                 f"status word {vals[0]} ({DEVICE_ERRORS.get(vals[0], 'unknown')})")
    capi.check("anchorkv_read_device_status", st)
    return vals


def codebook() -> tuple[float, float, float, float]:
    out = (ctypes.c_double * 4)()
    capi.check("anchorkv_codebook", capi.lib().anchorkv_codebook(out))
    return tuple(out)


class HostCompressor:
    """End-to-end compress from host (pinned) buffers through the C ABI's
    anchorkv_compress_host: per call, the library copies the layer's K, V,
    Q_obs into a preallocated device staging buffer, compresses there and
    copies the compressed bytes back into a pinned host buffer, all on the
    current stream.  Allocation happens once, in the constructor; `out` is a
    device view of the staged layout."""

    def __init__(self, p: AnchorKVParams, device="cuda"):
        self.p = p
        self.device = torch.device(device)
        L = anchorkv_bytes(p)
        self.staging = torch.empty(compress_host_staging_bytes(p), dtype=torch.uint8, device=device)
        self.ws = torch.empty(compress_workspace(p)["total_bytes"], dtype=torch.uint8, device=device)
        self.host_out = torch.empty(L["total_bytes"], dtype=torch.uint8, pin_memory=True)
        # the staged layout: the staging buffer's last section (256-byte aligned)
        self.out = self.staging[-((L["total_bytes"] + 255) // 256 * 256):][:L["total_bytes"]]

    def __call__(self, K_host, V_host, Q_host, layer: int | None = None, host_out: torch.Tensor | None = None):
        """Compress one layer; the compressed bytes land in `host_out` (pinned,
        total_bytes) or in the compressor's own pinned buffer.  Several
        compressors on different streams overlap the copies of one layer with
        the compression of another."""
        if layer is not None:
            self.p.layer = layer
        dst = self.host_out if host_out is None else host_out
        return compress_host(self.p, K_host, V_host, Q_host, dst, self.staging, self.ws, device=self.device)


N_STAGES = 16   # ANCHORKV_N_STAGES


def stage_timing(enable: bool) -> None:
    """Turn the library's per-stage CUDA-event timing on (clearing it) or off."""
    capi.check("anchorkv_stage_timing", capi.lib().anchorkv_stage_timing(1 if enable else 0))


def stage_times() -> dict:
    """{stage name: (total ms, timed calls)} since the last stage_timing(True)."""
    ms = (ctypes.c_double * N_STAGES)()
    calls = (ctypes.c_int64 * N_STAGES)()
    capi.check("anchorkv_stage_times", capi.lib().anchorkv_stage_times(ms, calls, N_STAGES))
    return {capi.lib().anchorkv_stage_name(i).decode(): (ms[i], calls[i]) for i in range(N_STAGES)}


def launch_count() -> int:
    n = ctypes.c_int64()
    capi.check("anchorkv_launch_count", capi.lib().anchorkv_launch_count(ctypes.byref(n)))
    return n.value
