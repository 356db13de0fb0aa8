"""ctypes declarations of the C ABI in include/anchorkv.h (argument
marshalling only: every step of the codec runs in the CUDA library)."""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libanchorkv.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "anchorkv.h")

OK, EINVAL, ENOSPC, EUNSUPPORTED, ECUDA, EDEVICE = 0, -1, -2, -3, -4, -5
FP32, BF16 = 0, 1


class Params(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("window", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("theta", ctypes.c_double), ("seed", ctypes.c_uint64), ("layer", ctypes.c_int32),
        ("anchor_div", ctypes.c_int32), ("rho_num", ctypes.c_int32), ("rho_den", ctypes.c_int32),
        ("pool_kernel", ctypes.c_int32), ("mode", ctypes.c_int32),
    ]


class Layout(ctypes.Structure):
    _fields_ = [
        ("total_bytes", ctypes.c_int64), ("base_bytes", ctypes.c_int64), ("budget_bytes", ctypes.c_int64),
        ("uncompressed_bytes", ctypes.c_int64), ("n_residuals", ctypes.c_int64),
        ("residual_cap", ctypes.c_int64), ("residual_bytes_each", ctypes.c_int64),
        ("n_anchors", ctypes.c_int32), ("n_scored", ctypes.c_int32), ("n_uniform", ctypes.c_int32),
        ("n_tiles", ctypes.c_int32),
        ("off_anchors_k", ctypes.c_int64), ("off_anchors_v", ctypes.c_int64), ("off_anchor_pos", ctypes.c_int64),
        ("off_tok", ctypes.c_int64), ("off_bitmap", ctypes.c_int64), ("off_tile_prefix", ctypes.c_int64),
        ("off_res_codes", ctypes.c_int64), ("off_res_sigma", ctypes.c_int64),
    ]


class WorkspaceView(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_int64), ("off_pooled", ctypes.c_int64),
                ("off_utility", ctypes.c_int64), ("off_counters", ctypes.c_int64),
                ("off_assign_probe", ctypes.c_int64)]


_P = ctypes.POINTER
_vp = ctypes.c_void_p
_SIGS = {
    "anchorkv_default_params": ([_P(Params)], ctypes.c_int),
    "anchorkv_bytes": ([_P(Params), _P(Layout)], ctypes.c_int),
    "anchorkv_compress_workspace": ([_P(Params), _P(WorkspaceView)], ctypes.c_int),
    "anchorkv_compress": ([_P(Params), _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "anchorkv_compress_host_staging_bytes": ([_P(Params), _P(ctypes.c_size_t)], ctypes.c_int),
    "anchorkv_compress_host": ([_P(Params), _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, ctypes.c_size_t, _vp,
                                ctypes.c_size_t, _vp], ctypes.c_int),
    "anchorkv_decode_workspace_bytes": ([_P(Params), ctypes.c_int32, _P(ctypes.c_size_t)], ctypes.c_int),
    "anchorkv_decode_attn": ([_P(Params), _vp, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp, ctypes.c_int32,
                              ctypes.c_int32, _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "anchorkv_decode_attn_noalloc": ([_P(Params), _vp, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp,
                                      ctypes.c_int32, ctypes.c_int32, _vp, _vp], ctypes.c_int),
    "anchorkv_decode_config": ([_P(Params), ctypes.c_int32, _P(ctypes.c_int32), _P(ctypes.c_int32)], ctypes.c_int),
    "anchorkv_decode_rope_workspace_bytes": ([_P(Params), ctypes.c_int32, _P(ctypes.c_size_t)], ctypes.c_int),
    "anchorkv_decode_attn_rope": ([_P(Params), _vp, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp, ctypes.c_int32,
                                   ctypes.c_int32, ctypes.c_double, _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "anchorkv_reconstruct": ([_P(Params), _vp, _vp, _vp, _vp], ctypes.c_int),
    "anchorkv_read_device_status": ([_vp, _P(ctypes.c_int32), _vp], ctypes.c_int),
    "anchorkv_codebook": ([_P(ctypes.c_double)], ctypes.c_int),
    "anchorkv_strerror": ([ctypes.c_int], ctypes.c_char_p),
    "anchorkv_stage_timing": ([ctypes.c_int], ctypes.c_int),
    "anchorkv_stage_times": ([_P(ctypes.c_double), _P(ctypes.c_int64), ctypes.c_int32], ctypes.c_int),
    "anchorkv_stage_name": ([ctypes.c_int32], ctypes.c_char_p),
    "anchorkv_launch_count": ([_P(ctypes.c_int64)], ctypes.c_int),
}

_lib = None


class AnchorKVError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str | None = None):
        msg = _lib.anchorkv_strerror(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {msg} ({status})" + (f": {detail}" if detail else ""))
        self.status = status
        self.detail = detail


def header_functions() -> list[str]:
    """Names of the functions include/anchorkv.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^(?:int|const char\*)\s+(anchorkv_\w+)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """The CUDA library.  Raises if it has not been built: there is no other
    implementation of the codec in this package."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m kv_cache_compression_anchorkv_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def check(fn: str, status: int) -> None:
    if status != OK:
        raise AnchorKVError(fn, status)
