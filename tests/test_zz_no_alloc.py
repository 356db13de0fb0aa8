"""anchorkv_decode_attn_noalloc (library-owned scratch, no workspace argument)
against anchorkv_decode_attn (caller workspace), both through the C ABI.

The file is collected last, so that a run stopping at the first failure has
already run every other test, and so that in a full run its calls find the
shared scratch holding whatever earlier decode calls left in it.  Run on its
own (pytest tests/test_zz_no_alloc.py), its first call is the one that looks
up the scratch array's device address.
"""
import ctypes

import pytest
import torch

from kv_cache_compression_anchorkv_b200 import api, capi
from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_decode_queries, make_layer, make_tail

DECODE_TOL = {"bf16": 2e-3, "fp32": 1e-5}   # the decode tolerance of the parity tests


def _params(spec: CacheSpec, theta: float) -> api.AnchorKVParams:
    return api.AnchorKVParams(n_tokens=spec.n_tokens, n_kv_heads=spec.n_kv_heads, n_q_heads=spec.n_q_heads,
                              theta=theta, window=spec.window, dtype=spec.dtype, seed=spec.seed)


def _vp(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _compressed_batch(p: api.AnchorKVParams, spec: CacheSpec, batch: int):
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": spec.seed + 100 * b})
        K, V, Q = make_layer(sb, 0)
        out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
        comp[b, :L["total_bytes"]] = out
    return comp, stride


def _decode_both(p, comp, stride, q, Kt, Vt, tail_len):
    """(workspace entry point output, no-alloc entry point output)."""
    lib = capi.lib()
    batch = comp.shape[0]
    cap = Kt.shape[2]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ws_bytes = ctypes.c_size_t(0)
    capi.check("anchorkv_decode_workspace_bytes",
               lib.anchorkv_decode_workspace_bytes(ctypes.byref(p.c()), batch, ctypes.byref(ws_bytes)))
    ws = torch.empty(ws_bytes.value, dtype=torch.uint8, device="cuda")
    ref = torch.full((batch, p.n_q_heads, p.head_dim), float("nan"), dtype=torch.float32, device="cuda")
    got = torch.full_like(ref, float("nan"))
    capi.check("anchorkv_decode_attn",
               lib.anchorkv_decode_attn(ctypes.byref(p.c()), _vp(comp), stride, batch, _vp(q), _vp(Kt), _vp(Vt),
                                        tail_len, cap, _vp(ref), _vp(ws), ws_bytes.value, stream))
    capi.check("anchorkv_decode_attn_noalloc",
               lib.anchorkv_decode_attn_noalloc(ctypes.byref(p.c()), _vp(comp), stride, batch, _vp(q), _vp(Kt),
                                                _vp(Vt), tail_len, cap, _vp(got), stream))
    torch.cuda.synchronize()
    return ref, got


CASES = {
    "bf16-ragged-n3000-batch2": (CacheSpec(1, 2, 8, 3000, n_dirs=64, seed=11), 0.1, 2),
    "fp32-window8-n700-batch3": (CacheSpec(1, 3, 3, 700, window=8, dtype="fp32", n_dirs=8, seed=12), 0.3, 3),
    # 16 query heads per KV head: the decode path that uses the scratch
    "bf16-gqa16-n1500-batch2": (CacheSpec(1, 1, 16, 1500, n_dirs=32, seed=13), 0.2, 2),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point(name):
    spec, theta, batch = CASES[name]
    p = _params(spec, theta)
    comp, stride = _compressed_batch(p, spec, batch)
    tol = DECODE_TOL[spec.dtype]
    cap = 40
    Kt, Vt = (x.cuda() for x in make_tail(spec, 0, cap, batch=batch))
    # two calls in a row with different queries and tail lengths: the second
    # runs over the scratch contents the first left behind
    for step, tail_len in ((0, 37), (1, 5)):
        q = make_decode_queries(spec, 0, step=step, batch=batch).cuda()
        ref, got = _decode_both(p, comp, stride, q, Kt, Vt, tail_len)
        assert torch.isfinite(ref).all() and torch.isfinite(got).all()
        err = (got - ref).abs().max().item()
        assert err <= tol, f"call {step}: max abs difference {err} > {tol}"


def test_noalloc_rejects_sizes_beyond_the_scratch():
    """A decode workspace above the static maximum is refused with ENOSPC
    before any device work.  With a GPU the arguments are real device buffers
    of the right sizes (a zeroed layout batch, queries, output), so nothing
    could read out of bounds even if a launch happened; without one they are
    aligned placeholders that the size check turns away first."""
    p = api.AnchorKVParams(n_tokens=131072, n_kv_heads=8, n_q_heads=128)
    batch = 4
    assert api.decode_workspace_bytes(p, batch) > api.NOALLOC_SCRATCH_BYTES
    stride = (api.anchorkv_bytes(p)["total_bytes"] + 255) // 256 * 256
    if torch.cuda.is_available():
        comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
        q = torch.zeros(batch, p.n_q_heads, p.head_dim, dtype=torch.bfloat16, device="cuda")
        out = torch.zeros(batch, p.n_q_heads, p.head_dim, dtype=torch.float32, device="cuda")
        ptrs = (_vp(comp), _vp(q), _vp(out))
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    else:
        fake = ctypes.c_void_p(1 << 20)
        ptrs, stream = (fake, fake, fake), None
    st = capi.lib().anchorkv_decode_attn_noalloc(ctypes.byref(p.c()), ptrs[0], stride, batch, ptrs[1], None, None,
                                                 0, 0, ptrs[2], stream)
    assert st == capi.ENOSPC
    if torch.cuda.is_available():
        torch.cuda.synchronize()
        assert torch.count_nonzero(out).item() == 0     # nothing ran
