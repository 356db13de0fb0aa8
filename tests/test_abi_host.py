"""The C-ABI library loads, exports what include/anchorkv.h declares, and its
host-side (pure) functions agree with the oracle.  No GPU needed."""
import ctypes
import math

import pytest

from kv_cache_compression_anchorkv_b200 import api, capi
from oracle import anchorkv_oracle as O


def test_library_exports_every_declared_symbol():
    L = capi.lib()
    names = capi.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(capi._SIGS), "binding and header disagree"


def test_struct_sizes_match_header_layout():
    assert ctypes.sizeof(capi.Params) == 4 * 6 + 8 + 8 + 4 * 6
    assert ctypes.sizeof(capi.Layout) == 8 * 7 + 4 * 4 + 8 * 8
    assert ctypes.sizeof(capi.WorkspaceView) == 8 * 5


CASES = [
    (1024, 1, 4, 0.1, "fp32"), (32768, 8, 32, 0.05, "bf16"), (131072, 8, 64, 0.05, "bf16"),
    (32768, 8, 32, 0.1, "bf16"), (8192, 8, 32, 0.2, "bf16"), (3000, 2, 8, 0.1, "bf16"),
    (33, 1, 2, 0.5, "bf16"), (256, 1, 4, 0.05, "bf16"), (777, 2, 4, 1.0, "fp32"), (5000, 3, 6, 0.07, "bf16"),
]


@pytest.mark.parametrize("N,H,Hq,theta,dtype", CASES)
def test_byte_accounting_matches_oracle(N, H, Hq, theta, dtype):
    p = api.AnchorKVParams(n_tokens=N, n_kv_heads=H, n_q_heads=Hq, theta=theta, dtype=dtype)
    got = api.anchorkv_bytes(p)
    want = O.layout(O.Params(n_tokens=N, n_kv_heads=H, n_q_heads=Hq, theta=theta, dtype=dtype))
    assert got["total_bytes"] == want["total"]
    assert got["base_bytes"] == want["base"]
    assert got["budget_bytes"] == want["B"]
    assert got["n_residuals"] == want["R"]
    assert got["residual_cap"] == want["cap"]
    assert got["n_anchors"] == want["k"]
    assert got["n_scored"] == want["n_s"] and got["n_uniform"] == want["n_u"]
    for name, off in want["off"].items():
        assert got["off_" + name.lower()] == off, name


@pytest.mark.parametrize("field,value", [
    ("head_dim", 64), ("n_kv_heads", 0), ("n_q_heads", 12), ("window", 0), ("n_tokens", 32),
    ("theta", 0.0), ("theta", float("nan")), ("theta", -1.0), ("pool_kernel", 6), ("rho_num", 11),
    ("layer", -1), ("anchor_div", 0), ("mode", 0x20), ("mode", api.mode_bits(rank=5)),
    ("mode", api.mode_bits(rank=7)), ("mode", -1)])
def test_invalid_params_rejected(field, value):
    p = api.AnchorKVParams(n_tokens=1024, n_kv_heads=8, n_q_heads=32)
    setattr(p, field, value)
    with pytest.raises(capi.AnchorKVError) as e:
        api.anchorkv_bytes(p)
    assert e.value.status in (capi.EINVAL, capi.EUNSUPPORTED)


def test_null_arguments_are_errors_not_crashes():
    L = capi.lib()
    assert L.anchorkv_bytes(None, None) == capi.EINVAL
    p = api.AnchorKVParams(n_tokens=1024).c()
    assert L.anchorkv_compress(ctypes.byref(p), None, None, None, None, 0, None, 0, None) == capi.EINVAL
    n = ctypes.c_size_t()
    assert L.anchorkv_decode_workspace_bytes(ctypes.byref(p), -1, ctypes.byref(n)) == capi.EINVAL
    assert L.anchorkv_read_device_status(None, None, None) == capi.EINVAL
    assert L.anchorkv_compress_host(ctypes.byref(p), None, None, None, None, 0, None, 0, None, 0, None) == capi.EINVAL
    assert L.anchorkv_compress_host_staging_bytes(ctypes.byref(p), None) == capi.EINVAL
    assert L.anchorkv_strerror(capi.ENOSPC) == b"buffer too small"


def test_small_output_buffer_is_enospc():
    L = capi.lib()
    p = api.AnchorKVParams(n_tokens=1024).c()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: size check fails first
    st = L.anchorkv_compress(ctypes.byref(p), fake, fake, fake, fake, 16, fake, 16, None)
    assert st == capi.ENOSPC


def test_host_compress_staging_and_checks():
    """The host-buffer compress: its staging size is K, V, Q_obs and the layout,
    each rounded up to 256 bytes, and a small staging or output buffer is
    refused before any copy (the fake pointers are never dereferenced)."""
    L = capi.lib()
    pp = api.AnchorKVParams(n_tokens=1000)
    n = api.compress_host_staging_bytes(pp)
    al = lambda x: (x + 255) // 256 * 256
    kv = pp.n_kv_heads * pp.n_tokens * pp.head_dim * 2
    q = pp.n_q_heads * pp.window * pp.head_dim * 2
    total = api.anchorkv_bytes(pp)["total_bytes"]
    assert n == 2 * al(kv) + al(q) + al(total)
    p = pp.c()
    fake = ctypes.c_void_p(1 << 20)
    assert L.anchorkv_compress_host(ctypes.byref(p), fake, fake, fake, fake, total, fake, n - 1, fake, 1 << 40,
                                    None) == capi.ENOSPC
    assert L.anchorkv_compress_host(ctypes.byref(p), fake, fake, fake, fake, total - 1, fake, n, fake, 1 << 40,
                                    None) == capi.ENOSPC
    misaligned = ctypes.c_void_p((1 << 20) + 8)
    assert L.anchorkv_compress_host(ctypes.byref(p), fake, fake, fake, fake, total, misaligned, n, fake, 1 << 40,
                                    None) == capi.EINVAL


def test_library_codebook_matches_oracle():
    tau, l1, l2, mse = api.codebook()
    o = O.lloyd_max_gaussian_4()
    for a, b in zip((tau, l1, l2, mse), o):
        assert abs(a - b) < 1e-13


def test_workspace_view(monkeypatch):
    p = api.AnchorKVParams(n_tokens=32768)
    v = api.compress_workspace(p)
    assert v["total_bytes"] > v["off_utility"] + 4 * 2 * 8 * 32768
    assert v["off_counters"] % 256 == 0 and v["off_pooled"] % 256 == 0
    # the slice decode needs tickets and slice partials only when a (sequence,
    # head) is cut into several slices: at batch 1 (8 heads on ~148 CTAs) it
    # is, at batch 32 (256 heads) every head is one slice; every shape needs
    # the anchor logits P (batch x H x k x G floats), and the key-logit
    # pre-pass's batch x R x G floats when it runs (by default at batch 32)
    assert api.decode_workspace_bytes(p, 1) > 0
    R = api.anchorkv_bytes(p)["n_residuals"]
    P32 = (32 * 8 * 288 * 4 * 4 + 255) // 256 * 256
    assert api.decode_workspace_bytes(p, 32) == (32 * R * 4 * 4 + 255) // 256 * 256 + P32
    monkeypatch.setenv("ANCHORKV_DECODE_KLOGIT", "0")
    assert api.decode_workspace_bytes(p, 32) == P32
    monkeypatch.setenv("ANCHORKV_DECODE_KLOGIT", "1")
    assert api.decode_workspace_bytes(p, 1) > (R * 4 * 4 + 255) // 256 * 256
    monkeypatch.delenv("ANCHORKV_DECODE_KLOGIT")
    # 16 query heads per KV head with 1056 anchors do not fit the slice
    # decode's shared memory: the split-token kernels and their workspace
    p16 = api.AnchorKVParams(n_tokens=131072, n_q_heads=128)
    assert api.decode_workspace_bytes(p16, 16) > api.decode_workspace_bytes(p16, 1) > 0


def test_misaligned_tails_rejected_before_any_launch():
    """K_tail / V_tail are read with 16-byte vector loads: a tail pointer off
    a 16-byte boundary is EINVAL on the host, for the workspace and the
    no-alloc entry points alike (placeholder pointers, never dereferenced)."""
    L = capi.lib()
    p = api.AnchorKVParams(n_tokens=1024).c()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 21) + 2)
    for kt, vt in ((odd, fake), (fake, odd)):
        assert L.anchorkv_decode_attn(ctypes.byref(p), fake, 1 << 20, 1, fake, kt, vt, 4, 8, fake, fake,
                                      1 << 30, None) == capi.EINVAL
        assert L.anchorkv_decode_attn_noalloc(ctypes.byref(p), fake, 1 << 20, 1, fake, kt, vt, 4, 8, fake,
                                              None) == capi.EINVAL


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    import bench
    # the committed record matches the committed kernel source
    assert bench.recorded_traffic("assign") is None or bench.recorded_traffic("assign") > 0
    assert bench.recorded_traffic("no_such_stage") is None
    # a record whose hash does not match its source reads as unknown
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text("kernel v2\n")
    (tmp_path / "profiles" / "traffic.txt").write_text("stage_x kern 123 k.cu " + "0" * 64 + " cap.md\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("stage_x") is None
    import hashlib
    h = hashlib.sha256(b"kernel v2\n").hexdigest()
    (tmp_path / "profiles" / "traffic.txt").write_text(f"stage_x kern 123 k.cu {h} cap.md\n")
    assert bench.recorded_traffic("stage_x") == 123


def test_mode_bits_match_header():
    text = open(capi.HEADER).read()
    for name, val in [("ANCHORKV_MODE_KEY_QUERIES", api.MODE_KEY_QUERIES), ("ANCHORKV_MODE_NAIVE_CODEC", api.MODE_NAIVE_CODEC),
                      ("ANCHORKV_MODE_RANK_SHIFT", api.MODE_RANK_SHIFT)]:
        assert f"#define {name} {val:#x}" in text or f"#define {name} {val}" in text, name
    for name, val in [("ANCHORKV_RANK_RESIDUAL_NORM", api.RANK_RESIDUAL_NORM), ("ANCHORKV_RANK_ATTENTION", api.RANK_ATTENTION),
                      ("ANCHORKV_RANK_COSINE", api.RANK_COSINE), ("ANCHORKV_RANK_RANDOM", api.RANK_RANDOM)]:
        assert f"{name} = {val}" in text, name
    assert api.mode_bits(True, api.RANK_RANDOM, True) == 0x1 | (4 << 1) | 0x10
    assert api.mode_bits(True, api.RANK_RANDOM, True) == O.MODE_KEY_QUERIES | (O.RANK_RANDOM << O.MODE_RANK_SHIFT) | O.MODE_NAIVE_CODEC


def test_every_valid_mode_is_accepted():
    for mode in range(0x20):
        p = api.AnchorKVParams(n_tokens=1024, mode=mode)
        rank = (mode >> 1) & 7
        if rank > api.RANK_RANDOM:
            with pytest.raises(capi.AnchorKVError):
                api.anchorkv_bytes(p)
        else:
            assert api.anchorkv_bytes(p)["total_bytes"] > 0


def test_queries_are_optional_only_with_key_queries():
    """Q_obs = NULL is EINVAL unless the key-as-query mode is set; then the
    proxy queries take workspace (size check first: never dereferenced)."""
    L = capi.lib()
    fake = ctypes.c_void_p(1 << 20)
    p = api.AnchorKVParams(n_tokens=1024).c()
    assert L.anchorkv_compress(ctypes.byref(p), fake, fake, None, fake, 1 << 40, fake, 1 << 40, None) == capi.EINVAL
    pk = api.AnchorKVParams(n_tokens=1024, mode=api.MODE_KEY_QUERIES)
    assert L.anchorkv_compress(ctypes.byref(pk.c()), fake, fake, None, fake, 16, fake, 16, None) == capi.ENOSPC
    base = api.compress_workspace(api.AnchorKVParams(n_tokens=1024))["total_bytes"]
    assert api.compress_workspace(pk)["total_bytes"] >= base + 32 * 32 * 128 * 2


def test_rope_decode_arguments_checked_on_the_host():
    L = capi.lib()
    p = api.AnchorKVParams(n_tokens=1024).c()
    fake = ctypes.c_void_p(1 << 20)
    n = ctypes.c_size_t()
    assert L.anchorkv_decode_rope_workspace_bytes(ctypes.byref(p), 4, ctypes.byref(n)) == capi.OK and n.value > 0
    for base in (1.0, 0.5, float("nan"), float("inf")):
        assert L.anchorkv_decode_attn_rope(ctypes.byref(p), fake, 1 << 20, 1, fake, None, None, 0, 0, base,
                                           fake, fake, 1 << 30, None) == capi.EINVAL
    assert L.anchorkv_decode_attn_rope(ctypes.byref(p), fake, 1 << 20, 1, fake, None, None, 0, 0, 10000.0,
                                       fake, fake, 16, None) == capi.ENOSPC
    # (sequence, head) pairs beyond one grid dimension
    assert L.anchorkv_decode_attn_rope(ctypes.byref(p), fake, 1 << 24, 10000, fake, None, None, 0, 0, 10000.0,
                                       fake, fake, 1 << 40, None) == capi.EUNSUPPORTED


def test_split_token_decode_grid_limit_on_the_host():
    """The split-token decode (more than 8 query heads per KV head) puts
    batch x H (sequence, head) pairs in one grid dimension: beyond 65535 it
    is refused before any launch."""
    L = capi.lib()
    p = api.AnchorKVParams(n_tokens=1024, n_kv_heads=8, n_q_heads=128).c()
    fake = ctypes.c_void_p(1 << 20)
    n = ctypes.c_size_t()
    assert L.anchorkv_decode_workspace_bytes(ctypes.byref(p), 9000, ctypes.byref(n)) == capi.OK
    st = L.anchorkv_decode_attn(ctypes.byref(p), fake, 1 << 24, 9000, fake, None, None, 0, 0, fake, fake,
                                n.value, None)
    assert st == capi.EUNSUPPORTED
