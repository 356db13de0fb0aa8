"""CUDA path vs the oracle, through the C ABI, on seeded synthetic caches."""
import numpy as np
import pytest
import torch

from kv_cache_compression_anchorkv_b200 import api, capi
from kv_cache_compression_anchorkv_b200.synthetic import (CacheSpec, make_decode_queries, make_layer,
                                                           make_tail)
from oracle import anchorkv_oracle as O
from tests import parity

pytestmark = pytest.mark.gpu

DECODE_TOL = {"bf16": 2e-3, "fp32": 1e-5}


def _params(spec: CacheSpec, theta, layer=0):
    return api.AnchorKVParams(n_tokens=spec.n_tokens, n_kv_heads=spec.n_kv_heads, n_q_heads=spec.n_q_heads,
                              theta=theta, window=spec.window, dtype=spec.dtype, seed=spec.seed, layer=layer)


def _f64(x):
    return x.detach().cpu().double().numpy()


CASES = {
    # name: (spec, theta)
    "tiny-fp32-n1024": (CacheSpec(1, 1, 4, 1024, dtype="fp32", n_dirs=32, seed=0), 0.1),
    "bf16-ragged-n3000": (CacheSpec(1, 2, 8, 3000, n_dirs=64, seed=1), 0.1),
    "bf16-gqa8-n2500": (CacheSpec(1, 2, 16, 2500, n_dirs=64, seed=2), 0.15),
    "bf16-every-residual": (CacheSpec(1, 1, 4, 1100, n_dirs=16, seed=3), 1.0),
    "bf16-no-residual": (CacheSpec(1, 2, 4, 1000, n_dirs=16, seed=4), 0.01),
    "fp32-all-anchors": (CacheSpec(1, 2, 4, 33, dtype="fp32", n_dirs=8, seed=5), 0.5),
    "fp32-window8-n700": (CacheSpec(1, 3, 3, 700, window=8, dtype="fp32", n_dirs=8, seed=6), 0.3),
    # 16 query heads per KV head (the split-K decode path)
    "bf16-gqa16-n1500": (CacheSpec(1, 1, 16, 1500, n_dirs=32, seed=8), 0.2),
    # enough tiles that every CTA of a 16-CTA decode cluster streams two chunks
    "bf16-n20000": (CacheSpec(1, 1, 4, 20000, n_dirs=64, seed=9), 0.1),
    # wide windows: k = W + ceil(N/128) anchors = 232 and 413 (up to six
    # assignment chunks; eight 128-row observation blocks)
    "bf16-window200-n4000": (CacheSpec(1, 1, 4, 4000, window=200, n_dirs=32, seed=10), 0.1),
    "bf16-window256-n20000": (CacheSpec(1, 1, 4, 20000, window=256, n_dirs=64, seed=11), 0.1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_compress_parity(name):
    spec, theta = CASES[name]
    K, V, Q = make_layer(spec, 0)
    p = _params(spec, theta, layer=3)
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    assert counters[0] == 0
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil)
    parity.log_report(name, rep, refined_rows=counters[1])
    print(name, rep, "refined rows:", counters[1])


def test_compress_exact_ties():
    """Duplicate rows and zero rows make exact ties: lowest slot / lowest index."""
    spec = CacheSpec(1, 1, 4, 600, n_dirs=8, seed=7)
    K, V, Q = make_layer(spec, 0)
    K[0, 100:140] = K[0, 10]          # many keys identical to one another
    V[0, 200:260] = V[0, 20]
    K[0, 300:310] = 0.0               # zero keys: every cosine 0 -> slot 0, gamma 0
    V[0, 400:405] = 0.0
    p = _params(spec, 0.3)
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil)
    g = O.unpack_layout(gb, parity.oracle_params(p))
    assert np.all(g["idx"][0, 0, 300:310] == 0) or 300 in g["anchor_pos"][0]
    parity.log_report("exact-ties-n600", rep, refined_rows=counters[1])
    print(rep)


def test_compress_deterministic():
    spec, theta = CASES["bf16-ragged-n3000"]
    K, V, Q = (x.cuda() for x in make_layer(spec, 0))
    p = _params(spec, theta)
    a, _ = api.compress(p, K, V, Q)
    b, _ = api.compress(p, K, V, Q)
    assert torch.equal(a, b)


def test_host_buffer_compress_matches_device_compress():
    """anchorkv_compress_host (copies inside the library, from pinned host
    buffers) gives the device compress's bytes, in the host buffer and in the
    staged layout; with key-as-query mode it takes no queries."""
    spec, theta = CASES["bf16-ragged-n3000"]
    K, V, Q = make_layer(spec, 0)
    for mode in (0, api.MODE_KEY_QUERIES):
        p = _params(spec, theta)
        p.mode = mode
        Qd = None if mode else Q.cuda()
        ref, _ = api.compress(p, K.cuda(), V.cuda(), Qd)
        hc = api.HostCompressor(p)
        Kh, Vh = K.pin_memory(), V.pin_memory()
        Qh = None if mode else Q.pin_memory()
        out = hc(Kh, Vh, Qh)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(out, ref.cpu())
        assert torch.equal(hc.out, ref)


def test_reconstruct_matches_oracle():
    spec, theta = CASES["bf16-ragged-n3000"]
    K, V, Q = make_layer(spec, 0)
    p = _params(spec, theta)
    out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
    Kh, Vh = api.reconstruct(p, out)
    parts = O.unpack_layout(out.cpu().numpy(), parity.oracle_params(p))
    Ko, Vo = O.reconstruct(parts, parity.oracle_params(p))
    assert np.abs(Kh.cpu().double().numpy() - Ko).max() < 1e-5 * max(1.0, np.abs(Ko).max())
    assert np.abs(Vh.cpu().double().numpy() - Vo).max() < 1e-5 * max(1.0, np.abs(Vo).max())
    # anchors reconstruct bit for bit
    ap = parts["anchor_pos"]
    for h in range(p.n_kv_heads):
        assert torch.equal(Kh[h][ap[h]].cpu(), K[h][ap[h]].float())


@pytest.mark.parametrize("name,batch,tail", [("tiny-fp32-n1024", 1, 0), ("tiny-fp32-n1024", 2, 5),
                                             ("bf16-ragged-n3000", 3, 17), ("bf16-gqa8-n2500", 2, 0),
                                             ("bf16-every-residual", 1, 3), ("bf16-no-residual", 2, 1),
                                             ("fp32-all-anchors", 1, 2), ("fp32-window8-n700", 2, 9),
                                             ("bf16-gqa16-n1500", 2, 4), ("bf16-n20000", 1, 0),
                                             ("bf16-n20000", 2, 1500)])
def test_decode_parity(name, batch, tail):
    spec, theta = CASES[name]
    p = _params(spec, theta)
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    layouts = []
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": spec.seed + 100 * b})
        K, V, Q = make_layer(sb, 0)
        out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
        comp[b, :L["total_bytes"]] = out
        layouts.append(out.cpu().numpy())
    q = make_decode_queries(spec, 0, step=0, batch=batch)
    cap = max(tail, 1) + 3
    Kt, Vt = make_tail(spec, 0, cap, batch=batch)
    o = api.decode_attn(p, comp, q.cuda(), Kt.cuda(), Vt.cuda(), tail_len=tail)
    err = parity.check_decode(p, layouts, _f64(q), _f64(Kt), _f64(Vt), tail, o.cpu().double().numpy(),
                              DECODE_TOL[spec.dtype])
    print(name, batch, tail, "max abs err", err)


@pytest.mark.parametrize("name,batch,tail,mode", [("tiny-fp32-n1024", 2, 5, 0), ("bf16-ragged-n3000", 3, 17, 0),
                                                  ("bf16-gqa8-n2500", 2, 0, 0), ("bf16-every-residual", 1, 3, 0),
                                                  ("fp32-window8-n700", 2, 9, 0), ("bf16-n20000", 2, 1500, 0),
                                                  ("bf16-ragged-n3000", 2, 4, 0x10)])
@pytest.mark.parametrize("klogit", ["1", "0"])
def test_decode_tensor_core_key_logits(name, batch, tail, mode, klogit, monkeypatch):
    """Both ways to the key-residual logits give the oracle's decode, whatever
    the launch shape would pick by default: ahead of the decode on the tensor
    cores (bit planes of the codes times a fixed-point query, kind::i8), or
    inside the decode on the CUDA cores."""
    monkeypatch.setenv("ANCHORKV_DECODE_KLOGIT", klogit)
    spec, theta = CASES[name]
    p = _params(spec, theta)
    p.mode = mode
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    layouts = []
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": spec.seed + 100 * b})
        K, V, Q = make_layer(sb, 0)
        out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
        comp[b, :L["total_bytes"]] = out
        layouts.append(out.cpu().numpy())
    q = make_decode_queries(spec, 0, step=3, batch=batch)
    cap = max(tail, 1) + 3
    Kt, Vt = make_tail(spec, 0, cap, batch=batch)
    o = api.decode_attn(p, comp, q.cuda(), Kt.cuda(), Vt.cuda(), tail_len=tail)
    err = parity.check_decode(p, layouts, _f64(q), _f64(Kt), _f64(Vt), tail, o.cpu().double().numpy(),
                              DECODE_TOL[spec.dtype])
    print(name, "tensor-core key logits", batch, tail, "max abs err", err)


@pytest.mark.parametrize("name,batch,tail,klogit", [("bf16-ragged-n3000", 1, 5, "0"), ("bf16-gqa8-n2500", 3, 0, "1"),
                                                    ("bf16-n20000", 1, 64, "0")])
def test_decode_replayed_in_a_cuda_graph(name, batch, tail, klogit, monkeypatch):
    """A decode captured in a CUDA graph (the anchor-logit pre-kernel, the
    decode launched as its programmatic dependent, and the pre-pass when on)
    and replayed gives the eager call's output bit for bit, replay after
    replay; the rotary decode likewise."""
    monkeypatch.setenv("ANCHORKV_DECODE_KLOGIT", klogit)
    spec, theta = CASES[name]
    p = _params(spec, theta)
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": spec.seed + 100 * b})
        K, V, Q = make_layer(sb, 0)
        out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
        comp[b, :L["total_bytes"]] = out
    q = make_decode_queries(spec, 0, step=0, batch=batch).cuda()
    Kt, Vt = (x.cuda() for x in make_tail(spec, 0, max(tail, 1) + 3, batch=batch))
    ws = torch.empty(api.decode_workspace_bytes(p, batch), dtype=torch.uint8, device="cuda")
    rws = torch.empty(api.decode_rope_workspace_bytes(p, batch), dtype=torch.uint8, device="cuda")
    eager = api.decode_attn(p, comp, q, Kt, Vt, tail_len=tail, workspace=ws).clone()
    eager_r = api.decode_attn_rope(p, comp, q, 500000.0, Kt, Vt, tail_len=tail, workspace=rws).clone()
    o = torch.empty_like(eager)
    orr = torch.empty_like(eager_r)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):          # warm the launch path on the capture stream
        api.decode_attn(p, comp, q, Kt, Vt, tail_len=tail, out=o, workspace=ws)
        api.decode_attn_rope(p, comp, q, 500000.0, Kt, Vt, tail_len=tail, out=orr, workspace=rws)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.decode_attn(p, comp, q, Kt, Vt, tail_len=tail, out=o, workspace=ws)
        api.decode_attn_rope(p, comp, q, 500000.0, Kt, Vt, tail_len=tail, out=orr, workspace=rws)
    for _ in range(3):
        o.zero_()
        orr.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, eager)
        assert torch.equal(orr, eager_r)
    del g


def test_decode_config():
    spec, theta = CASES["bf16-n20000"]
    cfg = api.decode_config(_params(spec, theta), 1)
    n_tiles = (spec.n_tokens + 127) // 128
    assert 1 < cfg["slices"] <= n_tiles and 0 < cfg["smem_bytes"] <= 227 * 1024
    # a batch with more (sequence, head) pairs than SMs: one slice each
    assert api.decode_config(_params(spec, theta), 200)["slices"] == 1
    # 16 query heads per KV head and 1056 anchors: the split-token kernels
    p = api.AnchorKVParams(n_tokens=131072, n_kv_heads=8, n_q_heads=128)
    assert api.decode_config(p, 1)["slices"] == 0


def test_error_paths_on_device():
    spec, theta = CASES["bf16-ragged-n3000"]
    K, V, Q = (x.cuda() for x in make_layer(spec, 0))
    p = _params(spec, theta)
    L = api.anchorkv_bytes(p)
    small = torch.empty(L["total_bytes"] - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(capi.AnchorKVError) as e:
        api.compress(p, K, V, Q, out=small)
    assert e.value.status == capi.ENOSPC
    buf = torch.empty(K.numel() * 2 + 64, dtype=torch.uint8, device="cuda")
    lib = capi.lib()
    ws = torch.empty(api.compress_workspace(p)["total_bytes"], dtype=torch.uint8, device="cuda")
    out = torch.empty(L["total_bytes"], dtype=torch.uint8, device="cuda")
    import ctypes
    st = lib.anchorkv_compress(ctypes.byref(p.c()), ctypes.c_void_p(buf.data_ptr() + 2), ctypes.c_void_p(V.data_ptr()),
                               ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(out.data_ptr()), out.numel(),
                               ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st == capi.EINVAL
    assert api.decode_attn(p, torch.zeros(0, 16, dtype=torch.uint8, device="cuda"),
                           torch.zeros(0, p.n_q_heads, 128, dtype=torch.bfloat16, device="cuda")).shape[0] == 0


@pytest.mark.slow
def test_full_size_layer_llama8b_shape():
    """One layer of the 8B-shaped cache (8 KV / 32 Q heads, N = 32768, bf16,
    theta = 0.05), generated on the device as the benchmark does, checked
    against the oracle in full (every head, both sides), plus a batch-1 decode."""
    spec = CacheSpec(32, 8, 32, 32768, n_dirs=128, seed=0)
    layer = 5
    K, V, Q = make_layer(spec, layer, device="cuda")
    p = _params(spec, 0.05, layer=layer)
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil, full_chain=False)
    parity.log_report("llama8b-layer5-n32768", rep, refined_rows=counters[1])
    print("full-size layer", rep, "refined rows:", counters[1])
    # decisions the fp32 paths cannot certify are re-taken in fp64, so near-ties
    # can only come from the fp32 observation scores and utilities at the
    # selection boundaries: a handful at most on half a million token-sides
    assert rep["near_ties"] <= 8, rep
    q = make_decode_queries(spec, layer, step=0, batch=1, device="cuda")
    comp = torch.from_numpy(gb).cuda()
    o = api.decode_attn(p, comp, q)
    parity.check_decode(p, [gb], _f64(q), None, None, 0, o.cpu().double().numpy(), DECODE_TOL["bf16"])


@pytest.mark.slow
def test_tensor_core_accumulation_error_on_8b_layer(monkeypatch):
    """The nearest-anchor decision is certified from fp32 scores: a row whose
    best two differ by more than 2^-13 ||x|| is not re-taken in fp64.  That
    margin assumes the tensor core's fp32 accumulation of the 128 exact bf16
    products of <x, a> errs by at most 2^-16 ||x|| ||a||.  Measured here on
    every (token, slot) pair of tokens 0..511 of the key side of head 0 of an
    8B-shaped layer (512 x 288 raw accumulators exported by the kernel)
    against the exact dot products."""
    monkeypatch.setenv("ANCHORKV_ASSIGN_PROBE", "1")
    spec = CacheSpec(32, 8, 32, 32768, n_dirs=128, seed=0)
    K, V, Q = make_layer(spec, 5, device="cuda")
    p = _params(spec, 0.05, layer=5)
    out, ws = api.compress(p, K, V, Q)
    assert api.read_status(ws)[0] == 0
    L = api.anchorkv_bytes(p)
    k = L["n_anchors"]
    assert k == 288            # one anchor group, chunked 2 x 144 (or 3 x 96): 288 columns
    view = api.compress_workspace(p)
    raw = ws[view["off_assign_probe"]:view["off_assign_probe"] + 4 * 512 * k].cpu().numpy()
    acc = raw.view(np.float32).reshape(512, k).astype(np.float64)
    ap = O.unpack_layout(out.cpu().numpy(), parity.oracle_params(p))["anchor_pos"][0]
    X = _f64(K[0, :512])
    A = _f64(K[0])[ap]
    exact = X @ A.T                      # products of bf16 values are exact in fp64
    scale = np.linalg.norm(X, axis=1)[:, None] * np.linalg.norm(A, axis=1)[None, :]
    rel = np.abs(acc - exact) / np.where(scale > 0, scale, 1.0)
    print("tensor-core accumulation: max |acc - <x,a>| / (||x|| ||a||) =", rel.max(),
          "= 2^%.1f" % np.log2(max(rel.max(), 1e-300)))
    parity.log_report("tc-accumulation-8b-layer5", {"max_rel_acc_err": float(rel.max()),
                                                     "pairs": int(rel.size)})
    assert rel.max() <= 2.0 ** -16


@pytest.mark.parametrize("name", ["bf16-ragged-n3000", "bf16-gqa8-n2500", "bf16-every-residual"])
def test_tensor_core_and_simt_assignment_agree(name, monkeypatch):
    """The tcgen05 assignment and the SIMT assignment both end in the same
    fp64-certified decisions, so their layouts are identical."""
    spec, theta = CASES[name]
    K, V, Q = (x.cuda() for x in make_layer(spec, 0))
    p = _params(spec, theta)
    tc_out, tc_ws = api.compress(p, K, V, Q)
    tc_refined = api.read_status(tc_ws)[1]
    monkeypatch.setenv("ANCHORKV_SIMT_ASSIGN", "1")
    simt_out, _ = api.compress(p, K, V, Q)
    assert torch.equal(tc_out, simt_out)
    print(name, "rows re-decided in fp64 (tensor-core path):", tc_refined)


@pytest.mark.parametrize("name", ["bf16-ragged-n3000", "bf16-gqa8-n2500"])
def test_simt_observation_path_parity(name, monkeypatch):
    """The SIMT observation passes (used for fp32 caches) also match the
    oracle on bf16 inputs, so both implementations stay covered."""
    monkeypatch.setenv("ANCHORKV_SIMT_OBS", "1")
    spec, theta = CASES[name]
    K, V, Q = make_layer(spec, 0)
    p = _params(spec, theta, layer=1)
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    assert counters[0] == 0
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil)
    parity.log_report(name + " (SIMT observation passes)", rep, refined_rows=counters[1])
    print(name, "simt observation passes", rep)


# optional modes: key-as-query proxies, the alternative rankings, the unrotated codec
MODE_CASES = [
    ("bf16-ragged-n3000", api.mode_bits(key_queries=True)),
    ("fp32-window8-n700", api.mode_bits(key_queries=True)),
    ("bf16-ragged-n3000", api.mode_bits(rank=api.RANK_RESIDUAL_NORM)),
    ("bf16-gqa8-n2500", api.mode_bits(rank=api.RANK_ATTENTION)),
    ("tiny-fp32-n1024", api.mode_bits(rank=api.RANK_ATTENTION)),
    ("bf16-ragged-n3000", api.mode_bits(rank=api.RANK_COSINE)),
    ("bf16-n20000", api.mode_bits(rank=api.RANK_RANDOM)),
    ("bf16-ragged-n3000", api.mode_bits(naive_codec=True)),
    ("tiny-fp32-n1024", api.mode_bits(naive_codec=True)),
    ("bf16-gqa16-n1500", api.mode_bits(key_queries=True, rank=api.RANK_COSINE, naive_codec=True)),
]


@pytest.mark.parametrize("name,mode", MODE_CASES)
def test_compress_modes(name, mode):
    spec, theta = CASES[name]
    K, V, Q = make_layer(spec, 0)
    p = _params(spec, theta, layer=2)
    p.mode = mode
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    assert counters[0] == 0
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil)
    parity.log_report(f"{name} mode {mode:#x}", rep, refined_rows=counters[1])
    print(name, hex(mode), rep)


@pytest.mark.parametrize("name,batch,tail", [("bf16-ragged-n3000", 2, 5), ("tiny-fp32-n1024", 1, 0),
                                             ("bf16-gqa16-n1500", 2, 3), ("bf16-n20000", 1, 700)])
def test_decode_naive_codec(name, batch, tail):
    """Decode of layouts written with the unrotated codec (cluster path for
    G <= 8, split-token path for G = 16)."""
    spec, theta = CASES[name]
    p = _params(spec, theta)
    p.mode = api.mode_bits(naive_codec=True)
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    layouts = []
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": spec.seed + 50 * b})
        K, V, Q = make_layer(sb, 0)
        out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
        comp[b, :L["total_bytes"]] = out
        layouts.append(out.cpu().numpy())
    q = make_decode_queries(spec, 0, step=0, batch=batch)
    cap = max(tail, 1) + 3
    Kt, Vt = make_tail(spec, 0, cap, batch=batch)
    o = api.decode_attn(p, comp, q.cuda(), Kt.cuda(), Vt.cuda(), tail_len=tail)
    err = parity.check_decode(p, layouts, _f64(q), _f64(Kt), _f64(Vt), tail, o.cpu().double().numpy(),
                              DECODE_TOL[spec.dtype])
    print(name, "naive codec", batch, tail, "max abs err", err)


def test_reconstruct_naive_codec():
    spec, theta = CASES["bf16-ragged-n3000"]
    K, V, Q = make_layer(spec, 0)
    p = _params(spec, theta)
    p.mode = api.mode_bits(naive_codec=True)
    out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
    Kh, Vh = api.reconstruct(p, out)
    po = parity.oracle_params(p)
    Ko, Vo = O.reconstruct(O.unpack_layout(out.cpu().numpy(), po), po)
    assert np.abs(Kh.cpu().double().numpy() - Ko).max() < 1e-5 * np.abs(Ko).max()
    assert np.abs(Vh.cpu().double().numpy() - Vo).max() < 1e-5 * np.abs(Vo).max()


@pytest.mark.parametrize("N,anchor_div,theta", [(8000, 16, 0.1), (8000, 8, 0.15)])
def test_compress_anchor_groups(N, anchor_div, theta):
    """More anchors than the tensor-core assignment keeps resident (k = 532
    and 1032: two and three anchor groups merged through the workspace)."""
    spec = CacheSpec(1, 1, 4, N, n_dirs=64, seed=12)
    K, V, Q = make_layer(spec, 0)
    p = _params(spec, theta, layer=1)
    p.anchor_div = anchor_div
    assert api.anchorkv_bytes(p)["n_anchors"] > 480
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    assert counters[0] == 0
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil)
    parity.log_report(f"anchor-groups-n{N}-k{api.anchorkv_bytes(p)['n_anchors']}", rep, refined_rows=counters[1])
    print("anchor groups", N, anchor_div, rep, "refined rows:", counters[1])


@pytest.mark.parametrize("name,batch,tail,base,mode", [
    ("tiny-fp32-n1024", 1, 0, 10000.0, 0), ("tiny-fp32-n1024", 2, 5, 500000.0, 0),
    ("bf16-ragged-n3000", 2, 17, 500000.0, 0), ("bf16-gqa8-n2500", 1, 3, 10000.0, 0),
    ("bf16-gqa16-n1500", 2, 4, 500000.0, 0), ("bf16-n20000", 1, 40, 500000.0, 0),
    ("bf16-ragged-n3000", 1, 2, 10000.0, 0x10),
    # one and two query heads per KV head, no residuals, every residual, and a
    # 33-token all-anchor cache whose tail makes a second, partial 32-token chunk
    ("fp32-window8-n700", 1, 3, 10000.0, 0), ("bf16-no-residual", 2, 0, 500000.0, 0),
    ("bf16-every-residual", 1, 1, 10000.0, 0), ("fp32-all-anchors", 1, 2, 10000.0, 0)])
def test_decode_rope_parity(name, batch, tail, base, mode):
    """Keys stored before the rotary map, rotated at decode (cached token t at
    position t, tail token i at N + i, the query at N + T)."""
    spec, theta = CASES[name]
    p = _params(spec, theta)
    p.mode = mode
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    layouts = []
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": spec.seed + 70 * b})
        K, V, Q = make_layer(sb, 0)
        out, _ = api.compress(p, K.cuda(), V.cuda(), Q.cuda())
        comp[b, :L["total_bytes"]] = out
        layouts.append(out.cpu().numpy())
    q = make_decode_queries(spec, 0, step=1, batch=batch)
    cap = max(tail, 1) + 2
    Kt, Vt = make_tail(spec, 0, cap, batch=batch)
    o = api.decode_attn_rope(p, comp, q.cuda(), base, Kt.cuda(), Vt.cuda(), tail_len=tail)
    err = parity.check_decode_rope(p, layouts, _f64(q), _f64(Kt), _f64(Vt), tail, base, o.cpu().double().numpy(),
                                   DECODE_TOL[spec.dtype])
    print(name, "rope", batch, tail, base, "max abs err", err)


@pytest.mark.slow
def test_batched_decode_8b_shape_sampled():
    """Batched decode as benchmarked for many sequences: 16 compressed
    sequences of the 8B shape (8 KV / 32 query heads, N = 32768, theta = 0.1)
    decoded in one launch; every sequence checked against the oracle."""
    spec = CacheSpec(32, 8, 32, 32768, n_dirs=128, seed=0)
    p = _params(spec, 0.1, layer=0)
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    batch = 16
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device="cuda")
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": 1000 + b})
        K, V, Q = make_layer(sb, 0, device="cuda")
        out, ws = api.compress(p, K, V, Q)
        assert api.read_status(ws)[0] == 0
        comp[b, :L["total_bytes"]] = out
    q = make_decode_queries(spec, 0, step=0, batch=batch, device="cuda")
    o = api.decode_attn(p, comp, q)
    po = parity.oracle_params(p)
    assert torch.isfinite(o).all()
    for b in range(batch):
        parts = O.unpack_layout(comp[b, :L["total_bytes"]].cpu().numpy(), po)
        Kh, Vh = O.reconstruct(parts, po)
        want = O.decode_attention(_f64(q[b]), Kh, Vh)
        err = float(np.abs(o[b].cpu().double().numpy() - want).max())
        assert err <= DECODE_TOL["bf16"], (b, err)
        print("batched decode sequence", b, "max abs err", err)


@pytest.mark.slow
def test_70b_shape_layer_stage_by_stage():
    """One layer of the 70B-shaped cache (8 KV / 64 query heads, N = 131072,
    theta = 0.05; k = 1056 anchors in three assignment groups), every stage
    against the oracle on every head and side: pooled scores, anchor sets,
    nearest-anchor slots, coefficients, utilities, the top-R selection, the
    residual codes and scales (mismatches only as counted near-ties); then the
    decode of all 64 query heads after 128 appended exact tokens."""
    spec = CacheSpec(80, 8, 64, 131072, n_dirs=256, seed=0)
    p = _params(spec, 0.05, layer=7)
    K, V, Q = make_layer(spec, 7, device="cuda")
    L = api.anchorkv_bytes(p)
    po = parity.oracle_params(p)
    Lo = O.layout(po)
    assert L["total_bytes"] == Lo["total"] and L["n_residuals"] == Lo["R"] and L["n_anchors"] == Lo["k"] == 1056
    gb, gpool, gutil, counters = parity.gpu_compress(p, K, V, Q)
    assert counters[0] == 0
    rep = parity.check_compress(p, _f64(K), _f64(V), _f64(Q), gb, gpool, gutil, full_chain=False)
    parity.log_report("llama70b-layer7-n131072", rep, refined_rows=counters[1])
    print("70B-shaped layer", rep, "refined rows:", counters[1])
    assert rep["near_ties"] <= 16, rep
    out = torch.from_numpy(gb).cuda()
    q = make_decode_queries(spec, 7, step=128, batch=1, device="cuda")
    Kt, Vt = make_tail(spec, 7, 128, batch=1, device="cuda")
    o = api.decode_attn(p, out, q, Kt, Vt, tail_len=128)
    parity.check_decode(p, [gb], _f64(q), _f64(Kt), _f64(Vt), 128, o.cpu().double().numpy(), DECODE_TOL["bf16"])


@pytest.mark.slow
def test_multi_stream_compress_matches_single_stream():
    """The benchmark compresses independent layers on four streams, each with
    its own workspace: the layouts must equal the single-stream ones byte for
    byte (8B-shaped layers, N = 32768, theta = 0.05)."""
    spec = CacheSpec(4, 8, 32, 32768, n_dirs=128, seed=0)
    layers = [make_layer(spec, l, device="cuda") for l in range(spec.n_layers)]
    params = [_params(spec, 0.05, layer=l) for l in range(spec.n_layers)]
    single = []
    ws = None
    for l, (K, V, Q) in enumerate(layers):
        out, ws = api.compress(params[l], K, V, Q, workspace=ws)
        single.append(out.clone())
    streams = [torch.cuda.Stream() for _ in range(4)]
    wss = [torch.empty_like(ws) for _ in range(4)]
    multi = [torch.empty_like(x) for x in single]
    torch.cuda.synchronize()
    for l, (K, V, Q) in enumerate(layers):
        with torch.cuda.stream(streams[l % 4]):
            api.compress(params[l], K, V, Q, out=multi[l], workspace=wss[l % 4])
    torch.cuda.synchronize()
    for w in wss:
        assert api.read_status(w)[0] == 0
    for l in range(spec.n_layers):
        assert torch.equal(single[l], multi[l]), l
