"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests retypes an oracle formula: each checks the oracle against a
published value, a library routine, a brute-force search, an invariant or a
perturbation experiment.  All run on the CPU.
"""
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.special
import scipy.stats
import torch

from oracle import anchorkv_oracle as O
from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_layer, gaussian_queries

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _small_layer(N=512, H=2, Hq=8, dtype="bf16", theta=0.1, seed=3, n_dirs=16):
    spec = CacheSpec(1, H, Hq, N, dtype=dtype, n_dirs=n_dirs, seed=seed)
    K, V, Q = make_layer(spec, 0)
    p = O.Params(n_tokens=N, n_kv_heads=H, n_q_heads=Hq, theta=theta, dtype=dtype, seed=seed)
    return K.double().numpy(), V.double().numpy(), Q.double().numpy(), p


# ---------------------------------------------------------------- codebook

def test_lloyd_max_matches_published_table():
    tau, l1, l2, mse = O.lloyd_max_gaussian_4()
    got = dict(threshold_outer=tau, level_inner=l1, level_outer=l2, mse=mse)
    for name, val, tol in _read_golden("lloyd_max_gaussian_4level.txt"):
        assert abs(got[name] - float(val)) <= float(tol), (name, got[name], val)


def test_lloyd_max_optimality_by_quadrature():
    """Centroid and nearest-neighbour conditions, integrated numerically."""
    tau, l1, l2, mse = O.lloyd_max_gaussian_4()
    pdf = scipy.stats.norm.pdf
    m0 = scipy.integrate.quad(lambda x: x * pdf(x), 0, tau, epsabs=1e-14)[0]
    p0 = scipy.integrate.quad(pdf, 0, tau, epsabs=1e-14)[0]
    m1 = scipy.integrate.quad(lambda x: x * pdf(x), tau, np.inf, epsabs=1e-14)[0]
    p1 = scipy.integrate.quad(pdf, tau, np.inf, epsabs=1e-14)[0]
    assert abs(m0 / p0 - l1) < 1e-9
    assert abs(m1 / p1 - l2) < 1e-9
    assert abs(0.5 * (l1 + l2) - tau) < 1e-12
    d = 2 * (scipy.integrate.quad(lambda x: (x - l1) ** 2 * pdf(x), 0, tau, epsabs=1e-14)[0]
             + scipy.integrate.quad(lambda x: (x - l2) ** 2 * pdf(x), tau, np.inf, epsabs=1e-14)[0])
    assert abs(d - mse) < 1e-9


# ---------------------------------------------------------------- generator

def test_splitmix64_published_outputs():
    want = [int(r[0]) for r in _read_golden("splitmix64_state1234567.txt")]
    got = [O.splitmix64(1234567 + i * 0x9E3779B97F4A7C15) for i in range(5)]
    assert got == want


def test_hadamard_matches_scipy_and_is_involution():
    for d in (4, 32, 128):
        H = O.hadamard_matrix(d)
        assert np.array_equal(H * math.sqrt(d), scipy.linalg.hadamard(d).astype(float))
        assert np.abs(H @ H - np.eye(d)).max() < 1e-12
    s = O.hadamard_signs(0, 128)
    assert set(np.unique(s)) <= {-1.0, 1.0}
    assert 40 < (s > 0).sum() < 88


# ---------------------------------------------------------------- codec

def test_codes_pick_nearest_level():
    rng = np.random.default_rng(0)
    r = rng.normal(size=(200, 128)) * rng.lognormal(size=(200, 1))
    sig, codes, y = O.quantize_residuals(r, seed=5)
    tau, l1, l2, _ = O.lloyd_max_gaussian_4()
    levels = np.array([-l2, -l1, l1, l2])
    s16 = sig.astype(np.float64)[:, None]
    dist = np.abs(y[:, :, None] - levels[None, None, :] * s16[:, :, None])
    nearest = dist.argmin(axis=2)
    assert np.array_equal(nearest, codes)
    # the rotation is orthonormal: ||y|| == ||r||
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(r, axis=1), rtol=1e-12)


def test_codec_roundtrip_reduces_error():
    """Quantized residual is strictly closer than storing nothing (also for
    residuals whose energy sits in one coordinate)."""
    rng = np.random.default_rng(1)
    r = rng.normal(size=(300, 128))
    r[:20] = 0.0
    r[:20, np.arange(20) * 3] = rng.normal(size=20) * 5
    sig, codes, _ = O.quantize_residuals(r, seed=9)
    rt = O.dequantize_residuals(sig, codes, seed=9)
    assert np.all(np.linalg.norm(r - rt, axis=1) < np.linalg.norm(r, axis=1))


def test_codec_distortion_matches_lloyd_max_mse():
    rng = np.random.default_rng(2)
    r = rng.normal(size=(4000, 128))
    sig, codes, _ = O.quantize_residuals(r, seed=11)
    rt = O.dequantize_residuals(sig, codes, seed=11)
    eta = (np.linalg.norm(r - rt, axis=1) ** 2 / np.linalg.norm(r, axis=1) ** 2).mean()
    mse = O.lloyd_max_gaussian_4()[3]
    assert abs(eta - mse) < 0.01


def test_pack_bit_positions():
    codes = np.array([[0, 1, 2, 3] * 32], dtype=np.uint8)
    packed = O.pack_codes(codes)
    assert packed.shape == (1, 32) and np.all(packed == 0b11100100)
    rng = np.random.default_rng(3)
    c = rng.integers(0, 4, size=(17, 128)).astype(np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(c), 128), c)


def test_zero_residual_decodes_to_zero():
    sig, codes, _ = O.quantize_residuals(np.zeros((2, 128)), seed=0)
    assert np.all(sig == 0)
    assert np.all(O.dequantize_residuals(sig, codes, seed=0) == 0)


# ---------------------------------------------------------------- projection

def test_gamma_orthogonality_and_exact_reconstruction():
    K, V, Q, p = _small_layer()
    ap = np.sort(np.random.default_rng(0).choice(p.n_tokens, 40, replace=False))
    idx, _, _ = O.assign(K[0], ap)
    gamma, g16, r, r2 = O.project(K[0], ap, idx)
    xa = K[0][ap][idx]
    res_unrounded = K[0] - gamma[:, None] * xa
    scale = np.linalg.norm(K[0], axis=1) * np.linalg.norm(xa, axis=1)
    assert np.all(np.abs((res_unrounded * xa).sum(axis=1)) <= 1e-12 * scale + 1e-300)
    # stored gamma~ plus the residual reproduces x bit for bit
    assert np.array_equal(g16.astype(np.float64)[:, None] * xa + r, K[0])
    # anchors: gamma 1, zero residual
    assert np.all(g16[ap] == 1.0) and np.all(r[ap] == 0.0)


def test_assign_brute_force_small():
    rng = np.random.default_rng(4)
    N, D = 96, 16
    X = rng.normal(size=(N, D)).round(3)
    ap = np.array([0, 5, 9, 20, 33, 47, 60, 90])
    X[9] = X[5]            # duplicate anchors: ties must go to the lower slot
    X[40] = 2.0 * X[5]     # exactly collinear with two slots -> slot 1
    X[33] = 0.0            # a zero anchor scores 0
    idx, _, _ = O.assign(X, ap)
    for i in range(N):
        if i in ap:
            assert idx[i] == list(ap).index(i)
            continue
        best, bs = -math.inf, -1
        for s, a in enumerate(ap):
            na = math.sqrt(math.fsum(v * v for v in X[a]))
            c = 0.0 if na == 0 else math.fsum(u * v for u, v in zip(X[i], X[a])) / na
            if c > best:
                best, bs = c, s
        assert idx[i] == bs, i
    assert idx[40] == 1


# ---------------------------------------------------------------- scoring

def test_single_query_score_is_softmax():
    rng = np.random.default_rng(5)
    N, D = 64, 16
    K = rng.normal(size=(N, D))
    V = rng.normal(size=(N, D))
    q = rng.normal(size=(1, D))
    att = O.obs_attention(q, K, V, window=1)
    ref = scipy.special.softmax(K @ q[0] / math.sqrt(D))
    assert np.abs(att["alpha"][0] - ref).max() < 1e-15
    assert np.abs(att["ybar"][0] - ref @ V).max() < 1e-12


def test_observation_rows_are_causal():
    rng = np.random.default_rng(6)
    N, D, W = 40, 8, 4
    K, V = rng.normal(size=(N, D)), rng.normal(size=(N, D))
    Qh = rng.normal(size=(2 * W, D))
    a = O.obs_attention(Qh, K, V, window=W)["alpha"]
    for r in range(2 * W):
        w = r % W
        assert np.all(a[r, N - W + w + 1:] == 0)
        ref = scipy.special.softmax(K[:N - W + w + 1] @ Qh[r] / math.sqrt(D))
        assert np.abs(a[r, :N - W + w + 1] - ref).max() < 1e-15


def test_pooling_of_a_spike():
    s = np.zeros(30)
    s[10] = 7.0
    p = O.pool_scores(s, 7)
    assert np.allclose(p[7:14], 1.0) and np.all(p[:7] == 0) and np.all(p[14:] == 0)
    e = np.zeros(30)
    e[0] = 7.0                            # zero padding at the edge
    assert np.allclose(O.pool_scores(e, 7)[:4], 1.0) and np.all(O.pool_scores(e, 7)[4:] == 0)


def _textbook_pooled_scores(K, Q, p, h):
    """The anchor score of KV head h recomputed from first principles: for
    every query head j of the head and every window row w, a textbook softmax
    (scipy) over the positions query (j, w) can see (t <= N - W + w); the
    weights are summed over all (j, w) at the non-window positions t < N - W,
    then averaged over a centred kappa-wide window with zero padding (numpy's
    'same' convolution with a box of ones, divided by kappa)."""
    N, D = K.shape[1], K.shape[2]
    W, G = p.window, p.group
    score = np.zeros(N - W)
    for j in range(h * G, (h + 1) * G):
        for w in range(W):
            vis = N - W + w + 1
            a = scipy.special.softmax(K[h, :vis] @ Q[j, w] / math.sqrt(D))
            score += a[:N - W]
    return np.convolve(score, np.ones(p.pool_kernel), mode="same") / p.pool_kernel


def test_pooled_scores_against_textbook_softmax():
    """[PITH] "Assumptions & free parameters": the last W queries' attention,
    pooled over every GQA query head of the KV head, then kappa = 7 pooling
    (Eq. 14).  The oracle's pooled scores (the values the GPU is compared
    with) must equal an independent per-row recomputation."""
    K, V, Q, p = _small_layer(N=300, H=2, Hq=8)
    st = O.compress_layer(K, V, Q, p)
    for h in range(p.n_kv_heads):
        ref = _textbook_pooled_scores(K, Q, p, h)
        assert np.abs(st["pooled"][h] - ref).max() <= 1e-12 * ref.max(), h


def test_anchor_sets():
    K, V, Q, p = _small_layer(N=700)
    L = O.layout(p)
    st = O.compress_layer(K, V, Q, p)
    for h in range(p.n_kv_heads):
        ap = st["anchor_pos"][h]
        assert len(set(ap.tolist())) == L["k"] == p.window + L["m"]
        assert set(range(p.n_tokens - p.window, p.n_tokens)) <= set(ap.tolist())
        pooled = st["pooled"][h]
        # brute force: the n_s best by (score desc, position asc) are all anchors
        ranked = sorted(range(p.n_tokens - p.window), key=lambda t: (-pooled[t], t))
        scored = set(ranked[:L["n_s"]])
        assert scored <= set(ap.tolist())
        rest = sorted(set(ap.tolist()) - scored - set(range(p.n_tokens - p.window, p.n_tokens)))
        assert len(rest) == L["n_u"]
        cand = [t for t in range(p.n_tokens - p.window) if t not in scored]
        by_key = sorted(cand, key=lambda t: (O.anchor_hash_key(p.seed, p.layer, h, t), t))
        assert rest == sorted(by_key[:L["n_u"]])


def test_uniform_sample_is_uniform():
    p = O.Params(n_tokens=1000, n_kv_heads=1, n_q_heads=1, theta=0.1, window=8, anchor_div=10)
    L = O.layout(p)
    pooled = np.zeros(p.n_tokens - p.window)   # every score ties -> scored = lowest positions
    hits = np.zeros(p.n_tokens - p.window)
    for seed in range(300):
        p.seed = seed
        ap = O.select_anchors(pooled, p, head=0)
        u = [t for t in ap if L["n_s"] <= t < p.n_tokens - p.window]
        assert len(u) == L["n_u"]
        hits[u] += 1
    obs = hits[L["n_s"]:]
    chi2 = ((obs - obs.mean()) ** 2 / obs.mean()).sum()
    dof = obs.size - 1
    assert scipy.stats.chi2.sf(chi2, dof) > 1e-3


def test_all_positions_anchor_when_short():
    p = O.Params(n_tokens=33, n_kv_heads=1, n_q_heads=2, theta=0.5, window=32)
    L = O.layout(p)
    assert L["k"] == 33 and L["cap"] == 0 and L["R"] == 0
    K, V, Q, _ = _small_layer(N=33, H=1, Hq=2)
    st = O.compress_layer(K, V, Q, p)
    assert np.array_equal(st["anchor_pos"][0], np.arange(33))
    assert st["sel"].sum() == 0


# ---------------------------------------------------------------- utilities

def _dense_out(Qh, K, V, W):
    return O.obs_attention(Qh, K, V, W)["ybar"]


def test_value_utility_equals_output_change():
    """Leaving out r^V_t changes every observation output by alpha_rt r_t; the
    summed squared change is the value utility (exact: y is linear in V)."""
    K, V, Q, p = _small_layer(N=300, H=1, Hq=2)
    st = O.compress_layer(K, V, Q, p)
    Qh = Q[:2].reshape(2 * p.window, -1)
    y0 = _dense_out(Qh, K[0], V[0], p.window)
    for t in np.nonzero(st["eligible"][1, 0])[0][:15]:
        Vp = V[0].copy()
        Vp[t] -= st["r"][1, 0, t]
        dy = _dense_out(Qh, K[0], Vp, p.window) - y0
        assert abs((dy ** 2).sum() - st["u"][1, 0, t]) <= 1e-9 * st["u"][1, 0, t] + 1e-300


def test_key_utility_is_first_order_isotropic_expectation():
    """Average, over an orthonormal basis of residual directions of norm
    ||r^K_t||, of the squared first-order output change (central finite
    differences through the real softmax) equals the key utility."""
    K, V, Q, p = _small_layer(N=200, H=1, Hq=2)
    st = O.compress_layer(K, V, Q, p)
    D = K.shape[2]
    Qh = Q[:2].reshape(2 * p.window, -1)
    h = 1e-5
    for t in np.nonzero(st["eligible"][0, 0])[0][:4]:
        nr = math.sqrt(st["r2"][0, 0, t])
        acc = 0.0
        for d in range(D):
            Kp, Km = K[0].copy(), K[0].copy()
            Kp[t, d] += h * nr
            Km[t, d] -= h * nr
            dy = (_dense_out(Qh, Kp, V[0], p.window) - _dense_out(Qh, Km, V[0], p.window)) / (2 * h)
            acc += (dy ** 2).sum()
        assert abs(acc / D - st["u"][0, 0, t]) <= 1e-6 * st["u"][0, 0, t]


# ---------------------------------------------------------------- budget

def test_select_residuals_brute_force():
    rng = np.random.default_rng(7)
    u = rng.integers(0, 6, size=(2, 3, 50)).astype(float)   # many exact ties
    el = rng.random(size=(2, 3, 50)) > 0.2
    for R in (0, 1, 17, 60, int(el.sum())):
        sel = O.select_residuals(u, el, R)
        flat = [(-u.reshape(-1)[f], f) for f in range(u.size) if el.reshape(-1)[f]]
        want = {f for _, f in sorted(flat)[:R]}
        assert set(np.nonzero(sel.reshape(-1))[0].tolist()) == want


def test_budget_pools_across_heads():
    rng = np.random.default_rng(8)
    u = rng.random(size=(2, 2, 400))
    el = np.ones_like(u, dtype=bool)
    base = O.select_residuals(u, el, 200)
    u2 = u.copy()
    u2[:, 1] *= 10.0
    boosted = O.select_residuals(u2, el, 200)
    assert boosted[:, 1].sum() > base[:, 1].sum()
    assert boosted[:, 1].sum() > boosted[:, 0].sum()


@pytest.mark.parametrize("N,H,theta,dtype", [
    (1024, 1, 0.1, "fp32"), (32768, 8, 0.05, "bf16"), (131072, 8, 0.05, "bf16"),
    (32768, 8, 0.1, "bf16"), (8192, 8, 0.2, "bf16"), (5000, 3, 0.07, "bf16"), (777, 2, 0.3, "fp32")])
def test_byte_accounting(N, H, theta, dtype):
    p = O.Params(n_tokens=N, n_kv_heads=H, n_q_heads=4 * H, theta=theta, dtype=dtype)
    L = O.layout(p)
    assert L["total"] == L["base"] + L["c"] * L["R"]
    if 0 < L["R"] < L["cap"]:
        assert L["total"] <= L["B"] < L["total"] + L["c"]
    offs = sorted(L["off"].items(), key=lambda kv: kv[1])
    for (name, o), (_, nxt) in zip(offs, offs[1:]):
        assert o % 16 == 0 or name == "res_sigma"
        assert o + L["sizes"].get(name, 0) <= nxt
    if (N, H, theta) == (32768, 8, 0.05):
        assert abs(L["U"] / L["total"] - 20.0) < 0.01      # theta = 0.05 -> 20x


def test_byte_image_length_and_roundtrip():
    K, V, Q, p = _small_layer(N=600, H=2, Hq=4, theta=0.2)
    st = O.compress_layer(K, V, Q, p)
    L = O.layout(p)
    assert st["bytes"].shape[0] == L["total"]
    parts = O.unpack_layout(st["bytes"], p)
    assert np.array_equal(parts["idx"], st["idx"])
    assert np.array_equal(parts["g16"].view(np.uint16), st["g16"].view(np.uint16))
    assert np.array_equal(parts["sel"], st["sel"])
    assert parts["tile_prefix"][-1, -1, -1] == L["R"]
    # every position keeps a record (no token is dropped)
    assert np.all(parts["idx"] < L["k"])


def test_small_scale_floors_to_zero_residuals():
    p = O.Params(n_tokens=256, n_kv_heads=1, n_q_heads=4, theta=0.05, dtype="bf16")
    L = O.layout(p)
    assert L["R"] == 0 and L["total"] > L["B"]


def test_theta_one_gives_every_token_a_residual():
    K, V, Q, p = _small_layer(N=300, H=1, Hq=2, theta=1.0)
    L = O.layout(p)
    assert L["R"] == L["cap"]
    st = O.compress_layer(K, V, Q, p)
    assert np.array_equal(st["sel"], st["eligible"])


def test_deterministic():
    K, V, Q, p = _small_layer(N=400)
    a = O.compress_layer(K, V, Q, p)["bytes"]
    b = O.compress_layer(K, V, Q, p)["bytes"]
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- decode

def _sdpa(q, K, V):
    """torch's scaled-dot-product attention in float64, GQA by repeat."""
    Hq, D = q.shape
    G = Hq // K.shape[0]
    Kr = torch.from_numpy(np.repeat(K, G, axis=0))
    Vr = torch.from_numpy(np.repeat(V, G, axis=0))
    qt = torch.from_numpy(q)[:, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kr, Vr)[:, 0].numpy()


def test_decode_with_exact_residuals_is_dense_attention():
    K, V, Q, p = _small_layer(N=300, H=2, Hq=8, theta=1.0)
    st = O.compress_layer(K, V, Q, p)
    parts = O.unpack_layout(st["bytes"], p)
    Kh, Vh = O.reconstruct(parts, p, identity_residuals=st["r"])
    assert np.abs(Kh - K).max() < 1e-12 and np.abs(Vh - V).max() < 1e-12
    q = np.random.default_rng(9).normal(size=(8, 128))
    Kt = np.random.default_rng(10).normal(size=(2, 5, 128))
    Vt = np.random.default_rng(11).normal(size=(2, 5, 128))
    o = O.decode_attention(q, Kh, Vh, Kt, Vt)
    ref = _sdpa(q, np.concatenate([K, Kt], 1), np.concatenate([V, Vt], 1))
    assert np.abs(o - ref).max() < 1e-12


def test_decode_anchor_only_cache():
    K, V, Q, p = _small_layer(N=400, H=1, Hq=4, theta=0.01)
    st = O.compress_layer(K, V, Q, p)
    assert O.layout(p)["R"] == 0
    parts = O.unpack_layout(st["bytes"], p)
    Kh, Vh = O.reconstruct(parts, p)
    ap = st["anchor_pos"][0]
    for side, X, Xh in ((0, K, Kh), (1, V, Vh)):
        want = st["g16"][side, 0].astype(np.float64)[:, None] * X[0][ap][st["idx"][side, 0]]
        assert np.array_equal(Xh[0], want)
        assert np.array_equal(Xh[0][ap], X[0][ap])                 # anchors bit-exact
    q = np.random.default_rng(12).normal(size=(4, 128))
    assert np.abs(O.decode_attention(q, Kh, Vh) - _sdpa(q, Kh, Vh)).max() < 1e-12


def test_theorem1_bound_holds():
    K, V, Q, p = _small_layer(N=1024, H=1, Hq=4, theta=0.1)
    st = O.compress_layer(K, V, Q, p)
    Kh, Vh = O.reconstruct(O.unpack_layout(st["bytes"], p), p)
    q = gaussian_queries(256, 128, seed=1).double().numpy()
    t = O.theorem1(q, K[0], V[0], Kh[0], Vh[0])
    assert np.all(t["err"] <= t["bound_a"] + 1e-12)
    assert np.all(t["err"] <= t["bound_b"] + 1e-12)
    assert np.all(t["err"] > 0)


# ---------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes(monkeypatch):
    """A dropped 1/D in the key utility or a flipped residual sign must be
    caught by the pins above."""
    orig_util = O.utilities

    def bad_util(*a, **k):
        uK, uV = orig_util(*a, **k)
        return uK * 128.0, uV
    monkeypatch.setattr(O, "utilities", bad_util)
    with pytest.raises(AssertionError):
        test_key_utility_is_first_order_isotropic_expectation()
    monkeypatch.setattr(O, "utilities", orig_util)

    orig_proj = O.project

    def bad_proj(X, ap, idx):
        g, g16, r, r2 = orig_proj(X, ap, idx)
        return g, g16, -r, r2
    monkeypatch.setattr(O, "project", bad_proj)
    with pytest.raises(AssertionError):
        test_gamma_orthogonality_and_exact_reconstruction()
    monkeypatch.setattr(O, "project", orig_proj)


def test_score_pin_catches_planted_mistakes(monkeypatch):
    """Anchor-score mistakes the textbook recomputation must catch: summing the
    window rows of one query head only, and pooling the weights of the window
    positions into the scores next to the window."""
    orig_scores, orig_pool = O.token_scores, O.pool_scores

    def one_head_only(alpha, n_tokens, window):
        return alpha[:window, : n_tokens - window].sum(axis=0)
    monkeypatch.setattr(O, "token_scores", one_head_only)
    with pytest.raises(AssertionError):
        test_pooled_scores_against_textbook_softmax()

    # the window's weights leak into the pooling: score over all N positions,
    # pooled, and only then cut to the non-window positions
    n_cut = {}

    def full_length(alpha, n_tokens, window):
        n_cut["n"] = n_tokens - window
        return alpha.sum(axis=0)

    def pool_then_cut(score, kappa):
        return orig_pool(score, kappa)[: n_cut["n"]]
    monkeypatch.setattr(O, "token_scores", full_length)
    monkeypatch.setattr(O, "pool_scores", pool_then_cut)
    with pytest.raises(AssertionError):
        test_pooled_scores_against_textbook_softmax()
    monkeypatch.setattr(O, "token_scores", orig_scores)
    monkeypatch.setattr(O, "pool_scores", orig_pool)
    test_pooled_scores_against_textbook_softmax()
