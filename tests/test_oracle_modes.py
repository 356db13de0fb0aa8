"""Pins of the oracle's optional modes: key-as-query proxies, the alternative
ranking criteria and the unrotated ("naive") 2-bit codec.

Each test recomputes what the mode must select or produce from the layout
bytes and the inputs by an independent route (brute force over the flat
index, a textbook softmax, nearest-level coding) rather than re-calling the
oracle's own helper for that mode.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import scipy.stats

from oracle import anchorkv_oracle as O
from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_layer


def _layer(N=600, H=2, Hq=4, theta=0.08, seed=5, n_dirs=12, window=16):
    spec = CacheSpec(1, H, Hq, N, dtype="bf16", n_dirs=n_dirs, seed=seed, window=window)
    K, V, Q = make_layer(spec, 0)
    return K.double().numpy(), V.double().numpy(), Q.double().numpy(), spec


def _params(spec, theta, mode):
    return O.Params(n_tokens=spec.n_tokens, n_kv_heads=spec.n_kv_heads, n_q_heads=spec.n_q_heads, theta=theta,
                    dtype="bf16", seed=spec.seed, window=spec.window, mode=mode)


def _residual_norms_from_bytes(K, V, p, parts):
    """||x - gamma~ x_a||^2 per token-side, from the unpacked layout only."""
    H, N = p.n_kv_heads, p.n_tokens
    r2 = np.zeros((2, H, N))
    for side, (X, A) in enumerate(((K, parts["anchors_K"]), (V, parts["anchors_V"]))):
        for h in range(H):
            xa = A[h][parts["idx"][side, h]]
            r = X[h] - parts["g16"][side, h].astype(np.float64)[:, None] * xa
            r2[side, h] = (r * r).sum(axis=1)
    return r2


def _brute_top(u, eligible, R):
    flat = sorted((-u.reshape(-1)[f], f) for f in range(u.size) if eligible.reshape(-1)[f])
    return {f for _, f in flat[:R]}


def _selected(parts):
    return set(np.nonzero(parts["sel"].reshape(-1))[0].tolist())


def _eligible(p, parts):
    el = np.ones((2, p.n_kv_heads, p.n_tokens), bool)
    for h in range(p.n_kv_heads):
        el[:, h, parts["anchor_pos"][h]] = False
    return el


def test_key_query_proxy_is_the_trailing_keys():
    """[VQ] Adaptation notes: the trailing window key rows stand in as the
    queries for anchor selection and residual scoring."""
    K, V, Q, spec = _layer()
    p = _params(spec, 0.08, O.MODE_KEY_QUERIES)
    got = O.compress_layer(K, V, None, p)
    N, W, G = spec.n_tokens, spec.window, p.group
    Qk = np.stack([K[j // G, N - W:N] for j in range(p.n_q_heads)])
    want = O.compress_layer(K, V, Qk, _params(spec, 0.08, 0))
    assert np.array_equal(got["bytes"], want["bytes"])


def test_key_query_proxy_single_row_is_a_softmax_over_the_keys():
    """G = 1, W = 1: the one proxy query is the last key, which sees every
    position, so the score of t is softmax_t(K_{N-1}.K_t / sqrt(D))."""
    spec = CacheSpec(1, 1, 1, 300, dtype="bf16", n_dirs=8, seed=2, window=1)
    K, V, _ = make_layer(spec, 0)
    K, V = K.double().numpy(), V.double().numpy()
    p = _params(spec, 0.2, O.MODE_KEY_QUERIES)
    out = O.compress_layer(K, V, None, p)
    s = K[0] @ K[0, -1] / math.sqrt(128)
    want = np.exp(s - s.max())
    want /= want.sum()
    assert np.allclose(out["alpha"][0][0], want, rtol=0, atol=1e-14)


def test_rank_residual_norm_takes_the_largest_residuals():
    K, V, Q, spec = _layer(seed=6)
    p = _params(spec, 0.08, O.RANK_RESIDUAL_NORM << O.MODE_RANK_SHIFT)
    out = O.compress_layer(K, V, Q, p)
    parts = O.unpack_layout(out["bytes"], p)
    r2 = _residual_norms_from_bytes(K, V, p, parts)
    assert _selected(parts) == _brute_top(r2, _eligible(p, parts), out["layout"]["R"])


def test_rank_attention_takes_the_most_attended_tokens():
    K, V, Q, spec = _layer(seed=7)
    p = _params(spec, 0.08, O.RANK_ATTENTION << O.MODE_RANK_SHIFT)
    out = O.compress_layer(K, V, Q, p)
    parts = O.unpack_layout(out["bytes"], p)
    H, N, W, G = spec.n_kv_heads, spec.n_tokens, spec.window, p.group
    u = np.zeros((2, H, N))
    for h in range(H):
        for j in range(h * G, (h + 1) * G):
            for w in range(W):
                lim = N - W + w                           # causal observation row
                s = K[h, :lim + 1] @ Q[j, w] / math.sqrt(128)
                a = np.exp(s - s.max())
                u[:, h, :lim + 1] += a / a.sum()
    assert _selected(parts) == _brute_top(u, _eligible(p, parts), out["layout"]["R"])


def test_rank_cosine_takes_the_worst_approximated_tokens():
    K, V, Q, spec = _layer(seed=8)
    p = _params(spec, 0.08, O.RANK_COSINE << O.MODE_RANK_SHIFT)
    out = O.compress_layer(K, V, Q, p)
    parts = O.unpack_layout(out["bytes"], p)
    H, N = spec.n_kv_heads, spec.n_tokens
    u = np.zeros((2, H, N))
    for side, (X, A) in enumerate(((K, parts["anchors_K"]), (V, parts["anchors_V"]))):
        for h in range(H):
            xa = A[h][parts["idx"][side, h]]
            c = (X[h] * xa).sum(axis=1) / (np.linalg.norm(X[h], axis=1) * np.linalg.norm(xa, axis=1))
            u[side, h] = 1.0 - c
    assert _selected(parts) == _brute_top(u, _eligible(p, parts), out["layout"]["R"])


def test_rank_random_is_uniform_and_seeded():
    K, V, Q, spec = _layer(N=2000, H=2, seed=9, theta=0.1)
    mode = O.RANK_RANDOM << O.MODE_RANK_SHIFT
    p = _params(spec, 0.1, mode)
    a = O.compress_layer(K, V, Q, p)
    assert np.array_equal(O.compress_layer(K, V, Q, p)["bytes"], a["bytes"])     # deterministic
    other = O.Params(**{**p.__dict__, "seed": p.seed + 1})
    b = O.compress_layer(K, V, Q, other)
    assert not np.array_equal(a["sel"], b["sel"])                                 # keyed by the seed
    # the selection does not follow the utilities: each (side, head) gets its
    # share of the eligible token-sides (binomial), and positions are uniform
    el = a["eligible"]
    frac = a["layout"]["R"] / el.sum()
    for side in range(2):
        for h in range(2):
            n, k = el[side, h].sum(), a["sel"][side, h].sum()
            assert abs(k - n * frac) < 5 * math.sqrt(n * frac * (1 - frac))
    pos = np.nonzero(a["sel"].reshape(-1, spec.n_tokens))[1]
    hist = np.histogram(pos, bins=10, range=(0, spec.n_tokens - spec.window))[0]
    assert scipy.stats.chisquare(hist).pvalue > 1e-3


def test_random_rank_key_is_splitmix_top_bits():
    z = O.splitmix64((77 ^ O.RANK_SALT ^ (3 << 48) ^ 12345) & ((1 << 64) - 1))
    assert O.random_rank_key(77, 3, 12345) == (z >> 40) / 2.0 ** 24


def test_naive_codec_codes_the_residual_itself():
    """No rotation: the code of coordinate j is the nearest of the four levels
    to r_j / sigma~ (levels +-l1, +-l2, decision points 0 and +-tau)."""
    rng = np.random.default_rng(4)
    r = rng.normal(size=(200, 128)) * rng.lognormal(size=(200, 1))
    sig, codes, y = O.quantize_residuals(r, seed=3, naive=True)
    tau, l1, l2, _ = O.lloyd_max_gaussian_4()
    lev = np.array([-l2, -l1, l1, l2])
    z = r / sig.astype(np.float64)[:, None]
    nearest = np.abs(z[:, :, None] - lev[None, None, :]).argmin(axis=2)
    margin = np.abs(np.abs(z) - tau).min(axis=1)
    ok = margin > 1e-9                                  # rows clear of a decision point
    assert np.array_equal(codes[ok], nearest[ok])
    rt = O.dequantize_residuals(sig, codes, seed=3, naive=True)
    assert np.allclose(rt, lev[codes] * sig.astype(np.float64)[:, None])


def test_naive_codec_loses_what_the_rotation_spreads():
    """A residual concentrated in a few coordinates: the rotation spreads it
    (every rotated coordinate carries ||r||^2 / D), the naive codec cannot, so
    its error is far larger; for Gaussian residuals both match the Lloyd-Max
    distortion."""
    rng = np.random.default_rng(5)
    spiky = np.zeros((50, 128))
    spiky[np.arange(50), rng.integers(0, 128, 50)] = rng.normal(size=50) * 8
    err = {}
    for naive in (False, True):
        sig, codes, _ = O.quantize_residuals(spiky, seed=1, naive=naive)
        rt = O.dequantize_residuals(sig, codes, seed=1, naive=naive)
        err[naive] = (np.linalg.norm(spiky - rt, axis=1) ** 2 / np.linalg.norm(spiky, axis=1) ** 2).mean()
    assert err[True] > 3 * err[False]
    g = rng.normal(size=(3000, 128))
    sig, codes, _ = O.quantize_residuals(g, seed=1, naive=True)
    rt = O.dequantize_residuals(sig, codes, seed=1, naive=True)
    eta = (np.linalg.norm(g - rt, axis=1) ** 2 / np.linalg.norm(g, axis=1) ** 2).mean()
    assert abs(eta - O.lloyd_max_gaussian_4()[3]) < 0.01


def test_naive_codec_layout_reconstructs():
    K, V, Q, spec = _layer(seed=10, theta=0.15)
    p = _params(spec, 0.15, O.MODE_NAIVE_CODEC)
    out = O.compress_layer(K, V, Q, p)
    parts = O.unpack_layout(out["bytes"], p)
    Kh, Vh = O.reconstruct(parts, p)
    tau, l1, l2, _ = O.lloyd_max_gaussian_4()
    lev = np.array([-l2, -l1, l1, l2])
    sel = parts["sel"]
    rec = np.cumsum(sel.reshape(-1)).reshape(sel.shape) - 1
    for side, (X, A, Xh) in enumerate(((K, parts["anchors_K"], Kh), (V, parts["anchors_V"], Vh))):
        for h in range(spec.n_kv_heads):
            base = parts["g16"][side, h].astype(np.float64)[:, None] * A[h][parts["idx"][side, h]]
            for t in np.nonzero(sel[side, h])[0][:20]:
                i = rec[side, h, t]
                want = base[t] + lev[parts["codes"][i]] * float(parts["sigma16"][i])
                assert np.allclose(Xh[h, t], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [1 << 1 | 1, 5 << 1, 7 << 1])
def test_unknown_or_combined_modes(mode):
    """Combinations are allowed (key queries with any ranking); ranking values
    above 4 are not defined."""
    K, V, Q, spec = _layer(N=300, H=1, Hq=2, seed=11)
    p = _params(spec, 0.1, mode)
    if p.rank > O.RANK_RANDOM:
        with pytest.raises(ValueError):
            O.compress_layer(K, V, Q, p)
    else:
        out = O.compress_layer(K, V, None if p.key_queries else Q, p)
        assert out["sel"].sum() == out["layout"]["R"]


def test_mode_pins_catch_planted_mistakes(monkeypatch):
    """Swapped sides in the residual-norm ranking, or a naive codec that still
    rotates, must be caught by the pins above."""
    orig_rank = O.ranking_values

    def swapped(p, h, alpha, ybar, Qh, K_h, V_h, r2, cos, ap):
        uK, uV = orig_rank(p, h, alpha, ybar, Qh, K_h, V_h, r2, cos, ap)
        return (uV, uK) if p.rank == O.RANK_RESIDUAL_NORM else (uK, uV)
    monkeypatch.setattr(O, "ranking_values", swapped)
    with pytest.raises(AssertionError):
        test_rank_residual_norm_takes_the_largest_residuals()
    monkeypatch.setattr(O, "ranking_values", orig_rank)

    orig_q = O.quantize_residuals
    monkeypatch.setattr(O, "quantize_residuals", lambda r, seed, codebook=None, naive=False: orig_q(r, seed, codebook))
    with pytest.raises(AssertionError):
        test_naive_codec_codes_the_residual_itself()


# ---------------------------------------------------------------- rotary positions

def test_rope_is_orthogonal_and_linear():
    """[PITH] Section 3.2 as quoted in the review: R_t is orthogonal and linear,
    so it distributes over the anchor-residual decomposition."""
    rng = np.random.default_rng(20)
    X, Y = rng.normal(size=(50, 128)), rng.normal(size=(50, 128))
    pos = rng.integers(0, 200000, 50)
    RX = O.rope_rotate(X, pos, 500000.0)
    assert np.allclose(np.linalg.norm(RX, axis=1), np.linalg.norm(X, axis=1), rtol=1e-13)
    assert np.allclose(O.rope_rotate(2.5 * X - Y, pos, 500000.0), 2.5 * RX - O.rope_rotate(Y, pos, 500000.0),
                       rtol=0, atol=1e-11)


def test_rope_matches_complex_rotation_and_hand_values():
    """Pair (x_i, x_{i+D/2}) as the complex number x_i + i x_{i+D/2}, turned by
    exp(i p base^(-2i/D)); and a hand-worked D = 4 case."""
    rng = np.random.default_rng(21)
    X = rng.normal(size=(7, 128))
    pos = np.array([0, 1, 2, 31, 1000, 32767, 131071])
    z = X[:, :64] + 1j * X[:, 64:]
    w = z * np.exp(1j * pos[:, None] * 10000.0 ** (-np.arange(64) / 64.0)[None, :])
    assert np.allclose(O.rope_rotate(X, pos, 10000.0), np.concatenate([w.real, w.imag], axis=1), rtol=0, atol=1e-11)
    # D = 4, base 100: frequencies 1 and 100^(-1/2) = 0.1; x = e_0 and e_1 at p = 1
    got = O.rope_rotate(np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]]), np.array([1, 1]), 100.0)
    assert np.allclose(got[0], [math.cos(1), 0, math.sin(1), 0])
    assert np.allclose(got[1], [0, math.cos(0.1), 0, math.sin(0.1)])


def test_rope_scores_depend_on_relative_position():
    rng = np.random.default_rng(22)
    q, k = rng.normal(size=(1, 128)), rng.normal(size=(1, 128))
    for a, b in [(5, 17), (1000, 1003), (70000, 12)]:
        lhs = O.rope_rotate(q, [a], 500000.0) @ O.rope_rotate(k, [b], 500000.0).T
        rhs = q @ O.rope_rotate(k, [b - a], 500000.0).T
        assert abs(lhs - rhs) < 1e-10 * (1 + abs(rhs))


def test_rope_decode_is_attention_over_rotated_keys():
    """The decode with rotary positions equals textbook softmax attention of
    the rotated query over the rotated keys (positions 0..N-1, then the tail,
    query at N + T), values unrotated."""
    rng = np.random.default_rng(23)
    H, G, N, T, D = 2, 3, 40, 5, 128
    q = rng.normal(size=(H * G, D))
    K, V = rng.normal(size=(H, N, D)), rng.normal(size=(H, N, D))
    Kt, Vt = rng.normal(size=(H, T, D)), rng.normal(size=(H, T, D))
    o = O.decode_attention_rope(q, K, V, 1000.0, Kt, Vt)
    for j in range(H * G):
        h = j // G
        keys = np.concatenate([K[h], Kt[h]])
        vals = np.concatenate([V[h], Vt[h]])
        z = keys[:, :64] + 1j * keys[:, 64:]
        zq = q[j, :64] + 1j * q[j, 64:]
        f = 1000.0 ** (-np.arange(64) / 64.0)
        zr = z * np.exp(1j * np.arange(N + T)[:, None] * f[None, :])
        zqr = zq * np.exp(1j * (N + T) * f)
        s = (zr.real @ zqr.real + zr.imag @ zqr.imag) / math.sqrt(D)
        p = np.exp(s - s.max())
        assert np.allclose(o[j], (p / p.sum()) @ vals, rtol=0, atol=1e-12)
