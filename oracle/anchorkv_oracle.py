"""AnchorKV oracle: a plain, slow, fp64 CPU restatement of the anchor-residual
KV-cache codec (compress at the end of prefill, decode attention over the
compressed cache).

TEST INFRASTRUCTURE ONLY.  The test-suite, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers allowed.  The product path
(the CUDA library and its Python binding) never imports, calls or links
anything in this directory, and nothing here imports the product path.

Sources (web pages about arXiv 2608.02901, cited by title and section):
  [PITH]  "AnchorKV: Anchor-Residual KV Cache Compression" (pith.science
          machine review): "What carries the argument", "Referee Report"
          (Summary, Significance, major and minor comments), "Circularity
          Check", "Assumptions & free parameters".
  [VQ]    "AnchorKV-adapted - Anchor-Residual Compression, No Eviction"
          (VeloxQuant-MLX docs): "The one setting worth tuning:
          anchorkv_theta", "Adaptation notes", "Evidence".

Every function follows one step of the method in the pages' order.  Where the
pages name a step without printing it, the docstring says "Reading:" and gives
the reading taken; the same readings are listed in the repository's design
notes.  Arithmetic is float64 throughout, except where the pages fix a storage
precision (2-byte coefficient and scale, 2-bit codes, input-precision anchors).

Library primitives used as steps: numpy matmul, argsort/lexsort, exp, erfc.
No blocking, fusion or reordering beyond what the definitions state.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------
# Parameters and fixed hyper-parameters
# --------------------------------------------------------------------------

# Mode bits (Params.mode; the C ABI's anchorkv_params.mode):
MODE_KEY_QUERIES = 1        # [VQ] "Adaptation notes": trailing key rows as proxy queries
MODE_RANK_SHIFT = 1         # bits 1..3: ranking criterion of the residual budget
MODE_RANK_MASK = 7 << MODE_RANK_SHIFT
MODE_NAIVE_CODEC = 1 << 4   # [PITH] minor comments, Figure 5 "Naive 2 bit": no rotation
RANK_UTILITY, RANK_RESIDUAL_NORM, RANK_ATTENTION, RANK_COSINE, RANK_RANDOM = 0, 1, 2, 3, 4
RANK_SALT = 0x72616E6B5F726E64   # "rank_rnd": separates the ranking keys from the anchor sample

B_INDEX = 2      # b_a: bytes per anchor index   [PITH] "Assumptions & free parameters", codec parameters
B_GAMMA = 2      # b_gamma: bytes per coefficient [PITH] same entry
CODE_BITS = 2    # 2-bit residual codes            [PITH] same entry
TILE = 128       # token tile of the residual bitmap / prefix table (layout reading)


@dataclass
class Params:
    """One layer's compression problem.

    theta: retained fraction of the uncompressed byte cost, the single user
        knob ([VQ] "The one setting worth tuning"; [PITH] free parameter
        "retained fraction theta", Eq. 9).
    window: W trailing positions always kept as anchors and used as the
        observation queries ([PITH] free parameter "recency window W = 32").
    anchor_div: k = S/128 ([PITH] free parameter "anchor budget k").
    rho_num/rho_den: scored fraction rho = 0.7 ([PITH] "scored anchor fraction").
    pool_kernel: kappa = 7 ([PITH] "pooling kernel width kappa").
    seed: the one seed behind the uniform anchor sample and the shared
        Hadamard sign vector ([PITH] "fixed Hadamard seed").
    """
    n_tokens: int
    n_kv_heads: int
    n_q_heads: int
    theta: float
    head_dim: int = 128
    window: int = 32
    dtype: str = "bf16"          # storage precision of K, V, Q_obs and anchors
    seed: int = 0
    layer: int = 0
    anchor_div: int = 128
    rho_num: int = 7
    rho_den: int = 10
    pool_kernel: int = 7
    mode: int = 0                # MODE_* bits; 0 = the method as the pages describe it

    @property
    def key_queries(self) -> bool:
        return bool(self.mode & MODE_KEY_QUERIES)

    @property
    def rank(self) -> int:
        return (self.mode & MODE_RANK_MASK) >> MODE_RANK_SHIFT

    @property
    def naive_codec(self) -> bool:
        return bool(self.mode & MODE_NAIVE_CODEC)

    @property
    def elem_bytes(self) -> int:
        return {"fp32": 4, "bf16": 2}[self.dtype]

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


def _align16(x: int) -> int:
    return (x + 15) // 16 * 16


# --------------------------------------------------------------------------
# Counter-based generator (splitmix64) used for the uniform anchor sample and
# the Hadamard signs.  Published definition: Steele, Lea & Flood, "Fast
# splittable pseudorandom number generators", OOPSLA 2014 (the mix function of
# SplitMix64 applied to state + golden gamma).
# --------------------------------------------------------------------------

_M64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One SplitMix64 output for state ``x`` (python integers, mod 2^64)."""
    z = (x + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def anchor_hash_key(seed: int, layer: int, head: int, t: int) -> int:
    """Reading: the uniform anchor sample is keyed per (layer, head, position)
    as splitmix64(seed ^ layer<<48 ^ head<<32 ^ t)."""
    return splitmix64((seed ^ (layer << 48) ^ (head << 32) ^ t) & _M64)


def hadamard_signs(seed: int, d: int) -> np.ndarray:
    """Shared random signs s_j of the randomized Hadamard rotation.

    [PITH] "Assumptions & free parameters": randomized Hadamard rotation with a
    shared fixed seed.  Reading: s_j = -1 when bit 0 of
    splitmix64(seed ^ 2^63 ^ j) is set, else +1; one vector for every layer,
    head and side.
    """
    return np.array([-1.0 if splitmix64((seed ^ (1 << 63) ^ j) & _M64) & 1 else 1.0
                     for j in range(d)])


def hadamard_matrix(d: int) -> np.ndarray:
    """Orthonormal Sylvester-Hadamard matrix H_d / sqrt(d) (d a power of two)."""
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    assert h.shape[0] == d, "head_dim must be a power of two"
    return h / math.sqrt(d)


# --------------------------------------------------------------------------
# 2-bit Lloyd-Max codebook for a unit Gaussian
# --------------------------------------------------------------------------

def lloyd_max_gaussian_4(tol: float = 1e-15, max_iter: int = 100000):
    """Four-level Lloyd-Max quantizer for N(0,1), by Lloyd's iteration.

    [PITH] "Assumptions & free parameters": two bits per coordinate with a
    four-level Lloyd-Max codebook for a unit Gaussian source (Lloyd 1982 is in
    the pages' reference list).  By symmetry the cells are (-inf,-tau),
    [-tau,0), [0,tau), [tau,inf) with levels -l2, -l1, l1, l2.  Each pass sets
    every threshold to the midpoint of its neighbouring levels and every level
    to the conditional mean of its cell.  Returns (tau, l1, l2, mse).
    """
    phi = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    Phi = lambda x: 0.5 * math.erfc(-x / math.sqrt(2.0))
    l1, l2 = 0.5, 1.5
    for _ in range(max_iter):
        tau = 0.5 * (l1 + l2)
        n1 = (phi(0.0) - phi(tau)) / (Phi(tau) - 0.5)
        n2 = phi(tau) / (1.0 - Phi(tau))
        done = abs(n1 - l1) < tol and abs(n2 - l2) < tol
        l1, l2 = n1, n2
        if done:
            break
    tau = 0.5 * (l1 + l2)
    p1 = Phi(tau) - 0.5
    p2 = 1.0 - Phi(tau)
    mse = 1.0 - 2.0 * (p1 * l1 * l1 + p2 * l2 * l2)
    return tau, l1, l2, mse


# --------------------------------------------------------------------------
# Byte accounting (Eq. 13 reading) and the compressed layout
# --------------------------------------------------------------------------

def layout(p: Params) -> dict:
    """Anchor count, byte budget, residual count R and section offsets.

    [PITH] Referee Report "Summary": an exact byte accounting (Eq. 13) maps the
    knob to a per-layer residual budget; minor comment 1: b_a = b_gamma = 2.
    [VQ] "The one setting worth tuning": at small scale the budget can floor to
    zero residual slots.

    Reading (Eq. 13 is not printed):
      m     = ceil(N / anchor_div) non-window anchor slots, k = W + m
              (k = N when N - W <= m: every position is an anchor);
      U     = 2 * H * N * D * e            uncompressed bytes of the layer;
      B     = floor(theta * U)             (one IEEE double product);
      base  = bytes of the layout below with no residual record;
      c     = D * 2 / 8 + 2 = 34 B         codes + fp16 scale per residual;
      cap   = 2 * H * (N - k)              eligible (non-anchor) token-sides;
      R     = min(cap, max(0, floor((B - base) / c)));
      total = base + c * R  (<= B whenever R > 0).
    Layout sections, each starting on a 16-byte boundary, in this order:
      anchors_K [H][k][D] (input dtype), anchors_V [H][k][D], anchor_pos
      [H][k] int32, tok [2][H][N] uint32 (low 16 bits: anchor slot, high 16:
      fp16 gamma), bitmap [2][H][ceil(N/128)][4] uint32, tile_prefix
      [2][H][ceil(N/128)+1] int32 (global residual record index at each tile
      start), res_codes [R][D/4] uint8, res_sigma [R] fp16.
    """
    N, H, D, W, e = p.n_tokens, p.n_kv_heads, p.head_dim, p.window, p.elem_bytes
    m = -(-N // p.anchor_div)
    if N - W <= m:
        k, n_s, n_u = N, 0, 0
    else:
        k = W + m
        n_s = (p.rho_num * m) // p.rho_den
        n_u = m - n_s
    n_t = -(-N // TILE)
    sizes = [
        ("anchors_K", H * k * D * e),
        ("anchors_V", H * k * D * e),
        ("anchor_pos", 4 * H * k),
        ("tok", 4 * 2 * H * N),
        ("bitmap", 2 * H * n_t * 16),
        ("tile_prefix", 4 * 2 * H * (n_t + 1)),
    ]
    off = {}
    cur = 0
    for name, sz in sizes:
        off[name] = cur
        cur = _align16(cur + sz)
    base = cur
    c = D * CODE_BITS // 8 + B_GAMMA
    U = 2 * H * N * D * e
    B = math.floor(p.theta * float(U))
    cap = 2 * H * (N - k)
    R = min(cap, max(0, (B - base) // c))
    off["res_codes"] = base
    off["res_sigma"] = base + (D * CODE_BITS // 8) * R
    total = base + c * R
    return dict(m=m, k=k, n_s=n_s, n_u=n_u, n_tiles=n_t, U=U, B=B, base=base,
                c=c, cap=cap, R=R, total=total, off=off, sizes=dict(sizes))


# --------------------------------------------------------------------------
# a1: observation-window attention score (SnapKV-style, Eq. 14)
# --------------------------------------------------------------------------

def obs_attention(Qh: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, window: int) -> dict:
    """Exact attention of the observation queries of one KV head.

    [PITH] "What carries the argument" (SnapKV observation-window score) and
    free parameter W: the final W positions are the observation queries.
    Qh: [G*W, D] rows ordered (query head j, window slot w) -> r = j*W + w;
    query (j, w) sits at position N - W + w and (Reading) sees t <= N - W + w,
    as in a causal prefill.  Returns alpha [G*W, N] (softmax weights, zero where
    masked), ybar [G*W, D] = alpha @ V (exact attention output), and the logits.
    """
    R_, D = Qh.shape
    N = Kh.shape[0]
    W = window
    s = (Qh @ Kh.T) / math.sqrt(D)
    w_of_row = np.arange(R_) % W
    limit = N - W + w_of_row                      # last visible position per row
    visible = np.arange(N)[None, :] <= limit[:, None]
    s_masked = np.where(visible, s, -np.inf)
    M = s_masked.max(axis=1, keepdims=True)
    E = np.where(visible, np.exp(s_masked - M), 0.0)
    Z = E.sum(axis=1, keepdims=True)
    alpha = E / Z
    ybar = alpha @ Vh
    return dict(alpha=alpha, ybar=ybar, logits=s, M=M[:, 0], Z=Z[:, 0])


def token_scores(alpha: np.ndarray, n_tokens: int, window: int) -> np.ndarray:
    """score_t = sum over observation rows (all G query heads of the KV head and
    all W window queries) of alpha, for the non-window positions t < N - W.

    [PITH] "Assumptions & free parameters": the last W tokens' attention is
    pooled over GQA query heads.  Reading: pooling is a plain sum (it ranks
    exactly like the mean).
    """
    return alpha[:, : n_tokens - window].sum(axis=0)


def pool_scores(score: np.ndarray, kappa: int) -> np.ndarray:
    """Positional pooling of width kappa (Eq. 14's kernel).

    Reading: average pooling, stride 1, centred window of kappa positions,
    zero padding outside [0, N - W), always divided by kappa.
    """
    n = score.shape[0]
    h = kappa // 2
    padded = np.concatenate([np.zeros(h), score, np.zeros(h)])
    out = np.zeros(n)
    for d in range(kappa):
        out += padded[d:d + n]
    return out / kappa


# --------------------------------------------------------------------------
# a2: anchor selection
# --------------------------------------------------------------------------

def select_anchors(pooled: np.ndarray, p: Params, head: int, scored: np.ndarray | None = None) -> np.ndarray:
    """Anchor positions of one KV head, ascending (slot s <-> position).

    [PITH] free parameters: the final W positions are always anchors; a
    fraction rho = 0.7 of the non-window slots goes to the highest pooled
    scores, the rest is a uniform sample; k = S/128.
    Reading: m = ceil(N/128) non-window slots, n_s = floor(7m/10) by score
    (ties -> lower position), n_u = m - n_s drawn without replacement from the
    remaining non-window positions as the n_u smallest counter-based hash keys
    (ties -> lower position).  If N - W <= m every position is an anchor.
    ``scored`` may carry the scored positions to use instead of recomputing
    them (tests use it to check the uniform sample on its own).
    """
    N, W = p.n_tokens, p.window
    L = layout(p)
    if L["k"] == N:
        return np.arange(N, dtype=np.int64)
    n_s, n_u = L["n_s"], L["n_u"]
    t = np.arange(N - W)
    if scored is None:
        order = np.lexsort((t, -pooled))        # primary: pooled desc; then t asc
        scored = order[:n_s]
    scored = np.asarray(scored, dtype=np.int64)
    taken = np.zeros(N - W, dtype=bool)
    taken[scored] = True
    rest = t[~taken]
    keys = np.array([anchor_hash_key(p.seed, p.layer, head, int(x)) for x in rest],
                    dtype=np.uint64)
    pick = rest[np.lexsort((rest, keys))[:n_u]]
    anchors = np.concatenate([scored, pick, np.arange(N - W, N)])
    return np.sort(anchors).astype(np.int64)


# --------------------------------------------------------------------------
# a3: nearest-anchor assignment, a4: coefficient and residual
# --------------------------------------------------------------------------

def assign(X: np.ndarray, anchor_pos: np.ndarray):
    """Nearest anchor of every token of one side (keys or values) of one head.

    [PITH] Referee "Summary": each key and value vector is assigned to its
    nearest anchor; [VQ] "one index, one coefficient per side".
    Reading: "nearest" = largest signed cosine, i.e. argmax over slots of
    <x, a_s> / ||a_s|| (||x|| is common to the row); a zero anchor scores 0;
    ties -> lowest slot; an anchor token takes its own slot.
    Returns (idx [N], dots [N, k], cos [N, k]).
    """
    A = X[anchor_pos]
    dots = X @ A.T
    n2 = (A * A).sum(axis=1)
    nrm = np.sqrt(n2)
    safe = np.where(nrm > 0, nrm, 1.0)
    cos = np.where(nrm[None, :] > 0, dots / safe[None, :], 0.0)
    idx = np.argmax(cos, axis=1)                # first maximum = lowest slot
    idx[anchor_pos] = np.arange(anchor_pos.shape[0])
    return idx.astype(np.int64), dots, cos


def to_fp16(x):
    """Round to fp16, nearest-even, saturating at +-65504 (Reading: the 2-byte
    coefficient/scale format is IEEE half)."""
    return np.asarray(np.clip(x, -65504.0, 65504.0), dtype=np.float64).astype(np.float16)


def project(X: np.ndarray, anchor_pos: np.ndarray, idx: np.ndarray):
    """gamma_i = <x_i, x_a> / ||x_a||^2 and r_i = x_i - gamma~_i x_a.

    [PITH] "What carries the argument": gamma_i = <x_i, x_a(i)>/||x_a(i)||^2,
    x^_i = gamma_i x_a(i) + r~_i.  [VQ] "Evidence": an anchor projected on
    itself has coefficient 1 and zero residual.
    Reading: gamma is stored as fp16 (b_gamma = 2 bytes) and the residual is
    taken against the stored gamma~ so that gamma~ x_a + r is exactly x; a zero
    anchor gives gamma = 0.
    Returns (gamma fp64, gamma~ as fp16 array, r [N, D], ||r||^2 [N]).
    """
    A = X[anchor_pos]
    xa = A[idx]
    n2 = (xa * xa).sum(axis=1)
    dot = (X * xa).sum(axis=1)
    gamma = np.where(n2 > 0, dot / np.where(n2 > 0, n2, 1.0), 0.0)
    gamma[anchor_pos] = 1.0
    g16 = to_fp16(gamma)
    r = X - g16.astype(np.float64)[:, None] * xa
    r[anchor_pos] = 0.0
    return gamma, g16, r, (r * r).sum(axis=1)


# --------------------------------------------------------------------------
# a4: first-order attention-output utility (Eq. 5 / Eq. 6 / Eq. 16 reading)
# --------------------------------------------------------------------------

def utilities(alpha: np.ndarray, ybar: np.ndarray, Qh: np.ndarray, Vh: np.ndarray,
              r2K: np.ndarray, r2V: np.ndarray, anchor_pos: np.ndarray):
    """Value- and key-induced utility of giving token t its residual.

    [PITH] "Circularity Check" / "Assumptions": Delta y is expanded to first
    order in the logit and value perturbations (softmax Jacobian
    d alpha_t/d s_u = alpha_t(delta_tu - alpha_u)); under the incoherence model
    per-token errors are zero-mean and independent, so E||Delta y||^2 is a sum
    of per-token key and value terms (Eq. 16).
    Reading (the equations are not printed): leaving r_t out perturbs
      value channel: Delta y_r = alpha_rt * r^V_t  ->  ||.||^2 = alpha_rt^2 ||r^V_t||^2
      key channel:   Delta s_rt = q_r . r^K_t / sqrt(D),
                     Delta y_r = alpha_rt (V_t - ybar_r) Delta s_rt, and for an
                     isotropic residual direction E (q.r)^2 = ||q||^2 ||r||^2 / D
    so, summed over the observation rows r,
      u^V_t = ||r^V_t||^2 * sum_r alpha_rt^2
      u^K_t = ||r^K_t||^2 / D^2 * sum_r alpha_rt^2 ||q_r||^2 ||V_t - ybar_r||^2.
    The common factor (1 - eta) of the fixed codec distortion is dropped (it
    does not change the ranking).  Anchors get utility 0 and are ineligible.
    """
    D = Qh.shape[1]
    a2 = alpha * alpha                                   # [GW, N]
    uV = r2V * a2.sum(axis=0)
    q2 = (Qh * Qh).sum(axis=1)                           # [GW]
    v2 = (Vh * Vh).sum(axis=1)                           # [N]
    y2 = (ybar * ybar).sum(axis=1)                       # [GW]
    vy = Vh @ ybar.T                                     # [N, GW]
    dist2 = v2[:, None] - 2.0 * vy + y2[None, :]         # ||V_t - ybar_r||^2
    ku = (a2.T * q2[None, :] * dist2).sum(axis=1)
    uK = r2K / (D * D) * ku
    uK[anchor_pos] = 0.0
    uV[anchor_pos] = 0.0
    return uK, uV


def key_queries(K: np.ndarray, p: Params) -> np.ndarray:
    """Proxy observation queries built from the keys alone: [Hq, W, D].

    [VQ] "Adaptation notes" (key-as-query proxy): a cache wrapper never sees
    queries, so the trailing anchorkv_window key rows stand in as the queries
    for both anchor selection and residual scoring.
    Reading: every query head j of KV head h = j // G uses K[h, N-W : N]
    (the G copies rank exactly like one copy); each proxy row keeps its
    position N - W + w, so the causal mask is unchanged.
    """
    H, N, D = K.shape
    W, G = p.window, p.group
    Q = np.zeros((p.n_q_heads, W, D))
    for j in range(p.n_q_heads):
        Q[j] = K[j // G, N - W:N]
    return Q


def random_rank_key(seed: int, layer: int, f: int) -> float:
    """Uniform ranking value in [0, 1) of flat token-side f: the top 24 bits of
    a SplitMix64 output (a 24-bit integer over 2^24, exact in fp32)."""
    z = splitmix64((seed ^ RANK_SALT ^ ((layer & 0x7FFF) << 48) ^ f) & _M64)
    return float(z >> 40) / float(1 << 24)


def ranking_values(p: Params, h: int, alpha: np.ndarray, ybar: np.ndarray, Qh: np.ndarray,
                   K_h: np.ndarray, V_h: np.ndarray, r2: np.ndarray, cos: list, anchor_pos: np.ndarray):
    """Per-side ranking values (uK, uV) of one head under the selected criterion.

    [PITH] "Circularity Check": the utility ranking is validated against
    random, attention, residual-norm and cosine alternatives (Figure 5).
    Readings (the alternatives are named, not defined):
      utility        the first-order utility (``utilities``);
      residual norm  ||r_t||^2 of the side;
      attention      sum over observation rows of alpha_rt (the un-pooled
                     observation score), the same for both sides;
      cosine         1 - cos(x_t, x_a(t)) (worst-approximated first; a zero
                     vector has cosine 0);
      random         ``random_rank_key`` of the flat index f.
    Anchors get 0 and are ineligible.  cos: per side, the true cosine of each
    token with its assigned anchor.
    """
    N = K_h.shape[0]
    H = p.n_kv_heads
    if p.rank == RANK_UTILITY:
        return utilities(alpha, ybar, Qh, V_h, r2[0], r2[1], anchor_pos)
    out = []
    for side in range(2):
        if p.rank == RANK_RESIDUAL_NORM:
            u = r2[side].copy()
        elif p.rank == RANK_ATTENTION:
            u = alpha.sum(axis=0)
        elif p.rank == RANK_COSINE:
            u = 1.0 - cos[side]
        elif p.rank == RANK_RANDOM:
            base = (side * H + h) * N
            u = np.array([random_rank_key(p.seed, p.layer, base + t) for t in range(N)])
        else:
            raise ValueError("unknown ranking criterion")
        u[anchor_pos] = 0.0
        out.append(u)
    return out[0], out[1]


def assigned_cosine(X: np.ndarray, anchor_pos: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """cos(x_t, x_a(t)) = <x, a> / (||x|| ||a||), 0 when either norm is 0."""
    xa = X[anchor_pos][idx]
    den = np.sqrt((X * X).sum(axis=1) * (xa * xa).sum(axis=1))
    dot = (X * xa).sum(axis=1)
    return np.where(den > 0, dot / np.where(den > 0, den, 1.0), 0.0)


# --------------------------------------------------------------------------
# a5: per-layer residual budget, pooled over heads and sides
# --------------------------------------------------------------------------

def select_residuals(u: np.ndarray, eligible: np.ndarray, R: int) -> np.ndarray:
    """The R largest utilities of the layer over all token-sides.

    [VQ] "Evidence": the residual budget pools across heads and favours the
    head with higher estimated utility; [PITH] "Referee Report": 17.3% of
    token-sides carry residuals at 20x (the budget is counted in token-sides).
    Reading: one pool per layer over both sides and all KV heads; flat index
    f = (side * H + h) * N + t with side 0 = keys; ties -> lower f.
    u, eligible: [2, H, N].  Returns a boolean mask [2, H, N].
    """
    flat_u = u.reshape(-1)
    flat_e = eligible.reshape(-1)
    f = np.nonzero(flat_e)[0]
    order = f[np.lexsort((f, -flat_u[f]))]
    sel = np.zeros(flat_u.shape[0], dtype=bool)
    sel[order[:R]] = True
    return sel.reshape(u.shape)


# --------------------------------------------------------------------------
# a6: randomized Hadamard rotation + 2-bit Lloyd-Max quantization + packing
# --------------------------------------------------------------------------

def quantize_residuals(r: np.ndarray, seed: int, codebook=None, naive: bool = False):
    """Encode residual rows r [n, D] to (sigma~ fp16 [n], codes [n, D] in 0..3).

    [PITH] Referee "Summary": 2-bit Hadamard-rotated, Lloyd-Max-quantized
    residuals; "Assumptions": after the randomized rotation each coordinate is
    about N(0, ||r||^2 / D), which justifies the unit-Gaussian codebook.
    Reading: y = H_D (s * r) with the orthonormal Sylvester matrix and the
    shared signs s; one fp16 scale sigma~ = fp16(||r|| / sqrt(D)) per residual
    vector (group = the whole head vector); code = 3 if y >= tau sigma~,
    2 if y >= 0, 1 if y >= -tau sigma~, else 0.
    naive: the ablation of [PITH] Figure 5 ("Naive 2 bit", minor comments);
    Reading: the same scale and codebook applied to r itself (no sign flip,
    no rotation), y = r.
    Returns (sigma16, codes, y).
    """
    D = r.shape[1]
    if codebook is None:
        codebook = lloyd_max_gaussian_4()
    tau = codebook[0]
    if naive:
        y = r.copy()
    else:
        s = hadamard_signs(seed, D)
        H = hadamard_matrix(D)
        y = (r * s[None, :]) @ H.T
    sigma = np.sqrt((r * r).sum(axis=1) / D)
    sig16 = to_fp16(sigma)
    th = tau * sig16.astype(np.float64)[:, None]
    codes = np.where(y >= th, 3, np.where(y >= 0.0, 2, np.where(y >= -th, 1, 0)))
    return sig16, codes.astype(np.uint8), y


def dequantize_residuals(sig16: np.ndarray, codes: np.ndarray, seed: int, codebook=None, naive: bool = False):
    """r~ = s * H_D (sigma~ * level(code)); H_D is symmetric and its own inverse.
    naive: r~ = sigma~ * level(code)."""
    D = codes.shape[1]
    if codebook is None:
        codebook = lloyd_max_gaussian_4()
    _, l1, l2, _ = codebook
    lev = np.array([-l2, -l1, l1, l2])
    z = lev[codes.astype(np.int64)] * sig16.astype(np.float64)[:, None]
    if naive:
        return z
    H = hadamard_matrix(D)
    return (z @ H.T) * hadamard_signs(seed, D)[None, :]


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Four 2-bit codes per byte: coordinate j -> byte j/4, bits 2*(j mod 4)."""
    n, D = codes.shape
    c = codes.reshape(n, D // 4, 4).astype(np.uint8)
    return (c[:, :, 0] | (c[:, :, 1] << 2) | (c[:, :, 2] << 4) | (c[:, :, 3] << 6)).astype(np.uint8)


def unpack_codes(packed: np.ndarray, D: int) -> np.ndarray:
    n = packed.shape[0]
    out = np.zeros((n, D), dtype=np.uint8)
    for q in range(4):
        out[:, q::4] = (packed >> (2 * q)) & 3
    return out


# --------------------------------------------------------------------------
# Whole-layer compress (the stages chained) and the byte image of the layout
# --------------------------------------------------------------------------

def _as_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Byte image of values that are exactly representable in ``dtype``."""
    f32 = np.asarray(x, dtype=np.float32)
    if dtype == "fp32":
        return f32.view(np.uint8).reshape(-1)
    bits = f32.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "value not representable in bf16"
    return (bits >> 16).astype(np.uint16).view(np.uint8).reshape(-1)


def compress_layer(K: np.ndarray, V: np.ndarray, Q: np.ndarray, p: Params,
                   stages: dict | None = None) -> dict:
    """Run every compress stage for one layer and build its byte layout.

    K, V: [H, N, D] and Q: [Hq, W, D], float64 holding the stored values.
    ``stages`` may carry decisions to use instead of recomputing them
    (keys "anchor_pos" [H, k], "idx" [2, H, N], "sel" [2, H, N]); tests use it
    to check each stage given the previous stage's result.
    """
    stages = stages or {}
    H, N, D = K.shape
    G, W = p.group, p.window
    if p.key_queries:
        Q = key_queries(K, p)
    L = layout(p)
    k = L["k"]
    out = dict(layout=L, anchor_pos=np.zeros((H, k), np.int64),
               pooled=np.zeros((H, max(N - W, 0))), idx=np.zeros((2, H, N), np.int64),
               gamma=np.zeros((2, H, N)), g16=np.zeros((2, H, N), np.float16),
               r=np.zeros((2, H, N, D)), r2=np.zeros((2, H, N)), u=np.zeros((2, H, N)),
               eligible=np.ones((2, H, N), bool), alpha=[], ybar=[], cos=[[None] * H, [None] * H])
    for h in range(H):
        Qh = Q[h * G:(h + 1) * G].reshape(G * W, D)
        att = obs_attention(Qh, K[h], V[h], W)
        out["alpha"].append(att["alpha"])
        out["ybar"].append(att["ybar"])
        score = token_scores(att["alpha"], N, W)
        pooled = pool_scores(score, p.pool_kernel)
        out["pooled"][h] = pooled
        ap = stages["anchor_pos"][h] if "anchor_pos" in stages else select_anchors(pooled, p, h)
        ap = np.asarray(ap, np.int64)
        out["anchor_pos"][h] = ap
        out["eligible"][:, h, ap] = False
        acos = []
        for side, X in enumerate((K[h], V[h])):
            idx, _, cos = assign(X, ap)
            if "idx" in stages:
                idx = np.asarray(stages["idx"][side, h], np.int64)
            out["cos"][side][h] = cos
            out["idx"][side, h] = idx
            g, g16, r, r2 = project(X, ap, idx)
            out["gamma"][side, h], out["g16"][side, h] = g, g16
            out["r"][side, h], out["r2"][side, h] = r, r2
            acos.append(assigned_cosine(X, ap, idx))
        uK, uV = ranking_values(p, h, att["alpha"], att["ybar"], Qh, K[h], V[h], out["r2"][:, h], acos, ap)
        out["u"][0, h], out["u"][1, h] = uK, uV
    sel = stages["sel"] if "sel" in stages else select_residuals(out["u"], out["eligible"], L["R"])
    out["sel"] = np.asarray(sel, bool)
    rows = out["r"][out["sel"]]                         # flat (side, h, t) order
    sig16, codes, y = quantize_residuals(rows, p.seed, naive=p.naive_codec)
    out["sigma16"], out["codes"], out["y"] = sig16, codes, y
    out["bytes"] = pack_layout(p, K, V, out)
    return out


def pack_layout(p: Params, K: np.ndarray, V: np.ndarray, st: dict) -> np.ndarray:
    """Byte image of the compressed layer (sections as in ``layout``)."""
    L = layout(p)
    H, N, D = K.shape
    k, n_t, R = L["k"], L["n_tiles"], L["R"]
    buf = np.zeros(L["total"], dtype=np.uint8)
    o = L["off"]
    ap = st["anchor_pos"]
    aK = np.stack([K[h][ap[h]] for h in range(H)])
    aV = np.stack([V[h][ap[h]] for h in range(H)])
    nb = H * k * D * p.elem_bytes
    buf[o["anchors_K"]:o["anchors_K"] + nb] = _as_storage(aK, p.dtype)
    buf[o["anchors_V"]:o["anchors_V"] + nb] = _as_storage(aV, p.dtype)
    buf[o["anchor_pos"]:o["anchor_pos"] + 4 * H * k] = ap.astype(np.int32).view(np.uint8).reshape(-1)
    tok = st["idx"].astype(np.uint32) | (st["g16"].view(np.uint16).astype(np.uint32) << 16)
    buf[o["tok"]:o["tok"] + 8 * H * N] = tok.astype(np.uint32).view(np.uint8).reshape(-1)
    sel = st["sel"]
    bits = np.zeros((2, H, n_t * TILE), dtype=np.uint64)
    bits[:, :, :N] = sel
    words = np.zeros((2, H, n_t, 4), dtype=np.uint32)
    for wd in range(n_t * 4):
        chunk = bits[:, :, wd * 32:(wd + 1) * 32]
        val = np.zeros((2, H), dtype=np.uint64)
        for b in range(32):
            val |= chunk[:, :, b] << np.uint64(b)
        words[:, :, wd // 4, wd % 4] = val.astype(np.uint32)
    buf[o["bitmap"]:o["bitmap"] + 2 * H * n_t * 16] = words.view(np.uint8).reshape(-1)
    per_tile = sel.reshape(2, H, -1)
    counts = np.zeros((2, H, n_t), dtype=np.int64)
    for t in range(n_t):
        counts[:, :, t] = per_tile[:, :, t * TILE:min((t + 1) * TILE, N)].sum(axis=2)
    flat = counts.reshape(-1)
    starts = np.concatenate([[0], np.cumsum(flat)])    # record index at each tile start
    prefix = np.zeros((2, H, n_t + 1), dtype=np.int64)
    cursor = 0
    for sh in range(2 * H):
        s_, h_ = divmod(sh, H)
        prefix[s_, h_, :n_t] = starts[cursor:cursor + n_t]
        prefix[s_, h_, n_t] = starts[cursor + n_t]
        cursor += n_t
    buf[o["tile_prefix"]:o["tile_prefix"] + 4 * 2 * H * (n_t + 1)] = \
        prefix.astype(np.int32).view(np.uint8).reshape(-1)
    if R:
        buf[o["res_codes"]:o["res_codes"] + R * D // 4] = pack_codes(st["codes"]).reshape(-1)
        buf[o["res_sigma"]:o["res_sigma"] + 2 * R] = st["sigma16"].view(np.uint8).reshape(-1)
    return buf


def unpack_layout(buf: np.ndarray, p: Params) -> dict:
    """Parse a compressed layer image back into arrays (inverse of pack_layout)."""
    L = layout(p)
    H, N, D, k, n_t, R = p.n_kv_heads, p.n_tokens, p.head_dim, L["k"], L["n_tiles"], L["R"]
    o = L["off"]
    buf = np.asarray(buf, dtype=np.uint8)

    def sec(name, nbytes):
        return buf[o[name]:o[name] + nbytes]

    def anchors(name):
        raw = sec(name, H * k * D * p.elem_bytes)
        if p.dtype == "fp32":
            v = raw.view(np.float32)
        else:
            v = (raw.view(np.uint16).astype(np.uint32) << 16).view(np.float32)
        return v.astype(np.float64).reshape(H, k, D)

    tok = sec("tok", 8 * H * N).view(np.uint32).reshape(2, H, N)
    words = sec("bitmap", 2 * H * n_t * 16).view(np.uint32).reshape(2, H, n_t * 4)
    sel = np.zeros((2, H, n_t * TILE), dtype=bool)
    for b in range(32):
        sel[:, :, b::32] = (words >> b) & 1
    return dict(
        anchors_K=anchors("anchors_K"), anchors_V=anchors("anchors_V"),
        anchor_pos=sec("anchor_pos", 4 * H * k).view(np.int32).reshape(H, k).astype(np.int64),
        idx=(tok & 0xFFFF).astype(np.int64),
        g16=(tok >> 16).astype(np.uint16).view(np.float16),
        sel=sel[:, :, :N],
        tile_prefix=sec("tile_prefix", 4 * 2 * H * (n_t + 1)).view(np.int32).reshape(2, H, n_t + 1),
        codes=unpack_codes(buf[o["res_codes"]:o["res_codes"] + R * D // 4].reshape(R, D // 4), D)
        if R else np.zeros((0, D), np.uint8),
        sigma16=buf[o["res_sigma"]:o["res_sigma"] + 2 * R].view(np.float16) if R else np.zeros(0, np.float16),
    )


def reconstruct(parts: dict, p: Params, identity_residuals: np.ndarray | None = None):
    """K^, V^ [H, N, D] from a parsed layout: x^_t = gamma~_t x_a(t) + r~_t.

    [PITH] "What carries the argument".  ``identity_residuals`` ([2, H, N, D])
    replaces the 2-bit codec by the exact residual (a test device that turns
    the decode into plain attention).
    """
    H, N, D = p.n_kv_heads, p.n_tokens, p.head_dim
    out = []
    res_rows = None
    if parts["codes"].shape[0]:
        res_rows = dequantize_residuals(parts["sigma16"], parts["codes"], p.seed, naive=p.naive_codec)
    cursor = 0
    flat_sel = parts["sel"].reshape(-1)
    rec_of = np.cumsum(flat_sel) - 1                    # record index per token-side
    rec_of = rec_of.reshape(2, H, N)
    for side, A in enumerate((parts["anchors_K"], parts["anchors_V"])):
        Xh = np.zeros((H, N, D))
        for h in range(H):
            Xh[h] = parts["g16"][side, h].astype(np.float64)[:, None] * A[h][parts["idx"][side, h]]
            sel = parts["sel"][side, h]
            if identity_residuals is not None:
                Xh[h][sel] += identity_residuals[side, h][sel]
            elif res_rows is not None and sel.any():
                Xh[h][sel] += res_rows[rec_of[side, h][sel]]
        out.append(Xh)
        cursor += 1
    return out[0], out[1]


# --------------------------------------------------------------------------
# a7: decode attention over the compressed cache (+ exact appended tail)
# --------------------------------------------------------------------------

def decode_attention(q: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray,
                     Ktail: np.ndarray | None = None, Vtail: np.ndarray | None = None) -> np.ndarray:
    """o_j = softmax_t(q_j . K_t / sqrt(D)) V over the N reconstructed prefix
    tokens and the T tokens appended exactly during decode.

    [VQ] "Adaptation notes": decode tokens are appended at full precision and
    never re-anchored; [PITH] Referee "Summary": a FlashAttention-style
    decoder reconstructs tiles as they are consumed (same result as the dense
    rebuild written here).  q: [Hq, D]; Khat, Vhat: [H, N, D]; tails [H, T, D].
    No mask: the decode query is newer than every cached token.
    """
    Hq, D = q.shape
    H = Khat.shape[0]
    G = Hq // H
    o = np.zeros((Hq, D))
    for j in range(Hq):
        h = j // G
        Kf, Vf = Khat[h], Vhat[h]
        if Ktail is not None and Ktail.shape[1]:
            Kf = np.concatenate([Kf, Ktail[h]], axis=0)
            Vf = np.concatenate([Vf, Vtail[h]], axis=0)
        s = Kf @ q[j] / math.sqrt(D)
        w = np.exp(s - s.max())
        o[j] = (w / w.sum()) @ Vf
    return o


# --------------------------------------------------------------------------
# a7 with rotary positions: keys stored pre-RoPE, rotated at decode
# --------------------------------------------------------------------------

def rope_rotate(X: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """R_p x for every row: the rotary position map of each row's position.

    [PITH] "Assumptions & free parameters" (standard math, Section 3.2): RoPE
    is a per-position orthogonal linear map R_t, so R_t K_t = R_t K~_t +
    R_t r_t and ||R_t r_t|| = ||r_t||, which justifies storing keys pre-RoPE
    and rotating them at decode time.
    Reading (the pages name no convention): the rotate-half pairing of
    Llama-family models, coordinate i paired with i + D/2 for i < D/2 and
    turned by the angle p * base^(-2i/D).
    X: [n, D]; positions: [n] integers.
    """
    n, D = X.shape
    half = D // 2
    inv = base ** (-2.0 * np.arange(half) / D)
    ang = np.asarray(positions, np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = X[:, :half], X[:, half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=1)


def decode_attention_rope(q: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray, base: float,
                          Ktail: np.ndarray | None = None, Vtail: np.ndarray | None = None) -> np.ndarray:
    """Decode attention when the cached keys are stored before the rotary map.

    [PITH] "Assumptions & free parameters": pre-RoPE storage, rotation at
    decode time.  Reading: cached token t sits at position t, appended tail
    token i at N + i, and the decode query at N + T (the position of the token
    being decoded); keys and the query are rotated at their positions, values
    are not; no mask.  q: [Hq, D]; Khat, Vhat: [H, N, D]; tails [H, T, D].
    """
    Hq, D = q.shape
    H, N, _ = Khat.shape
    G = Hq // H
    T = 0 if Ktail is None else Ktail.shape[1]
    pos = np.arange(N + T)
    o = np.zeros((Hq, D))
    for j in range(Hq):
        h = j // G
        Kf, Vf = Khat[h], Vhat[h]
        if T:
            Kf = np.concatenate([Kf, Ktail[h]], axis=0)
            Vf = np.concatenate([Vf, Vtail[h]], axis=0)
        kr = rope_rotate(Kf, pos, base)
        qr = rope_rotate(q[j][None, :], np.array([N + T]), base)[0]
        s = kr @ qr / math.sqrt(D)
        w = np.exp(s - s.max())
        o[j] = (w / w.sum()) @ Vf
    return o


# --------------------------------------------------------------------------
# Theorem 1 (output-error bound) terms
# --------------------------------------------------------------------------

def theorem1(q: np.ndarray, K: np.ndarray, V: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray) -> dict:
    """Per-query error ||y^ - y|| and the two Theorem-1 bounds, for one head.

    [PITH] "What carries the argument" and major comment (Eq. 17): the output
    error is at most an attention-weighted value term plus 2 V_max tanh(mu),
    mu = ||q|| Delta_K / sqrt(D), Delta_K = max_t ||K_t - K^_t||.
    Reading (which weights and which V_max are not printed): both provable
    pairings are returned - (alpha^, max||V||) and (alpha, max||V^||).
    q: [nq, D]; K, V, Khat, Vhat: [N, D].
    """
    D = K.shape[1]
    dK = math.sqrt(((K - Khat) ** 2).sum(axis=1).max())
    dV = np.sqrt(((V - Vhat) ** 2).sum(axis=1))
    vmax = math.sqrt((V * V).sum(axis=1).max())
    vhmax = math.sqrt((Vhat * Vhat).sum(axis=1).max())
    res = dict(err=[], bound_a=[], bound_b=[], mu=[])
    for x in q:
        s = K @ x / math.sqrt(D)
        sh = Khat @ x / math.sqrt(D)
        a = np.exp(s - s.max()); a /= a.sum()
        ah = np.exp(sh - sh.max()); ah /= ah.sum()
        mu = np.linalg.norm(x) * dK / math.sqrt(D)
        res["err"].append(np.linalg.norm(ah @ Vhat - a @ V))
        res["bound_a"].append(float(ah @ dV) + 2.0 * vmax * math.tanh(mu))
        res["bound_b"].append(float(a @ dV) + 2.0 * vhmax * math.tanh(mu))
        res["mu"].append(mu)
    return {k_: np.array(v) for k_, v in res.items()}
