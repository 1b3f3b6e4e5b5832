"""fp64 CPU oracle for the ZipMap global large-chunk TTT layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` may call it.  It shares no code with the CUDA
path (``recon_chunk_ttt_b200``); both only consume the seeded arrays of
``recon_chunk_ttt_b200.workloads``.

Sources (pages on the web, cited by title and section):
  [review]  kimjy99, "[논문리뷰] ZipMap: Linear-Time Stateful 3D Reconstruction
            via Test-Time Training", section 2 "Feature Backbone" (Eq. 1
            SwiGLU fast weights, Eq. 2 virtual loss, Eq. 3 eta-weighted
            gradient, Newton-Schulz + L2 renormalisation, apply o' = f(q),
            ray-map queries) and section 3 "Streaming Reconstruction".
  [notes]   67656.sbs reading notes "ZipMap：基于 Test-Time Training 的线性时间
            有状态 3D 重建", section "TTT 模块：核心公式" (virtual objective,
            one gradient step with per-token eta, SwiGLU), section
            "为什么它像 attention（线性情形的直观推导）" (the linear case) and
            "流式更新（streaming）".
  [survey]  mhpn.cn survey of TTSA3R / LaCT / ZipMap / LoGeR, part "二、LaCT,
            2、架构" (update = summed chunk gradient, then L2 normalisation).

Everything is float64.  Inputs are the same (bf16-exact or fp32) values the
GPU receives, upcast exactly.  Per head:
  W1, W3 : [hidden, d]   (rows are the fan-in vectors of hidden units)
  W2     : [d, hidden]
  K, V, Q: [n, d] token-major
  eta    : [n]

Readings taken where the pages are silent or ambiguous (each is also listed in
the design notes; the gated output unit's readings sit with gated_output):
  * SiLU(x) = x * sigmoid(x) with the logistic sigmoid (the pages name SiLU
    without defining it).
  * One gradient step (the review says one step; the notes say "one (or a
    few)").
  * The Eq. 3 sum runs over every image token of the chunk (its index letter
    is a typo in the review).
  * Renormalisation axis: row-wise (each row of W1, W3 of length d, each row
    of W2 of length hidden) to the pre-update row norm, no epsilon; a zero
    updated row is left as is.  "frobenius" (whole matrix per head, the
    literal reading of the unindexed norm) and "off" are kept as switches.
  * Newton-Schulz orthonormalisation of the gradient ([review] section 2,
    the update after Eq. 3, "following the Muon optimizer") is a switch,
    ns_steps, off (0) by default.  The pages give neither the polynomial nor
    the step count; the reading taken is Muon's published quintic iteration
    (Jordan et al. 2024, "Muon: An optimizer for hidden layers in neural
    networks"): X0 = g / ||g||_F, then ns_steps times
    X <- a X + b (X X^T) X + c (X X^T)^2 X with (a, b, c) =
    (3.4445, -4.7750, 2.0315), worked on the wide orientation of g; each of
    g1, g2, g3 is orthonormalised on its own, per head; g = 0 gives 0.
  * Heads are independent fast-weight MLPs.
"""
from __future__ import annotations

import numpy as np

RENORM_OFF, RENORM_ROW, RENORM_FROB = 0, 1, 2


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    """Logistic function, evaluated without overflow."""
    x = _f64(x)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def silu(x):
    """SiLU(x) = x * sigmoid(x)."""
    x = _f64(x)
    return x * sigmoid(x)


def silu_prime(x):
    """d/dx SiLU(x) = s + x s (1 - s), s = sigmoid(x)."""
    x = _f64(x)
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


# --------------------------------------------------------------------------
# Eq. 1 of [review] / "Fast-weight MLP：SwiGLU" of [notes]:
#   f_W(x) = W2 [ SiLU(W1 x) ⊙ (W3 x) ]
# --------------------------------------------------------------------------
def fast_weight_mlp(W1, W2, W3, X):
    """Rows of X are tokens; returns f_W(x) for each row.  [n, d] -> [n, d]."""
    W1, W2, W3, X = map(_f64, (W1, W2, W3, X))
    h1 = X @ W1.T              # [n, hidden]  = (W1 x)^T
    h3 = X @ W3.T              # [n, hidden]  = (W3 x)^T
    return (silu(h1) * h3) @ W2.T


# --------------------------------------------------------------------------
# Eq. 2 of [review] / "虚拟目标" of [notes]:  L_i = -f_W(k_i)^T v_i,
# weighted by the per-token write strength eta_i (Eq. 3 of [review]).
# --------------------------------------------------------------------------
def virtual_loss(W1, W2, W3, K, V, eta):
    """sum_i eta_i * L(f_W(k_i), v_i) with L = -f_W(k)^T v."""
    F = fast_weight_mlp(W1, W2, W3, K)
    return float(-np.sum(_f64(eta) * np.sum(F * _f64(V), axis=1)))


def gradient(W1, W2, W3, K, V, eta):
    """g = ∇_W sum_i eta_i L(f_W(k_i), v_i)  (Eq. 3 of [review]).

    Chain rule for one token with h1 = W1 k, h3 = W3 k, a = SiLU(h1),
    u = a ⊙ h3, L = -v^T W2 u:
        dL/dW2 = -v u^T
        dL/du  = -W2^T v =: du
        dL/dh3 = du ⊙ a,          dL/dW3 = (du ⊙ a) k^T
        dL/dh1 = du ⊙ h3 ⊙ SiLU'(h1),  dL/dW1 = (...) k^T
    Summed over all tokens with weights eta_i.  Returns (G1, G2, G3) shaped
    like (W1, W2, W3).
    """
    W1, W2, W3, K, V, eta = map(_f64, (W1, W2, W3, K, V, eta))
    h1 = K @ W1.T
    h3 = K @ W3.T
    a = silu(h1)
    u = a * h3
    du = -(V @ W2)                      # row i = (-W2^T v_i)^T
    dh3 = du * a
    dh1 = du * h3 * silu_prime(h1)
    e = eta[:, None]
    G2 = -(V * e).T @ u                 # [d, hidden]
    G1 = (dh1 * e).T @ K                # [hidden, d]
    G3 = (dh3 * e).T @ K                # [hidden, d]
    return G1, G2, G3


def gradient_rows_w13(W1, W2, W3, K, V, eta, rows):
    """Selected rows r of G1 and G3 only, by the same formulas as
    ``gradient`` restricted to hidden unit r (each row needs only row r of W1
    and W3 and column r of W2).  Returns (G1[rows], G3[rows])."""
    W1, W2, W3, K, V, eta = map(_f64, (W1, W2, W3, K, V, eta))
    rows = np.asarray(rows)
    h1 = K @ W1[rows].T                 # [n, r]
    h3 = K @ W3[rows].T
    du = -(V @ W2[:, rows])
    e = eta[:, None]
    dh3 = du * silu(h1)
    dh1 = du * h3 * silu_prime(h1)
    return (dh1 * e).T @ K, (dh3 * e).T @ K


def gradient_cols_w2(W1, W2, W3, K, V, eta, cols):
    """Selected columns j of G2 only: G2[:, j] = -sum_i eta_i v_i u_i[j]."""
    W1, W3, K, V, eta = map(_f64, (W1, W3, K, V, eta))
    cols = np.asarray(cols)
    u = silu(K @ W1[cols].T) * (K @ W3[cols].T)      # [n, c]
    return -(V * eta[:, None]).T @ u                 # [d, c]


def gradient_rows_w2(W1, W2, W3, K, V, eta, rows):
    """Selected rows c of G2 only (output coordinate c of the fast-weight MLP):
    G2[c, :] = -sum_i eta_i v_i[c] u_i^T, with u_i over every hidden unit."""
    W1, W3, K, V, eta = map(_f64, (W1, W3, K, V, eta))
    rows = np.asarray(rows)
    u = silu(K @ W1.T) * (K @ W3.T)                  # [n, hidden]
    return -(V[:, rows] * eta[:, None]).T @ u        # [r, hidden]


# --------------------------------------------------------------------------
# Update and L2 renormalisation ([review] section 2, the two-line update after
# Eq. 3; [survey] LaCT 架构 "L2 归一化"):
#   W' = W - g,   Ŵ = ||W|| * W' / ||W'||
# --------------------------------------------------------------------------
def renorm(W, Wp, mode):
    """Rescale the updated matrix Wp to the norm of the pre-update W.
    mode: RENORM_OFF, RENORM_ROW (each row to its own pre-update row norm)
    or RENORM_FROB (whole matrix)."""
    W, Wp = _f64(W), _f64(Wp)
    if mode == RENORM_OFF:
        return Wp.copy()
    if mode == RENORM_ROW:
        n_old = np.sqrt(np.sum(W * W, axis=-1, keepdims=True))
        n_new = np.sqrt(np.sum(Wp * Wp, axis=-1, keepdims=True))
        scale = np.divide(n_old, n_new, out=np.ones_like(n_new), where=n_new > 0)
        return Wp * scale
    if mode == RENORM_FROB:
        n_old = np.sqrt(np.sum(W * W))
        n_new = np.sqrt(np.sum(Wp * Wp))
        return Wp * (n_old / n_new) if n_new > 0 else Wp.copy()
    raise ValueError(f"unknown renorm mode {mode}")


# --------------------------------------------------------------------------
# Newton-Schulz orthonormalisation ([review] section 2, the update after
# Eq. 3: Delta <- NewtonSchulz(g), following the Muon optimizer).  The
# polynomial is Muon's quintic; see the module header for the reading.
# --------------------------------------------------------------------------
NS_COEFFS = (3.4445, -4.7750, 2.0315)


def newton_schulz(G, steps, coeffs=NS_COEFFS):
    """Approximate orthonormalisation of one matrix: with X0 = G/||G||_F,
    repeat X <- a X + b A X + c A^2 X, A = X X^T, `steps` times.  A tall G is
    worked as G^T (A is then the smaller Gram matrix; the result is the same
    polynomial in the singular values either way) and transposed back."""
    a, b, c = coeffs
    X = _f64(G)
    nrm = np.sqrt(np.sum(X * X))
    if nrm == 0.0:
        return np.zeros_like(X)
    X = X / nrm
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    for _ in range(steps):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.T if tall else X


def update_head(W1, W2, W3, K, V, eta, renorm_mode=RENORM_ROW, ns_steps=0):
    """One TTT update of one head: Ŵ = renorm(W - Delta) with Delta = g, or
    Delta = NewtonSchulz(g) per matrix when ns_steps > 0."""
    G = gradient(W1, W2, W3, K, V, eta)
    if ns_steps > 0:
        G = tuple(newton_schulz(g, ns_steps) for g in G)
    G1, G2, G3 = G
    return (renorm(W1, _f64(W1) - G1, renorm_mode),
            renorm(W2, _f64(W2) - G2, renorm_mode),
            renorm(W3, _f64(W3) - G3, renorm_mode))


def _split_heads(X, heads):
    X = _f64(X)
    n = X.shape[0]
    return X.reshape(n, heads, -1)


def ttt_update(W1, W2, W3, K, V, eta, renorm_mode=RENORM_ROW, ns_steps=0):
    """All heads.  W1, W3: [H, hidden, d]; W2: [H, d, hidden];
    K, V: [n, H*d]; eta: [n, H].  Returns (Ŵ1, Ŵ2, Ŵ3) in fp64."""
    H = np.shape(W1)[0]
    Kh, Vh = _split_heads(K, H), _split_heads(V, H)
    eta = _f64(eta).reshape(-1, H)
    out = [update_head(W1[h], W2[h], W3[h], Kh[:, h], Vh[:, h], eta[:, h],
                       renorm_mode, ns_steps) for h in range(H)]
    return tuple(np.stack([o[i] for o in out]) for i in range(3))


def ttt_apply(W1, W2, W3, Q):
    """o'_i = f_Ŵ(q_i) for every query row and head ([review] section 2,
    the apply equation; ray-map queries use the same map).  Q: [m, H*d]."""
    H = np.shape(W1)[0]
    Qh = _split_heads(Q, H)
    m = Qh.shape[0]
    O = np.stack([fast_weight_mlp(W1[h], W2[h], W3[h], Qh[:, h])
                  for h in range(H)], axis=1)
    return O.reshape(m, -1)


def ttt_stream(W1, W2, W3, K, V, eta, Q, frame_tokens, renorm_mode=RENORM_ROW,
               ns_steps=0):
    """Streaming ([review] section 3, [notes] "流式更新"): for each frame t,
    W^(t) = TTTUpdate(W^(t-1); the frame's tokens), then the frame's queries
    read f_{W^(t)}.  Returns the final weights and the per-frame outputs
    concatenated in frame order."""
    n = np.shape(K)[0]
    Ws = (_f64(W1), _f64(W2), _f64(W3))
    outs = []
    for s in range(0, n, frame_tokens):
        e = min(n, s + frame_tokens)
        Ws = ttt_update(*Ws, K[s:e], V[s:e], eta[s:e], renorm_mode, ns_steps)
        outs.append(ttt_apply(*Ws, Q[s:e]))
    return Ws, np.concatenate(outs, axis=0)


# --------------------------------------------------------------------------
# Gated output unit ([review] section 2, the last equation of "Feature
# Backbone"): o = RMSNorm(o') * SiLU(W_g o').  Readings: per head (o' of one
# head is a d-vector, W_g is d x d, rows = outputs), RMSNorm(x) =
# x / sqrt(mean(x^2) + eps) with eps = 1e-6 and no learned gain.
# --------------------------------------------------------------------------
GATE_EPS = 1e-6


def rms_norm(X, eps=GATE_EPS):
    X = _f64(X)
    return X / np.sqrt(np.mean(X * X, axis=-1, keepdims=True) + eps)


def gated_output(Oprime, Wg, eps=GATE_EPS):
    """Oprime: [m, H*d]; Wg: [H, d, d].  Returns o for every row and head."""
    H = np.shape(Wg)[0]
    X = _split_heads(Oprime, H)
    out = np.stack([rms_norm(X[:, h], eps) * silu(X[:, h] @ _f64(Wg[h]).T)
                    for h in range(H)], axis=1)
    return out.reshape(X.shape[0], -1)


# --------------------------------------------------------------------------
# Token-sharded form of Eq. 3 ([review] section 2: g sums over every token, so
# any split of the tokens into shards sums to the same g).  Partial layout per
# head: [g1 (hidden x d), g3 (hidden x d), -g2 (d x hidden)], flattened.
# --------------------------------------------------------------------------
def gradient_partial(W1, W2, W3, K, V, eta):
    """All heads' gradient partial of the given tokens, [H, 3, hidden*d]."""
    H = np.shape(W1)[0]
    Kh, Vh = _split_heads(K, H), _split_heads(V, H)
    eta = _f64(eta).reshape(-1, H)
    out = []
    for h in range(H):
        G1, G2, G3 = gradient(W1[h], W2[h], W3[h], Kh[:, h], Vh[:, h], eta[:, h])
        out.append(np.stack([G1.reshape(-1), G3.reshape(-1), -G2.reshape(-1)]))
    return np.stack(out)


def update_from_partials(W1, W2, W3, partials, renorm_mode=RENORM_ROW, ns_steps=0):
    """Ŵ from partials [ranks, H, 3, hidden*d] summed in rank order."""
    P = np.zeros_like(_f64(partials[0]))
    for r in range(len(partials)):
        P = P + _f64(partials[r])
    H, hid, d = np.shape(W1)
    outs = ([], [], [])
    for h in range(H):
        G = (P[h, 0].reshape(hid, d), -P[h, 2].reshape(d, hid), P[h, 1].reshape(hid, d))
        if ns_steps > 0:
            G = tuple(newton_schulz(g, ns_steps) for g in G)
        for i, W in enumerate((W1, W2, W3)):
            outs[i].append(renorm(W[h], _f64(W[h]) - G[i], renorm_mode))
    return tuple(np.stack(o) for o in outs)


# --------------------------------------------------------------------------
# Chunked orderings ([survey] part "二、LaCT", "3应用场景"): the sequence is cut
# into consecutive chunks of b tokens (the last one shorter); per chunk the
# update U and the apply A run in one of two orders, and U may be skipped on
# chosen chunks:
#   update-then-apply (block-causal):  W_i = U(W_{i-1}; c_i), o_i = A(W_i; c_i)
#   apply-then-update (shifted):       o_i = A(W_{i-1}; c_i), W_i = U(W_{i-1}; c_i)
#   update mask (cross-chunk causal):  U only where mask[i] is true
# Fully bidirectional LaCT is apply-then-update with one chunk; the ZipMap
# layer itself is update-then-apply with one chunk.
# --------------------------------------------------------------------------
ORDER_UPDATE_THEN_APPLY, ORDER_APPLY_THEN_UPDATE = 0, 1


def chunked(update_fn, apply_fn, W, K, V, eta, Q, b, order, update_mask=None):
    """Generic chunk loop over any fast-weight model: update_fn(W, K, V, eta)
    returns the new state, apply_fn(W, Q) the outputs.  Returns the final
    state and the outputs of every token, in order."""
    n = np.shape(K)[0]
    nchunks = (n + b - 1) // b
    outs = []
    for i in range(nchunks):
        s, e = i * b, min(n, (i + 1) * b)
        upd = True if update_mask is None else bool(update_mask[i])
        if order == ORDER_APPLY_THEN_UPDATE:
            outs.append(apply_fn(W, Q[s:e]))
        if upd:
            W = update_fn(W, K[s:e], V[s:e], eta[s:e])
        if order == ORDER_UPDATE_THEN_APPLY:
            outs.append(apply_fn(W, Q[s:e]))
    O = np.concatenate(outs, axis=0) if outs else np.zeros((0, np.shape(Q)[1]))
    return W, O


def ttt_chunked(W1, W2, W3, K, V, eta, Q, b, order, update_mask=None,
                renorm_mode=RENORM_ROW, ns_steps=0):
    """The chunk loop over the SwiGLU layer (all heads)."""
    def upd(W, K_, V_, e_):
        return ttt_update(*W, K_, V_, e_, renorm_mode, ns_steps)

    def app(W, Q_):
        return ttt_apply(*W, Q_)

    return chunked(upd, app, (_f64(W1), _f64(W2), _f64(W3)), K, V, eta, Q, b, order,
                   update_mask)


# --------------------------------------------------------------------------
# Linear fast weights ([notes], "为什么它像 attention（线性情形的直观推导）"):
#   f_W(k) = W k,  L = -(W k)^T v  =>  ∇_W L = -v k^T
# --------------------------------------------------------------------------
def linear_gradient(W, K, V, eta):
    """g = ∇_W sum_i eta_i (-(W k_i)^T v_i) = -sum_i eta_i v_i k_i^T."""
    K, V, eta = map(_f64, (K, V, eta))
    return -(V * eta[:, None]).T @ K


def linear_update(W, K, V, eta, renorm_mode=RENORM_OFF):
    W = _f64(W)
    return renorm(W, W - linear_gradient(W, K, V, eta), renorm_mode)


def linear_apply(W, Q):
    return _f64(Q) @ _f64(W).T


def linear_loss(W, K, V, eta):
    return float(-np.sum(_f64(eta) * np.sum((_f64(K) @ _f64(W).T) * _f64(V), axis=1)))


# --------------------------------------------------------------------------
# State size ([notes], "Fast-weight state 大小与训练规模"): three matrices of
# d x hidden each.
# --------------------------------------------------------------------------
def state_params(d, hidden, heads=1):
    return 3 * d * hidden * heads


# --------------------------------------------------------------------------
# Error measures used by the parity tests.
# --------------------------------------------------------------------------
def rel_fro(x, ref):
    """||x - ref||_F / ||ref||_F in fp64 (returns the absolute error if the
    reference is exactly zero)."""
    x, ref = _f64(x), _f64(ref)
    den = np.sqrt(np.sum(ref * ref))
    num = np.sqrt(np.sum((x - ref) ** 2))
    return float(num / den) if den > 0 else float(num)
