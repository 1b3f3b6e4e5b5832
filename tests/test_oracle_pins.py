"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test is chosen so that a plausible mistake in the oracle (a dropped term,
a wrong sign or index, a transposed operand, a wrong renorm axis) fails it:
finite differences of the virtual loss (Eq. 2) pin the gradient (Eq. 3); the
linear case of the reading notes pins the update direction and the apply; the
W1 = 0 special case has a closed form; invariants (eta = 0, linearity in eta,
token permutation, zero padding, norm preservation) pin the structure.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny(seed=0, n=5, d=4, hidden=8, scale=0.7):
    rng = np.random.default_rng(seed)
    W1 = rng.standard_normal((hidden, d)) * scale
    W3 = rng.standard_normal((hidden, d)) * scale
    W2 = rng.standard_normal((d, hidden)) * scale
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    eta = 0.1 + rng.random(n)
    return W1, W2, W3, K, V, eta


# ---------------------------------------------------------------- SiLU facts
def test_sigmoid_silu_values():
    assert O.sigmoid(np.array([0.0]))[0] == 0.5
    # exp(-ln 3) = 1/3, so sigmoid(ln 3) = 3/4
    assert abs(O.sigmoid(np.array([math.log(3.0)]))[0] - 0.75) < 1e-15
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert O.silu_prime(np.array([0.0]))[0] == 0.5
    x = np.linspace(-8, 8, 33)
    # SiLU(x) - SiLU(-x) = x (since sigmoid(-x) = 1 - sigmoid(x))
    np.testing.assert_allclose(O.silu(x) - O.silu(-x), x, atol=1e-14)
    # large arguments: no overflow, SiLU -> x and -> 0
    big = np.array([800.0, -800.0])
    np.testing.assert_allclose(O.silu(big), [800.0, 0.0], atol=1e-300)


def test_silu_prime_matches_finite_difference():
    x = np.linspace(-6, 6, 97)
    h = 1e-6
    fd = (O.silu(x + h) - O.silu(x - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_prime(x), fd, rtol=1e-8, atol=1e-9)


# ----------------------------------------------------- Eq. 1 forward pieces
def test_forward_homogeneity_and_zero_cases():
    W1, W2, W3, K, V, eta = _tiny(1)
    f = O.fast_weight_mlp(W1, W2, W3, K)
    np.testing.assert_allclose(O.fast_weight_mlp(W1, 3 * W2, W3, K), 3 * f, rtol=1e-14)
    np.testing.assert_allclose(O.fast_weight_mlp(W1, W2, -2 * W3, K), -2 * f, rtol=1e-14)
    assert np.all(O.fast_weight_mlp(0 * W1, W2, W3, K) == 0)  # SiLU(0) = 0
    assert np.all(O.fast_weight_mlp(W1, W2, 0 * W3, K) == 0)
    # Each output row depends on its own token only.
    f2 = O.fast_weight_mlp(W1, W2, W3, K[::-1])
    np.testing.assert_allclose(f2, f[::-1], rtol=1e-14)


def test_forward_against_torch_library():
    torch = pytest.importorskip("torch")
    W1, W2, W3, K, V, eta = _tiny(2, n=7, d=5, hidden=6)
    t = lambda a: torch.tensor(a, dtype=torch.float64)  # noqa: E731
    ref = (torch.nn.functional.silu(t(K) @ t(W1).T) * (t(K) @ t(W3).T)) @ t(W2).T
    np.testing.assert_allclose(O.fast_weight_mlp(W1, W2, W3, K), ref.numpy(), rtol=1e-13)


# --------------------------------------------------------- Eq. 3 gradient
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gradient_matches_central_differences(seed):
    W1, W2, W3, K, V, eta = _tiny(seed)
    G = O.gradient(W1, W2, W3, K, V, eta)
    Ws = [W1, W2, W3]
    h = 1e-6
    for idx in range(3):
        fd = np.zeros_like(Ws[idx])
        for pos in np.ndindex(Ws[idx].shape):
            plus = [w.copy() for w in Ws]
            minus = [w.copy() for w in Ws]
            plus[idx][pos] += h
            minus[idx][pos] -= h
            fd[pos] = (O.virtual_loss(*plus, K, V, eta) - O.virtual_loss(*minus, K, V, eta)) / (2 * h)
        err = np.max(np.abs(fd - G[idx])) / np.max(np.abs(G[idx]))
        assert err <= 1e-7, (idx, err)


def test_gradient_against_torch_autograd():
    torch = pytest.importorskip("torch")
    W1, W2, W3, K, V, eta = _tiny(3, n=9, d=6, hidden=10)
    ws = [torch.tensor(w, dtype=torch.float64, requires_grad=True) for w in (W1, W2, W3)]
    Kt, Vt, et = (torch.tensor(a, dtype=torch.float64) for a in (K, V, eta))
    f = (torch.nn.functional.silu(Kt @ ws[0].T) * (Kt @ ws[2].T)) @ ws[1].T
    loss = -(et * (f * Vt).sum(1)).sum()
    loss.backward()
    G = O.gradient(W1, W2, W3, K, V, eta)
    for g, w in zip(G, ws):
        np.testing.assert_allclose(g, w.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_w1_zero_closed_form():
    """W1 = 0: SiLU(0) = 0 and SiLU'(0) = 1/2, so u = 0, G2 = G3 = 0 and
    W1_hat = sum_i eta_i * 1/2 * ((W2^T v_i) ⊙ (W3 k_i)) k_i^T."""
    W1, W2, W3, K, V, eta = _tiny(4)
    W1 = np.zeros_like(W1)
    G1, G2, G3 = O.gradient(W1, W2, W3, K, V, eta)
    assert np.all(G2 == 0) and np.all(G3 == 0)
    expect = np.zeros_like(W1)
    for i in range(K.shape[0]):
        expect += eta[i] * 0.5 * np.outer((W2.T @ V[i]) * (W3 @ K[i]), K[i])
    np.testing.assert_allclose(W1 - G1, expect, rtol=1e-13, atol=1e-15)
    Wh = O.update_head(W1, W2, W3, K, V, eta, O.RENORM_OFF)
    np.testing.assert_allclose(Wh[0], expect, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(Wh[1], W2)
    np.testing.assert_array_equal(Wh[2], W3)


def test_selected_rows_and_columns_match_full_gradient():
    W1, W2, W3, K, V, eta = _tiny(5, n=40, d=8, hidden=16)
    G1, G2, G3 = O.gradient(W1, W2, W3, K, V, eta)
    rows = [0, 5, 15]
    g1, g3 = O.gradient_rows_w13(W1, W2, W3, K, V, eta, rows)
    np.testing.assert_allclose(g1, G1[rows], rtol=1e-13)
    np.testing.assert_allclose(g3, G3[rows], rtol=1e-13)
    cols = [1, 7, 14]
    np.testing.assert_allclose(O.gradient_cols_w2(W1, W2, W3, K, V, eta, cols),
                               G2[:, cols], rtol=1e-13)
    r2 = [0, 3, 7]
    np.testing.assert_allclose(O.gradient_rows_w2(W1, W2, W3, K, V, eta, r2), G2[r2],
                               rtol=1e-13)


# ------------------------------------------------------------ error measure
def test_rel_fro_hand_computed():
    """The parity measure ||x - ref||_F / ||ref||_F on values worked by hand:
    the denominator is the reference's norm (not x's), both norms are square
    roots of sums of squares over every entry, and an all-zero reference gives
    the absolute error."""
    # 3-4-5: x = 0 against ref = (3, 4): |x - ref| = 5, |ref| = 5
    assert O.rel_fro([0.0, 0.0], [3.0, 4.0]) == 1.0
    # (1, 1) vs (3, 4): sqrt(4 + 9) / 5 = sqrt(13) / 5 (a missing square root gives 13/25)
    assert math.isclose(O.rel_fro([1.0, 1.0], [3.0, 4.0]), math.sqrt(13.0) / 5.0, rel_tol=1e-15)
    # asymmetric: the reference's norm is the denominator
    assert O.rel_fro([2.0, 0.0], [1.0, 0.0]) == 1.0
    assert O.rel_fro([1.0, 0.0], [2.0, 0.0]) == 0.5
    # matrices: the Frobenius norm runs over all entries
    x = np.array([[1.0, 2.0], [3.0, 4.0]])
    ref = np.array([[1.0, 2.0], [3.0, 2.0]])
    assert math.isclose(O.rel_fro(x, ref), 2.0 / math.sqrt(18.0), rel_tol=1e-15)
    # relative: scaling both by 1000 changes nothing
    assert math.isclose(O.rel_fro(1e3 * x, 1e3 * ref), 2.0 / math.sqrt(18.0), rel_tol=1e-15)
    # zero reference: the absolute error, sqrt(9 + 16)
    assert O.rel_fro([3.0, -4.0], [0.0, 0.0]) == 5.0
    assert O.rel_fro(np.zeros(3), np.zeros(3)) == 0.0
    # identical inputs
    assert O.rel_fro(x, x) == 0.0


# ------------------------------------------------------------ invariants
def test_eta_zero_gives_identity_bitwise():
    W1, W2, W3, K, V, eta = _tiny(6)
    for mode in (O.RENORM_OFF, O.RENORM_ROW, O.RENORM_FROB):
        Wh = O.update_head(W1, W2, W3, K, V, 0 * eta, mode)
        for a, b in zip(Wh, (W1, W2, W3)):
            np.testing.assert_array_equal(a, b)


def test_gradient_linear_in_eta():
    W1, W2, W3, K, V, eta = _tiny(7, n=12)
    rng = np.random.default_rng(0)
    eb = rng.random(12)
    Ga = O.gradient(W1, W2, W3, K, V, eta)
    Gb = O.gradient(W1, W2, W3, K, V, eb)
    Gab = O.gradient(W1, W2, W3, K, V, eta + eb)
    Gc = O.gradient(W1, W2, W3, K, V, 2.5 * eta)
    for a, b, ab, c in zip(Ga, Gb, Gab, Gc):
        np.testing.assert_allclose(ab, a + b, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(c, 2.5 * a, rtol=1e-12, atol=1e-14)


def test_token_permutation_invariance():
    W1, W2, W3, K, V, eta = _tiny(8, n=30)
    perm = np.random.default_rng(1).permutation(30)
    a = O.update_head(W1, W2, W3, K, V, eta, O.RENORM_ROW)
    b = O.update_head(W1, W2, W3, K[perm], V[perm], eta[perm], O.RENORM_ROW)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-14)


def test_zero_eta_padding_changes_nothing():
    W1, W2, W3, K, V, eta = _tiny(9, n=11)
    rng = np.random.default_rng(2)
    Kp = np.concatenate([K, rng.standard_normal((5, 4))])
    Vp = np.concatenate([V, rng.standard_normal((5, 4))])
    ep = np.concatenate([eta, np.zeros(5)])
    a = O.gradient(W1, W2, W3, K, V, eta)
    b = O.gradient(W1, W2, W3, Kp, Vp, ep)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-15)


def test_row_renorm_keeps_row_norms_and_directions():
    W1, W2, W3, K, V, eta = _tiny(10, n=20)
    G = O.gradient(W1, W2, W3, K, V, eta)
    Wh = O.update_head(W1, W2, W3, K, V, eta, O.RENORM_ROW)
    for W, g, w in zip((W1, W2, W3), G, Wh):
        np.testing.assert_allclose(np.linalg.norm(w, axis=1), np.linalg.norm(W, axis=1), rtol=1e-13)
        Wp = W - g
        cos = np.sum(w * Wp, axis=1) / (np.linalg.norm(w, axis=1) * np.linalg.norm(Wp, axis=1))
        np.testing.assert_allclose(cos, 1.0, rtol=1e-13)
    Wf = O.update_head(W1, W2, W3, K, V, eta, O.RENORM_FROB)
    for W, w in zip((W1, W2, W3), Wf):
        np.testing.assert_allclose(np.linalg.norm(w), np.linalg.norm(W), rtol=1e-13)


def test_renorm_axis_is_rows_of_math_layout():
    """W2 is [d, hidden]: its rows have length hidden.  A row-wise rescale of
    W2 must not equal a column-wise one (catches a transposed axis)."""
    W1, W2, W3, K, V, eta = _tiny(11, n=20)
    G = O.gradient(W1, W2, W3, K, V, eta)
    w2 = O.renorm(W2, W2 - G[1], O.RENORM_ROW)
    assert w2.shape == W2.shape
    np.testing.assert_allclose(np.linalg.norm(w2, axis=1), np.linalg.norm(W2, axis=1), rtol=1e-13)
    assert not np.allclose(np.linalg.norm(w2, axis=0), np.linalg.norm(W2, axis=0))


def test_zero_row_left_unchanged():
    W = np.array([[1.0, 0.0], [0.0, 2.0]])
    Wp = np.array([[0.0, 0.0], [0.0, 3.0]])
    out = O.renorm(W, Wp, O.RENORM_ROW)
    np.testing.assert_array_equal(out, [[0.0, 0.0], [0.0, 2.0]])


def test_heads_are_independent():
    rng = np.random.default_rng(3)
    H, d, hid, n = 3, 4, 8, 10
    W1 = rng.standard_normal((H, hid, d))
    W3 = rng.standard_normal((H, hid, d))
    W2 = rng.standard_normal((H, d, hid))
    K = rng.standard_normal((n, H * d))
    V = rng.standard_normal((n, H * d))
    Q = rng.standard_normal((7, H * d))
    eta = rng.random((n, H))
    Wh = O.ttt_update(W1, W2, W3, K, V, eta)
    Oo = O.ttt_apply(*Wh, Q)
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        w = O.update_head(W1[h], W2[h], W3[h], K[:, sl], V[:, sl], eta[:, h])
        for a, b in zip(w, Wh):
            np.testing.assert_allclose(b[h], a, rtol=1e-14)
        np.testing.assert_allclose(Oo[:, sl], O.fast_weight_mlp(*w, Q[:, sl]), rtol=1e-14)


# --------------------------------------------- linear case ([notes])
def test_linear_case_gradient_by_finite_differences():
    rng = np.random.default_rng(4)
    W = rng.standard_normal((4, 4))
    K = rng.standard_normal((6, 4))
    V = rng.standard_normal((6, 4))
    eta = rng.random(6)
    g = O.linear_gradient(W, K, V, eta)
    h = 1e-6
    for pos in np.ndindex(W.shape):
        p, m = W.copy(), W.copy()
        p[pos] += h
        m[pos] -= h
        fd = (O.linear_loss(p, K, V, eta) - O.linear_loss(m, K, V, eta)) / (2 * h)
        assert abs(fd - g[pos]) <= 1e-8 * max(1.0, abs(g[pos]))


def test_linear_case_closed_form_and_attention_readout():
    """W_hat = W + sum eta v k^T; f_W_hat(q) = W q + sum_i eta_i v_i (k_i^T q),
    the latter summed token by token like un-normalised linear attention."""
    rng = np.random.default_rng(5)
    d, n, m = 6, 25, 9
    W = rng.standard_normal((d, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    Q = rng.standard_normal((m, d))
    eta = rng.random(n)
    Wh = O.linear_update(W, K, V, eta, O.RENORM_OFF)
    expect = W.copy()
    for i in range(n):
        expect += eta[i] * np.outer(V[i], K[i])
    np.testing.assert_allclose(Wh, expect, rtol=1e-14, atol=1e-14)
    out = O.linear_apply(Wh, Q)
    for j in range(m):
        attn = W @ Q[j]
        for i in range(n):
            attn = attn + eta[i] * V[i] * float(K[i] @ Q[j])
        np.testing.assert_allclose(out[j], attn, rtol=1e-12, atol=1e-13)


def test_linear_streaming_equals_one_chunk():
    """Linear fast weights, renorm off: the gradient does not depend on W, so
    frame-by-frame updates sum to the one-chunk update."""
    rng = np.random.default_rng(6)
    d, n, p = 5, 40, 8
    W = rng.standard_normal((d, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    eta = rng.random(n)
    Ws = W.copy()
    for s in range(0, n, p):
        Ws = O.linear_update(Ws, K[s:s + p], V[s:s + p], eta[s:s + p], O.RENORM_OFF)
    np.testing.assert_allclose(Ws, O.linear_update(W, K, V, eta, O.RENORM_OFF), rtol=1e-13)


# ------------------------------------------------------------ streaming
def test_streaming_is_sum_of_per_frame_steps_renorm_off():
    rng = np.random.default_rng(7)
    H, d, hid, n, p = 2, 4, 8, 24, 6
    W1 = rng.standard_normal((H, hid, d)) * 0.5
    W3 = rng.standard_normal((H, hid, d)) * 0.5
    W2 = rng.standard_normal((H, d, hid)) * 0.5
    K = rng.standard_normal((n, H * d))
    V = rng.standard_normal((n, H * d))
    Q = rng.standard_normal((n, H * d))
    eta = 0.05 * rng.random((n, H))
    (f1, f2, f3), out = O.ttt_stream(W1, W2, W3, K, V, eta, Q, p, O.RENORM_OFF)
    # W^(T) = W^(0) - sum_t G_t(W^(t-1)), each G_t from that frame only.
    acc = [W1.copy(), W2.copy(), W3.copy()]
    cur = [W1.copy(), W2.copy(), W3.copy()]
    for s in range(0, n, p):
        for h in range(H):
            sl = slice(h * d, (h + 1) * d)
            g = O.gradient(cur[0][h], cur[1][h], cur[2][h], K[s:s + p, sl],
                           V[s:s + p, sl], eta[s:s + p, h])
            for i in range(3):
                acc[i][h] -= g[i]
        cur = [a.copy() for a in acc]
    for a, b in zip((f1, f2, f3), acc):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    # The outputs of the last frame read the final weights.
    np.testing.assert_allclose(out[-p:], O.ttt_apply(f1, f2, f3, Q[-p:]), rtol=1e-13)


def test_single_frame_stream_equals_update_then_apply():
    rng = np.random.default_rng(8)
    H, d, hid, n = 2, 4, 8, 9
    W1 = rng.standard_normal((H, hid, d))
    W3 = rng.standard_normal((H, hid, d))
    W2 = rng.standard_normal((H, d, hid))
    K, V, Q = (rng.standard_normal((n, H * d)) for _ in range(3))
    eta = rng.random((n, H))
    Ws, out = O.ttt_stream(W1, W2, W3, K, V, eta, Q, n)
    Wu = O.ttt_update(W1, W2, W3, K, V, eta)
    for a, b in zip(Ws, Wu):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(out, O.ttt_apply(*Wu, Q))


# ------------------------------------------------------ page-printed values
def test_page_values():
    with open(os.path.join(GOLDEN, "page_values.json")) as f:
        g = json.load(f)
    t = g["tokens_per_frame"]
    assert wl.tokens_per_frame(t[0]["height"], t[0]["width"]) == t[0]["p"]
    assert wl.tokens_per_frame(t[1]["height"], t[1]["width"]) == t[1]["p"]
    assert wl.tokens_per_frame(224, 224) - wl.SPECIAL_TOKENS == t[2]["p_patches"]
    s = g["state_size"][0]
    per_layer = O.state_params(s["d"], s["hidden"])
    assert round(per_layer / 1e6, 2) == s["params_per_layer_millions"]
    assert round(per_layer * s["layers"] / 1e8, 1) == s["total_params_hundred_millions"]


def test_workload_token_counts():
    assert wl.WORKLOADS["tiny"].n_tokens == 108
    assert wl.WORKLOADS["layer8"].n_tokens == 10992
    assert wl.WORKLOADS["scale100"].n_tokens == 137400
    assert wl.WORKLOADS["scene700"].n_tokens == 961800
    assert wl.WORKLOADS["scene700"].n_ray == 21984
    assert wl.WORKLOADS["stream256"].n_tokens == 256 * 1374


def test_golden_tiny_regression():
    """Digest of the oracle on the tiny workload, written by
    tests/golden/make_golden.py (which calls only the oracle)."""
    with open(os.path.join(GOLDEN, "tiny_oracle.json")) as f:
        g = json.load(f)
    x = wl.make_inputs("tiny")
    Wh = O.ttt_update(x.W1, x.W2, x.W3, x.K, x.V, x.eta, O.RENORM_ROW)
    out = O.ttt_apply(*Wh, x.Q)
    for i, name in enumerate(("dW1", "dW2", "dW3")):
        d = Wh[i] - x.W1 if i == 0 else (Wh[i] - (x.W2 if i == 1 else x.W3))
        np.testing.assert_allclose(np.linalg.norm(d), g[name + "_fro"], rtol=1e-12)
        np.testing.assert_allclose(d.reshape(-1)[:8], g[name + "_head8"], rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(np.linalg.norm(out), g["O_fro"], rtol=1e-12)
    np.testing.assert_allclose(out.reshape(-1)[:8], g["O_head8"], rtol=1e-12, atol=1e-18)


# ---------------------------------------------------- Newton-Schulz (switch)
def _ns_scalar(x, steps):
    """The scalar quintic that the matrix iteration applies to each singular
    value of X0 = G/||G||_F (Muon's coefficients)."""
    a, b, c = 3.4445, -4.7750, 2.0315
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (7, 7)])
@pytest.mark.parametrize("steps", [1, 2, 5])
def test_newton_schulz_acts_on_singular_values(shape, steps):
    """For G = U diag(s) V^T the iteration is U diag(p^k(s/||s||)) V^T: pins the
    coefficient order, the Frobenius normalisation and the tall/wide handling
    against an SVD built by hand (a rank-deficient part stays zero)."""
    m, n = shape
    r = min(m, n)
    rng = np.random.default_rng(11 + steps)
    U, _ = np.linalg.qr(rng.standard_normal((m, r)))
    Vt, _ = np.linalg.qr(rng.standard_normal((n, r)))
    s = np.linspace(3.0, 0.2, r)
    s[-1] = 0.0  # one zero singular value
    G = U @ np.diag(s) @ Vt.T
    want = U @ np.diag(_ns_scalar(s / np.linalg.norm(s), steps)) @ Vt.T
    np.testing.assert_allclose(O.newton_schulz(G, steps), want, rtol=0, atol=1e-12)


def test_newton_schulz_worked_scalar_and_invariants():
    # 1x1: X0 = sign(g), one step gives a + b + c = 0.701 with the sign kept
    assert abs(O.newton_schulz(np.array([[-3.0]]), 1)[0, 0] + 0.701) < 1e-15
    rng = np.random.default_rng(5)
    G = rng.standard_normal((8, 12))
    X = O.newton_schulz(G, 5)
    np.testing.assert_allclose(O.newton_schulz(7.5 * G, 5), X, atol=1e-13)  # scale
    np.testing.assert_allclose(O.newton_schulz(-G, 5), -X, atol=1e-13)      # odd
    np.testing.assert_allclose(O.newton_schulz(G.T, 5), X.T, atol=1e-13)    # transpose
    np.testing.assert_allclose(O.newton_schulz(G, 0), G / np.linalg.norm(G), atol=1e-15)
    assert not np.any(O.newton_schulz(np.zeros((4, 6)), 5))
    # five steps leave every singular value inside Muon's band around 1
    sv = np.linalg.svd(X, compute_uv=False)
    assert sv.min() > 0.6 and sv.max() < 1.25


def test_update_with_newton_schulz():
    """With NS the update shares the gradient's singular vectors (g^T Delta
    and g Delta^T are symmetric positive semi-definite), it no longer depends
    on the global scale of eta, and eta = 0 still leaves W bitwise."""
    W1, W2, W3, K, V, eta = _tiny(seed=4, n=9, d=6, hidden=10)
    G = O.gradient(W1, W2, W3, K, V, eta)
    Wn = O.update_head(W1, W2, W3, K, V, eta, O.RENORM_OFF, ns_steps=5)
    for g, W, Wh in zip(G, (W1, W2, W3), Wn):
        D = W - Wh
        for P in (g.T @ D, g @ D.T):
            np.testing.assert_allclose(P, P.T, atol=1e-12)
            assert np.linalg.eigvalsh(0.5 * (P + P.T)).min() > -1e-12
    Wc = O.update_head(W1, W2, W3, K, V, 3.0 * eta, O.RENORM_OFF, ns_steps=5)
    for a_, b_ in zip(Wn, Wc):
        np.testing.assert_allclose(a_, b_, atol=1e-12)
    Wz = O.update_head(W1, W2, W3, K, V, 0 * eta, O.RENORM_ROW, ns_steps=5)
    for a_, b_ in zip(Wz, (W1, W2, W3)):
        assert np.array_equal(a_, b_)
    # renorm on: row norms kept
    Wr = O.update_head(W1, W2, W3, K, V, eta, O.RENORM_ROW, ns_steps=3)
    for a_, b_ in zip(Wr, (W1, W2, W3)):
        np.testing.assert_allclose(np.linalg.norm(a_, axis=1), np.linalg.norm(b_, axis=1), rtol=1e-13)


# ------------------------------------------------------- chunked orderings
def _block_causal_linear_attention(W0, K, V, eta, Q, b, strict, mask=None):
    """Brute force: o_t = W0 q_t + sum over earlier tokens s of eta_s v_s (k_s.q_t)
    where s runs over the updating chunks before t's chunk, plus t's own chunk
    unless `strict`.  This is linear attention with a block mask."""
    n = K.shape[0]
    O = Q @ W0.T
    for t in range(n):
        ct = t // b
        for s_ in range(n):
            cs = s_ // b
            if mask is not None and not mask[cs]:
                continue
            if cs < ct or (cs == ct and not strict):
                O[t] += eta[s_] * V[s_] * (K[s_] @ Q[t])
    return O


@pytest.mark.parametrize("b", [1, 3, 4, 11])
def test_chunked_orders_are_block_causal_linear_attention(b):
    """Linear fast weights, renorm off ([notes] linear case): update-then-apply
    is inclusive block-causal linear attention, apply-then-update the strict
    (shifted) one, and an update mask drops the masked chunks' keys."""
    rng = np.random.default_rng(b)
    n, d = 11, 5
    W0 = rng.standard_normal((d, d)) * 0.3
    K, V, Q = (rng.standard_normal((n, d)) for _ in range(3))
    eta = 0.05 + rng.random(n)
    upd = lambda W, K_, V_, e_: O.linear_update(W, K_, V_, e_, O.RENORM_OFF)  # noqa: E731
    app = O.linear_apply
    for order, strict in ((O.ORDER_UPDATE_THEN_APPLY, False), (O.ORDER_APPLY_THEN_UPDATE, True)):
        Wf, Out = O.chunked(upd, app, W0, K, V, eta, Q, b, order)
        np.testing.assert_allclose(Out, _block_causal_linear_attention(W0, K, V, eta, Q, b, strict),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Wf, O.linear_update(W0, K, V, eta), rtol=1e-12, atol=1e-12)
    mask = [(i % 2) == 0 for i in range((n + b - 1) // b)]
    _, Out = O.chunked(upd, app, W0, K, V, eta, Q, b, O.ORDER_UPDATE_THEN_APPLY, mask)
    np.testing.assert_allclose(Out, _block_causal_linear_attention(W0, K, V, eta, Q, b, False, mask),
                               rtol=1e-12, atol=1e-12)


def test_chunked_swiglu_special_cases():
    x = wl.make_inputs("tiny")
    W = (x.W1, x.W2, x.W3)
    n = x.K.shape[0]
    # one chunk, update-then-apply: the ZipMap layer
    Wf, Out = O.ttt_chunked(*W, x.K, x.V, x.eta, x.Q, n, O.ORDER_UPDATE_THEN_APPLY)
    Wu = O.ttt_update(*W, x.K, x.V, x.eta)
    np.testing.assert_allclose(Out, rtol=1e-13, atol=1e-15, desired=O.ttt_apply(*Wu, x.Q))
    # one chunk, apply-then-update: outputs read the initial state
    Wf, Out = O.ttt_chunked(*W, x.K, x.V, x.eta, x.Q, n, O.ORDER_APPLY_THEN_UPDATE)
    np.testing.assert_allclose(Out, rtol=1e-13, atol=1e-15, desired=O.ttt_apply(*W, x.Q))
    for a_, b_ in zip(Wf, Wu):
        np.testing.assert_allclose(a_, b_, rtol=1e-13, atol=1e-15)
    # no chunk updates: every output reads the initial state, W unchanged
    Wf, Out = O.ttt_chunked(*W, x.K, x.V, x.eta, x.Q, 40, O.ORDER_UPDATE_THEN_APPLY,
                            update_mask=[0, 0, 0])
    np.testing.assert_allclose(Out, rtol=1e-13, atol=1e-15, desired=O.ttt_apply(*W, x.Q))
    # update-then-apply with frame-sized chunks is the streaming recurrence
    Wf, Out = O.ttt_chunked(*W, x.K, x.V, x.eta, x.Q, 49, O.ORDER_UPDATE_THEN_APPLY)
    Ws, Os = O.ttt_stream(*W, x.K, x.V, x.eta, x.Q, 49)
    np.testing.assert_allclose(Out, rtol=1e-13, atol=1e-15, desired=Os)


# --------------------------------------------------- token-sharded update
def test_partials_sum_to_the_full_update():
    """Any split of the tokens: the shards' partials, summed, give the one-chunk
    update (Eq. 3 is a sum over tokens); block 2 holds -g2."""
    x = wl.make_inputs("tiny")
    W = (x.W1, x.W2, x.W3)
    full = O.ttt_update(*W, x.K, x.V, x.eta)
    for cuts in ([0, 108], [0, 40, 108], [0, 1, 2, 57, 108]):
        parts = [O.gradient_partial(*W, x.K[a:b], x.V[a:b], x.eta[a:b])
                 for a, b in zip(cuts[:-1], cuts[1:])]
        got = O.update_from_partials(*W, parts)
        for g, f in zip(got, full):
            np.testing.assert_allclose(g, f, rtol=1e-12, atol=1e-14)
    P = O.gradient_partial(*W, x.K, x.V, x.eta)
    G1, G2, G3 = O.gradient(x.W1[0], x.W2[0], x.W3[0], x.K, x.V, x.eta[:, 0])
    np.testing.assert_allclose(P[0, 2].reshape(G2.shape), -G2, rtol=1e-15)
    # with Newton-Schulz the orthonormalised sum matches the one-chunk path
    got = O.update_from_partials(*W, [O.gradient_partial(*W, x.K[:50], x.V[:50], x.eta[:50]),
                                      O.gradient_partial(*W, x.K[50:], x.V[50:], x.eta[50:])],
                                 ns_steps=5)
    want = O.ttt_update(*W, x.K, x.V, x.eta, ns_steps=5)
    for g, f in zip(got, want):
        np.testing.assert_allclose(g, f, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------- gated output unit
def test_gated_output_against_torch_and_closed_forms():
    import torch
    rng = np.random.default_rng(9)
    m, H, d = 7, 3, 16
    Op = rng.standard_normal((m, H * d))
    Wg = rng.standard_normal((H, d, d)) / 4
    got = O.gated_output(Op, Wg)
    # library routines: torch's rms_norm, linear and silu, per head
    X = torch.from_numpy(Op).view(m, H, d)
    want = torch.stack([torch.nn.functional.rms_norm(X[:, h], (d,), eps=1e-6) *
                        torch.nn.functional.silu(torch.nn.functional.linear(
                            X[:, h], torch.from_numpy(Wg[h])))
                        for h in range(H)], dim=1).reshape(m, -1).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)
    # W_g = 0: SiLU(0) = 0 silences the unit
    assert not np.any(O.gated_output(Op, np.zeros_like(Wg)))
    # constant o' = c 1 and W_g = a I: o_j = c / sqrt(c^2 + eps) * SiLU(a c)
    c, a = -0.7, 1.3
    got = O.gated_output(np.full((1, d), c), a * np.eye(d)[None])
    silu = a * c / (1.0 + math.exp(-a * c))
    np.testing.assert_allclose(got, np.full((1, d), c / math.sqrt(c * c + 1e-6) * silu),
                               rtol=1e-14)
    # heads do not mix: changing head 1's o' leaves heads 0 and 2
    Op2 = Op.copy()
    Op2[:, d:2 * d] += 1.0
    g2 = O.gated_output(Op2, Wg)
    np.testing.assert_array_equal(g2[:, :d], O.gated_output(Op, Wg)[:, :d])
    np.testing.assert_array_equal(g2[:, 2 * d:], O.gated_output(Op, Wg)[:, 2 * d:])
