"""Randomised pins of the fp64 oracle (hypothesis): the same laws as
test_oracle_pins.py, over random small shapes, seeds and chunkings, so that a
mistake that happens to cancel for one fixed draw still shows."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle as O

SETTINGS = settings(max_examples=25, deadline=None)


def _draw(seed, n, d, h, scale=0.6):
    rng = np.random.default_rng(seed)
    W1 = rng.standard_normal((h, d)) * scale
    W3 = rng.standard_normal((h, d)) * scale
    W2 = rng.standard_normal((d, h)) * scale
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    eta = 0.05 + rng.random(n)
    return W1, W2, W3, K, V, eta


@SETTINGS
@given(seed=st.integers(0, 10**6), n=st.integers(1, 6), d=st.integers(1, 4), h=st.integers(1, 5))
def test_gradient_is_the_derivative_of_the_virtual_loss(seed, n, d, h):
    W1, W2, W3, K, V, eta = _draw(seed, n, d, h)
    G = O.gradient(W1, W2, W3, K, V, eta)
    Ws = [W1, W2, W3]
    step = 1e-6
    rng = np.random.default_rng(seed + 1)
    for i in range(3):
        D = rng.standard_normal(Ws[i].shape)  # directional derivative along D
        Wp = [w.copy() for w in Ws]
        Wm = [w.copy() for w in Ws]
        Wp[i] += step * D
        Wm[i] -= step * D
        num = (O.virtual_loss(*Wp, K, V, eta) - O.virtual_loss(*Wm, K, V, eta)) / (2 * step)
        ana = float(np.sum(G[i] * D))
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana))


@SETTINGS
@given(seed=st.integers(0, 10**6), n=st.integers(2, 12), cut=st.integers(1, 11))
def test_gradient_is_additive_over_any_token_split(seed, n, cut):
    W1, W2, W3, K, V, eta = _draw(seed, n, 3, 4)
    c = min(cut, n - 1)
    Ga = O.gradient(W1, W2, W3, K[:c], V[:c], eta[:c])
    Gb = O.gradient(W1, W2, W3, K[c:], V[c:], eta[c:])
    G = O.gradient(W1, W2, W3, K, V, eta)
    for a, b, g in zip(Ga, Gb, G):
        np.testing.assert_allclose(a + b, g, rtol=1e-12, atol=1e-13)


@SETTINGS
@given(seed=st.integers(0, 10**6), mode=st.sampled_from([O.RENORM_ROW, O.RENORM_FROB]))
def test_renorm_keeps_norms(seed, mode):
    W1, W2, W3, K, V, eta = _draw(seed, 5, 4, 6)
    Wh = O.ttt_update(W1[None], W2[None], W3[None], K, V, eta[:, None], mode)
    for w, wh in zip((W1, W2, W3), Wh):
        if mode == O.RENORM_ROW:
            np.testing.assert_allclose(np.linalg.norm(wh[0], axis=1), np.linalg.norm(w, axis=1),
                                       rtol=1e-12)
        else:
            np.testing.assert_allclose(np.linalg.norm(wh[0]), np.linalg.norm(w), rtol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 10**6), n=st.integers(1, 9), b=st.integers(1, 9),
       order=st.sampled_from([O.ORDER_UPDATE_THEN_APPLY, O.ORDER_APPLY_THEN_UPDATE]),
       mask_bits=st.integers(0, 511))
def test_chunked_linear_is_block_masked_attention(seed, n, b, order, mask_bits):
    rng = np.random.default_rng(seed)
    d = 3
    W0 = rng.standard_normal((d, d)) * 0.3
    K, V, Q = (rng.standard_normal((n, d)) for _ in range(3))
    eta = 0.05 + rng.random(n)
    nch = (n + b - 1) // b
    mask = [(mask_bits >> i) & 1 for i in range(nch)]
    upd = lambda W, K_, V_, e_: O.linear_update(W, K_, V_, e_, O.RENORM_OFF)  # noqa: E731
    _, Out = O.chunked(upd, O.linear_apply, W0, K, V, eta, Q, b, order, mask)
    strict = order == O.ORDER_APPLY_THEN_UPDATE
    want = Q @ W0.T
    for t in range(n):
        for s_ in range(n):
            cs, ct = s_ // b, t // b
            if mask[cs] and (cs < ct or (cs == ct and not strict)):
                want[t] += eta[s_] * V[s_] * (K[s_] @ Q[t])
    np.testing.assert_allclose(Out, want, rtol=1e-12, atol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 10**6), m=st.integers(1, 6), n=st.integers(1, 6),
       steps=st.integers(0, 6))
def test_newton_schulz_is_the_scalar_quintic_on_singular_values(seed, m, n, steps):
    rng = np.random.default_rng(seed)
    G = rng.standard_normal((m, n))
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    x = s / np.linalg.norm(s)
    for _ in range(steps):
        x = 3.4445 * x - 4.7750 * x ** 3 + 2.0315 * x ** 5
    np.testing.assert_allclose(O.newton_schulz(G, steps), (U * x) @ Vt, rtol=0, atol=1e-11)


@SETTINGS
@given(seed=st.integers(0, 10**6), m=st.integers(1, 5), H=st.integers(1, 3), d=st.integers(1, 8))
def test_gate_matches_its_definition_elementwise(seed, m, H, d):
    rng = np.random.default_rng(seed)
    Op = rng.standard_normal((m, H * d))
    Wg = rng.standard_normal((H, d, d))
    got = O.gated_output(Op, Wg)
    for r in range(m):
        for h in range(H):
            x = Op[r, h * d:(h + 1) * d]
            rms = np.sqrt(np.mean(x * x) + 1e-6)
            for j in range(d):
                z = float(Wg[h, j] @ x)
                want = x[j] / rms * z / (1.0 + np.exp(-z))
                assert got[r, h * d + j] == pytest.approx(want, rel=1e-12, abs=1e-14)
