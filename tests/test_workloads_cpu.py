"""The seeded input generators against the recipe they state (token counts from
the ZipMap review's tokenisation, distributions, seeds, layouts), and the
bf16 rounding both sides of the parity tests rely on.  CPU only."""
import numpy as np
import pytest

from recon_chunk_ttt_b200 import workloads as wl

torch = pytest.importorskip("torch")


def test_tokens_per_frame_and_workload_sizes():
    assert wl.tokens_per_frame(518, 518) == 37 * 37 + 5 == 1374
    assert wl.tokens_per_frame(98, 98) == 54
    with pytest.raises(ValueError):
        wl.tokens_per_frame(500, 518)
    W = wl.WORKLOADS
    assert W["tiny"].n_tokens == 108
    assert W["layer8"].n_tokens == 10992
    assert W["scale100"].n_tokens == 137400
    assert W["scene700"].n_tokens == 961800 and W["scene700"].n_ray == 21984
    assert W["scene700"].layers == 24
    assert W["stream256"].n_tokens == 256 * 1374


def test_bf16_round_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(
        -20, 20, 20000), np.float32([0.0, -0.0, 1.0, 65504.0, 3.0e38, -1e-30])])
    # exact ties between two bf16 neighbours: the low 16 bits are 0x8000
    ties = ((rng.integers(0x3F80, 0x4100, 64).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = wl.bf16_round(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(wl.bits_to_f32(wl.bf16_bits(got)), got)


def test_tiny_recipe():
    x = wl.make_inputs("tiny")
    assert x.K.shape == (108, 64) and x.K.dtype == np.float32
    assert x.W1.shape == (1, 128, 64) and x.W2.shape == (1, 64, 128)
    for a in (x.K, x.V, x.Q):                        # N(0, 1) / 8
        assert abs(a.std() - 1 / 8) < 0.01 and abs(a.mean()) < 0.01
    assert abs(x.W1.var() - 1 / 64) < 0.002 and abs(x.W2.var() - 1 / 128) < 0.001
    assert np.all(x.eta > 0) and abs(x.eta.mean() - 0.01 * 0.806) < 0.002  # 0.01 softplus(N(0,1))
    assert x.Qray is None


def test_layer_recipe_normalised_bf16_tokens():
    x = wl.make_inputs("layer8", n_tokens=3000)
    H, d = 4, 256
    for a in (x.K, x.V, x.Q):
        assert a.shape == (3000, H * d)
        assert np.array_equal(wl.bf16_round(a), a)  # bf16-exact values
        norms = np.linalg.norm(a.reshape(-1, H, d).astype(np.float64), axis=2)
        assert np.all(np.abs(norms - 1.0) < 2e-3)   # unit per token and head, then rounded
    assert abs(x.W1.var() - 1 / 256) < 2e-4 and abs(x.W3.var() - 1 / 256) < 2e-4
    assert abs(x.W2.var() - 1 / 512) < 1e-4
    z_mean = np.mean(np.log1p(np.exp(np.random.default_rng(9).standard_normal(10 ** 6) - 3.0)))
    assert x.eta.shape == (3000, H) and abs(x.eta.mean() - z_mean) < 0.01


def test_seeds_layers_and_bits():
    w = wl.WORKLOADS["scene700"]
    a = wl.make_inputs(w, n_tokens=500, layer=0)
    b = wl.make_inputs(w, n_tokens=500, layer=3)
    c = wl.make_inputs(w, n_tokens=500, layer=3)
    for t in ("K", "V", "Q", "eta", "Qray"):       # tokens: the same for every layer
        assert np.array_equal(getattr(a, t), getattr(b, t))
    assert not np.array_equal(a.W1, b.W1)           # weights: seed pair (4, layer)
    for t in ("W1", "W2", "W3", "K"):               # and reproducible
        assert np.array_equal(getattr(b, t), getattr(c, t))
    assert a.Qray.shape == (21984, 1024)
    bits = wl.make_inputs(w, n_tokens=500, layer=0, bits=True)
    assert bits.K.dtype == np.uint16 and np.array_equal(wl.bits_to_f32(bits.K), a.K)
