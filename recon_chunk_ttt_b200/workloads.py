"""Seeded synthetic inputs for the large-chunk TTT layer.

This module only draws random numbers and lays them out.  It holds none of the
layer's arithmetic (no fast-weight MLP, no gradient, no renormalisation), so
both the fp64 oracle (tests only) and the CUDA path may consume its arrays.

Token arithmetic follows the ZipMap review (kimjy99, "1. Input Tokenization"):
an H x W frame with patch size 14 gives HW/14^2 patch tokens plus one camera
token and four register tokens, so p = HW/14^2 + 5 (1374 for 518 x 518).

Workloads (all inputs are synthetic; the pages' image datasets are not used):

  tiny      N=2 frames of 98x98 (54 tokens each, T=108), one head, d=64,
            hidden 128, fp32 q/k/v ~ N(0,1)/8, W1,W3 ~ N(0,1/64),
            W2 ~ N(0,1/128), eta = 0.01*softplus(N(0,1)), seed 0.
  layer8    N=8 frames at 518x518 (T=10,992), 4 heads x d=256, hidden 512,
            q/k/v ~ N(0,1) L2-normalised per token per head then rounded to
            bf16, W ~ N(0, 1/fan_in) fp32, eta = softplus(N(0,1)-3), seed 2.
  scale100  as layer8 with N=100 frames (T=137,400), seed 3.
  scene700  as layer8 with N=700 frames (T=961,800) plus 16 ray-map target
            views (21,984 query tokens); 24 layers whose weights use the seed
            pair (4, layer); token inputs use seed 4.
  stream256 as layer8 with 256 frames fed one frame (1374 tokens) at a time,
            seed 5.

Draw order inside one generator: W1, W3, W2, k, v, q, eta, ray q.
Arrays are token-major: K, V, Q are [T, heads*d]; eta is [T, heads];
W1, W3 are [heads, hidden, d]; W2 is [heads, d, hidden].
"""
from __future__ import annotations

import dataclasses

import numpy as np

PATCH = 14
SPECIAL_TOKENS = 5  # one camera token + four register tokens per frame


def tokens_per_frame(height: int, width: int, patch: int = PATCH) -> int:
    """p = HW/P^2 + 5 (ZipMap review, "1. Input Tokenization")."""
    if height % patch or width % patch:
        raise ValueError("frame size must be a multiple of the patch size")
    return (height // patch) * (width // patch) + SPECIAL_TOKENS


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    frames: int
    frame_px: int
    heads: int
    d: int
    hidden: int
    seed: int
    bf16_inputs: bool          # q/k/v rounded to bf16 (False: fp32 values)
    normalise: bool            # per-token per-head L2 normalisation of q/k/v
    layers: int = 1
    ray_views: int = 0
    streaming: bool = False

    @property
    def p(self) -> int:
        return tokens_per_frame(self.frame_px, self.frame_px)

    @property
    def n_tokens(self) -> int:
        return self.frames * self.p

    @property
    def n_ray(self) -> int:
        return self.ray_views * self.p


WORKLOADS = {
    "tiny": Workload("tiny", 2, 98, 1, 64, 128, 0, False, False),
    "layer8": Workload("layer8", 8, 518, 4, 256, 512, 2, True, True),
    "scale100": Workload("scale100", 100, 518, 4, 256, 512, 3, True, True),
    "scene700": Workload("scene700", 700, 518, 4, 256, 512, 4, True, True,
                         layers=24, ray_views=16),
    "stream256": Workload("stream256", 256, 518, 4, 256, 512, 5, True, True,
                          streaming=True),
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); the result
    is float32 holding exactly representable bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    lsb = (bits >> 16) & np.uint32(1)
    rounded = (bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return rounded.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _softplus(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    return np.where(x > 30.0, x, np.log1p(np.exp(np.minimum(x, 30.0))))


def draw_weights(rng: np.random.Generator, heads: int, d: int, hidden: int,
                 w13_var: float, w2_var: float):
    """W1, W3 ~ N(0, w13_var) as [heads, hidden, d]; W2 ~ N(0, w2_var) as
    [heads, d, hidden]; fp32."""
    w1 = (rng.standard_normal((heads, hidden, d)) * np.sqrt(w13_var)).astype(np.float32)
    w3 = (rng.standard_normal((heads, hidden, d)) * np.sqrt(w13_var)).astype(np.float32)
    w2 = (rng.standard_normal((heads, d, hidden)) * np.sqrt(w2_var)).astype(np.float32)
    return w1, w2, w3


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to the float32 values they encode."""
    return (np.ascontiguousarray(bits).astype(np.uint32) << 16).view(np.float32)


def _tokens(rng: np.random.Generator, n: int, heads: int, d: int,
            normalise: bool, scale: float, bf16: bool, chunk: int = 65536,
            bits: bool = False):
    out = np.empty((n, heads * d), dtype=np.uint16 if (bits and bf16) else np.float32)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal((e - s, heads * d), dtype=np.float32)
        if normalise:
            xh = x.reshape(e - s, heads, d).astype(np.float64)
            xh /= np.sqrt(np.sum(xh * xh, axis=2, keepdims=True))
            x = xh.reshape(e - s, heads * d).astype(np.float32)
        else:
            x = x * np.float32(scale)
        if bits and bf16:
            out[s:e] = bf16_bits(bf16_round(x))
        else:
            out[s:e] = bf16_round(x) if bf16 else x
    return out


@dataclasses.dataclass
class LayerInputs:
    W1: np.ndarray
    W2: np.ndarray
    W3: np.ndarray
    K: np.ndarray
    V: np.ndarray
    Q: np.ndarray
    eta: np.ndarray
    Qray: np.ndarray | None


def make_inputs(w: Workload | str, n_tokens: int | None = None,
                layer: int = 0, bits: bool = False) -> LayerInputs:
    """Draw one layer's inputs for a workload.  With n_tokens given, the same
    recipe and seed are used for a chunk of that many tokens (a different
    draw from the first n_tokens of the full-size chunk).  With bits=True the
    bf16 token arrays (K, V, Q, Qray) are returned as uint16 bit patterns,
    half the host memory of float32 (same values)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    n = w.n_tokens if n_tokens is None else int(n_tokens)
    if w.layers > 1:
        wrng = np.random.default_rng([w.seed, layer])
        rng = np.random.default_rng(w.seed)
    else:
        wrng = rng = np.random.default_rng(w.seed)
    if w.name == "tiny":
        W1, W2, W3 = draw_weights(wrng, w.heads, w.d, w.hidden, 1 / 64, 1 / 128)
    else:
        W1, W2, W3 = draw_weights(wrng, w.heads, w.d, w.hidden,
                                  1.0 / w.d, 1.0 / w.hidden)
    scale = 1.0 / np.sqrt(w.d)
    K = _tokens(rng, n, w.heads, w.d, w.normalise, scale, w.bf16_inputs, bits=bits)
    V = _tokens(rng, n, w.heads, w.d, w.normalise, scale, w.bf16_inputs, bits=bits)
    Q = _tokens(rng, n, w.heads, w.d, w.normalise, scale, w.bf16_inputs, bits=bits)
    z = rng.standard_normal((n, w.heads))
    if w.name == "tiny":
        eta = (0.01 * _softplus(z)).astype(np.float32)
    else:
        eta = _softplus(z - 3.0).astype(np.float32)
    Qray = None
    if w.ray_views:
        Qray = _tokens(rng, w.n_ray, w.heads, w.d, w.normalise, scale, w.bf16_inputs,
                       bits=bits)
    return LayerInputs(W1, W2, W3, K, V, Q, eta, Qray)


def random_layer(seed: int, n: int, heads: int, d: int, hidden: int,
                 m: int | None = None, bf16: bool = True,
                 eta_scale: float = 1.0) -> LayerInputs:
    """Inputs of arbitrary size with the layer8 distributions (used for
    ragged and edge-case sizes)."""
    rng = np.random.default_rng(seed)
    W1, W2, W3 = draw_weights(rng, heads, d, hidden, 1.0 / d, 1.0 / hidden)
    K = _tokens(rng, n, heads, d, True, 1.0, bf16)
    V = _tokens(rng, n, heads, d, True, 1.0, bf16)
    Q = _tokens(rng, n if m is None else m, heads, d, True, 1.0, bf16)
    eta = (eta_scale * _softplus(rng.standard_normal((n, heads)) - 3.0)).astype(np.float32)
    return LayerInputs(W1, W2, W3, K, V, Q, eta, None)
