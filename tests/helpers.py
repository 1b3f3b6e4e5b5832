"""Shared test plumbing: move seeded inputs to the GPU, run the library through
its C ABI, and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

# Tolerances on the relative Frobenius error of (Ŵ - W) and of O.
TOL_TC = 1e-2      # bf16 tensor-core operands, fp32 accumulation
TOL_F32 = 1e-5     # fp32 CUDA-core check mode


def torch_mod():
    import torch
    return torch


def to_dev(x, dtype):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(dtype)


def gpu_inputs(x: wl.LayerInputs, precision: int):
    """Device copies: weights fp32; tokens bf16 (tensor-core mode) or fp32."""
    import recon_chunk_ttt_b200 as R
    torch = torch_mod()
    tdt = torch.bfloat16 if precision == R.PREC_BF16_TC else torch.float32
    d = dict(W1=to_dev(x.W1, torch.float32), W2=to_dev(x.W2, torch.float32),
             W3=to_dev(x.W3, torch.float32), K=to_dev(x.K, tdt), V=to_dev(x.V, tdt),
             Q=to_dev(x.Q, tdt), eta=to_dev(x.eta, torch.float32))
    if x.Qray is not None:
        d["Qray"] = to_dev(x.Qray, tdt)
    return d


def oracle_inputs(x: wl.LayerInputs, precision: int):
    """What the oracle sees: in tensor-core mode the bf16-rounded token values
    (the GPU's exact inputs)."""
    import recon_chunk_ttt_b200 as R
    if precision == R.PREC_BF16_TC:
        r = wl.bf16_round
        return wl.LayerInputs(x.W1, x.W2, x.W3, r(x.K), r(x.V), r(x.Q), x.eta,
                              None if x.Qray is None else r(x.Qray))
    return x


def run_update_apply(x: wl.LayerInputs, precision: int, renorm: int, ns_steps: int = 0):
    import recon_chunk_ttt_b200 as R
    torch = torch_mod()
    H, hid, d = x.W1.shape
    cfg = R.make_config(H, d, hid, renorm=renorm, precision=precision, ns_steps=ns_steps)
    g = gpu_inputs(x, precision)
    shadow = R.alloc_shadow(cfg)
    W1o, W2o, W3o = R.ttt_update(cfg, g["W1"], g["W2"], g["W3"], g["K"], g["V"], g["eta"],
                                 shadow=shadow)
    O_ = R.ttt_apply(cfg, g["Q"], W1=W1o, W2=W2o, W3=W3o, shadow=shadow)
    R.ttt_check_device_error()
    torch.cuda.synchronize()
    return (W1o.cpu().double().numpy(), W2o.cpu().double().numpy(),
            W3o.cpu().double().numpy(), O_.float().cpu().double().numpy())


def oracle_update_apply(x: wl.LayerInputs, precision: int, renorm: int, ns_steps: int = 0):
    xo = oracle_inputs(x, precision)
    Wh = O.ttt_update(xo.W1, xo.W2, xo.W3, xo.K, xo.V, xo.eta, renorm, ns_steps)
    return Wh, O.ttt_apply(*Wh, xo.Q)


def as_output_type(W_ref):
    """The oracle's Ŵ rounded to the library's output type (fp32).  Ŵ - W taken
    from an fp32 Ŵ cannot be finer than ulp(W); comparing with the rounded
    reference removes that floor (which dominates when the update is tiny,
    e.g. one token) and leaves the kernels' own error."""
    return np.asarray(W_ref, dtype=np.float32).astype(np.float64)


def rel_fro_heads(x, ref, heads, token_major=False):
    """The relative Frobenius error over all heads and of every single head,
    the largest of them: one wrong head cannot hide among correct ones.
    Weights are [H, ...]; token-major outputs are [m, H*d]."""
    x, ref = np.asarray(x, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    if token_major:
        per = [(x.reshape(x.shape[0], heads, -1)[:, h], ref.reshape(ref.shape[0], heads, -1)[:, h])
               for h in range(heads)]
    else:
        per = [(x[h], ref[h]) for h in range(heads)]
    return max([O.rel_fro(x, ref)] + [O.rel_fro(a, b) for a, b in per])


def rel_errors(gpu, ref, x):
    """Relative Frobenius errors on Ŵ - W (per matrix) and on O, each the
    maximum over the whole tensor and every head."""
    W = (x.W1, x.W2, x.W3)
    H = x.W1.shape[0]
    errs = [rel_fro_heads(g - w, as_output_type(r) - w, H) for g, r, w in zip(gpu[:3], ref[0], W)]
    errs.append(rel_fro_heads(gpu[3], ref[1], H, token_major=True))
    return errs
