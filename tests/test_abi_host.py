"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/ttt.h declares, and rejects bad arguments before
anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttt.h")


@pytest.fixture(scope="module")
def B():
    from recon_chunk_ttt_b200 import build
    build.build()
    from recon_chunk_ttt_b200 import _binding
    return _binding


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("ttt_update", "ttt_apply", "ttt_stream_step", "ttt_update_workspace_bytes",
              "ttt_status_string", "ttt_shadow_bytes", "ttt_pack_shadow",
              "ttt_check_device_error", "ttt_chunked", "ttt_gate", "ttt_update_partial",
              "ttt_update_finish", "ttt_partial_floats", "ttt_finish_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol(B):
    L = B.lib()
    for n in declared_functions():
        assert hasattr(L, n), n


def test_status_strings(B):
    assert B.status_string(0) == "ok"
    assert "alignment" in B.status_string(B.TTT_ERR_ALIGNMENT) or \
        "aligned" in B.status_string(B.TTT_ERR_ALIGNMENT)
    assert B.status_string(99) == "unknown status"


def _cfg(B, **kw):
    base = dict(heads=4, d=256, hidden=512, renorm=B.RENORM_ROW, precision=B.PREC_BF16_TC)
    base.update(kw)
    return B.make_config(**base)


def test_workspace_sizes(B):
    cfg = _cfg(B)
    n = 961800
    ws = B.ttt_update_workspace_bytes(cfg, n)
    # the fused update keeps η·u, η·dh1, η·dh3 on chip: the workspace is the
    # S fp32 gradient partials and the renorm scratch, independent of n once
    # S stops growing
    S = B.ttt_update_splits(cfg, n)
    mat = 3 * 4 * 256 * 512
    assert 1 <= S <= 16
    assert S * mat * 4 <= ws < S * mat * 4 + 2**20
    assert ws < 64 * 2**20
    assert B.ttt_update_workspace_bytes(cfg, 10 * n) == ws
    assert B.ttt_update_workspace_bytes(cfg, 0) > 0
    f32 = B.ttt_update_workspace_bytes(_cfg(B, precision=B.PREC_FP32_CHECK), 1000)
    assert f32 >= 3 * 4 * 1000 * 512 * 4
    assert B.ttt_shadow_bytes(cfg) == 3 * 4 * 256 * 512 * 2
    assert B.ttt_update_workspace_bytes(_cfg(B, d=100), 10) == 0
    assert B.ttt_update_workspace_bytes(cfg, -1) == 0
    assert B.ttt_update_splits(_cfg(B, d=100), 10) == 0


def test_linear_mode_validation_and_sizes(B):
    """Linear fast weights (f_W(k) = W k): hidden must equal d, no
    Newton-Schulz; one d x d matrix per head in W1 (W2, W3 may be NULL), a
    one-matrix shadow and partial; an unknown form is an invalid argument."""
    lin = _cfg(B, hidden=256, mlp=B.MLP_LINEAR)
    assert B.ttt_shadow_bytes(lin) == 4 * 256 * 256 * 2
    assert B.ttt_partial_floats(lin) == 4 * 256 * 256
    assert B.ttt_update_workspace_bytes(lin, 1000) >= B.ttt_update_splits(lin, 1000) * 4 * 256 * 256 * 4
    assert B.ttt_update_workspace_bytes(_cfg(B, mlp=B.MLP_LINEAR), 10) == 0       # hidden != d
    assert B.ttt_update_workspace_bytes(_cfg(B, d=64, hidden=64, mlp=B.MLP_LINEAR), 10) > 0
    assert _update(B, _cfg(B, mlp=B.MLP_LINEAR)) == B.TTT_ERR_UNSUPPORTED_SHAPE
    assert _update(B, _cfg(B, hidden=256, mlp=B.MLP_LINEAR, ns_steps=2)) == B.TTT_ERR_UNSUPPORTED_SHAPE
    assert _update(B, _cfg(B, mlp=2)) == B.TTT_ERR_INVALID_ARG
    # W2, W3 and their outputs are not needed in linear mode: validation runs
    # on to the workspace check
    assert _update(B, lin, W2=None, W3=None, W2o=None, W3o=None, ws_bytes=100) == B.TTT_ERR_WORKSPACE
    assert _update(B, lin, W1=None) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B), W2=None) == B.TTT_ERR_INVALID_ARG                  # SwiGLU needs W2


def test_split_plan(B):
    """The gradient slots of the update: sets of (hidden / 128) 3-CTA clusters,
    as many as one wave holds (45 clusters resident on a B200: 11 sets for
    hidden 512), split the head-major tile space evenly with at least 4 tiles
    (512 tokens) per set, or, with at most 64 tiles per head, are aligned to
    heads (one slot per set of a head); a head's pieces fill at most S slots."""
    cfg = _cfg(B)
    assert B.ttt_update_splits(cfg, 0) == 1
    assert B.ttt_update_splits(cfg, 1) == 1
    assert B.ttt_update_splits(cfg, 512) == 1
    assert B.ttt_update_splits(cfg, 8192) == 2       # 64 tiles per head, aligned
    assert B.ttt_update_splits(cfg, 8193) == 4       # 65 tiles per head: 11 sets over 4 heads
    assert B.ttt_update_splits(cfg, 1374) == 2       # one 518 x 518 frame: 2 sets per head
    assert B.ttt_update_splits(cfg, 961800) == 4     # 11 sets over 4 heads
    assert B.ttt_update_splits(_cfg(B, heads=1), 961800) == 11
    assert B.ttt_update_splits(_cfg(B, heads=1, d=64, hidden=128), 108) == 1
    assert B.ttt_update_splits(_cfg(B, heads=64), 961800) == 2
    # Newton-Schulz: two d x hidden iterates, two d x d products and Delta per
    # matrix, on top of the update's own workspace (both precisions)
    for prec in (B.PREC_BF16_TC, B.PREC_FP32_CHECK):
        base = B.ttt_update_workspace_bytes(_cfg(B, precision=prec), 1000)
        ns = B.ttt_update_workspace_bytes(_cfg(B, precision=prec, ns_steps=5), 1000)
        assert ns - base >= 12 * (2 * 256 * 512 + 2 * 256 * 256 + 256 * 512) * 4


FAKE = 0x10000  # aligned, never dereferenced: validation fails first


def _update(B, cfg, n=10, ws_bytes=1 << 40, **over):
    args = dict(W1=FAKE, W2=FAKE, W3=FAKE, K=FAKE, V=FAKE, eta=FAKE, W1o=FAKE, W2o=FAKE,
                W3o=FAKE, shadow=None, ws=FAKE)
    args.update(over)
    L = B.lib()
    cp = ctypes.byref(cfg) if cfg is not None else None
    return L.ttt_update(cp, args["W1"], args["W2"], args["W3"], args["K"], args["V"],
                        args["eta"], n, args["W1o"], args["W2o"], args["W3o"], args["shadow"],
                        args["ws"], ws_bytes, None)


def test_update_rejects_bad_arguments(B):
    assert _update(B, None) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B, d=128, hidden=256)) == B.TTT_ERR_UNSUPPORTED_SHAPE
    assert _update(B, _cfg(B, ns_steps=-1)) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B, ns_steps=B.MAX_NS_STEPS + 1)) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B, renorm=7)) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B, precision=5)) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B, heads=0)) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B), n=-1) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B), W1=None) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B), K=None) == B.TTT_ERR_INVALID_ARG
    assert _update(B, _cfg(B), K=FAKE + 8) == B.TTT_ERR_ALIGNMENT
    assert _update(B, _cfg(B), eta=FAKE + 4) == B.TTT_ERR_ALIGNMENT
    assert _update(B, _cfg(B), ws=None) == B.TTT_ERR_WORKSPACE
    assert _update(B, _cfg(B), ws_bytes=100) == B.TTT_ERR_WORKSPACE


def test_apply_and_stream_reject_bad_arguments(B):
    L = B.lib()
    cfg = _cfg(B)
    # bf16 apply needs the shadow
    assert L.ttt_apply(ctypes.byref(cfg), None, None, None, None, FAKE, 5, FAKE,
                       None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_apply(ctypes.byref(cfg), None, None, None, FAKE, FAKE + 2, 5, FAKE,
                       None) == B.TTT_ERR_ALIGNMENT
    assert L.ttt_apply(ctypes.byref(cfg), None, None, None, FAKE, FAKE, -3, FAKE,
                       None) == B.TTT_ERR_INVALID_ARG
    f32 = _cfg(B, precision=B.PREC_FP32_CHECK)
    assert L.ttt_apply(ctypes.byref(f32), None, FAKE, FAKE, None, FAKE, 5, FAKE,
                       None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_stream_step(ctypes.byref(cfg), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 5,
                             FAKE, 5, FAKE, FAKE, 1 << 40, None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_pack_shadow(ctypes.byref(cfg), FAKE, FAKE, FAKE, None,
                             None) == B.TTT_ERR_INVALID_ARG


def test_product_path_does_not_touch_the_oracle():
    """The package and the kernels never import or link the oracle."""
    pkg = os.path.join(ROOT, "recon_chunk_ttt_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "ttt_oracle" not in txt, f


def test_chunked_rejects_bad_arguments(B):
    """Validation of ttt_chunked happens before any launch (FAKE pointers are
    never dereferenced)."""
    L = B.lib()
    cfg = _cfg(B)

    def call(cfg_, n=100, chunk=16, order=0, shadow=FAKE, eta=FAKE, ws=FAKE, ws_bytes=1 << 40,
             mask=None):
        return L.ttt_chunked(ctypes.byref(cfg_), FAKE, FAKE, FAKE, shadow, FAKE, FAKE, eta, FAKE,
                             n, chunk, order, mask, FAKE, ws, ws_bytes, None)

    assert call(cfg, order=2) == B.TTT_ERR_INVALID_ARG
    assert call(cfg, chunk=0) == B.TTT_ERR_INVALID_ARG
    assert call(cfg, n=-1) == B.TTT_ERR_INVALID_ARG
    assert call(cfg, shadow=None) == B.TTT_ERR_INVALID_ARG      # bf16 needs the shadow
    assert call(cfg, eta=FAKE + 4) == B.TTT_ERR_ALIGNMENT
    one_head = _cfg(B, heads=1)
    assert call(one_head, chunk=6) == B.TTT_ERR_ALIGNMENT       # eta rows of chunk 2 misaligned
    assert call(cfg, ws=None) == B.TTT_ERR_WORKSPACE
    assert call(cfg, ws_bytes=100) == B.TTT_ERR_WORKSPACE
    # the workspace is sized for the first (longest) chunk
    need = B.ttt_update_workspace_bytes(cfg, 16)
    assert need > 0 and call(cfg, ws_bytes=need - 1) == B.TTT_ERR_WORKSPACE
    # no chunk updates: no workspace needed; n = 0 is a no-op
    none = (ctypes.c_uint8 * 7)(*([0] * 7))
    assert call(cfg, n=0, ws=None) == B.TTT_OK
    f32 = _cfg(B, precision=B.PREC_FP32_CHECK)
    assert call(f32, n=0, shadow=None) == B.TTT_OK
    assert call(cfg, ws=None, mask=none, n=0) == B.TTT_OK


def test_gate_partial_finish_reject_bad_arguments(B):
    """Validation of ttt_gate, ttt_update_partial and ttt_update_finish happens
    before any launch (FAKE pointers are never dereferenced)."""
    L = B.lib()
    cfg = _cfg(B)
    c = ctypes.byref(cfg)
    # gate
    assert L.ttt_gate(None, FAKE, FAKE, 5, FAKE, None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_gate(c, None, FAKE, 5, FAKE, None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_gate(c, FAKE, None, 5, FAKE, None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_gate(c, FAKE, FAKE, -1, FAKE, None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_gate(c, FAKE + 8, FAKE, 5, FAKE, None) == B.TTT_ERR_ALIGNMENT
    assert L.ttt_gate(c, FAKE, FAKE, 0, None, None) == B.TTT_OK  # nothing to do
    assert L.ttt_gate(ctypes.byref(_cfg(B, d=128, hidden=256)), FAKE, FAKE, 5, FAKE,
                      None) == B.TTT_ERR_UNSUPPORTED_SHAPE
    # partial
    assert B.ttt_partial_floats(cfg) == 3 * 4 * 256 * 512
    assert L.ttt_update_partial(c, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10, None, FAKE, 1 << 40,
                                None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_update_partial(c, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, FAKE, FAKE, 1 << 40,
                                None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_update_partial(c, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 10, FAKE, FAKE,
                                1 << 40, None) == B.TTT_ERR_ALIGNMENT
    assert L.ttt_update_partial(c, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10, FAKE, FAKE, 100,
                                None) == B.TTT_ERR_WORKSPACE
    # finish
    need = B.ttt_finish_workspace_bytes(cfg)
    assert need > 0
    ns5 = _cfg(B, ns_steps=5)
    assert B.ttt_finish_workspace_bytes(ns5) > need  # the Newton-Schulz region
    args = [FAKE, FAKE, FAKE, FAKE]
    assert L.ttt_update_finish(c, *args, 0, FAKE, FAKE, FAKE, None, FAKE, need,
                               None) == B.TTT_ERR_INVALID_ARG   # no ranks
    assert L.ttt_update_finish(c, *args, 2, None, FAKE, FAKE, None, FAKE, need,
                               None) == B.TTT_ERR_INVALID_ARG
    assert L.ttt_update_finish(c, *args, 2, FAKE, FAKE, FAKE, None, FAKE, need - 1,
                               None) == B.TTT_ERR_WORKSPACE
    assert L.ttt_update_finish(c, *args, 2, FAKE, FAKE, FAKE, FAKE + 2, FAKE, need,
                               None) == B.TTT_ERR_ALIGNMENT


def test_static_stream_step_limit_and_rejection(B):
    """ttt_stream_step_static's fixed 96 MiB scratch, per configuration (the
    limits the header states): BF16_TC keeps its intermediates on chip, so 4
    heads of d = 256 fit for every n with and without Newton-Schulz, and for
    every n up to 31 (ns_steps = 0) or 6 (ns_steps > 0) such heads fit;
    FP32_CHECK fits 3,836 tokens (2,044 with Newton-Schulz).  A call over the
    limit is rejected with TTT_ERR_WORKSPACE before anything touches a device."""
    cap = 96 << 20
    ws = B.ttt_update_workspace_bytes
    for ns in (0, 5):
        cfg = _cfg(B, ns_steps=ns)
        assert ws(cfg, 1374) <= cap and ws(cfg, 10**9) <= cap
    assert ws(_cfg(B, heads=31), 10**9) <= cap < ws(_cfg(B, heads=32), 10**9)
    assert ws(_cfg(B, heads=6, ns_steps=5), 10**9) <= cap < ws(_cfg(B, heads=7, ns_steps=5), 10**9)
    f32 = _cfg(B, precision=B.PREC_FP32_CHECK)
    f32ns = _cfg(B, precision=B.PREC_FP32_CHECK, ns_steps=5)
    assert ws(f32, 3836) <= cap < ws(f32, 3837)
    assert ws(f32ns, 2044) <= cap < ws(f32ns, 2045)
    assert ws(f32, 1374) <= cap and ws(f32ns, 1374) <= cap   # one frame fits either way
    L = B.lib()
    f = L.ttt_stream_step_static
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [ctypes.POINTER(B.ttt_config), P, P, P, P, P, P, P, I64, P, I64, P, P]
    f.restype = ctypes.c_int
    for cfg, n in ((f32, 3837), (f32ns, 2045), (_cfg(B, heads=32), 10**6)):
        args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, n, FAKE, 5, FAKE, None]
        assert f(ctypes.byref(cfg), *args) == B.TTT_ERR_WORKSPACE
    assert f(None, *[FAKE] * 7, 5, FAKE, 5, FAKE, None) == B.TTT_ERR_INVALID_ARG
