"""ctypes binding of libttt.so (include/ttt.h).

Argument marshalling only: torch tensors are turned into device pointers and
sizes, the C function runs every step of the layer in the library's CUDA
kernels, and a non-OK status raises TTTError.  PyTorch serves only for device
memory and streams.  There is no fallback: if libttt.so is missing or fails to
load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# RECON_CHUNK_TTT_LIB may name another build of the same library (the debug
# build, libttt_debug.so); it must exist, there is no fallback.
LIB_PATH = os.environ.get("RECON_CHUNK_TTT_LIB") or os.path.join(_HERE, "libttt.so")

TTT_OK, TTT_ERR_INVALID_ARG, TTT_ERR_UNSUPPORTED_SHAPE, TTT_ERR_ALIGNMENT, \
    TTT_ERR_WORKSPACE, TTT_ERR_CUDA, TTT_ERR_DEVICE = range(7)
MAX_NS_STEPS = 32  # TTT_MAX_NS_STEPS
MLP_SWIGLU, MLP_LINEAR = 0, 1
RENORM_OFF, RENORM_ROW, RENORM_FROB = 0, 1, 2
PREC_BF16_TC, PREC_FP32_CHECK = 0, 1


class ttt_config(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("d", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("mlp", ctypes.c_int32), ("renorm", ctypes.c_int32),
                ("ns_steps", ctypes.c_int32), ("precision", ctypes.c_int32)]


def make_config(heads: int, d: int, hidden: int, renorm: int = RENORM_ROW,
                precision: int = PREC_BF16_TC, mlp: int = MLP_SWIGLU,
                ns_steps: int = 0) -> ttt_config:
    return ttt_config(heads, d, hidden, mlp, renorm, ns_steps, precision)


class ttt_trace_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


class TTTError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_CFG = ctypes.POINTER(ttt_config)


def lib() -> ctypes.CDLL:
    """Load libttt.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m recon_chunk_ttt_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.ttt_status_string.argtypes = [ctypes.c_int]
        L.ttt_status_string.restype = ctypes.c_char_p
        L.ttt_update_workspace_bytes.argtypes = [_CFG, _I64]
        L.ttt_update_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_shadow_bytes.argtypes = [_CFG]
        L.ttt_shadow_bytes.restype = ctypes.c_size_t
        L.ttt_update.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _P,
                                 ctypes.c_size_t, _P]
        L.ttt_update.restype = ctypes.c_int
        L.ttt_apply.argtypes = [_CFG, _P, _P, _P, _P, _P, _I64, _P, _P]
        L.ttt_apply.restype = ctypes.c_int
        L.ttt_pack_shadow.argtypes = [_CFG, _P, _P, _P, _P, _P]
        L.ttt_pack_shadow.restype = ctypes.c_int
        L.ttt_stream_step.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I64, _P, _P,
                                      ctypes.c_size_t, _P]
        L.ttt_stream_step.restype = ctypes.c_int
        L.ttt_gate.argtypes = [_CFG, _P, _P, _I64, _P, _P]
        L.ttt_gate.restype = ctypes.c_int
        L.ttt_partial_floats.argtypes = [_CFG]
        L.ttt_partial_floats.restype = ctypes.c_size_t
        L.ttt_update_splits.argtypes = [_CFG, _I64]
        L.ttt_update_splits.restype = ctypes.c_int32
        L.ttt_finish_workspace_bytes.argtypes = [_CFG]
        L.ttt_finish_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_update_partial.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _I64, _P, _P,
                                         ctypes.c_size_t, _P]
        L.ttt_update_partial.restype = ctypes.c_int
        L.ttt_update_finish.argtypes = [_CFG, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]
        L.ttt_update_finish.restype = ctypes.c_int
        L.ttt_chunked.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64,
                                  ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]
        L.ttt_chunked.restype = ctypes.c_int
        L.ttt_selftest_wait_timeout.argtypes = [_I64, _P]
        L.ttt_selftest_wait_timeout.restype = ctypes.c_int
        L.ttt_check_device_error.argtypes = [_P, ctypes.POINTER(ctypes.c_int32)]
        L.ttt_check_device_error.restype = ctypes.c_int
        L.ttt_trace_enable.argtypes = [ctypes.c_int32]
        L.ttt_trace_enable.restype = ctypes.c_int
        L.ttt_trace_read.argtypes = [ctypes.POINTER(ttt_trace_entry), ctypes.c_int32,
                                     ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
        L.ttt_trace_read.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ttt_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str):
    if status != TTT_OK:
        raise TTTError(status, what)


def _token_dtype(cfg: ttt_config):
    return torch.float32 if cfg.precision == PREC_FP32_CHECK else torch.bfloat16


def ttt_update_workspace_bytes(cfg: ttt_config, n_tokens: int) -> int:
    return int(lib().ttt_update_workspace_bytes(ctypes.byref(cfg), int(n_tokens)))


def ttt_shadow_bytes(cfg: ttt_config) -> int:
    return int(lib().ttt_shadow_bytes(ctypes.byref(cfg)))


def alloc_workspace(cfg: ttt_config, n_tokens: int, device=None) -> torch.Tensor:
    nbytes = ttt_update_workspace_bytes(cfg, n_tokens)
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device or "cuda")


def alloc_shadow(cfg: ttt_config, device=None) -> torch.Tensor:
    return torch.empty(ttt_shadow_bytes(cfg) // 2, dtype=torch.bfloat16, device=device or "cuda")


def ttt_update(cfg: ttt_config, W1, W2, W3, K, V, eta, W1_out=None, W2_out=None, W3_out=None,
               shadow=None, workspace=None, stream=None):
    """Ŵ = renorm(W - ∇_W Σ η_i (-f_W(k_i)^T v_i)); returns (W1_out, W2_out, W3_out)."""
    n = int(K.shape[0]) if K is not None else 0
    W1_out = torch.empty_like(W1) if W1_out is None else W1_out
    W2_out = torch.empty_like(W2) if W2_out is None and W2 is not None else W2_out
    W3_out = torch.empty_like(W3) if W3_out is None and W3 is not None else W3_out
    if workspace is None:
        workspace = alloc_workspace(cfg, n, W1.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().ttt_update(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3), _ptr(K), _ptr(V),
                            _ptr(eta), n, _ptr(W1_out), _ptr(W2_out), _ptr(W3_out),
                            _ptr(shadow), _ptr(workspace), nbytes, _stream(stream)),
           "ttt_update")
    return W1_out, W2_out, W3_out


def ttt_apply(cfg: ttt_config, Q, O=None, W1=None, W2=None, W3=None, shadow=None, stream=None):
    """O[i] = f_Ŵ(Q[i]) per head; returns O."""
    m = int(Q.shape[0])
    if O is None:
        O = torch.empty((m, cfg.heads * cfg.d), dtype=_token_dtype(cfg), device=Q.device)
    _check(lib().ttt_apply(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3), _ptr(shadow),
                           _ptr(Q), m, _ptr(O), _stream(stream)), "ttt_apply")
    return O


def ttt_pack_shadow(cfg: ttt_config, W1, W2, W3, shadow=None, stream=None):
    if shadow is None:
        shadow = alloc_shadow(cfg, W1.device)
    _check(lib().ttt_pack_shadow(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3),
                                 _ptr(shadow), _stream(stream)), "ttt_pack_shadow")
    return shadow


def ttt_stream_step(cfg: ttt_config, W1, W2, W3, shadow, K, V, eta, Q, O=None,
                    workspace=None, stream=None):
    """Update the state (W1, W2, W3, shadow) in place with one frame, then
    apply it to the frame's queries; returns O."""
    n, m = int(K.shape[0]), int(Q.shape[0])
    if O is None:
        O = torch.empty((m, cfg.heads * cfg.d), dtype=_token_dtype(cfg), device=Q.device)
    if workspace is None:
        workspace = alloc_workspace(cfg, n, W1.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().ttt_stream_step(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3), _ptr(shadow),
                                 _ptr(K), _ptr(V), _ptr(eta), n, _ptr(Q), m, _ptr(O),
                                 _ptr(workspace), nbytes, _stream(stream)), "ttt_stream_step")
    return O


GATE_EPS = 1e-6  # TTT_GATE_EPS


def ttt_gate(cfg: ttt_config, Wg, O_prime, O=None, stream=None):
    """o = RMSNorm(o') * SiLU(W_g o') per head; O may be O_prime (in place)."""
    m = int(O_prime.shape[0])
    if O is None:
        O = torch.empty_like(O_prime)
    _check(lib().ttt_gate(ctypes.byref(cfg), _ptr(Wg), _ptr(O_prime), m, _ptr(O),
                          _stream(stream)), "ttt_gate")
    return O


def ttt_partial_floats(cfg: ttt_config) -> int:
    return int(lib().ttt_partial_floats(ctypes.byref(cfg)))


def ttt_update_splits(cfg: ttt_config, n_tokens: int) -> int:
    return int(lib().ttt_update_splits(ctypes.byref(cfg), n_tokens))


def ttt_finish_workspace_bytes(cfg: ttt_config) -> int:
    return int(lib().ttt_finish_workspace_bytes(ctypes.byref(cfg)))


def ttt_update_partial(cfg: ttt_config, W1, W2, W3, K, V, eta, partial=None, workspace=None,
                       stream=None):
    """This rank's gradient partial ([H][3][hidden*d] fp32: g1, g3, -g2)."""
    n = int(K.shape[0])
    if partial is None:
        partial = torch.empty(ttt_partial_floats(cfg), dtype=torch.float32, device=W1.device)
    if workspace is None:
        workspace = alloc_workspace(cfg, n, W1.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().ttt_update_partial(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3), _ptr(K),
                                    _ptr(V), _ptr(eta), n, _ptr(partial), _ptr(workspace), nbytes,
                                    _stream(stream)), "ttt_update_partial")
    return partial


def ttt_update_finish(cfg: ttt_config, W1, W2, W3, partials, W1_out=None, W2_out=None,
                      W3_out=None, shadow=None, workspace=None, stream=None):
    """Ŵ from the ranks' partials ([ranks, partial_floats], summed in rank
    order); returns (W1_out, W2_out, W3_out)."""
    ranks = int(partials.shape[0]) if partials.dim() == 2 else 1
    outs = [o if o is not None or w is None else torch.empty_like(w)
            for o, w in ((W1_out, W1), (W2_out, W2), (W3_out, W3))]
    if workspace is None:
        workspace = torch.empty(max(ttt_finish_workspace_bytes(cfg), 1), dtype=torch.uint8,
                                device=W1.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().ttt_update_finish(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3),
                                   _ptr(partials), ranks, _ptr(outs[0]), _ptr(outs[1]),
                                   _ptr(outs[2]), _ptr(shadow), _ptr(workspace), nbytes,
                                   _stream(stream)), "ttt_update_finish")
    return tuple(outs)


ORDER_UPDATE_THEN_APPLY, ORDER_APPLY_THEN_UPDATE = 0, 1  # TTT_ORDER_*


def ttt_chunked(cfg: ttt_config, W1, W2, W3, shadow, K, V, eta, Q, chunk: int,
                order: int = ORDER_UPDATE_THEN_APPLY, update_mask=None, O=None,
                workspace=None, stream=None):
    """Chunk loop over the n tokens (update and apply per chunk in `order`,
    updates only where update_mask is nonzero); the state (W1, W2, W3,
    shadow) is updated in place; returns O for all n tokens."""
    n = int(K.shape[0])
    if O is None:
        O = torch.empty((n, cfg.heads * cfg.d), dtype=_token_dtype(cfg), device=Q.device)
    first = min(int(chunk), n) if n else 0
    if workspace is None:
        workspace = alloc_workspace(cfg, first, W1.device)
    nbytes = workspace.numel() * workspace.element_size()
    mask = None
    if update_mask is not None:
        mask = (ctypes.c_uint8 * len(update_mask))(*[1 if m else 0 for m in update_mask])
    _check(lib().ttt_chunked(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3), _ptr(shadow),
                             _ptr(K), _ptr(V), _ptr(eta), _ptr(Q), n, int(chunk), int(order),
                             mask, _ptr(O), _ptr(workspace), nbytes, _stream(stream)),
           "ttt_chunked")
    return O


DEVICE_ERR_SELFTEST = 7  # TTT_DEVICE_ERR_SELFTEST


def ttt_selftest_wait_timeout(limit_cycles: int = 1 << 24, stream=None) -> None:
    """Launch the failure-detection self-test: a bounded wait that runs out
    after limit_cycles and reports DEVICE_ERR_SELFTEST in the error word."""
    _check(lib().ttt_selftest_wait_timeout(int(limit_cycles), _stream(stream)),
           "ttt_selftest_wait_timeout")


def ttt_check_device_error(stream=None) -> int:
    """Synchronise and read/clear the device error word; raises TTTError on a
    kernel-reported error."""
    code = ctypes.c_int32(0)
    st = lib().ttt_check_device_error(_stream(stream), ctypes.byref(code))
    if st != TTT_OK:
        raise TTTError(st, f"device error word = {code.value}")
    return code.value


def ttt_trace_enable(on: bool = True) -> None:
    """Bracket every kernel launch of the library with CUDA events."""
    _check(lib().ttt_trace_enable(1 if on else 0), "ttt_trace_enable")


def ttt_trace_read(reset: bool = True) -> dict:
    """{kernel name: (launches, total device ms)} since the last reset."""
    cap = 64
    arr = (ttt_trace_entry * cap)()
    cnt = ctypes.c_int32(0)
    _check(lib().ttt_trace_read(arr, cap, ctypes.byref(cnt), 1 if reset else 0),
           "ttt_trace_read")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms))
            for i in range(min(cnt.value, cap))}


def ttt_stream_step_static(cfg: ttt_config, W1, W2, W3, shadow, K, V, eta, Q, O=None,
                           stream=None):
    """ttt_stream_step without a workspace argument: the library's fixed
    device scratch is used, so the call allocates nothing on the device (O is
    allocated here only when not given)."""
    L = lib()
    if not hasattr(L.ttt_stream_step_static, "_typed"):
        L.ttt_stream_step_static.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I64,
                                             _P, _P]
        L.ttt_stream_step_static.restype = ctypes.c_int
        L.ttt_stream_step_static._typed = True
    n, m = int(K.shape[0]), int(Q.shape[0])
    if O is None:
        O = torch.empty((m, cfg.heads * cfg.d), dtype=_token_dtype(cfg), device=Q.device)
    _check(L.ttt_stream_step_static(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W3),
                                    _ptr(shadow), _ptr(K), _ptr(V), _ptr(eta), n, _ptr(Q), m,
                                    _ptr(O), _stream(stream)), "ttt_stream_step_static")
    return O
