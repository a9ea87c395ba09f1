"""ctypes binding of libttt_b200.so (include/ttt.h).

Argument marshalling only: every function forwards plain pointers and sizes
to the C ABI of the same name.  Tensors are passed by ``data_ptr()``; streams
by their CUDA handle.  Nothing here computes any part of the layer.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttt_b200.so")

TTT_OK, TTT_ERR_ARG, TTT_ERR_SHAPE, TTT_ERR_ALIGN, TTT_ERR_DTYPE = 0, -1, -2, -3, -4
TTT_ERR_UNSUPPORTED, TTT_ERR_WORKSPACE, TTT_ERR_CUDA, TTT_ERR_TIMEOUT = -5, -6, -7, -8
TTT_F32, TTT_BF16 = 0, 1
TTT_CAUSAL, TTT_BIDIRECTIONAL = 0, 1
TTT_OPT_GD, TTT_OPT_MOMENTUM, TTT_OPT_MUON = 0, 1, 2
TTT_STATUS_BYTES = 256


class TTTError(RuntimeError):
    def __init__(self, fn: str, status: int, name: str):
        super().__init__(f"{fn} failed: {name} ({status})")
        self.status = status


class ttt_linear_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("order", ctypes.c_int), ("include_diag", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int)]


class lact_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N_in", ctypes.c_int),
                ("N_q", ctypes.c_int), ("d", ctypes.c_int), ("dh", ctypes.c_int),
                ("chunk", ctypes.c_int), ("order", ctypes.c_int), ("opt", ctypes.c_int),
                ("beta", ctypes.c_float), ("ns_steps", ctypes.c_int),
                ("ns_coef", ctypes.c_float * 3), ("ns_eps", ctypes.c_float),
                ("normalize_rows", ctypes.c_int), ("norm_eps", ctypes.c_float),
                ("update_mask", ctypes.c_int), ("in_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("split_operands", ctypes.c_int)]


class ttt_window_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("window", ctypes.c_int), ("scale", ctypes.c_float), ("in_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("accumulate", ctypes.c_int)]


class ttt_prof_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


_VP, _SZ, _SZP, _I = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t), ctypes.c_int
_SIGS = {
    "ttt_linear_workspace_bytes": [ctypes.POINTER(ttt_linear_desc), _SZP],
    "ttt_linear_state_init": [ctypes.POINTER(ttt_linear_desc), _VP, _VP, _VP],
    "ttt_linear_state_readout": [ctypes.POINTER(ttt_linear_desc), _VP, _VP, _VP],
    "ttt_linear_fwd": [ctypes.POINTER(ttt_linear_desc), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ,
                       _VP],
    "ttt_linear_bwd_workspace_bytes": [ctypes.POINTER(ttt_linear_desc), _SZP],
    "ttt_linear_bwd": [ctypes.POINTER(ttt_linear_desc)] + [_VP] * 13 + [_SZ, _VP],
    "ttt_window_attn_fwd": [ctypes.POINTER(ttt_window_desc), _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "lact_layer_fwd": [ctypes.POINTER(lact_desc), _I, ctypes.c_float, _VP, _VP, _VP, _VP, _VP, _VP,
                       _VP, _SZ, _VP],
    "lact_state_bytes": [ctypes.POINTER(lact_desc), _SZP],
    "lact_workspace_bytes": [ctypes.POINTER(lact_desc), _SZP],
    "lact_workspace_bytes_min": [ctypes.POINTER(lact_desc), _SZP],
    "lact_state_init": [ctypes.POINTER(lact_desc), _VP, _VP, _VP, _I, _VP, _VP],
    "lact_state_readout": [ctypes.POINTER(lact_desc), _VP, _VP, _VP, _VP, _VP, _VP],
    "lact_chunk_fwd": [ctypes.POINTER(lact_desc), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "lact_grad_bytes": [ctypes.POINTER(lact_desc), _SZP],
    "lact_chunk_grad": [ctypes.POINTER(lact_desc), _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "lact_apply_grad": [ctypes.POINTER(lact_desc), _VP, _VP, _VP, _SZ, _VP],
    "lact_read": [ctypes.POINTER(lact_desc), _I, _I, _VP, _VP, _VP, _VP, _SZ, _VP],
    "lact_bwd_workspace_bytes": [ctypes.POINTER(lact_desc), _SZP],
    "lact_chunk_bwd": [ctypes.POINTER(lact_desc)] + [_VP] * 13 + [_SZ, _VP],
    "lact_chunk_fwd_noalloc": [ctypes.POINTER(lact_desc), _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "lact_noalloc_check_status": [_VP],
    "ttt_check_device_status": [_VP, _VP],
    "ttt_selftest_wait_timeout": [_VP, _SZ, _I, _VP],
    "ttt_profile_begin": [],
    "ttt_profile_end": [ctypes.POINTER(ttt_prof_entry), _I, ctypes.POINTER(ctypes.c_int)],
    "ttt_status_string": [_I],
    "ttt_build_info": [],
}

_lib = None


def load():
    """Load the in-tree library; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m learned_linear_attention_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name in ("ttt_status_string", "ttt_build_info") \
                else ctypes.c_int
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().ttt_status_string(int(status)).decode()


def _check(fn: str, status: int) -> int:
    if status != TTT_OK:
        raise TTTError(fn, status, status_string(status))
    return status


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ linear
def ttt_linear_workspace_bytes(desc: ttt_linear_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("ttt_linear_workspace_bytes", load().ttt_linear_workspace_bytes(ctypes.byref(desc),
                                                                          ctypes.byref(n)))
    return n.value


def ttt_linear_state_init(desc, S0, S, stream=None):
    return _check("ttt_linear_state_init",
                  load().ttt_linear_state_init(ctypes.byref(desc), _ptr(S0), _ptr(S),
                                               _stream(stream)))


def ttt_linear_state_readout(desc, S, dst, stream=None):
    return _check("ttt_linear_state_readout",
                  load().ttt_linear_state_readout(ctypes.byref(desc), _ptr(S), _ptr(dst),
                                                  _stream(stream)))


def ttt_linear_fwd(desc, q, k, v, lr, S, out, ws, ws_bytes=None, stream=None, check=True):
    nbytes = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    st = load().ttt_linear_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(S),
                               _ptr(out), _ptr(ws), nbytes, _stream(stream))
    return _check("ttt_linear_fwd", st) if check else st


def ttt_linear_bwd_workspace_bytes(desc: ttt_linear_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("ttt_linear_bwd_workspace_bytes",
           load().ttt_linear_bwd_workspace_bytes(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def ttt_linear_bwd(desc, q, k, v, lr, S0, dout, dS_end, dq, dk, dv, dlr, dS0, ws, ws_bytes=None,
                   stream=None, check=True):
    """Gradients of sum <dout, out> + <dS_end, S_end> (see include/ttt.h);
    S0 and dS_end may be None (zeros)."""
    nbytes = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    st = load().ttt_linear_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(S0),
                               _ptr(dout), _ptr(dS_end), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlr),
                               _ptr(dS0), _ptr(ws), nbytes, _stream(stream))
    return _check("ttt_linear_bwd", st) if check else st


def ttt_window_attn_fwd(desc, q, k, v, out, ws, ws_bytes=None, stream=None, check=True):
    nbytes = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    st = load().ttt_window_attn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                    _ptr(ws), nbytes, _stream(stream))
    return _check("ttt_window_attn_fwd", st) if check else st


def lact_layer_fwd(desc, window, scale, q, k, v, lr, state, out, ws, ws_bytes=None, stream=None,
                   check=True):
    nbytes = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    st = load().lact_layer_fwd(ctypes.byref(desc), int(window), float(scale), _ptr(q), _ptr(k),
                               _ptr(v), _ptr(lr), _ptr(state), _ptr(out), _ptr(ws), nbytes,
                               _stream(stream))
    return _check("lact_layer_fwd", st) if check else st


# ------------------------------------------------------------------ LaCT
def lact_state_bytes(desc: lact_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("lact_state_bytes", load().lact_state_bytes(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def lact_workspace_bytes(desc: lact_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("lact_workspace_bytes", load().lact_workspace_bytes(ctypes.byref(desc),
                                                              ctypes.byref(n)))
    return n.value


def lact_workspace_bytes_min(desc: lact_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("lact_workspace_bytes_min", load().lact_workspace_bytes_min(ctypes.byref(desc),
                                                                      ctypes.byref(n)))
    return n.value


def lact_state_init(desc, W1, W3, W2, w_per_batch, state, stream=None):
    return _check("lact_state_init",
                  load().lact_state_init(ctypes.byref(desc), _ptr(W1), _ptr(W3), _ptr(W2),
                                         int(w_per_batch), _ptr(state), _stream(stream)))


def lact_state_readout(desc, state, W1, W3, W2, M=None, stream=None):
    return _check("lact_state_readout",
                  load().lact_state_readout(ctypes.byref(desc), _ptr(state), _ptr(W1), _ptr(W3),
                                            _ptr(W2), _ptr(M), _stream(stream)))


def lact_chunk_fwd(desc, q, k, v, lr, state, out, ws, ws_bytes=None, stream=None, check=True):
    nbytes = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    st = load().lact_chunk_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lr),
                               _ptr(state), _ptr(out), _ptr(ws), nbytes, _stream(stream))
    return _check("lact_chunk_fwd", st) if check else st


def lact_grad_bytes(desc: lact_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("lact_grad_bytes", load().lact_grad_bytes(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def _nbytes(ws, ws_bytes):
    return ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()


def lact_chunk_grad(desc, t0, n, k, v, lr, state, G, ws, ws_bytes=None, stream=None, check=True):
    st = load().lact_chunk_grad(ctypes.byref(desc), int(t0), int(n), _ptr(k), _ptr(v), _ptr(lr),
                                _ptr(state), _ptr(G), _ptr(ws), _nbytes(ws, ws_bytes),
                                _stream(stream))
    return _check("lact_chunk_grad", st) if check else st


def lact_apply_grad(desc, G, state, ws, ws_bytes=None, stream=None, check=True):
    st = load().lact_apply_grad(ctypes.byref(desc), _ptr(G), _ptr(state), _ptr(ws),
                                _nbytes(ws, ws_bytes), _stream(stream))
    return _check("lact_apply_grad", st) if check else st


def lact_read(desc, t0, n, q, state, out, ws, ws_bytes=None, stream=None, check=True):
    st = load().lact_read(ctypes.byref(desc), int(t0), int(n), _ptr(q), _ptr(state), _ptr(out),
                          _ptr(ws), _nbytes(ws, ws_bytes), _stream(stream))
    return _check("lact_read", st) if check else st


def lact_bwd_workspace_bytes(desc: lact_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("lact_bwd_workspace_bytes",
           load().lact_bwd_workspace_bytes(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def lact_chunk_bwd(desc, q, k, v, lr, state0, dout, dW_end, dq, dk, dv, dlr, dW0, ws,
                   ws_bytes=None, stream=None, check=True):
    """Gradients of sum <dout, out> + <dW_end, W_end> (see include/ttt.h)."""
    st = load().lact_chunk_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lr),
                               _ptr(state0), _ptr(dout), _ptr(dW_end), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(dlr), _ptr(dW0), _ptr(ws), _nbytes(ws, ws_bytes),
                               _stream(stream))
    return _check("lact_chunk_bwd", st) if check else st


def lact_chunk_fwd_noalloc(desc, q, k, v, lr, state, out, stream=None, check=True):
    """lact_chunk_fwd with the library's fixed device scratch as workspace."""
    st = load().lact_chunk_fwd_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lr),
                                       _ptr(state), _ptr(out), _stream(stream))
    return _check("lact_chunk_fwd_noalloc", st) if check else st


def lact_noalloc_check_status(stream=None) -> int:
    """Status of the last lact_chunk_fwd_noalloc call on the current device."""
    return load().lact_noalloc_check_status(_stream(stream))


# ------------------------------------------------------------------ status
def ttt_check_device_status(ws, stream=None) -> int:
    return load().ttt_check_device_status(_ptr(ws), _stream(stream))


def ttt_selftest_wait_timeout(ws, timeout_us: int, stream=None) -> int:
    return load().ttt_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(),
                                            int(timeout_us), _stream(stream))


def ttt_profile_begin() -> int:
    return _check("ttt_profile_begin", load().ttt_profile_begin())


def ttt_profile_end() -> dict:
    """Per kernel kind: {"launches": n, "total_ms": t} (event-timed)."""
    arr = (ttt_prof_entry * 32)()
    n = ctypes.c_int(0)
    _check("ttt_profile_end", load().ttt_profile_end(arr, 32, ctypes.byref(n)))
    return {arr[i].name.decode(): {"launches": arr[i].launches, "total_ms": arr[i].total_ms}
            for i in range(min(n.value, 32))}


def ttt_build_info() -> str:
    return load().ttt_build_info().decode()
