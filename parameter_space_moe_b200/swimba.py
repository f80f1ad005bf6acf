"""Python binding of libswimba.so (include/swimba.h): argument marshalling only.

Every function here has the name of the C entry point without the "swimba_" prefix, takes torch
tensors that already live on the GPU, passes their data pointers and the current CUDA stream to the
library and raises SwimbaError on a non-OK status.  No arithmetic of the layer happens in Python; if
the compiled library is missing, importing this module fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswimba.so")

F32, BF16, F16 = 0, 1, 2
MIX_UNSCALED_B = 1
STATUS = {0: "SWIMBA_OK", 1: "SWIMBA_ERR_INVALID_ARG", 2: "SWIMBA_ERR_UNSUPPORTED", 3: "SWIMBA_ERR_CUDA",
          4: "SWIMBA_ERR_WORKSPACE", 5: "SWIMBA_ERR_TIMEOUT", 6: "SWIMBA_ERR_RANGE", 7: "SWIMBA_ERR_INDEX",
          8: "SWIMBA_ERR_UNSTABLE"}
EXPORTS = ("swimba_workspace_size", "swimba_stream_dtype", "swimba_router_topk", "swimba_dispatch",
           "swimba_expert_proj", "swimba_mix", "swimba_ssd_scan", "swimba_layer_fwd", "swimba_step",
           "swimba_separated_scan", "swimba_check_device_status", "swimba_status_string",
           "swimba_profile_enable", "swimba_profile_read", "swimba_launch_count", "swimba_dispatch_noalloc",
           "swimba_layer_fwd_host", "swimba_debug_scan_lost_first_chunk", "swimba_out_proj",
           "swimba_ssd_scan_bwd", "swimba_layer_bwd", "swimba_layer_bwd_workspace_size")


class SwimbaError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "seqlen", "d_model", "nheads", "headdim", "dstate",
                                              "ngroups", "n_experts", "top_k", "chunk", "dtype")]


class Weights(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("w_dt", ctypes.c_void_p), ("b_dt", ctypes.c_void_p),
                ("A", ctypes.c_void_p), ("w_exp", ctypes.c_void_p), ("A_exp", ctypes.c_void_p)]


_lib = None


def lib():
    """Load the compiled library (raises OSError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libswimba.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        P = ctypes.POINTER
        L.swimba_workspace_size.restype = sz
        L.swimba_workspace_size.argtypes = [P(Dims)]
        L.swimba_stream_dtype.restype = ctypes.c_int
        L.swimba_stream_dtype.argtypes = [P(Dims)]
        L.swimba_layer_bwd_workspace_size.restype = sz
        L.swimba_layer_bwd_workspace_size.argtypes = [P(Dims)]
        L.swimba_status_string.restype = ctypes.c_char_p
        L.swimba_status_string.argtypes = [ctypes.c_int]
        sig = {
            "swimba_router_topk": [P(Dims), vp, P(Weights), vp, vp, vp, vp],
            "swimba_dispatch": [P(Dims), vp, vp, vp, vp, sz, vp],
            "swimba_dispatch_noalloc": [P(Dims), vp, vp, vp, vp],
            "swimba_expert_proj": [P(Dims), vp, P(Weights), vp, vp, vp, sz, vp],
            "swimba_mix": [P(Dims), vp, vp, i32, vp, vp, vp, vp],
            "swimba_ssd_scan": [P(Dims), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "swimba_layer_fwd": [P(Dims), vp, P(Weights), vp, vp, vp, vp, vp, vp, sz, vp],
            "swimba_layer_fwd_host": [P(Dims), vp, P(Weights), vp, vp, vp, vp, vp, vp, sz, i32, vp],
            "swimba_debug_scan_lost_first_chunk": [P(Dims), vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "swimba_step": [P(Dims), vp, P(Weights), vp, vp, vp, vp, sz, vp],
            "swimba_separated_scan": [P(Dims), vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "swimba_out_proj": [P(Dims), vp, vp, vp, vp],
            "swimba_ssd_scan_bwd": [P(Dims), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "swimba_layer_bwd": [P(Dims), vp, P(Weights), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "swimba_check_device_status": [vp],
        }
        L.swimba_profile_enable.restype = ctypes.c_int
        L.swimba_profile_enable.argtypes = [ctypes.c_int]
        L.swimba_profile_read.restype = ctypes.c_int
        L.swimba_profile_read.argtypes = [P(ctypes.c_char_p), P(ctypes.c_float), ctypes.c_int]
        L.swimba_launch_count.restype = ctypes.c_longlong
        L.swimba_launch_count.argtypes = []
        for name, args in sig.items():
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = args
        _lib = L
    return _lib


def dims(batch, seqlen, d_model, nheads, headdim, dstate, ngroups, n_experts, top_k, chunk, dtype):
    return Dims(batch, seqlen, d_model, nheads, headdim, dstate, ngroups, n_experts, top_k, chunk, dtype)


def dims_of(w, seqlen=None, batch=None):
    """Dims of a configs.Workload (optionally overriding seqlen / batch)."""
    return dims(batch or w.batch, seqlen or w.seqlen, w.d_model, w.nheads, w.headdim, w.dstate, w.G,
                w.n_experts, w.top_k, w.chunk, BF16 if w.dtype == "bf16" else F32)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise SwimbaError(fn, code)


class WeightSet:
    """Device weights plus the C struct pointing at them (keeps the tensors alive)."""

    def __init__(self, w_router, w_dt, b_dt, A, w_exp, A_exp=None):
        self.tensors = (w_router, w_dt, b_dt, A, w_exp, A_exp)
        self.c = Weights(*(None if t is None else t.data_ptr() for t in self.tensors))


def workspace_size(d):
    return lib().swimba_workspace_size(ctypes.byref(d))


def stream_dtype(d):
    return lib().swimba_stream_dtype(ctypes.byref(d))


def router_topk(d, X, W, topk_idx, topk_w, dt, stream=None):
    _check("swimba_router_topk", lib().swimba_router_topk(ctypes.byref(d), _p(X), ctypes.byref(W.c), _p(topk_idx),
                                                           _p(topk_w), _p(dt), _stream(stream)))


def dispatch(d, topk_idx, expert_offsets, perm, ws, stream=None):
    _check("swimba_dispatch", lib().swimba_dispatch(ctypes.byref(d), _p(topk_idx), _p(expert_offsets), _p(perm),
                                                     _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def dispatch_noalloc(d, topk_idx, expert_offsets, perm, stream=None):
    """swimba_dispatch without a workspace (scratch in a fixed array inside the library); for callers
    that cannot allocate device memory."""
    _check("swimba_dispatch_noalloc", lib().swimba_dispatch_noalloc(ctypes.byref(d), _p(topk_idx),
                                                                     _p(expert_offsets), _p(perm), _stream(stream)))


def expert_proj(d, X, W, topk_idx, Z, ws, stream=None):
    _check("swimba_expert_proj", lib().swimba_expert_proj(ctypes.byref(d), _p(X), ctypes.byref(W.c), _p(topk_idx),
                                                           _p(Z), _p(ws), ws.numel() * ws.element_size(),
                                                           _stream(stream)))


def mix(d, Z, topk_w, flags, Bpi, Xs, Cpi, stream=None):
    _check("swimba_mix", lib().swimba_mix(ctypes.byref(d), _p(Z), _p(topk_w), flags, _p(Bpi), _p(Xs), _p(Cpi),
                                          _stream(stream)))


def ssd_scan(d, Bpi, Xs, Cpi, dt, A, init_state, y, final_state, chunk_states, ws, stream=None):
    _check("swimba_ssd_scan", lib().swimba_ssd_scan(ctypes.byref(d), _p(Bpi), _p(Xs), _p(Cpi), _p(dt), _p(A),
                                                     _p(init_state), _p(y), _p(final_state), _p(chunk_states),
                                                     _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def layer_fwd(d, X, W, init_state, y, final_state, topk_idx_out, topk_w_out, ws, stream=None):
    _check("swimba_layer_fwd", lib().swimba_layer_fwd(ctypes.byref(d), _p(X), ctypes.byref(W.c), _p(init_state),
                                                       _p(y), _p(final_state), _p(topk_idx_out), _p(topk_w_out),
                                                       _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def layer_fwd_host(d, X_host, W, init_state, y_host, final_state, X_dev, y_dev, ws, chunks=4, stream=None):
    """X_host / y_host: pinned CPU tensors; X_dev / y_dev: device staging tensors of the same shapes."""
    _check("swimba_layer_fwd_host", lib().swimba_layer_fwd_host(
        ctypes.byref(d), _p(X_host), ctypes.byref(W.c), _p(init_state), _p(y_host), _p(final_state), _p(X_dev),
        _p(y_dev), _p(ws), ws.numel() * ws.element_size(), int(chunks), _stream(stream)))


def step(d, X, W, state, y, topk_idx_out, ws, stream=None):
    _check("swimba_step", lib().swimba_step(ctypes.byref(d), _p(X), ctypes.byref(W.c), _p(state), _p(y),
                                             _p(topk_idx_out), _p(ws), ws.numel() * ws.element_size(),
                                             _stream(stream)))


def separated_scan(d, B, Xs, Cpi, dt, A, init_states, y, final_states, ws, stream=None):
    _check("swimba_separated_scan", lib().swimba_separated_scan(ctypes.byref(d), _p(B), _p(Xs), _p(Cpi), _p(dt),
                                                                 _p(A), _p(init_states), _p(y), _p(final_states),
                                                                 _p(ws), ws.numel() * ws.element_size(),
                                                                 _stream(stream)))


def ssd_scan_bwd(d, Bpi, Xs, Cpi, dt, A, init_state, dy, dBpi, dXs, dCt, d_dt, dA, d_init, ws, stream=None):
    _check("swimba_ssd_scan_bwd", lib().swimba_ssd_scan_bwd(
        ctypes.byref(d), _p(Bpi), _p(Xs), _p(Cpi), _p(dt), _p(A), _p(init_state), _p(dy), _p(dBpi), _p(dXs),
        _p(dCt), _p(d_dt), _p(dA), _p(d_init), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def layer_bwd_workspace_size(d):
    return lib().swimba_layer_bwd_workspace_size(ctypes.byref(d))


def layer_bwd(d, X, W, init_state, dy, dX, dW_r, dW_dt, db_dt, dA, dW_exp, d_init, ws, stream=None):
    _check("swimba_layer_bwd", lib().swimba_layer_bwd(
        ctypes.byref(d), _p(X), ctypes.byref(W.c), _p(init_state), _p(dy), _p(dX), _p(dW_r), _p(dW_dt), _p(db_dt),
        _p(dA), _p(dW_exp), _p(d_init), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def out_proj(d, y, w_out, out, stream=None):
    _check("swimba_out_proj", lib().swimba_out_proj(ctypes.byref(d), _p(y), _p(w_out), _p(out), _stream(stream)))


def debug_scan_lost_first_chunk(d, Bpi, Xs, Cpi, dt, A, y, ws, stream=None):
    _check("swimba_debug_scan_lost_first_chunk", lib().swimba_debug_scan_lost_first_chunk(
        ctypes.byref(d), _p(Bpi), _p(Xs), _p(Cpi), _p(dt), _p(A), _p(y), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def check_device_status(stream=None):
    """Synchronise the stream and return the device status code (0 = OK); clears the status word."""
    return lib().swimba_check_device_status(_stream(stream))


def status_string(code):
    return lib().swimba_status_string(code).decode()


def profile_enable(on=True):
    _check("swimba_profile_enable", lib().swimba_profile_enable(1 if on else 0))


def profile_read(max_stages=16):
    """[(stage name, milliseconds)] of the most recent entry-point call (waits for its events)."""
    names = (ctypes.c_char_p * max_stages)()
    ms = (ctypes.c_float * max_stages)()
    n = lib().swimba_profile_read(names, ms, max_stages)
    if n < 0:
        raise SwimbaError("swimba_profile_read", 3)
    return [(names[i].decode(), ms[i]) for i in range(n)]


def launch_count():
    return lib().swimba_launch_count()
