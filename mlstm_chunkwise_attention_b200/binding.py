"""Thin Python binding of libmlstm.so (ctypes).

The functions named like the C ABI (``mlstm_fwd``, ``mlstm_bwd``, the size
queries) marshal plain integers (device pointers, sizes, a stream handle) and
return the C status.  ``forward`` / ``backward`` are conveniences for torch
tensors: they allocate outputs and buffers through PyTorch (plumbing only) and
call the same entry points.  Every step of the computation runs in the CUDA
library; if it is not built this module raises instead of computing anything.
"""

import ctypes
import os

SIG = 0
EXP = 1
BF16 = 0
FP32 = 1

STATUS_OK = 0
STATUS_INVALID = 1
STATUS_UNSUPPORTED = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmlstm.so")
_lib = None


class MLSTMError(RuntimeError):
    def __init__(self, status, where):
        lib = load()
        msg = lib.mlstm_status_string(status).decode()
        detail = lib.mlstm_last_error().decode()
        super().__init__(f"{where}: {msg} ({status}){': ' + detail if detail else ''}")
        self.status = status


class SavedLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "gate_b", "gate_li", "gate_m", "norm", "state_c", "state_n", "tile_table",
        "gate_b_bytes", "gate_li_bytes", "gate_m_bytes", "norm_bytes", "state_c_bytes",
        "state_n_bytes", "tile_table_bytes", "total")]


_SIZES = [ctypes.c_int] * 8  # B, NH, T, d_qk, d_hv, chunk, variant, dtype
_P = ctypes.c_void_p

EXPORTS = {
    "mlstm_saved_layout": (ctypes.c_int, _SIZES + [ctypes.POINTER(SavedLayout)]),
    "mlstm_saved_size": (ctypes.c_size_t, _SIZES),
    "mlstm_fwd_workspace_size": (ctypes.c_size_t, _SIZES),
    "mlstm_bwd_workspace_size": (ctypes.c_size_t, _SIZES),
    "mlstm_fwd_launch_count": (ctypes.c_int, _SIZES),
    "mlstm_bwd_launch_count": (ctypes.c_int, _SIZES),
    "mlstm_fwd": (ctypes.c_int, [_P] * 7 + [_P, ctypes.c_size_t] + _SIZES + [_P]),
    "mlstm_bwd": (ctypes.c_int, [_P] * 13 + [_P, ctypes.c_size_t] + _SIZES + [_P]),
    "mlstm_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mlstm_last_error": (ctypes.c_char_p, []),
    "mlstm_launch_name": (ctypes.c_char_p, [ctypes.c_int, ctypes.c_int] + _SIZES),
    "mlstm_set_timing_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
    "mlstm_set_serial_launches": (ctypes.c_int, [ctypes.c_int]),
    "mlstm_device_status": (ctypes.c_int, [_P]),
    "mlstm_selftest_timeout": (ctypes.c_int, [_P]),
    "mlstm_fwd_noalloc": (ctypes.c_int, [_P] * 6 + _SIZES + [_P]),
    "mlstm_state_size": (ctypes.c_size_t, [ctypes.c_int] * 5),
    "mlstm_state_zero": (ctypes.c_int, [_P] + [ctypes.c_int] * 5 + [_P]),
    "mlstm_final_state": (ctypes.c_int, [_P] * 4 + _SIZES + [_P]),
    "mlstm_step": (ctypes.c_int, [_P] * 8 + [ctypes.c_int] * 6 + [_P]),
    "mlstm_fwd_state": (ctypes.c_int, [_P] * 7 + [_P, ctypes.c_size_t, _P, _P] + _SIZES + [_P]),
    "mlstm_bwd_state": (ctypes.c_int, [_P] * 16 + [_P, ctypes.c_size_t] + _SIZES + [_P]),
    "mlstm_log_decay": (ctypes.c_int, [_P, _P] + [ctypes.c_int] * 4 + [_P]),
    "mlstm_state_chain": (ctypes.c_int, [_P] * 4 + [ctypes.c_int] * 5 + [_P]),
    "mlstm_dstate_chain": (ctypes.c_int, [_P] * 6 + [ctypes.c_int] * 5 + [_P]),
}


def load(path=None):
    """Load the CUDA library once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} is missing "
                          "(run __graft_entry__.build() or python -m mlstm_chunkwise_attention_b200._build)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


# --------------------------------------------------------------------------
# C ABI, same names
# --------------------------------------------------------------------------

def mlstm_saved_layout(B, NH, T, d_qk, d_hv, chunk, variant, dtype):
    lay = SavedLayout()
    st = load().mlstm_saved_layout(B, NH, T, d_qk, d_hv, chunk, variant, dtype, ctypes.byref(lay))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_saved_layout")
    return {n: getattr(lay, n) for n, _ in SavedLayout._fields_}


def mlstm_saved_size(*sizes):
    return load().mlstm_saved_size(*sizes)


def mlstm_fwd_workspace_size(*sizes):
    return load().mlstm_fwd_workspace_size(*sizes)


def mlstm_bwd_workspace_size(*sizes):
    return load().mlstm_bwd_workspace_size(*sizes)


def mlstm_fwd_launch_count(*sizes):
    return load().mlstm_fwd_launch_count(*sizes)


def mlstm_bwd_launch_count(*sizes):
    return load().mlstm_bwd_launch_count(*sizes)


def mlstm_fwd(q, k, v, igate_pre, fgate_pre, h, saved, workspace, workspace_bytes,
              B, NH, T, d_qk, d_hv, chunk, variant, dtype, stream):
    return load().mlstm_fwd(q, k, v, igate_pre, fgate_pre, h, saved, workspace, workspace_bytes,
                            B, NH, T, d_qk, d_hv, chunk, variant, dtype, stream)


def mlstm_fwd_noalloc(q, k, v, igate_pre, fgate_pre, h, B, NH, T, d_qk, d_hv, chunk, variant,
                      dtype, stream):
    """Forward whose scratch is a fixed array inside the library (no allocation)."""
    return load().mlstm_fwd_noalloc(q, k, v, igate_pre, fgate_pre, h, B, NH, T, d_qk, d_hv, chunk,
                                    variant, dtype, stream)


def mlstm_bwd(q, k, v, igate_pre, fgate_pre, h, dh, saved, dq, dk, dv, digate_pre, dfgate_pre,
              workspace, workspace_bytes, B, NH, T, d_qk, d_hv, chunk, variant, dtype, stream):
    return load().mlstm_bwd(q, k, v, igate_pre, fgate_pre, h, dh, saved, dq, dk, dv, digate_pre,
                            dfgate_pre, workspace, workspace_bytes, B, NH, T, d_qk, d_hv, chunk,
                            variant, dtype, stream)


def mlstm_fwd_state(q, k, v, igate_pre, fgate_pre, h, saved, workspace, workspace_bytes,
                    state_in, state_out, B, NH, T, d_qk, d_hv, chunk, variant, dtype, stream):
    return load().mlstm_fwd_state(q, k, v, igate_pre, fgate_pre, h, saved, workspace,
                                  workspace_bytes, state_in, state_out, B, NH, T, d_qk, d_hv, chunk,
                                  variant, dtype, stream)


def mlstm_bwd_state(q, k, v, igate_pre, fgate_pre, h, dh, saved, state_in, dstate_in, dstate_out,
                    dq, dk, dv, digate_pre, dfgate_pre, workspace, workspace_bytes, B, NH, T, d_qk,
                    d_hv, chunk, variant, dtype, stream):
    return load().mlstm_bwd_state(q, k, v, igate_pre, fgate_pre, h, dh, saved, state_in, dstate_in,
                                  dstate_out, dq, dk, dv, digate_pre, dfgate_pre, workspace,
                                  workspace_bytes, B, NH, T, d_qk, d_hv, chunk, variant, dtype,
                                  stream)


def mlstm_status_string(status):
    return load().mlstm_status_string(status).decode()


def mlstm_device_status(stream=None):
    return load().mlstm_device_status(stream)


def mlstm_selftest_timeout(stream=None):
    return load().mlstm_selftest_timeout(stream)


def check_device(stream=None):
    """Raise if a kernel enqueued so far reported a timeout or a CUDA error."""
    st = mlstm_device_status(stream)
    if st != STATUS_OK:
        raise MLSTMError(st, "device status")


def mlstm_last_error():
    return load().mlstm_last_error().decode()


def mlstm_launch_name(pass_, index, *sizes):
    return load().mlstm_launch_name(pass_, index, *sizes).decode()


def mlstm_set_timing_events(events, count):
    """events: a ctypes array of void* (cudaEvent_t handles), or None."""
    return load().mlstm_set_timing_events(events, count)


def mlstm_set_serial_launches(serial):
    """True: every kernel of this thread's later calls on the caller's stream (for timing
    each kernel alone); False (the default): the backward may overlap two of them."""
    return load().mlstm_set_serial_launches(1 if serial else 0)


# --------------------------------------------------------------------------
# torch conveniences (allocation through PyTorch, compute in the library)
# --------------------------------------------------------------------------

def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _check(tensors, dtype):
    for name, t in tensors.items():
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype != dtype:
            raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def problem_sizes(q, v, chunk, variant):
    B, NH, T, d_qk = q.shape
    d_hv = v.shape[-1]
    return (B, NH, T, d_qk, d_hv, int(chunk), int(variant), _dtype_code(q))


def forward(q, k, v, igate_pre, fgate_pre, chunk, variant, *, keep_saved=True, h=None,
            saved=None, stream=None):
    """h = mLSTM(q, k, v, gates) on the current (or given) stream.

    Returns (h, saved); ``saved`` (a uint8 tensor) is what ``backward`` needs,
    or None when keep_saved is False (then a transient workspace is used).
    """
    import torch
    _check({"q": q, "k": k, "v": v, "igate_pre": igate_pre, "fgate_pre": fgate_pre}, q.dtype)
    sizes = problem_sizes(q, v, chunk, variant)
    if h is None:
        h = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ws = None
    if keep_saved:
        if saved is None:
            saved = torch.empty(max(mlstm_saved_size(*sizes), 1), dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = None, 0
    else:
        nbytes = mlstm_fwd_workspace_size(*sizes)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = ws.data_ptr(), nbytes
    st = mlstm_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), igate_pre.data_ptr(),
                   fgate_pre.data_ptr(), h.data_ptr(), saved.data_ptr() if keep_saved else None,
                   ws_ptr, ws_bytes, *sizes, _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_fwd")
    return h, (saved if keep_saved else None)


def backward(q, k, v, igate_pre, fgate_pre, h, dh, saved, chunk, variant, *, workspace=None,
             stream=None):
    """Gradients of sum(dh * h): dict of dq, dk, dv, digate_pre, dfgate_pre."""
    import torch
    _check({"q": q, "k": k, "v": v, "igate_pre": igate_pre, "fgate_pre": fgate_pre, "h": h,
            "dh": dh}, q.dtype)
    sizes = problem_sizes(q, v, chunk, variant)
    out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "digate_pre": torch.empty_like(igate_pre), "dfgate_pre": torch.empty_like(fgate_pre)}
    nbytes = mlstm_bwd_workspace_size(*sizes)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    st = mlstm_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), igate_pre.data_ptr(),
                   fgate_pre.data_ptr(), h.data_ptr(), dh.data_ptr(), saved.data_ptr(),
                   out["dq"].data_ptr(), out["dk"].data_ptr(), out["dv"].data_ptr(),
                   out["digate_pre"].data_ptr(), out["dfgate_pre"].data_ptr(),
                   workspace.data_ptr(), workspace.numel(), *sizes, _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_bwd")
    return out


# ---------------------------------------------------------------------------
# Recurrent form: state buffers, hand-off from a forward pass, one-token steps
# ---------------------------------------------------------------------------

def state_views(state, B, NH, d_qk, d_hv, variant):
    """C [B, NH, d_qk, d_hv] and, for EXP, n [B, NH, d_qk] and m [B, NH] views of a state
    buffer (layout in include/mlstm.h)."""
    import torch
    BH = B * NH
    c_bytes = BH * d_qk * d_hv * 4
    out = {"C": state[:c_bytes].view(torch.float32).view(B, NH, d_qk, d_hv), "n": None, "m": None}
    if variant == EXP:
        off = (c_bytes + 255) // 256 * 256
        out["n"] = state[off: off + BH * d_qk * 4].view(torch.float32).view(B, NH, d_qk)
        off = (off + BH * d_qk * 4 + 255) // 256 * 256
        out["m"] = state[off: off + BH * 4].view(torch.float32).view(B, NH)
    return out


def new_state(B, NH, d_qk, d_hv, variant, device, stream=None):
    """A zero state (C = 0, n = 0, m = -inf) in a fresh uint8 buffer."""
    import torch
    nbytes = load().mlstm_state_size(B, NH, d_qk, d_hv, variant)
    if nbytes == 0:
        raise MLSTMError(STATUS_UNSUPPORTED, "mlstm_state_size")
    state = torch.empty(nbytes, dtype=torch.uint8, device=device)
    st = load().mlstm_state_zero(state.data_ptr(), B, NH, d_qk, d_hv, variant, _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_state_zero")
    return state


def final_state(k, v, saved, chunk, variant, *, state=None, stream=None):
    """State after the last token of a forward that kept ``saved`` (same sizes)."""
    import torch
    B, NH, T, d_qk = k.shape
    d_hv = v.shape[-1]
    if state is None:
        state = torch.empty(load().mlstm_state_size(B, NH, d_qk, d_hv, variant), dtype=torch.uint8,
                            device=k.device)
    st = load().mlstm_final_state(k.data_ptr(), v.data_ptr(), saved.data_ptr(), state.data_ptr(),
                                  *problem_sizes(k, v, chunk, variant), _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_final_state")
    return state


def forward_state(q, k, v, igate_pre, fgate_pre, chunk, variant, state_in=None, *,
                  keep_saved=True, want_h=True, stream=None):
    """Chunkwise forward continuing from ``state_in`` (None: the zero state).

    Returns (h, saved, state_out): state_out is a fresh state buffer holding the state
    after the last token; saved (None when keep_saved is False) is for backward_state;
    h is None when want_h is False (the state-only pass).
    """
    import torch
    _check({"q": q, "k": k, "v": v, "igate_pre": igate_pre, "fgate_pre": fgate_pre}, q.dtype)
    sizes = problem_sizes(q, v, chunk, variant)
    B, NH, T, d_qk, d_hv = sizes[:5]
    h = torch.empty(v.shape, dtype=q.dtype, device=q.device) if want_h else None
    state_out = torch.empty(load().mlstm_state_size(B, NH, d_qk, d_hv, variant), dtype=torch.uint8,
                            device=q.device)
    saved = ws = None
    if keep_saved:
        saved = torch.empty(max(mlstm_saved_size(*sizes), 1), dtype=torch.uint8, device=q.device)
    else:
        ws = torch.empty(max(mlstm_fwd_workspace_size(*sizes), 1), dtype=torch.uint8,
                         device=q.device)
    st = mlstm_fwd_state(q.data_ptr(), k.data_ptr(), v.data_ptr(), igate_pre.data_ptr(),
                         fgate_pre.data_ptr(), h.data_ptr() if h is not None else None,
                         saved.data_ptr() if saved is not None else None,
                         ws.data_ptr() if ws is not None else None,
                         ws.numel() if ws is not None else 0,
                         state_in.data_ptr() if state_in is not None else None,
                         state_out.data_ptr(), *sizes, _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_fwd_state")
    return h, saved, state_out


def log_decay(fgate_pre, *, stream=None):
    """sum_t log sigmoid(fgate_pre) per head: float32 [B, NH]."""
    import torch
    B, NH, T = fgate_pre.shape
    out = torch.empty((B, NH), dtype=torch.float32, device=fgate_pre.device)
    st = load().mlstm_log_decay(fgate_pre.data_ptr(), out.data_ptr(), B, NH, T,
                                _dtype_code(fgate_pre), _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_log_decay")
    return out


def state_chain(state_a, state_b, log_decay_b, B, NH, d_qk, d_hv, variant, *, out=None,
                stream=None):
    """The state after segment b when it starts from state_a (see include/mlstm.h)."""
    import torch
    if out is None:
        out = torch.empty_like(state_a)
    st = load().mlstm_state_chain(state_a.data_ptr(), state_b.data_ptr(), log_decay_b.data_ptr(),
                                  out.data_ptr(), B, NH, d_qk, d_hv, variant,
                                  _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_state_chain")
    return out


def dstate_chain(dstate_local, dstate_out, state_in, state_out, log_decay_b, B, NH, d_qk, d_hv,
                 variant, *, out=None, stream=None):
    """Gradient with respect to segment b's initial state (see include/mlstm.h)."""
    import torch
    if out is None:
        out = torch.zeros_like(dstate_local)
    st = load().mlstm_dstate_chain(dstate_local.data_ptr(), dstate_out.data_ptr(),
                                   state_in.data_ptr(), state_out.data_ptr(), log_decay_b.data_ptr(),
                                   out.data_ptr(), B, NH, d_qk, d_hv, variant,
                                   _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_dstate_chain")
    return out


def state_gradient(q, k, v, igate_pre, fgate_pre, h, dh, saved, chunk, variant, state_in=None, *,
                   stream=None):
    """The state-gradient-only pass: gradient of sum(dh * h) with respect to state_in."""
    import torch
    sizes = problem_sizes(q, v, chunk, variant)
    B, NH, T, d_qk, d_hv = sizes[:5]
    dstate = torch.zeros(load().mlstm_state_size(B, NH, d_qk, d_hv, variant), dtype=torch.uint8,
                         device=q.device)
    ws = torch.empty(max(mlstm_bwd_workspace_size(*sizes), 1), dtype=torch.uint8, device=q.device)
    st = mlstm_bwd_state(q.data_ptr(), k.data_ptr(), v.data_ptr(), igate_pre.data_ptr(),
                         fgate_pre.data_ptr(), h.data_ptr(), dh.data_ptr(), saved.data_ptr(),
                         state_in.data_ptr() if state_in is not None else None, dstate.data_ptr(),
                         None, None, None, None, None, None, ws.data_ptr(), ws.numel(), *sizes,
                         _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_bwd_state")
    return dstate


def backward_state(q, k, v, igate_pre, fgate_pre, h, dh, saved, chunk, variant, state_in=None, *,
                   dstate_out=None, want_dstate=True, stream=None):
    """Gradients of sum(dh * h) (+ <dstate_out, final state> when dstate_out, a state-layout
    buffer, is given) for a forward_state call, the initial state held constant.

    Returns the dict of ``backward`` plus "dstate_in" (a state-layout buffer whose C and,
    for EXP, n regions hold the gradient with respect to state_in) when want_dstate.
    """
    import torch
    _check({"q": q, "k": k, "v": v, "igate_pre": igate_pre, "fgate_pre": fgate_pre, "h": h,
            "dh": dh}, q.dtype)
    sizes = problem_sizes(q, v, chunk, variant)
    B, NH, T, d_qk, d_hv = sizes[:5]
    out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "digate_pre": torch.empty_like(igate_pre), "dfgate_pre": torch.empty_like(fgate_pre)}
    if want_dstate:
        out["dstate_in"] = torch.zeros(load().mlstm_state_size(B, NH, d_qk, d_hv, variant),
                                       dtype=torch.uint8, device=q.device)
    ws = torch.empty(max(mlstm_bwd_workspace_size(*sizes), 1), dtype=torch.uint8, device=q.device)
    st = mlstm_bwd_state(q.data_ptr(), k.data_ptr(), v.data_ptr(), igate_pre.data_ptr(),
                         fgate_pre.data_ptr(), h.data_ptr(), dh.data_ptr(), saved.data_ptr(),
                         state_in.data_ptr() if state_in is not None else None,
                         out["dstate_in"].data_ptr() if want_dstate else None,
                         dstate_out.data_ptr() if dstate_out is not None else None,
                         out["dq"].data_ptr(), out["dk"].data_ptr(), out["dv"].data_ptr(),
                         out["digate_pre"].data_ptr(), out["dfgate_pre"].data_ptr(),
                         ws.data_ptr(), ws.numel(), *sizes, _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_bwd_state")
    return out


def step(q, k, v, igate_pre, fgate_pre, state_in, state_out, variant, *, h=None, stream=None):
    """One token: q, k [B, NH, d_qk], v [B, NH, d_hv], gates [B, NH]; returns h [B, NH, d_hv]."""
    import torch
    _check({"q": q, "k": k, "v": v, "igate_pre": igate_pre, "fgate_pre": fgate_pre}, q.dtype)
    B, NH, d_qk = q.shape
    d_hv = v.shape[-1]
    if h is None:
        h = torch.empty((B, NH, d_hv), dtype=q.dtype, device=q.device)
    st = load().mlstm_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), igate_pre.data_ptr(),
                           fgate_pre.data_ptr(), h.data_ptr(), state_in.data_ptr(), state_out.data_ptr(),
                           B, NH, d_qk, d_hv, int(variant), _dtype_code(q), _stream_handle(stream))
    if st != STATUS_OK:
        raise MLSTMError(st, "mlstm_step")
    return h


def saved_views(saved, q, v, chunk, variant):
    """Typed views of the saved regions (for tests and diagnostics)."""
    import torch
    B, NH, T, d_qk, d_hv, chunk, variant, dtype = problem_sizes(q, v, chunk, variant)
    lay = mlstm_saved_layout(B, NH, T, d_qk, d_hv, chunk, variant, dtype)
    NC = (T + chunk - 1) // chunk
    BH = B * NH

    def view(name, shape, dt):
        nbytes = lay[name + "_bytes"]
        if nbytes == 0:
            return None
        return saved[lay[name]: lay[name] + nbytes].view(dt).view(*shape)

    if dtype == BF16:  # two bf16 planes: hi then lo
        planes = view("state_c", (2, BH, NC, d_qk, d_hv), torch.bfloat16)
        C = planes[0].float() + planes[1].float()
    else:
        C = view("state_c", (BH, NC, d_qk, d_hv), torch.float32)
    return {
        "b": view("gate_b", (BH, T), torch.float32),
        "log_i": view("gate_li", (BH, T), torch.float32),
        "m": view("gate_m", (BH, T), torch.float32),
        "abar": view("norm", (BH, T), torch.float32),
        "C": C,
        "n": view("state_n", (BH, NC, d_qk), torch.float32),
    }
