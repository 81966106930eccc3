"""Python binding of liblinattn.so — B200 (sm_100a) kernelized linear attention
with the elu(x)+1 feature map.

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  PyTorch provides device memory (outputs, state and
workspace buffers) and the current CUDA stream.  The binding's functions carry
the C ABI's names (``include/linattn.h``):

    la_prefill_causal(q, k, v, decay=None, eps=1e-6, chunk=64, ...)
    la_forward_noncausal(q, k, v, eps=1e-6, ...)
    la_decode_step(q, k, v, state_S, state_z, decay=None, eps=1e-6, ...)

If the shared library has not been built, importing works but every call
raises: there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "LinAttnError", "lib", "la_prefill_causal", "la_forward_noncausal", "la_decode_step",
    "la_prefill_causal_mlstm", "la_decode_step_mlstm", "la_prefill_causal_flash",
    "la_prefill_causal_summary", "la_state_combine",
    "la_prefill_workspace_size", "la_noncausal_workspace_size", "la_status_string",
    "la_prefill_path", "la_launch_count", "la_workspace_status", "la_set_wait_limit_ns", "LA_F32", "LA_BF16", "LA_F16", "LA_STATE_NONE", "LA_STATE_OUT",
    "LA_STATE_INOUT", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblinattn.so")

LA_F32, LA_BF16, LA_F16 = 0, 1, 2
LA_STATE_NONE, LA_STATE_OUT, LA_STATE_INOUT = 0, 1, 2
LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT = 0, 1, 2, 3, 4

_DT = {torch.float32: LA_F32, torch.bfloat16: LA_BF16, torch.float16: LA_F16}

_lib = None
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class LinAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = f"{fn} returned {status}: {la_status_string(status)}"
        if status == LA_ERR_CUDA:
            msg += f" ({lib().la_last_error_string().decode()})"
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m kernelized_causal_sequence_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        L.la_prefill_causal.restype = _i
        L.la_prefill_causal.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _f, _i, _vp,
                                        _vp, _i, _vp, _i, _vp, _sz, _vp]
        L.la_prefill_causal_ev.restype = _i
        L.la_prefill_causal_ev.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _f, _i, _vp,
                                           _vp, _i, _vp, _i, _vp, _sz, _vp, _vp]
        L.la_prefill_causal_gated.restype = _i
        L.la_prefill_causal_gated.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _f, _i,
                                              _vp, _vp, _i, _vp, _i, _vp, _sz, _vp]
        L.la_prefill_causal_mlstm.restype = _i
        L.la_prefill_causal_mlstm.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                              _vp, _vp, _i, _vp, _i, _vp, _sz, _vp]
        L.la_prefill_causal_flash.restype = _i
        L.la_prefill_causal_flash.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _i,
                                              _vp, _i, _vp, _sz, _vp]
        L.la_prefill_causal_summary.restype = _i
        L.la_prefill_causal_summary.argtypes = [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                                _vp, _sz, _vp]
        L.la_state_combine.restype = _i
        L.la_state_combine.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]
        L.la_prefill_workspace_size.restype = _sz
        L.la_prefill_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i]
        L.la_forward_noncausal.restype = _i
        L.la_forward_noncausal.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _f, _vp,
                                           _vp, _i, _vp, _i, _vp, _sz, _vp]
        L.la_noncausal_workspace_size.restype = _sz
        L.la_noncausal_workspace_size.argtypes = [_i, _i, _i, _i, _i]
        L.la_decode_step.restype = _i
        L.la_decode_step.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp,
                                     _i, _vp]
        L.la_decode_step_gated.restype = _i
        L.la_decode_step_gated.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp,
                                           _vp, _i, _vp]
        L.la_decode_step_mlstm.restype = _i
        L.la_decode_step_mlstm.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _vp, _vp,
                                           _vp, _i, _vp]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_status_string.argtypes = [_i]
        L.la_prefill_plan.restype = _i
        L.la_prefill_plan.argtypes = [_i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)]
        L.la_prefill_path.restype = _i
        L.la_prefill_path.argtypes = [_i, _i, _i, _i, _i]
        L.la_launch_count.restype = ctypes.c_uint64
        L.la_launch_count.argtypes = []
        L.la_last_error_string.restype = ctypes.c_char_p
        L.la_last_error_string.argtypes = []
        L.la_workspace_status.restype = _i
        L.la_workspace_status.argtypes = [_vp, ctypes.POINTER(_i), _vp]
        L.la_noalloc_status.restype = _i
        L.la_noalloc_status.argtypes = [ctypes.POINTER(_i), _vp]
        L.la_set_wait_limit_ns.restype = ctypes.c_uint64
        L.la_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        _lib = L
    return _lib


def la_launch_count() -> int:
    return int(lib().la_launch_count())


def la_workspace_status(workspace, stream=None):
    """(status, waiter) of the last call that used ``workspace``: status is
    LA_OK or LA_ERR_TIMEOUT (a bounded device-side wait of that call gave up),
    waiter the id of the first wait that gave up.  Synchronises the stream."""
    w = ctypes.c_int(0)
    st = lib().la_workspace_status(_ptr(workspace), ctypes.byref(w), _stream(stream))
    if st not in (LA_OK, LA_ERR_TIMEOUT):
        raise LinAttnError("la_workspace_status", st)
    return st, w.value


def la_set_wait_limit_ns(ns: int) -> int:
    """Limit of every bounded device-side wait of later calls (process-wide);
    returns the previous limit."""
    return int(lib().la_set_wait_limit_ns(int(ns)))


def la_status_string(status: int) -> str:
    return lib().la_status_string(int(status)).decode()


def la_prefill_workspace_size(B, H, T, d_k, d_v, chunk) -> int:
    return int(lib().la_prefill_workspace_size(B, H, T, d_k, d_v, chunk))


def la_prefill_plan(B, H, T, d_k, chunk):
    """(segments per head, tokens per segment) of la_prefill_causal's plan."""
    n, sl = ctypes.c_int(0), ctypes.c_int(0)
    _check("la_prefill_plan", lib().la_prefill_plan(B, H, T, d_k, chunk, ctypes.byref(n), ctypes.byref(sl)))
    return n.value, sl.value


def la_noncausal_workspace_size(B, H, Lk, d_k, d_v) -> int:
    return int(lib().la_noncausal_workspace_size(B, H, Lk, d_k, d_v))


def la_prefill_path(in_dtype, d_k, d_v, chunk, has_decay=False) -> int:
    if isinstance(in_dtype, torch.dtype):
        in_dtype = _DT[in_dtype]
    return int(lib().la_prefill_path(in_dtype, d_k, d_v, chunk, int(bool(has_decay))))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, st):
    if st != LA_OK:
        raise LinAttnError(fn, st)


def _workspace(nbytes, device):
    # 256-byte aligned by the caching allocator
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def la_prefill_causal(q, k, v, decay=None, eps=1e-6, chunk=64, state_S=None, state_z=None,
                      mode=None, out=None, out_dtype=None, workspace=None, stream=None,
                      events=None, gain=None):
    """Causal chunked prefill.  q, k: [B,H,T,d_k]; v: [B,H,T,d_v] (f32/bf16/f16, CUDA,
    contiguous); decay: [B,H,T] fp32 or None.  state_S [B,H,d_k,d_v] / state_z [B,H,d_k]
    fp32 with ``mode`` LA_STATE_NONE/OUT/INOUT (default: OUT if given, else NONE).
    ``gain``: [B,H,T] fp32 (>= 0) or None — the gated form, token t's new term
    scaled by gain[t] (la_prefill_causal_gated; the RFA gate is decay=g, gain=1-g).
    ``events``: None, or 4 recorded-once ``torch.cuda.Event(enable_timing=True)``
    objects that la_prefill_causal_ev records around the state pass, the scan and
    the output pass (not with ``gain``).  Returns ``out`` [B,H,T,d_v]."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    if mode is None:
        mode = LA_STATE_OUT if state_S is not None else LA_STATE_NONE
    if workspace is None:
        workspace = _workspace(la_prefill_workspace_size(B, H, T, dk, dv, chunk), q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(decay), B, H, T, dk, dv, float(eps),
            int(chunk), _ptr(state_S), _ptr(state_z), int(mode), _ptr(out), _DT[out.dtype],
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if gain is not None:
        if events is not None:
            raise ValueError("events are not recorded by the gated prefill")
        st = lib().la_prefill_causal_gated(*args[:5], _ptr(gain), *args[5:])
        _check("la_prefill_causal_gated", st)
    elif events is None:
        st = lib().la_prefill_causal(*args)
        _check("la_prefill_causal", st)
    else:
        if len(events) != 4:
            raise ValueError("events: 4 CUDA events")
        for e in events:   # torch creates the CUDA event at its first record
            if int(e.cuda_event) == 0:
                e.record()
        arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(int(e.cuda_event)) for e in events])
        st = lib().la_prefill_causal_ev(*args, arr)
        _check("la_prefill_causal_ev", st)
    return out


def la_prefill_causal_mlstm(q, k, v, forget=None, input_gate=None, chunk=64, state_S=None, state_z=None,
                            mode=None, out=None, out_dtype=None, workspace=None, stream=None):
    """Causal prefill with the mLSTM read-out: identity feature map, forget gate
    f and input gate i (``[B,H,T]`` fp32 or None), out = q^T S / max(|q^T z|, 1)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    if mode is None:
        mode = LA_STATE_OUT if state_S is not None else LA_STATE_NONE
    if workspace is None:
        workspace = _workspace(la_prefill_workspace_size(B, H, T, dk, dv, chunk), q.device)
    st = lib().la_prefill_causal_mlstm(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(forget), _ptr(input_gate),
                                       B, H, T, dk, dv, int(chunk), _ptr(state_S), _ptr(state_z), int(mode),
                                       _ptr(out), _DT[out.dtype], _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream))
    _check("la_prefill_causal_mlstm", st)
    return out


def la_prefill_causal_flash(q, k, v, chunk=64, scaled=False, state_S=None, state_z=None, mode=None, out=None,
                            out_dtype=None, workspace=None, stream=None):
    """The FLASH chunk form: exact relu(q.k / s)^2 attention inside each chunk
    plus q^T (sum of the earlier chunks' k v^T) / s; s = chunk if ``scaled``
    (the listings' convention) else 1.  The state is the raw sum of k v^T
    (and of k) over all tokens.  Returns ``out`` [B,H,T,d_v]."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=out_dtype, device=q.device)
    if mode is None:
        mode = LA_STATE_OUT if state_S is not None else LA_STATE_NONE
    if workspace is None:
        workspace = _workspace(la_prefill_workspace_size(B, H, T, dk, dv, chunk), q.device)
    st = lib().la_prefill_causal_flash(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], B, H, T, dk, dv, int(chunk),
                                       int(bool(scaled)), _ptr(state_S), _ptr(state_z), int(mode), _ptr(out),
                                       _DT[out.dtype], _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream))
    _check("la_prefill_causal_flash", st)
    return out


def la_prefill_causal_summary(k, v, decay=None, gain=None, chunk=64, sum_S=None, sum_z=None, sum_A=None,
                              workspace=None, stream=None):
    """A shard's summary: (dS [B,H,dk,dv], dz [B,H,dk], A [B,H]) fp32, the
    shard's contribution to the state from a zero entry state and its decay
    product (la_prefill_causal_summary)."""
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    dev = k.device
    sum_S = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if sum_S is None else sum_S
    sum_z = torch.empty((B, H, dk), dtype=torch.float32, device=dev) if sum_z is None else sum_z
    sum_A = torch.empty((B, H), dtype=torch.float32, device=dev) if sum_A is None else sum_A
    if workspace is None:
        workspace = _workspace(max(256, la_prefill_workspace_size(B, H, max(T, 1), dk, dv, chunk)), dev)
    st = lib().la_prefill_causal_summary(_ptr(k), _ptr(v), _DT[k.dtype], _ptr(decay), _ptr(gain), B, H, T, dk, dv,
                                         int(chunk), _ptr(sum_S), _ptr(sum_z), _ptr(sum_A), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream))
    _check("la_prefill_causal_summary", st)
    return sum_S, sum_z, sum_A


def la_state_combine(S_all, z_all, A_all, r, S_in=None, z_in=None, S_out=None, z_out=None, stream=None):
    """Entry state of shard r from the gathered summaries [R, B, H, ...]
    (la_state_combine).  Returns (S_out, z_out)."""
    R, B, H, dk, dv = S_all.shape
    dev = S_all.device
    S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if S_out is None else S_out
    z_out = torch.empty((B, H, dk), dtype=torch.float32, device=dev) if z_out is None else z_out
    st = lib().la_state_combine(_ptr(S_all), _ptr(z_all), _ptr(A_all), R, int(r), B, H, dk, dv, _ptr(S_in),
                                _ptr(z_in), _ptr(S_out), _ptr(z_out), _stream(stream))
    _check("la_state_combine", st)
    return S_out, z_out


def la_decode_step_mlstm(q, k, v, state_S, state_z, forget=None, input_gate=None, out=None,
                         out_dtype=None, stream=None):
    """One mLSTM decode step (``forget``, ``input_gate``: [B,H] fp32 or None);
    the state is updated in place."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype, device=q.device)
    st = lib().la_decode_step_mlstm(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(forget), _ptr(input_gate),
                                    B, H, dk, dv, _ptr(state_S), _ptr(state_z), _ptr(out), _DT[out.dtype],
                                    _stream(stream))
    _check("la_decode_step_mlstm", st)
    return out


def la_forward_noncausal(q, k, v, eps=1e-6, state_S=None, state_z=None, mode=None, out=None,
                         out_dtype=None, workspace=None, stream=None, decay=None):
    """Non-causal form.  q: [B,H,Lq,d_k]; k: [B,H,Lk,d_k]; v: [B,H,Lk,d_v]."""
    B, H, Lq, dk = q.shape
    Lk, dv = v.shape[2], v.shape[3]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, Lq, dv), dtype=out_dtype, device=q.device)
    if mode is None:
        mode = LA_STATE_OUT if state_S is not None else LA_STATE_NONE
    if workspace is None:
        workspace = _workspace(la_noncausal_workspace_size(B, H, Lk, dk, dv), q.device)
    st = lib().la_forward_noncausal(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(decay), B, H,
                                    Lq, Lk, dk, dv, float(eps), _ptr(state_S), _ptr(state_z),
                                    int(mode), _ptr(out), _DT[out.dtype], _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check("la_forward_noncausal", st)
    return out


def la_decode_step(q, k, v, state_S, state_z, decay=None, eps=1e-6, out=None, out_dtype=None,
                   stream=None, gain=None):
    """One decode step; q, k: [B,H,d_k]; v: [B,H,d_v]; state updated in place.
    ``decay``, ``gain``: [B,H] fp32 or None (gated step: S <- a S + b phi(k) v^T)."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype, device=q.device)
    st = lib().la_decode_step_gated(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(decay), _ptr(gain), B, H,
                                    dk, dv, float(eps), _ptr(state_S), _ptr(state_z), _ptr(out),
                                    _DT[out.dtype], _stream(stream))
    _check("la_decode_step_gated" if gain is not None else "la_decode_step", st)
    return out
