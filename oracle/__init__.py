"""fp64 CPU oracle for elu(x)+1 kernelized linear attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``, never by the product path.  It
shares no code with the CUDA library; both sides receive the same arrays from
the seeded generator and nothing else.

The arithmetic lives in ``linattn_oracle.c`` (plain C, fp64, token by token).
This module only builds that file with gcc when needed and marshals numpy
arrays to it.  Inputs of any float dtype are converted to float64 exactly
(bf16/fp16/fp32 values are all representable in fp64).

Pinned by ``tests/test_oracle_pins.py`` against the masked quadratic form, the
decayed (1-semiseparable) quadratic form, the gated form's weighted quadratic
form and its constant-gate closed form, the mLSTM read-out's weighted
quadratic form with the max(|.|, 1) normaliser, associativity of the non-causal
bracketing, closed forms on constructed inputs and the linear-attention
lesson's printed N=8, d=4 example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "linattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblinattn_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle to a shared library next to its source (gcc, -O2,
    OpenMP, no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.orc_causal_form.restype = ctypes.c_int
        lib.orc_causal_form.argtypes = [ctypes.c_int, _D, _D, _D, _D, _D, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        _D, _D, _D, _D, _D]
        lib.orc_noncausal.restype = ctypes.c_int
        lib.orc_noncausal.argtypes = [_D, _D, _D, ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                      ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                      _D, _D, _D, _D, _D]
        lib.orc_decode_step_form.restype = ctypes.c_int
        lib.orc_decode_step_form.argtypes = [ctypes.c_int, _D, _D, _D, _D, _D, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, _D, _D]
        lib.orc_flash.restype = ctypes.c_int
        lib.orc_flash.argtypes = [_D, _D, _D, ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int, ctypes.c_int, _D, _D]
        lib.orc_max_threads.restype = ctypes.c_int
        lib.orc_set_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _f64(x):
    """Exact conversion of a numpy array or CPU torch tensor to C-contiguous fp64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (CPU): widen in torch, bf16 has no numpy dtype
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def max_threads() -> int:
    return int(_load().orc_max_threads())


def causal(q, k, v, decay=None, eps=1e-6, S_in=None, z_in=None, gain=None, mlstm=False):
    """Causal recurrence.  q, k: [B,H,T,dk]; v: [B,H,T,dv]; decay, gain: [B,H,T] or
    None (gain b_t scales the new term: S_t = a_t S_{t-1} + b_t phi(k_t) v_t^T).
    ``mlstm``: the identity feature map and the max(|q^T z|, 1) read-out (decay =
    forget gate, gain = input gate; eps unused).
    Returns (out [B,H,T,dv], S [B,H,dk,dv], z [B,H,dk]) in fp64."""
    q, k, v, decay, S_in, z_in, gain = map(_f64, (q, k, v, decay, S_in, z_in, gain))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, T, dk) and v.shape == (B, H, T, dv)
    if decay is not None:
        assert decay.shape == (B, H, T)
    if gain is not None:
        assert gain.shape == (B, H, T)
    if S_in is not None:
        assert S_in.shape == (B, H, dk, dv)
    if z_in is not None:
        assert z_in.shape == (B, H, dk)
    out = np.zeros((B, H, T, dv))
    S = np.zeros((B, H, dk, dv))
    z = np.zeros((B, H, dk))
    rc = _load().orc_causal_form(int(bool(mlstm)), _ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(gain), B, H,
                                 T, dk, dv, float(eps), _ptr(S_in), _ptr(z_in), _ptr(out), _ptr(S), _ptr(z))
    if rc != 0:
        raise RuntimeError("orc_causal failed")
    return out, S, z


def noncausal(q, k, v, eps=1e-6, S_in=None, z_in=None):
    """Non-causal form.  q: [B,H,Lq,dk]; k: [B,H,Lk,dk]; v: [B,H,Lk,dv].
    Returns (out [B,H,Lq,dv], S, z) in fp64; S, z are the totals."""
    q, k, v, S_in, z_in = map(_f64, (q, k, v, S_in, z_in))
    B, H, Lq, dk = q.shape
    Lk, dv = v.shape[2], v.shape[3]
    assert k.shape == (B, H, Lk, dk) and v.shape[:2] == (B, H)
    out = np.zeros((B, H, Lq, dv))
    S = np.zeros((B, H, dk, dv))
    z = np.zeros((B, H, dk))
    rc = _load().orc_noncausal(_ptr(q), _ptr(k), _ptr(v), B, H, Lq, Lk, dk, dv, float(eps),
                               _ptr(S_in), _ptr(z_in), _ptr(out), _ptr(S), _ptr(z))
    if rc != 0:
        raise RuntimeError("orc_noncausal failed")
    return out, S, z


def decode_step(q, k, v, S, z, decay=None, eps=1e-6, gain=None, mlstm=False):
    """One decode step.  q, k: [B,H,dk]; v: [B,H,dv]; S: [B,H,dk,dv]; z: [B,H,dk];
    decay, gain: [B,H] or None; ``mlstm`` as in causal().
    Returns (out [B,H,dv], S_new, z_new); inputs untouched."""
    q, k, v, decay, gain = map(_f64, (q, k, v, decay, gain))
    S = _f64(S).copy()
    z = _f64(z).copy()
    B, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, H, dv))
    rc = _load().orc_decode_step_form(int(bool(mlstm)), _ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(gain),
                                      B, H, dk, dv, float(eps), _ptr(S), _ptr(z), _ptr(out))
    if rc != 0:
        raise RuntimeError("orc_decode_step failed")
    return out, S, z


def flash(q, k, v, chunk, scaled=False):
    """FLASH chunk form (causal): exact squared-ReLU attention inside each chunk
    plus a linear term over the earlier chunks' summaries; no feature map, no
    normaliser.  ``scaled``: the listings' convention (scores and summaries
    divided by the chunk length) instead of the equations'.  q, k: [B,H,T,dk];
    v: [B,H,T,dv].  Returns (out [B,H,T,dv], S [B,H,dk,dv] = all summaries)."""
    q, k, v = map(_f64, (q, k, v))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, H, T, dv))
    S = np.zeros((B, H, dk, dv))
    rc = _load().orc_flash(_ptr(q), _ptr(k), _ptr(v), B, H, T, dk, dv, int(chunk), int(bool(scaled)),
                           _ptr(out), _ptr(S))
    if rc != 0:
        raise RuntimeError("orc_flash failed")
    return out, S

