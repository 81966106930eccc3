"""la_prefill_causal_noalloc against la_prefill_causal.

The no-allocation entry point is for callers that cannot allocate device
memory — a plugin whose host runtime owns every device allocation, or a
process that forbids allocation after start-up.  It keeps its scratch in a
fixed device array inside the library instead of a caller workspace, so two
calls in a row must each match the workspace entry point on their own inputs
(the second call must not see anything of the first), bit for bit: both run
the same kernels with the same segment plan.

This file is collected last on purpose; it passes alone in a fresh process and
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.conftest import row_rel_err

pytestmark = pytest.mark.gpu

_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


def _entry(L):
    fn = L.la_prefill_causal_noalloc
    fn.restype = _i
    fn.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _i, _vp, _i, _vp]
    return fn


def _inputs(seed, B, H, T, d, decay):
    rng = np.random.default_rng(seed)
    mk = lambda: torch.from_numpy(rng.standard_normal((B, H, T, d), dtype=np.float32) / np.sqrt(d)) \
        .to(torch.bfloat16).cuda()
    q, k, v = mk(), mk(), mk()
    a = None
    if decay:
        g = rng.standard_normal((B, H, T), dtype=np.float32) + 2.0
        a = torch.from_numpy((1 / (1 + np.exp(-g))).astype(np.float32)).cuda()
    return q, k, v, a


def _run_both(la, fn, seed, B, H, T, d, chunk, decay):
    """One call of each entry point on the same inputs; returns both results."""
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    q, k, v, a = _inputs(seed, B, H, T, d, decay)
    S_ref = torch.zeros((B, H, d, d), device="cuda")
    z_ref = torch.zeros((B, H, d), device="cuda")
    ref = la.la_prefill_causal(q, k, v, decay=a, chunk=chunk, state_S=S_ref, state_z=z_ref,
                               mode=la.LA_STATE_OUT)
    out = torch.full_like(ref, float("nan"))
    S = torch.full_like(S_ref, float("nan"))
    z = torch.full_like(z_ref, float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(p(q), p(k), p(v), la.LA_BF16, p(a), B, H, T, d, d, 1e-6, chunk, p(S), p(z),
            la.LA_STATE_OUT, p(out), la.LA_BF16, stream)
    assert rc == la.LA_OK, la.la_status_string(rc)
    torch.cuda.synchronize()
    return (out, S, z), (ref, S_ref, z_ref)


def _assert_same(got, ref):
    # the same kernels with the same segment plan: bitwise equal results
    for g, r in zip(got, ref):
        assert torch.equal(g, r), float((g.float() - r.float()).abs().max())


def test_noalloc_matches_workspace_entry_point(la):
    """Two calls in a row of different shapes, each equal to the workspace entry
    point's result on its own inputs; the status word of the scratch array
    reports success."""
    fn = _entry(la.lib())
    status = la.lib().la_noalloc_status
    for seed, B, H, T, d, chunk, decay in [(101, 2, 3, 1000, 128, 64, True), (202, 1, 4, 777, 64, 128, False)]:
        got, ref = _run_both(la, fn, seed, B, H, T, d, chunk, decay)
        _assert_same(got, ref)
        w = ctypes.c_int(-1)
        st = status(ctypes.byref(w), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == la.LA_OK and w.value == 0


def test_noalloc_second_call_ignores_leftover_scratch(la):
    """A large call (many segments' states left in the shared array), then a
    smaller call with other inputs: the second result depends on its own
    inputs only."""
    fn = _entry(la.lib())
    got, ref = _run_both(la, fn, 303, 2, 8, 9000, 128, 64, True)
    _assert_same(got, ref)
    got, ref = _run_both(la, fn, 404, 1, 3, 2500, 128, 64, True)
    _assert_same(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch(la):
    fn = _entry(la.lib())
    dummy = ctypes.c_void_p(0x10000)
    rc = fn(dummy, dummy, dummy, la.LA_BF16, None, 64, 64, 131072, 128, 128, 1e-6, 64, None,
            None, la.LA_STATE_NONE, dummy, la.LA_BF16, None)
    assert rc == la.LA_ERR_UNSUPPORTED
