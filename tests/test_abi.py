"""Host-side checks of the C ABI: the library loads, exports every entry point
include/linattn.h declares, and rejects bad arguments on the host before
anything is launched (these calls never reach the GPU, so they run anywhere).
"""
import ctypes
import os
import re

import pytest

import kernelized_causal_sequence_b200 as la

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "linattn.h")

P = ctypes.c_void_p(0x10000)      # 16-byte aligned dummy address, never dereferenced
P_ODD = ctypes.c_void_p(0x10004)  # misaligned dummy address


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(la_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    from kernelized_causal_sequence_b200 import build
    build.build()
    return la.lib()


@pytest.fixture(autouse=True)
def no_kernel_launched(L):
    """Every call in this file must be settled on the host: the dummy device
    addresses above are never dereferenced because no kernel is launched."""
    before = L.la_launch_count()
    yield
    assert L.la_launch_count() == before, "a host-side check let a kernel launch"


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"la_prefill_causal", "la_forward_noncausal", "la_decode_step",
            "la_prefill_workspace_size", "la_noncausal_workspace_size",
            "la_status_string", "la_prefill_path"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in linattn.h but not exported"


def test_status_strings(L):
    for s in range(5):
        assert la.la_status_string(s).startswith("LA_")
    assert "unknown" in la.la_status_string(99)


def test_workspace_sizes(L):
    assert la.la_prefill_workspace_size(1, 16, 131072, 128, 128, 128) > 0
    assert la.la_prefill_workspace_size(1, 16, 131072, 128, 64, 128) == 0
    assert la.la_prefill_workspace_size(1, 1, 256, 64, 64, 32) == 0
    assert la.la_prefill_workspace_size(0, 1, 256, 64, 64, 64) == 0
    assert la.la_noncausal_workspace_size(8, 8, 4800, 32, 32) > 0
    small = la.la_prefill_workspace_size(1, 1, 64, 64, 64, 64)
    assert small % 256 == 0 and small >= 4 * (64 * 64 + 64)


def test_prefill_path_selection(L):
    assert la.la_prefill_path(la.LA_F32, 64, 64, 64) == 0
    assert la.la_prefill_path(la.LA_BF16, 64, 64, 96) == -1
    assert la.la_prefill_path(la.LA_BF16, 48, 48, 64) == -1
    # 16-bit inputs with d in {64, 128} run on tensor cores, either chunk, with or without decay
    assert la.la_prefill_path(la.LA_BF16, 128, 128, 128) == 1
    assert la.la_prefill_path(la.LA_F16, 64, 64, 64, has_decay=True) == 1
    assert la.la_prefill_path(la.LA_BF16, 128, 128, 128, has_decay=True) == 1
    assert la.la_prefill_path(la.LA_BF16, 32, 32, 64) == 0


def _prefill(L, q=P, k=P, v=P, dt=la.LA_BF16, decay=None, B=1, H=2, T=128, dk=64, dv=64,
             eps=1e-6, chunk=64, S=P, z=P, mode=la.LA_STATE_OUT, out=P, odt=la.LA_BF16,
             ws=P, ws_bytes=1 << 30):
    return L.la_prefill_causal(q, k, v, dt, decay, B, H, T, dk, dv, eps, chunk, S, z, mode, out,
                               odt, ws, ws_bytes, None)


def test_prefill_rejects_bad_arguments(L):
    E_ARG, E_UNS = la.LA_ERR_INVALID_ARG, la.LA_ERR_UNSUPPORTED
    assert _prefill(L, dk=48, dv=48) == E_UNS
    assert _prefill(L, dk=64, dv=128) == E_UNS
    assert _prefill(L, chunk=32) == E_UNS
    assert _prefill(L, eps=-1.0) == E_ARG
    assert _prefill(L, eps=float("nan")) == E_ARG
    assert _prefill(L, eps=float("inf")) == E_ARG
    assert _prefill(L, dt=la.LA_F16, odt=la.LA_BF16) == E_UNS
    assert _prefill(L, dt=7) == E_ARG
    assert _prefill(L, T=-1) == E_ARG
    assert _prefill(L, q=None) == E_ARG
    assert _prefill(L, out=None) == E_ARG
    assert _prefill(L, k=P_ODD) == E_ARG
    assert _prefill(L, S=None) == E_ARG
    assert _prefill(L, mode=9) == E_ARG
    assert _prefill(L, ws_bytes=16) == E_ARG
    assert _prefill(L, ws=None) == E_ARG
    assert _prefill(L, ws=ctypes.c_void_p(0x10010)) == E_ARG  # workspace not 256-B aligned
    # empty batch: nothing to do, nothing launched
    assert _prefill(L, B=0) == la.LA_OK


def test_noncausal_and_decode_reject_bad_arguments(L):
    E_ARG, E_UNS = la.LA_ERR_INVALID_ARG, la.LA_ERR_UNSUPPORTED
    nc = lambda **kw: L.la_forward_noncausal(
        kw.get("q", P), P, P, la.LA_F16, kw.get("decay", None), 8, 8, kw.get("Lq", 100), 100,
        kw.get("d", 32), kw.get("d", 32), 1e-6, None, None, la.LA_STATE_NONE, kw.get("out", P),
        la.LA_F32, P, 1 << 30, None)
    assert nc(decay=P) == E_UNS
    assert nc(d=16) == E_UNS
    assert nc(q=None) == E_ARG
    assert nc(Lq=-5) == E_ARG
    dec = lambda **kw: L.la_decode_step(P, P, P, la.LA_BF16, None, 4, 4, kw.get("d", 128),
                                        kw.get("d", 128), 1e-6, kw.get("S", P), P, P, la.LA_BF16,
                                        None)
    assert dec(S=None) == E_ARG
    assert dec(S=P_ODD) == E_ARG
    assert dec(d=96) == E_UNS


def test_header_documents_each_entry_point():
    src = open(HEADER).read()
    for name in ("la_prefill_causal", "la_forward_noncausal", "la_decode_step"):
        i = src.index(name + "(")
        assert "/*" in src[max(0, i - 1500):i], f"{name} lacks a comment block"


def test_prefill_plan(L):
    # long-context workload: 16 heads x 1024 chunks of 128 -> 9 segments (144 CTAs)
    assert la.la_prefill_plan(1, 16, 131072, 128, 128) == (9, 14592)
    # SSD workload: 32 heads x 128 chunks of 64 -> 4 segments (128 CTAs)
    assert la.la_prefill_plan(2, 16, 8192, 128, 64) == (4, 2048)
    n, sl = la.la_prefill_plan(1, 1, 5000, 128, 64)
    assert n * sl >= 5000 and (n - 1) * sl < 5000 and sl % 64 == 0
    with pytest.raises(la.LinAttnError):
        la.la_prefill_plan(1, 1, 100, 64, 96)


@pytest.mark.parametrize("B,H,T,d,C", [(1, 1, 1 << 30, 128, 128), (1, 1, (1 << 31) - 1, 128, 64),
                                       (1024, 64, 1 << 20, 128, 128), (1, 65535, 1 << 16, 128, 64)])
def test_plan_and_workspace_at_extreme_sizes(L, B, H, T, d, C):
    """Sizes near the ABI's limits: the plan still covers every token with
    whole chunks, and the workspace size is computed in 64 bits."""
    n, sl = la.la_prefill_plan(B, H, T, d, C)
    assert n >= 1 and sl % C == 0 and n * sl >= T and (n - 1) * sl < T
    ws = la.la_prefill_workspace_size(B, H, T, d, d, C)
    assert ws >= 4 * B * H * n * (d * d + d)


def test_gated_and_mlstm_reject_bad_arguments(L):
    """The gated and mLSTM entry points share the prefill's and the decode
    step's host checks, and add the alignment of the gain / gate arrays."""
    E_ARG, E_UNS = la.LA_ERR_INVALID_ARG, la.LA_ERR_UNSUPPORTED

    def gated(gain=P, decay=None, B=1, T=128, dk=64, dv=64, chunk=64, eps=1e-6):
        return L.la_prefill_causal_gated(P, P, P, la.LA_BF16, decay, gain, B, 2, T, dk, dv, eps, chunk, P, P,
                                         la.LA_STATE_OUT, P, la.LA_BF16, P, 1 << 30, None)

    def mlstm(forget=None, igate=P, B=1, T=128, dk=64, dv=64, chunk=64):
        return L.la_prefill_causal_mlstm(P, P, P, la.LA_BF16, forget, igate, B, 2, T, dk, dv, chunk, P, P,
                                         la.LA_STATE_OUT, P, la.LA_BF16, P, 1 << 30, None)

    assert gated(gain=P_ODD) == E_ARG
    assert gated(decay=P_ODD) == E_ARG
    assert gated(B=-1) == E_ARG
    assert gated(chunk=96) == E_UNS
    assert gated(dk=64, dv=128) == E_UNS
    assert gated(eps=-1.0) == E_ARG
    assert gated(B=0) == la.LA_OK              # nothing to do, nothing launched
    assert mlstm(igate=P_ODD) == E_ARG
    assert mlstm(forget=P_ODD) == E_ARG
    assert mlstm(B=-1) == E_ARG
    assert mlstm(chunk=32) == E_UNS
    assert mlstm(dk=48, dv=48) == E_UNS
    assert mlstm(B=0) == la.LA_OK

    def dec_gated(gain=P, S=P, z=P, B=2):
        return L.la_decode_step_gated(P, P, P, la.LA_BF16, None, gain, B, 2, 64, 64, 1e-6, S, z, P, la.LA_BF16,
                                      None)

    def dec_mlstm(igate=P, S=P, z=P, B=2, d=64):
        return L.la_decode_step_mlstm(P, P, P, la.LA_BF16, None, igate, B, 2, d, d, S, z, P, la.LA_BF16, None)

    assert dec_gated(gain=P_ODD) == E_ARG
    assert dec_gated(S=None) == E_ARG
    assert dec_gated(B=0) == la.LA_OK
    assert dec_mlstm(igate=P_ODD) == E_ARG
    assert dec_mlstm(z=None) == E_ARG
    assert dec_mlstm(d=96) == E_UNS
    assert dec_mlstm(B=0) == la.LA_OK


def test_status_query_and_wait_limit(L):
    """la_workspace_status rejects a null or misaligned workspace on the host;
    la_set_wait_limit_ns returns the previous limit (default 2 s)."""
    w = ctypes.c_int(0)
    assert L.la_workspace_status(None, ctypes.byref(w), None) == la.LA_ERR_INVALID_ARG
    assert L.la_workspace_status(ctypes.c_void_p(0x10010), ctypes.byref(w), None) == la.LA_ERR_INVALID_ARG
    old = la.la_set_wait_limit_ns(12345)
    try:
        assert old == 2_000_000_000
        assert la.la_set_wait_limit_ns(0) == 12345
    finally:
        la.la_set_wait_limit_ns(old)
    assert la.la_set_wait_limit_ns(old) == old
