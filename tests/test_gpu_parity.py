"""CUDA path vs the fp64 oracle, element by element, on the same seeded inputs.

Bar: max over output rows of ||o_gpu - o_ref||_inf / ||o_ref||_inf below
1e-4 for fp32 inputs and 2e-2 for bf16/fp16 inputs (fp32 state).  Full-size
workloads run on the GPU exactly as the bench launches them; where the
oracle would take too long, whole heads are sampled (heads are independent,
so a sampled head's reference is exact).
"""
import numpy as np
import pytest
import torch

from kernelized_causal_sequence_b200 import inputs
from tests.conftest import row_rel_err, tol_for

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS
DEV = "cuda"


def gpu_prefill(la, q, k, v, decay, chunk, out_dtype, S_in=None, z_in=None, eps=1e-6):
    B, H, T, d = q.shape
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    ad = None if decay is None else decay.to(DEV)
    S = torch.zeros((B, H, d, d), dtype=torch.float32, device=DEV)
    z = torch.zeros((B, H, d), dtype=torch.float32, device=DEV)
    mode = la.LA_STATE_OUT
    if S_in is not None:
        S.copy_(S_in)
        z.copy_(z_in)
        mode = la.LA_STATE_INOUT
    out = la.la_prefill_causal(qd, kd, vd, decay=ad, eps=eps, chunk=chunk, state_S=S, state_z=z,
                               mode=mode, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), S.cpu().numpy(), z.cpu().numpy()


def check_prefill(la, orc, q, k, v, decay, chunk, out_dtype, tol, S_in=None, z_in=None):
    o, S, z = gpu_prefill(la, q, k, v, decay, chunk, out_dtype, S_in, z_in)
    ro, rS, rz = orc.causal(q, k, v, decay, 1e-6, S_in, z_in)
    err = row_rel_err(o, ro)
    assert err < tol, f"output rel err {err}"
    assert row_rel_err(S.reshape(S.shape[0], S.shape[1], -1),
                       rS.reshape(rS.shape[0], rS.shape[1], -1)) < tol
    assert row_rel_err(z, rz) < tol
    return err


# --------------------------------------------------------------- small cases
SMALL = [
    # (dtype, d, T, chunk, decay, B, H)
    (torch.float32, 64, 1, 64, False, 1, 1),
    (torch.float32, 32, 65, 64, False, 2, 3),
    (torch.float32, 128, 200, 128, True, 1, 2),
    (torch.float32, 64, 1000, 64, True, 1, 2),
    (torch.bfloat16, 64, 63, 64, False, 2, 2),
    (torch.bfloat16, 64, 777, 64, True, 1, 3),
    (torch.bfloat16, 128, 129, 128, False, 1, 2),
    (torch.bfloat16, 128, 1500, 64, True, 2, 1),
    (torch.bfloat16, 128, 3000, 128, False, 1, 2),
    (torch.float16, 32, 300, 128, False, 2, 2),
    (torch.float16, 128, 513, 64, True, 1, 2),
    # chunk 64 without decay at d 128 (bf16 out) and d 64 (fp16 out): the
    # output epilogues' half-warp column split, ragged tails
    (torch.bfloat16, 128, 700, 64, False, 1, 2),
    (torch.float16, 64, 450, 64, False, 2, 1),
    # chunk 128 with decay on the tensor cores (in-place decay weights)
    (torch.bfloat16, 128, 1000, 128, True, 1, 2),
    (torch.bfloat16, 64, 777, 128, True, 2, 1),
    (torch.float16, 128, 2500, 128, True, 1, 1),
    # more than 64 segments per head (the scan's shuffle form)
    (torch.bfloat16, 128, 5000, 64, True, 1, 1),
    (torch.float32, 64, 10000, 64, False, 1, 1),
]


def _small_inputs(dtype, d, T, decay, B, H, seed):
    rng = np.random.default_rng(seed)
    s = 1.0 / np.sqrt(d)
    mk = lambda: torch.from_numpy((rng.standard_normal((B, H, T, d), dtype=np.float32) * s)).to(dtype)
    q, k, v = mk(), mk(), mk()
    a = None
    if decay:
        g = rng.standard_normal((B, H, T), dtype=np.float32) + 2.0
        a = torch.from_numpy((1.0 / (1.0 + np.exp(-g))).astype(np.float32))
    return q, k, v, a


@pytest.mark.parametrize("dtype,d,T,chunk,decay,B,H", SMALL)
def test_prefill_small(la, orc, dtype, d, T, chunk, decay, B, H):
    q, k, v, a = _small_inputs(dtype, d, T, decay, B, H, seed=T * 7 + d)
    check_prefill(la, orc, q, k, v, a, chunk, torch.float32, tol_for(dtype))
    if dtype != torch.float32:
        check_prefill(la, orc, q, k, v, a, chunk, dtype, tol_for(dtype))


def test_prefill_state_inout_and_split(la, orc):
    dtype, d, T1, T2 = torch.bfloat16, 64, 300, 457
    q, k, v, a = _small_inputs(dtype, d, T1 + T2, True, 2, 2, seed=5)
    o_full, S_full, z_full = gpu_prefill(la, q, k, v, a, 64, torch.float32)
    o1, S1, z1 = gpu_prefill(la, q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], a[:, :, :T1], 64,
                             torch.float32)
    o2, S2, z2 = gpu_prefill(la, q[:, :, T1:], k[:, :, T1:], v[:, :, T1:], a[:, :, T1:], 64,
                             torch.float32, S_in=torch.from_numpy(S1).to(DEV),
                             z_in=torch.from_numpy(z1).to(DEV))
    ro, rS, rz = orc.causal(q, k, v, a)
    assert row_rel_err(np.concatenate([o1, o2], 2), ro) < 2e-2
    assert row_rel_err(S2.reshape(2, 2, -1), rS.reshape(2, 2, -1)) < 2e-2
    assert row_rel_err(o_full, ro) < 2e-2


def test_decay_one_matches_no_decay(la):
    """Decay 1 is the plain causal form.  On the fp32 CUDA-core path every
    decay factor is exactly 1 (2^0), so the results are bitwise equal.  On the
    tensor-core path every decay weight is exactly 1 too and both kernel
    families carry the normaliser as the same hi + lo bf16 pair, so the
    results agree to fp32 rounding (the state is summed in a different order
    of MMA issue)."""
    q, k, v, _ = _small_inputs(torch.float32, 64, 700, False, 1, 2, seed=9)
    ones = torch.ones((1, 2, 700), dtype=torch.float32)
    o1, S1, _ = gpu_prefill(la, q, k, v, None, 64, torch.float32)
    o2, S2, _ = gpu_prefill(la, q, k, v, ones, 64, torch.float32)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)
    q, k, v, _ = _small_inputs(torch.bfloat16, 128, 1000, False, 1, 2, seed=9)
    ones = torch.ones((1, 2, 1000), dtype=torch.float32)
    o1, S1, _ = gpu_prefill(la, q, k, v, None, 64, torch.float32)
    o2, S2, _ = gpu_prefill(la, q, k, v, ones, 64, torch.float32)
    assert row_rel_err(o2, o1) < 1e-5
    assert row_rel_err(S2.reshape(1, 2, -1), S1.reshape(1, 2, -1)) < 1e-5


def test_prefill_deterministic(la):
    q, k, v, a = _small_inputs(torch.bfloat16, 128, 4096, True, 1, 4, seed=10)
    o1, S1, _ = gpu_prefill(la, q, k, v, a, 64, torch.bfloat16)
    o2, S2, _ = gpu_prefill(la, q, k, v, a, 64, torch.bfloat16)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


@pytest.mark.parametrize("decay", [False, True])
def test_chunk_64_vs_128_agree(la, decay):
    q, k, v, a = _small_inputs(torch.bfloat16, 128, 2000, decay, 1, 2, seed=11)
    o1, S1, _ = gpu_prefill(la, q, k, v, a, 64, torch.float32)
    o2, S2, _ = gpu_prefill(la, q, k, v, a, 128, torch.float32)
    assert row_rel_err(o1, o2) < 2e-2
    assert row_rel_err(S1.reshape(1, 2, -1), S2.reshape(1, 2, -1)) < 2e-2


def test_workload_ssd_decay_chunk128(la, orc):
    """The SSD-decay workload's inputs processed with 128-token chunks (the
    result equals the per-token recurrence up to rounding for any chunk)."""
    w = W["ssd_decay_bf16_b2h16_t8192_d128"]
    q, k, v, a = inputs.qkv(w)
    o = la.la_prefill_causal(q.to(DEV), k.to(DEV), v.to(DEV), decay=a.to(DEV), chunk=128)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy()
    for b, h in ((0, 0), (1, 15)):
        ro, _, _ = orc.causal(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                              a[b:b + 1, h:h + 1])
        assert row_rel_err(o[b:b + 1, h:h + 1], ro) < 2e-2


def test_empty_and_state_only(la):
    q = torch.empty((2, 2, 0, 64), dtype=torch.bfloat16, device=DEV)
    S = torch.full((2, 2, 64, 64), 3.0, device=DEV)
    z = torch.full((2, 2, 64), 3.0, device=DEV)
    la.la_prefill_causal(q, q, q, state_S=S, state_z=z, mode=la.LA_STATE_OUT)
    torch.cuda.synchronize()
    assert float(S.abs().max()) == 0.0 and float(z.abs().max()) == 0.0
    S.fill_(2.0)
    la.la_prefill_causal(q, q, q, state_S=S, state_z=z, mode=la.LA_STATE_INOUT)
    torch.cuda.synchronize()
    assert float(S.min()) == 2.0


@pytest.mark.parametrize("dtype,d,T,chunk,decay", [(torch.bfloat16, 128, 3000, 128, True),
                                                   (torch.bfloat16, 64, 2000, 64, False),
                                                   (torch.float32, 64, 1000, 64, True)])
def test_state_mode_none_matches_out(la, dtype, d, T, chunk, decay):
    """Without a state output the output is bitwise the same, and no state
    buffer is written (the last segment of the output pass writes the final
    state only when one is asked for)."""
    B, H = 1, 2
    assert la.la_prefill_plan(B, H, T, d, chunk)[0] > 1   # several segments per head
    q, k, v, a = _small_inputs(dtype, d, T, decay, B, H, seed=41)
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    ad = None if a is None else a.to(DEV)
    S = torch.full((B, H, d, d), 7.0, device=DEV)
    z = torch.full((B, H, d), 7.0, device=DEV)
    o_none = la.la_prefill_causal(qd, kd, vd, decay=ad, chunk=chunk, state_S=S, state_z=z,
                                  mode=la.LA_STATE_NONE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert float(S.min()) == 7.0 and float(S.max()) == 7.0
    assert float(z.min()) == 7.0 and float(z.max()) == 7.0
    o_out = la.la_prefill_causal(qd, kd, vd, decay=ad, chunk=chunk, state_S=S, state_z=z,
                                 mode=la.LA_STATE_OUT, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o_none, o_out)
    assert float(z.min()) > 0.0   # phi > 0: the written normaliser is positive


# -------------------------------------------------------- full-size workloads
def test_workload_causal_f32(la, orc):
    w = W["causal_f32_t256_d64"]
    q, k, v, a = inputs.qkv(w)
    err = check_prefill(la, orc, q, k, v, a, w.chunk, w.torch_out_dtype, 1e-4)
    assert err < 1e-4


def test_workload_causal_bf16(la, orc):
    w = W["causal_bf16_b4h8_t2048_d64"]
    q, k, v, a = inputs.qkv(w)
    check_prefill(la, orc, q, k, v, a, w.chunk, w.torch_out_dtype, 2e-2)


def _sampled_heads(la, orc, w, heads):
    q, k, v, a = inputs.qkv(w)
    o, S, z = gpu_prefill(la, q, k, v, a, w.chunk, w.torch_out_dtype)
    for (b, h) in heads:
        sl = lambda x: None if x is None else x[b:b + 1, h:h + 1]
        ro, rS, rz = orc.causal(sl(q), sl(k), sl(v), sl(a))
        assert row_rel_err(o[b:b + 1, h:h + 1], ro) < 2e-2
        assert row_rel_err(S[b:b + 1, h:h + 1].reshape(1, 1, -1), rS.reshape(1, 1, -1)) < 2e-2
        assert row_rel_err(z[b:b + 1, h:h + 1], rz) < 2e-2


def test_workload_ssd_decay(la, orc):
    w = W["ssd_decay_bf16_b2h16_t8192_d128"]
    _sampled_heads(la, orc, w, [(0, 0), (1, 15), (0, 7)])


def test_workload_long_prefill(la, orc):
    w = W["prefill_bf16_h16_t131072_d128"]
    _sampled_heads(la, orc, w, [(0, 0), (0, 11)])


@pytest.mark.parametrize("cross", [False, True])
def test_workload_noncausal(la, orc, cross):
    w = W["noncausal_f16_b8h8_l4800_d32"]
    q, k, v, _ = inputs.qkv(w)
    if cross:
        k, v = inputs.cross_kv(w)
    S = torch.zeros((w.B, w.H, w.d, w.d), device=DEV)
    z = torch.zeros((w.B, w.H, w.d), device=DEV)
    o = la.la_forward_noncausal(q.to(DEV), k.to(DEV), v.to(DEV), state_S=S, state_z=z,
                                out_dtype=w.torch_out_dtype)
    torch.cuda.synchronize()
    ro, rS, rz = orc.noncausal(q, k, v)
    assert row_rel_err(o.cpu().numpy(), ro) < 2e-2
    assert row_rel_err(S.cpu().numpy().reshape(w.B, w.H, -1), rS.reshape(w.B, w.H, -1)) < 2e-2


@pytest.mark.parametrize("dtype,d,Lq,Lk", [(torch.float32, 64, 100, 333), (torch.bfloat16, 128, 17, 1000),
                                           (torch.float16, 32, 129, 0), (torch.bfloat16, 64, 0, 50),
                                           (torch.float32, 32, 300, 700), (torch.bfloat16, 32, 1000, 517),
                                           (torch.float16, 32, 513, 5000),
                                           # tensor-core path at d = 32: no queries (state only),
                                           # one key, one query, many heads per key segment
                                           (torch.bfloat16, 32, 0, 700), (torch.float16, 32, 1, 1),
                                           (torch.bfloat16, 32, 4800, 128), (torch.float16, 32, 257, 129)])
def test_noncausal_small(la, orc, dtype, d, Lq, Lk):
    rng = np.random.default_rng(Lq + Lk)
    mk = lambda L: torch.from_numpy(rng.standard_normal((2, 3, L, d), dtype=np.float32)).to(dtype)
    q, k, v = mk(Lq), mk(Lk), mk(Lk)
    S0 = torch.from_numpy(rng.standard_normal((2, 3, d, d), dtype=np.float32))
    z0 = torch.from_numpy(np.abs(rng.standard_normal((2, 3, d), dtype=np.float32)) + 1.0)
    S = S0.to(DEV).clone()
    z = z0.to(DEV).clone()
    o = la.la_forward_noncausal(q.to(DEV), k.to(DEV), v.to(DEV), state_S=S, state_z=z,
                                mode=la.LA_STATE_INOUT, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rS, rz = orc.noncausal(q, k, v, S_in=S0, z_in=z0)
    tol = tol_for(dtype)
    if Lq:
        assert row_rel_err(o.cpu().numpy(), ro) < tol
    assert row_rel_err(S.cpu().numpy().reshape(2, 3, -1), rS.reshape(2, 3, -1)) < tol


@pytest.mark.parametrize("dtype,d,decay", [(torch.float32, 64, False), (torch.bfloat16, 128, True),
                                           (torch.float16, 32, True), (torch.bfloat16, 64, False)])
def test_decode_small(la, orc, dtype, d, decay):
    rng = np.random.default_rng(d)
    B, H = 3, 5
    S0 = torch.from_numpy(rng.standard_normal((B, H, d, d), dtype=np.float32))
    z0 = torch.from_numpy(np.abs(rng.standard_normal((B, H, d), dtype=np.float32)) * 10 + 1)
    S, z = S0.to(DEV).clone(), z0.to(DEV).clone()
    rS, rz = S0.double().numpy(), z0.double().numpy()
    for step in range(5):
        mk = lambda: torch.from_numpy(rng.standard_normal((B, H, d), dtype=np.float32)).to(dtype)
        q, k, v = mk(), mk(), mk()
        a = torch.from_numpy(rng.uniform(0.5, 1.0, (B, H)).astype(np.float32)) if decay else None
        o = la.la_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), S, z,
                              decay=None if a is None else a.to(DEV), out_dtype=torch.float32)
        torch.cuda.synchronize()
        ro, rS, rz = orc.decode_step(q, k, v, rS, rz, decay=a)
        tol = tol_for(dtype)
        assert row_rel_err(o.cpu().numpy(), ro) < tol
        assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < tol


def test_workload_decode(la, orc):
    w = W["decode_bf16_b64h16_d128"]
    S0, z0 = inputs.decode_state(w)
    S, z = S0.to(DEV).clone(), z0.to(DEV).clone()
    rS, rz = S0.double().numpy(), z0.double().numpy()
    for step in range(6):
        q, k, v, _ = inputs.decode_inputs(w, step)
        o = la.la_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), S, z, out_dtype=w.torch_out_dtype)
        torch.cuda.synchronize()
        ro, rS, rz = orc.decode_step(q, k, v, rS, rz)
        assert row_rel_err(o.float().cpu().numpy(), ro) < 2e-2
    assert row_rel_err(S.cpu().numpy().reshape(w.B, w.H, -1), rS.reshape(w.B, w.H, -1)) < 2e-2


def test_prefill_then_decode_is_prefill_plus_one(la, orc):
    q, k, v, a = _small_inputs(torch.bfloat16, 128, 513, True, 2, 2, seed=12)
    T = 512
    _, S, z = gpu_prefill(la, q[:, :, :T], k[:, :, :T], v[:, :, :T], a[:, :, :T], 128,
                          torch.float32)
    Sd, zd = torch.from_numpy(S).to(DEV), torch.from_numpy(z).to(DEV)
    o = la.la_decode_step(q[:, :, T].to(DEV), k[:, :, T].to(DEV), v[:, :, T].to(DEV), Sd, zd,
                          decay=a[:, :, T].to(DEV), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, _, _ = orc.causal(q, k, v, a)
    assert row_rel_err(o.cpu().numpy(), ro[:, :, T]) < 2e-2


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_noncausal_d32_native_out(la, orc, dtype):
    """d = 32 read-out writing the input dtype (ragged query and key tiles)."""
    rng = np.random.default_rng(32)
    mk = lambda L: torch.from_numpy(rng.standard_normal((1, 4, L, 32), dtype=np.float32) * 0.5).to(dtype)
    q, k, v = mk(333), mk(1100), mk(1100)
    o = la.la_forward_noncausal(q.to(DEV), k.to(DEV), v.to(DEV), out_dtype=dtype)
    torch.cuda.synchronize()
    ro, _, _ = orc.noncausal(q, k, v)
    assert o.dtype == dtype
    assert row_rel_err(o.float().cpu().numpy(), ro) < 2e-2


@pytest.mark.parametrize("dtype,d,chunk,decay", [(torch.bfloat16, 128, 128, False), (torch.bfloat16, 128, 64, True),
                                                 (torch.float32, 64, 64, False)])
def test_prefill_events_entry_point(la, dtype, d, chunk, decay):
    """la_prefill_causal_ev: the same kernels as la_prefill_causal (bitwise equal
    results) plus four events recorded around the passes, in order."""
    q, k, v, a = _small_inputs(dtype, d, 3000, decay, 1, 2, seed=12)
    o1, S1, _ = gpu_prefill(la, q, k, v, a, chunk, torch.float32)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    S = torch.zeros((1, 2, d, d), device=DEV)
    z = torch.zeros((1, 2, d), device=DEV)
    o2 = la.la_prefill_causal(q.to(DEV), k.to(DEV), v.to(DEV), decay=None if a is None else a.to(DEV),
                              chunk=chunk, state_S=S, state_z=z, out_dtype=torch.float32, events=ev)
    torch.cuda.synchronize()
    assert np.array_equal(o1, o2.cpu().numpy()) and np.array_equal(S1, S.cpu().numpy())
    times = [ev[j].elapsed_time(ev[j + 1]) for j in range(3)]
    assert all(t >= 0 for t in times) and sum(times) > 0


# ------------------------------------------------------------- gated form
# Per-token gain b_t on the new term (S_t = a_t S_{t-1} + b_t phi(k_t) v_t^T);
# the RFA gate is a = g, b = 1 - g.
GATED = [
    # (dtype, d, T, chunk, kind, B, H)
    (torch.bfloat16, 128, 1000, 128, "rfa", 1, 2),
    (torch.bfloat16, 128, 1500, 64, "rfa", 2, 1),
    (torch.bfloat16, 64, 777, 64, "gain", 1, 3),
    (torch.bfloat16, 64, 777, 128, "decay_gain", 2, 1),
    (torch.float16, 128, 513, 64, "gain", 1, 2),
    (torch.float32, 64, 1000, 64, "rfa", 1, 2),
    (torch.float32, 32, 300, 128, "gain", 2, 2),
    (torch.bfloat16, 128, 5000, 64, "rfa", 1, 1),   # > 64 segments per head
]


def _gated_inputs(dtype, d, T, kind, B, H, seed):
    q, k, v, a = _small_inputs(dtype, d, T, kind != "gain", B, H, seed)
    rng = np.random.default_rng(seed + 1)
    if kind == "rfa":
        b = (1.0 - a.numpy()).astype(np.float32)
    else:
        b = rng.uniform(0.0, 2.0, (B, H, T)).astype(np.float32)
        b[..., T // 3] = 0.0     # keys that enter with weight zero
        b[..., T // 2] = 0.0
    return q, k, v, a, torch.from_numpy(b)


def gpu_prefill_gated(la, q, k, v, a, b, chunk, out_dtype):
    B, H, T, d = q.shape
    S = torch.zeros((B, H, d, d), dtype=torch.float32, device=DEV)
    z = torch.zeros((B, H, d), dtype=torch.float32, device=DEV)
    out = la.la_prefill_causal(q.to(DEV), k.to(DEV), v.to(DEV), decay=None if a is None else a.to(DEV),
                               chunk=chunk, state_S=S, state_z=z, out_dtype=out_dtype, gain=b.to(DEV))
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), S.cpu().numpy(), z.cpu().numpy()


@pytest.mark.parametrize("dtype,d,T,chunk,kind,B,H", GATED)
def test_gated_prefill_small(la, orc, dtype, d, T, chunk, kind, B, H):
    q, k, v, a, b = _gated_inputs(dtype, d, T, kind, B, H, seed=T * 5 + d)
    ro, rS, rz = orc.causal(q, k, v, a, 1e-6, gain=b)
    tol = tol_for(dtype)
    for out_dtype in ([torch.float32] if dtype == torch.float32 else [torch.float32, dtype]):
        o, S, z = gpu_prefill_gated(la, q, k, v, a, b, chunk, out_dtype)
        assert row_rel_err(o, ro) < tol, f"output rel err {row_rel_err(o, ro)}"
        assert row_rel_err(S.reshape(B, H, -1), rS.reshape(B, H, -1)) < tol
        assert row_rel_err(z, rz) < tol


def test_gain_one_matches_ungated(la):
    """b = 1 is the ungated form: the CUDA-core path multiplies by 1.0 (bitwise
    equal); on the tensor-core path the gain enters the key weights through
    log2(1) = 0 (equal up to the exponent approximation)."""
    q, k, v, a = _small_inputs(torch.float32, 64, 700, True, 1, 2, seed=12)
    ones = torch.ones((1, 2, 700), dtype=torch.float32)
    o1, S1, _ = gpu_prefill(la, q, k, v, a, 64, torch.float32)
    o2, S2, _ = gpu_prefill_gated(la, q, k, v, a, ones, 64, torch.float32)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)
    q, k, v, a = _small_inputs(torch.bfloat16, 128, 1000, True, 1, 2, seed=12)
    ones = torch.ones((1, 2, 1000), dtype=torch.float32)
    o1, S1, _ = gpu_prefill(la, q, k, v, a, 128, torch.float32)
    o2, S2, _ = gpu_prefill_gated(la, q, k, v, a, ones, 128, torch.float32)
    assert row_rel_err(o2, o1) < 1e-5
    assert row_rel_err(S2.reshape(1, 2, -1), S1.reshape(1, 2, -1)) < 1e-5


def test_workload_rfa_gated(la, orc):
    """The RFA-gated workload at full size, launched as the bench launches it;
    whole heads are compared with the oracle (heads are independent)."""
    w = W["rfa_gated_bf16_b2h16_t8192_d128"]
    q, k, v, a = inputs.qkv(w)
    b = inputs.gate_gain(w, a)
    S = torch.zeros((w.B, w.H, w.d, w.d), device=DEV)
    z = torch.zeros((w.B, w.H, w.d), device=DEV)
    o = la.la_prefill_causal(q.to(DEV), k.to(DEV), v.to(DEV), decay=a.to(DEV), chunk=w.chunk, state_S=S,
                             state_z=z, gain=b.to(DEV)).float().cpu().numpy()
    S = S.cpu().numpy()
    for bb, h in ((0, 0), (1, 15)):
        sl = (slice(bb, bb + 1), slice(h, h + 1))
        ro, rS, _ = orc.causal(q[sl], k[sl], v[sl], a[sl], w.eps, gain=b[sl])
        assert row_rel_err(o[sl], ro) < 2e-2
        assert row_rel_err(S[sl].reshape(1, 1, -1), rS.reshape(1, 1, -1)) < 2e-2


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.float16, 32)])
def test_gated_decode(la, orc, dtype, d):
    rng = np.random.default_rng(d)
    B, H = 3, 4
    q, k, v = (torch.from_numpy(rng.standard_normal((B, H, d), dtype=np.float32) / np.sqrt(d)).to(dtype)
               for _ in range(3))
    g = torch.from_numpy((1 / (1 + np.exp(-(rng.standard_normal((B, H)) + 2)))).astype(np.float32))
    b = 1.0 - g
    S0 = torch.from_numpy(rng.uniform(0, 1, (B, H, d, d)).astype(np.float32))
    z0 = torch.from_numpy(rng.uniform(1, 2, (B, H, d)).astype(np.float32))
    S, z = S0.to(DEV), z0.to(DEV)
    o = la.la_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), S, z, decay=g.to(DEV), gain=b.to(DEV),
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rS, rz = orc.decode_step(q, k, v, S0, z0, decay=g, gain=b)
    tol = tol_for(dtype)
    assert row_rel_err(o.cpu().numpy(), ro) < tol
    assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < 1e-5
    assert row_rel_err(z.cpu().numpy(), rz) < 1e-5


# ------------------------------------------------------------ mLSTM read-out
# Identity feature map, forget gate f (decay) and input gate i (gain), and the
# read-out q^T S / max(|q^T z|, 1).
MLSTM = [
    # (dtype, d, T, chunk, gates, B, H)
    (torch.bfloat16, 128, 1000, 128, True, 1, 2),
    (torch.bfloat16, 128, 1500, 64, True, 2, 1),
    (torch.bfloat16, 64, 777, 64, True, 1, 3),
    (torch.bfloat16, 64, 600, 128, False, 1, 2),   # no gates: f = i = 1
    (torch.float16, 128, 513, 64, True, 1, 2),
    (torch.float32, 64, 1000, 64, True, 1, 2),
    (torch.float32, 32, 300, 128, True, 2, 2),
]


def _mlstm_inputs(dtype, d, T, gates, B, H, seed):
    rng = np.random.default_rng(seed)
    mk = lambda s: torch.from_numpy((rng.standard_normal((B, H, T, d), dtype=np.float32) * s)).to(dtype)
    q, k, v = mk(1.0), mk(1.0 / np.sqrt(d)), mk(1.0 / np.sqrt(d))
    f = i = None
    if gates:
        f = torch.from_numpy((1 / (1 + np.exp(-(rng.standard_normal((B, H, T)) + 2)))).astype(np.float32))
        i = torch.from_numpy(np.exp(0.5 * rng.standard_normal((B, H, T)) - 0.5).astype(np.float32))
    return q, k, v, f, i


@pytest.mark.parametrize("dtype,d,T,chunk,gates,B,H", MLSTM)
def test_mlstm_prefill_small(la, orc, dtype, d, T, chunk, gates, B, H):
    q, k, v, f, i = _mlstm_inputs(dtype, d, T, gates, B, H, seed=T * 3 + d)
    ro, rS, rz = orc.causal(q, k, v, f, gain=i, mlstm=True)
    if gates:
        # rows on both sides of the max(|q^T z|, 1) clamp
        qn, kn = q.double().numpy(), k.double().numpy()
        zt = np.zeros((B, H, d))
        den = np.empty((B, H, T))
        for t in range(T):
            zt = f.numpy()[:, :, t, None] * zt + i.numpy()[:, :, t, None] * kn[:, :, t]
            den[:, :, t] = np.abs((qn[:, :, t] * zt).sum(-1))
        assert (den < 1).any() and (den > 1).any()
    tol = tol_for(dtype)
    dev = lambda x: None if x is None else x.to(DEV)
    for out_dtype in ([torch.float32] if dtype == torch.float32 else [torch.float32, dtype]):
        S = torch.zeros((B, H, d, d), device=DEV)
        z = torch.zeros((B, H, d), device=DEV)
        o = la.la_prefill_causal_mlstm(dev(q), dev(k), dev(v), forget=dev(f), input_gate=dev(i), chunk=chunk,
                                       state_S=S, state_z=z, out_dtype=out_dtype)
        torch.cuda.synchronize()
        o = o.float().cpu().numpy()
        assert row_rel_err(o, ro) < tol, f"output rel err {row_rel_err(o, ro)}"
        assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < tol
        assert row_rel_err(z.cpu().numpy(), rz) < tol


@pytest.mark.parametrize("form,d,chunk", [("rfa", 128, 64), ("gain", 64, 128), ("mlstm", 128, 128),
                                          ("mlstm", 64, 64)])
def test_gated_and_mlstm_state_split(la, orc, form, d, chunk):
    """The gated and mLSTM prefills in two calls, the state carried in place
    (INOUT) and the first piece ragged (not a whole number of chunks): equal to
    the oracle over the whole sequence, outputs and final state."""
    B, H, T1, T2 = 2, 2, 333, 470
    T = T1 + T2
    if form == "mlstm":
        q, k, v, a, b = _mlstm_inputs(torch.bfloat16, d, T, True, B, H, seed=61)
        ro, rS, rz = orc.causal(q, k, v, a, gain=b, mlstm=True)
    else:
        q, k, v, a, b = _gated_inputs(torch.bfloat16, d, T, form, B, H, seed=62)
        ro, rS, rz = orc.causal(q, k, v, a, 1e-6, gain=b)
    dev = lambda x, lo, hi: None if x is None else x[:, :, lo:hi].contiguous().to(DEV)
    S = torch.zeros((B, H, d, d), device=DEV)
    z = torch.zeros((B, H, d), device=DEV)
    outs = []
    for lo, hi in ((0, T1), (T1, T)):
        if form == "mlstm":
            o = la.la_prefill_causal_mlstm(dev(q, lo, hi), dev(k, lo, hi), dev(v, lo, hi), forget=dev(a, lo, hi),
                                           input_gate=dev(b, lo, hi), chunk=chunk, state_S=S, state_z=z,
                                           mode=la.LA_STATE_INOUT, out_dtype=torch.float32)
        else:
            o = la.la_prefill_causal(dev(q, lo, hi), dev(k, lo, hi), dev(v, lo, hi), decay=dev(a, lo, hi),
                                     gain=dev(b, lo, hi), chunk=chunk, state_S=S, state_z=z,
                                     mode=la.LA_STATE_INOUT, out_dtype=torch.float32)
        outs.append(o)
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=2).cpu().numpy()
    assert row_rel_err(o, ro) < 2e-2, f"output rel err {row_rel_err(o, ro)}"
    assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < 2e-2
    assert row_rel_err(z.cpu().numpy(), rz) < 2e-2


def test_workload_mlstm(la, orc):
    w = W["mlstm_bf16_b2h16_t8192_d128"]
    q, k, v, f = inputs.qkv(w)
    i = inputs.input_gate(w)
    S = torch.zeros((w.B, w.H, w.d, w.d), device=DEV)
    z = torch.zeros((w.B, w.H, w.d), device=DEV)
    o = la.la_prefill_causal_mlstm(q.to(DEV), k.to(DEV), v.to(DEV), forget=f.to(DEV), input_gate=i.to(DEV),
                                   chunk=w.chunk, state_S=S, state_z=z).float().cpu().numpy()
    S = S.cpu().numpy()
    for bb, h in ((0, 0), (1, 15)):
        sl = (slice(bb, bb + 1), slice(h, h + 1))
        ro, rS, rz = orc.causal(q[sl], k[sl], v[sl], f[sl], gain=i[sl], mlstm=True)
        assert row_rel_err(o[sl], ro) < 2e-2, row_rel_err(o[sl], ro)
        assert row_rel_err(S[sl].reshape(1, 1, -1), rS.reshape(1, 1, -1)) < 2e-2


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.float16, 32)])
def test_mlstm_decode(la, orc, dtype, d):
    rng = np.random.default_rng(d + 1)
    B, H = 3, 4
    q = torch.from_numpy(rng.standard_normal((B, H, d), dtype=np.float32)).to(dtype)
    k, v = (torch.from_numpy(rng.standard_normal((B, H, d), dtype=np.float32) / np.sqrt(d)).to(dtype)
            for _ in range(2))
    f = torch.from_numpy((1 / (1 + np.exp(-(rng.standard_normal((B, H)) + 2)))).astype(np.float32))
    i = torch.from_numpy(np.exp(0.5 * rng.standard_normal((B, H)) - 0.5).astype(np.float32))
    S0 = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.3)
    z0 = torch.from_numpy(rng.standard_normal((B, H, d)).astype(np.float32) * 0.3)
    S, z = S0.to(DEV), z0.to(DEV)
    o = la.la_decode_step_mlstm(q.to(DEV), k.to(DEV), v.to(DEV), S, z, forget=f.to(DEV), input_gate=i.to(DEV),
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rS, rz = orc.decode_step(q, k, v, S0, z0, decay=f, gain=i, mlstm=True)
    assert row_rel_err(o.cpu().numpy(), ro) < tol_for(dtype)
    assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < 1e-5
    assert row_rel_err(z.cpu().numpy(), rz) < 1e-5


# ------------------------------------------- decode exactly as the bench runs it
def test_workload_decode_as_benched(la, orc):
    """The long-context decode as the bench runs it: fp32 states from the
    library's own prefill of the seeded 512-token prompt (B64 H16, chunk 128),
    then all 1024 steps updating the states in place, the distinct step inputs
    cycled.  The oracle receives the same fp32 states and runs its decode step
    1024 times on sampled heads; every step's output and the final state are
    compared.  The prompt's states are also checked against the oracle's
    prefill of the prompt (the prefill -> decode hand-off)."""
    wd = W["decode_bf16_b64h16_d128"]
    B, H, d = wd.B, wd.H, wd.d
    pq, pk, pv = inputs.decode_prompt(wd)
    S = torch.zeros((B, H, d, d), device=DEV)
    z = torch.zeros((B, H, d), device=DEV)
    la.la_prefill_causal(pq.to(DEV), pk.to(DEV), pv.to(DEV), chunk=128, state_S=S, state_z=z,
                         mode=la.LA_STATE_OUT)
    torch.cuda.synchronize()
    S0, z0 = S.cpu().numpy().astype(np.float64), z.cpu().numpy().astype(np.float64)
    bidx = np.array([0, 17, 40, 63])
    hidx = np.array([0, 5, 11, 15])
    sel = lambda x: x[bidx, hidx][None]          # [1, n_sampled, ...]
    _, rS_p, rz_p = orc.causal(sel(pq), sel(pk), sel(pv))
    assert row_rel_err(sel(S0).reshape(1, len(bidx), -1), rS_p.reshape(1, len(bidx), -1)) < 2e-2
    assert row_rel_err(sel(z0), rz_p) < 2e-2

    n_in = inputs.DECODE_DISTINCT_INPUTS
    steps_in = [inputs.decode_inputs(wd, i) for i in range(n_in)]
    dq = torch.stack([s[0] for s in steps_in]).to(DEV)
    dk = torch.stack([s[1] for s in steps_in]).to(DEV)
    dv = torch.stack([s[2] for s in steps_in]).to(DEV)
    outs = torch.empty((wd.steps, B, H, d), dtype=wd.torch_out_dtype, device=DEV)
    for i in range(wd.steps):
        j = i % n_in
        la.la_decode_step(dq[j], dk[j], dv[j], S, z, eps=wd.eps, out=outs[i])
    torch.cuda.synchronize()
    got = outs[:, bidx, hidx].float().cpu().numpy()          # [steps, n_sampled, d]
    rS, rz = sel(S0), sel(z0)
    worst = 0.0
    for i in range(wd.steps):
        q, k, v, _ = steps_in[i % n_in]
        ro, rS, rz = orc.decode_step(sel(q), sel(k), sel(v), rS, rz, eps=wd.eps)
        worst = max(worst, row_rel_err(got[i][None], ro))
    assert worst < 2e-2, f"worst step output rel err {worst}"
    Sg, zg = S.cpu().numpy(), z.cpu().numpy()
    assert row_rel_err(sel(Sg).reshape(1, len(bidx), -1), rS.reshape(1, len(bidx), -1)) < 2e-2
    assert row_rel_err(sel(zg), rz) < 2e-2


# ------------------------------------------------- feature-map and decay range
def _scaled_inputs(dtype, d, T, B, H, seed, qk_std, decay=None):
    rng = np.random.default_rng(seed)
    mk = lambda s: torch.from_numpy((rng.standard_normal((B, H, T, d), dtype=np.float32) * s)).to(dtype)
    q, k, v = mk(qk_std), mk(qk_std), mk(1.0 / np.sqrt(d))
    return q, k, v


# (dtype, d, chunk, qk_std): the workloads' N(0,1)/sqrt(d) scaled x4 and x8,
# and unit-variance inputs x3, whose e^x branch reaches x < -10 (phi(x) of
# order 1e-5) while the x + 1 branch reaches x > 10
PHI_RANGE = [
    (torch.bfloat16, 128, 128, 4.0 / np.sqrt(128)),
    (torch.bfloat16, 128, 64, 8.0 / np.sqrt(128)),
    (torch.bfloat16, 64, 64, 8.0 / np.sqrt(64)),
    (torch.float16, 128, 128, 8.0 / np.sqrt(128)),
    (torch.bfloat16, 128, 128, 3.0),
    (torch.bfloat16, 64, 64, 3.0),
    (torch.float16, 64, 128, 3.0),
]


@pytest.mark.parametrize("dtype,d,chunk,qk_std", PHI_RANGE)
@pytest.mark.parametrize("decay", [False, True])
def test_prefill_phi_range(la, orc, dtype, d, chunk, qk_std, decay):
    """The tensor-core feature map on both branches far from 0: phi(x) = x + 1
    for large x and e^x for x << 0 (2^(x log2 e) on the ex2 unit, rounded to
    bf16)."""
    B, H, T = 1, 2, 1100
    q, k, v = _scaled_inputs(dtype, d, T, B, H, seed=int(qk_std * 1000) + d, qk_std=qk_std)
    a = None
    if decay:
        rng = np.random.default_rng(d)
        a = torch.from_numpy((1 / (1 + np.exp(-(rng.standard_normal((B, H, T)) + 2)))).astype(np.float32))
    if qk_std >= 2.0:
        assert float(q.float().min()) < -10 and float(k.float().max()) > 10
    check_prefill(la, orc, q, k, v, a, chunk, torch.float32, 2e-2)


@pytest.mark.parametrize("dtype,d,chunk", [(torch.bfloat16, 128, 64), (torch.bfloat16, 128, 128),
                                           (torch.bfloat16, 64, 64), (torch.float32, 64, 64),
                                           (torch.float16, 32, 128)])
def test_prefill_decay_extremes(la, orc, dtype, d, chunk):
    """Decays of 1 mixed inside every chunk with decays of 1e-6 and 1e-30,
    where the in-chunk weights 2^(L_i - L_j) underflow to 0 and the carried
    state is wiped; the exact answer is the recurrence's."""
    B, H, T = 2, 2, 1500
    q, k, v, _ = _small_inputs(dtype, d, T, False, B, H, seed=71 + d)
    rng = np.random.default_rng(72 + d)
    u = rng.uniform(size=(B, H, T))
    a = np.ones((B, H, T), dtype=np.float32)
    a[u < 0.08] = 1e-6
    a[(u >= 0.08) & (u < 0.12)] = 1e-30
    a[(u >= 0.12) & (u < 0.5)] = rng.uniform(0.2, 1.0, size=int(((u >= 0.12) & (u < 0.5)).sum()))
    a = torch.from_numpy(a)
    check_prefill(la, orc, q, k, v, a, chunk, torch.float32, tol_for(dtype))


# ------------------------------------------------------------- timeout path
@pytest.mark.parametrize("d,chunk,decay", [(128, 128, False), (128, 64, True)])
def test_wait_timeout_is_reported_and_next_call_is_exact(la, d, chunk, decay):
    """With the wait limit set to 0 every device-side wait that is not already
    satisfied gives up at once: the blocks drain their copies and products,
    free their tensor memory and exit, and the workspace's status word reports
    LA_ERR_TIMEOUT with the id of the wait.  The next call with the default
    limit is bitwise equal to the call before the timeout."""
    B, H, T = 1, 2, 3000
    q, k, v, a = _small_inputs(torch.bfloat16, d, T, decay, B, H, seed=81)
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    ad = None if a is None else a.to(DEV)
    ws = torch.empty(la.la_prefill_workspace_size(B, H, T, d, d, chunk), dtype=torch.uint8, device=DEV)

    def call():
        S = torch.zeros((B, H, d, d), device=DEV)
        z = torch.zeros((B, H, d), device=DEV)
        o = la.la_prefill_causal(qd, kd, vd, decay=ad, chunk=chunk, state_S=S, state_z=z,
                                 out_dtype=torch.float32, workspace=ws)
        return o, S

    o1, S1 = call()
    assert la.la_workspace_status(ws) == (la.LA_OK, 0)
    old = la.la_set_wait_limit_ns(0)
    try:
        call()
        st, waiter = la.la_workspace_status(ws)
    finally:
        la.la_set_wait_limit_ns(old)
    assert st == la.LA_ERR_TIMEOUT and waiter > 0
    o3, S3 = call()
    assert la.la_workspace_status(ws) == (la.LA_OK, 0)
    assert torch.equal(o1, o3) and torch.equal(S1, S3)


@pytest.mark.parametrize("dtype,d,chunk,decay,gain", [(torch.bfloat16, 128, 128, False, False),
                                                       (torch.bfloat16, 64, 64, True, True),
                                                       (torch.float32, 64, 64, True, False)])
def test_prefill_from_host(la, orc, dtype, d, chunk, decay, gain):
    """The host-input prefill (pinned host tensors, the sequence in pieces with
    the copies overlapped, the state carried between the pieces): equal to the
    oracle over the whole sequence, with a state in and out, the last piece
    ragged."""
    from kernelized_causal_sequence_b200 import hostio
    B, H = 2, 3
    T = 1000 if chunk == 128 else 1024   # pieces of 256 with a ragged last one / whole pieces only
    q, k, v, a = _small_inputs(dtype, d, T, decay, B, H, seed=91)
    rng = np.random.default_rng(92)
    b = torch.from_numpy(rng.uniform(0.2, 1.5, (B, H, T)).astype(np.float32)) if gain else None
    S0 = torch.from_numpy(rng.standard_normal((B, H, d, d), dtype=np.float32) * 0.1)
    z0 = torch.from_numpy(np.abs(rng.standard_normal((B, H, d), dtype=np.float32)) + 1.0)
    pin = lambda x: None if x is None else x.contiguous().pin_memory()
    S, z = S0.to(DEV).clone(), z0.to(DEV).clone()
    out, S, z = hostio.prefill_causal_from_host(pin(q), pin(k), pin(v), decay=pin(a), gain=pin(b), chunk=chunk,
                                                out_dtype=torch.float32, state_S=S, state_z=z, piece_tokens=256)
    torch.cuda.synchronize()
    ro, rS, rz = orc.causal(q, k, v, a, 1e-6, S_in=S0.double().numpy(), z_in=z0.double().numpy(),
                            gain=None if b is None else b.double().numpy())
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert row_rel_err(out.numpy(), ro) < tol
    assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < tol
    assert row_rel_err(z.cpu().numpy(), rz) < tol


def test_prefill_from_host_one_short_piece(la, orc):
    """The host-input prefill when the whole sequence is shorter than one
    chunk (a single ragged piece), no state given."""
    from kernelized_causal_sequence_b200 import hostio
    q, k, v, a = _small_inputs(torch.bfloat16, 128, 100, True, 1, 2, seed=93)
    pin = lambda x: x.contiguous().pin_memory()
    out, S, z = hostio.prefill_causal_from_host(pin(q), pin(k), pin(v), decay=pin(a), chunk=128,
                                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rS, rz = orc.causal(q, k, v, a)
    assert row_rel_err(out.numpy(), ro) < 2e-2
    assert row_rel_err(S.cpu().numpy().reshape(1, 2, -1), rS.reshape(1, 2, -1)) < 2e-2


@pytest.mark.parametrize("B,H,Lq,Lk", [(16, 16, 500, 2000), (16, 64, 129, 65), (2, 3, 1, 5000)])
def test_noncausal_tc_many_heads(la, orc, B, H, Lq, Lk):
    """The tensor-core non-causal path with many heads per SM (256 and 1024
    heads), or one group of heads split into many key segments: equal to the
    oracle with a state in and out, and bitwise repeatable."""
    rng = np.random.default_rng(B * H + Lq)
    mk = lambda L: torch.from_numpy(rng.standard_normal((B, H, L, 32), dtype=np.float32) * 0.6).to(torch.bfloat16)
    q, k, v = mk(Lq), mk(Lk), mk(Lk)
    S0 = torch.from_numpy(rng.standard_normal((B, H, 32, 32), dtype=np.float32))
    z0 = torch.from_numpy(np.abs(rng.standard_normal((B, H, 32), dtype=np.float32)) + 1.0)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    ro, rS, rz = orc.noncausal(q, k, v, S_in=S0, z_in=z0)
    outs = []
    for _ in range(2):
        S, z = S0.to(DEV).clone(), z0.to(DEV).clone()
        o = la.la_forward_noncausal(qd, kd, vd, state_S=S, state_z=z, mode=la.LA_STATE_INOUT,
                                    out_dtype=torch.float32)
        outs.append((o, S, z))
    torch.cuda.synchronize()
    o, S, z = outs[0]
    assert row_rel_err(o.cpu().numpy(), ro) < 2e-2
    assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < 2e-2
    assert row_rel_err(z.cpu().numpy(), rz) < 2e-2
    assert all(torch.equal(x, y) for x, y in zip(outs[0], outs[1]))


def test_noncausal_wait_limit_zero(la):
    """The non-causal tensor-core call under a wait limit of 0: every wait not
    satisfied at once gives up, the blocks drain and exit, the status word
    reports LA_ERR_TIMEOUT; the next call with the default limit is bitwise
    equal to the call before."""
    B, H, Lq, Lk = 2, 8, 3000, 3000
    rng = np.random.default_rng(83)
    mk = lambda L: torch.from_numpy(rng.standard_normal((B, H, L, 32), dtype=np.float32) * 0.6).to(DEV).half()
    q, k, v = mk(Lq), mk(Lk), mk(Lk)
    ws = torch.empty(la.la_noncausal_workspace_size(B, H, Lk, 32, 32), dtype=torch.uint8, device=DEV)

    def call():
        S = torch.zeros((B, H, 32, 32), device=DEV)
        z = torch.zeros((B, H, 32), device=DEV)
        o = la.la_forward_noncausal(q, k, v, state_S=S, state_z=z, mode=la.LA_STATE_OUT, out_dtype=torch.float32,
                                    workspace=ws)
        return o, S, z

    r1 = call()
    assert la.la_workspace_status(ws) == (la.LA_OK, 0)
    old = la.la_set_wait_limit_ns(0)
    try:
        call()
        st, waiter = la.la_workspace_status(ws)
    finally:
        la.la_set_wait_limit_ns(old)
    assert st == la.LA_ERR_TIMEOUT and waiter > 0
    r3 = call()
    assert la.la_workspace_status(ws) == (la.LA_OK, 0)
    assert all(torch.equal(x, y) for x, y in zip(r1, r3))


@pytest.mark.parametrize("B,H,Lq,Lk", [(1, 3, 700, 900), (3, 7, 300, 2000), (1, 1, 128, 128)])
def test_noncausal_tc_head_groups(la, orc, B, H, Lq, Lk):
    """Head counts that leave the tensor-core state pass's last group of four
    heads partly empty, in every state mode; the output is deterministic and
    the same without a state output."""
    rng = np.random.default_rng(B * 100 + H)
    mk = lambda L: torch.from_numpy(rng.standard_normal((B, H, L, 32), dtype=np.float32) * 0.7).to(torch.float16)
    q, k, v = mk(Lq), mk(Lk), mk(Lk)
    S0 = torch.from_numpy(rng.standard_normal((B, H, 32, 32), dtype=np.float32))
    z0 = torch.from_numpy(np.abs(rng.standard_normal((B, H, 32), dtype=np.float32)) + 1.0)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    ro, rS, rz = orc.noncausal(q, k, v, S_in=S0, z_in=z0)
    S, z = S0.to(DEV).clone(), z0.to(DEV).clone()
    o1 = la.la_forward_noncausal(qd, kd, vd, state_S=S, state_z=z, mode=la.LA_STATE_INOUT, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert row_rel_err(o1.cpu().numpy(), ro) < 2e-2
    assert row_rel_err(S.cpu().numpy().reshape(B, H, -1), rS.reshape(B, H, -1)) < 2e-2
    assert row_rel_err(z.cpu().numpy(), rz) < 2e-2
    ro0, rS0, _ = orc.noncausal(q, k, v)
    S2 = torch.full((B, H, 32, 32), 5.0, device=DEV)
    z2 = torch.full((B, H, 32), 5.0, device=DEV)
    o2 = la.la_forward_noncausal(qd, kd, vd, state_S=S2, state_z=z2, mode=la.LA_STATE_OUT, out_dtype=torch.float32)
    o3 = la.la_forward_noncausal(qd, kd, vd, out_dtype=torch.float32)
    o4 = la.la_forward_noncausal(qd, kd, vd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert row_rel_err(o2.cpu().numpy(), ro0) < 2e-2
    assert row_rel_err(S2.cpu().numpy().reshape(B, H, -1), rS0.reshape(B, H, -1)) < 2e-2
    assert torch.equal(o2, o3) and torch.equal(o3, o4)


# ------------------------------------------------------------- FLASH chunk form
# Exact relu(q.k / s)^2 attention inside each chunk, q^T (earlier chunks'
# summaries) / s across chunks; s = 1 (equations) or s = chunk (listings).
FLASH = [
    # (dtype, d, T, chunk, B, H)
    (torch.bfloat16, 128, 1000, 128, 1, 2),    # ragged last chunk
    (torch.bfloat16, 128, 1500, 64, 2, 1),
    (torch.bfloat16, 64, 777, 64, 1, 3),
    (torch.bfloat16, 64, 600, 128, 1, 2),
    (torch.float16, 128, 513, 64, 1, 2),
    (torch.bfloat16, 128, 5000, 64, 1, 1),     # > 64 segments per head
    (torch.bfloat16, 128, 64, 64, 1, 1),       # one chunk: causal squared-ReLU attention alone
]


def _flash_inputs(dtype, d, T, B, H, seed):
    rng = np.random.default_rng(seed)
    s = d ** -0.25   # q.k ~ N(0, 1)
    mk = lambda sc: torch.from_numpy(rng.standard_normal((B, H, T, d), dtype=np.float32) * sc).to(dtype)
    return mk(s), mk(s), mk(1.0)


@pytest.mark.parametrize("dtype,d,T,chunk,B,H", FLASH)
@pytest.mark.parametrize("scaled", [False, True])
def test_flash_prefill(la, orc, dtype, d, T, chunk, B, H, scaled):
    q, k, v = _flash_inputs(dtype, d, T, B, H, seed=T + d + chunk)
    ro, rS = orc.flash(q, k, v, chunk, scaled=scaled)
    inv_s = 1.0 / chunk if scaled else 1.0
    for out_dtype in (torch.float32, dtype):
        S = torch.zeros((B, H, d, d), device=DEV)
        z = torch.zeros((B, H, d), device=DEV)
        o = la.la_prefill_causal_flash(q.to(DEV), k.to(DEV), v.to(DEV), chunk=chunk, scaled=scaled, state_S=S,
                                       state_z=z, out_dtype=out_dtype)
        torch.cuda.synchronize()
        o = o.float().cpu().numpy()
        err = row_rel_err(o, ro)
        assert err < 2e-2, f"output rel err {err}"
        Sg = S.cpu().numpy() * inv_s
        assert row_rel_err(Sg.reshape(B, H, -1), rS.reshape(B, H, -1)) < 2e-2
        rz = k.double().numpy().sum(axis=2)
        assert row_rel_err(z.cpu().numpy(), rz) < 2e-2


@pytest.mark.parametrize("scaled", [False, True])
def test_flash_state_handoff(la, orc, scaled):
    """A prefill split at a chunk boundary, the second part starting from the
    first part's state, equals the whole prefill."""
    d, T1, T2, chunk = 128, 640, 517, 64
    q, k, v = _flash_inputs(torch.bfloat16, d, T1 + T2, 1, 2, seed=5)
    ro, _ = orc.flash(q, k, v, chunk, scaled=scaled)
    S = torch.zeros((1, 2, d, d), device=DEV)
    z = torch.zeros((1, 2, d), device=DEV)
    dv = lambda x, a, b: x[:, :, a:b].contiguous().to(DEV)
    o1 = la.la_prefill_causal_flash(dv(q, 0, T1), dv(k, 0, T1), dv(v, 0, T1), chunk=chunk, scaled=scaled,
                                    state_S=S, state_z=z, out_dtype=torch.float32)
    o2 = la.la_prefill_causal_flash(dv(q, T1, T1 + T2), dv(k, T1, T1 + T2), dv(v, T1, T1 + T2), chunk=chunk,
                                    scaled=scaled, state_S=S, state_z=z, mode=la.LA_STATE_INOUT,
                                    out_dtype=torch.float32)
    torch.cuda.synchronize()
    o = np.concatenate([o1.cpu().numpy(), o2.cpu().numpy()], axis=2)
    assert row_rel_err(o, ro) < 2e-2


def test_flash_rejects_unsupported(la):
    q = torch.zeros((1, 1, 64, 32), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(la.LinAttnError):
        la.la_prefill_causal_flash(q, q, q, chunk=64)          # d = 32: no tensor-core path
    q = torch.zeros((1, 1, 64, 64), dtype=torch.float32, device=DEV)
    with pytest.raises(la.LinAttnError):
        la.la_prefill_causal_flash(q, q, q, chunk=64)          # fp32 inputs
