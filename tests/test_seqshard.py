"""Sequence sharding of one causal prefill over ranks (one exchange step).

CPU: two and three gloo ranks run kernelized_causal_sequence_b200.seqshard
with the library's compute steps replaced by stand-ins built on the fp64
oracle (the library's kernels need a GPU).  What is checked is the exchange
and its ordering: every rank's summary reaches the others in rank order,
each rank's entry state is the oracle's state of the whole sequence at that
rank's first token, and each rank's output is the whole-sequence output on
its tokens.

GPU (marked gpu): the same sharded computation through the library's kernels
(la_prefill_causal_summary, la_state_combine, la_prefill_causal with INOUT),
the ranks emulated one after the other on one GPU (the steps of different
ranks never wait on one another, so this is exact), compared with the oracle
and with the unsharded prefill.
"""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tests.conftest import row_rel_err  # noqa: E402

B, H, T, D = 1, 2, 96, 8


def _inputs():
    rng = np.random.default_rng(2024)
    q = rng.standard_normal((B, H, T, D)) / np.sqrt(D)
    k = rng.standard_normal((B, H, T, D)) / np.sqrt(D)
    v = rng.standard_normal((B, H, T, D))
    a = 1.0 / (1.0 + np.exp(-(rng.standard_normal((B, H, T)) + 2.0)))
    b = rng.uniform(0.0, 1.5, (B, H, T))
    return q, k, v, a, b


def _oracle_ops():
    """Stand-in compute steps on the fp64 oracle (CPU tensors)."""
    import oracle
    from kernelized_causal_sequence_b200.seqshard import ShardOps

    def summary(k, v, decay, gain, chunk):
        zq = torch.zeros_like(k)
        _, S, z = oracle.causal(zq, k, v, decay, 1e-6, gain=gain)
        A = np.prod(decay.numpy(), axis=-1) if decay is not None else np.ones(k.shape[:2])
        return torch.from_numpy(S), torch.from_numpy(z), torch.from_numpy(A)

    def combine(S_all, z_all, A_all, r, S_in, z_in):
        S = torch.zeros_like(S_all[0]) if S_in is None else S_in.clone()
        z = torch.zeros_like(z_all[0]) if z_in is None else z_in.clone()
        for i in range(r):
            S = A_all[i][..., None, None] * S + S_all[i]
            z = A_all[i][..., None] * z + z_all[i]
        return S, z

    def prefill(q, k, v, decay, gain, eps, chunk, S, z, out_dtype):
        o, S1, z1 = oracle.causal(q, k, v, decay, eps, S_in=S, z_in=z, gain=gain)
        S.copy_(torch.from_numpy(S1))
        z.copy_(torch.from_numpy(z1))
        return torch.from_numpy(o)

    return ShardOps(summary=summary, combine=combine, prefill=prefill)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, with_state, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from kernelized_causal_sequence_b200 import seqshard
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    q, k, v, a, b = (torch.from_numpy(x) for x in _inputs())
    n = T // world
    sl = slice(rank * n, (rank + 1) * n)
    S0 = torch.full((B, H, D, D), 0.25, dtype=torch.float64) if with_state else None
    z0 = torch.full((B, H, D), 2.0, dtype=torch.float64) if with_state else None
    ops = _oracle_ops()
    # record the entry state the combine step hands to the prefill
    entry = {}
    inner = ops.prefill

    def prefill(q_, k_, v_, decay, gain, eps, chunk, S, z, out_dtype):
        entry["S"], entry["z"] = S.clone(), z.clone()
        return inner(q_, k_, v_, decay, gain, eps, chunk, S, z, out_dtype)

    ops.prefill = prefill
    o, S, z = seqshard.sharded_prefill(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                       v[:, :, sl].contiguous(), decay=a[:, :, sl].contiguous(),
                                       gain=b[:, :, sl].contiguous(), chunk=64, state_S=S0, state_z=z0, ops=ops)
    dist.destroy_process_group()
    out.put((rank, o.numpy(), S.numpy(), z.numpy(), entry["S"].numpy(), entry["z"].numpy()))


def _run(world, with_state):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, with_state, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in procs], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world,with_state", [(2, False), (3, True)])
def test_sharded_prefill_matches_whole_sequence(orc, world, with_state):
    res = _run(world, with_state)
    q, k, v, a, b = _inputs()
    S0 = np.full((B, H, D, D), 0.25) if with_state else None
    z0 = np.full((B, H, D), 2.0) if with_state else None
    ro, rS, rz = orc.causal(q, k, v, a, 1e-6, S_in=S0, z_in=z0, gain=b)
    n = T // world
    for rank, o, S, z, eS, ez in res:
        # entry state = the oracle's state after the tokens before this shard
        if rank == 0:
            pS = np.zeros((B, H, D, D)) if S0 is None else S0
            pz = np.zeros((B, H, D)) if z0 is None else z0
        else:
            _, pS, pz = orc.causal(q[:, :, :rank * n], k[:, :, :rank * n], v[:, :, :rank * n],
                                   a[:, :, :rank * n], 1e-6, S_in=S0, z_in=z0, gain=b[:, :, :rank * n])
        np.testing.assert_allclose(eS, pS, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(ez, pz, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o, ro[:, :, rank * n:(rank + 1) * n], rtol=1e-10, atol=1e-12)
    # the last rank ends with the whole sequence's state
    np.testing.assert_allclose(res[-1][2], rS, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[-1][3], rz, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- GPU: real kernels
@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d,chunk,shards,decay", [(torch.bfloat16, 128, 128, 2, False),
                                                        (torch.bfloat16, 128, 64, 3, True),
                                                        (torch.float32, 64, 64, 2, True),
                                                        (torch.float16, 64, 128, 4, True)])
def test_sharded_prefill_kernels_emulated_ranks(la, orc, dtype, d, chunk, shards, decay):
    """The sharded prefill through the library's kernels, ranks emulated one
    after the other on one GPU: summaries -> stacked as an all-gather would ->
    combine -> prefill with the entry state (INOUT).  Equal to the oracle on
    the whole sequence, and the last shard's state is the final state."""
    Bq, Hq, Tq = 2, 3, 2600
    rng = np.random.default_rng(d + shards)
    mk = lambda: torch.from_numpy(rng.standard_normal((Bq, Hq, Tq, d), dtype=np.float32) / np.sqrt(d)).to(dtype)
    q, k, v = mk(), mk(), mk()
    a = None
    if decay:
        a = torch.from_numpy((1 / (1 + np.exp(-(rng.standard_normal((Bq, Hq, Tq)) + 2)))).astype(np.float32))
    ro, rS, rz = orc.causal(q, k, v, a)
    bounds = [Tq * i // shards for i in range(shards + 1)]
    dev = lambda x, lo, hi: None if x is None else x[:, :, lo:hi].contiguous().cuda()
    sums = [la.la_prefill_causal_summary(dev(k, lo, hi), dev(v, lo, hi), decay=dev(a, lo, hi), chunk=chunk)
            for lo, hi in zip(bounds[:-1], bounds[1:])]
    S_all = torch.stack([s[0] for s in sums])
    z_all = torch.stack([s[1] for s in sums])
    A_all = torch.stack([s[2] for s in sums])
    outs = []
    for r, (lo, hi) in enumerate(zip(bounds[:-1], bounds[1:])):
        S, z = la.la_state_combine(S_all, z_all, A_all, r)
        if r > 0:
            _, pS, pz = orc.causal(q[:, :, :lo], k[:, :, :lo], v[:, :, :lo], None if a is None else a[:, :, :lo])
            assert row_rel_err(S.cpu().numpy().reshape(Bq, Hq, -1), pS.reshape(Bq, Hq, -1)) < 2e-2
            assert row_rel_err(z.cpu().numpy(), pz) < 2e-2
        o = la.la_prefill_causal(dev(q, lo, hi), dev(k, lo, hi), dev(v, lo, hi), decay=dev(a, lo, hi), chunk=chunk,
                                 state_S=S, state_z=z, mode=la.LA_STATE_INOUT, out_dtype=torch.float32)
        outs.append(o.cpu().numpy())
    torch.cuda.synchronize()
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert row_rel_err(np.concatenate(outs, axis=2), ro) < tol
    assert row_rel_err(S.cpu().numpy().reshape(Bq, Hq, -1), rS.reshape(Bq, Hq, -1)) < tol
    assert row_rel_err(z.cpu().numpy(), rz) < tol
    # the decay products
    if a is not None:
        for i, (lo, hi) in enumerate(zip(bounds[:-1], bounds[1:])):
            # products of ~900 decays of ~0.88 underflow fp32 to 0 (the exact ones are ~1e-60)
            np.testing.assert_allclose(A_all[i].cpu().numpy(), np.prod(a[:, :, lo:hi].double().numpy(), axis=-1),
                                       rtol=1e-4, atol=1e-37)
    else:
        assert torch.all(A_all == 1)
