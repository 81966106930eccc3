"""Causal prefill of one sequence sharded along its tokens over the ranks of a
process group (one GPU per rank), with one exchange step.

The recurrence of the causal form is affine in the carried state: a block of
tokens maps an entry state X = (S, z) to A X + dX ("Linear attention" concept
card, SSD variant: the chunked algorithm carries one state between blocks).
Rank r holds tokens [r T_r, (r + 1) T_r) of every head.  Each rank

  1. summarises its shard on its GPU (la_prefill_causal_summary: the shard's
     contribution dS, dz from a zero state, and the decay product A),
  2. all-gathers the summaries (one collective; NCCL over NVLink on GPUs),
  3. folds the earlier shards' summaries into its entry state on its GPU
     (la_state_combine), and
  4. runs la_prefill_causal on its shard with that entry state (INOUT).

The summaries are (d_k d_v + d_k + 1) fp32 per head (66 KB at d = 128), so the
exchange is small next to the shard's own tokens.  The last rank's state
after step 4 is the state of the whole sequence.

The compute steps are the library's kernels; ``ops`` only exists so that the
exchange and its ordering can be exercised on CPU ranks (gloo) with
stand-in steps.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional

import torch

import kernelized_causal_sequence_b200 as _la


@dataclasses.dataclass
class ShardOps:
    """The three compute steps of a sharded prefill.

    summary(k, v, decay, gain, chunk) -> (dS [B,H,dk,dv], dz [B,H,dk], A [B,H]) fp32
    combine(S_all, z_all, A_all, r, S_in, z_in) -> (S [B,H,dk,dv], z [B,H,dk]) entry state of shard r
    prefill(q, k, v, decay, gain, eps, chunk, S, z, out_dtype) -> out; updates S, z in place to the
        state after the shard
    """
    summary: Callable
    combine: Callable
    prefill: Callable


def _gpu_summary(k, v, decay, gain, chunk):
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    S = torch.empty((B, H, dk, dv), dtype=torch.float32, device=k.device)
    z = torch.empty((B, H, dk), dtype=torch.float32, device=k.device)
    A = torch.empty((B, H), dtype=torch.float32, device=k.device)
    _la.la_prefill_causal_summary(k, v, decay=decay, gain=gain, chunk=chunk, sum_S=S, sum_z=z, sum_A=A)
    return S, z, A


def _gpu_combine(S_all, z_all, A_all, r, S_in, z_in):
    return _la.la_state_combine(S_all, z_all, A_all, r, S_in=S_in, z_in=z_in)


def _gpu_prefill(q, k, v, decay, gain, eps, chunk, S, z, out_dtype):
    return _la.la_prefill_causal(q, k, v, decay=decay, eps=eps, chunk=chunk, state_S=S, state_z=z,
                                 mode=_la.LA_STATE_INOUT, out_dtype=out_dtype, gain=gain)


GPU_OPS = ShardOps(summary=_gpu_summary, combine=_gpu_combine, prefill=_gpu_prefill)


def sharded_prefill(q, k, v, decay=None, gain=None, eps=1e-6, chunk=64, group=None, state_S=None,
                    state_z=None, out_dtype=None, ops: Optional[ShardOps] = None):
    """This rank's part of a causal prefill whose tokens are split over the
    ranks of ``group`` in rank order.

    q, k, v: this rank's shard [B, H, T_r, d]; decay, gain: [B, H, T_r] or
    None.  ``state_S``/``state_z`` (optional, fp32): the state entering the
    whole sequence, the same on every rank.  Returns (out, S, z): the shard's
    output and the state after the shard (on the last rank, the state after
    the whole sequence).  Every rank takes part in the one all-gather.
    """
    import torch.distributed as dist
    ops = GPU_OPS if ops is None else ops
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    dS, dz, A = ops.summary(k, v, decay, gain, chunk)
    # one exchange: every rank's summary, packed into one buffer
    flat = torch.cat([dS.reshape(-1), dz.reshape(-1), A.reshape(-1)])
    gathered = torch.empty(world * flat.numel(), dtype=flat.dtype, device=flat.device)
    dist.all_gather_into_tensor(gathered, flat, group=group)
    gathered = gathered.view(world, flat.numel())
    nS, nz = dS.numel(), dz.numel()
    S_all = gathered[:, :nS].reshape((world,) + tuple(dS.shape))
    z_all = gathered[:, nS:nS + nz].reshape((world,) + tuple(dz.shape))
    A_all = gathered[:, nS + nz:].reshape((world,) + tuple(A.shape))
    S, z = ops.combine(S_all.contiguous(), z_all.contiguous(), A_all.contiguous(), rank, state_S, state_z)
    out = ops.prefill(q, k, v, decay, gain, eps, chunk, S, z, out_dtype)
    return out, S, z
