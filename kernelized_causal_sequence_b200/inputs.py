"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds the input recipes only — shapes, dtypes, value
distributions and seeds — and none of the method's arithmetic (no feature
map, no sums, no read-out).  Both sides receive the arrays it returns, cast
once to the workload dtype; the oracle widens them to fp64 exactly.

Recipe: ``numpy.random.default_rng(seed)`` (PCG64) draws standard normals as
float32 in C order, in the order q, k, v, then the decay logits g, then (for
decode) q, k, v of each step.  Values are scaled as the workload states and
then rounded once to the workload dtype with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

_TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One workload of the hot path.  ``kind`` is causal | noncausal | decode."""
    name: str
    kind: str
    B: int
    H: int
    T: int              # tokens (causal), Lq (non-causal); 1 for decode
    d: int              # d_k = d_v
    dtype: str          # f32 | bf16 | f16
    out_dtype: str
    chunk: int = 64
    decay: bool = False
    gated: bool = False   # RFA gate: decay a_t = g_t and gain b_t = 1 - g_t on the new term
    mlstm: bool = False   # mLSTM read-out: decay = forget gate, plus an input gate (input_gate())
    flash: bool = False   # the FLASH chunk form (its own entry point)
    k_scale: float = 0.0  # keys' scale when it differs from qk_scale (0: qk_scale)
    eps: float = 1e-6
    Lk: int = 0         # non-causal only
    qk_scale: float = 1.0
    v_scale: float = 1.0
    seed: int = 0
    steps: int = 0      # decode only
    prompt: int = 0     # decode only: tokens summarised by the initial state

    @property
    def torch_dtype(self):
        return _TORCH_DTYPES[self.dtype]

    @property
    def torch_out_dtype(self):
        return _TORCH_DTYPES[self.out_dtype]


# The five workloads of the hot path.  Seeds are 1000 + index; the non-causal
# "cross" keys/values use seed 1000 + 4 + 100.
WORKLOADS = {
    # causal, fp32 inputs, no decay: B=1, H=1, T=256, d=64, chunk 64
    "causal_f32_t256_d64": Workload("causal_f32_t256_d64", "causal", 1, 1, 256, 64, "f32", "f32",
                                    chunk=64, seed=1001),
    # causal bf16, no decay: B=4, H=8, T=2048, d=64, inputs N(0,1)/sqrt(64)
    "causal_bf16_b4h8_t2048_d64": Workload("causal_bf16_b4h8_t2048_d64", "causal", 4, 8, 2048, 64,
                                           "bf16", "bf16", chunk=64, qk_scale=1 / 8, v_scale=1 / 8,
                                           seed=1002),
    # SSD-style scalar decay a_t = sigmoid(g_t), g_t ~ N(2, 1): B=2, H=16, T=8192, d=128
    "ssd_decay_bf16_b2h16_t8192_d128": Workload("ssd_decay_bf16_b2h16_t8192_d128", "causal", 2, 16,
                                                8192, 128, "bf16", "bf16", chunk=64, decay=True,
                                                qk_scale=1 / math.sqrt(128),
                                                v_scale=1 / math.sqrt(128), seed=1003),
    # the gated form (RFA's sigmoid gate g_t = sigmoid(N(2, 1)), decay g_t and gain 1 - g_t)
    # at the SSD workload's shape and chunk
    "rfa_gated_bf16_b2h16_t8192_d128": Workload("rfa_gated_bf16_b2h16_t8192_d128", "causal", 2, 16,
                                                8192, 128, "bf16", "bf16", chunk=64, decay=True,
                                                gated=True, qk_scale=1 / math.sqrt(128),
                                                v_scale=1 / math.sqrt(128), seed=1006),
    # the mLSTM read-out at the same shape: q ~ N(0,1), k and v ~ N(0,1)/sqrt(128),
    # forget gate sigmoid(N(2, 1)), input gate exp(0.5 N(0, 1) - 0.5)
    "mlstm_bf16_b2h16_t8192_d128": Workload("mlstm_bf16_b2h16_t8192_d128", "causal", 2, 16, 8192, 128,
                                            "bf16", "bf16", chunk=64, decay=True, mlstm=True,
                                            qk_scale=1.0, k_scale=1 / math.sqrt(128),
                                            v_scale=1 / math.sqrt(128), seed=1007),
    # the FLASH chunk form at the same shape: q, k ~ N(0,1)/128^(1/4) (so q.k ~ N(0,1)),
    # v ~ N(0,1)/sqrt(128); the chunk is part of the form's definition
    "flash_bf16_b2h16_t8192_d128": Workload("flash_bf16_b2h16_t8192_d128", "causal", 2, 16, 8192, 128,
                                            "bf16", "bf16", chunk=64, flash=True, qk_scale=128 ** -0.25,
                                            v_scale=1 / math.sqrt(128), seed=1008),
    # non-causal, LoFTR-coarse shape: B=8, H=8, L=4800, d=32, fp16, V pre-scaled by 1/Lk
    "noncausal_f16_b8h8_l4800_d32": Workload("noncausal_f16_b8h8_l4800_d32", "noncausal", 8, 8,
                                             4800, 32, "f16", "f32", chunk=128, Lk=4800,
                                             v_scale=1 / 4800, seed=1004),
    # long-context prefill: B=1, H=16, T=131072, d=128, chunk 128
    "prefill_bf16_h16_t131072_d128": Workload("prefill_bf16_h16_t131072_d128", "causal", 1, 16,
                                              131072, 128, "bf16", "bf16", chunk=128,
                                              qk_scale=1 / math.sqrt(128),
                                              v_scale=1 / math.sqrt(128), seed=1005),
    # 1024 decode steps at B=64, H=16 from fp32 states of a 512-token prompt
    "decode_bf16_b64h16_d128": Workload("decode_bf16_b64h16_d128", "decode", 64, 16, 1, 128,
                                        "bf16", "bf16", qk_scale=1 / math.sqrt(128),
                                        v_scale=1 / math.sqrt(128), seed=1005 + 200, steps=1024,
                                        prompt=512),
}


def _normals(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _cast(a32: np.ndarray, dtype: str) -> torch.Tensor:
    """Round an fp32 array once to the workload dtype (round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(a32)).to(_TORCH_DTYPES[dtype])


def qkv(w: Workload, seed: int | None = None, T: int | None = None, B: int | None = None,
        H: int | None = None):
    """Q, K, V ([B,H,T,d] each, workload dtype, CPU) plus decay [B,H,T] fp32 or None.

    ``T``/``B``/``H`` override the workload's sizes (smaller parity cases with
    the same distributions)."""
    seed = w.seed if seed is None else seed
    B = w.B if B is None else B
    H = w.H if H is None else H
    T = w.T if T is None else T
    rng = np.random.default_rng(seed)
    shape = (B, H, T, w.d)
    q = _cast(_normals(rng, shape) * np.float32(w.qk_scale), w.dtype)
    k = _cast(_normals(rng, shape) * np.float32(w.k_scale or w.qk_scale), w.dtype)
    v = _cast(_normals(rng, shape) * np.float32(w.v_scale), w.dtype)
    decay = None
    if w.decay:
        g = _normals(rng, (B, H, T)) + np.float32(2.0)
        a = (np.float32(1.0) / (np.float32(1.0) + np.exp(-g))).astype(np.float32)
        decay = torch.from_numpy(a)
    return q, k, v, decay


def gate_gain(w: Workload, decay: torch.Tensor | None) -> torch.Tensor | None:
    """The gain input of a gated workload: 1 - g for the gate g drawn as its
    decay (fp32, rounded once), else None."""
    if not w.gated or decay is None:
        return None
    return torch.from_numpy((np.float32(1.0) - decay.numpy()).astype(np.float32))


def input_gate(w: Workload, T: int | None = None, B: int | None = None,
               H: int | None = None) -> torch.Tensor | None:
    """The input gate of an mLSTM workload, exp(0.5 x - 0.5) with x ~ N(0, 1)
    drawn from its own stream (seed + 50), [B,H,T] fp32; else None."""
    if not w.mlstm:
        return None
    B = w.B if B is None else B
    H = w.H if H is None else H
    T = w.T if T is None else T
    rng = np.random.default_rng(w.seed + 50)
    x = _normals(rng, (B, H, T))
    return torch.from_numpy(np.exp(np.float32(0.5) * x - np.float32(0.5)).astype(np.float32))


def cross_kv(w: Workload, Lk: int | None = None, B: int | None = None, H: int | None = None):
    """Second key/value set for the non-causal cross-attention case (seed + 100)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    Lk = w.Lk if Lk is None else Lk
    rng = np.random.default_rng(w.seed + 100)
    shape = (B, H, Lk, w.d)
    k = _cast(_normals(rng, shape) * np.float32(w.qk_scale), w.dtype)
    v = _cast(_normals(rng, shape) * np.float32(w.v_scale), w.dtype)
    return k, v


def decode_state(w: Workload, B: int | None = None, H: int | None = None):
    """Synthetic fp32 starting state (S [B,H,d,d], z [B,H,d]) with the magnitudes
    of a ``w.prompt``-token prefill of the workload's inputs: z ~= prompt (the
    feature means are ~1 at this input scale), S ~= a sum of ``prompt`` value
    rows (std sqrt(prompt) * v_scale).  Drawn directly, not computed."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    rng = np.random.default_rng(w.seed + 7)
    S = _normals(rng, (B, H, w.d, w.d)) * np.float32(math.sqrt(w.prompt) * w.v_scale)
    z = np.float32(w.prompt) * (np.float32(1.0) + np.float32(0.05) * _normals(rng, (B, H, w.d)))
    return torch.from_numpy(S.astype(np.float32)), torch.from_numpy(z.astype(np.float32))


# Distinct per-step decode inputs; a longer decode loop cycles through them.
DECODE_DISTINCT_INPUTS = 64


def decode_prompt(w: Workload):
    """The prompt whose prefill state starts a decode workload: q, k, v
    [B, H, w.prompt, d] drawn like the long-context prefill's inputs (same
    scales and dtype) from the decode workload's seed + 1."""
    pw = WORKLOADS["prefill_bf16_h16_t131072_d128"]
    q, k, v, _ = qkv(pw, T=w.prompt, B=w.B, H=w.H, seed=w.seed + 1)
    return q, k, v


def decode_inputs(w: Workload, step: int, B: int | None = None, H: int | None = None,
                  decay: bool = False):
    """q, k, v [B,H,d] for one decode step (step-major streams), optional decay [B,H]."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    rng = np.random.default_rng([w.seed, step])
    shape = (B, H, w.d)
    q = _cast(_normals(rng, shape) * np.float32(w.qk_scale), w.dtype)
    k = _cast(_normals(rng, shape) * np.float32(w.qk_scale), w.dtype)
    v = _cast(_normals(rng, shape) * np.float32(w.v_scale), w.dtype)
    a = None
    if decay:
        g = _normals(rng, (B, H)) + np.float32(2.0)
        a = torch.from_numpy((np.float32(1.0) / (np.float32(1.0) + np.exp(-g))).astype(np.float32))
    return q, k, v, a
