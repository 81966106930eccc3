"""Host-side checks of the seeded input recipes shared by the CUDA path's
tests/bench and the oracle: determinism, shapes and dtypes, and the gate
inputs of the gated and mLSTM workloads."""
import math

import numpy as np
import torch

from kernelized_causal_sequence_b200 import inputs

W = inputs.WORKLOADS


def test_recipes_are_deterministic_and_typed():
    for name in ("causal_bf16_b4h8_t2048_d64", "ssd_decay_bf16_b2h16_t8192_d128",
                 "rfa_gated_bf16_b2h16_t8192_d128", "mlstm_bf16_b2h16_t8192_d128"):
        w = W[name]
        a1 = inputs.qkv(w, T=96, B=1, H=2)
        a2 = inputs.qkv(w, T=96, B=1, H=2)
        for x, y in zip(a1[:3], a2[:3]):
            assert x.dtype == w.torch_dtype and x.shape == (1, 2, 96, w.d)
            assert torch.equal(x, y)
        if w.decay:
            assert a1[3].dtype == torch.float32 and a1[3].shape == (1, 2, 96)
            assert torch.equal(a1[3], a2[3])
            assert float(a1[3].min()) > 0.0 and float(a1[3].max()) < 1.0
        else:
            assert a1[3] is None


def test_rfa_gain_is_one_minus_gate():
    w = W["rfa_gated_bf16_b2h16_t8192_d128"]
    _, _, _, g = inputs.qkv(w, T=64, B=1, H=2)
    b = inputs.gate_gain(w, g)
    assert b.dtype == torch.float32
    assert np.array_equal(b.numpy(), (np.float32(1.0) - g.numpy()).astype(np.float32))
    assert inputs.gate_gain(W["ssd_decay_bf16_b2h16_t8192_d128"], g) is None


def test_mlstm_inputs():
    w = W["mlstm_bf16_b2h16_t8192_d128"]
    q, k, v, f = inputs.qkv(w, T=4096, B=1, H=2)
    i1 = inputs.input_gate(w, T=4096, B=1, H=2)
    i2 = inputs.input_gate(w, T=4096, B=1, H=2)
    assert torch.equal(i1, i2) and i1.shape == (1, 2, 4096) and float(i1.min()) > 0.0
    # log of the input gate ~ N(-0.5, 0.5^2); queries unscaled, keys by 1/sqrt(d)
    li = np.log(i1.numpy().astype(np.float64))
    assert abs(li.mean() + 0.5) < 0.05 and abs(li.std() - 0.5) < 0.05
    assert abs(q.float().std().item() - 1.0) < 0.05
    assert abs(k.float().std().item() - 1 / math.sqrt(w.d)) < 0.01
    assert inputs.input_gate(W["ssd_decay_bf16_b2h16_t8192_d128"]) is None
