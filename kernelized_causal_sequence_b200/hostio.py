"""Causal prefill of inputs that live in pinned host memory.

The sequence is cut into pieces of whole chunks along T.  Piece i's inputs
are copied to the device on one stream while piece i-1 is computed on the
caller's stream (la_prefill_causal with the state carried in place, mode
INOUT: the chunked recurrence is the same whether the tokens arrive in one
call or in several) and piece i-2's output is copied back on a third stream.
A piece's rows are strided in the [B, H, T, d] host tensors (one block per
head), so each copy is one 2-D copy (cudaMemcpy2DAsync): B*H rows of the
piece's bytes per head.  Two device buffers per tensor alternate between the
pieces; events order every reuse.

The result equals one la_prefill_causal call over the whole sequence up to
rounding (the pieces set their own segment plans).
"""
from __future__ import annotations

import torch

import kernelized_causal_sequence_b200 as _la

_STREAMS = {}


def _streams(dev):
    # the copy streams of device `dev` (an explicit index), made once
    if dev.index not in _STREAMS:
        _STREAMS[dev.index] = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev))
    return _STREAMS[dev.index]


def _copy2d(dst_ptr, dpitch, src_ptr, spitch, width, height, stream):
    from cuda.bindings import runtime as rt
    (err,) = rt.cudaMemcpy2DAsync(dst_ptr, dpitch, src_ptr, spitch, width, height,
                                  rt.cudaMemcpyKind.cudaMemcpyDefault, rt.cudaStream_t(stream.cuda_stream))
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaMemcpy2DAsync failed: {err}")


def prefill_causal_from_host(q, k, v, decay=None, gain=None, eps=1e-6, chunk=64, out=None, out_dtype=None,
                             state_S=None, state_z=None, piece_tokens=16384, device="cuda"):
    """Causal prefill of pinned host tensors, copies overlapped with the kernels.

    q, k: [B, H, T, d_k]; v: [B, H, T, d_v] (pinned CPU, contiguous, bf16/f16/f32);
    decay, gain: [B, H, T] fp32 pinned or None.  ``out``: pinned CPU [B, H, T, d_v]
    (allocated, pinned, when None).  ``state_S`` [B, H, d_k, d_v] / ``state_z``
    [B, H, d_k] fp32 on the device: the state entering the sequence (zeros when
    None); on return they hold the state after it.  ``piece_tokens`` is rounded
    down to whole chunks.  Work is queued on the current stream of ``device``,
    which waits for the last copy back; returns (out, state_S, state_z).
    """
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    BH = B * H
    dev = torch.device(device)
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    out_dtype = q.dtype if out_dtype is None else out_dtype
    for x in (q, k, v) + tuple(y for y in (decay, gain) if y is not None):
        if x.is_cuda or not x.is_contiguous() or not x.is_pinned():
            raise ValueError("inputs: contiguous pinned host tensors")
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=out_dtype).pin_memory()
    elif out.is_cuda or not out.is_contiguous() or not out.is_pinned() or tuple(out.shape) != (B, H, T, dv):
        raise ValueError("out: a contiguous pinned host tensor [B, H, T, d_v]")
    if state_S is None:
        state_S = torch.zeros((B, H, dk, dv), dtype=torch.float32, device=dev)
        state_z = torch.zeros((B, H, dk), dtype=torch.float32, device=dev)
    tp = max(chunk, (min(piece_tokens, max(T, 1)) // chunk) * chunk)
    bounds = [(t0, min(T, t0 + tp)) for t0 in range(0, T, tp)]
    main = torch.cuda.current_stream(dev)
    s_in, s_out = _streams(dev)
    eq, ek, ev, eo = q.element_size(), k.element_size(), v.element_size(), out.element_size()
    bufs = [dict(q=torch.empty((B, H, tp, dk), dtype=q.dtype, device=dev),
                 k=torch.empty((B, H, tp, dk), dtype=k.dtype, device=dev),
                 v=torch.empty((B, H, tp, dv), dtype=v.dtype, device=dev),
                 a=None if decay is None else torch.empty((B, H, tp), dtype=torch.float32, device=dev),
                 b=None if gain is None else torch.empty((B, H, tp), dtype=torch.float32, device=dev),
                 o=torch.empty((B, H, tp, dv), dtype=out_dtype, device=dev)) for _ in range(2)]
    ws = _la._workspace(_la.la_prefill_workspace_size(B, H, tp, dk, dv, chunk), dev)
    computed = [torch.cuda.Event() for _ in range(2)]   # piece's kernels done: its input buffers are free
    copied_out = [torch.cuda.Event() for _ in range(2)]   # piece's output copied back: its out buffer is free
    start = torch.cuda.Event()
    start.record(main)
    s_in.wait_event(start)
    s_out.wait_event(start)
    for i, (t0, t1) in enumerate(bounds):
        n = t1 - t0
        bf = bufs[i & 1]
        if i >= 2:
            s_in.wait_event(computed[i & 1])
        for name, host, w in (("q", q, dk * eq), ("k", k, dk * ek), ("v", v, dv * ev), ("a", decay, 4),
                              ("b", gain, 4)):
            if host is None:
                continue
            _copy2d(bf[name].data_ptr(), n * w, host.data_ptr() + t0 * w, T * w, n * w, BH, s_in)
        loaded = torch.cuda.Event()
        loaded.record(s_in)
        main.wait_event(loaded)
        if i >= 2:
            main.wait_event(copied_out[i & 1])
        view = lambda x, last: None if x is None else x.view(-1)[:BH * n * last].view(B, H, n, last)
        sub = lambda x: None if x is None else x.view(-1)[:BH * n].view(B, H, n)
        o = view(bf["o"], dv)
        _la.la_prefill_causal(view(bf["q"], dk), view(bf["k"], dk), view(bf["v"], dv), decay=sub(bf["a"]),
                              gain=sub(bf["b"]), eps=eps, chunk=chunk, state_S=state_S, state_z=state_z,
                              mode=_la.LA_STATE_INOUT, out=o, workspace=ws, stream=main)
        computed[i & 1].record(main)
        s_out.wait_event(computed[i & 1])
        _copy2d(out.data_ptr() + t0 * dv * eo, T * dv * eo, o.data_ptr(), n * dv * eo, n * dv * eo, BH, s_out)
        copied_out[i & 1].record(s_out)
    done = torch.cuda.Event()
    done.record(s_out)
    main.wait_event(done)
    # the piece buffers stay in use on the side streams until `done`
    for bf in bufs:
        for x in bf.values():
            if x is not None:
                x.record_stream(s_in)
                x.record_stream(s_out)
    return out, state_S, state_z
