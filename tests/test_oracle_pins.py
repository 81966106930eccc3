"""Pins for the fp64 oracle, checked against things the pages and the
mathematics fix, never against the oracle itself:

* the linear-attention lesson's worked N=8, d=4, seed-0 example and its
  masked quadratic check (tests/golden/lesson_n8_d4_seed0.txt);
* brute-force masked quadratic attention on tiny inputs (the lesson's
  "same thing written as masked quadratic attention");
* the decayed, 1-semiseparable weighted quadratic form (the lesson's "Try it
  yourself" decay exercise; the concept card's SSD variant);
* decay 1 being the plain causal form (concept card, SSD variant);
* associativity of the non-causal bracketing (knowledge-base page, section 3;
  lesson, "Two ways to bracket the same product");
* closed forms on constructed inputs, the feature map against torch's elu,
  invariances, state split / hand-off equivalences.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def phi_ref(x):
    """elu(x)+1 through torch's own elu, in fp64 (library routine)."""
    return torch.nn.functional.elu(torch.as_tensor(x, dtype=torch.float64)).numpy() + 1.0


def quad_causal(q, k, v, eps, weights=None):
    """Brute force masked quadratic form for one head: scores = phi(Q) phi(K)^T,
    masked to j <= i (and weighted if given), rows normalised by their sums."""
    fq, fk = phi_ref(q), phi_ref(k)
    T = q.shape[0]
    scores = fq @ fk.T
    mask = np.tril(np.ones((T, T)))
    scores = scores * mask
    if weights is not None:
        scores = scores * weights
    return (scores @ v) / (scores.sum(-1, keepdims=True) + eps)


def read_golden(name):
    vals = {}
    multi = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = [s.strip() for s in line.split("=", 1)]
            if key in vals:
                multi.setdefault(key, [vals[key]]).append(val)
            vals[key] = val
    return vals, multi


def test_lesson_worked_example(orc):
    g, multi = read_golden("lesson_n8_d4_seed0.txt")
    N, d, eps = int(g["N"]), int(g["d"]), float(g["eps"])
    torch.manual_seed(int(g["seed"]))
    Q, K, V = torch.randn(N, d), torch.randn(N, d), torch.randn(N, d)
    out, S, z = orc.causal(Q[None, None], K[None, None], V[None, None], eps=eps)
    out = out[0, 0]
    # the page's fp32 masked quadratic form, recomputed in fp32 with torch
    q32, k32 = torch.nn.functional.elu(Q) + 1, torch.nn.functional.elu(K) + 1
    sc = (q32 @ k32.T) * torch.tril(torch.ones(N, N))
    quad32 = ((sc @ V) / (sc.sum(-1, keepdim=True) + eps)).double().numpy()
    # the oracle agrees with the page's check at the page's tolerance, and with
    # the fp32 result to the magnitude the page prints (4.77e-7, fp32 rounding)
    atol = float(g["recurrent_matches_quadratic_atol"])
    assert np.abs(out - quad32).max() <= atol
    assert np.abs(out - quad32).max() <= 10 * float(g["max_difference_fp32"])
    # fp64 brute force: agreement to rounding
    np.testing.assert_allclose(out, quad_causal(Q.double().numpy(), K.double().numpy(),
                                                V.double().numpy(), eps), rtol=1e-12, atol=1e-13)
    # state carried: d x d numbers, independent of t
    assert S[0, 0].size == int(g["state_numbers"]) == d * d
    assert 2 * N * d == int(g["kv_cache_numbers_at_t8"])
    # bracketing: (q k^T) V == q (k^T V) in the non-causal form
    onc, _, _ = orc.noncausal(Q[None, None], K[None, None], V[None, None], eps=eps)
    fq, fk = phi_ref(Q.double().numpy()), phi_ref(K.double().numpy())
    left = (fq @ fk.T) @ V.double().numpy() / ((fq @ fk.T).sum(-1, keepdims=True) + eps)
    np.testing.assert_allclose(onc[0, 0], left, rtol=1e-12, atol=1e-13)
    assert g["scores_shape"] == f"{N}x{N}" and g["kTv_shape"] == f"{d}x{d}"
    for row in multi["crossover"]:
        n, a, b, r = row.split()
        n = int(n)
        assert n * n * d == int(a) and n * d * d == int(b) and float(r) == n * n * d / (n * d * d)


@pytest.mark.parametrize("seed,T,dk,dv", [(1, 1, 1, 1), (2, 5, 3, 2), (3, 17, 4, 4),
                                          (4, 64, 8, 5), (5, 33, 2, 7)])
def test_masked_quadratic_bruteforce(orc, seed, T, dk, dv):
    rng = np.random.default_rng(seed)
    B, H = 2, 3
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    out, S, z = orc.causal(q, k, v, eps=1e-6)
    for b in range(B):
        for h in range(H):
            ref = quad_causal(q[b, h], k[b, h], v[b, h], 1e-6)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-11, atol=1e-12)
            # final state is the full prefix sum
            fk = phi_ref(k[b, h])
            np.testing.assert_allclose(S[b, h], fk.T @ v[b, h], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(z[b, h], fk.sum(0), rtol=1e-12)


def _semiseparable(a):
    """W[i, j] = prod_{l=j+1..i} a_l for j <= i, else 0 — explicit products."""
    T = a.shape[0]
    W = np.zeros((T, T))
    for i in range(T):
        for j in range(i + 1):
            p = 1.0
            for l in range(j + 1, i + 1):
                p *= a[l]
            W[i, j] = p
    return W


@pytest.mark.parametrize("seed,T,d", [(11, 9, 3), (12, 40, 4), (13, 64, 6)])
def test_decayed_quadratic(orc, seed, T, d):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 2, T, d))
    k = rng.standard_normal((1, 2, T, d))
    v = rng.standard_normal((1, 2, T, d))
    a = 1.0 / (1.0 + np.exp(-(rng.standard_normal((1, 2, T)) + 2.0)))
    out, S, z = orc.causal(q, k, v, decay=a, eps=1e-6)
    for h in range(2):
        W = _semiseparable(a[0, h])
        ref = quad_causal(q[0, h], k[0, h], v[0, h], 1e-6, weights=W)
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-11, atol=1e-12)
        # final state: sum_j (prod_{l>j} a_l) phi(k_j) v_j^T
        fk = phi_ref(k[0, h])
        np.testing.assert_allclose(S[0, h], (fk * W[-1][:, None]).T @ v[0, h], rtol=1e-11,
                                   atol=1e-12)


def test_lesson_decay_exercise(orc):
    """S = 0.9 S + outer(k, v): no longer the unweighted quadratic form, but the
    one weighted by 0.9^(i-j)."""
    torch.manual_seed(0)
    N, d = 8, 4
    Q, K, V = (torch.randn(N, d).double().numpy() for _ in range(3))
    a = np.full((1, 1, N), 0.9)
    out, _, _ = orc.causal(Q[None, None], K[None, None], V[None, None], decay=a, eps=1e-6)
    plain = quad_causal(Q, K, V, 1e-6)
    assert np.abs(out[0, 0] - plain).max() > 1e-3
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    W = np.where(j <= i, 0.9 ** (i - j).astype(float), 0.0)
    np.testing.assert_allclose(out[0, 0], quad_causal(Q, K, V, 1e-6, weights=W), rtol=1e-12,
                               atol=1e-13)


def test_decay_one_is_plain_bitwise(orc):
    rng = np.random.default_rng(21)
    q, k, v = (rng.standard_normal((2, 2, 50, 6)) for _ in range(3))
    o1, S1, z1 = orc.causal(q, k, v, eps=1e-6)
    o2, S2, z2 = orc.causal(q, k, v, decay=np.ones((2, 2, 50)), eps=1e-6)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2) and np.array_equal(z1, z2)


def test_feature_map_against_torch_elu(orc):
    """Two tokens, v = (1, 0), k_1 = 0 (phi = 1): o_1 = phi(k_0) / (phi(k_0) + 1),
    so phi(k_0) is recovered from the oracle's output and compared with torch's
    elu(x)+1 on both branches."""
    xs = np.array([-30.0, -3.0, -1.0, -0.25, -1e-8, 0.0, 1e-8, 0.3, 1.0, 4.0])
    for x in xs:
        q = np.zeros((1, 1, 2, 1))
        k = np.array([x, 0.0]).reshape(1, 1, 2, 1)
        v = np.array([1.0, 0.0]).reshape(1, 1, 2, 1)
        out, _, _ = orc.causal(q, k, v, eps=0.0)
        o = out[0, 0, 1, 0]
        # torch forms elu(x)+1 as (expm1(x)) + 1, exact to ~1 ulp of 1.0 in
        # absolute terms; hence the absolute floor
        np.testing.assert_allclose(o / (1 - o), phi_ref(x), rtol=1e-12, atol=1e-15)


def test_noncausal_associativity_and_state_in(orc):
    rng = np.random.default_rng(31)
    B, H, Lq, Lk, d, e = 2, 2, 23, 37, 5, 3
    q = rng.standard_normal((B, H, Lq, d))
    k = rng.standard_normal((B, H, Lk, d))
    v = rng.standard_normal((B, H, Lk, e))
    out, S, z = orc.noncausal(q, k, v, eps=1e-6)
    for b in range(B):
        for h in range(H):
            fq, fk = phi_ref(q[b, h]), phi_ref(k[b, h])
            sc = fq @ fk.T
            ref = (sc @ v[b, h]) / (sc.sum(-1, keepdims=True) + 1e-6)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-13)
    # state-in equals an extra prefix of keys
    k2 = rng.standard_normal((B, H, 11, d))
    v2 = rng.standard_normal((B, H, 11, e))
    o_split, S_split, z_split = orc.noncausal(q, k2, v2, eps=1e-6, S_in=S, z_in=z)
    o_all, S_all, z_all = orc.noncausal(q, np.concatenate([k, k2], 2),
                                        np.concatenate([v, v2], 2), eps=1e-6)
    np.testing.assert_allclose(o_split, o_all, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S_split, S_all, rtol=1e-12, atol=1e-12)
    # V scaled by c scales the output by c; key order does not matter
    o_c, _, _ = orc.noncausal(q, k, 3.5 * v, eps=1e-6)
    np.testing.assert_allclose(o_c, 3.5 * out, rtol=1e-12, atol=1e-13)
    perm = rng.permutation(Lk)
    o_p, _, _ = orc.noncausal(q, k[:, :, perm], v[:, :, perm], eps=1e-6)
    np.testing.assert_allclose(o_p, out, rtol=1e-12, atol=1e-13)


def test_causal_last_row_is_noncausal(orc):
    rng = np.random.default_rng(41)
    q, k, v = (rng.standard_normal((1, 3, 30, 4)) for _ in range(3))
    oc, Sc, zc = orc.causal(q, k, v, eps=1e-6)
    on, Sn, zn = orc.noncausal(q[:, :, -1:], k, v, eps=1e-6)
    np.testing.assert_allclose(oc[:, :, -1:], on, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sc, Sn, rtol=1e-12, atol=1e-12)


def test_closed_forms(orc):
    rng = np.random.default_rng(51)
    eps = 1e-6
    # T = 1: o = v w / (w + eps), w = phi(q).phi(k)
    q, k, v = (rng.standard_normal((1, 1, 1, 6)) for _ in range(3))
    out, _, _ = orc.causal(q, k, v, eps=eps)
    w = float(phi_ref(q[0, 0, 0]) @ phi_ref(k[0, 0, 0]))
    np.testing.assert_allclose(out[0, 0, 0], v[0, 0, 0] * w / (w + eps), rtol=1e-14)
    # constant value rows: o_t = c den_t / (den_t + eps)
    T = 20
    q, k = (rng.standard_normal((1, 1, T, 4)) for _ in range(2))
    c = rng.standard_normal(3)
    v = np.broadcast_to(c, (1, 1, T, 3)).copy()
    out, _, _ = orc.causal(q, k, v, eps=eps)
    fq, fk = phi_ref(q[0, 0]), phi_ref(k[0, 0])
    den = np.array([fq[t] @ fk[: t + 1].sum(0) for t in range(T)])
    np.testing.assert_allclose(out[0, 0], c[None] * (den / (den + eps))[:, None], rtol=1e-13)
    # all keys equal: o_t = (sum_{j<=t} v_j) / ((t + 1) + eps / w_t)
    kk = np.broadcast_to(rng.standard_normal(4), (1, 1, T, 4)).copy()
    v = rng.standard_normal((1, 1, T, 3))
    out, _, _ = orc.causal(q, kk, v, eps=eps)
    wt = fq @ phi_ref(kk[0, 0, 0])
    ref = np.cumsum(v[0, 0], 0) / (np.arange(1, T + 1) + eps / wt)[:, None]
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12)


@pytest.mark.parametrize("with_decay", [False, True])
def test_state_split_and_decode_handoff(orc, with_decay):
    rng = np.random.default_rng(61 + with_decay)
    B, H, T1, T2, d, e = 2, 2, 13, 19, 5, 4
    q = rng.standard_normal((B, H, T1 + T2 + 1, d))
    k = rng.standard_normal((B, H, T1 + T2 + 1, d))
    v = rng.standard_normal((B, H, T1 + T2 + 1, e))
    a = rng.uniform(0.5, 1.0, (B, H, T1 + T2 + 1)) if with_decay else None
    sl = lambda x, s: None if x is None else x[:, :, s]
    T = T1 + T2
    o_full, S_full, z_full = orc.causal(q[:, :, :T], k[:, :, :T], v[:, :, :T], sl(a, slice(0, T)))
    o1, S1, z1 = orc.causal(sl(q, slice(0, T1)), sl(k, slice(0, T1)), sl(v, slice(0, T1)),
                            sl(a, slice(0, T1)))
    o2, S2, z2 = orc.causal(sl(q, slice(T1, T)), sl(k, slice(T1, T)), sl(v, slice(T1, T)),
                            sl(a, slice(T1, T)), S_in=S1, z_in=z1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 2), o_full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S_full, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z2, z_full, rtol=1e-12)
    # prefill(T) then one decode step == prefill(T + 1), last row
    od, Sd, zd = orc.decode_step(q[:, :, T], k[:, :, T], v[:, :, T], S_full, z_full,
                                 decay=None if a is None else a[:, :, T])
    o_next, S_next, z_next = orc.causal(q, k, v, a)
    np.testing.assert_allclose(od, o_next[:, :, T], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sd, S_next, rtol=1e-12, atol=1e-12)


def test_kb_opcount_closed_form():
    """The knowledge-base page's op counts are T d' d_h and T^2 d_h."""
    g, _ = read_golden("kb_opcount_d128_t100k.txt")
    T, dp, dh = int(g["T"]), int(g["d_feature"]), int(g["d_head"])
    tol = float(g["rel_rounding"])
    assert abs(T * dp * dh / float(g["linear_ops_approx"]) - 1) < tol
    assert abs(T * T * dh / float(g["softmax_ops_approx"]) - 1) < tol


def test_oracle_thread_count_invariance(orc):
    rng = np.random.default_rng(71)
    q, k, v = (rng.standard_normal((3, 3, 40, 4)) for _ in range(3))
    n = orc.max_threads()
    orc.set_threads(1)
    o1, _, _ = orc.causal(q, k, v)
    orc.set_threads(max(n, 2))
    o2, _, _ = orc.causal(q, k, v)
    orc.set_threads(n)
    assert np.array_equal(o1, o2)


# ------------------------------------------------------------------ gated form
# A per-token gain b_t on the new term, S_t = a_t S_{t-1} + b_t phi(k_t) v_t^T
# (and z alike).  Random Feature Attention's sigmoid gate is a_t = g_t,
# b_t = 1 - g_t (concept card, RFA variant and the closing paragraph of its
# implementation sketch; RFA eq. 7).

@pytest.mark.parametrize("seed,T,d", [(81, 9, 3), (82, 40, 4), (83, 64, 6)])
def test_gated_quadratic(orc, seed, T, d):
    """The gated recurrence equals the quadratic form weighted by
    W_ij = (prod_{l=j+1..i} a_l) * b_j: the gain belongs to the key's token and
    is not decayed at its own step."""
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, 2, T, d)) for _ in range(3))
    a = 1.0 / (1.0 + np.exp(-(rng.standard_normal((1, 2, T)) + 2.0)))
    b = rng.uniform(0.0, 2.0, (1, 2, T))
    b[0, 0, T // 3] = 0.0   # a key that enters with weight zero
    out, S, z = orc.causal(q, k, v, decay=a, eps=1e-6, gain=b)
    for h in range(2):
        W = _semiseparable(a[0, h]) * b[0, h][None, :]
        ref = quad_causal(q[0, h], k[0, h], v[0, h], 1e-6, weights=W)
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-11, atol=1e-12)
        fk = phi_ref(k[0, h])
        np.testing.assert_allclose(S[0, h], (fk * W[-1][:, None]).T @ v[0, h], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(z[0, h], (fk * W[-1][:, None]).sum(0), rtol=1e-11, atol=1e-12)
    # the gain is not the decay: moving it onto the query index changes the result
    W_wrong = _semiseparable(a[0, 1]) * b[0, 1][:, None]
    assert np.abs(out[0, 1] - quad_causal(q[0, 1], k[0, 1], v[0, 1], 1e-6, weights=W_wrong)).max() > 1e-3


def test_rfa_gate_closed_form(orc):
    """Constant gate g, all keys equal (w = phi(q_t).phi(k) per query): the
    gated sums are geometric, z_t = (1 - g^(t+1)) phi(k) and
    o_t = w (1-g) sum_{j<=t} g^(t-j) v_j / (w (1 - g^(t+1)) + eps)."""
    rng = np.random.default_rng(91)
    T, d, e, g, eps = 30, 4, 3, 0.8, 1e-3
    q = rng.standard_normal((1, 1, T, d))
    kk = np.broadcast_to(rng.standard_normal((1, 1, 1, d)), (1, 1, T, d)).copy()
    v = rng.standard_normal((1, 1, T, e))
    out, S, z = orc.causal(q, kk, v, decay=np.full((1, 1, T), g), eps=eps, gain=np.full((1, 1, T), 1.0 - g))
    fk = phi_ref(kk[0, 0, 0])
    w = phi_ref(q[0, 0]) @ fk
    t = np.arange(T)
    num = np.stack([(1.0 - g) * (g ** (tt - np.arange(tt + 1)))[:, None].T @ v[0, 0, :tt + 1] for tt in t])[:, 0]
    ref = (w[:, None] * num) / (w * (1.0 - g ** (t + 1)) + eps)[:, None]
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(z[0, 0], (1.0 - g ** T) * fk, rtol=1e-12)


@pytest.mark.parametrize("with_decay", [False, True])
def test_gain_one_is_plain_bitwise(orc, with_decay):
    rng = np.random.default_rng(95 + with_decay)
    q, k, v = (rng.standard_normal((2, 2, 50, 6)) for _ in range(3))
    a = rng.uniform(0.5, 1.0, (2, 2, 50)) if with_decay else None
    o1, S1, z1 = orc.causal(q, k, v, decay=a, eps=1e-6)
    o2, S2, z2 = orc.causal(q, k, v, decay=a, eps=1e-6, gain=np.ones((2, 2, 50)))
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2) and np.array_equal(z1, z2)


def test_gain_scale_invariance(orc):
    """With eps = 0 the read-out is a ratio, so scaling every gain by c leaves
    the outputs unchanged while the state scales by c."""
    rng = np.random.default_rng(97)
    q, k, v = (rng.standard_normal((1, 2, 33, 5)) for _ in range(3))
    a = rng.uniform(0.6, 1.0, (1, 2, 33))
    b = rng.uniform(0.1, 1.0, (1, 2, 33))
    o1, S1, z1 = orc.causal(q, k, v, decay=a, eps=0.0, gain=b)
    o2, S2, z2 = orc.causal(q, k, v, decay=a, eps=0.0, gain=3.0 * b)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, 3.0 * S1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(z2, 3.0 * z1, rtol=1e-12)


def test_gated_split_and_decode_handoff(orc):
    rng = np.random.default_rng(99)
    B, H, T1, T2, d, e = 1, 2, 11, 17, 4, 3
    T = T1 + T2
    q = rng.standard_normal((B, H, T + 1, d))
    k = rng.standard_normal((B, H, T + 1, d))
    v = rng.standard_normal((B, H, T + 1, e))
    g = 1.0 / (1.0 + np.exp(-(rng.standard_normal((B, H, T + 1)) + 2.0)))
    a, b = g, 1.0 - g
    o_full, S_full, z_full = orc.causal(q[:, :, :T], k[:, :, :T], v[:, :, :T], a[:, :, :T], gain=b[:, :, :T])
    o1, S1, z1 = orc.causal(q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], a[:, :, :T1], gain=b[:, :, :T1])
    o2, S2, z2 = orc.causal(q[:, :, T1:T], k[:, :, T1:T], v[:, :, T1:T], a[:, :, T1:T], S_in=S1, z_in=z1,
                            gain=b[:, :, T1:T])
    np.testing.assert_allclose(np.concatenate([o1, o2], 2), o_full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S_full, rtol=1e-12, atol=1e-12)
    od, Sd, zd = orc.decode_step(q[:, :, T], k[:, :, T], v[:, :, T], S_full, z_full, decay=a[:, :, T],
                                 gain=b[:, :, T])
    o_next, S_next, z_next = orc.causal(q, k, v, a, gain=b)
    np.testing.assert_allclose(od, o_next[:, :, T], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sd, S_next, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(zd, z_next, rtol=1e-12)


# ------------------------------------------------------------- mLSTM read-out
# Concept card, "Matrix memory with exponential gates (mLSTM)":
# C_t = f_t C_{t-1} + i_t v_t k_t^T, n_t = f_t n_{t-1} + i_t k_t, and the
# read-out C_t q_t / max(|n_t^T q_t|, 1); its implementation sketch places it
# in the running-sum loop with the identity as the feature map.

def _mlstm_quadratic(q, k, v, f, i):
    """Quadratic form of one head: raw scores q_t.k_j weighted by
    (prod_{l=j+1..t} f_l) i_j for j <= t; numerator = weighted scores @ v,
    denominator max(|row sum|, 1)."""
    W = _semiseparable(f) * i[None, :]
    sc = (q @ k.T) * W
    den = np.maximum(np.abs(sc.sum(-1)), 1.0)
    return (sc @ v) / den[:, None], sc.sum(-1)


@pytest.mark.parametrize("seed,T,d,qs", [(101, 12, 3, 1.0), (102, 48, 4, 0.7), (103, 64, 8, 1.5)])
def test_mlstm_quadratic(orc, seed, T, d, qs):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 2, T, d)) * qs
    k, v = (rng.standard_normal((1, 2, T, d)) for _ in range(2))
    f = 1.0 / (1.0 + np.exp(-(rng.standard_normal((1, 2, T)) + 2.0)))
    i = np.exp(rng.standard_normal((1, 2, T)) * 0.5)
    out, S, z = orc.causal(q, k, v, decay=f, gain=i, mlstm=True)
    seen_small = seen_large = False
    for h in range(2):
        ref, den = _mlstm_quadratic(q[0, h], k[0, h], v[0, h], f[0, h], i[0, h])
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-11, atol=1e-12)
        seen_small |= bool((np.abs(den) < 1).any())
        seen_large |= bool((np.abs(den) > 1).any())
        # the memory holds the raw keys: S = sum_j w_j k_j v_j^T, z = sum_j w_j k_j
        w = _semiseparable(f[0, h])[-1] * i[0, h]
        np.testing.assert_allclose(S[0, h], (k[0, h] * w[:, None]).T @ v[0, h], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(z[0, h], (k[0, h] * w[:, None]).sum(0), rtol=1e-11, atol=1e-12)
    assert seen_small and seen_large   # both sides of the max(|.|, 1) are exercised


def test_mlstm_normaliser_homogeneity(orc):
    """Rows with |n^T q| < 1 are divided by 1, so they scale linearly with q;
    rows with |n^T q| > 1 are divided by |n^T q|, so scaling q by c only
    flips their sign with c."""
    rng = np.random.default_rng(105)
    T, d = 40, 4
    q, k, v = (rng.standard_normal((1, 1, T, d)) for _ in range(3))
    f = np.full((1, 1, T), 0.9)
    tiny = 1e-3 * q
    o1, _, z = orc.causal(tiny, k, v, decay=f, mlstm=True)
    o2, _, _ = orc.causal(0.5 * tiny, k, v, decay=f, mlstm=True)
    np.testing.assert_allclose(o2, 0.5 * o1, rtol=1e-12, atol=1e-16)
    big = 1e3 * q
    o3, _, _ = orc.causal(big, k, v, decay=f, mlstm=True)
    o4, _, _ = orc.causal(-2.0 * big, k, v, decay=f, mlstm=True)
    np.testing.assert_allclose(o4, -o3, rtol=1e-12, atol=1e-12)
    # the elu+1 form is a different read-out on the same inputs
    o5, _, _ = orc.causal(big, k, v, decay=f)
    assert np.abs(o5 - o3).max() > 1e-3


def test_mlstm_split_and_decode_handoff(orc):
    rng = np.random.default_rng(107)
    B, H, T1, T2, d, e = 1, 2, 9, 14, 4, 3
    T = T1 + T2
    q, k = (rng.standard_normal((B, H, T + 1, d)) for _ in range(2))
    v = rng.standard_normal((B, H, T + 1, e))
    f = 1.0 / (1.0 + np.exp(-(rng.standard_normal((B, H, T + 1)) + 2.0)))
    i = np.exp(rng.standard_normal((B, H, T + 1)) * 0.5)
    kw = dict(mlstm=True)
    o_full, S_full, z_full = orc.causal(q[:, :, :T], k[:, :, :T], v[:, :, :T], f[:, :, :T], gain=i[:, :, :T], **kw)
    o1, S1, z1 = orc.causal(q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], f[:, :, :T1], gain=i[:, :, :T1], **kw)
    o2, S2, z2 = orc.causal(q[:, :, T1:T], k[:, :, T1:T], v[:, :, T1:T], f[:, :, T1:T], S_in=S1, z_in=z1,
                            gain=i[:, :, T1:T], **kw)
    np.testing.assert_allclose(np.concatenate([o1, o2], 2), o_full, rtol=1e-12, atol=1e-13)
    od, Sd, zd = orc.decode_step(q[:, :, T], k[:, :, T], v[:, :, T], S_full, z_full, decay=f[:, :, T],
                                 gain=i[:, :, T], **kw)
    o_next, S_next, z_next = orc.causal(q, k, v, f, gain=i, **kw)
    np.testing.assert_allclose(od, o_next[:, :, T], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sd, S_next, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ FLASH chunk form
# Concept card, "Chunked attention: exact inside blocks, linear across them
# (FLASH)" and the closing paragraph of its implementation sketch: exact
# squared-ReLU attention inside each chunk, a linear term over the earlier
# chunks' summaries, no normaliser; equations vs listings differ by the
# chunk-length factors, so both are checked.

def _flash_dense(q, k, v, C, scaled):
    """Token-level form of one head: a T x T weight matrix with
    relu(q_t.k_j / s)^2 for j <= t in t's chunk and (q_t.k_j) / s for j in an
    earlier chunk (s = C in the listings' form, 1 in the equations')."""
    T = q.shape[0]
    s = float(C) if scaled else 1.0
    raw = q @ k.T
    ch = np.arange(T) // C
    same = (ch[:, None] == ch[None, :]) & (np.arange(T)[None, :] <= np.arange(T)[:, None])
    earlier = ch[None, :] < ch[:, None]
    W = np.where(same, np.maximum(raw / s, 0.0) ** 2, 0.0) + np.where(earlier, raw / s, 0.0)
    return W @ v


@pytest.mark.parametrize("seed,T,d,C", [(111, 10, 3, 4), (112, 37, 4, 8), (113, 64, 5, 16)])
@pytest.mark.parametrize("scaled", [False, True])
def test_flash_dense_form(orc, seed, T, d, C, scaled):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, 2, T, d)) for _ in range(3))
    out, S = orc.flash(q, k, v, C, scaled=scaled)
    s = float(C) if scaled else 1.0
    for h in range(2):
        np.testing.assert_allclose(out[0, h], _flash_dense(q[0, h], k[0, h], v[0, h], C, scaled),
                                   rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S[0, h], k[0, h].T @ v[0, h] / s, rtol=1e-11, atol=1e-12)


def test_flash_special_chunks(orc):
    rng = np.random.default_rng(115)
    T, d = 20, 4
    q, k, v = (rng.standard_normal((1, 1, T, d)) for _ in range(3))
    # one chunk covering the sequence: causal squared-ReLU attention (torch's relu)
    out, _ = orc.flash(q, k, v, T)
    sc = torch.relu(torch.as_tensor(q[0, 0] @ k[0, 0].T)) ** 2 * torch.tril(torch.ones(T, T, dtype=torch.float64))
    np.testing.assert_allclose(out[0, 0], (sc @ torch.as_tensor(v[0, 0])).numpy(), rtol=1e-12, atol=1e-12)
    # chunk 1: linear attention over the earlier tokens plus relu(q_t.k_t)^2 v_t;
    # both conventions coincide
    o_eq, _ = orc.flash(q, k, v, 1)
    o_ls, _ = orc.flash(q, k, v, 1, scaled=True)
    assert np.array_equal(o_eq, o_ls)
    raw = q[0, 0] @ k[0, 0].T
    ref = np.tril(raw, -1) @ v[0, 0] + (np.maximum(np.diag(raw), 0) ** 2)[:, None] * v[0, 0]
    np.testing.assert_allclose(o_eq[0, 0], ref, rtol=1e-12, atol=1e-12)


def test_flash_causal_and_linear_in_v(orc):
    rng = np.random.default_rng(117)
    T, d, C = 30, 4, 8
    q, k, v = (rng.standard_normal((1, 1, T, d)) for _ in range(3))
    out, _ = orc.flash(q, k, v, C, scaled=True)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[..., 17:, :] += 1.0
    k2[..., 17:, :] -= 2.0
    v2[..., 17:, :] *= 3.0
    out2, _ = orc.flash(q2, k2, v2, C, scaled=True)
    assert np.array_equal(out[..., :17, :], out2[..., :17, :])
    v3 = rng.standard_normal(v.shape)
    o3, _ = orc.flash(q, k, v3, C, scaled=True)
    o4, _ = orc.flash(q, k, 2.0 * v - v3, C, scaled=True)
    np.testing.assert_allclose(o4, 2.0 * out - o3, rtol=1e-11, atol=1e-12)
