"""Pins for the backward oracle (oracle/backward.py), each against something
other than its own formulas:

- torch autograd in fp64 through an explicit softmax (scores, mask, a virtual
  sink key with a zero value, logsumexp), for dense / GQA, MLA (autograd sums the
  shared k_rope over the heads) and sparse top-k (autograd accumulates repeated
  indices);
- central finite differences of the forward C oracle, so the backward is tied to
  the forward's own definition;
- invariants of softmax: without a sink every row's dS sums to zero, so the key
  gradients of a kv head sum to zero, identical keys give dQ = 0, and the value
  gradients sum to the rows' dO;
- the chunked form: gradients of K/V chunks evaluated with the merged forward's O
  and LSE add up to the whole-sequence gradients ("TransformerEngine: FA4 in
  context-parallel attention", its comparison of context-parallel gradients with
  full-sequence attention);
- a planted mistake (the D_i term dropped) that these pins must catch.
"""
import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng


def case(B, H, Hkv, Tq, Tk, D, Dv, seed, sinks):
    r = RNG(seed)
    q = r.standard_normal((B, H, Tq, D))
    k = r.standard_normal((B, Hkv, Tk, D))
    v = r.standard_normal((B, Hkv, Tk, Dv))
    do = r.standard_normal((B, H, Tq, Dv))
    dlse = r.standard_normal((B, H, Tq))
    s = r.standard_normal(H) if sinks else None
    return q, k, v, do, dlse, s


def torch_dense(q, k, v, do, dlse, sinks, scale, causal):
    """Autograd reference: explicit scores and softmax, K/V repeated kv-major, the sink a zero-value key."""
    t = lambda x: torch.tensor(x, dtype=torch.float64, requires_grad=True)
    tq, tk, tv = t(q), t(k), t(v)
    ts = t(sinks) if sinks is not None else None
    B, H, Tq, _ = q.shape
    Tk, Dv = v.shape[2], v.shape[3]
    g = H // k.shape[1]
    kr, vr = tk.repeat_interleave(g, dim=1), tv.repeat_interleave(g, dim=1)
    s = scale * tq @ kr.transpose(-1, -2)
    if causal:
        vis = torch.ones(Tq, Tk, dtype=torch.bool).tril(diagonal=Tk - Tq)
        s = s.masked_fill(~vis, float("-inf"))
    if ts is not None:
        s = torch.cat([s, ts.view(1, H, 1, 1).expand(B, H, Tq, 1)], dim=-1)
        vr = torch.cat([vr, torch.zeros(B, H, 1, Dv, dtype=torch.float64)], dim=-2)
    lse = torch.logsumexp(s, dim=-1)
    o = torch.softmax(s, dim=-1) @ vr
    loss = (o * torch.tensor(do)).sum() + (lse * torch.tensor(dlse)).sum()
    loss.backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), None if ts is None else ts.grad.numpy()


DENSE = [
    # B, H, Hkv, Tq, Tk, D, Dv, causal, sinks
    (1, 4, 1, 7, 9, 8, 8, True, True),      # MQA, bottom-right causal, Tq < Tk, sinks
    (2, 6, 3, 5, 5, 16, 4, True, False),    # GQA g = 2, Dv < D
    (1, 2, 2, 6, 11, 4, 12, False, True),   # no mask, Dv > D
    (1, 4, 2, 9, 4, 8, 8, True, True),      # Tq > Tk: the first rows see only the sink
]


@pytest.mark.parametrize("B,H,Hkv,Tq,Tk,D,Dv,causal,sinks", DENSE)
@pytest.mark.parametrize("with_dlse", [False, True])
def test_dense_bwd_matches_torch_autograd(B, H, Hkv, Tq, Tk, D, Dv, causal, sinks, with_dlse):
    q, k, v, do, dlse, s = case(B, H, Hkv, Tq, Tk, D, Dv, 70 + Tq, sinks)
    dlse = dlse if with_dlse else np.zeros_like(dlse)
    scale = D ** -0.5
    ref = torch_dense(q, k, v, do, dlse, s, scale, causal)
    got = oracle.attn_bwd(q, k, v, do, scale=scale, causal=causal, sinks=s, dlse=dlse if with_dlse else None)
    for name, a, b in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        if b is None:
            assert a is None
            continue
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12, err_msg=name)


def test_rows_without_keys_or_sink_have_no_gradient():
    q, k, v, do, _, _ = case(1, 2, 1, 6, 3, 4, 4, 81, False)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, do, scale=0.5, causal=True)
    assert np.all(dq[:, :, :3] == 0)          # rows 0..2 see no key (Tq - Tk = 3)
    ref = oracle.attn_bwd(q[:, :, 3:], k, v, do[:, :, 3:], scale=0.5, causal=True)
    np.testing.assert_allclose(dk, ref[1], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv, ref[2], rtol=1e-12, atol=1e-14)


def loss_via_forward_oracle(q, k, v, s, do, dlse, scale, causal):
    o, lse = oracle.attn(q, k, v, scale=scale, causal=causal, sinks=s)
    return float((o * do).sum() + (lse * dlse).sum())


def test_directional_derivatives_match_finite_differences_of_the_forward_oracle():
    q, k, v, do, dlse, s = case(1, 4, 2, 6, 8, 8, 4, 90, True)
    scale, causal, eps = 0.4, True, 1e-5
    dq, dk, dv, ds = oracle.attn_bwd(q, k, v, do, scale=scale, causal=causal, sinks=s, dlse=dlse)
    r = RNG(91)
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("s", s, ds)):
        u = r.standard_normal(x.shape)
        args = dict(q=q, k=k, v=v, s=s)
        args[name] = x + eps * u
        up = loss_via_forward_oracle(args["q"], args["k"], args["v"], args["s"], do, dlse, scale, causal)
        args[name] = x - eps * u
        dn = loss_via_forward_oracle(args["q"], args["k"], args["v"], args["s"], do, dlse, scale, causal)
        fd = (up - dn) / (2 * eps)
        assert abs(fd - float((grad * u).sum())) <= 1e-6 * max(1.0, abs(fd)), name


def test_softmax_invariants_without_a_sink():
    q, k, v, do, _, _ = case(2, 8, 2, 10, 10, 16, 8, 92, False)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, do, scale=0.25, causal=True)
    # shifting every key of a kv head by one vector leaves every row's softmax unchanged
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # the weights of a row sum to one, so the value gradients add up to the rows' dO
    np.testing.assert_allclose(dv.sum(axis=2), do.reshape(2, 2, 4, 10, 8).sum(axis=(2, 3)), rtol=1e-12, atol=1e-12)
    # identical keys: S is constant along each row, so Q has no gradient
    k_same = np.broadcast_to(k[:, :, :1], k.shape).copy()
    dq_same = oracle.attn_bwd(q, k_same, v, do, scale=0.25, causal=True)[0]
    np.testing.assert_allclose(dq_same, 0.0, atol=1e-12)


def test_sink_gradient_closed_form():
    """One key and a sink: p_sink = 1 / (1 + e^(s - sink)), O = (1 - p_sink) v, so
    dL/d sink = -p_sink (1 - p_sink) dO.v."""
    q, k, v, do, _, s = case(1, 1, 1, 1, 1, 4, 3, 93, True)
    _, _, _, ds = oracle.attn_bwd(q, k, v, do, scale=1.0, causal=False, sinks=s)
    score = float(q[0, 0, 0] @ k[0, 0, 0])
    ps = 1.0 / (1.0 + np.exp(score - s[0]))
    want = -ps * (1 - ps) * float(do[0, 0, 0] @ v[0, 0, 0])
    assert abs(ds[0] - want) <= 1e-12


@pytest.mark.parametrize("world", [2, 3])
def test_chunked_backward_with_the_merged_forward_equals_the_whole_sequence(world):
    L = 5
    T = world * L
    q, k, v, do, _, s = case(1, 4, 2, T, T, 8, 8, 94 + world, True)
    scale = 8 ** -0.5
    o, lse = oracle.attn(q, k, v, scale=scale, causal=True, sinks=s)
    whole = oracle.attn_bwd(q, k, v, do, scale=scale, causal=True, sinks=s)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dsinks = np.zeros(4)
    for r in range(world):               # query chunk r
        rows = slice(r * L, (r + 1) * L)
        for c in range(r + 1):           # key chunk c: causal within its own chunk, whole below it
            cols = slice(c * L, (c + 1) * L)
            g = oracle.attn_bwd(q[:, :, rows], k[:, :, cols], v[:, :, cols], do[:, :, rows], scale=scale,
                                causal=(c == r), sinks=s, o=o[:, :, rows], lse=lse[:, :, rows])
            dq[:, :, rows] += g[0]
            dk[:, :, cols] += g[1]
            dv[:, :, cols] += g[2]
            if c == r:                   # the sink enters once per row
                dsinks += g[3]
    for a, b in zip((dq, dk, dv, dsinks), whole):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_mla_bwd_matches_torch_autograd_through_the_concat():
    r = RNG(96)
    B, H, T, Dn, Dr, Dv = 2, 3, 7, 8, 4, 6
    qn, qr = r.standard_normal((B, H, T, Dn)), r.standard_normal((B, H, T, Dr))
    kn, kr = r.standard_normal((B, H, T, Dn)), r.standard_normal((B, T, Dr))
    v, do = r.standard_normal((B, H, T, Dv)), r.standard_normal((B, H, T, Dv))
    scale = (Dn + Dr) ** -0.5
    t = lambda x: torch.tensor(x, dtype=torch.float64, requires_grad=True)
    tqn, tqr, tkn, tkr, tv = t(qn), t(qr), t(kn), t(kr), t(v)
    q = torch.cat([tqn, tqr], dim=-1)
    k = torch.cat([tkn, tkr[:, None].expand(B, H, T, Dr)], dim=-1)
    sc = (scale * q @ k.transpose(-1, -2)).masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(), float("-inf"))
    (torch.softmax(sc, dim=-1) @ tv * torch.tensor(do)).sum().backward()
    got = oracle.mla_bwd(qn, qr, kn, kr, v, do, scale=scale, causal=True)
    for a, b in zip(got, (tqn.grad, tqr.grad, tkn.grad, tkr.grad, tv.grad)):
        np.testing.assert_allclose(a, b.numpy(), rtol=1e-10, atol=1e-12)


def sparse_case(Sq, H, Skv, D, Dv, topk, seed, sep_v, sinks):
    r = RNG(seed)
    q = r.standard_normal((Sq, H, D))
    kv = r.standard_normal((Skv, D))
    v = r.standard_normal((Skv, Dv)) if sep_v else None
    idx = r.integers(0, Skv, size=(Sq, topk)).astype(np.int32)      # repeats on purpose
    idx[r.random((Sq, topk)) < 0.2] = -1
    idx[0, 0] = Skv + 3                                              # out of range: masked
    do = r.standard_normal((Sq, H, Dv))
    s = r.standard_normal(H) if sinks else None
    return q, kv, v, idx, do, s


@pytest.mark.parametrize("sep_v,sinks", [(False, True), (True, False)])
def test_sparse_bwd_matches_torch_autograd(sep_v, sinks):
    Sq, H, Skv, D, Dv, topk = 4, 3, 9, 8, 6, 7
    q, kv, v, idx, do, s = sparse_case(Sq, H, Skv, D, Dv, topk, 97, sep_v, sinks)
    scale = D ** -0.5
    t = lambda x: torch.tensor(x, dtype=torch.float64, requires_grad=True)
    tq, tkv = t(q), t(kv)
    tv = t(v) if sep_v else None
    ts = t(s) if sinks else None
    loss = 0
    for i in range(Sq):
        slots = torch.tensor(idx[i][(idx[i] >= 0) & (idx[i] < Skv)], dtype=torch.long)
        k_i = tkv[slots]
        v_i = tv[slots] if sep_v else tkv[slots, :Dv]
        sc = scale * tq[i] @ k_i.T
        if ts is not None:
            sc = torch.cat([sc, ts[:, None]], dim=1)
            v_i = torch.cat([v_i, torch.zeros(1, Dv, dtype=torch.float64)], dim=0)
        loss = loss + (torch.softmax(sc, dim=1) @ v_i * torch.tensor(do[i])).sum()
    loss.backward()
    dq, dkv, dv, ds = oracle.sparse_bwd(q, kv, idx, do, scale=scale, Dv=Dv, v=v, sinks=s)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dkv, tkv.grad.numpy(), rtol=1e-10, atol=1e-12)
    if sep_v:
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)
    if sinks:
        np.testing.assert_allclose(ds, ts.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_sparse_over_all_keys_equals_dense_mqa_backward():
    """Every query listing every pool row (in its own order) is MQA attention without a mask."""
    r = RNG(98)
    Sq, H, Skv, D, Dv = 5, 4, 6, 8, 8
    q, kv, do = r.standard_normal((Sq, H, D)), r.standard_normal((Skv, D)), r.standard_normal((Sq, H, Dv))
    idx = np.stack([r.permutation(Skv) for _ in range(Sq)]).astype(np.int32)
    dq, dkv, _, _ = oracle.sparse_bwd(q, kv, idx, do, scale=0.3, Dv=Dv)
    qd = q.transpose(1, 0, 2)[None]                      # [1, H, Sq, D]
    dqd, dkd, dvd, _ = oracle.attn_bwd(qd, kv[None, None], kv[None, None, :, :Dv], do.transpose(1, 0, 2)[None],
                                       scale=0.3, causal=False)
    np.testing.assert_allclose(dq, dqd[0].transpose(1, 0, 2), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dkv, dkd[0, 0] + dvd[0, 0], rtol=1e-11, atol=1e-12)


def test_mutation_dropped_delta_is_caught(mutation):
    q, k, v, do, dlse, s = case(*DENSE[1][:7], 75, False)
    scale = 16 ** -0.5
    ref = torch_dense(q, k, v, do, np.zeros_like(dlse), None, scale, True)
    mutation(oracle.MUT_BWD_DROP_DELTA)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, do, scale=scale, causal=True)
    assert not np.allclose(dq, ref[0], rtol=1e-6)
    assert not np.allclose(dk.sum(axis=2), 0.0, atol=1e-6)
