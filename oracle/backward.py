"""fp64 CPU oracle for the attention backward pass -- TEST INFRASTRUCTURE ONLY.

Like the rest of ``oracle/``, only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the CUDA library shares
no code with it.

What it computes is the derivative of the forward definition in this package.
"TransformerEngine: FA4 in context-parallel attention" (flowchart) runs FA4's raw
backward per K/V chunk to get the Q/K/V gradients, and its comparison script
checks context-parallel gradients against full-sequence attention.  "pith-train:
FA4 b19 return arity and MLA q/k concat" feeds the q/k concatenation to the
attention call inside the model, so MLA gradients reach q_nope, q_rope, k_nope and
the shared k_rope through that concatenation.  The pages print no formula for the
backward, so the oracle is the plain derivative, written out per (batch, head).
For a loss with upstream gradients dO (and optionally dLSE):

    S = scale * Q K^T (masked entries -inf),  P = exp(S - LSE),  p_sink = exp(sink - LSE)
    dV  = P^T dO                      dP = dO V^T
    D_i = sum_d dO_id O_id            dS = P * (dP - D_i [+ dLSE_i])
    dQ  = scale * dS K                dK = scale * dS^T Q
    d sink_h = sum_i p_sink_i * (dLSE_i - D_i)

The sink is a key with a zero value, so it adds nothing to dP. GQA sums dK and dV
over the g query heads that read a kv head (kv-major: head h reads kv head h // g).
A row with no visible key and no sink has O = 0 and LSE = -inf, and no gradient.
Passing ``o`` and ``lse`` evaluates P and D from them rather than from the row's
own keys. This is the form that a chunked (ring) backward takes: each chunk uses
the merged forward's O and LSE.

Matrix products are numpy's; there is no blocking and no reordering beyond the
definition.  Pins: tests/test_oracle_backward_pins.py.
"""
from __future__ import annotations

import numpy as np


def _widen(x):
    from . import widen
    return widen(x)


def _mutation():
    from . import _load
    return int(_load().oracle_get_mutation())


def _visible(Tq, Tk, causal):
    """[Tq, Tk] visibility: bottom-right causal (key j <= i + Tk - Tq) or all."""
    if not causal:
        return np.ones((Tq, Tk), dtype=bool)
    return np.arange(Tk)[None, :] <= np.arange(Tq)[:, None] + (Tk - Tq)


def _row_softmax(s, sink):
    """P over the row's keys, the sink's share, and the LSE; rows with nothing visible give zeros / -inf."""
    m = np.maximum(s.max(axis=1, initial=-np.inf), sink)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe[:, None])
    es = np.exp(sink - m_safe)
    total = e.sum(axis=1) + es
    total_safe = np.where(empty, 1.0, total)
    p = np.where(empty[:, None], 0.0, e / total_safe[:, None])
    ps = np.where(empty, 0.0, es / total_safe)
    lse = np.where(empty, -np.inf, m_safe + np.log(total_safe))
    return p, ps, lse


def _head_bwd(q, k, v, do, vis, scale, sink, dlse, o_in, lse_in):
    """Gradients for one (batch, query head) against one K/V set.  Returns dq, dk, dv, dsink."""
    s = scale * (q @ k.T)
    s = np.where(vis, s, -np.inf)
    if lse_in is None:
        p, ps, _ = _row_softmax(s, sink)
        o = p @ v
    else:
        live = ~np.isneginf(lse_in)
        lse_safe = np.where(live, lse_in, 0.0)
        p = np.where(live[:, None], np.exp(s - lse_safe[:, None]), 0.0)
        ps = np.where(live, np.exp(sink - lse_safe), 0.0)
        o = o_in
    delta = (do * o).sum(axis=1)
    if _mutation() == MUT_BWD_DROP_DELTA:
        delta = np.zeros_like(delta)
    dp = do @ v.T
    g = dp - delta[:, None]
    if dlse is not None:
        g = g + dlse[:, None]
    ds = p * g
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    dv = p.T @ do
    dsink = float(np.sum(ps * ((dlse if dlse is not None else 0.0) - delta)))
    return dq, dk, dv, dsink


# a planted mistake for the pins to catch: the D_i term dropped from dS
MUT_BWD_DROP_DELTA = 7


def attn_bwd(q, k, v, do, *, scale, causal=True, sinks=None, dlse=None, o=None, lse=None):
    """Gradients of dense / GQA attention.

    q [B,H,Tq,D], k [B,Hkv,Tk,D], v [B,Hkv,Tk,Dv], do [B,H,Tq,Dv]; sinks [H] or None;
    dlse [B,H,Tq] or None.  o [B,H,Tq,Dv] and lse [B,H,Tq], if given, replace the
    forward's own (the chunked form).  Returns dq, dk, dv and dsinks ([H], or None).
    """
    q, k, v, do = _widen(q), _widen(k), _widen(v), _widen(do)
    B, H, Tq, D = q.shape
    _, Hkv, Tk, Dv = v.shape
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    g = H // Hkv
    vis = _visible(Tq, Tk, causal)
    sk = None if sinks is None else _widen(sinks)
    dlse = None if dlse is None else _widen(dlse)
    o = None if o is None else _widen(o)
    lse = None if lse is None else _widen(lse)
    if (o is None) != (lse is None):
        raise ValueError("o and lse are given together")
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dsinks = None if sinks is None else np.zeros(H)
    for b in range(B):
        for h in range(H):
            kv = h // g
            sink = -np.inf if sk is None else sk[h]
            r = _head_bwd(q[b, h], k[b, kv], v[b, kv], do[b, h], vis, scale, sink,
                          None if dlse is None else dlse[b, h],
                          None if o is None else o[b, h],
                          None if lse is None else lse[b, h])
            dq[b, h] = r[0]
            dk[b, kv] += r[1]
            dv[b, kv] += r[2]
            if dsinks is not None:
                dsinks[h] += r[3]
    return dq, dk, dv, dsinks


def mla_bwd(q_nope, q_rope, k_nope, k_rope, v, do, *, scale, causal=True, dlse=None):
    """Gradients of MLA attention (q = q_nope||q_rope, k = k_nope[h]||k_rope shared by all heads).

    Returns dq_nope [B,H,Tq,Dn], dq_rope [B,H,Tq,Dr], dk_nope [B,H,Tk,Dn],
    dk_rope [B,Tk,Dr] (summed over the heads that share it), dv [B,H,Tk,Dv].
    """
    qn, qr, kn, kr = _widen(q_nope), _widen(q_rope), _widen(k_nope), _widen(k_rope)
    Dn = qn.shape[-1]
    H = qn.shape[1]
    q = np.concatenate([qn, qr], axis=-1)
    k = np.concatenate([kn, np.repeat(kr[:, None], H, axis=1)], axis=-1)
    dq, dk, dv, _ = attn_bwd(q, k, v, do, scale=scale, causal=causal, dlse=dlse)
    return dq[..., :Dn], dq[..., Dn:], dk[..., :Dn], dk[..., Dn:].sum(axis=1), dv


def sparse_bwd(q, kv, idx, do, *, scale, Dv=None, v=None, sinks=None, dlse=None):
    """Gradients of sparse top-k attention.

    q [Sq,H,Dqk], kv [Skv,Dqk], idx [Sq,topk] int32 (slots outside [0, Skv) are
    masked; a repeated index counts once per slot), do [Sq,H,Dv].  V is kv[:, :Dv]
    unless a separate v [Skv,Dv] is given.  Returns dq, dkv (which also carries the
    V gradient when V is part of the kv row), dv (None unless v is given) and dsinks.
    """
    q, kv, do = _widen(q), _widen(kv), _widen(do)
    Sq, H, Dqk = q.shape
    Skv = kv.shape[0]
    vv = None if v is None else _widen(v)
    Dv = vv.shape[1] if vv is not None else (Dqk if Dv is None else Dv)
    sk = None if sinks is None else _widen(sinks)
    dlse = None if dlse is None else _widen(dlse)
    dq = np.zeros_like(q)
    dkv = np.zeros_like(kv)
    dv = None if vv is None else np.zeros_like(vv)
    dsinks = None if sinks is None else np.zeros(H)
    idx = np.asarray(idx)
    for i in range(Sq):
        slots = idx[i][(idx[i] >= 0) & (idx[i] < Skv)]
        k_i = kv[slots]
        v_i = vv[slots] if vv is not None else kv[slots, :Dv]
        vis = np.ones((1, len(slots)), dtype=bool)
        for h in range(H):
            sink = -np.inf if sk is None else sk[h]
            r = _head_bwd(q[i, h][None], k_i, v_i, do[i, h][None], vis, scale, sink,
                          None if dlse is None else dlse[i, h][None], None, None)
            dq[i, h] = r[0][0]
            np.add.at(dkv, slots, r[1])
            if vv is not None:
                np.add.at(dv, slots, r[2])
            else:
                np.add.at(dkv[:, :Dv], slots, r[2])
            if dsinks is not None:
                dsinks[h] += r[3]
    return dq, dkv, dv, dsinks
