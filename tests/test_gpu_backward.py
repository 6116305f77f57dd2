"""The tcgen05 backward (arc_attn_bwd) against the fp64 oracle's derivative.

"TransformerEngine: FA4 in context-parallel attention" (flowchart) runs FA4's
raw backward per chunk, and its comparison script checks the gradients of
context-parallel attention against full-sequence attention.  Here every
gradient of the library's backward -- dQ, dK, dV and the sink gradient -- is
compared element by element with oracle/backward.py, the plain derivative of the
forward definition evaluated in fp64 from the same bf16 inputs.  The GPU side
takes O and LSE from the library's own forward, as a training step would.

Tolerance: the inputs are exact on both sides; the GPU rounds P and dS to bf16
for the tensor cores (relative 2^-9 each), O to bf16 in the forward (which
enters delta = rowsum(dO * O)), and each gradient to bf16 on output (2^-9).
Those roundings are independent from element to element, so their sums stay
well inside 2e-2 of the largest gradient magnitude, which is the bar:
max|gpu - ref| <= 2e-2 * max|ref| per tensor.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import exact_attention_131_b200 as arc
from tests._util import dev, host, status_word

pytestmark = pytest.mark.gpu

TOL_GRAD = 2e-2


def check(name, got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    got = host(got) if torch.is_tensor(got) else np.asarray(got, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    scale = float(np.abs(ref).max())
    assert scale > 0, f"{name}: reference is all zero"
    err = float(np.abs(got - ref).max())
    assert err <= TOL_GRAD * scale, f"{name}: max|d| = {err:.3e} > {TOL_GRAD} * {scale:.3e}"
    return err / scale


def run_case(B, H, Hkv, Tq, Tk, D, Dv, causal, sinks, dlse, seed):
    c = W.dense_case(B, H, Hkv, Tq, Tk, D, Dv, dtype="bf16", std=0.5, causal=causal, sinks=sinks, seed=seed)
    up = W.upstream(B, H, Tq, Dv, dlse=dlse, seed=seed + 1000)
    q, k, v = dev(c.q), dev(c.k), dev(c.v)
    s = dev(c.sinks) if sinks else None
    o, lse = arc.attn_fwd(q, k, v, scale=c.scale, causal=causal, sinks=s)
    do = dev(up.do)
    dl = dev(up.dlse) if dlse else None
    st = status_word()
    dq, dk, dv, ds = arc.attn_bwd(q, k, v, o, lse, do, scale=c.scale, causal=causal, sinks=s, dlse=dl, status=st)
    torch.cuda.synchronize()
    assert arc.check_device_error(st) == arc.ARC_OK
    rq, rk, rv, rs = oracle.attn_bwd(c.q, c.k, c.v, up.do, scale=c.scale, causal=causal, sinks=c.sinks,
                                     dlse=up.dlse)
    return c, (dq, dk, dv, ds), (rq, rk, rv, rs), (q, k, v, o, lse, do, s)


@pytest.mark.parametrize("B,H,Hkv,Tq,Tk,D,Dv,causal,sinks,dlse", [
    (1, 8, 2, 300, 300, 128, 128, True, True, False),    # GQA-4 with sinks, ragged tiles
    (2, 4, 4, 200, 200, 64, 64, True, False, True),      # MHA, upstream dLSE
    (1, 4, 1, 150, 260, 128, 128, True, False, False),   # MQA, Tq < Tk: bottom-right causal
    (1, 4, 2, 200, 100, 64, 64, True, True, False),      # Tq > Tk: the first rows see only the sink
    (1, 2, 2, 257, 257, 192, 128, False, True, True),    # d_qk 192, d_v 128 (64-row dK/dV tiles), non-causal
    (2, 6, 3, 160, 160, 192, 128, True, False, False),   # d_qk 192 causal, GQA-2
])
def test_backward_matches_oracle(B, H, Hkv, Tq, Tk, D, Dv, causal, sinks, dlse):
    c, got, ref, t = run_case(B, H, Hkv, Tq, Tk, D, Dv, causal, sinks, dlse, seed=400 + D + Tq)
    q, k, v, o, lse, do, s = t
    info = arc.plan_attn_bwd(q, k, v, o, lse, do, causal=causal, sinks=s)
    assert info["kernel"] == "bwd_dkdv_kernel+bwd_dq_kernel" and info["tensor_cores"] == 1
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        check(name, g, r)
    if sinks:
        check("dsinks", got[3], ref[3])


def test_backward_row_split_dk_dv_and_bit_identical_repeats():
    """Few key tiles: the dK/dV work of each key tile is split over CTAs along the fold
    rows and reduced; a second call gives the same bits."""
    c, got, ref, t = run_case(1, 16, 2, 260, 260, 128, 128, True, True, False, seed=451)
    q, k, v, o, lse, do, s = t
    info = arc.plan_attn_bwd(q, k, v, o, lse, do, causal=True, sinks=s)
    assert info["splits"] > 1
    for name, g, r in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        check(name, g, r)
    again = arc.attn_bwd(q, k, v, o, lse, do, scale=c.scale, causal=True, sinks=s)
    torch.cuda.synchronize()
    for a, b in zip(got, again):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


def test_backward_c2_shape_gqa8_with_sinks_at_d128():
    """The GQA prefill's structure (64 query heads over 8 kv heads, causal, sinks) at
    head dim 128 and 1400 positions."""
    c, got, ref, _ = run_case(1, 64, 8, 1400, 1400, 128, 128, True, True, False, seed=452)
    for name, g, r in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        check(name, g, r)


def test_backward_mla_shaped_head_dims():
    """d_qk 192 / d_v 128 (the MLA prefill's head dims, on concatenated q/k) at B=2, H=4, T=1024."""
    c, got, ref, _ = run_case(2, 4, 4, 1024, 1024, 192, 128, True, False, False, seed=453)
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        check(name, g, r)


@pytest.mark.parametrize("B,H,T,Dn,Dr,Dv,causal,dlse", [
    (1, 3, 300, 128, 64, 128, True, False),     # the MLA prefill's head dims, ragged tiles
    (2, 2, 200, 64, 64, 128, False, True),      # d_qk 128, non-causal, upstream dLSE
    (1, 4, 260, 128, 64, 128, True, False),     # four heads summed into dk_rope
])
def test_mla_backward_matches_oracle(B, H, T, Dn, Dr, Dv, causal, dlse):
    """arc_mla_bwd: gradients through the q_nope||q_rope and k_nope||k_rope concatenation,
    dk_rope summed over the heads that share it, against oracle/backward.py's mla_bwd."""
    c = W.mla_case(B, H, T, T, Dn, Dr, Dv, causal=causal, seed=470 + T)
    up = W.upstream(B, H, T, Dv, dlse=dlse, seed=471 + T)
    t = [dev(x) for x in (c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v)]
    o, lse = arc.mla_fwd(*t, scale=c.scale, causal=causal)
    do = dev(up.do)
    dl = dev(up.dlse) if dlse else None
    st = status_word()
    got = arc.mla_bwd(*t, o, lse, do, scale=c.scale, causal=causal, dlse=dl, status=st)
    torch.cuda.synchronize()
    assert arc.check_device_error(st) == arc.ARC_OK
    info = arc.plan_mla_bwd(*t, o, lse, do, causal=causal)
    assert info["kernel"] == "bwd_dkdv_kernel<mla>+bwd_dq_kernel" and info["tensor_cores"] == 1
    ref = oracle.mla_bwd(c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v, up.do, scale=c.scale, causal=causal,
                         dlse=up.dlse)
    for name, g, r in zip(("dq_nope", "dq_rope", "dk_nope", "dk_rope", "dv"), got, ref):
        check(name, g, r)
