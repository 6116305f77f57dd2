"""Every tensor-core instantiation the C ABI advertises, against the fp64 oracle.

include/arc_attn.h lists the (d_qk, d_v) pairs each call runs on tensor cores.
Each pair is a separate template instantiation (another tile count, another d_v
slicing), so each gets its own element-by-element comparison here, with the
kernel that ran asserted through arc_plan: the engagement record of "ArcFlash -
Arc's own attention kernel, rung 0" (section D18) and the review note of
"unsloth llama.cpp: dequantize q4_0/q8_0 K/V tiles in the FA MMA kernel" that
equal numbers do not show which path ran.  Sizes span several query tiles and
key tiles with ragged tails.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import exact_attention_131_b200 as arc
from tests._util import TOL_O_BF16, compare, dev, status_word

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ dense

# (D, Dv) -> the kernel arc_plan must name (default flags)
DENSE = {
    (64, 64): "tc_attn2_kernel",
    (128, 64): "tc_attn2_kernel",
    (128, 128): "tc_attn_pair_kernel",
    (192, 128): "tc_attn_pair_kernel",
    (256, 128): "tc_attn_pair_kernel",
    (256, 256): "tc_attn_pair_kernel",
    (256, 512): "tc_attn_pair_kernel",     # two 256-wide d_v slices
    (512, 128): "tc_attn_kernel",
    (512, 256): "tc_attn_pair_kernel",
    (512, 512): "tc_attn_pair_kernel",
}


@pytest.mark.parametrize("D,Dv", sorted(DENSE), ids=[f"d{d}-dv{v}" for d, v in sorted(DENSE)])
def test_dense_every_listed_head_dim_pair(D, Dv):
    c = W.dense_case(1, 8, 2, 203, 203, D, Dv, dtype="bf16", std=0.5, causal=True, sinks=True,
                     seed=200 + D + Dv)
    q, k, v, s = dev(c.q), dev(c.k), dev(c.v), dev(c.sinks)
    st = status_word()
    o, lse = arc.attn_fwd(q, k, v, scale=c.scale, causal=True, sinks=s, status=st)
    torch.cuda.synchronize()
    info = arc.plan_attn(q, k, v, o, lse, causal=True, sinks=s)
    assert info["kernel"] == DENSE[(D, Dv)] and info["tensor_cores"] == 1
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


def test_dense_default_scale_is_one_over_root_d():
    """scale=None sets ARC_FLAG_DEFAULT_SCALE: the library resolves 1/sqrt(D) itself,
    and the result is bit-identical to passing that scale explicitly."""
    c = W.dense_case(1, 8, 2, 150, 150, 128, dtype="bf16", std=0.5, sinks=True, seed=211)
    q, k, v, s = dev(c.q), dev(c.k), dev(c.v), dev(c.sinks)
    o1, l1 = arc.attn_fwd(q, k, v, sinks=s)
    o2, l2 = arc.attn_fwd(q, k, v, scale=float(np.float32(1.0 / np.sqrt(128.0))), sinks=s)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)
    ro, rl = oracle.run_case(c)
    compare(o1, l1, ro, rl, TOL_O_BF16)


# ------------------------------------------------------------------ MLA

MLA = {
    (64, 64, 128): "tc_attn2_kernel<mla>",     # d_qk 128
    (128, 64, 64): "tc_attn2_kernel<mla>",     # d_qk 192
    (128, 64, 128): "tc_attn_pair_kernel<mla>",
    (192, 64, 128): "tc_attn2_kernel<mla>",    # d_qk 256
    (128, 128, 128): "tc_attn2_kernel<mla>",   # d_qk 256, rope 128
    (192, 64, 256): "tc_attn_kernel<mla>",     # d_qk 256, d_v 256
}


@pytest.mark.parametrize("Dn,Dr,Dv", sorted(MLA), ids=[f"n{a}-r{b}-dv{c}" for a, b, c in sorted(MLA)])
def test_mla_every_listed_head_dim_pair(Dn, Dr, Dv):
    c = W.mla_case(2, 2, 270, 270, Dn, Dr, Dv, seed=220 + Dn + Dr + Dv)
    t = [dev(x) for x in (c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v)]
    st = status_word()
    o, lse = arc.mla_fwd(*t, scale=c.scale, causal=True, status=st)
    torch.cuda.synchronize()
    info = arc.plan_mla(*t, o, lse)
    assert info["kernel"] == MLA[(Dn, Dr, Dv)] and info["tensor_cores"] == 1
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


def test_mla_default_scale_is_one_over_root_dqk():
    c = W.mla_case(1, 2, 140, 140, 128, 64, 128, seed=229)
    t = [dev(x) for x in (c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v)]
    o, lse = arc.mla_fwd(*t)
    torch.cuda.synchronize()
    ro, rl = oracle.run_case(c)          # the case's scale is 1/sqrt(192)
    compare(o, lse, ro, rl, TOL_O_BF16)


# ------------------------------------------------------------------ sparse

# (Dqk, Dv, separate v)
SPARSE = [(512, 512, False), (512, 256, False), (256, 256, False), (128, 128, False),
          (128, 64, True), (128, 128, True), (256, 256, True)]


@pytest.mark.parametrize("Dqk,Dv,sep_v", SPARSE, ids=[f"d{a}-dv{b}-{'sepv' if s else 'row'}" for a, b, s in SPARSE])
def test_sparse_every_listed_head_dim_pair(Dqk, Dv, sep_v):
    c = W.sparse_case(11, 64, 1500, Dqk, Dv, 203, pad_mode="random", separate_v=sep_v, seed=240 + Dqk + Dv)
    q, kv, idx = dev(c.q), dev(c.kv), dev(c.idx)
    v = dev(c.v) if sep_v else None
    st = status_word()
    o, lse = arc.sparse_mla_fwd(q, kv, idx, Dv=Dv, v=v, scale=c.scale, status=st)
    torch.cuda.synchronize()
    info = arc.plan_sparse(q, kv, idx, o, lse, Dv=Dv, v=v)
    assert info["kernel"] == "sparse_tc_kernel" and info["tensor_cores"] == 1
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


@pytest.mark.parametrize("Dqk,Dv,sep_v", [(512, 512, False), (128, 64, True)])
def test_sparse_invalid_slots_read_no_pool_row(Dqk, Dv, sep_v):
    """The kernel gathers rows four slots at a time.  Invalid slots (-1, negative,
    Skv and beyond) are placed as whole tiles, whole groups of four, one to three
    slots of a group, every other slot, and a ragged last tile; every pool row that
    no valid slot names holds NaN.  An invalid slot adds nothing, so the output must
    be finite and equal the oracle's, which never reads such a row."""
    c = W.sparse_case(8, 64, 3000, Dqk, Dv, 203, pad_frac=0.0, separate_v=sep_v, seed=262)
    bad = np.array([-1, -5, c.Skv, c.Skv + 77, 2**31 - 1], dtype=np.int64)
    rng = np.random.default_rng(263)
    slots = np.arange(c.topk)
    patterns = [
        slots < 64,                                  # a whole tile
        (slots // 4) % 3 == 1,                       # whole groups of four
        slots % 4 == 1,                              # one slot of each group
        slots % 4 != 0,                              # three slots of each group
        slots % 2 == 0,                              # every other slot
        slots >= 192,                                # the ragged last tile
        rng.random(c.topk) < 0.5,
        np.ones(c.topk, dtype=bool),                 # no valid slot at all
    ]
    for t, m in enumerate(patterns):
        c.idx[t, m] = rng.choice(bad, size=int(m.sum())).astype(np.int32)
    valid = c.idx[(c.idx >= 0) & (c.idx < c.Skv)]
    unnamed = np.setdiff1d(np.arange(c.Skv), valid)
    assert unnamed.size > 0
    nan = np.uint16(0x7FC0)
    c.kv[unnamed] = nan
    if sep_v:
        c.v[unnamed] = nan
    q, kv, idx = dev(c.q), dev(c.kv), dev(c.idx)
    v = dev(c.v) if sep_v else None
    st = status_word()
    o, lse = arc.sparse_mla_fwd(q, kv, idx, Dv=Dv, v=v, scale=c.scale, status=st)
    torch.cuda.synchronize()
    assert arc.plan_sparse(q, kv, idx, o, lse, Dv=Dv, v=v)["kernel"] == "sparse_tc_kernel"
    assert bool(torch.isfinite(o).all())
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert float(o[7].abs().max()) == 0.0
    assert arc.check_device_error(st) == arc.ARC_OK


@pytest.mark.parametrize("Dqk,Dv", [(512, 512), (128, 64)])
def test_sparse_sinks_and_a_row_with_no_valid_slot(Dqk, Dv):
    """Sinks in the sparse kernel's epilogue (sink max, rescale, the sink in the
    denominator only), -1 padding, and one query whose every slot is invalid: its
    output is 0 and its LSE the sink."""
    c = W.sparse_case(9, 16, 700, Dqk, Dv, 130, pad_mode="random", separate_v=Dv != Dqk, sinks=True, seed=251)
    c.idx[4, :] = -1
    q, kv, idx, s = dev(c.q), dev(c.kv), dev(c.idx), dev(c.sinks)
    v = dev(c.v) if c.v is not None else None
    st = status_word()
    o, lse = arc.sparse_mla_fwd(q, kv, idx, Dv=Dv, v=v, scale=c.scale, sinks=s, status=st)
    torch.cuda.synchronize()
    assert arc.plan_sparse(q, kv, idx, o, lse, Dv=Dv, v=v, sinks=s)["kernel"] == "sparse_tc_kernel"
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert float(o[4].abs().max()) == 0.0
    assert np.allclose(lse[4].cpu().numpy(), c.sinks, atol=1e-6)
    assert arc.check_device_error(st) == arc.ARC_OK
