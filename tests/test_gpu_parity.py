"""CUDA path vs the fp64 CPU oracle, element by element, through the C ABI.

Small cases span several query-row tiles, several KV tiles and ragged tails;
full-size cases (the five workload configurations) compare sampled rows that
the oracle evaluates one by one, in the launch configuration bench.py times.
Engagement is asserted separately: arc_plan names the tensor-core kernel for
every bf16 case and the CUDA-core kernel only under ARC_FLAG_FORCE_SIMPLE.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import exact_attention_131_b200 as arc
from tests._util import TOL_LSE, TOL_O_BF16, TOL_O_F32, compare, dev, status_word

pytestmark = pytest.mark.gpu


def run_dense(c, flags=0, status=None):
    q, k, v = dev(c.q), dev(c.k), dev(c.v)
    s = dev(c.sinks) if c.sinks is not None else None
    o, lse = arc.attn_fwd(q, k, v, scale=c.scale, causal=c.causal, sinks=s, flags=flags, status=status)
    torch.cuda.synchronize()
    return o, lse, (q, k, v, s)


# ------------------------------------------------------------------ dense / GQA

def test_config1_fp32_reference_mode():
    c = W.config(1)
    o, lse, _ = run_dense(c)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_F32)


@pytest.mark.parametrize("B,H,Hkv,Tq,Tk,D,Dv,causal,sinks", [
    (1, 8, 2, 300, 300, 128, 128, True, False),     # ragged fold rows and KV tail
    (2, 4, 4, 129, 129, 64, 64, True, True),        # one row past a tile
    (1, 16, 2, 200, 200, 512, 512, True, True),     # d=512 with sinks: two d_v slices
    (1, 8, 1, 100, 260, 256, 256, True, False),     # Tq < Tk: bottom-right causal
    (1, 4, 2, 77, 333, 128, 64, False, True),       # non-causal, Dv < D
    (1, 6, 3, 64, 40, 192, 128, True, False),       # Tq > Tk: first rows see nothing
])
def test_dense_bf16_small(B, H, Hkv, Tq, Tk, D, Dv, causal, sinks):
    c = W.dense_case(B, H, Hkv, Tq, Tk, D, Dv, dtype="bf16", std=0.5, causal=causal, sinks=sinks, seed=31)
    st = status_word()
    o, lse, (q, k, v, s) = run_dense(c, status=st)
    info = arc.plan_attn(q, k, v, o, lse, causal=causal, sinks=s)
    assert info["kernel"] == expected_dense_kernel(D, Dv) and info["tensor_cores"] == 1
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


def expected_dense_kernel(D, Dv):
    # a CTA pair (M = 256) for d_qk 128-256 with d_v 128 and for d_qk 256 / 512 with a
    # 256-wide d_v slice; other d_v <= 128: two query tiles per CTA; else one tile per slice
    if (D, Dv) in ((128, 128), (192, 128), (256, 128)):
        return "tc_attn_pair_kernel"
    if Dv <= 128:
        return "tc_attn2_kernel"
    if D in (256, 512) and Dv in (256, 512):
        return "tc_attn_pair_kernel"
    return "tc_attn_kernel"


@pytest.mark.parametrize("B,H,Hkv,Tq,Tk,D,causal,sinks", [
    (1, 16, 2, 200, 200, 512, True, True),     # odd tile count: the last pair's second CTA has no rows
    (2, 8, 1, 190, 450, 256, True, False),      # Tq < Tk, two batches
    (1, 4, 4, 300, 300, 512, False, True),      # non-causal, G = 1
])
def test_dense_pair_and_single_cta_agree_with_oracle(B, H, Hkv, Tq, Tk, D, causal, sinks):
    c = W.dense_case(B, H, Hkv, Tq, Tk, D, D, dtype="bf16", std=0.5, causal=causal, sinks=sinks, seed=34)
    ro, rl = oracle.run_case(c)
    for flags, name in ((0, "tc_attn_pair_kernel"), (arc.ARC_FLAG_SINGLE_CTA, "tc_attn_kernel")):
        st = status_word()
        o, lse, (q, k, v, s) = run_dense(c, flags=flags, status=st)
        info = arc.plan_attn(q, k, v, o, lse, causal=causal, sinks=s, flags=flags)
        assert info["kernel"] == name
        compare(o, lse, ro, rl, TOL_O_BF16)
        assert arc.check_device_error(st) == arc.ARC_OK


@pytest.mark.parametrize("B,H,Hkv,Tq,Tk,D,causal,sinks", [
    (1, 8, 2, 300, 300, 128, True, True),      # G = 4: t-major fold
    (2, 6, 3, 260, 400, 192, True, False),     # Tq < Tk, 3 row tiles: last pair half empty
    (1, 4, 4, 200, 200, 256, False, True),     # non-causal, G = 1
])
def test_dense_small_d_pair_and_two_tile_agree_with_oracle(B, H, Hkv, Tq, Tk, D, causal, sinks):
    c = W.dense_case(B, H, Hkv, Tq, Tk, D, 128, dtype="bf16", std=0.5, causal=causal, sinks=sinks, seed=35)
    ro, rl = oracle.run_case(c)
    for flags, name in ((0, "tc_attn_pair_kernel"), (arc.ARC_FLAG_SINGLE_CTA, "tc_attn2_kernel")):
        st = status_word()
        o, lse, (q, k, v, s) = run_dense(c, flags=flags, status=st)
        info = arc.plan_attn(q, k, v, o, lse, causal=causal, sinks=s, flags=flags)
        assert info["kernel"] == name
        compare(o, lse, ro, rl, TOL_O_BF16)
        assert arc.check_device_error(st) == arc.ARC_OK


def test_dense_control_arm_runs_the_simple_kernel():
    c = W.dense_case(1, 8, 2, 150, 150, 128, dtype="bf16", std=0.5, sinks=True, seed=32)
    o, lse, (q, k, v, s) = run_dense(c, flags=arc.ARC_FLAG_FORCE_SIMPLE)
    info = arc.plan_attn(q, k, v, o, lse, sinks=s, flags=arc.ARC_FLAG_FORCE_SIMPLE)
    assert info["kernel"] == "simple_attn_kernel" and info["tensor_cores"] == 0
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)


def sample_rows(T, n, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(T, size=n - 4, replace=False).tolist()) | {0, 1, T - 2, T - 1}
    return np.array(sorted(rows), dtype=np.int32)


def test_config2_gqa_sinks_full_size_sampled_rows():
    c = W.config(2)
    st = status_word()
    o, lse, (q, k, v, s) = run_dense(c, status=st)
    info = arc.plan_attn(q, k, v, o, lse, sinks=s)
    assert info["kernel"] == "tc_attn_pair_kernel" and info["d_slice"] == 256 and info["tile_m"] == 256
    rows = sample_rows(c.Tq, 40, 2)
    ro, rl = oracle.run_case(c, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


# ------------------------------------------------------------------ MLA

def run_mla(c, flags=0, status=None):
    t = [dev(x) for x in (c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v)]
    o, lse = arc.mla_fwd(*t, scale=c.scale, causal=c.causal, flags=flags, status=status)
    torch.cuda.synchronize()
    return o, lse, t


@pytest.mark.parametrize("B,H,T,Dn,Dr,Dv", [(1, 3, 300, 128, 64, 128), (2, 2, 130, 128, 64, 64),
                                             (1, 2, 257, 64, 64, 128)])
def test_mla_small(B, H, T, Dn, Dr, Dv):
    c = W.mla_case(B, H, T, T, Dn, Dr, Dv, seed=33)
    st = status_word()
    o, lse, t = run_mla(c, status=st)
    info = arc.plan_mla(*t, o, lse)
    # d_qk 128 + 64 with d_v 128 runs on a CTA pair (M = 256); other shapes on two tiles per CTA
    assert info["kernel"] == ("tc_attn_pair_kernel<mla>" if (Dn + Dr, Dv) == (192, 128) else "tc_attn2_kernel<mla>")
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


@pytest.mark.parametrize("B,H,T,causal", [(1, 2, 700, True),    # 3 row tiles: the last pair's second CTA is empty
                                          (2, 3, 520, False),
                                          (1, 1, 1000, True)])
def test_mla_pair_and_two_tile_agree_with_oracle(B, H, T, causal):
    c = W.mla_case(B, H, T, T, 128, 64, 128, causal=causal, seed=34)
    ro, rl = oracle.run_case(c)
    for flags, name in ((0, "tc_attn_pair_kernel<mla>"), (arc.ARC_FLAG_SINGLE_CTA, "tc_attn2_kernel<mla>")):
        st = status_word()
        o, lse, t = run_mla(c, flags=flags, status=st)
        assert arc.plan_mla(*t, o, lse, causal=causal, flags=flags)["kernel"] == name
        compare(o, lse, ro, rl, TOL_O_BF16)
        assert arc.check_device_error(st) == arc.ARC_OK


def test_config3_mla_full_size_sampled_rows():
    c = W.config(3)
    o, lse, t = run_mla(c)
    assert arc.plan_mla(*t, o, lse)["kernel"] == "tc_attn_pair_kernel<mla>"
    rows = sample_rows(c.Tq, 24, 3)
    ro, rl = oracle.run_case(c, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], ro, rl, TOL_O_BF16)


# ------------------------------------------------------------------ sparse

def run_sparse(c, flags=0, status=None):
    q, kv, idx = dev(c.q), dev(c.kv), dev(c.idx)
    v = dev(c.v) if c.v is not None else None
    o, lse = arc.sparse_mla_fwd(q, kv, idx, Dv=c.Dv, v=v, scale=c.scale, flags=flags, status=status)
    torch.cuda.synchronize()
    return o, lse, (q, kv, idx, v)


@pytest.mark.parametrize("Sq,H,Skv,D,Dv,topk,pad_mode,sep_v", [
    (37, 64, 5000, 512, 512, 300, "random", False),
    (20, 64, 3000, 512, 512, 250, "tail", False),
    (9, 16, 700, 128, 64, 130, "random", True),
])
def test_sparse_small(Sq, H, Skv, D, Dv, topk, pad_mode, sep_v):
    c = W.sparse_case(Sq, H, Skv, D, Dv, topk, pad_mode=pad_mode, separate_v=sep_v, seed=34)
    st = status_word()
    o, lse, (q, kv, idx, v) = run_sparse(c, status=st)
    info = arc.plan_sparse(q, kv, idx, o, lse, Dv=Dv, v=v)
    assert info["kernel"] == "sparse_tc_kernel" and info["tensor_cores"] == 1
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


def test_sparse_more_than_64_heads_and_control_arm():
    c = W.sparse_case(7, 96, 900, 256, 256, 200, seed=43)
    o, lse, (q, kv, idx, v) = run_sparse(c)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    o2, lse2, _ = run_sparse(c, flags=arc.ARC_FLAG_FORCE_SIMPLE)
    assert arc.plan_sparse(q, kv, idx, o2, lse2, flags=arc.ARC_FLAG_FORCE_SIMPLE)["kernel"] == \
        "simple_attn_kernel<sparse>"
    compare(o2, lse2, ro, rl, TOL_O_BF16)


def test_config4_sparse_full_size_sampled_queries():
    c = W.config(4)
    o, lse, _ = run_sparse(c)
    rows = sample_rows(c.Sq, 24, 4)
    ro, rl = oracle.run_case(c, rows=rows)
    compare(o[rows], lse[rows], ro, rl, TOL_O_BF16)


# ------------------------------------------------------------------ decode

def run_decode(c, flags=0, status=None):
    q, kc, vc = dev(c.q), dev(c.k_cache), dev(c.v_cache)
    o, lse = arc.attn_decode_q8(q, kc, vc, kv_type=c.kv_type, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q,
                                kv_begin=c.kv_begin, n_kv=c.n_kv, scale=c.scale, flags=flags, status=status)
    torch.cuda.synchronize()
    return o, lse, (q, kc, vc)


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
def test_config5_decode_full(kv_type):
    c = W.config(5, kv_type=kv_type)
    st = status_word()
    o, lse, (q, kc, vc) = run_decode(c, status=st)
    info = arc.plan_decode(kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    # 16-byte aligned caches with a 16-byte multiple cell stride take the TMA kernel
    assert info["kernel"].startswith("decode_ws_kernel") and info["splits"] > 1
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
def test_decode_ragged_sequences(kv_type):
    c = W.decode_case(5, 0, 0, 16, 4, 128, kv_type=kv_type, seed=35, n_q_list=[4, 1, 3, 2, 4],
                      n_kv_list=[1000, 17, 3, 333, 4])
    o, lse, _ = run_decode(c)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
@pytest.mark.parametrize("H,Hkv,D,kernel", [
    (6, 3, 128, "decode_split_kernel"),   # cell = 3 head rows (408 / 216 bytes): no TMA, cp.async path
    (16, 4, 64, "decode_ws_kernel"),      # cell = 4 rows of 68 / 36 bytes = 272 / 144: TMA path at D = 64
])
def test_decode_both_load_paths(kv_type, H, Hkv, D, kernel):
    c = W.decode_case(3, 2, 700, H, Hkv, D, kv_type=kv_type, seed=40)
    st = status_word()
    o, lse, (q, kc, vc) = run_decode(c, status=st)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    assert info["kernel"].startswith(kernel)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


def _decode_into(c, q, kc, vc, ws, o, lse):
    arc.attn_decode_q8(q, kc, vc, kv_type=c.kv_type, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                       n_kv=c.n_kv, scale=c.scale, workspace=ws, out=o, lse=lse)


def test_decode_workspace_garbage_reuse_and_graph_replay():
    """The workspace needs no initialisation (stale bytes are never read before they
    are written), may be reused call after call, and a captured launch (split kernel
    plus its programmatic-dependent combine) replays correctly."""
    c = W.decode_case(2, 4, 3000, 16, 4, 128, kv_type=W.KV_Q8_0, seed=43)
    q, kc, vc = dev(c.q), dev(c.k_cache), dev(c.v_cache)
    n = arc.decode_workspace_size(c.kv_type, q, c.Hkv, c.k_cache.shape[0], c.q_begin, c.n_q, c.kv_begin, c.n_kv)
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")
    o = torch.empty(c.n_tok, c.H, c.D, dtype=torch.float32, device="cuda")
    lse = torch.empty(c.n_tok, c.H, dtype=torch.float32, device="cuda")
    ro, rl = oracle.run_case(c)
    for _ in range(3):
        o.fill_(float("nan"))
        _decode_into(c, q, kc, vc, ws, o, lse)
        torch.cuda.synchronize()
        compare(o, lse, ro, rl, TOL_O_BF16)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        _decode_into(c, q, kc, vc, ws, o, lse)   # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            _decode_into(c, q, kc, vc, ws, o, lse)
    torch.cuda.synchronize()
    for _ in range(3):
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        compare(o, lse, ro, rl, TOL_O_BF16)
    del g


def test_decode_head_dim_64_and_control_arm():
    c = W.decode_case(2, 3, 500, 8, 2, 64, kv_type=W.KV_Q8_0, seed=36)
    o, lse, _ = run_decode(c)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    o2, lse2, (q, kc, vc) = run_decode(c, flags=arc.ARC_FLAG_FORCE_SIMPLE)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q,
                           kv_begin=c.kv_begin, n_kv=c.n_kv, flags=arc.ARC_FLAG_FORCE_SIMPLE)
    assert info["kernel"] == "simple_decode_kernel"
    compare(o2, lse2, ro, rl, TOL_O_BF16)


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
@pytest.mark.parametrize("D", [256, 512])
def test_decode_wide_head_dims(kv_type, D):
    """Head dims 256 / 512 (the sliced tensor-core split kernel): ragged sequences, GQA 4."""
    c = W.decode_case(3, 0, 0, 8, 2, D, kv_type=kv_type, seed=62, n_q_list=[2, 1, 4], n_kv_list=[700, 1, 130])
    st = status_word()
    o, lse, (q, kc, vc) = run_decode(c, status=st)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    assert info["kernel"].startswith("decode_ws_kernel") and info["d_slice"] == 128
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK
    o2, lse2 = arc.attn_decode_q8(q, kc, vc, kv_type=c.kv_type, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q,
                                  kv_begin=c.kv_begin, n_kv=c.n_kv, scale=c.scale, flags=arc.ARC_FLAG_FORCE_SIMPLE)
    torch.cuda.synchronize()
    compare(o2, lse2, ro, rl, TOL_O_BF16)                 # the CUDA-core control arm


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
@pytest.mark.parametrize("D,G,n_q", [(128, 8, 4), (128, 4, 16), (256, 8, 4), (512, 4, 16), (64, 32, 4)])
def test_decode_more_than_16_fold_rows_full_length(kv_type, D, G, n_q):
    """Several sequences of G * n_q = 32 to 128 fold rows over 8192-cell caches: two m16
    fragments per CTA (one at D = 512) in row groups, many splits and the combine."""
    c = W.decode_case(2, n_q, 8192, 4 * G, 4, D, kv_type=kv_type, seed=63 + D + G)
    st = status_word()
    o, lse, (q, kc, vc) = run_decode(c, status=st)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    assert info["kernel"].startswith("decode_ws_kernel") and info["tile_m"] == (16 if D == 512 else 32)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


# ------------------------------------------------------------------ edge cases and failure reporting

def test_empty_and_degenerate_shapes():
    # Tq = 0: nothing to do.  Tk = 0: every row sees nothing -> O = 0, LSE = -inf (or the sink).
    c = W.dense_case(1, 4, 2, 0, 10, 64, dtype="bf16", seed=37)
    o, lse, _ = run_dense(c)
    assert o.numel() == 0
    c = W.dense_case(1, 4, 2, 5, 0, 64, dtype="bf16", sinks=True, seed=38)
    o, lse, _ = run_dense(c)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)


def test_bounded_wait_reports_a_timeout():
    st = status_word()
    assert arc.selftest_timeout(st, 2_000_000) == arc.ARC_OK     # 2 ms bound
    assert arc.check_device_error(st) == arc.ARC_ERR_DEVICE_TIMEOUT
    # The context stays usable afterwards.
    c = W.dense_case(1, 2, 2, 64, 64, 64, dtype="bf16", seed=39)
    o, lse, _ = run_dense(c)
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)


def test_invalid_arguments_launch_nothing():
    q = torch.zeros(1, 3, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.full((1, 3, 8, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(arc.ArcError) as e:
        arc.attn_fwd(q, k, k, out=out)
    assert e.value.status == arc.ARC_ERR_INVALID_ARG
    assert torch.all(out == 7.0)


# ------------------------------------------------------------------ merge over disjoint key sets

@pytest.mark.parametrize("n_parts,dv,dtype,sinks", [(1, 64, "f32", False), (3, 128, "f32", True),
                                                     (5, 512, "bf16", True), (2, 256, "bf16", False),
                                                     (2, 94, "bf16", True)])   # dv % 8 != 0: 2-element path
def test_merge_matches_oracle(n_parts, dv, dtype, sinks):
    rng = np.random.default_rng(50 + n_parts)
    B, H, T = 2, 6, 97
    o_np = [rng.standard_normal((B, H, T, dv)).astype(np.float32) for _ in range(n_parts)]
    l_np = [(3.0 * rng.standard_normal((B, H, T))).astype(np.float32) for _ in range(n_parts)]
    for i in range(n_parts):                      # scattered empty parts, and some rows empty in every part
        l_np[i][rng.random((B, H, T)) < 0.2] = -np.inf
    for i in range(n_parts):
        l_np[i][0, 0, :5] = -np.inf
    s_np = rng.standard_normal(H).astype(np.float32) if sinks else None
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    o_dev = [torch.from_numpy(x).cuda().to(tdt) for x in o_np]
    l_dev = [torch.from_numpy(x).cuda() for x in l_np]
    s_dev = torch.from_numpy(s_np).cuda() if sinks else None
    o, lse = arc.attn_merge(o_dev, l_dev, sinks=s_dev, sink_rows=T if sinks else None)
    torch.cuda.synchronize()
    o_in = [x.float().cpu().numpy() for x in o_dev]          # the oracle merges the same (rounded) parts
    rows = None if s_np is None else np.broadcast_to(s_np.astype(np.float64)[None, :, None], (B, H, T))
    ro, rl = oracle.merge(o_in, l_np, sink_rows=rows)
    compare(o, lse, ro, rl, TOL_O_F32 if dtype == "f32" else TOL_O_BF16)
    info = arc.plan_merge(o_dev, l_dev, o, lse)
    assert info["kernel"] == "merge_kernel" and info["launches"] == 1


def test_merge_in_place_over_the_first_part():
    rng = np.random.default_rng(57)
    o_np = [rng.standard_normal((40, 128)).astype(np.float32) for _ in range(2)]
    l_np = [rng.standard_normal(40).astype(np.float32) for _ in range(2)]
    o_dev = [torch.from_numpy(x).cuda() for x in o_np]
    l_dev = [torch.from_numpy(x).cuda() for x in l_np]
    o, lse = arc.attn_merge(o_dev, l_dev, out=o_dev[0], lse=l_dev[0])
    torch.cuda.synchronize()
    ro, rl = oracle.merge(o_np, l_np)
    compare(o, lse, ro, rl, TOL_O_F32)


@pytest.mark.parametrize("world,B,H,Hkv,L,D,sinks", [(2, 1, 8, 2, 200, 128, True), (4, 2, 4, 4, 130, 64, False)])
def test_context_parallel_chunks_merge_to_attention_over_the_whole_sequence(world, B, H, Hkv, L, D, sinks):
    """Each emulated rank runs the ring schedule with the library's attention and merge
    kernels on one GPU; its chunk of O / LSE matches the oracle over the whole sequence."""
    from exact_attention_131_b200 import cp

    c = W.dense_case(B, H, Hkv, world * L, world * L, D, dtype="bf16", std=0.5, causal=True, sinks=sinks, seed=58)
    q, k, v = dev(c.q, torch.bfloat16), dev(c.k, torch.bfloat16), dev(c.v, torch.bfloat16)
    s = dev(c.sinks) if sinks else None
    outs = cp.context_parallel_forward_local(q, k, v, world, causal=True, scale=c.scale, sinks=s)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=True, sinks=c.sinks if sinks else None)
    for r, (o, lse) in enumerate(outs):
        compare(o, lse, ro[:, :, r * L:(r + 1) * L], rl[:, :, r * L:(r + 1) * L], TOL_O_BF16)


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
def test_single_stream_decode_one_token_long_context(kv_type):
    """One sequence, one new token (t_q = 1), a long cache: few (sequence, kv head)
    pairs, so many splits and the two-kernel merge."""
    c = W.decode_case(1, 1, 40000, 32, 4, 128, kv_type=kv_type, seed=59)
    st = status_word()
    o, lse, (q, kc, vc) = run_decode(c, status=st)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    assert info["kernel"].startswith("decode_ws_kernel") and info["splits"] > 16 and info["launches"] == 2
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK


def test_merge_sixteen_parts_and_empty_call():
    rng = np.random.default_rng(61)
    o_np = [rng.standard_normal((33, 64)).astype(np.float32) for _ in range(16)]
    l_np = [rng.standard_normal(33).astype(np.float32) for _ in range(16)]
    o, lse = arc.attn_merge([torch.from_numpy(x).cuda() for x in o_np], [torch.from_numpy(x).cuda() for x in l_np])
    torch.cuda.synchronize()
    ro, rl = oracle.merge(o_np, l_np)
    compare(o, lse, ro, rl, TOL_O_F32)
    e = [torch.empty(0, 64, device="cuda")] * 2
    el = [torch.empty(0, device="cuda")] * 2
    o0, l0 = arc.attn_merge(e, el)                      # zero rows: nothing launched, nothing written
    assert o0.shape == (0, 64) and l0.shape == (0,)


def test_repeated_calls_are_bit_identical():
    """Every kernel sums in a fixed order (static tile assignment, no atomics), so the
    same call twice gives the same bits ("TensorRT-LLM: FlashMLA without -rdc" holds
    its build change to bit-identical outputs)."""
    def twice(run):
        a = [t.clone() for t in run()]
        b = run()
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int32) if x.dtype == torch.float32 else x.view(torch.int16),
                               y.view(torch.int32) if y.dtype == torch.float32 else y.view(torch.int16))

    c = W.dense_case(1, 16, 2, 200, 200, 512, 512, dtype="bf16", std=0.5, causal=True, sinks=True, seed=31)
    twice(lambda: run_dense(c)[:2])
    m = W.mla_case(1, 3, 300, 300, 128, 64, 128, seed=33)
    twice(lambda: run_mla(m)[:2])
    s = W.sparse_case(20, 64, 3000, 512, 512, 250, pad_mode="tail", seed=34)
    twice(lambda: run_sparse(s)[:2])
    d = W.decode_case(2, 4, 3000, 16, 4, 128, kv_type=W.KV_Q4_0, seed=43)
    twice(lambda: run_decode(d)[:2])
