"""Pins for the fp64 CPU oracle, against things other than the oracle itself.

Each pin is chosen so that a plausible mistake (a dropped term, a wrong sign
or index, a transposed operand, a misplaced mask) fails at least one of them;
the mutation tests at the end plant such mistakes in the oracle and check
that they are caught, as the ArcFlash rung-0 page does with its
"four mutations, four caught" table.

Independent references used:
  * torch.nn.functional.scaled_dot_product_attention in float64 on the CPU
    (a library implementation of the same definition), including its
    enable_gqa head map and float-bias masks;
  * closed forms: zero queries (LSE = ln #visible), a single key, identical keys;
  * numpy's own float16 decoding, for the q8_0 / q4_0 block scale.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as W

TOL = 1e-11


def t64(x):
    return torch.from_numpy(oracle.widen(x))


def sdpa(q, k, v, *, scale, mask=None, causal_br=False, gqa=False):
    """torch fp64 SDPA; causal_br builds a bottom-right causal boolean mask."""
    q, k, v = t64(q), t64(k), t64(v)
    Tq, Tk = q.shape[-2], k.shape[-2]
    if causal_br:
        i = torch.arange(Tq)[:, None]
        j = torch.arange(Tk)[None, :]
        bm = j <= i + (Tk - Tq)
        mask = bm if mask is None else mask.masked_fill(~bm, float("-inf"))
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale,
                                          enable_gqa=gqa).numpy()


def logsumexp_scores(q, k, scale, causal_br):
    """LSE from torch's logsumexp over explicitly masked fp64 scores (MHA only)."""
    q, k = t64(q), t64(k)
    s = torch.einsum("bhid,bhjd->bhij", q, k) * scale
    if causal_br:
        Tq, Tk = s.shape[-2:]
        i = torch.arange(Tq)[:, None]
        j = torch.arange(Tk)[None, :]
        s = s.masked_fill(~(j <= i + (Tk - Tq)), float("-inf"))
    return torch.logsumexp(s, dim=-1).numpy()


# ------------------------------------------------------------------ softmax core

@pytest.mark.parametrize("B,H,Tq,Tk,D,Dv,causal", [
    (1, 2, 7, 7, 16, 16, True),
    (2, 3, 5, 9, 8, 12, True),      # Tq < Tk: bottom-right alignment
    (1, 1, 33, 33, 64, 64, False),
    (2, 2, 1, 17, 32, 32, True),    # a single decode-like query
])
def test_attn_matches_torch_sdpa(B, H, Tq, Tk, D, Dv, causal):
    c = W.dense_case(B, H, H, Tq, Tk, D, Dv, dtype="f32", causal=causal, seed=11)
    o, lse = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=causal)
    ref = sdpa(c.q, c.k, c.v, scale=c.scale, causal_br=causal)
    assert np.abs(o - ref).max() < TOL
    ref_lse = logsumexp_scores(c.q, c.k, c.scale, causal)
    assert np.abs(lse - ref_lse).max() < TOL


def test_zero_query_lse_counts_visible_keys():
    """q = 0: every score is 0, so LSE_i = ln(#visible) = ln(i + Tk - Tq + 1), O = mean of visible V."""
    B, H, Tq, Tk, D = 1, 2, 6, 10, 8
    c = W.dense_case(B, H, H, Tq, Tk, D, dtype="f32", seed=3)
    q = np.zeros_like(c.q)
    o, lse = oracle.attn(q, c.k, c.v, scale=0.3, causal=True)
    n = np.arange(Tq) + (Tk - Tq) + 1
    assert np.abs(lse - np.log(n)[None, None, :]).max() < 1e-14
    vm = np.cumsum(c.v.astype(np.float64), axis=2)[:, :, Tk - Tq:, :] / n[None, None, :, None]
    assert np.abs(o - vm).max() < 1e-13


def test_single_key_closed_form():
    c = W.dense_case(2, 3, 3, 4, 1, 16, dtype="f32", causal=False, seed=4)
    o, lse = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=False)
    assert np.abs(o - np.broadcast_to(c.v, o.shape)).max() < 1e-15
    s0 = c.scale * np.einsum("bhid,bhjd->bhi", c.q.astype(np.float64), c.k.astype(np.float64))
    assert np.abs(lse - s0).max() < 1e-13


def test_identical_keys_closed_form():
    """All keys equal: O = mean of visible values, LSE = s + ln|visible|."""
    c = W.dense_case(1, 2, 2, 5, 5, 8, dtype="f32", causal=True, seed=5)
    k = np.broadcast_to(c.k[:, :, :1, :], c.k.shape).copy()
    o, lse = oracle.attn(c.q, k, c.v, scale=c.scale, causal=True)
    n = np.arange(1, 6)
    vm = np.cumsum(c.v.astype(np.float64), axis=2) / n[None, None, :, None]
    assert np.abs(o - vm).max() < 1e-13
    s = c.scale * np.einsum("bhid,bhd->bhi", c.q.astype(np.float64), k[:, :, 0, :].astype(np.float64))
    assert np.abs(lse - (s + np.log(n))).max() < 1e-13


def test_empty_visible_set_reading():
    """Tq > Tk with bottom-right causal leaves the first rows with no key: O = 0, LSE = -inf."""
    c = W.dense_case(1, 1, 1, 5, 3, 8, dtype="f32", causal=True, seed=6)
    o, lse = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=True)
    assert np.all(o[0, 0, :2] == 0) and np.all(np.isneginf(lse[0, 0, :2]))
    assert np.all(np.isfinite(lse[0, 0, 2:]))


def test_row_subset_equals_full():
    c = W.dense_case(1, 4, 2, 40, 40, 16, dtype="bf16", seed=7)
    o, lse = oracle.attn(c.q, c.k, c.v, scale=c.scale)
    rows = [0, 3, 17, 39]
    os_, ls_ = oracle.attn(c.q, c.k, c.v, scale=c.scale, rows=rows)
    assert np.array_equal(os_, o[:, :, rows]) and np.array_equal(ls_, lse[:, :, rows])


# ------------------------------------------------------------------ GQA fold

def gqa_max_diff(g, causal=True, seed=8):
    Hkv = 64 // g if g > 8 else 2
    H = Hkv * g
    c = W.dense_case(1, H, Hkv, 9, 9, 16, dtype="f32", causal=causal, seed=seed)
    o, _ = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=causal)
    ref = sdpa(c.q, c.k, c.v, scale=c.scale, causal_br=causal, gqa=True)
    return np.abs(o - ref).max(), c, o


@pytest.mark.parametrize("g", [1, 2, 4, 8, 64])
def test_gqa_matches_torch_enable_gqa_and_repeat_kv(g):
    d, c, o = gqa_max_diff(g)
    assert d < TOL
    # repeat_kv: y[b, kv*g + rep] = x[b, kv]  (kv-major), written with numpy's repeat.
    kr, vr = np.repeat(c.k, g, axis=1), np.repeat(c.v, g, axis=1)
    o2, _ = oracle.attn(c.q, kr, vr, scale=c.scale)
    assert np.abs(o - o2).max() < 1e-14


def test_fold_view_equals_per_head_definition():
    c = W.dense_case(2, 8, 2, 13, 13, 16, dtype="bf16", sinks=True, seed=9)
    of, lf = oracle.attn_fold(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks)
    o, lse = oracle.attn(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks)
    # [B,Hkv,g*Tq,Dv] is the same memory as [B,H,Tq,Dv] when heads are kv-major.
    assert np.array_equal(of.reshape(o.shape), o)
    assert np.array_equal(lf.reshape(lse.shape), lse)


# ------------------------------------------------------------------ sinks

def sink_reference(c):
    """Sinks through torch SDPA: one extra key with score sigma_h (zero q.k plus a float bias) and a zero value."""
    q, k, v = t64(c.q), t64(c.k), t64(c.v)
    B, H, Tq, D = q.shape
    g = H // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    v = v.repeat_interleave(g, dim=1)
    Tk = k.shape[2]
    k = torch.cat([k, torch.zeros(B, H, 1, D, dtype=k.dtype)], dim=2)
    v = torch.cat([v, torch.zeros(B, H, 1, v.shape[-1], dtype=v.dtype)], dim=2)
    i = torch.arange(Tq)[:, None]
    j = torch.arange(Tk)[None, :]
    bias = torch.zeros(H, Tq, Tk + 1, dtype=torch.float64)
    bias[:, :, :Tk] = bias[:, :, :Tk].masked_fill(~(j <= i + (Tk - Tq)), float("-inf"))
    bias[:, :, Tk] = torch.from_numpy(c.sinks.astype(np.float64))[:, None]
    return F.scaled_dot_product_attention(q, k, v, attn_mask=bias[None], scale=c.scale).numpy()


def test_sinks_match_torch_with_virtual_key():
    c = W.dense_case(1, 8, 2, 11, 11, 32, dtype="bf16", sinks=True, seed=12)
    o, _ = oracle.attn(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks)
    assert np.abs(o - sink_reference(c)).max() < TOL


def test_sinks_closed_forms():
    c = W.dense_case(1, 4, 4, 6, 6, 16, dtype="f32", sinks=True, seed=13)
    o0, l0 = oracle.attn(c.q, c.k, c.v, scale=c.scale)
    o1, l1 = oracle.attn(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks)
    sig = c.sinks.astype(np.float64)[None, :, None]
    # The sink only enlarges the denominator: LSE adds it in log space, O shrinks uniformly.
    assert np.abs(l1 - np.logaddexp(l0, sig)).max() < 1e-13
    assert np.abs(o1 - o0 * np.exp(l0 - l1)[..., None]).max() < 1e-13
    # sigma -> -inf is no sink at all.
    o2, l2 = oracle.attn(c.q, c.k, c.v, scale=c.scale, sinks=np.full(4, -np.inf))
    assert np.array_equal(o2, o0) and np.array_equal(l2, l0)
    # q = 0: LSE = ln(n + e^sigma).
    _, l3 = oracle.attn(np.zeros_like(c.q), c.k, c.v, scale=c.scale, sinks=c.sinks)
    n = np.arange(1, 7)[None, None, :]
    assert np.abs(l3 - np.log(n + np.exp(sig))).max() < 1e-13


# ------------------------------------------------------------------ query-row tiling

def test_query_tiling_is_exact_and_the_mask_follows_the_tile():
    c = W.dense_case(1, 8, 2, 150, 150, 32, dtype="bf16", sinks=True, seed=14)
    o, lse = oracle.attn(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks)
    budget = 8 * 20 * 150 * 4            # 20 rows per tile
    ot, lt, nt = oracle.attn_tiled(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks, tile_bytes=budget)
    assert nt > 1, "the shape must actually tile"
    assert nt == math.ceil(150 / 20)
    assert np.array_equal(ot, o) and np.array_equal(lt, lse)


def test_rung0_tile_count_at_the_prefill_shape():
    """H=64, T=1400 under a 32 MiB fp32 score budget: 93 rows per tile, 16 tiles."""
    c = W.dense_case(1, 64, 8, 1400, 1400, 8, dtype="bf16", sinks=True, seed=15)
    rows = (32 << 20) // (64 * 1400 * 4)
    assert rows == 93
    _, _, nt = oracle.attn_tiled(c.q[:, :, :, :], c.k, c.v, scale=c.scale, sinks=c.sinks)
    assert nt == 16


# ------------------------------------------------------------------ MLA

def test_mla_matches_torch_on_explicit_concat():
    c = W.mla_case(2, 4, 37, 37, 32, 16, 24, seed=16)
    o, lse = oracle.mla(c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v, scale=c.scale)
    q = np.concatenate([oracle.widen(c.q_nope), oracle.widen(c.q_rope)], axis=-1)
    kr = np.broadcast_to(oracle.widen(c.k_rope)[:, None], (2, 4, 37, 16))
    k = np.concatenate([oracle.widen(c.k_nope), kr], axis=-1)
    ref = sdpa(q, k, c.v, scale=c.scale, causal_br=True)
    assert np.abs(o - ref).max() < TOL
    assert np.abs(lse - logsumexp_scores(q, k, c.scale, True)).max() < TOL


# ------------------------------------------------------------------ sparse

def test_sparse_all_keys_permuted_equals_dense_noncausal():
    rng = np.random.default_rng(17)
    c = W.sparse_case(6, 4, 50, 32, 32, 50, pad_frac=0.0, seed=17)
    idx = np.stack([rng.permutation(50) for _ in range(6)]).astype(np.int32)
    o, lse = oracle.sparse(c.q, c.kv, idx, scale=c.scale)
    q = oracle.widen(c.q).transpose(1, 0, 2)[None]          # [1,H,nq,D]
    k = np.broadcast_to(oracle.widen(c.kv)[None, None], (1, 4, 50, 32))
    ref = sdpa(q, k, k, scale=c.scale)
    assert np.abs(o - ref[0].transpose(1, 0, 2)).max() < TOL


def test_sparse_padding_and_out_of_range_are_masked():
    c = W.sparse_case(5, 4, 80, 32, 32, 40, pad_frac=0.0, seed=18)
    o, lse = oracle.sparse(c.q, c.kv, c.idx, scale=c.scale)
    idx2 = np.concatenate([c.idx, np.full((5, 7), -1, np.int32), np.full((5, 2), 80, np.int32)], 1)
    o2, l2 = oracle.sparse(c.q, c.kv, idx2, scale=c.scale)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_sparse_duplicate_index_doubles_its_weight():
    c = W.sparse_case(3, 2, 30, 16, 16, 30, pad_frac=0.0, seed=19)
    idx = np.tile(np.arange(30, dtype=np.int32), (3, 1))
    idx_dup = np.concatenate([idx, np.full((3, 1), 7, np.int32)], axis=1)
    o, lse = oracle.sparse(c.q, c.kv, idx_dup, scale=c.scale)
    q = oracle.widen(c.q).transpose(1, 0, 2)[None]
    k = np.broadcast_to(oracle.widen(c.kv)[None, None], (1, 2, 30, 16))
    bias = torch.zeros(30, dtype=torch.float64)
    bias[7] = math.log(2.0)
    ref = sdpa(q, k, k, scale=c.scale, mask=bias[None, :])
    assert np.abs(o - ref[0].transpose(1, 0, 2)).max() < TOL


def test_sparse_separate_v_and_slot_order():
    c = W.sparse_case(4, 3, 64, 32, 16, 20, pad_frac=0.1, separate_v=True, seed=20)
    o, lse = oracle.sparse(c.q, c.kv, c.idx, scale=c.scale, v=c.v)
    perm = np.random.default_rng(0).permutation(20)
    o2, l2 = oracle.sparse(c.q, c.kv, c.idx[:, perm], scale=c.scale, v=c.v)
    assert np.abs(o - o2).max() < 1e-14 and np.abs(lse - l2).max() < 1e-14
    # V = kv[:, :Dv] when no separate V is given.
    o3, _ = oracle.sparse(c.q, c.kv, c.idx, scale=c.scale, Dv=16)
    o4, _ = oracle.sparse(c.q, c.kv, c.idx, scale=c.scale, v=c.kv[:, :16])
    assert np.array_equal(o3, o4)


# ------------------------------------------------------------------ q8_0 / q4_0 and decode

def test_fp16_scale_decoding_matches_numpy():
    vals = np.array([0.5, -3.25, 6.1e-5, 1e-7, 65504.0, -0.0, 1.0 / 3.0], dtype=np.float16)
    x = np.zeros((len(vals), 1, 32), np.float32)
    blocks = W.encode_q8_0(x)
    blocks[:, :, 0:2] = vals.view(np.uint8).reshape(-1, 1, 2)
    blocks[:, :, 2] = 1                                   # q_0 = 1 -> value = d
    out = oracle.dequant_cache(W.KV_Q8_0, blocks.reshape(len(vals), 1, 34), len(vals), 1, 32)
    assert np.array_equal(out[:, 0, 0], vals.astype(np.float64))


def test_golden_q8_0_and_q4_0_blocks():
    """Hand-written blocks from the format definition (tests/golden/quant_blocks.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "quant_blocks.txt")
    cases = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, kind, payload = line.split(" ", 2)
        cases.setdefault(name, {})[kind] = payload
    assert cases
    for name, c in cases.items():
        kv_type = W.KV_Q8_0 if name.startswith("q8") else W.KV_Q4_0
        blk = np.array([int(b, 16) for b in c["bytes"].split()], np.uint8)
        expect = np.array([float(x) for x in c["values"].split()])
        out = oracle.dequant_cache(kv_type, blk.reshape(1, 1, -1), 1, 1, 32)
        assert np.array_equal(out[0, 0], expect), name


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
def test_quant_roundtrip_within_half_step(kv_type):
    rng = W.make_rng(21)
    x = rng.standard_normal((64, 4, 128)).astype(np.float32)
    enc = W.encode_q8_0(x) if kv_type == W.KV_Q8_0 else W.encode_q4_0(x)
    deq = oracle.dequant_cache(kv_type, enc, 64, 4, 128)
    xb = x.reshape(64, 4, 4, 32).astype(np.float64)
    err = np.abs(deq.reshape(64, 4, 4, 32) - xb)
    if kv_type == W.KV_Q8_0:
        step = np.abs(xb).max(-1, keepdims=True) / 127.0
        assert np.all(err <= 0.57 * step)
    else:
        step = np.abs(xb).max(-1, keepdims=True) / 8.0
        assert np.all(err <= 1.01 * step)
        assert np.mean(err <= 0.51 * step) > 0.99


@pytest.mark.parametrize("kv_type", [W.KV_Q8_0, W.KV_Q4_0])
@pytest.mark.parametrize("D", [64, 512])
def test_decode_matches_torch_per_sequence(kv_type, D):
    c = W.decode_case(3, 4, 0, 8, 2, D, kv_type=kv_type, seed=22, n_q_list=[4, 1, 3],
                      n_kv_list=[40, 17, 3])
    o, lse = oracle.decode_q(c)
    K = oracle.dequant_cache(kv_type, c.k_cache, c.n_cells, c.Hkv, c.D)
    V = oracle.dequant_cache(kv_type, c.v_cache, c.n_cells, c.Hkv, c.D)
    for s in range(c.n_seq):
        qs = c.q[c.q_begin[s]:c.q_begin[s] + c.n_q[s]].transpose(1, 0, 2)[None]
        ks = K[c.kv_begin[s]:c.kv_begin[s] + c.n_kv[s]].transpose(1, 0, 2)[None]
        vs = V[c.kv_begin[s]:c.kv_begin[s] + c.n_kv[s]].transpose(1, 0, 2)[None]
        ref = sdpa(qs, ks, vs, scale=c.scale, causal_br=True, gqa=True)[0].transpose(1, 0, 2)
        got = o[c.q_begin[s]:c.q_begin[s] + c.n_q[s]]
        assert np.abs(got - ref).max() < TOL


# ------------------------------------------------------------------ merge over disjoint key sets

def ref_lse_gqa(q, k, scale, causal_br):
    """LSE over explicitly masked fp64 scores, K repeated kv-major to every query head."""
    g = q.shape[1] // k.shape[1]
    return logsumexp_scores(q, np.repeat(oracle.widen(k), g, axis=1), scale, causal_br)


def test_merge_of_key_chunks_equals_attention_over_all_keys():
    """Attention over random disjoint chunks of the keys (no mask), merged by
    log-sum-exp, equals torch's fp64 SDPA over all keys.  With sinks the chunks are
    computed without them and the merge adds the sink once; that equals attention
    with the sink inside the softmax (pinned against torch elsewhere)."""
    c = W.dense_case(2, 4, 2, 37, 101, 16, 24, dtype="bf16", causal=False, sinks=True, seed=40)
    cuts = [0, 13, 14, 70, 101]                                   # one chunk of a single key
    parts = [oracle.attn(c.q, c.k[:, :, a:b], c.v[:, :, a:b], scale=c.scale, causal=False)
             for a, b in zip(cuts, cuts[1:])]
    o, lse = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
    ref_o = sdpa(c.q, c.k, c.v, scale=c.scale, gqa=True)
    ref_lse = ref_lse_gqa(c.q, c.k, c.scale, False)
    assert np.abs(o - ref_o).max() < TOL and np.abs(lse - ref_lse).max() < TOL
    sink_rows = np.broadcast_to(oracle.widen(c.sinks)[None, :, None], lse.shape)
    os_, ls_ = oracle.merge([p[0] for p in parts], [p[1] for p in parts], sink_rows=sink_rows)
    so, sl = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=False, sinks=c.sinks)
    assert np.abs(os_ - so).max() < TOL and np.abs(ls_ - sl).max() < TOL


def test_merge_reassembles_causal_attention_from_sequence_chunks():
    """The context-parallel split: with Q and K/V cut into n equal sequence chunks,
    query chunk r merges its own chunk under the causal mask with every earlier
    chunk unmasked; later chunks are invisible.  Equals causal SDPA over the whole
    sequence."""
    n, L = 4, 23
    c = W.dense_case(1, 6, 3, n * L, n * L, 16, dtype="bf16", causal=True, seed=41)
    ref_o = sdpa(c.q, c.k, c.v, scale=c.scale, causal_br=True, gqa=True)
    ref_lse = ref_lse_gqa(c.q, c.k, c.scale, True)
    for r in range(n):
        q = c.q[:, :, r * L:(r + 1) * L]
        parts = []
        for s_ in range(r + 1):
            k, v = c.k[:, :, s_ * L:(s_ + 1) * L], c.v[:, :, s_ * L:(s_ + 1) * L]
            parts.append(oracle.attn(q, k, v, scale=c.scale, causal=(s_ == r)))
        o, lse = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
        assert np.abs(o - ref_o[:, :, r * L:(r + 1) * L]).max() < TOL
        assert np.abs(lse - ref_lse[:, :, r * L:(r + 1) * L]).max() < TOL


def test_merge_special_cases():
    rng = np.random.default_rng(42)
    o1 = rng.standard_normal((5, 8))
    l1 = rng.standard_normal(5)
    o, lse = oracle.merge([o1], [l1])                             # one part: identity
    assert np.abs(o - o1).max() < TOL and np.abs(lse - l1).max() < TOL
    empty = np.full(5, -np.inf)
    o, lse = oracle.merge([o1, rng.standard_normal((5, 8))], [l1, empty])   # an empty part adds nothing
    assert np.abs(o - o1).max() < TOL and np.abs(lse - l1).max() < TOL
    o, lse = oracle.merge([o1, o1], [empty, empty])               # nothing visible
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    sink = rng.standard_normal(5)
    o, lse = oracle.merge([o1], [empty], sink_rows=sink)          # only the sink: LSE = sink, O = 0
    assert np.all(o == 0) and np.abs(lse - sink).max() < TOL
    o, lse = oracle.merge([o1, 3 * o1], [l1, l1])                 # equal weights: the mean, LSE + ln 2
    assert np.abs(o - 2 * o1).max() < TOL and np.abs(lse - (l1 + math.log(2))).max() < TOL


# ------------------------------------------------------------------ mutations are caught

def test_mutation_rep_major_is_caught(mutation):
    mutation(oracle.MUT_REP_MAJOR)
    d, _, _ = gqa_max_diff(4)
    assert d > 0.1


def test_mutation_mask_not_following_tile_is_caught(mutation):
    c = W.dense_case(1, 4, 2, 60, 60, 16, dtype="bf16", seed=23)
    o, _ = oracle.attn(c.q, c.k, c.v, scale=c.scale)
    mutation(oracle.MUT_TILE_LOCAL_MASK)
    ot, _, nt = oracle.attn_tiled(c.q, c.k, c.v, scale=c.scale, tile_bytes=4 * 15 * 60 * 4)
    assert nt > 1 and np.abs(ot - o).max() > 0.1


def test_mutation_dropped_sink_is_caught(mutation):
    c = W.dense_case(1, 8, 2, 11, 11, 32, dtype="bf16", sinks=True, seed=12)
    mutation(oracle.MUT_DROP_SINK)
    o, _ = oracle.attn(c.q, c.k, c.v, scale=c.scale, sinks=c.sinks)
    assert np.abs(o - sink_reference(c)).max() > 1e-3


def test_mutation_top_left_causal_is_caught(mutation):
    mutation(oracle.MUT_TOP_LEFT_CAUSAL)
    c = W.dense_case(1, 2, 2, 5, 9, 8, dtype="f32", seed=24)
    o, _ = oracle.attn(c.q, c.k, c.v, scale=c.scale, causal=True)
    assert np.abs(o - sdpa(c.q, c.k, c.v, scale=c.scale, causal_br=True)).max() > 0.1


def test_mutation_swapped_nibbles_is_caught(mutation):
    rng = W.make_rng(25)
    x = rng.standard_normal((8, 1, 64)).astype(np.float32)
    enc = W.encode_q4_0(x)
    mutation(oracle.MUT_SWAP_NIBBLES)
    deq = oracle.dequant_cache(W.KV_Q4_0, enc, 8, 1, 64)
    step = np.abs(x.reshape(8, 1, 2, 32)).max(-1, keepdims=True) / 8.0
    assert not np.all(np.abs(deq.reshape(8, 1, 2, 32) - x.reshape(8, 1, 2, 32)) <= 1.01 * step)


def test_mutation_unweighted_merge_is_caught(mutation):
    c = W.dense_case(1, 4, 4, 20, 60, 16, dtype="bf16", causal=False, seed=43)
    parts = [oracle.attn(c.q, c.k[:, :, a:b], c.v[:, :, a:b], scale=c.scale, causal=False)
             for a, b in ((0, 10), (10, 60))]
    mutation(oracle.MUT_MERGE_UNWEIGHTED)
    o, _ = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
    assert np.abs(o - sdpa(c.q, c.k, c.v, scale=c.scale, gqa=True)).max() > 1e-2
