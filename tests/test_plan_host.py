"""Host-side checks of dispatch and validation for every call: which kernel
arc_plan names for each workload shape, the split-KV plan's arithmetic, and the
error each malformed call returns (as documented in include/arc_attn.h).
Nothing here launches a kernel: either validation refuses first, or arc_plan
answers without launching."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20          # a 256-byte-aligned non-NULL placeholder; nothing here dereferences it
SMS = 148               # the planner's SM count when no device is present


@pytest.fixture(scope="module")
def arc():
    import exact_attention_131_b200 as arc
    if not os.path.exists(arc.LIB_PATH):
        from exact_attention_131_b200 import build
        build.build()
    arc.lib()
    return arc


def contiguous(*shape):
    """Element strides of a contiguous tensor of this shape, outermost first, without the last (unit) one."""
    out, acc = [], 1
    for n in reversed(shape[1:]):
        acc *= n
        out.append(acc)
    return tuple(reversed(out))


# ----------------------------------------------------------------------------------- MLA
def mla_args(arc, B=2, H=16, Tq=4096, Tk=4096, Dn=128, Dr=64, Dv=128):
    m = arc.MlaArgs()
    m.B, m.H, m.Tq, m.Tk, m.Dn, m.Dr, m.Dv = B, H, Tq, Tk, Dn, Dr, Dv
    m.q_nope, m.q_rope, m.k_nope, m.k_rope, m.v, m.o, m.lse = (FAKE,) * 7
    m.q_nope_strides = (arc._i64 * 3)(*contiguous(B, H, Tq, Dn))
    m.q_rope_strides = (arc._i64 * 3)(*contiguous(B, H, Tq, Dr))
    m.k_nope_strides = (arc._i64 * 3)(*contiguous(B, H, Tk, Dn))
    m.k_rope_strides = (arc._i64 * 2)(*contiguous(B, Tk, Dr))
    m.v_strides = (arc._i64 * 3)(*contiguous(B, H, Tk, Dv))
    m.o_strides = (arc._i64 * 3)(*contiguous(B, H, Tq, Dv))
    m.scale, m.causal = 192 ** -0.5, 1
    return m


def test_mla_prefill_plans_the_cta_pair(arc):
    """q_nope/k_nope/v [2,16,4096,128], rope 64: the pair kernel, one d_v pass, persistent over SM pairs."""
    m = mla_args(arc)
    info = arc.plan(arc.ARC_OP_MLA, m)
    assert info["kernel"] == "tc_attn_pair_kernel<mla>" and info["tensor_cores"] == 1
    assert info["tile_m"] == 256 and info["d_slice"] == 128 and info["launches"] == 1
    items = (4096 // 128 + 1) // 2 * 2 * 16           # row-tile pairs x (B * H)
    assert info["n_ctas"] == 2 * min(items, SMS // 2)
    assert 0 < info["smem_bytes"] <= 227 * 1024
    m.flags = arc.ARC_FLAG_SINGLE_CTA
    info = arc.plan(arc.ARC_OP_MLA, m)
    assert info["kernel"] in ("tc_attn2_kernel<mla>", "tc_attn_kernel<mla>") and info["tile_m"] in (128, 256)
    m.flags = arc.ARC_FLAG_FORCE_SIMPLE
    assert arc.plan(arc.ARC_OP_MLA, m)["kernel"] == "simple_attn_kernel"


def test_mla_layouts_the_tensor_cores_cannot_take_are_refused(arc):
    m = mla_args(arc, Tq=256, Tk=256)
    m.k_rope = FAKE + 8                                 # not 16-byte aligned
    assert arc.lib().arc_plan(arc.ARC_OP_MLA, ctypes.byref(m), ctypes.byref(arc.PlanInfo())) == arc.ARC_ERR_UNSUPPORTED
    assert arc.lib().arc_mla_fwd(ctypes.byref(m), None) == arc.ARC_ERR_UNSUPPORTED
    m = mla_args(arc, Tq=256, Tk=256, Dn=96)            # Dn not a multiple of 64
    assert arc.lib().arc_mla_fwd(ctypes.byref(m), None) == arc.ARC_ERR_UNSUPPORTED
    m.flags = arc.ARC_FLAG_FORCE_SIMPLE                 # the CUDA-core kernel takes it
    assert arc.plan(arc.ARC_OP_MLA, m)["kernel"] == "simple_attn_kernel"


@pytest.mark.parametrize("field,value,want", [
    ("H", 0, "ARC_ERR_INVALID_ARG"), ("Tq", -1, "ARC_ERR_INVALID_ARG"), ("Dn", 0, "ARC_ERR_INVALID_ARG"),
    ("Dr", -64, "ARC_ERR_INVALID_ARG"), ("Dv", 0, "ARC_ERR_INVALID_ARG"), ("Dn", 512, "ARC_ERR_UNSUPPORTED"),
    ("Dv", 576, "ARC_ERR_UNSUPPORTED"), ("q_nope", None, "ARC_ERR_INVALID_ARG"), ("k_rope", None, "ARC_ERR_INVALID_ARG"),
    ("v", None, "ARC_ERR_INVALID_ARG"), ("lse", None, "ARC_ERR_INVALID_ARG"),
])
def test_mla_validation(arc, field, value, want):
    m = mla_args(arc, Tq=256, Tk=256)
    setattr(m, field, value)
    assert arc.lib().arc_mla_fwd(ctypes.byref(m), None) == getattr(arc, want)
    assert arc.lib().arc_plan(arc.ARC_OP_MLA, ctypes.byref(m), ctypes.byref(arc.PlanInfo())) == getattr(arc, want)


# -------------------------------------------------------------------------------- sparse
def sparse_args(arc, Sq=13312, H=64, Skv=65536, D=512, Dv=512, topk=2176):
    s = arc.SparseArgs()
    s.Sq, s.H, s.Skv, s.Dqk, s.Dv, s.topk = Sq, H, Skv, D, Dv, topk
    s.q, s.kv, s.idx, s.o, s.lse = (FAKE,) * 5
    s.q_strides = (arc._i64 * 2)(H * D, D)
    s.kv_stride, s.idx_stride = D, topk
    s.o_strides = (arc._i64 * 2)(H * Dv, Dv)
    s.scale = D ** -0.5
    return s


def test_sparse_prefill_plans_one_cta_per_query(arc):
    """13312 queries x 64 heads x 2176 top-k at d 512: the tcgen05 kernel, 64 rows per CTA."""
    info = arc.plan(arc.ARC_OP_SPARSE, sparse_args(arc))
    assert info["kernel"] == "sparse_tc_kernel" and info["tensor_cores"] == 1
    assert info["tile_m"] == 64 and info["d_slice"] == 512 and info["n_ctas"] == 13312
    assert 0 < info["smem_bytes"] <= 227 * 1024
    # more heads than one CTA's 64 rows: one CTA per (query, 64-head group)
    assert arc.plan(arc.ARC_OP_SPARSE, sparse_args(arc, Sq=10, H=128, topk=64))["n_ctas"] == 20


@pytest.mark.parametrize("change", ["q+8", "kv_stride", "FORCE_SIMPLE", "Dqk384"])
def test_sparse_other_layouts_run_the_cuda_core_kernel(arc, change):
    s = sparse_args(arc, Sq=4, topk=64)
    if change == "q+8":
        s.q = FAKE + 8
    elif change == "kv_stride":
        s.kv_stride = 516                               # rows not 16-byte aligned
    elif change == "FORCE_SIMPLE":
        s.flags = arc.ARC_FLAG_FORCE_SIMPLE
    else:
        s.Dqk, s.Dv, s.kv_stride = 384, 384, 384        # a shape without a tensor-core instantiation
        s.q_strides = (arc._i64 * 2)(64 * 384, 384)
    info = arc.plan(arc.ARC_OP_SPARSE, s)
    assert info["kernel"] == "simple_attn_kernel<sparse>" and info["tensor_cores"] == 0


@pytest.mark.parametrize("field,value,want", [
    ("Sq", -1, "ARC_ERR_INVALID_ARG"), ("H", 0, "ARC_ERR_INVALID_ARG"), ("topk", -1, "ARC_ERR_INVALID_ARG"),
    ("Dqk", 576, "ARC_ERR_UNSUPPORTED"), ("Dv", 0, "ARC_ERR_INVALID_ARG"), ("idx", None, "ARC_ERR_INVALID_ARG"),
    ("kv", None, "ARC_ERR_INVALID_ARG"), ("o", None, "ARC_ERR_INVALID_ARG"),
])
def test_sparse_validation(arc, field, value, want):
    s = sparse_args(arc, Sq=4, topk=64)
    setattr(s, field, value)
    assert arc.lib().arc_sparse_mla_fwd(ctypes.byref(s), None) == getattr(arc, want)


def test_sparse_v_wider_than_the_latent_needs_a_separate_v(arc):
    s = sparse_args(arc, Sq=4, topk=64, D=256, Dv=512)
    s.q_strides, s.kv_stride = (arc._i64 * 2)(64 * 256, 256), 256
    assert arc.lib().arc_sparse_mla_fwd(ctypes.byref(s), None) == arc.ARC_ERR_INVALID_ARG
    s.Sq = 0                                            # an empty call with bad shapes is still refused
    assert arc.lib().arc_sparse_mla_fwd(ctypes.byref(s), None) == arc.ARC_ERR_INVALID_ARG


# -------------------------------------------------------------------------------- decode
def decode_args(arc, kv_type, n_seq=4, n_q=4, n_kv=8192, H=32, Hkv=8, D=128):
    seqs = arc.make_seqs([n_q * s for s in range(n_seq)], [n_q] * n_seq,
                         [n_kv * s for s in range(n_seq)], [n_kv] * n_seq)
    d = arc.DecodeArgs()
    d.kv_type, d.n_tok, d.H, d.Hkv, d.D, d.n_cells, d.n_seq = kv_type, n_q * n_seq, H, Hkv, D, n_kv * n_seq, n_seq
    d.seqs = ctypes.cast(seqs, ctypes.POINTER(arc.Seq))
    d.q, d.k_cache, d.v_cache, d.o, d.lse = (FAKE,) * 5
    d.scale = D ** -0.5
    d._keep = seqs                                      # keep the host array alive with the struct
    return d


@pytest.mark.parametrize("kv", ["q8_0", "q4_0"])
def test_decode_split_plan_covers_every_cell_in_one_wave(arc, kv):
    """4 sequences x 4 tokens, 32 heads over 8 kv heads, 8192 cells each."""
    kv_type = arc.ARC_KV_Q8_0 if kv == "q8_0" else arc.ARC_KV_Q4_0
    d = decode_args(arc, kv_type)
    info = arc.plan(arc.ARC_OP_DECODE, d)
    assert info["kernel"] == f"decode_ws_kernel<{kv}>" and info["launches"] == 2
    splits = info["splits"]
    chunk = -(-8192 // splits)
    chunk = -(-chunk // 128) * 128                      # chunks are whole 128-cell tiles
    assert -(-8192 // chunk) == splits                  # no empty split
    assert info["n_ctas"] == 4 * 8 * splits <= SMS * 4  # one wave at <= 4 CTAs per SM
    ws = arc.lib().arc_decode_workspace_size(ctypes.byref(d))
    assert ws == 4 * 8 * splits * 16 * (128 + 2) * 4    # per (seq, kv head, split): 16 rows of O, m and l
    # caches that are 8- but not 16-byte aligned: the plain-load kernel
    d.k_cache = FAKE + 8
    assert arc.plan(arc.ARC_OP_DECODE, d)["kernel"] == f"decode_split_kernel<{kv}>"


def test_decode_single_stream_and_empty_caches(arc):
    d = decode_args(arc, arc.ARC_KV_Q8_0, n_seq=1, n_q=1, n_kv=32768)
    info = arc.plan(arc.ARC_OP_DECODE, d)
    assert info["kernel"] == "decode_ws_kernel<q8_0>" and info["splits"] * 8 <= SMS * 4
    assert info["splits"] >= SMS // 8                   # a lone sequence still spreads over the SMs
    d = decode_args(arc, arc.ARC_KV_Q8_0, n_seq=2, n_q=0, n_kv=0)
    assert arc.plan(arc.ARC_OP_DECODE, d)["kernel"] == "simple_decode_kernel"


@pytest.mark.parametrize("kv", ["q8_0", "q4_0"])
@pytest.mark.parametrize("D", [256, 512])
def test_decode_wide_heads_run_the_sliced_tensor_core_kernel(arc, kv, D):
    """Head dims 256 / 512: the TMA split kernel with the head dim cut into 128-dim
    slices (the four warps of a CTA: 2 cell groups x 2 slices, or 1 x 4)."""
    kv_type = arc.ARC_KV_Q8_0 if kv == "q8_0" else arc.ARC_KV_Q4_0
    d = decode_args(arc, kv_type, D=D)
    info = arc.plan(arc.ARC_OP_DECODE, d)
    assert info["kernel"] == f"decode_ws_kernel<{kv}>" and info["launches"] == 2 and info["tensor_cores"] == 1
    assert info["d_slice"] == 128 and info["tile_m"] == 16 and info["tile_n"] == 16 * 4 // (D // 128)
    ws = arc.lib().arc_decode_workspace_size(ctypes.byref(d))
    assert ws == 4 * 8 * info["splits"] * 16 * (D + 2) * 4
    d.flags = arc.ARC_FLAG_FORCE_SIMPLE
    info = arc.plan(arc.ARC_OP_DECODE, d)
    assert info["kernel"] == "simple_decode_kernel" and info["launches"] == 1 and info["tensor_cores"] == 0
    assert arc.lib().arc_decode_workspace_size(ctypes.byref(d)) == 0


@pytest.mark.parametrize("D,G,n_q,mf,groups", [(128, 8, 4, 2, 1), (128, 4, 16, 2, 2), (64, 16, 4, 2, 2),
                                                (256, 8, 4, 2, 1), (512, 8, 4, 1, 2), (128, 16, 8, 2, 4)])
def test_decode_more_than_16_fold_rows(arc, D, G, n_q, mf, groups):
    """GQA-8 x 4 tokens (32 rows), GQA-4 x a 16-token ubatch (64 rows) and more: 32 fold
    rows per CTA (two m16 fragments; one at D = 512) in row groups along the fold."""
    d = decode_args(arc, arc.ARC_KV_Q8_0, n_seq=2, n_q=n_q, H=8 * G, Hkv=8, D=D, n_kv=4096)
    info = arc.plan(arc.ARC_OP_DECODE, d)
    assert info["kernel"] == "decode_ws_kernel<q8_0>" and info["tile_m"] == 16 * mf
    assert info["n_ctas"] == 2 * 8 * groups * info["splits"]
    ws = arc.lib().arc_decode_workspace_size(ctypes.byref(d))
    assert ws == 2 * 8 * groups * info["splits"] * 16 * mf * (D + 2) * 4
    d.k_cache = FAKE + 8                                # not 16-byte aligned: the CUDA-core kernel
    assert arc.plan(arc.ARC_OP_DECODE, d)["kernel"] == "simple_decode_kernel"


def test_decode_workspace_errors_come_before_any_launch(arc):
    L = arc.lib()
    d = decode_args(arc, arc.ARC_KV_Q8_0)
    ws = L.arc_decode_workspace_size(ctypes.byref(d))
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, ws, None) == arc.ARC_ERR_WORKSPACE            # missing
    assert L.arc_attn_decode_q8(ctypes.byref(d), FAKE, ws - 4, None) == arc.ARC_ERR_WORKSPACE        # short
    assert L.arc_attn_decode_q8(ctypes.byref(d), FAKE + 128, ws, None) == arc.ARC_ERR_WORKSPACE      # unaligned


@pytest.mark.parametrize("change,want", [
    ("D=384", "ARC_ERR_UNSUPPORTED"), ("H%Hkv", "ARC_ERR_INVALID_ARG"), ("q misaligned", "ARC_ERR_INVALID_ARG"),
    ("cache misaligned", "ARC_ERR_INVALID_ARG"), ("tokens past n_tok", "ARC_ERR_INVALID_ARG"),
    ("cells past n_cells", "ARC_ERR_INVALID_ARG"), ("lse NULL", "ARC_ERR_INVALID_ARG"),
    ("negative kv_begin", "ARC_ERR_INVALID_ARG"),
])
def test_decode_validation(arc, change, want):
    d = decode_args(arc, arc.ARC_KV_Q4_0, n_seq=2, n_q=2, n_kv=256)
    if change == "D=384":
        d.D = 384
    elif change == "H%Hkv":
        d.Hkv = 6
    elif change == "q misaligned":
        d.q = FAKE + 4
    elif change == "cache misaligned":
        d.v_cache = FAKE + 2
    elif change == "tokens past n_tok":
        d.n_tok = 3
    elif change == "cells past n_cells":
        d.n_cells = 511
    elif change == "lse NULL":
        d.lse = None
    else:
        d.seqs[1].kv_begin = -1
    assert arc.lib().arc_attn_decode_q8(ctypes.byref(d), FAKE, 1 << 30, None) == getattr(arc, want)


# --------------------------------------------------------------------------------- dense
def test_dense_simple_fallback_and_unsupported_layouts(arc):
    """bf16 with rows that are not 16-byte aligned: refused unless FORCE_SIMPLE asks for the CUDA-core kernel."""
    a = arc.AttnArgs()
    a.dtype, a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = arc.ARC_DTYPE_BF16, 1, 4, 1, 64, 64, 64, 64
    a.q, a.k, a.v, a.o, a.lse = (FAKE,) * 5
    for name, shape in (("q", (1, 4, 64, 64)), ("k", (1, 1, 64, 64)), ("v", (1, 1, 64, 64)), ("o", (1, 4, 64, 64))):
        setattr(a, name + "_strides", (arc._i64 * 3)(*contiguous(*shape)))
    assert arc.plan(arc.ARC_OP_ATTN, a)["tensor_cores"] == 1
    a.k = FAKE + 2
    assert arc.lib().arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_UNSUPPORTED
    a.flags = arc.ARC_FLAG_FORCE_SIMPLE
    info = arc.plan(arc.ARC_OP_ATTN, a)
    assert info["kernel"] == "simple_attn_kernel" and info["n_ctas"] == (4 * 64 + 3) // 4


# ----------------------------------------------------------------------- broadcast strides
def dense_args(arc, B=2, H=4, Hkv=2, T=64, D=64):
    a = arc.AttnArgs()
    a.dtype, a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = arc.ARC_DTYPE_BF16, B, H, Hkv, T, T, D, D
    a.q, a.k, a.v, a.o, a.lse = (FAKE,) * 5
    for name, shape in (("q", (B, H, T, D)), ("k", (B, Hkv, T, D)), ("v", (B, Hkv, T, D)), ("o", (B, H, T, D))):
        setattr(a, name + "_strides", (arc._i64 * 3)(*contiguous(*shape)))
    return a


@pytest.mark.parametrize("name,dim", [("k", 0), ("v", 0), ("q", 0), ("k", 1), ("v", 1)])
def test_broadcast_inputs_are_refused_by_the_tma_path(arc, name, dim):
    """A zero stride over an extent above one cannot be a TMA map stride; it must not be
    replaced by the contiguous default (that map would run past the allocation)."""
    a = dense_args(arc)
    assert arc.plan(arc.ARC_OP_ATTN, a)["tensor_cores"] == 1
    getattr(a, name + "_strides")[dim] = 0
    assert arc.lib().arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_UNSUPPORTED
    a.flags = arc.ARC_FLAG_FORCE_SIMPLE
    assert arc.plan(arc.ARC_OP_ATTN, a)["kernel"] == "simple_attn_kernel"


def test_zero_strides_over_extent_one_still_take_the_tma_path(arc):
    a = dense_args(arc, B=1, Hkv=1)
    a.q_strides[0] = a.k_strides[0] = a.v_strides[0] = a.k_strides[1] = a.v_strides[1] = 0
    assert arc.plan(arc.ARC_OP_ATTN, a)["tensor_cores"] == 1


@pytest.mark.parametrize("dim", [0, 1, 2])
def test_aliasing_output_rows_are_invalid(arc, dim):
    a = dense_args(arc)
    a.o_strides[dim] = 0
    assert arc.lib().arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_INVALID_ARG
    m = mla_args(arc, Tq=256, Tk=256)
    m.o_strides[dim] = 0
    assert arc.lib().arc_mla_fwd(ctypes.byref(m), None) == arc.ARC_ERR_INVALID_ARG
    if dim < 2:
        s = sparse_args(arc, Sq=4, topk=64)
        s.o_strides[dim] = 0
        assert arc.lib().arc_sparse_mla_fwd(ctypes.byref(s), None) == arc.ARC_ERR_INVALID_ARG


@pytest.mark.parametrize("field,dim", [("k_rope_strides", 0), ("k_nope_strides", 1), ("v_strides", 0),
                                       ("q_rope_strides", 0)])
def test_mla_broadcast_inputs_are_refused_by_the_tma_path(arc, field, dim):
    m = mla_args(arc, Tq=256, Tk=256)
    getattr(m, field)[dim] = 0
    assert arc.lib().arc_mla_fwd(ctypes.byref(m), None) == arc.ARC_ERR_UNSUPPORTED
    m.flags = arc.ARC_FLAG_FORCE_SIMPLE
    assert arc.plan(arc.ARC_OP_MLA, m)["kernel"] == "simple_attn_kernel"


@pytest.mark.parametrize("call,field,dim", [("mla", "q_nope_strides", 2), ("mla", "k_rope_strides", 1),
                                            ("mla", "o_strides", 0), ("sparse", "kv_stride", None),
                                            ("sparse", "idx_stride", None), ("sparse", "q_strides", 1)])
def test_negative_strides_are_invalid(arc, call, field, dim):
    x = mla_args(arc, Tq=256, Tk=256) if call == "mla" else sparse_args(arc, Sq=4, topk=64)
    if dim is None:
        setattr(x, field, -8)
    else:
        getattr(x, field)[dim] = -8
    fn = arc.lib().arc_mla_fwd if call == "mla" else arc.lib().arc_sparse_mla_fwd
    assert fn(ctypes.byref(x), None) == arc.ARC_ERR_INVALID_ARG



def test_tensor_core_shape_sets_match_the_header(arc):
    """The (D, Dv) pairs arc_plan sends to tensor-core kernels are exactly those the header lists."""
    import re
    text = open(os.path.join(ROOT, "include", "arc_attn.h")).read()

    def pairs_after(marker):
        seg = text[text.index(marker):]
        seg = seg[:seg.index("}") + 1]
        return {tuple(int(x) for x in m) for m in re.findall(r"\((\d+),\s*(\d+)\)", seg)}

    dense_doc = pairs_after("dtype BF16: (D, Dv) in {")
    mla_doc = pairs_after("with (Dn + Dr, Dv) in {")
    dense, mla = set(), set()
    for D in (64, 128, 192, 256, 320, 384, 512):
        for Dv in (64, 128, 192, 256, 384, 512):
            a = arc.AttnArgs()
            B, H, Hkv, T = 1, 4, 2, 64
            a.dtype, a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = arc.ARC_DTYPE_BF16, B, H, Hkv, T, T, D, Dv
            a.q, a.k, a.v, a.o, a.lse = (FAKE,) * 5
            for name, shape in (("q", (B, H, T, D)), ("k", (B, Hkv, T, D)), ("v", (B, Hkv, T, Dv)), ("o", (B, H, T, Dv))):
                setattr(a, name + "_strides", (arc._i64 * 3)(*contiguous(*shape)))
            info = arc.PlanInfo()
            if arc.lib().arc_plan(arc.ARC_OP_ATTN, ctypes.byref(a), ctypes.byref(info)) == arc.ARC_OK:
                assert info.tensor_cores == 1
                dense.add((D, Dv))
    for Dn in (64, 128, 192):
        for Dr in (64, 128):
            for Dv in (64, 128, 256):
                m = mla_args(arc, B=1, H=2, Tq=64, Tk=64, Dn=Dn, Dr=Dr, Dv=Dv)
                if arc.lib().arc_plan(arc.ARC_OP_MLA, ctypes.byref(m), ctypes.byref(arc.PlanInfo())) == arc.ARC_OK:
                    mla.add((Dn + Dr, Dv))
    assert dense == dense_doc and len(dense) == 10
    assert mla == mla_doc and len(mla) == 5


# -------------------------------------------------------------------------- sparse decode
@pytest.mark.parametrize("Sq,want_splits", [(1, 12), (4, 12), (37, 4), (74, 2), (148, 1), (400, 1)])
def test_sparse_decode_splits_the_top_k_when_tokens_leave_sms_idle(arc, Sq, want_splits):
    """64 heads, 2176 slots (34 tiles of 64): few tokens cut their lists into chunks of whole
    tiles, at least two tiles each and at most 16 chunks; enough tokens run one CTA each."""
    s = sparse_args(arc, Sq=Sq, topk=2176, D=512, Dv=512)
    info = arc.plan(arc.ARC_OP_SPARSE_DECODE, s)
    assert info["splits"] == want_splits and info["tensor_cores"] == 1
    ws = arc.lib().arc_sparse_decode_workspace_size(ctypes.byref(s))
    if want_splits == 1:
        assert info["kernel"] == "sparse_tc_kernel" and info["launches"] == 1 and ws == 0
    else:
        assert info["kernel"] == "sparse_tc_kernel<split>" and info["launches"] == 2
        tiles = -(-34 // min(16, SMS // Sq, 17))
        assert want_splits == -(-2176 // (tiles * 64))
        assert ws == want_splits * Sq * 64 * (512 + 1) * 4
        assert info["n_ctas"] == Sq * want_splits
        # a missing or short workspace is refused before anything launches
        assert arc.lib().arc_sparse_mla_decode(ctypes.byref(s), None, ws, None) == arc.ARC_ERR_WORKSPACE
        assert arc.lib().arc_sparse_mla_decode(ctypes.byref(s), FAKE, ws - 4, None) == arc.ARC_ERR_WORKSPACE


# ------------------------------------------------------------------------------- backward
def bwd_args(arc, B=1, H=64, Hkv=8, T=1400, D=128, Dv=128, sinks=True):
    a = arc.BwdArgs()
    a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = B, H, Hkv, T, T, D, Dv
    for f in ("q", "k", "v", "o", "dout", "lse", "dq", "dk", "dv"):
        setattr(a, f, FAKE)
    if sinks:
        a.sinks, a.dsinks = FAKE, FAKE
    a.q_strides = a.o_strides = a.do_strides = a.dq_strides = (arc._i64 * 3)(*contiguous(B, H, T, D))
    a.o_strides = a.do_strides = (arc._i64 * 3)(*contiguous(B, H, T, Dv))
    a.k_strides = a.dk_strides = (arc._i64 * 3)(*contiguous(B, Hkv, T, D))
    a.v_strides = a.dv_strides = (arc._i64 * 3)(*contiguous(B, Hkv, T, Dv))
    a.scale, a.causal = D ** -0.5, 1
    return a


def test_backward_plans_the_tensor_core_kernels_and_its_workspace(arc):
    """GQA-8 at d 128, T 1400 with sinks: 8 kv heads x 11 key tiles = 88 dK/dV CTAs, fewer
    than two per SM, so each key tile's 88 fold tiles are split over 4 CTAs (22 each) whose
    fp32 partials a fifth launch adds up; delta and the partials in the workspace."""
    def expect_split(base, n_qt):
        want = 2 * SMS
        r = 1 if base >= want else min(-(-want // base), n_qt // 4)
        r = max(1, min(r, 64))
        tps = -(-n_qt // r)
        return -(-n_qt // tps)

    a = bwd_args(arc)
    info = arc.plan(arc.ARC_OP_ATTN_BWD, a)
    assert info["kernel"] == "bwd_dkdv_kernel+bwd_dq_kernel" and info["tensor_cores"] == 1
    assert info["splits"] == expect_split(8 * 11, 88) == 4
    assert info["n_ctas"] == 8 * 11 * 4 and info["launches"] == 5
    delta = 64 * 1400 * 4
    assert arc.lib().arc_attn_bwd_workspace_size(ctypes.byref(a)) == delta + 4 * 8 * 1400 * 256 * 4
    # few key tiles, no sinks
    a = bwd_args(arc, H=16, Hkv=2, T=260, sinks=False)
    info = arc.plan(arc.ARC_OP_ATTN_BWD, a)
    n_qt = -(-8 * 260 // 128)
    assert info["splits"] == expect_split(2 * 3, n_qt) > 1 and info["launches"] == 4
    delta = -(-16 * 260 * 4 // 256) * 256
    assert arc.lib().arc_attn_bwd_workspace_size(ctypes.byref(a)) == delta + info["splits"] * 2 * 260 * 256 * 4
    # enough key tiles: no split, no reduction
    info = arc.plan(arc.ARC_OP_ATTN_BWD, bwd_args(arc, B=2, H=16, Hkv=16, T=4096, sinks=False))
    assert info["splits"] == 1 and info["launches"] == 3
    # d_qk 192 / d_v 128: 64-row fold tiles for dK / dV (TMEM room)
    info = arc.plan(arc.ARC_OP_ATTN_BWD, bwd_args(arc, H=16, Hkv=16, T=4096, D=192, Dv=128, sinks=False))
    assert info["tile_n"] == 64 and info["d_slice"] == 192


def test_backward_validation_before_any_launch(arc):
    L = arc.lib()
    a = bwd_args(arc, D=256, Dv=256)
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == arc.ARC_ERR_UNSUPPORTED
    a = bwd_args(arc)
    a.dsinks = None                                     # sinks without a place for their gradient
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == arc.ARC_ERR_INVALID_ARG
    a = bwd_args(arc)
    a.Hkv = 7
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == arc.ARC_ERR_INVALID_ARG
    a = bwd_args(arc)
    a.q = FAKE + 8                                      # not 16-byte aligned
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == arc.ARC_ERR_UNSUPPORTED
    a = bwd_args(arc)
    ws = L.arc_attn_bwd_workspace_size(ctypes.byref(a))
    assert L.arc_attn_bwd(ctypes.byref(a), None, ws, None) == arc.ARC_ERR_WORKSPACE
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE, ws - 4, None) == arc.ARC_ERR_WORKSPACE
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE + 16, ws, None) == arc.ARC_ERR_WORKSPACE
    a.scale = float("nan")
    assert L.arc_attn_bwd(ctypes.byref(a), FAKE, ws, None) == arc.ARC_ERR_INVALID_ARG


def mla_bwd_args(arc, B=2, H=16, T=4096, Dn=128, Dr=64, Dv=128):
    a = arc.MlaBwdArgs()
    a.B, a.H, a.Tq, a.Tk, a.Dn, a.Dr, a.Dv = B, H, T, T, Dn, Dr, Dv
    for f in ("q_nope", "q_rope", "k_nope", "k_rope", "v", "o", "dout", "lse", "dq_nope", "dq_rope", "dk_nope",
              "dk_rope", "dv"):
        setattr(a, f, FAKE)
    a.q_nope_strides = a.k_nope_strides = a.dq_nope_strides = a.dk_nope_strides = (arc._i64 * 3)(*contiguous(B, H, T, Dn))
    a.q_rope_strides = a.dq_rope_strides = (arc._i64 * 3)(*contiguous(B, H, T, Dr))
    a.k_rope_strides = a.dk_rope_strides = (arc._i64 * 2)(*contiguous(B, T, Dr))
    a.v_strides = a.o_strides = a.do_strides = a.dv_strides = (arc._i64 * 3)(*contiguous(B, H, T, Dv))
    a.scale, a.causal = (Dn + Dr) ** -0.5, 1
    return a


def test_mla_backward_plan_workspace_and_validation(arc):
    """MLA prefill's shape: 2 x 16 heads x 32 key tiles = 1024 dK/dV CTAs (no split), 64-row
    fold tiles at d_qk 192; the workspace holds delta and each head's fp32 share of dk_rope;
    four launches: delta, dK / dV, the sum over heads, dQ."""
    L = arc.lib()
    a = mla_bwd_args(arc)
    info = arc.plan(arc.ARC_OP_MLA_BWD, a)
    assert info["kernel"] == "bwd_dkdv_kernel<mla>+bwd_dq_kernel" and info["splits"] == 1
    assert info["n_ctas"] == 2 * 16 * 32 and info["tile_n"] == 64 and info["launches"] == 4
    ws = L.arc_mla_bwd_workspace_size(ctypes.byref(a))
    assert ws == 2 * 16 * 4096 * 4 + 2 * 16 * 4096 * 64 * 4
    assert L.arc_mla_bwd(ctypes.byref(a), None, ws, None) == arc.ARC_ERR_WORKSPACE
    for field, value, want in (("Dr", 0, arc.ARC_ERR_UNSUPPORTED), ("Dn", 96, arc.ARC_ERR_UNSUPPORTED),
                               ("Dv", 256, arc.ARC_ERR_UNSUPPORTED)):
        b = mla_bwd_args(arc)
        setattr(b, field, value)
        assert L.arc_mla_bwd(ctypes.byref(b), FAKE, 1 << 34, None) == want, field
    b = mla_bwd_args(arc)
    b.k_rope = FAKE + 8                                  # not 16-byte aligned
    assert L.arc_mla_bwd(ctypes.byref(b), FAKE, 1 << 34, None) == arc.ARC_ERR_UNSUPPORTED
    b = mla_bwd_args(arc)
    b.dq_rope = None
    assert L.arc_mla_bwd(ctypes.byref(b), FAKE, 1 << 34, None) == arc.ARC_ERR_INVALID_ARG
