"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, the ctypes mirror matches the C struct layout, and argument
validation refuses bad calls before any CUDA work (no GPU needed)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "arc_attn.h")


@pytest.fixture(scope="module")
def arc():
    import exact_attention_131_b200 as arc
    if not os.path.exists(arc.LIB_PATH):
        from exact_attention_131_b200 import build
        build.build()
    arc.lib()
    return arc


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(arc_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(arc):
    names = declared_functions()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", arc.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(arc.EXPORTS) <= set(names)


def test_abi_version_and_status_strings(arc):
    m = re.search(r"#define ARC_ABI_VERSION (\d+)", open(HEADER).read())
    assert arc.abi_version() == int(m.group(1))
    for s in range(6):
        assert arc.status_string(s) and "unknown" not in arc.status_string(s)


STRUCTS = {
    "arc_attn_args": ("AttnArgs", ["q", "k_strides", "o", "lse", "sinks", "scale", "causal", "flags", "status"]),
    "arc_mla_args": ("MlaArgs", ["q_rope", "k_rope_strides", "v", "lse", "scale", "status"]),
    "arc_sparse_args": ("SparseArgs", ["kv", "v_stride", "idx", "o_strides", "sinks", "scale", "status"]),
    "arc_decode_args": ("DecodeArgs", ["q", "seqs", "o", "lse", "scale", "flags", "status"]),
    "arc_plan_info": ("PlanInfo", ["kernel", "tensor_cores", "splits", "launches"]),
    "arc_seq": ("Seq", ["q_begin", "n_kv"]),
    "arc_merge_args": ("MergeArgs", ["dtype", "o_parts", "lse_parts", "sinks", "sink_rows", "o", "lse"]),
}


def test_ctypes_mirror_matches_c_layout(arc):
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void){"]
    for cname, (_, fields) in STRUCTS.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f in fields:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(src, "w").write("\n".join(lines))
        subprocess.check_call(["gcc", src, "-o", exe])
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    for line in out.splitlines():
        cname, f, val = line.split()
        cls = getattr(arc, STRUCTS[cname][0])
        got = ctypes.sizeof(cls) if f == "size" else getattr(cls, f).offset
        assert got == int(val), (cname, f, got, val)


def test_validation_rejects_before_any_launch(arc):
    L = arc.lib()
    a = arc.AttnArgs()
    a.dtype, a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = arc.ARC_DTYPE_BF16, 1, 3, 2, 8, 8, 64, 64
    assert L.arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_INVALID_ARG        # H % Hkv
    a.H = 4
    assert L.arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_INVALID_ARG        # NULL pointers
    a.D = 1024
    assert L.arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_UNSUPPORTED
    a.dtype = 7
    assert L.arc_attn_fwd(ctypes.byref(a), None) == arc.ARC_ERR_INVALID_ARG
    assert L.arc_attn_fwd(None, None) == arc.ARC_ERR_INVALID_ARG
    # B == 0 or Tq == 0 is a valid call with nothing to do
    b = arc.AttnArgs()
    b.dtype, b.B, b.H, b.Hkv, b.Tq, b.Tk, b.D, b.Dv = arc.ARC_DTYPE_BF16, 0, 4, 2, 8, 8, 64, 64
    assert L.arc_attn_fwd(ctypes.byref(b), None) == arc.ARC_OK

    m = arc.MlaArgs()
    m.B, m.H, m.Tq, m.Tk, m.Dn, m.Dr, m.Dv = 1, 2, 4, 4, 128, 64, 128
    assert L.arc_mla_fwd(ctypes.byref(m), None) == arc.ARC_ERR_INVALID_ARG

    s = arc.SparseArgs()
    s.Sq, s.H, s.Skv, s.Dqk, s.Dv, s.topk = 2, 64, 10, 512, 600, 4
    assert L.arc_sparse_mla_fwd(ctypes.byref(s), None) == arc.ARC_ERR_UNSUPPORTED   # Dv > 512


def test_decode_validation_and_workspace_size(arc):
    L = arc.lib()
    seqs = arc.make_seqs([0, 4], [4, 4], [0, 100], [100, 50])
    d = arc.DecodeArgs()
    d.kv_type, d.n_tok, d.H, d.Hkv, d.D, d.n_cells, d.n_seq = arc.ARC_KV_Q8_0, 8, 32, 8, 128, 150, 2
    d.seqs = ctypes.cast(seqs, ctypes.POINTER(arc.Seq))
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, 0, None) == arc.ARC_ERR_INVALID_ARG  # NULL tensors
    ws = L.arc_decode_workspace_size(ctypes.byref(d))
    assert ws > 0 and ws % 4 == 0
    d.kv_type = 3
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, 0, None) == arc.ARC_ERR_INVALID_ARG
    assert L.arc_decode_workspace_size(ctypes.byref(d)) == 0
    d.kv_type = arc.ARC_KV_Q8_0
    bad = arc.make_seqs([0], [5], [0], [4])                  # n_kv < n_q
    d.seqs, d.n_seq = ctypes.cast(bad, ctypes.POINTER(arc.Seq)), 1
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, 0, None) == arc.ARC_ERR_INVALID_ARG
    many = arc.make_seqs([0] * 65, [0] * 65, [0] * 65, [0] * 65)
    d.seqs, d.n_seq = ctypes.cast(many, ctypes.POINTER(arc.Seq)), 65
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, 0, None) == arc.ARC_ERR_UNSUPPORTED
    wide = arc.make_seqs([0], [33], [0], [40])               # g * n_q = 4 * 33 = 132 > 128 fold rows
    d.seqs, d.n_seq, d.H, d.Hkv, d.n_tok = ctypes.cast(wide, ctypes.POINTER(arc.Seq)), 1, 32, 8, 33
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, 0, None) == arc.ARC_ERR_UNSUPPORTED
    ok = arc.make_seqs([0], [32], [0], [40])                 # 128 fold rows: accepted (NULL tensors refused next)
    d.seqs = ctypes.cast(ok, ctypes.POINTER(arc.Seq))
    assert L.arc_attn_decode_q8(ctypes.byref(d), None, 0, None) == arc.ARC_ERR_INVALID_ARG


def test_merge_validation_before_any_launch(arc):
    L = arc.lib()
    m = arc.MergeArgs()
    m.n_parts, m.rows, m.dv, m.dtype = 2, 10, 128, arc.ARC_DTYPE_F32
    assert L.arc_attn_merge(ctypes.byref(m), None) == arc.ARC_ERR_INVALID_ARG     # NULL pointers
    fake = 1 << 20                                                                # never dereferenced
    for i in range(2):
        m.o_parts[i], m.lse_parts[i] = fake, fake
    m.o, m.lse = fake, fake
    for field, value, want in (("n_parts", 0, arc.ARC_ERR_INVALID_ARG), ("n_parts", 17, arc.ARC_ERR_INVALID_ARG),
                               ("dv", 127, arc.ARC_ERR_INVALID_ARG), ("dv", 2048, arc.ARC_ERR_UNSUPPORTED),
                               ("dtype", 7, arc.ARC_ERR_INVALID_ARG), ("rows", -1, arc.ARC_ERR_INVALID_ARG)):
        old = getattr(m, field)
        setattr(m, field, value)
        assert L.arc_attn_merge(ctypes.byref(m), None) == want, (field, value)
        setattr(m, field, old)
    m.o_parts[1] = fake + 4                                                       # misaligned part
    assert L.arc_attn_merge(ctypes.byref(m), None) == arc.ARC_ERR_INVALID_ARG
    m.o_parts[1] = fake
    m.sinks, m.sink_heads, m.sink_rows = fake, 0, 5                               # sinks without a head count
    assert L.arc_attn_merge(ctypes.byref(m), None) == arc.ARC_ERR_INVALID_ARG
    m.sinks, m.rows = None, 0                                                     # nothing to do
    assert L.arc_attn_merge(ctypes.byref(m), None) == arc.ARC_OK
    info = arc.PlanInfo()
    m.rows = 100
    assert L.arc_plan(arc.ARC_OP_MERGE, ctypes.byref(m), ctypes.byref(info)) == arc.ARC_OK
    assert info.kernel.decode() == "merge_kernel" and info.launches == 1 and info.n_ctas == 13


def test_plan_names_the_tensor_core_kernels(arc):
    """The engagement record is pure host logic: bf16 shapes plan tcgen05 / mma kernels."""
    a = arc.AttnArgs()
    a.dtype, a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = arc.ARC_DTYPE_BF16, 1, 64, 8, 1400, 1400, 512, 512
    base = 1 << 20  # any 16-byte-aligned non-NULL placeholder; arc_plan never dereferences
    a.q, a.k, a.v, a.o, a.lse = base, base, base, base, base
    a.q_strides = (arc._i64 * 3)(64 * 1400 * 512, 1400 * 512, 512)
    a.k_strides = (arc._i64 * 3)(8 * 1400 * 512, 1400 * 512, 512)
    a.v_strides = (arc._i64 * 3)(8 * 1400 * 512, 1400 * 512, 512)
    a.o_strides = (arc._i64 * 3)(64 * 1400 * 512, 1400 * 512, 512)
    info = arc.plan(arc.ARC_OP_ATTN, a)
    assert info["kernel"] == "tc_attn_pair_kernel" and info["d_slice"] == 256 and info["tmem_cols"] == 512
    # persistent: one cluster per two SMs (148 on B200; the planner's default without a GPU)
    # walks the 44 x 8 row-tile pairs, running both d_v slices of each in turn
    assert info["n_ctas"] == 2 * min(44 * 8, 148 // 2)
    assert info["tile_m"] == 256
    a.flags = arc.ARC_FLAG_SINGLE_CTA
    info = arc.plan(arc.ARC_OP_ATTN, a)
    assert info["kernel"] == "tc_attn_kernel" and info["d_slice"] == 256
    assert info["n_ctas"] == 88 * 8 * 2            # ceil(8*1400/128) tiles x 8 kv heads x 2 slices
    a.flags = arc.ARC_FLAG_FORCE_SIMPLE
    assert arc.plan(arc.ARC_OP_ATTN, a)["kernel"] == "simple_attn_kernel"
    a.flags, a.dtype = 0, arc.ARC_DTYPE_F32
    assert arc.plan(arc.ARC_OP_ATTN, a)["kernel"] == "simple_attn_kernel"


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "exact_attention_131_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "arc_oracle" not in text and "liboracle" not in text, f
