"""The boundary is a C ABI: a plain C program, compiled against include/arc_attn.h
and linked to the built library with no Python or torch in between, plans the
GQA prefill and the quantised decode, sizes a decode workspace, asks for the
library's default softmax scale by flag, and gets the documented validation errors back (host logic only: nothing is launched)."""
import os
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CLIENT = r"""
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "arc_attn.h"

#define FAKE ((const void *)(size_t)(1u << 20))   /* never dereferenced: nothing launches */

int main(void)
{
    if (arc_abi_version() != ARC_ABI_VERSION) return 1;

    arc_attn_args a;
    memset(&a, 0, sizeof a);
    a.dtype = ARC_DTYPE_BF16;
    a.B = 1; a.H = 64; a.Hkv = 8; a.Tq = 1400; a.Tk = 1400; a.D = 512; a.Dv = 512;
    a.q = FAKE; a.k = FAKE; a.v = FAKE; a.o = (void *)FAKE; a.lse = (float *)FAKE;
    int64_t qs[3] = {64LL * 1400 * 512, 1400LL * 512, 512}, ks[3] = {8LL * 1400 * 512, 1400LL * 512, 512};
    memcpy(a.q_strides, qs, sizeof qs); memcpy(a.o_strides, qs, sizeof qs);
    memcpy(a.k_strides, ks, sizeof ks); memcpy(a.v_strides, ks, sizeof ks);
    a.scale = 0.044194173f; a.causal = 1;
    arc_plan_info info;
    memset(&info, 0, sizeof info);
    if (arc_plan(ARC_OP_ATTN, &a, &info) != ARC_OK) return 2;
    printf("attn %s tensor_cores=%d tile_m=%d d_slice=%d\n", info.kernel, info.tensor_cores, info.tile_m, info.d_slice);

    /* ARC_FLAG_DEFAULT_SCALE: the library takes 1/sqrt(D) and ignores the field, so
       even a NaN there is accepted; without the flag a NaN scale is refused */
    a.scale = NAN;
    if (arc_plan(ARC_OP_ATTN, &a, &info) != ARC_ERR_INVALID_ARG) return 6;
    a.flags = ARC_FLAG_DEFAULT_SCALE;
    if (arc_plan(ARC_OP_ATTN, &a, &info) != ARC_OK) return 7;
    a.flags = 0;
    a.scale = 0.044194173f;

    a.Hkv = 7;                                   /* 64 heads do not divide over 7 kv heads */
    if (arc_attn_fwd(&a, NULL) != ARC_ERR_INVALID_ARG) return 3;
    printf("status %s\n", arc_status_string(ARC_ERR_INVALID_ARG));

    arc_seq seqs[4];
    for (int s = 0; s < 4; ++s) { seqs[s].q_begin = 4 * s; seqs[s].n_q = 4; seqs[s].kv_begin = 8192 * s; seqs[s].n_kv = 8192; }
    arc_decode_args d;
    memset(&d, 0, sizeof d);
    d.kv_type = ARC_KV_Q8_0; d.n_tok = 16; d.H = 32; d.Hkv = 8; d.D = 128; d.n_cells = 32768; d.n_seq = 4;
    d.q = (const float *)FAKE; d.k_cache = FAKE; d.v_cache = FAKE; d.seqs = seqs;
    d.o = (float *)FAKE; d.lse = (float *)FAKE; d.scale = 0.088388348f;
    memset(&info, 0, sizeof info);
    if (arc_plan(ARC_OP_DECODE, &d, &info) != ARC_OK) return 4;
    size_t ws = arc_decode_workspace_size(&d);
    printf("decode %s splits=%d launches=%d workspace=%zu\n", info.kernel, info.splits, info.launches, ws);
    if (ws == 0 || arc_attn_decode_q8(&d, NULL, ws, NULL) != ARC_ERR_WORKSPACE) return 5;
    return 0;
}
"""


def test_plain_c_client_plans_and_validates():
    import exact_attention_131_b200 as arc
    if not os.path.exists(arc.LIB_PATH):
        from exact_attention_131_b200 import build
        build.build()
    libdir = os.path.dirname(arc.LIB_PATH)
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "client.c"), os.path.join(d, "client")
        open(src, "w").write(CLIENT)
        subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                               "-o", exe, "-L", libdir, "-larc_attn", "-lm", "-Wl,-rpath," + libdir])
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    lines = r.stdout.splitlines()
    assert lines[0] == "attn tc_attn_pair_kernel tensor_cores=1 tile_m=256 d_slice=256"
    assert lines[1] == "status invalid argument"
    assert lines[2].startswith("decode decode_ws_kernel<q8_0> ") and "launches=2" in lines[2]
