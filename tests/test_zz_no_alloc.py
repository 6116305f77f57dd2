"""The allocation-free decode entry point, against the workspace entry point.

arc_attn_decode_q8_noalloc serves callers that cannot call cudaMalloc (an
engine whose planner owns all device memory, a fixed memory budget): it keeps
its split-KV partials in the library's own static 8 MiB device buffer.  These
checks call it through the C ABI and compare it with arc_attn_decode_q8 fed a
caller workspace, over consecutive calls that reuse the shared buffer.  The
file name sorts last so a stop-at-first-failure run has run everything else.
"""
import numpy as np
import pytest
import torch

import workloads as W
import exact_attention_131_b200 as arc
from tests._util import TOL_LSE, TOL_O_BF16, compare, dev, host

pytestmark = pytest.mark.gpu


def _inputs(c):
    return dev(c.q), dev(c.k_cache), dev(c.v_cache)


def _kw(c):
    return dict(kv_type=c.kv_type, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                n_kv=c.n_kv, scale=c.scale)


def test_noalloc_decode_matches_workspace_entry_on_consecutive_calls():
    cases = [W.config(5, kv_type=W.KV_Q8_0), W.config(5, kv_type=W.KV_Q4_0),
             W.decode_case(3, 2, 0, 16, 4, 64, kv_type=W.KV_Q8_0, seed=41, n_q_list=[2, 4, 1],
                           n_kv_list=[900, 33, 5])]
    for c in cases:
        q, kc, vc = _inputs(c)
        o_ref, l_ref = arc.attn_decode_q8(q, kc, vc, **_kw(c))
        torch.cuda.synchronize()
        ro, rl = host(o_ref), host(l_ref)
        for _ in range(2):                      # two calls in a row on the shared buffer
            o = torch.full_like(o_ref, float("nan"))
            lse = torch.full_like(l_ref, float("nan"))
            arc.attn_decode_q8_noalloc(q, kc, vc, out=o, lse=lse, **_kw(c))
            torch.cuda.synchronize()
            compare(o, lse, ro, rl, TOL_O_BF16, TOL_LSE)


def test_noalloc_decode_rejects_calls_beyond_its_buffer():
    # 64 sequences x 32 kv heads of partials need more than the 8 MiB buffer.
    c = W.decode_case(64, 1, 8, 32, 32, 128, kv_type=W.KV_Q8_0, seed=42)
    q, kc, vc = _inputs(c)
    need = arc.decode_workspace_size(c.kv_type, q, c.Hkv, c.n_cells, c.q_begin, c.n_q, c.kv_begin, c.n_kv)
    assert need > arc.NOALLOC_SCRATCH_BYTES
    o = torch.full((c.n_tok, c.H, c.D), 3.0, device="cuda")
    with pytest.raises(arc.ArcError) as e:
        arc.attn_decode_q8_noalloc(q, kc, vc, out=o, **_kw(c))
    assert e.value.status == arc.ARC_ERR_WORKSPACE
    assert torch.all(o == 3.0)
