"""Decode-shaped sparse MLA (arc_sparse_mla_decode) against the fp64 oracle.

"TensorRT-LLM: FlashMLA without -rdc" lists a sparse decode kernel for 64 heads
beside the sparse prefill.  A decode batch has few query tokens, each attending
with its 64 heads to its own top-k rows of a shared latent pool; the call cuts
each token's list over several CTAs and merges the parts by their LSE.  Every
case is compared element by element with the oracle's sparse attention (with
sinks where given), the split count is asserted through arc_plan, and the
one-CTA-per-token arc_sparse_mla_fwd is run on the same inputs as a control.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import exact_attention_131_b200 as arc
from tests._util import TOL_O_BF16, compare, dev, status_word

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Sq,Skv,Dqk,Dv,topk,sep_v,sinks", [
    (1, 8192, 512, 512, 2176, False, False),     # one token, the page's top-k at d_qk 512
    (4, 8192, 512, 512, 2176, False, True),      # sinks enter once, in the merge
    (5, 4000, 512, 512, 700, False, False),      # a ragged last chunk
    (37, 8192, 512, 512, 2176, False, True),     # fewer, longer chunks
    (3, 3000, 128, 64, 1000, True, True),        # a separate V
    (200, 3000, 512, 512, 300, False, False),    # enough tokens: one CTA per token, no split
])
def test_sparse_decode_matches_oracle(Sq, Skv, Dqk, Dv, topk, sep_v, sinks):
    c = W.sparse_case(Sq, 64, Skv, Dqk, Dv, topk, pad_mode="random", separate_v=sep_v, sinks=sinks,
                      seed=300 + Sq + topk)
    if Sq > 2:
        c.idx[1, :] = -1                       # a token whose every slot is padding
    q, kv, idx = dev(c.q), dev(c.kv), dev(c.idx)
    v = dev(c.v) if sep_v else None
    s = dev(c.sinks) if sinks else None
    st = status_word()
    o, lse = arc.sparse_mla_decode(q, kv, idx, Dv=Dv, v=v, scale=c.scale, sinks=s, status=st)
    torch.cuda.synchronize()
    info = arc.plan_sparse_decode(q, kv, idx, o, lse, Dv=Dv, v=v, sinks=s)
    if Sq * 1 >= 148:
        assert info["kernel"] == "sparse_tc_kernel" and info["splits"] == 1
    else:
        assert info["kernel"] == "sparse_tc_kernel<split>" and info["splits"] >= 2 and info["launches"] == 2
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK
    o2, l2 = arc.sparse_mla_fwd(q, kv, idx, Dv=Dv, v=v, scale=c.scale, sinks=s)
    torch.cuda.synchronize()
    compare(o2, l2, ro, rl, TOL_O_BF16)


def test_sparse_decode_workspace_reuse_with_garbage():
    """The workspace needs no initialisation and may be reused call after call."""
    c = W.sparse_case(4, 64, 8192, 512, 512, 2176, seed=310)
    q, kv, idx = dev(c.q), dev(c.kv), dev(c.idx)
    o = torch.empty(4, 64, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(4, 64, device="cuda")
    n = arc.sparse_decode_workspace_size(q, kv, idx, o, lse)
    assert n > 0
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")
    ro, rl = oracle.run_case(c)
    for _ in range(3):
        o.fill_(float("nan"))
        arc.sparse_mla_decode(q, kv, idx, scale=c.scale, out=o, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        compare(o, lse, ro, rl, TOL_O_BF16)
