"""Seeded shape sweep of the quantised decode against the oracle.

"unsloth llama.cpp: dequantize q4_0/q8_0 K/V tiles in the FA MMA kernel" checks its
in-tile dequantising kernel against the CPU backend over a family of
multi-sequence shapes and both cache types, at head dims 128 / 256 / 512 and 3 to
16 tokens per ubatch.  This is the same design over this library's decode: every
combination of cache type, head dim (64 to 512), GQA ratio (1, 4, 16) and
sequence layout (one new token over a long cache; four sequences of up to four
new tokens; ragged sequences up to 16 fold rows; 32 and 64 fold rows, as GQA-8
with 4 tokens or GQA-4 with a 16-token ubatch give), each compared element by
element with the oracle.  The layouts include a sequence whose cache holds only
its new tokens and cache lengths that end inside a tile; the GQA ratios give cell
strides that are and are not 16-byte multiples, so both load paths run where
both exist.
"""
import itertools

import pytest

import oracle
import workloads as W
import exact_attention_131_b200 as arc
from tests._util import TOL_O_BF16, compare, dev, status_word

pytestmark = pytest.mark.gpu

HEADS = [(8, 8), (16, 4), (32, 2)]          # (H, Hkv): g = 1, 4, 16


def layout(name, g):
    """(n_q per sequence, n_kv per sequence)."""
    top = max(1, 16 // g)
    if name == "single":
        return [1], [777]
    if name == "full":
        n = min(4, top)
        return [n] * 4, [130, 64, 1000, n]
    if name == "ragged":
        return [top, 1, max(1, top // 2)], [max(top, 70), 200, 513]
    rows = 32 if name == "rows32" else 64
    n = rows // g
    return [n, max(1, n // 2)], [max(n, 300), 90]


NAMES = ["single", "full", "ragged", "rows32", "rows64"]
CASES = list(itertools.product([W.KV_Q8_0, W.KV_Q4_0], [64, 128, 256, 512], HEADS, NAMES))


def expected_kernel(kv_type, D, H, Hkv, n_q):
    cell = Hkv * D // 32 * (34 if kv_type == W.KV_Q8_0 else 18)
    rows = max(H // Hkv * n for n in n_q)
    if cell % 16 == 0:
        return "decode_ws_kernel"
    return "decode_split_kernel" if D <= 128 and rows <= 16 else "simple_decode_kernel"


@pytest.mark.parametrize("kv_type,D,heads,name", CASES,
                         ids=[f"{'q8' if k == W.KV_Q8_0 else 'q4'}-D{d}-g{h[0] // h[1]}-{n}" for k, d, h, n in CASES])
def test_decode_shape_sweep(kv_type, D, heads, name):
    H, Hkv = heads
    n_q, n_kv = layout(name, H // Hkv)
    seed = 100 + CASES.index((kv_type, D, heads, name))
    c = W.decode_case(len(n_q), 0, 0, H, Hkv, D, kv_type=kv_type, seed=seed, n_q_list=n_q, n_kv_list=n_kv)
    q, kc, vc = dev(c.q), dev(c.k_cache), dev(c.v_cache)
    st = status_word()
    o, lse = arc.attn_decode_q8(q, kc, vc, kv_type=c.kv_type, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q,
                                kv_begin=c.kv_begin, n_kv=c.n_kv, scale=c.scale, status=st)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    assert info["kernel"].startswith(expected_kernel(kv_type, D, H, Hkv, n_q))
    ro, rl = oracle.run_case(c)
    compare(o, lse, ro, rl, TOL_O_BF16)
    assert arc.check_device_error(st) == arc.ARC_OK
