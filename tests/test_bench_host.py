"""The numerator of every roofline fraction: bench.work() counts the algorithmic
FLOPs (visible (q, k) pairs x (2 d_qk + 2 d_v)) or bytes of one call.  Checked here
against brute-force counts of the visible pairs and against the exact figures of
the workloads (no GPU needed)."""
import numpy as np
import pytest

import bench
import workloads as W


@pytest.mark.parametrize("Tq,Tk,causal", [(7, 7, True), (5, 9, True), (9, 5, True), (6, 4, False), (1, 1, True),
                                          (0, 5, True), (5, 0, True)])
def test_visible_pairs_match_an_explicit_mask(Tq, Tk, causal):
    i = np.arange(Tq)[:, None]
    j = np.arange(Tk)[None, :]
    mask = (j <= i + (Tk - Tq)) if causal else np.ones((Tq, Tk), dtype=bool)
    assert bench.dense_pairs(Tq, Tk, causal) == int(mask.sum())


def test_gqa_prefill_flops():
    """B1 H64 Hkv8 T1400 D512, causal: 1400 * 1401 / 2 pairs per head, 2048 FLOP each."""
    flop, unit = bench.work(W.config(2))
    assert unit == "flop" and flop == 64 * (1400 * 1401 // 2) * (2 * 512 + 2 * 512) == 128_542_310_400


def test_mla_prefill_flops():
    """B2 H16 T4096, d_qk 128 + 64, d_v 128, causal."""
    flop, unit = bench.work(W.config(3))
    assert unit == "flop" and flop == 2 * 16 * (4096 * 4097 // 2) * (2 * 192 + 2 * 128) == 171_840_634_880


def test_sparse_flops_count_valid_slots_only():
    c = W.sparse_case(6, 64, 65536, 512, 512, 2176, seed=4)
    per_row = ((c.idx >= 0) & (c.idx < c.Skv)).sum(axis=1)
    assert np.all(per_row == 2176 - round(0.05 * 2176))          # 109 padded slots per query
    flop, unit = bench.work(c)
    assert unit == "flop" and flop == 6 * 2067 * 64 * 2048
    # the full workload, 13312 queries with the same padding: 3.607 TFLOP
    assert 13312 * 2067 * 64 * 2048 == 3_606_564_569_088


def test_sparse_flops_ignore_out_of_range_and_count_duplicates():
    c = W.sparse_case(2, 8, 100, 64, 64, 10, seed=9)
    c.idx[0, :3] = [100, -7, 5]
    c.idx[1, :] = 5                                              # one row, ten slots
    valid = int(((c.idx >= 0) & (c.idx < 100)).sum())
    assert bench.work(c) == (valid * 8 * 256, "flop")


@pytest.mark.parametrize("kv_type,block", [(W.KV_Q8_0, 34), (W.KV_Q4_0, 18)])
def test_decode_bytes_are_the_quantised_cache_read_once(kv_type, block):
    c = W.config(5, kv_type=kv_type)
    nbytes, unit = bench.work(c)
    cache = 2 * 32768 * 8 * (128 // 32) * block                  # K and V
    qo = 16 * 32 * 128 * 4 * 2 + 16 * 32 * 4                      # q and o fp32, lse
    assert unit == "byte" and nbytes == cache + qo
    assert round(cache / 1e6, 1) == (71.3 if kv_type == W.KV_Q8_0 else 37.7)


def test_merge_bytes():
    c = W.merge_case(n_parts=2, B=1, H=4, T=10, Dv=8, seed=1)
    o_bytes = 1 * 4 * 10 * 8 * 2
    lse_bytes = 1 * 4 * 10 * 4
    assert bench.work(c) == (3 * (o_bytes + lse_bytes), "byte")


def test_every_measured_kernel_maps_to_its_source_and_has_a_traffic_record():
    """roofline.traffic is taken from profiles/traffic.json only while the recorded source
    hash matches the kernel's source file: every kernel a measured workload names must map
    to a file, and every measured workload must have a record naming that kernel."""
    import json
    import os
    names = {"c2": "tc_attn_pair_kernel", "c3": "tc_attn_pair_kernel<mla>", "c4": "sparse_tc_kernel",
             "c4d": "sparse_tc_kernel<split>", "c5q8": "decode_ws_kernel<q8_0>", "c5q4": "decode_ws_kernel<q4_0>",
             "c5d256": "decode_ws_kernel<q8_0>", "c5g8": "decode_ws_kernel<q8_0>",
             "bwd_gqa": "bwd_dkdv_kernel+bwd_dq_kernel", "bwd_mla": "bwd_dkdv_kernel<mla>+bwd_dq_kernel",
             "merge": "merge_kernel"}
    assert set(bench.GRADED) | {"merge"} == set(names)
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for cfg, kernel in names.items():
        assert bench.kernel_source_hash(kernel) is not None, kernel
        assert rec[cfg]["kernel"] == kernel, cfg
        assert rec[cfg]["dram_bytes_per_launch"] > 0, cfg
