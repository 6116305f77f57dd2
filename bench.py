#!/usr/bin/env python
"""Benchmark of the fused exact-attention forward on B200.

One step = one call of the hot path on one batch of seeded synthetic input,
inputs already resident in HBM.  Default workload: GQA prefill with per-head
sinks (B=1, H=64 over Hkv=8, T=1400 causal, D=512, bf16) -- the configuration
the headline metric is quoted on.  Other workloads: --config c1 c3 c4 c5q8 c5q4.

Timing: W untimed warm-up steps, then K steps; before each timed step a
256 MiB buffer is written and another 256 MiB read to flush L2 (outside the
timed interval, leaving no dirty line behind), and the
step is bracketed by CUDA events on the launching stream.  A single-GPU run
also times every other graded workload (c2, c3, c4, c5q8, c5q4) in the same
way, each on a loop of at least --per-config-wall seconds so the clock sampler
sees it, and adds them under "per_config"; the decode workloads are timed a
second time replaying the call from a CUDA graph.  Multi-GPU (torchrun):
every rank runs the same per-GPU work (weak scaling, no data-path collective);
the time is the max over ranks.  --impl reference times the CPU oracle on the
host cores on a bounded sample of the same workload.

Prints ONE JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

CONFIGS = {
    "c1": dict(cfg=1, name="tiny dense causal fp32, B=1 H=4 Hkv=1 T=64 D=64", metric="attention fwd TFLOP/s",
               dtype="f32"),
    "c2": dict(cfg=2, name="GQA prefill with sinks, B=1 H=64 Hkv=8 T=1400 D=512 causal", metric="attention fwd TFLOP/s",
               dtype="bf16"),
    "c3": dict(cfg=3, name="MLA prefill, B=2 H=16 T=4096 d_qk=192 (128+64) d_v=128 causal",
               metric="attention fwd TFLOP/s", dtype="bf16"),
    "c4": dict(cfg=4, name="sparse MLA fwd, 13312 q x 64 h x 2176 top-k, d_qk=d_v=512, pool 65536",
               metric="attention fwd TFLOP/s", dtype="bf16"),
    "c5q8": dict(cfg=5, kv_type=W.KV_Q8_0, name="multi-seq decode, 4 seq x 4 tok, H=32 Hkv=8 D=128, 8192 cells/seq, q8_0",
                 metric="decode GB/s", dtype="q8_0"),
    "c5q4": dict(cfg=5, kv_type=W.KV_Q4_0, name="multi-seq decode, 4 seq x 4 tok, H=32 Hkv=8 D=128, 8192 cells/seq, q4_0",
                 metric="decode GB/s", dtype="q4_0"),
    # quantised decode at head dim 256 and with 32 fold rows per (sequence, kv head)
    "c5d256": dict(cfg=8, decode=dict(n_seq=4, n_q=4, n_kv=8192, H=32, Hkv=8, D=256, kv_type=W.KV_Q8_0),
                   name="multi-seq decode, 4 seq x 4 tok, H=32 Hkv=8 D=256, 8192 cells/seq, q8_0",
                   metric="decode GB/s", dtype="q8_0"),
    "c5g8": dict(cfg=9, decode=dict(n_seq=4, n_q=4, n_kv=8192, H=64, Hkv=8, D=128, kv_type=W.KV_Q8_0),
                 name="multi-seq decode, 4 seq x 4 tok, H=64 Hkv=8 (32 fold rows) D=128, 8192 cells/seq, q8_0",
                 metric="decode GB/s", dtype="q8_0"),
    # the backward: the GQA prefill's structure (64 heads over 8, causal, sinks) at head
    # dim 128, and the MLA prefill's head dims (192 / 128) on concatenated q/k
    "bwd_gqa": dict(cfg=10, bwd=dict(B=1, H=64, Hkv=8, T=1400, D=128, Dv=128, sinks=True),
                    name="attention bwd, B=1 H=64 Hkv=8 T=1400 D=128 causal, sinks",
                    metric="attention bwd TFLOP/s", dtype="bf16"),
    "bwd_mla": dict(cfg=11, bwd_mla=dict(B=2, H=16, T=4096, Dn=128, Dr=64, Dv=128),
                    name="MLA bwd, B=2 H=16 T=4096 d_qk=192 (128+64) d_v=128 causal",
                    metric="attention bwd TFLOP/s", dtype="bf16"),
    # decode-shaped sparse MLA: c4's per-token shape at a decode batch of 32 tokens
    "c4d": dict(cfg=7, sparse_decode=dict(Sq=32, H=64, Skv=65536, Dqk=512, Dv=512, topk=2176),
                name="sparse MLA decode, 32 tokens x 64 h x 2176 top-k, d_qk=d_v=512, pool 65536",
                metric="sparse decode GB/s", dtype="bf16"),
    # the context-parallel output merge (not a configuration of the method's own benchmark):
    # two bf16 partial outputs shaped like c2's, with sinks
    "merge": dict(cfg=6, merge=dict(n_parts=2, B=1, H=64, T=1400, Dv=512), name="LSE output merge, 2 parts of "
                  "B=1 H=64 T=1400 Dv=512 bf16, sinks", metric="merge GB/s", dtype="bf16"),
}


def make_case(spec):
    if "merge" in spec:
        return W.merge_case(**spec["merge"], seed=spec["cfg"])
    if "sparse_decode" in spec:
        return SparseDecode(W.sparse_case(**spec["sparse_decode"], seed=spec["cfg"]))
    if "decode" in spec:
        return W.decode_case(**spec["decode"], seed=spec["cfg"])
    if "bwd_mla" in spec:
        b = spec["bwd_mla"]
        case = W.mla_case(b["B"], b["H"], b["T"], b["T"], b["Dn"], b["Dr"], b["Dv"], std=0.3, causal=True,
                          seed=spec["cfg"])
        return Backward(case, W.upstream(b["B"], b["H"], b["T"], b["Dv"], seed=spec["cfg"] + 1000))
    if "bwd" in spec:
        b = spec["bwd"]
        case = W.dense_case(b["B"], b["H"], b["Hkv"], b["T"], b["T"], b["D"], b["Dv"], dtype="bf16", std=0.5,
                            causal=True, sinks=b["sinks"], seed=spec["cfg"])
        return Backward(case, W.upstream(b["B"], b["H"], b["T"], b["Dv"], seed=spec["cfg"] + 1000))
    kw = {"kv_type": spec["kv_type"]} if "kv_type" in spec else {}
    return W.config(spec["cfg"], **kw)


# ------------------------------------------------------------------ algorithmic work

class Backward:
    """A dense case run through arc_attn_bwd, with seeded upstream gradients."""

    def __init__(self, case, up):
        self.case, self.up = case, up


class SparseDecode:
    """A sparse case run through arc_sparse_mla_decode (few tokens, top-k split over CTAs)."""

    def __init__(self, case):
        self.case = case

def dense_pairs(Tq, Tk, causal):
    if not causal:
        return Tq * Tk
    return sum(max(0, min(Tk, t + (Tk - Tq) + 1)) for t in range(Tq))


def work(case):
    """(algorithmic units, unit name) of one call: FLOPs over visible pairs, or bytes for decode."""
    if isinstance(case, Backward):
        # per visible (row, key) pair, each product counted once: 2*d_qk (S) + 2*d_v (dP)
        # + 2*d_v (dV) + 2*d_qk (dK) + 2*d_qk (dQ)
        c = case.case
        dqk = c.D if isinstance(c, W.DenseCase) else c.Dn + c.Dr
        pairs = c.B * c.H * dense_pairs(c.Tq, c.Tk, c.causal)
        return pairs * (6 * dqk + 4 * c.Dv), "flop"
    if isinstance(case, SparseDecode):
        # memory-bound: every distinct pool row a call gathers crosses HBM once, plus Q, O,
        # LSE and the index lists
        c = case.case
        valid = c.idx[(c.idx >= 0) & (c.idx < c.Skv)]
        rows = int(np.unique(valid).size)
        return rows * c.Dqk * 2 + c.q.nbytes + c.Sq * c.H * (c.Dv * 2 + 4) + c.idx.nbytes, "byte"
    if isinstance(case, W.DenseCase):
        pairs = case.B * case.H * dense_pairs(case.Tq, case.Tk, case.causal)
        return pairs * (2 * case.D + 2 * case.Dv), "flop"
    if isinstance(case, W.MlaCase):
        pairs = case.B * case.H * dense_pairs(case.Tq, case.Tk, case.causal)
        return pairs * (2 * (case.Dn + case.Dr) + 2 * case.Dv), "flop"
    if isinstance(case, W.SparseCase):
        valid = int(((case.idx >= 0) & (case.idx < case.Skv)).sum())
        return valid * case.H * (2 * case.Dqk + 2 * case.Dv), "flop"
    if isinstance(case, W.DecodeCase):
        kv = case.k_cache.nbytes + case.v_cache.nbytes
        qo = case.q.nbytes * 2 + case.n_tok * case.H * 4
        return kv + qo, "byte"
    if isinstance(case, W.MergeCase):
        # every part's O and LSE read once, the merged O and LSE written once
        return (len(case.o_parts) + 1) * (case.o_parts[0].nbytes + case.lse_parts[0].nbytes), "byte"
    raise TypeError(type(case))


# ------------------------------------------------------------------ GPU arm

class Uploaded:
    """Device copies of a case plus the call that runs one step."""

    def __init__(self, case, torch, arc):
        self.case, self.torch, self.arc = case, torch, arc
        self.h2d = 0

    def to_dev(self, x):
        torch = self.torch
        x = np.ascontiguousarray(x)
        t = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x)
        t = t.cuda()
        return t.view(torch.bfloat16) if x.dtype == np.uint16 else t


def build_call(case, torch, arc, status):
    """Returns (call(), inputs dict of device tensors, outputs list, n_launches, kernel name)."""
    U = Uploaded(case, torch, arc)
    if isinstance(case, Backward) and isinstance(case.case, W.MlaCase):
        c = case.case
        t = [U.to_dev(x) for x in (c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v)]
        o, lse = arc.mla_fwd(*t, scale=c.scale, causal=c.causal)
        do = U.to_dev(case.up.do)
        info = arc.plan_mla_bwd(*t, o, lse, do, causal=c.causal)

        def call():
            arc.mla_bwd(*t, o, lse, do, scale=c.scale, causal=c.causal, status=status)
        ins = dict(zip(["q_nope", "q_rope", "k_nope", "k_rope", "v"], t))
        ins.update({"o": o, "lse": lse, "do": do})
        return call, ins, [o], info
    if isinstance(case, Backward):
        c = case.case
        q, k, v = U.to_dev(c.q), U.to_dev(c.k), U.to_dev(c.v)
        s = U.to_dev(c.sinks) if c.sinks is not None else None
        o, lse = arc.attn_fwd(q, k, v, scale=c.scale, causal=c.causal, sinks=s)
        do = U.to_dev(case.up.do)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dsk = torch.empty_like(s) if s is not None else None
        info = arc.plan_attn_bwd(q, k, v, o, lse, do, causal=c.causal, sinks=s)
        ws = torch.empty(max(256, arc.attn_bwd_workspace_size(q, k, v, o, lse, do, causal=c.causal, sinks=s)),
                         dtype=torch.uint8, device="cuda")

        def call():
            arc.attn_bwd(q, k, v, o, lse, do, scale=c.scale, causal=c.causal, sinks=s, dq=dq, dk=dk, dv=dv,
                         dsinks=dsk, workspace=ws, status=status)
        ins = {"q": q, "k": k, "v": v, "o": o, "lse": lse, "do": do}
        if s is not None:
            ins["sinks"] = s
        outs = [dq, dk, dv] + ([dsk] if dsk is not None else [])
        return call, ins, outs, info
    if isinstance(case, SparseDecode):
        c = case.case
        q, kv, idx = U.to_dev(c.q), U.to_dev(c.kv), U.to_dev(c.idx)
        o = torch.empty(c.Sq, c.H, c.Dv, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(c.Sq, c.H, dtype=torch.float32, device="cuda")
        info = arc.plan_sparse_decode(q, kv, idx, o, lse, Dv=c.Dv)
        ws = torch.empty(max(256, arc.sparse_decode_workspace_size(q, kv, idx, o, lse, Dv=c.Dv)), dtype=torch.uint8,
                         device="cuda")

        def call():
            arc.sparse_mla_decode(q, kv, idx, Dv=c.Dv, scale=c.scale, out=o, lse=lse, workspace=ws, status=status)
        return call, {"q": q, "kv": kv, "idx": idx}, [o, lse], info
    if isinstance(case, W.DenseCase):
        q, k, v = U.to_dev(case.q), U.to_dev(case.k), U.to_dev(case.v)
        s = U.to_dev(case.sinks) if case.sinks is not None else None
        o = torch.empty(case.B, case.H, case.Tq, case.Dv, dtype=q.dtype, device="cuda")
        lse = torch.empty(case.B, case.H, case.Tq, dtype=torch.float32, device="cuda")
        info = arc.plan_attn(q, k, v, o, lse, causal=case.causal, sinks=s)

        def call():
            arc.attn_fwd(q, k, v, scale=case.scale, causal=case.causal, sinks=s, out=o, lse=lse, status=status)
        ins = {"q": q, "k": k, "v": v}
        if s is not None:
            ins["sinks"] = s
        return call, ins, [o, lse], info
    if isinstance(case, W.MlaCase):
        t = [U.to_dev(x) for x in (case.q_nope, case.q_rope, case.k_nope, case.k_rope, case.v)]
        o = torch.empty(case.B, case.H, case.Tq, case.Dv, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(case.B, case.H, case.Tq, dtype=torch.float32, device="cuda")
        info = arc.plan_mla(*t, o, lse, causal=case.causal)

        def call():
            arc.mla_fwd(*t, scale=case.scale, causal=case.causal, out=o, lse=lse, status=status)
        return call, dict(zip(["q_nope", "q_rope", "k_nope", "k_rope", "v"], t)), [o, lse], info
    if isinstance(case, W.SparseCase):
        q, kv, idx = U.to_dev(case.q), U.to_dev(case.kv), U.to_dev(case.idx)
        o = torch.empty(case.Sq, case.H, case.Dv, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(case.Sq, case.H, dtype=torch.float32, device="cuda")
        info = arc.plan_sparse(q, kv, idx, o, lse, Dv=case.Dv)

        def call():
            arc.sparse_mla_fwd(q, kv, idx, Dv=case.Dv, scale=case.scale, out=o, lse=lse, status=status)
        return call, {"q": q, "kv": kv, "idx": idx}, [o, lse], info
    if isinstance(case, W.DecodeCase):
        q, kc, vc = U.to_dev(case.q), U.to_dev(case.k_cache), U.to_dev(case.v_cache)
        o = torch.empty(case.n_tok, case.H, case.D, dtype=torch.float32, device="cuda")
        lse = torch.empty(case.n_tok, case.H, dtype=torch.float32, device="cuda")
        kw = dict(Hkv=case.Hkv, q_begin=case.q_begin, n_q=case.n_q, kv_begin=case.kv_begin, n_kv=case.n_kv)
        ws_n = arc.decode_workspace_size(case.kv_type, q, case.Hkv, case.n_cells, case.q_begin, case.n_q,
                                         case.kv_begin, case.n_kv)
        ws = torch.empty(max(ws_n, 256), dtype=torch.uint8, device="cuda")
        info = arc.plan_decode(case.kv_type, q, kc, vc, **kw)

        def call():
            arc.attn_decode_q8(q, kc, vc, kv_type=case.kv_type, scale=case.scale, workspace=ws, out=o, lse=lse,
                               status=status, **kw)
        return call, {"q": q, "k_cache": kc, "v_cache": vc}, [o, lse], info
    if isinstance(case, W.MergeCase):
        parts = [U.to_dev(x) for x in case.o_parts]
        lses = [U.to_dev(x) for x in case.lse_parts]
        sinks = U.to_dev(case.sinks) if case.sinks is not None else None
        o = torch.empty_like(parts[0])
        lse = torch.empty_like(lses[0])
        info = arc.plan_merge(parts, lses, o, lse)

        def call():
            arc.attn_merge(parts, lses, sinks=sinks, sink_rows=case.T, out=o, lse=lse)
        ins = {f"o{i}": x for i, x in enumerate(parts)}
        ins.update({f"lse{i}": x for i, x in enumerate(lses)})
        return call, ins, [o, lse], info
    raise TypeError(type(case))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report no clocks rather than guess
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def result(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvml unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(kernel):
    files = {"tc_attn_kernel": "attn_tc.cu", "tc_attn_kernel<mla>": "attn_tc.cu", "tc_attn_pair_kernel": "attn_pair.cu",
             "tc_attn_pair_kernel<mla>": "attn_pair.cu",
             "tc_attn2_kernel": "attn_tc.cu", "tc_attn2_kernel<mla>": "attn_tc.cu",
             "sparse_tc_kernel": "sparse_tc.cu", "simple_attn_kernel<sparse>": "simple_kernels.cu",
             "simple_attn_kernel": "simple_kernels.cu", "merge_kernel": "merge.cu",
             "sparse_tc_kernel<split>": "sparse_tc.cu", "bwd_dkdv_kernel+bwd_dq_kernel": "attn_bwd.cu",
             "bwd_dkdv_kernel<mla>+bwd_dq_kernel": "attn_bwd.cu"}
    f = files.get(kernel)
    if kernel.startswith("decode_split_kernel") or kernel.startswith("decode_ws_kernel"):
        f = "decode.cu"
    if not f:
        return None
    path = os.path.join(ROOT, "exact_attention_131_b200", "csrc", f)
    h = hashlib.sha256(open(path, "rb").read())
    h.update(open(os.path.join(ROOT, "exact_attention_131_b200", "csrc", "ptx.cuh"), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(config_key, kernel):
    """DRAM bytes per launch from a committed ncu summary, if its kernel source still matches."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(config_key)
    if not rec or rec.get("kernel") != kernel or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


def cpu_baseline(case, key, budget_s=(10.0, 30.0)):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload."""
    import oracle
    oracle.build()
    cores = oracle.num_threads()
    if isinstance(case, Backward):
        units, _ = work(case)
        reps, spent = 0, 0.0
        while spent < budget_s[0] and reps < 20:
            t0 = time.perf_counter()
            oracle_backward(oracle, case)
            spent += time.perf_counter() - t0
            reps += 1
        return {"value": units * reps / spent / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                "sample": f"the whole backward, {reps} repetitions", "seconds": round(spent, 2)}
    if isinstance(case, SparseDecode):
        units, _ = work(case)
        reps, spent = 0, 0.0
        while spent < budget_s[0] and reps < 50:
            t0 = time.perf_counter()
            oracle.run_case(case.case)
            spent += time.perf_counter() - t0
            reps += 1
        return {"value": units * reps / spent / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": f"the whole decode batch, {reps} repetitions", "seconds": round(spent, 2)}
    rng = np.random.default_rng(0)
    done_units, spent, n_rows = 0, 0.0, 0
    if isinstance(case, (W.DenseCase, W.MlaCase)):
        T = case.Tq
        batch = 8
        while spent < budget_s[0]:
            rows = np.sort(rng.choice(T, size=batch, replace=False)).astype(np.int32)
            t0 = time.perf_counter()
            oracle.run_case(case, rows=rows)
            spent += time.perf_counter() - t0
            Dqk = case.D if isinstance(case, W.DenseCase) else case.Dn + case.Dr
            heads = case.B * case.H
            vis = sum(min(case.Tk, int(r) + case.Tk - case.Tq + 1) if case.causal else case.Tk for r in rows)
            done_units += int(heads) * int(vis) * (2 * Dqk + 2 * case.Dv)
            n_rows += batch
            if spent > budget_s[1]:
                break
        sample = f"{n_rows} random query positions x all {case.B * case.H} (batch, head) rows"
        return {"value": done_units / spent / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                "sample": sample, "seconds": round(spent, 2)}
    if isinstance(case, W.SparseCase):
        batch = 4
        while spent < budget_s[0]:
            rows = np.sort(rng.choice(case.Sq, size=batch, replace=False))
            t0 = time.perf_counter()
            oracle.run_case(case, rows=rows)
            spent += time.perf_counter() - t0
            valid = int(((case.idx[rows] >= 0) & (case.idx[rows] < case.Skv)).sum())
            done_units += int(valid) * case.H * (2 * case.Dqk + 2 * case.Dv)
            n_rows += batch
            if spent > budget_s[1]:
                break
        return {"value": done_units / spent / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                "sample": f"{n_rows} random query tokens x 64 heads x all top-k slots", "seconds": round(spent, 2)}
    if isinstance(case, W.MergeCase):
        rows_done, T = 0, case.T
        row_bytes = work(case)[0] / T
        while spent < budget_s[0]:
            rows = np.sort(rng.choice(T, size=16, replace=False))
            t0 = time.perf_counter()
            oracle.run_case(case, rows=rows)
            spent += time.perf_counter() - t0
            rows_done += len(rows)
            if spent > budget_s[1]:
                break
        return {"value": row_bytes * rows_done / spent / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": f"{rows_done} random positions x all {case.B * case.H} (batch, head) rows",
                "seconds": round(spent, 2)}
    if isinstance(case, W.DecodeCase):
        reps = 0
        units, _ = work(case)
        while spent < budget_s[0] and reps < 50:
            t0 = time.perf_counter()
            oracle.run_case(case)
            spent += time.perf_counter() - t0
            reps += 1
        return {"value": units * reps / spent / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": f"the whole decode step, {reps} repetitions", "seconds": round(spent, 2)}
    raise TypeError(type(case))


def oracle_backward(oracle, case):
    c = case.case
    if isinstance(c, W.MlaCase):
        return oracle.mla_bwd(c.q_nope, c.q_rope, c.k_nope, c.k_rope, c.v, case.up.do, scale=c.scale, causal=c.causal)
    return oracle.attn_bwd(c.q, c.k, c.v, case.up.do, scale=c.scale, causal=c.causal, sinks=c.sinks)


def unit_is_flop(spec):
    return "TFLOP" in spec["metric"]


def max_over_ranks(x, world, device):
    """The largest x over all ranks; every rank takes this collective step."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step, world, steps, total_ms, unit_kind):
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    scale = 1e12 if unit_kind == "flop" else 1e9
    return units_per_step * world * steps / (total_ms * 1e-3) / scale


class L2Flush:
    """Evicts the timed call's data from the 126 MB L2 before each timed step: a 256 MiB
    write, then (mode "write+read") a 256 MiB read of another buffer.  The read leaves
    L2 holding clean lines only; after the write alone it holds dirty lines, whose
    write-back the next step's own reads would then pay for in the timed interval."""

    def __init__(self, torch, mode):
        self.mode = mode
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.rd = torch.ones(64 << 20, dtype=torch.float32, device="cuda") if mode == "write+read" else None

    def __call__(self, i):
        self.buf.fill_(i & 0xFF)
        if self.rd is not None:
            self.rd.sum()

    def describe(self):
        return ("flushed before every timed step: 256 MiB write, then 256 MiB read (no dirty line left)"
                if self.rd is not None else "flushed (256 MiB write) before every timed step")


def time_steps(call, steps, stream, flush, local, graph=None):
    """Device time of `steps` calls: L2 is flushed before each, CUDA events on
    the launching stream bracket the call only.  With `graph`, each step replays it instead
    of calling.  Returns (per-step ms list, wall seconds of the loop, clock record)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(local)
    torch.cuda.synchronize()
    with sampler:
        wall0 = time.perf_counter()
        for i in range(steps):
            flush(i)
            ev[i][0].record(stream)
            if graph is None:
                call()
            else:
                graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    return [a.elapsed_time(b) for a, b in ev], wall, sampler.result()


def capture(call, stream):
    """One call captured into a CUDA graph (the serving form of a decode step)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        call()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            call()
    torch.cuda.synchronize()
    return g


def steps_for(call, stream, flush, local, min_wall_s):
    """Enough steps that the timed loop lasts min_wall_s (so the clock sampler sees it)."""
    _, wall, _ = time_steps(call, 20, stream, flush, local)
    return max(20, int(math.ceil(min_wall_s / max(wall / 20, 1e-6))))


def roofline(units, unit_kind, mean_ms, peaks, config_key, kernel, launches=1):
    if unit_kind == "flop":
        achieved = units / (mean_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "peak_source": peaks["source"] + " burst bf16",
                "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                      if peaks.get("bf16_tflops_sustained") else None)}
    else:
        achieved = units / (mean_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"] + " copy bandwidth",
                "note": f"whole call timed ({launches} launch{'es' if launches > 1 else ''})"}
    roof["traffic"] = recorded_traffic(config_key, kernel)
    roof["kernel"] = kernel
    return roof


def measure_config(key, status, stream, flush, local, peaks, min_wall_s):
    """One graded workload on this GPU, for the per-workload record beside the headline:
    device time over a loop long enough for the clock sampler, and for the decode
    workloads the same call replayed from a CUDA graph as well."""
    import torch
    import exact_attention_131_b200 as arc
    spec = CONFIGS[key]
    case = make_case(spec)
    call, ins, outs, info = build_call(case, torch, arc, status)
    units, unit_kind = work(case)
    for _ in range(5):
        call()
    steps = steps_for(call, stream, flush, local, min_wall_s)
    times, wall, clocks = time_steps(call, steps, stream, flush, local)
    mean_ms = sum(times) / len(times)
    scale = 1e12 if unit_kind == "flop" else 1e9
    rec = {"workload": spec["name"], "metric": spec["metric"], "value": units / (mean_ms * 1e-3) / scale,
           "unit": "TFLOP/s" if unit_kind == "flop" else "GB/s", "ms_per_step": mean_ms, "steps": steps,
           "dtype": spec["dtype"], "roofline": roofline(units, unit_kind, mean_ms, peaks, key, info["kernel"], info["launches"]),
           "clocks": clocks, "wall_s_timed_region": wall, "gpu_launches": int(info["launches"]) * steps,
           "l2": flush.describe()}
    if isinstance(case, (W.DecodeCase, SparseDecode)):
        g = capture(call, stream)
        for _ in range(5):
            g.replay()
        gsteps = max(steps, 20)
        gt, gwall, gclocks = time_steps(call, gsteps, stream, flush, local, graph=g)
        gmean = sum(gt) / len(gt)
        rec["graph_replay"] = {"value": units / (gmean * 1e-3) / scale, "ms_per_step": gmean, "steps": gsteps,
                               "frac": units / (gmean * 1e-3) / scale / peaks["hbm_gbs"], "clocks": gclocks,
                               "note": "the same call captured once into a CUDA graph and replayed"}
        del g
    del call, ins, outs, case
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


# The graded workloads: the headline (--config) plus these, each measured in the same run.
GRADED = ["c2", "c3", "c4", "c5q8", "c5q4",
          "c5d256", "c5g8", "c4d",          # the decode variants beyond the five workloads
          "bwd_gqa", "bwd_mla"]             # and the backward


def run_ours(args, spec, case):
    import torch
    import torch.distributed as dist
    import exact_attention_131_b200 as arc

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    call, ins, outs, info = build_call(case, torch, arc, status)
    units, unit_kind = work(case)
    stream = torch.cuda.current_stream()
    flush = L2Flush(torch, args.flush)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()

    barrier()
    times_ms, wall, clocks = time_steps(call, args.steps, stream, flush, local)
    barrier()
    mean_ms = sum(times_ms) / len(times_ms)
    total_ms = sum(times_ms)
    total_ms = max_over_ranks(total_ms, world, "cuda")
    assert arc.check_device_error(status) == arc.ARC_OK, "a device-side wait timed out"

    # ---- end to end through the public API with host buffers: H2D of the inputs from
    # pinned memory, the call, D2H of the outputs, all inside one timed interval
    host_ins = {k: v.cpu().pin_memory() for k, v in ins.items()}
    host_outs = [o.cpu().pin_memory() for o in outs]
    h2d = sum(v.numel() * v.element_size() for v in host_ins.values())
    d2h = sum(o.numel() * o.element_size() for o in host_outs)
    e2e_ms = []
    for i in range(0 if args.no_e2e else max(3, min(args.steps, 20)) + 2):
        flush(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for kname, hv in host_ins.items():
            ins[kname].copy_(hv, non_blocking=True)
        call()
        for o, ho in zip(outs, host_outs):
            ho.copy_(o, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if i >= 2:
            e2e_ms.append(a.elapsed_time(b))
    e2e_mean = sum(e2e_ms) / len(e2e_ms) if e2e_ms else float("nan")

    peaks = load_peaks()
    scale = 1e12 if unit_kind == "flop" else 1e9
    unit = "TFLOP/s" if unit_kind == "flop" else "GB/s"
    value = job_throughput(units, world, args.steps, total_ms, unit_kind)
    roof = roofline(units, unit_kind, mean_ms, peaks, args.config, info["kernel"], info["launches"])
    e2e_val = units / (e2e_mean * 1e-3) / scale
    if not e2e_ms:                      # --no-e2e: no host-buffer leg; JSON null rather than NaN
        e2e_val = e2e_mean = None

    line = {
        "metric": spec["metric"], "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": spec["dtype"], "data": "synthetic",
        "config": {"workload": spec["name"], "config": args.config, "seed": spec["cfg"],
                   "l2": flush.describe(),
                   "parallelism": f"replicas x{world}, no collective" if world > 1 else "single GPU"},
        "roofline": roof,
        "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_mean},
        "gpu_launches": int(info["launches"]) * args.steps,
        "clocks": clocks,
        "wall_s_timed_region": wall,
    }
    del call, ins, outs, host_ins, host_outs
    torch.cuda.empty_cache()
    # Every graded workload, each on its own long-enough loop, in the same run (rank 0 of a
    # single-GPU run only: under torchrun each rank would time its own replicas again).
    if world == 1 and not args.no_per_config:
        line["per_config"] = {k: measure_config(k, status, stream, flush, local, peaks, args.per_config_wall)
                              for k in GRADED if k != args.config}
        assert arc.check_device_error(status) == arc.ARC_OK, "a device-side wait timed out"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, args.config)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args, spec, case):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = oracle.num_threads()
    rng = np.random.default_rng(1)
    per_step_units, times = [], []
    for i in range(args.warmup + args.steps):
        if isinstance(case, (W.DenseCase, W.MlaCase)):
            rows = np.sort(rng.choice(case.Tq, size=2, replace=False)).astype(np.int32)
            Dqk = case.D if isinstance(case, W.DenseCase) else case.Dn + case.Dr
            vis = sum(min(case.Tk, int(r) + case.Tk - case.Tq + 1) if case.causal else case.Tk for r in rows)
            u = case.B * case.H * vis * (2 * Dqk + 2 * case.Dv)
            t0 = time.perf_counter()
            oracle.run_case(case, rows=rows)
        elif isinstance(case, W.MergeCase):
            rows = np.sort(rng.choice(case.T, size=4, replace=False))
            u = work(case)[0] / case.T * len(rows)
            t0 = time.perf_counter()
            oracle.run_case(case, rows=rows)
        elif isinstance(case, W.SparseCase):
            rows = np.array([rng.integers(case.Sq)])
            valid = int(((case.idx[rows] >= 0) & (case.idx[rows] < case.Skv)).sum())
            u = valid * case.H * (2 * case.Dqk + 2 * case.Dv)
            t0 = time.perf_counter()
            oracle.run_case(case, rows=rows)
        elif isinstance(case, Backward):
            u, _ = work(case)
            t0 = time.perf_counter()
            oracle_backward(oracle, case)
        else:
            u, _ = work(case)
            t0 = time.perf_counter()
            oracle.run_case(case.case if isinstance(case, SparseDecode) else case)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            per_step_units.append(u)
    total = sum(times)
    scale = 1e12 if unit_is_flop(spec) else 1e9
    unit = "TFLOP/s" if scale == 1e12 else "GB/s"
    value = sum(per_step_units) / total / scale
    sample = ("2 random query positions x all heads per step" if isinstance(case, (W.DenseCase, W.MlaCase))
              else "4 random positions x all heads per step" if isinstance(case, W.MergeCase)
              else "1 random query token x all heads x all slots per step" if isinstance(case, W.SparseCase)
              else "the whole decode step per step")
    line = {"impl": "reference", "metric": spec["metric"], "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": spec["name"], "config": args.config, "seed": spec["cfg"]},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="c2")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (for profiler runs)")
    ap.add_argument("--no-per-config", action="store_true", help="time the --config workload only")
    ap.add_argument("--flush", choices=["write", "write+read"], default="write+read",
                    help="how L2 is flushed before each timed step")
    ap.add_argument("--per-config-wall", type=float, default=1.5,
                    help="seconds each extra graded workload's timed loop lasts at least")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    spec = CONFIGS[args.config]
    case = make_case(spec)
    if args.impl == "reference":
        run_reference(args, spec, case)
    else:
        run_ours(args, spec, case)


if __name__ == "__main__":
    main()
