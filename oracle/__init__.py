"""fp64 CPU oracle for exact softmax attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library does not use it and
shares no code with it; the only thing both sides read is the seeded inputs
from ``workloads``.

The forward arithmetic lives in ``arc_oracle.c`` (plain loops, double precision,
OpenMP over independent rows); the backward (``backward.py``) is numpy fp64, the
derivative of the same definition.  This module builds it with gcc, widens the
stored inputs exactly to float64 (bf16 bits -> fp32 -> fp64, fp32 -> fp64) and
marshals arguments.  Every forward function returns ``(o, lse)`` as float64 arrays.

Pins: tests/test_oracle_pins.py (forward) and tests/test_oracle_backward_pins.py
(backward).  Every function here is pinned there against something other than
itself (torch's fp64 SDPA or autograd, finite differences, closed forms,
invariants the pages state); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "arc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

MUT_NONE = 0
MUT_REP_MAJOR = 1
MUT_TILE_LOCAL_MASK = 2
MUT_DROP_SINK = 3
MUT_TOP_LEFT_CAUSAL = 4
MUT_SWAP_NIBBLES = 5
MUT_MERGE_UNWEIGHTED = 6

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_bp = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile arc_oracle.c into liboracle.so next to it (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        I, D = ctypes.c_int, ctypes.c_double
        lib.oracle_attn.argtypes = [I, I, I, I, I, I, I, I, _ip, _dp, _dp, _dp, D, I, _dp, _dp, _dp]
        lib.oracle_attn_tiled.argtypes = [I, I, I, I, I, I, I, _dp, _dp, _dp, D, I, _dp,
                                          ctypes.c_longlong, _dp, _dp, ctypes.POINTER(I)]
        lib.oracle_attn_fold.argtypes = [I, I, I, I, I, I, I, _dp, _dp, _dp, D, I, _dp, _dp, _dp]
        lib.oracle_mla.argtypes = [I, I, I, I, I, I, I, I, _ip, _dp, _dp, _dp, _dp, _dp, D, I,
                                   _dp, _dp]
        lib.oracle_sparse.argtypes = [I, I, I, I, I, I, _dp, _dp, _dp, _ip, D, _dp, _dp, _dp]
        lib.oracle_decode_q.argtypes = [I, I, _ip, _ip, _ip, _ip, I, I, I, I, _dp, I, _bp, _bp,
                                        D, _dp, _dp]
        lib.oracle_dequant_cache.argtypes = [I, I, I, I, _bp, _dp]
        lib.oracle_merge.argtypes = [I, ctypes.c_long, I, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_set_mutation.argtypes = [I]
        lib.oracle_set_num_threads.argtypes = [I]
        for f in ("oracle_attn", "oracle_attn_tiled", "oracle_attn_fold", "oracle_mla",
                  "oracle_sparse", "oracle_decode_q", "oracle_dequant_cache", "oracle_merge"):
            getattr(lib, f).restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def set_mutation(m: int) -> None:
    _load().oracle_set_mutation(int(m))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


# ------------------------------------------------------------------ widening

def widen(x: np.ndarray, dtype: str | None = None) -> np.ndarray:
    """Exact conversion of stored inputs to float64.  uint16 arrays are bf16 bits."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def _c(x, dt=np.float64):
    return np.ascontiguousarray(x, dtype=dt)


def _ptr(a, p):
    return a.ctypes.data_as(p) if a is not None else None


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: oracle rejected its arguments (rc={rc})")


# ------------------------------------------------------------------ entry points

def attn(q, k, v, *, scale, causal=True, sinks=None, rows=None):
    """Dense / GQA attention.  q [B,H,Tq,D], k [B,Hkv,Tk,D], v [B,Hkv,Tk,Dv].

    rows: optional sorted list of query positions to evaluate (default all);
    the outputs then have nr = len(rows) in place of Tq.
    """
    q, k, v = widen(q), widen(k), widen(v)
    B, H, Tq, D = q.shape
    _, Hkv, Tk, Dv = v.shape
    pos = np.arange(Tq, dtype=np.int32) if rows is None else _c(rows, np.int32)
    qs = _c(q if rows is None else q[:, :, pos, :])
    nr = len(pos)
    o = np.zeros((B, H, nr, Dv))
    lse = np.zeros((B, H, nr))
    s = None if sinks is None else _c(widen(sinks))
    rc = _load().oracle_attn(B, H, Hkv, Tq, Tk, D, Dv, nr, _ptr(pos, _ip), _ptr(qs, _dp),
                             _ptr(_c(k), _dp), _ptr(_c(v), _dp), float(scale), int(bool(causal)),
                             _ptr(s, _dp), _ptr(o, _dp), _ptr(lse, _dp))
    _check(rc, "attn")
    return o, lse


def attn_tiled(q, k, v, *, scale, causal=True, sinks=None, tile_bytes=32 << 20):
    """Query-row tiled evaluation; returns (o, lse, n_tiles)."""
    q, k, v = _c(widen(q)), _c(widen(k)), _c(widen(v))
    B, H, Tq, D = q.shape
    _, Hkv, Tk, Dv = v.shape
    o = np.zeros((B, H, Tq, Dv))
    lse = np.zeros((B, H, Tq))
    nt = ctypes.c_int(0)
    s = None if sinks is None else _c(widen(sinks))
    rc = _load().oracle_attn_tiled(B, H, Hkv, Tq, Tk, D, Dv, _ptr(q, _dp), _ptr(k, _dp),
                                   _ptr(v, _dp), float(scale), int(bool(causal)), _ptr(s, _dp),
                                   int(tile_bytes), _ptr(o, _dp), _ptr(lse, _dp), ctypes.byref(nt))
    _check(rc, "attn_tiled")
    return o, lse, nt.value


def attn_fold(q, k, v, *, scale, causal=True, sinks=None):
    """GQA fold view: returns (o_fold [B,Hkv,g*Tq,Dv], lse_fold [B,Hkv,g*Tq])."""
    q, k, v = _c(widen(q)), _c(widen(k)), _c(widen(v))
    B, H, Tq, D = q.shape
    _, Hkv, Tk, Dv = v.shape
    g = H // Hkv
    o = np.zeros((B, Hkv, g * Tq, Dv))
    lse = np.zeros((B, Hkv, g * Tq))
    s = None if sinks is None else _c(widen(sinks))
    rc = _load().oracle_attn_fold(B, H, Hkv, Tq, Tk, D, Dv, _ptr(q, _dp), _ptr(k, _dp),
                                  _ptr(v, _dp), float(scale), int(bool(causal)), _ptr(s, _dp),
                                  _ptr(o, _dp), _ptr(lse, _dp))
    _check(rc, "attn_fold")
    return o, lse


def mla(q_nope, q_rope, k_nope, k_rope, v, *, scale, causal=True, rows=None):
    """MLA: q = q_nope||q_rope [B,H,Tq,*], k = k_nope[B,H,Tk,Dn] || k_rope[B,Tk,Dr] (shared)."""
    qn, qr = widen(q_nope), widen(q_rope)
    kn, kr, vv = _c(widen(k_nope)), _c(widen(k_rope)), _c(widen(v))
    B, H, Tq, Dn = qn.shape
    Dr = qr.shape[-1]
    Tk, Dv = vv.shape[2], vv.shape[3]
    pos = np.arange(Tq, dtype=np.int32) if rows is None else _c(rows, np.int32)
    if rows is not None:
        qn, qr = qn[:, :, pos, :], qr[:, :, pos, :]
    qn, qr = _c(qn), _c(qr)
    nr = len(pos)
    o = np.zeros((B, H, nr, Dv))
    lse = np.zeros((B, H, nr))
    rc = _load().oracle_mla(B, H, Tq, Tk, Dn, Dr, Dv, nr, _ptr(pos, _ip), _ptr(qn, _dp),
                            _ptr(qr, _dp), _ptr(kn, _dp), _ptr(kr, _dp), _ptr(vv, _dp),
                            float(scale), int(bool(causal)), _ptr(o, _dp), _ptr(lse, _dp))
    _check(rc, "mla")
    return o, lse


def sparse(q, kv, idx, *, scale, Dv=None, v=None, sinks=None):
    """Sparse attention: q [nq,H,Dqk], kv [Skv,Dqk], idx [nq,topk] int32 (-1 = masked)."""
    q, kvw = _c(widen(q)), _c(widen(kv))
    nq, H, Dqk = q.shape
    Skv = kvw.shape[0]
    vw = None if v is None else _c(widen(v))
    if Dv is None:
        Dv = vw.shape[1] if vw is not None else Dqk
    idx = _c(idx, np.int32)
    topk = idx.shape[1]
    o = np.zeros((nq, H, Dv))
    lse = np.zeros((nq, H))
    s = None if sinks is None else _c(widen(sinks))
    rc = _load().oracle_sparse(nq, H, Skv, Dqk, Dv, topk, _ptr(q, _dp), _ptr(kvw, _dp),
                               _ptr(vw, _dp), _ptr(idx, _ip), float(scale), _ptr(s, _dp),
                               _ptr(o, _dp), _ptr(lse, _dp))
    _check(rc, "sparse")
    return o, lse


def decode_q(case, *, seqs=None):
    """Multi-sequence quantised decode on a workloads.DecodeCase; seqs limits the sequences."""
    sel = list(range(case.n_seq)) if seqs is None else list(seqs)
    qb = _c(case.q_begin[sel], np.int32)
    nq = _c(case.n_q[sel], np.int32)
    kb = _c(case.kv_begin[sel], np.int32)
    nkv = _c(case.n_kv[sel], np.int32)
    q = _c(widen(case.q))
    n_tok = q.shape[0]
    o = np.zeros((n_tok, case.H, case.D))
    lse = np.full((n_tok, case.H), np.nan)
    kc, vc = _c(case.k_cache, np.uint8), _c(case.v_cache, np.uint8)
    rc = _load().oracle_decode_q(case.kv_type, len(sel), _ptr(qb, _ip), _ptr(nq, _ip),
                                 _ptr(kb, _ip), _ptr(nkv, _ip), n_tok, case.H, case.Hkv, case.D,
                                 _ptr(q, _dp), case.n_cells, _ptr(kc, _bp), _ptr(vc, _bp),
                                 float(case.scale), _ptr(o, _dp), _ptr(lse, _dp))
    _check(rc, "decode_q")
    return o, lse


def dequant_cache(kv_type, cache, n_cells, Hkv, D):
    """Dequantise a [n_cells,Hkv,D/32 blocks] cache to float64 [n_cells,Hkv,D]."""
    c = _c(cache, np.uint8)
    out = np.zeros((n_cells, Hkv, D))
    rc = _load().oracle_dequant_cache(int(kv_type), n_cells, Hkv, D, _ptr(c, _bp), _ptr(out, _dp))
    _check(rc, "dequant_cache")
    return out


# ------------------------------------------------------------------ whole cases

def run_case(case, rows=None):
    """Evaluate a workloads case (Dense/Mla/Sparse/Decode/Merge).  rows selects query rows."""
    import workloads as W
    if isinstance(case, W.DenseCase):
        return attn(case.q, case.k, case.v, scale=case.scale, causal=case.causal,
                    sinks=case.sinks, rows=rows)
    if isinstance(case, W.MlaCase):
        return mla(case.q_nope, case.q_rope, case.k_nope, case.k_rope, case.v, scale=case.scale,
                   causal=case.causal, rows=rows)
    if isinstance(case, W.SparseCase):
        if rows is None:
            return sparse(case.q, case.kv, case.idx, scale=case.scale, Dv=case.Dv, v=case.v,
                          sinks=case.sinks)
        rows = np.asarray(rows)
        return sparse(case.q[rows], case.kv, case.idx[rows], scale=case.scale, Dv=case.Dv,
                      v=case.v, sinks=case.sinks)
    if isinstance(case, W.DecodeCase):
        return decode_q(case)
    if isinstance(case, W.MergeCase):
        sl = slice(None) if rows is None else np.asarray(rows)
        parts = [x[:, :, sl] for x in case.o_parts]
        lses = [x[:, :, sl] for x in case.lse_parts]
        sr = None if case.sinks is None else np.broadcast_to(case.sinks.astype(np.float64)[None, :, None],
                                                              lses[0].shape)
        return merge(parts, lses, sink_rows=sr)
    raise TypeError(type(case))


def merge(o_parts, lse_parts, *, sink_rows=None):
    """Merge of results over disjoint key sets: o_parts, a list of [..., dv] outputs,
    lse_parts the matching [...] natural-log LSEs (-inf = empty part); sink_rows,
    optional [...] sink logits added once.  Returns (o, lse) over the union of the keys.
    Follows the output merge of "TransformerEngine: FA4 in context-parallel attention"
    (flowchart); see oracle_merge in arc_oracle.c."""
    shape = np.shape(o_parts[0])
    dv = shape[-1]
    rows = int(np.prod(shape[:-1]))
    op = _c(np.stack([widen(x).reshape(rows, dv) for x in o_parts]))
    lp = _c(np.stack([widen(x).reshape(rows) for x in lse_parts]))
    sr = None if sink_rows is None else _c(np.broadcast_to(widen(sink_rows), shape[:-1]).reshape(rows))
    o = np.zeros((rows, dv))
    lse = np.zeros(rows)
    rc = _load().oracle_merge(len(o_parts), rows, dv, _ptr(op, _dp), _ptr(lp, _dp), _ptr(sr, _dp),
                              _ptr(o, _dp), _ptr(lse, _dp))
    _check(rc, "merge")
    return o.reshape(shape), lse.reshape(shape[:-1])


from .backward import MUT_BWD_DROP_DELTA, attn_bwd, mla_bwd, sparse_bwd  # noqa: E402
