"""Seeded synthetic inputs shaped like the pages' attention workloads.

This module is shared by the CPU oracle side and the CUDA side, and by
nothing else's arithmetic: it draws random numbers, rounds them to the
storage type (bf16 round-to-nearest-even, or a q8_0 / q4_0 block encoding)
and lays them out.  It computes no attention, no softmax and no dequantised
value; each side decodes the stored bytes on its own.

Workload shapes follow the pages:
  * GQA prefill with per-head sinks, head_dim 512, T=1400, 64 query heads
    over 8 kv heads ("ArcFlash - Arc's own attention kernel, rung 0",
    rung-0 table and the Fold/Tile sections).
  * MLA prefill with q = q_nope || q_rope, d_qk 192, d_v 128
    (pith-train PR "FA4 b19 ...", the MLA concat section).
  * Sparse MLA forward, 13312 queries x 64 heads x 2176 top-k, d_qk 512
    (TensorRT-LLM PR "FlashMLA without -rdc", the timing paragraph).
  * Multi-sequence decode over a unified q8_0 / q4_0 KV cache, 4 streams of
    a few tokens (unsloth llama.cpp PR "dequantize q4_0/q8_0 K/V tiles in the
    FA MMA kernel", summary paragraph).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# q8_0 / q4_0 block geometry: 32 values per block, an fp16 scale first.
QK = 32
Q8_0_BLOCK_BYTES = 2 + QK          # 34
Q4_0_BLOCK_BYTES = 2 + QK // 2     # 18
KV_Q8_0 = 8                        # ggml type ids, used as the ABI's kv_type
KV_Q4_0 = 2


def make_rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the raw uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


# ---------------------------------------------------------------- q8_0 / q4_0

def encode_q8_0(x: np.ndarray) -> np.ndarray:
    """Encode rows of fp32 values (last dim a multiple of 32) as q8_0 blocks.

    Block = fp16 scale d (little endian) then 32 signed bytes q; the stored
    value is d*q.  Encoder: d = amax/127, q = round-half-away(x/d).
    Returns uint8 array [..., n_blocks * 34].
    """
    x = np.asarray(x, dtype=np.float32)
    lead = x.shape[:-1]
    nb = x.shape[-1] // QK
    xb = x.reshape(-1, nb, QK)
    amax = np.abs(xb).max(axis=-1)
    d = amax / np.float32(127.0)
    inv = np.where(d > 0, np.float32(1.0) / np.where(d > 0, d, 1), np.float32(0.0)).astype(np.float32)
    y = xb * inv[..., None]
    q = np.clip(np.sign(y) * np.floor(np.abs(y) + np.float32(0.5)), -127, 127).astype(np.int8)
    out = np.empty((xb.shape[0], nb, Q8_0_BLOCK_BYTES), dtype=np.uint8)
    out[..., 0:2] = d.astype(np.float16).reshape(xb.shape[0], nb, 1).view(np.uint8)
    out[..., 2:] = q.view(np.uint8)
    return out.reshape(*lead, nb * Q8_0_BLOCK_BYTES)


def encode_q4_0(x: np.ndarray) -> np.ndarray:
    """Encode rows of fp32 values as q4_0 blocks.

    Block = fp16 scale d then 16 bytes; byte j holds element j in its low
    nibble and element j+16 in its high nibble; the stored value is d*(n-8).
    Encoder: m = the element of largest magnitude (with its sign), d = m/-8,
    n = clamp(floor(x/d + 8.5), 0, 15).
    Returns uint8 array [..., n_blocks * 18].
    """
    x = np.asarray(x, dtype=np.float32)
    lead = x.shape[:-1]
    nb = x.shape[-1] // QK
    xb = x.reshape(-1, nb, QK)
    arg = np.abs(xb).argmax(axis=-1)
    m = np.take_along_axis(xb, arg[..., None], axis=-1)[..., 0]
    d = m / np.float32(-8.0)
    inv = np.where(d != 0, np.float32(1.0) / np.where(d != 0, d, 1), np.float32(0.0)).astype(np.float32)
    n = np.clip(np.floor(xb * inv[..., None] + np.float32(8.5)), 0, 15).astype(np.uint8)
    out = np.empty((xb.shape[0], nb, Q4_0_BLOCK_BYTES), dtype=np.uint8)
    out[..., 0:2] = d.astype(np.float16).reshape(xb.shape[0], nb, 1).view(np.uint8)
    out[..., 2:] = n[..., :16] | (n[..., 16:] << np.uint8(4))
    return out.reshape(*lead, nb * Q4_0_BLOCK_BYTES)


def block_bytes(kv_type: int) -> int:
    if kv_type == KV_Q8_0:
        return Q8_0_BLOCK_BYTES
    if kv_type == KV_Q4_0:
        return Q4_0_BLOCK_BYTES
    raise ValueError(f"unknown kv_type {kv_type}")


# ------------------------------------------------------------------ workloads

@dataclass
class DenseCase:
    """Dense / GQA attention inputs in BHSD layout.  bf16 tensors are uint16 bits."""
    B: int
    H: int
    Hkv: int
    Tq: int
    Tk: int
    D: int
    Dv: int
    dtype: str              # "bf16" or "f32"
    causal: bool
    scale: float
    q: np.ndarray           # [B,H,Tq,D]
    k: np.ndarray           # [B,Hkv,Tk,D]
    v: np.ndarray           # [B,Hkv,Tk,Dv]
    sinks: np.ndarray | None = None   # [H] fp32
    seed: int = 0


def dense_case(B, H, Hkv, Tq, Tk, D, Dv=None, *, dtype="bf16", std=1.0, causal=True,
               sinks=False, seed=0, scale=None) -> DenseCase:
    Dv = D if Dv is None else Dv
    rng = make_rng(seed)
    q = normal(rng, (B, H, Tq, D), std)
    k = normal(rng, (B, Hkv, Tk, D), std)
    v = normal(rng, (B, Hkv, Tk, Dv), std)
    s = normal(rng, (H,), 1.0) if sinks else None
    if dtype == "bf16":
        q, k, v = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    elif dtype != "f32":
        raise ValueError(dtype)
    return DenseCase(B, H, Hkv, Tq, Tk, D, Dv, dtype, causal,
                     float(1.0 / math.sqrt(D)) if scale is None else float(scale),
                     q, k, v, s, seed)


@dataclass
class MlaCase:
    """MLA inputs: q = q_nope || q_rope, k = k_nope[h] || k_rope (k_rope shared by all heads)."""
    B: int
    H: int
    Tq: int
    Tk: int
    Dn: int
    Dr: int
    Dv: int
    causal: bool
    scale: float
    q_nope: np.ndarray      # [B,H,Tq,Dn] bf16 bits
    q_rope: np.ndarray      # [B,H,Tq,Dr]
    k_nope: np.ndarray      # [B,H,Tk,Dn]
    k_rope: np.ndarray      # [B,Tk,Dr]
    v: np.ndarray           # [B,H,Tk,Dv]
    seed: int = 0


def mla_case(B, H, Tq, Tk, Dn=128, Dr=64, Dv=128, *, std=0.3, causal=True, seed=0) -> MlaCase:
    rng = make_rng(seed)
    qn = bf16_bits(normal(rng, (B, H, Tq, Dn), std))
    qr = bf16_bits(normal(rng, (B, H, Tq, Dr), std))
    kn = bf16_bits(normal(rng, (B, H, Tk, Dn), std))
    kr = bf16_bits(normal(rng, (B, Tk, Dr), std))
    v = bf16_bits(normal(rng, (B, H, Tk, Dv), std))
    return MlaCase(B, H, Tq, Tk, Dn, Dr, Dv, causal, float(1.0 / math.sqrt(Dn + Dr)),
                   qn, qr, kn, kr, v, seed)


@dataclass
class SparseCase:
    """Sparse MLA inputs: every query token attends to its own top-k rows of a shared pool."""
    Sq: int
    H: int
    Skv: int
    Dqk: int
    Dv: int
    topk: int
    scale: float
    q: np.ndarray           # [Sq,H,Dqk] bf16 bits
    kv: np.ndarray          # [Skv,Dqk] bf16 bits; V is kv[:, :Dv] unless v is given
    idx: np.ndarray         # [Sq,topk] int32, -1 = padding
    v: np.ndarray | None = None
    seed: int = 0
    sinks: np.ndarray | None = None   # [H] fp32


def sparse_indices(rng, Sq, Skv, topk, pad_frac=0.05, pad_mode="random") -> np.ndarray:
    """Per query: topk distinct pool rows drawn uniformly, then pad_frac of slots set to -1."""
    idx = np.empty((Sq, topk), dtype=np.int32)
    draw = min(Skv, max(topk + 64, int(topk * 1.25)))
    for i in range(Sq):
        row = None
        if topk <= Skv // 2:
            # rejection draws; when topk is near Skv / 2 a draw can keep falling short
            # of topk distinct values, so after a bounded number of tries take a permutation
            for _ in range(64):
                cand = rng.integers(0, Skv, size=draw)
                _, first = np.unique(cand, return_index=True)
                if first.size >= topk:
                    row = cand[np.sort(first)][:topk]
                    break
        if row is None:
            row = rng.permutation(Skv)[:topk]
        idx[i] = row
    n_pad = int(round(pad_frac * topk))
    if n_pad > 0:
        if pad_mode == "random":
            for i in range(Sq):
                idx[i, rng.choice(topk, size=n_pad, replace=False)] = -1
        elif pad_mode == "tail":
            idx[:, topk - n_pad:] = -1
        else:
            raise ValueError(pad_mode)
    return idx


def sparse_case(Sq, H, Skv, Dqk=512, Dv=512, topk=2176, *, std=0.3, pad_frac=0.05,
                pad_mode="random", separate_v=False, sinks=False, seed=0) -> SparseCase:
    rng = make_rng(seed)
    q = bf16_bits(normal(rng, (Sq, H, Dqk), std))
    kv = bf16_bits(normal(rng, (Skv, Dqk), std))
    v = bf16_bits(normal(rng, (Skv, Dv), std)) if separate_v else None
    idx = sparse_indices(rng, Sq, Skv, topk, pad_frac, pad_mode)
    # drawn last, so a case without sinks is unchanged by the option
    s = normal(rng, (H,), 1.0).astype(np.float32) if sinks else None
    return SparseCase(Sq, H, Skv, Dqk, Dv, topk, float(1.0 / math.sqrt(Dqk)), q, kv, idx, v, seed, s)


@dataclass
class DecodeCase:
    """Multi-sequence decode over one unified quantised KV cache.

    Sequence s owns query tokens [q_begin[s], q_begin[s]+n_q[s]) and cache
    cells [kv_begin[s], kv_begin[s]+n_kv[s]); its n_q new tokens are the last
    n_q of its n_kv cells, so query t of the sequence sees cells
    kv_begin .. kv_begin + n_kv - n_q + t.
    """
    kv_type: int
    n_seq: int
    H: int
    Hkv: int
    D: int
    n_cells: int
    scale: float
    q: np.ndarray           # [n_tok,H,D] fp32
    k_cache: np.ndarray     # [n_cells,Hkv,D/32*block_bytes] uint8
    v_cache: np.ndarray
    q_begin: np.ndarray     # [n_seq] int32
    n_q: np.ndarray
    kv_begin: np.ndarray
    n_kv: np.ndarray
    seed: int = 0

    @property
    def n_tok(self) -> int:
        return int(self.q.shape[0])


def decode_case(n_seq=4, n_q=4, n_kv=8192, H=32, Hkv=8, D=128, *, kv_type=KV_Q8_0,
                seed=0, n_q_list=None, n_kv_list=None) -> DecodeCase:
    rng = make_rng(seed)
    nq = np.array(n_q_list if n_q_list is not None else [n_q] * n_seq, dtype=np.int32)
    nkv = np.array(n_kv_list if n_kv_list is not None else [n_kv] * n_seq, dtype=np.int32)
    qb = np.concatenate([[0], np.cumsum(nq)[:-1]]).astype(np.int32)
    kb = np.concatenate([[0], np.cumsum(nkv)[:-1]]).astype(np.int32)
    n_tok = int(nq.sum())
    n_cells = int(nkv.sum())
    q = normal(rng, (n_tok, H, D), 1.0)
    k = normal(rng, (n_cells, Hkv, D), 1.0)
    v = normal(rng, (n_cells, Hkv, D), 1.0)
    enc = encode_q8_0 if kv_type == KV_Q8_0 else encode_q4_0
    return DecodeCase(kv_type, len(nq), H, Hkv, D, n_cells, float(1.0 / math.sqrt(D)), q,
                      enc(k), enc(v), qb, nq, kb, nkv, seed)


@dataclass
class MergeCase:
    """Partial results over disjoint key sets, to be merged (context-parallel output merge)."""
    B: int
    H: int
    T: int
    Dv: int
    o_parts: list           # n_parts x [B,H,T,Dv] bf16 bits
    lse_parts: list         # n_parts x [B,H,T] fp32, natural log; -inf marks an empty part
    sinks: np.ndarray | None = None   # [H] fp32
    seed: int = 0


def merge_case(n_parts=2, B=1, H=64, T=1400, Dv=512, *, sinks=True, empty_frac=0.02, seed=6) -> MergeCase:
    """Seeded parts shaped like an attention output: O ~ 0.5*N(0,1) in bf16, LSE ~ 3 + N(0,1),
    a few rows empty in each part."""
    rng = make_rng(seed)
    o = [bf16_bits(normal(rng, (B, H, T, Dv), 0.5)) for _ in range(n_parts)]
    lse = []
    for _ in range(n_parts):
        l = (3.0 + normal(rng, (B, H, T), 1.0)).astype(np.float32)
        l[rng.random((B, H, T)) < empty_frac] = -np.inf
        lse.append(l)
    s = normal(rng, (H,), 1.0).astype(np.float32) if sinks else None
    return MergeCase(B, H, T, Dv, o, lse, s, seed)


@dataclass
class Upstream:
    """Upstream gradients for a backward pass: dO (bf16 bits) and optionally dLSE (fp32)."""
    do: np.ndarray                    # [B,H,Tq,Dv] bf16 bits
    dlse: np.ndarray | None = None    # [B,H,Tq] fp32


def upstream(B, H, Tq, Dv, *, dlse=False, std=1.0, seed=0) -> Upstream:
    rng = make_rng(seed)
    do = bf16_bits(normal(rng, (B, H, Tq, Dv), std))
    dl = normal(rng, (B, H, Tq), 0.5) if dlse else None
    return Upstream(do, dl)


# The five workload configurations, by number, with seed = number.
def config(i: int, **over):
    if i == 1:
        return dense_case(1, 4, 1, 64, 64, 64, dtype="f32", std=1.0, causal=True, seed=1, **over)
    if i == 2:
        return dense_case(1, 64, 8, 1400, 1400, 512, dtype="bf16", std=0.5, causal=True,
                          sinks=True, seed=2, **over)
    if i == 3:
        return mla_case(2, 16, 4096, 4096, 128, 64, 128, std=0.3, causal=True, seed=3, **over)
    if i == 4:
        return sparse_case(13312, 64, 65536, 512, 512, 2176, std=0.3, pad_frac=0.05, seed=4, **over)
    if i == 5:
        return decode_case(4, 4, 8192, 32, 8, 128, seed=5, **over)
    raise ValueError(i)
