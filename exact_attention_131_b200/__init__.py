"""exact_attention_131_b200 -- Python binding of libarc_attn.so (the C ABI in include/arc_attn.h).

Argument marshalling only: every step of the attention forward runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  There is
no fallback: if the library is missing, importing a function raises.

Names follow the C ABI:
    attn_fwd            -> arc_attn_fwd         dense / GQA / MQA (+ sinks)
    attn_bwd            -> arc_attn_bwd         its gradients: dq, dk, dv, d sinks
    mla_bwd             -> arc_mla_bwd          mla_fwd's gradients (dk_rope summed over heads)
    mla_fwd             -> arc_mla_fwd          q_nope||q_rope, d_qk != d_v
    sparse_mla_fwd      -> arc_sparse_mla_fwd   per-query top-k index lists
    sparse_mla_decode   -> arc_sparse_mla_decode   the same, top-k split over CTAs for few tokens
    attn_decode_q8      -> arc_attn_decode_q8   q8_0 / q4_0 cache, multi-sequence
    attn_merge          -> arc_attn_merge       results over disjoint key sets -> the whole
    plan                -> arc_plan             engagement record, no launch
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libarc_attn.so")
_lib = None

ARC_OK, ARC_ERR_INVALID_ARG, ARC_ERR_UNSUPPORTED, ARC_ERR_CUDA, ARC_ERR_DEVICE_TIMEOUT, ARC_ERR_WORKSPACE = range(6)
ARC_DTYPE_BF16, ARC_DTYPE_F32 = 0, 1
ARC_KV_Q4_0, ARC_KV_Q8_0 = 2, 8
(ARC_OP_ATTN, ARC_OP_MLA, ARC_OP_SPARSE, ARC_OP_DECODE, ARC_OP_MERGE, ARC_OP_SPARSE_DECODE, ARC_OP_ATTN_BWD,
 ARC_OP_MLA_BWD) = range(1, 9)
ARC_MERGE_MAX_PARTS = 16
ARC_FLAG_FORCE_SIMPLE = 1
ARC_FLAG_SINGLE_CTA = 2
ARC_FLAG_DEFAULT_SCALE = 4
ARC_DECODE_MAX_SEQ = 64

_i32, _i64, _u32, _f32, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float, ctypes.c_void_p


class AttnArgs(ctypes.Structure):
    _fields_ = [("dtype", _i32), ("B", _i32), ("H", _i32), ("Hkv", _i32), ("Tq", _i32), ("Tk", _i32),
                ("D", _i32), ("Dv", _i32),
                ("q", _vp), ("q_strides", _i64 * 3), ("k", _vp), ("k_strides", _i64 * 3),
                ("v", _vp), ("v_strides", _i64 * 3), ("o", _vp), ("o_strides", _i64 * 3),
                ("lse", _vp), ("sinks", _vp), ("scale", _f32), ("causal", _i32), ("flags", _u32),
                ("status", _vp)]


class MlaArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("Tq", _i32), ("Tk", _i32), ("Dn", _i32), ("Dr", _i32), ("Dv", _i32),
                ("q_nope", _vp), ("q_nope_strides", _i64 * 3), ("q_rope", _vp), ("q_rope_strides", _i64 * 3),
                ("k_nope", _vp), ("k_nope_strides", _i64 * 3), ("k_rope", _vp), ("k_rope_strides", _i64 * 2),
                ("v", _vp), ("v_strides", _i64 * 3), ("o", _vp), ("o_strides", _i64 * 3),
                ("lse", _vp), ("scale", _f32), ("causal", _i32), ("flags", _u32), ("status", _vp)]


class SparseArgs(ctypes.Structure):
    _fields_ = [("Sq", _i32), ("H", _i32), ("Skv", _i32), ("Dqk", _i32), ("Dv", _i32), ("topk", _i32),
                ("q", _vp), ("q_strides", _i64 * 2), ("kv", _vp), ("kv_stride", _i64),
                ("v", _vp), ("v_stride", _i64), ("idx", _vp), ("idx_stride", _i64),
                ("o", _vp), ("o_strides", _i64 * 2), ("lse", _vp), ("sinks", _vp), ("scale", _f32),
                ("flags", _u32), ("status", _vp)]


class BwdArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("Hkv", _i32), ("Tq", _i32), ("Tk", _i32), ("D", _i32), ("Dv", _i32),
                ("q", _vp), ("q_strides", _i64 * 3), ("k", _vp), ("k_strides", _i64 * 3),
                ("v", _vp), ("v_strides", _i64 * 3), ("o", _vp), ("o_strides", _i64 * 3),
                ("dout", _vp), ("do_strides", _i64 * 3), ("lse", _vp), ("dlse", _vp), ("sinks", _vp),
                ("dq", _vp), ("dq_strides", _i64 * 3), ("dk", _vp), ("dk_strides", _i64 * 3),
                ("dv", _vp), ("dv_strides", _i64 * 3), ("dsinks", _vp), ("scale", _f32), ("causal", _i32),
                ("flags", _u32), ("status", _vp)]


class MlaBwdArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("Tq", _i32), ("Tk", _i32), ("Dn", _i32), ("Dr", _i32), ("Dv", _i32),
                ("q_nope", _vp), ("q_nope_strides", _i64 * 3), ("q_rope", _vp), ("q_rope_strides", _i64 * 3),
                ("k_nope", _vp), ("k_nope_strides", _i64 * 3), ("k_rope", _vp), ("k_rope_strides", _i64 * 2),
                ("v", _vp), ("v_strides", _i64 * 3), ("o", _vp), ("o_strides", _i64 * 3),
                ("dout", _vp), ("do_strides", _i64 * 3), ("lse", _vp), ("dlse", _vp),
                ("dq_nope", _vp), ("dq_nope_strides", _i64 * 3), ("dq_rope", _vp), ("dq_rope_strides", _i64 * 3),
                ("dk_nope", _vp), ("dk_nope_strides", _i64 * 3), ("dk_rope", _vp), ("dk_rope_strides", _i64 * 2),
                ("dv", _vp), ("dv_strides", _i64 * 3), ("scale", _f32), ("causal", _i32), ("flags", _u32),
                ("status", _vp)]


class Seq(ctypes.Structure):
    _fields_ = [("q_begin", _i32), ("n_q", _i32), ("kv_begin", _i32), ("n_kv", _i32)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("kv_type", _i32), ("n_tok", _i32), ("H", _i32), ("Hkv", _i32), ("D", _i32),
                ("n_cells", _i32), ("n_seq", _i32), ("q", _vp), ("k_cache", _vp), ("v_cache", _vp),
                ("seqs", ctypes.POINTER(Seq)), ("o", _vp), ("lse", _vp), ("scale", _f32), ("flags", _u32),
                ("status", _vp)]


class MergeArgs(ctypes.Structure):
    _fields_ = [("n_parts", _i32), ("rows", _i32), ("dv", _i32), ("dtype", _i32),
                ("o_parts", _vp * ARC_MERGE_MAX_PARTS), ("lse_parts", _vp * ARC_MERGE_MAX_PARTS),
                ("sinks", _vp), ("sink_heads", _i32), ("sink_rows", _i32), ("o", _vp), ("lse", _vp)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char * 64), ("tensor_cores", _i32), ("tile_m", _i32), ("tile_n", _i32),
                ("d_slice", _i32), ("n_ctas", _i32), ("splits", _i32), ("smem_bytes", _i32),
                ("tmem_cols", _i32), ("launches", _i32)]


EXPORTS = ["arc_attn_fwd", "arc_mla_fwd", "arc_sparse_mla_fwd", "arc_attn_decode_q8",
           "arc_decode_workspace_size", "arc_plan", "arc_abi_version", "arc_status_string",
           "arc_check_device_error", "arc_selftest_timeout", "arc_attn_decode_q8_noalloc", "arc_attn_merge",
           "arc_sparse_mla_decode", "arc_sparse_decode_workspace_size", "arc_attn_bwd", "arc_attn_bwd_workspace_size",
           "arc_mla_bwd", "arc_mla_bwd_workspace_size"]


class ArcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib():
    """Load libarc_attn.so (built in-tree).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m exact_attention_131_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.arc_attn_fwd.argtypes = [ctypes.POINTER(AttnArgs), _vp]
        L.arc_mla_fwd.argtypes = [ctypes.POINTER(MlaArgs), _vp]
        L.arc_sparse_mla_fwd.argtypes = [ctypes.POINTER(SparseArgs), _vp]
        L.arc_sparse_mla_decode.argtypes = [ctypes.POINTER(SparseArgs), _vp, ctypes.c_size_t, _vp]
        L.arc_sparse_decode_workspace_size.argtypes = [ctypes.POINTER(SparseArgs)]
        L.arc_sparse_decode_workspace_size.restype = ctypes.c_size_t
        L.arc_attn_bwd.argtypes = [ctypes.POINTER(BwdArgs), _vp, ctypes.c_size_t, _vp]
        L.arc_attn_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs)]
        L.arc_attn_bwd_workspace_size.restype = ctypes.c_size_t
        L.arc_mla_bwd.argtypes = [ctypes.POINTER(MlaBwdArgs), _vp, ctypes.c_size_t, _vp]
        L.arc_mla_bwd_workspace_size.argtypes = [ctypes.POINTER(MlaBwdArgs)]
        L.arc_mla_bwd_workspace_size.restype = ctypes.c_size_t
        L.arc_attn_decode_q8.argtypes = [ctypes.POINTER(DecodeArgs), _vp, ctypes.c_size_t, _vp]
        L.arc_attn_decode_q8_noalloc.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
        L.arc_attn_merge.argtypes = [ctypes.POINTER(MergeArgs), _vp]
        L.arc_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs)]
        L.arc_decode_workspace_size.restype = ctypes.c_size_t
        L.arc_plan.argtypes = [_i32, _vp, ctypes.POINTER(PlanInfo)]
        L.arc_status_string.argtypes = [_i32]
        L.arc_status_string.restype = ctypes.c_char_p
        L.arc_check_device_error.argtypes = [_vp, _vp]
        L.arc_selftest_timeout.argtypes = [_vp, ctypes.c_uint64, _vp]
        for f in ("arc_attn_fwd", "arc_attn_bwd", "arc_mla_bwd", "arc_mla_fwd", "arc_sparse_mla_fwd", "arc_sparse_mla_decode",
                  "arc_attn_decode_q8",
                  "arc_attn_decode_q8_noalloc", "arc_attn_merge", "arc_plan",
                  "arc_check_device_error", "arc_selftest_timeout", "arc_abi_version"):
            getattr(L, f).restype = _i32
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().arc_status_string(int(s)).decode()


def abi_version() -> int:
    return int(lib().arc_abi_version())


def _check(st: int, where: str):
    if st != ARC_OK:
        raise ArcError(st, where)


# ------------------------------------------------------------------ marshalling helpers

def _torch():
    import torch
    return torch


def _dev(t, name, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() > 0 and t.dim() > 0 and t.stride(-1) != 1 and t.shape[-1] > 1:
        raise ValueError(f"{name} must have a contiguous last dimension")
    return t


def _p(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _s3(t):
    return (_i64 * 3)(*t.stride()[:3])


def _scale_flags(scale, flags):
    """scale=None asks the library for its default 1/sqrt(d_qk) (ARC_FLAG_DEFAULT_SCALE)."""
    if scale is None:
        return 0.0, int(flags) | ARC_FLAG_DEFAULT_SCALE
    return float(scale), int(flags)


# ------------------------------------------------------------------ entry points

def _attn_args(q, k, v, o, lse, sinks, scale, causal, flags, status):
    torch = _torch()
    dt = {torch.bfloat16: ARC_DTYPE_BF16, torch.float32: ARC_DTYPE_F32}.get(q.dtype)
    if dt is None:
        raise ValueError("q must be bf16 or fp32")
    B, H, Tq, D = q.shape
    _, Hkv, Tk, Dv = v.shape
    a = AttnArgs()
    a.dtype, a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = dt, B, H, Hkv, Tq, Tk, D, Dv
    a.q, a.q_strides = _p(q), _s3(q)
    a.k, a.k_strides = _p(k), _s3(k)
    a.v, a.v_strides = _p(v), _s3(v)
    a.o, a.o_strides = _p(o), _s3(o)
    a.lse, a.sinks = _p(lse), _p(sinks)
    a.scale, a.flags = _scale_flags(scale, flags)
    a.causal = int(bool(causal))
    a.status = _p(status)
    return a


def attn_fwd(q, k, v, *, scale=None, causal=True, sinks=None, out=None, lse=None, flags=0, status=None,
             stream=None):
    """O, LSE = arc_attn_fwd(q [B,H,Tq,D], k [B,Hkv,Tk,D], v [B,Hkv,Tk,Dv])."""
    torch = _torch()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev(t, n, q.dtype)
    _dev(sinks, "sinks", torch.float32)
    B, H, Tq, D = q.shape
    Dv = v.shape[-1]
    if out is None:
        out = torch.empty(B, H, Tq, Dv, dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty(B, H, Tq, dtype=torch.float32, device=q.device)
    a = _attn_args(q, k, v, out, lse, sinks, scale, causal, flags, status)
    _check(lib().arc_attn_fwd(ctypes.byref(a), _stream(stream)), "arc_attn_fwd")
    return out, lse


def _bwd_args(q, k, v, o, lse, dout, dlse, sinks, dq, dk, dv, dsinks, scale, causal, flags, status):
    B, H, Tq, D = q.shape
    _, Hkv, Tk, Dv = v.shape
    a = BwdArgs()
    a.B, a.H, a.Hkv, a.Tq, a.Tk, a.D, a.Dv = B, H, Hkv, Tq, Tk, D, Dv
    a.q, a.q_strides = _p(q), _s3(q)
    a.k, a.k_strides = _p(k), _s3(k)
    a.v, a.v_strides = _p(v), _s3(v)
    a.o, a.o_strides = _p(o), _s3(o)
    a.dout, a.do_strides = _p(dout), _s3(dout)
    a.lse, a.dlse, a.sinks = _p(lse), _p(dlse), _p(sinks)
    a.dq, a.dq_strides = _p(dq), _s3(dq)
    a.dk, a.dk_strides = _p(dk), _s3(dk)
    a.dv, a.dv_strides = _p(dv), _s3(dv)
    a.dsinks = _p(dsinks)
    a.scale, a.flags = _scale_flags(scale, flags)
    a.causal = int(bool(causal))
    a.status = _p(status)
    return a


def attn_bwd(q, k, v, o, lse, dout, *, scale=None, causal=True, sinks=None, dlse=None, dq=None, dk=None, dv=None,
             dsinks=None, workspace=None, flags=0, status=None, stream=None):
    """dq, dk, dv, dsinks = arc_attn_bwd: gradients of attn_fwd(q, k, v) given its o, lse and
    the upstream dout (and optionally dlse).  dsinks is None without sinks."""
    torch = _torch()
    bf = torch.bfloat16
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _dev(t, n, bf)
    for n, t in (("lse", lse), ("dlse", dlse), ("sinks", sinks)):
        _dev(t, n, torch.float32)
    for n, t in (("lse", lse), ("dlse", dlse)):
        if t is not None and (tuple(t.shape) != tuple(q.shape[:3]) or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous [B, H, Tq] fp32 tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if sinks is not None and dsinks is None:
        dsinks = torch.empty_like(sinks)
    a = _bwd_args(q, k, v, o, lse, dout, dlse, sinks, dq, dk, dv, dsinks, scale, causal, flags, status)
    need = int(lib().arc_attn_bwd_workspace_size(ctypes.byref(a)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _p(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().arc_attn_bwd(ctypes.byref(a), ws_ptr, ws_len, _stream(stream)), "arc_attn_bwd")
    return dq, dk, dv, dsinks


def attn_bwd_workspace_size(q, k, v, o, lse, dout, *, causal=True, sinks=None, flags=0) -> int:
    a = _bwd_args(q, k, v, o, lse, dout, None, sinks, q, k, v, sinks, 1.0, causal, flags, None)
    return int(lib().arc_attn_bwd_workspace_size(ctypes.byref(a)))


def plan_attn_bwd(q, k, v, o, lse, dout, *, causal=True, sinks=None, flags=0):
    dq, dk, dv = q, k, v            # shapes and strides only: nothing is launched
    ds = sinks if sinks is not None else None
    return plan(ARC_OP_ATTN_BWD, _bwd_args(q, k, v, o, lse, dout, None, sinks, dq, dk, dv, ds, 1.0, causal, flags,
                                           None))


def _mla_bwd_args(q_nope, q_rope, k_nope, k_rope, v, o, lse, dout, dlse, dq_nope, dq_rope, dk_nope, dk_rope, dv,
                  scale, causal, flags, status):
    B, H, Tq, Dn = q_nope.shape
    a = MlaBwdArgs()
    a.B, a.H, a.Tq, a.Tk, a.Dn, a.Dr, a.Dv = B, H, Tq, v.shape[2], Dn, q_rope.shape[-1], v.shape[3]
    for f, t in (("q_nope", q_nope), ("q_rope", q_rope), ("k_nope", k_nope), ("v", v), ("o", o),
                 ("dq_nope", dq_nope), ("dq_rope", dq_rope), ("dk_nope", dk_nope), ("dv", dv)):
        setattr(a, f, _p(t))
        setattr(a, f + "_strides", _s3(t))
    a.dout, a.do_strides = _p(dout), _s3(dout)
    a.k_rope, a.k_rope_strides = _p(k_rope), (_i64 * 2)(*k_rope.stride()[:2])
    a.dk_rope, a.dk_rope_strides = _p(dk_rope), (_i64 * 2)(*dk_rope.stride()[:2])
    a.lse, a.dlse = _p(lse), _p(dlse)
    a.scale, a.flags = _scale_flags(scale, flags)
    a.causal = int(bool(causal))
    a.status = _p(status)
    return a


def mla_bwd(q_nope, q_rope, k_nope, k_rope, v, o, lse, dout, *, scale=None, causal=True, dlse=None, workspace=None,
            flags=0, status=None, stream=None):
    """dq_nope, dq_rope, dk_nope, dk_rope, dv = arc_mla_bwd: gradients of mla_fwd given its o,
    lse and the upstream dout (and optionally dlse); dk_rope is summed over the heads."""
    torch = _torch()
    bf = torch.bfloat16
    for n, t in (("q_nope", q_nope), ("q_rope", q_rope), ("k_nope", k_nope), ("k_rope", k_rope), ("v", v),
                 ("o", o), ("dout", dout)):
        _dev(t, n, bf)
    for n, t in (("lse", lse), ("dlse", dlse)):
        _dev(t, n, torch.float32)
        if t is not None and (tuple(t.shape) != tuple(q_nope.shape[:3]) or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous [B, H, Tq] fp32 tensor")
    dq_nope, dq_rope = torch.empty_like(q_nope), torch.empty_like(q_rope)
    dk_nope, dk_rope, dv = torch.empty_like(k_nope), torch.empty_like(k_rope), torch.empty_like(v)
    a = _mla_bwd_args(q_nope, q_rope, k_nope, k_rope, v, o, lse, dout, dlse, dq_nope, dq_rope, dk_nope, dk_rope, dv,
                      scale, causal, flags, status)
    need = int(lib().arc_mla_bwd_workspace_size(ctypes.byref(a)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    ws_ptr = _p(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().arc_mla_bwd(ctypes.byref(a), ws_ptr, ws_len, _stream(stream)), "arc_mla_bwd")
    return dq_nope, dq_rope, dk_nope, dk_rope, dv


def plan_mla_bwd(q_nope, q_rope, k_nope, k_rope, v, o, lse, dout, *, causal=True, flags=0):
    return plan(ARC_OP_MLA_BWD, _mla_bwd_args(q_nope, q_rope, k_nope, k_rope, v, o, lse, dout, None, q_nope, q_rope,
                                              k_nope, k_rope, v, 1.0, causal, flags, None))


def _mla_args(q_nope, q_rope, k_nope, k_rope, v, o, lse, scale, causal, flags, status):
    B, H, Tq, Dn = q_nope.shape
    Dr = q_rope.shape[-1]
    Tk, Dv = v.shape[2], v.shape[3]
    a = MlaArgs()
    a.B, a.H, a.Tq, a.Tk, a.Dn, a.Dr, a.Dv = B, H, Tq, Tk, Dn, Dr, Dv
    a.q_nope, a.q_nope_strides = _p(q_nope), _s3(q_nope)
    a.q_rope, a.q_rope_strides = _p(q_rope), _s3(q_rope)
    a.k_nope, a.k_nope_strides = _p(k_nope), _s3(k_nope)
    a.k_rope, a.k_rope_strides = _p(k_rope), (_i64 * 2)(*k_rope.stride()[:2])
    a.v, a.v_strides = _p(v), _s3(v)
    a.o, a.o_strides = _p(o), _s3(o)
    a.lse = _p(lse)
    a.scale, a.flags = _scale_flags(scale, flags)
    a.causal = int(bool(causal))
    a.status = _p(status)
    return a


def mla_fwd(q_nope, q_rope, k_nope, k_rope, v, *, scale=None, causal=True, out=None, lse=None, flags=0,
            status=None, stream=None):
    """O, LSE = arc_mla_fwd: q = q_nope||q_rope [B,H,Tq,*], k = k_nope[B,H,Tk,Dn]||k_rope[B,Tk,Dr]."""
    torch = _torch()
    bf = torch.bfloat16
    for n, t in (("q_nope", q_nope), ("q_rope", q_rope), ("k_nope", k_nope), ("k_rope", k_rope), ("v", v)):
        _dev(t, n, bf)
    B, H, Tq, Dn = q_nope.shape
    Dv = v.shape[-1]
    if out is None:
        out = torch.empty(B, H, Tq, Dv, dtype=bf, device=q_nope.device)
    if lse is None:
        lse = torch.empty(B, H, Tq, dtype=torch.float32, device=q_nope.device)
    a = _mla_args(q_nope, q_rope, k_nope, k_rope, v, out, lse, scale, causal, flags, status)
    _check(lib().arc_mla_fwd(ctypes.byref(a), _stream(stream)), "arc_mla_fwd")
    return out, lse


def _sparse_args(q, kv, idx, v, o, lse, sinks, Dv, scale, flags, status):
    Sq, H, Dqk = q.shape
    a = SparseArgs()
    a.Sq, a.H, a.Skv, a.Dqk, a.Dv, a.topk = Sq, H, kv.shape[0], Dqk, Dv, idx.shape[1]
    a.q, a.q_strides = _p(q), (_i64 * 2)(*q.stride()[:2])
    a.kv, a.kv_stride = _p(kv), kv.stride(0)
    a.v, a.v_stride = (_p(v), v.stride(0)) if v is not None else (None, 0)
    a.idx, a.idx_stride = _p(idx), idx.stride(0)
    a.o, a.o_strides = _p(o), (_i64 * 2)(*o.stride()[:2])
    a.lse, a.sinks = _p(lse), _p(sinks)
    a.scale, a.flags = _scale_flags(scale, flags)
    a.status = _p(status)
    return a


def sparse_mla_fwd(q, kv, idx, *, Dv=None, v=None, scale=None, sinks=None, out=None, lse=None, flags=0,
                   status=None, stream=None):
    """O, LSE = arc_sparse_mla_fwd(q [Sq,H,Dqk], kv [Skv,Dqk], idx [Sq,topk] int32)."""
    torch = _torch()
    bf = torch.bfloat16
    _dev(q, "q", bf), _dev(kv, "kv", bf), _dev(idx, "idx", torch.int32), _dev(v, "v", bf)
    _dev(sinks, "sinks", torch.float32)
    Sq, H, Dqk = q.shape
    if Dv is None:
        Dv = v.shape[1] if v is not None else Dqk
    if out is None:
        out = torch.empty(Sq, H, Dv, dtype=bf, device=q.device)
    if lse is None:
        lse = torch.empty(Sq, H, dtype=torch.float32, device=q.device)
    a = _sparse_args(q, kv, idx, v, out, lse, sinks, Dv, scale, flags, status)
    _check(lib().arc_sparse_mla_fwd(ctypes.byref(a), _stream(stream)), "arc_sparse_mla_fwd")
    return out, lse


def sparse_mla_decode(q, kv, idx, *, Dv=None, v=None, scale=None, sinks=None, out=None, lse=None, workspace=None,
                      flags=0, status=None, stream=None):
    """O, LSE = arc_sparse_mla_decode: arc_sparse_mla_fwd with each token's top-k list split
    over several CTAs when the tokens do not fill the GPU (a workspace holds the partials)."""
    torch = _torch()
    bf = torch.bfloat16
    _dev(q, "q", bf), _dev(kv, "kv", bf), _dev(idx, "idx", torch.int32), _dev(v, "v", bf)
    _dev(sinks, "sinks", torch.float32)
    Sq, H, Dqk = q.shape
    if Dv is None:
        Dv = v.shape[1] if v is not None else Dqk
    if out is None:
        out = torch.empty(Sq, H, Dv, dtype=bf, device=q.device)
    if lse is None:
        lse = torch.empty(Sq, H, dtype=torch.float32, device=q.device)
    a = _sparse_args(q, kv, idx, v, out, lse, sinks, Dv, scale, flags, status)
    need = int(lib().arc_sparse_decode_workspace_size(ctypes.byref(a)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _p(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().arc_sparse_mla_decode(ctypes.byref(a), ws_ptr, ws_len, _stream(stream)), "arc_sparse_mla_decode")
    return out, lse


def sparse_decode_workspace_size(q, kv, idx, out, lse, *, Dv=None, v=None, sinks=None, flags=0) -> int:
    Dv = Dv if Dv is not None else (v.shape[1] if v is not None else q.shape[-1])
    a = _sparse_args(q, kv, idx, v, out, lse, sinks, Dv, 1.0, flags, None)
    return int(lib().arc_sparse_decode_workspace_size(ctypes.byref(a)))


def make_seqs(q_begin, n_q, kv_begin, n_kv):
    n = len(q_begin)
    arr = (Seq * max(n, 1))()
    for i in range(n):
        arr[i] = Seq(int(q_begin[i]), int(n_q[i]), int(kv_begin[i]), int(n_kv[i]))
    return arr


def _decode_args(kv_type, q, k_cache, v_cache, seqs, n_seq, Hkv, n_cells, o, lse, scale, flags, status):
    n_tok, H, D = q.shape
    a = DecodeArgs()
    a.kv_type, a.n_tok, a.H, a.Hkv, a.D, a.n_cells, a.n_seq = kv_type, n_tok, H, Hkv, D, n_cells, n_seq
    a.q, a.k_cache, a.v_cache = _p(q), _p(k_cache), _p(v_cache)
    a.seqs = ctypes.cast(seqs, ctypes.POINTER(Seq))
    a.o, a.lse = _p(o), _p(lse)
    a.scale, a.flags = _scale_flags(scale, flags)
    a.status = _p(status)
    return a


def decode_workspace_size(kv_type, q, Hkv, n_cells, q_begin, n_q, kv_begin, n_kv, flags=0) -> int:
    seqs = make_seqs(q_begin, n_q, kv_begin, n_kv)
    a = _decode_args(kv_type, q, None, None, seqs, len(q_begin), Hkv, n_cells, None, None, 1.0, flags, None)
    return int(lib().arc_decode_workspace_size(ctypes.byref(a)))


def _decode_tensors(kv_type, q, k_cache, v_cache, Hkv, out, lse):
    """The decode ABI takes no strides: every tensor must be contiguous and of the shape
    the call implies, or the kernels would read or write past it.  Returns (out, lse),
    created when not given."""
    torch = _torch()
    _dev(q, "q", torch.float32), _dev(k_cache, "k_cache", torch.uint8), _dev(v_cache, "v_cache", torch.uint8)
    if q.dim() != 3 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [n_tok, H, D] tensor")
    n_tok, H, D = q.shape
    if Hkv <= 0 or H % Hkv or D % 32:
        raise ValueError("H must be a multiple of Hkv and D a multiple of 32")
    block = {ARC_KV_Q8_0: 34, ARC_KV_Q4_0: 18}.get(kv_type)
    if block is None:
        raise ValueError(f"unknown kv_type {kv_type}")
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if not t.is_contiguous() or t.dim() < 1 or t.device != q.device:
            raise ValueError(f"{n} must be contiguous and on q's device")
        if t.numel() != t.shape[0] * Hkv * (D // 32) * block:
            raise ValueError(f"{n} rows must hold Hkv * D/32 blocks of {block} bytes")
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    for n, t, shape in (("out", out, (n_tok, H, D)), ("lse", lse, (n_tok, H))):
        if t is None:
            continue
        if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{n} must be a contiguous fp32 {list(shape)} tensor on q's device")
    if out is None:
        out = torch.empty(n_tok, H, D, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(n_tok, H, dtype=torch.float32, device=q.device)
    return out, lse


def attn_decode_q8(q, k_cache, v_cache, *, kv_type, Hkv, q_begin, n_q, kv_begin, n_kv, scale=None,
                   workspace=None, out=None, lse=None, flags=0, status=None, stream=None):
    """O, LSE = arc_attn_decode_q8(q [n_tok,H,D] fp32, caches [n_cells,Hkv,D/32 blocks] uint8)."""
    torch = _torch()
    out, lse = _decode_tensors(kv_type, q, k_cache, v_cache, Hkv, out, lse)
    n_cells = k_cache.shape[0]
    seqs = make_seqs(q_begin, n_q, kv_begin, n_kv)
    a = _decode_args(kv_type, q, k_cache, v_cache, seqs, len(q_begin), Hkv, n_cells, out, lse, scale, flags,
                     status)
    need = int(lib().arc_decode_workspace_size(ctypes.byref(a)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _p(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().arc_attn_decode_q8(ctypes.byref(a), ws_ptr, ws_len, _stream(stream)), "arc_attn_decode_q8")
    return out, lse


NOALLOC_SCRATCH_BYTES = 8 << 20


def attn_decode_q8_noalloc(q, k_cache, v_cache, *, kv_type, Hkv, q_begin, n_q, kv_begin, n_kv, scale=None,
                           out=None, lse=None, flags=0, status=None, stream=None):
    """arc_attn_decode_q8_noalloc: the decode with the library's own 8 MiB static scratch.

    For callers that must not allocate device memory: no workspace is passed and
    the library allocates nothing.  (This wrapper still creates `out` / `lse`
    with torch when they are not given; pass them to keep the call allocation-free.)
    Calls on unordered streams race on the shared scratch.
    """
    out, lse = _decode_tensors(kv_type, q, k_cache, v_cache, Hkv, out, lse)
    seqs = make_seqs(q_begin, n_q, kv_begin, n_kv)
    a = _decode_args(kv_type, q, k_cache, v_cache, seqs, len(q_begin), Hkv, k_cache.shape[0], out, lse, scale,
                     flags, status)
    _check(lib().arc_attn_decode_q8_noalloc(ctypes.byref(a), _stream(stream)), "arc_attn_decode_q8_noalloc")
    return out, lse


def _merge_args(o_parts, lse_parts, o, lse, sinks, sink_rows):
    n = len(o_parts)
    if not 1 <= n <= ARC_MERGE_MAX_PARTS or len(lse_parts) != n:
        raise ValueError(f"1..{ARC_MERGE_MAX_PARTS} parts, one LSE per O")
    dv = int(o_parts[0].shape[-1])
    rows = int(o_parts[0].numel() // dv) if dv else 0
    a = MergeArgs()
    a.n_parts, a.rows, a.dv = n, rows, dv
    torch = _torch()
    a.dtype = ARC_DTYPE_F32 if o_parts[0].dtype == torch.float32 else ARC_DTYPE_BF16
    for i in range(n):
        a.o_parts[i], a.lse_parts[i] = _p(o_parts[i]), _p(lse_parts[i])
    a.sinks = _p(sinks)
    a.sink_heads = int(sinks.numel()) if sinks is not None else 0
    a.sink_rows = int(sink_rows) if sinks is not None else 0
    a.o, a.lse = _p(o), _p(lse)
    return a


def attn_merge(o_parts, lse_parts, *, sinks=None, sink_rows=None, out=None, lse=None, stream=None):
    """O, LSE = arc_attn_merge over parts computed on disjoint key sets.

    o_parts: tensors of one shape [..., dv] (bf16 or fp32, contiguous); lse_parts: the
    matching [...] fp32 log-sum-exps (natural log, -inf = empty part).  sinks: optional
    [H] fp32 sink logits added once (parts computed without them); for [B, H, Tq, dv]
    outputs pass sink_rows = Tq.
    """
    torch = _torch()
    if not o_parts:
        raise ValueError("at least one part")
    shape, dt = o_parts[0].shape, o_parts[0].dtype
    for i, (o_i, l_i) in enumerate(zip(o_parts, lse_parts)):
        _dev(o_i, f"o_parts[{i}]", dt), _dev(l_i, f"lse_parts[{i}]", torch.float32)
        if o_i.shape != shape or tuple(l_i.shape) != tuple(shape[:-1]):
            raise ValueError("every part must have the shape of the first, and LSE its leading dims")
        if not (o_i.is_contiguous() and l_i.is_contiguous()):
            raise ValueError("parts must be contiguous")
    if sinks is not None:
        _dev(sinks, "sinks", torch.float32)
        if sink_rows is None:
            raise ValueError("sink_rows is needed with sinks (Tq for [B, H, Tq, dv] rows)")
    if out is None:
        out = torch.empty(shape, dtype=dt, device=o_parts[0].device)
    if lse is None:
        lse = torch.empty(shape[:-1], dtype=torch.float32, device=o_parts[0].device)
    a = _merge_args(o_parts, lse_parts, out, lse, sinks, sink_rows)
    _check(lib().arc_attn_merge(ctypes.byref(a), _stream(stream)), "arc_attn_merge")
    return out, lse


def plan(op: int, args) -> dict:
    """arc_plan on a filled args struct: which kernel a call launches, without launching it."""
    info = PlanInfo()
    _check(lib().arc_plan(int(op), ctypes.byref(args), ctypes.byref(info)), "arc_plan")
    return {f: (getattr(info, f).decode() if f == "kernel" else getattr(info, f)) for f, _ in PlanInfo._fields_}


def plan_attn(q, k, v, out, lse, *, causal=True, sinks=None, flags=0):
    """Engagement record for an attn_fwd call with these tensors (nothing is launched)."""
    return plan(ARC_OP_ATTN, _attn_args(q, k, v, out, lse, sinks, 1.0, causal, flags, None))


def plan_mla(q_nope, q_rope, k_nope, k_rope, v, out, lse, *, causal=True, flags=0):
    return plan(ARC_OP_MLA, _mla_args(q_nope, q_rope, k_nope, k_rope, v, out, lse, 1.0, causal, flags, None))


def plan_sparse(q, kv, idx, out, lse, *, Dv=None, v=None, sinks=None, flags=0):
    Dv = Dv if Dv is not None else (v.shape[1] if v is not None else q.shape[-1])
    return plan(ARC_OP_SPARSE, _sparse_args(q, kv, idx, v, out, lse, sinks, Dv, 1.0, flags, None))


def plan_sparse_decode(q, kv, idx, out, lse, *, Dv=None, v=None, sinks=None, flags=0):
    Dv = Dv if Dv is not None else (v.shape[1] if v is not None else q.shape[-1])
    return plan(ARC_OP_SPARSE_DECODE, _sparse_args(q, kv, idx, v, out, lse, sinks, Dv, 1.0, flags, None))


def plan_decode(kv_type, q, k_cache, v_cache, *, Hkv, q_begin, n_q, kv_begin, n_kv, flags=0):
    seqs = make_seqs(q_begin, n_q, kv_begin, n_kv)
    a = _decode_args(kv_type, q, k_cache, v_cache, seqs, len(q_begin), Hkv, k_cache.shape[0], q, q, 1.0,
                     flags, None)
    return plan(ARC_OP_DECODE, a)


def plan_merge(o_parts, lse_parts, out, lse) -> dict:
    return plan(ARC_OP_MERGE, _merge_args(o_parts, lse_parts, out, lse, None, None))


def check_device_error(status, stream=None) -> int:
    return int(lib().arc_check_device_error(_p(status), _stream(stream)))


def selftest_timeout(status, timeout_ns: int, stream=None) -> int:
    return int(lib().arc_selftest_timeout(_p(status), int(timeout_ns), _stream(stream)))
