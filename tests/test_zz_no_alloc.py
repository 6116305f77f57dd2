"""The allocation-free decode entry point, against the oracle and the workspace entry point.

arc_attn_decode_q8_noalloc serves callers that cannot call cudaMalloc (an
engine whose planner owns all device memory, a fixed memory budget): it keeps
its split-KV partials in the library's own static 8 MiB device buffer.  These
checks call it through the C ABI, twice in a row on the shared buffer, and
compare each result element by element with the fp64 oracle and with
arc_attn_decode_q8 fed a caller workspace.  The cases reach every decode
kernel: the TMA split kernel, the cp.async split kernel (a cell stride that is
not a multiple of 16 bytes) and the CUDA-core kernel (ARC_FLAG_FORCE_SIMPLE).  The file
name sorts last so a stop-at-first-failure run has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import exact_attention_131_b200 as arc
from tests._util import TOL_LSE, TOL_O_BF16, compare, dev, host

pytestmark = pytest.mark.gpu


def _inputs(c):
    return dev(c.q), dev(c.k_cache), dev(c.v_cache)


def _kw(c):
    return dict(kv_type=c.kv_type, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                n_kv=c.n_kv, scale=c.scale)


# name -> (case, flags, the kernel arc_plan must name)
CASES = {
    "c5-q8_0": (lambda: W.config(5, kv_type=W.KV_Q8_0), 0, "decode_ws_kernel"),
    "c5-q4_0": (lambda: W.config(5, kv_type=W.KV_Q4_0), 0, "decode_ws_kernel"),
    "d64-ragged": (lambda: W.decode_case(3, 2, 0, 16, 4, 64, kv_type=W.KV_Q8_0, seed=41, n_q_list=[2, 4, 1],
                                         n_kv_list=[900, 33, 5]), 0, "decode_ws_kernel"),
    "cp_async-path": (lambda: W.decode_case(3, 2, 700, 6, 3, 128, kv_type=W.KV_Q4_0, seed=44), 0,
                      "decode_split_kernel"),
    "d256-32-rows": (lambda: W.decode_case(2, 0, 0, 32, 2, 256, kv_type=W.KV_Q8_0, seed=45, n_q_list=[2, 1],
                                           n_kv_list=[300, 77]), 0, "decode_ws_kernel"),
    "cuda-cores": (lambda: W.decode_case(2, 0, 0, 8, 2, 256, kv_type=W.KV_Q4_0, seed=46, n_q_list=[2, 1],
                                         n_kv_list=[300, 77]), 1, "simple_decode_kernel"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_decode_matches_oracle_and_workspace_entry_on_consecutive_calls(name):
    make, flags, kernel = CASES[name]
    c = make()
    q, kc, vc = _inputs(c)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv, flags=flags)
    assert info["kernel"].startswith(kernel)
    ro, rl = oracle.run_case(c)
    o_ws, l_ws = arc.attn_decode_q8(q, kc, vc, flags=flags, **_kw(c))
    torch.cuda.synchronize()
    compare(o_ws, l_ws, ro, rl, TOL_O_BF16, TOL_LSE)
    for _ in range(2):                      # two calls in a row on the shared buffer
        o = torch.full_like(o_ws, float("nan"))
        lse = torch.full_like(l_ws, float("nan"))
        arc.attn_decode_q8_noalloc(q, kc, vc, out=o, lse=lse, flags=flags, **_kw(c))
        torch.cuda.synchronize()
        compare(o, lse, ro, rl, TOL_O_BF16, TOL_LSE)
        compare(o, lse, host(o_ws), host(l_ws), TOL_O_BF16, TOL_LSE)


def test_noalloc_decode_takes_no_device_memory():
    """With out / lse passed in, a call changes the device's free memory by nothing:
    no allocation happens on either side of the C ABI."""
    c = W.config(5, kv_type=W.KV_Q8_0)
    q, kc, vc = _inputs(c)
    o = torch.empty(c.n_tok, c.H, c.D, device="cuda")
    lse = torch.empty(c.n_tok, c.H, device="cuda")
    arc.attn_decode_q8_noalloc(q, kc, vc, out=o, lse=lse, **_kw(c))      # first call: address lookup
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        arc.attn_decode_q8_noalloc(q, kc, vc, out=o, lse=lse, **_kw(c))
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    ro, rl = oracle.run_case(c)
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


class _DevBuf:
    """A raw device allocation of the current driver context, shaped like the tensor it holds."""

    def __init__(self, cu, host):
        self.cu, self.host = cu, np.ascontiguousarray(host)
        self.shape = self.host.shape
        err, self.ptr = cu.cuMemAlloc(max(1, self.host.nbytes))
        assert err == cu.CUresult.CUDA_SUCCESS, err
        if self.host.nbytes:
            (err,) = cu.cuMemcpyHtoD(self.ptr, self.host.ctypes.data, self.host.nbytes)
            assert err == cu.CUresult.CUDA_SUCCESS, err

    def data_ptr(self):
        return int(self.ptr)

    def read(self):
        out = np.empty_like(self.host)
        (err,) = self.cu.cuMemcpyDtoH(out.ctypes.data, self.ptr, out.nbytes)
        assert err == self.cu.CUresult.CUDA_SUCCESS, err
        return out

    def free(self):
        self.cu.cuMemFree(self.ptr)


def test_noalloc_decode_in_a_second_context():
    """The static scratch has a different device address in every CUDA context.  After a
    call in the primary context (torch's), a call made with a second context current
    (created through the driver API, its buffers allocated there) must use that context's
    address; both results are checked against the oracle."""
    from cuda.bindings import driver as cu

    c = W.decode_case(2, 4, 700, 16, 4, 128, kv_type=W.KV_Q8_0, seed=47)
    q, kc, vc = _inputs(c)
    info = arc.plan_decode(c.kv_type, q, kc, vc, Hkv=c.Hkv, q_begin=c.q_begin, n_q=c.n_q, kv_begin=c.kv_begin,
                           n_kv=c.n_kv)
    assert info["splits"] > 1                       # the partials go through the scratch
    ro, rl = oracle.run_case(c)
    o, lse = arc.attn_decode_q8_noalloc(q, kc, vc, **_kw(c))
    torch.cuda.synchronize()
    compare(o, lse, ro, rl, TOL_O_BF16, TOL_LSE)

    (err,) = cu.cuInit(0)
    assert err == cu.CUresult.CUDA_SUCCESS, err
    err, device = cu.cuDeviceGet(torch.cuda.current_device())
    assert err == cu.CUresult.CUDA_SUCCESS, err
    err, ctx = cu.cuCtxCreate(0, device)            # made current on this thread
    assert err == cu.CUresult.CUDA_SUCCESS, err
    bufs = []
    try:
        dq, dkc, dvc = (_DevBuf(cu, x) for x in (c.q.astype(np.float32), c.k_cache, c.v_cache))
        do = _DevBuf(cu, np.full((c.n_tok, c.H, c.D), np.nan, dtype=np.float32))
        dl = _DevBuf(cu, np.full((c.n_tok, c.H), np.nan, dtype=np.float32))
        bufs = [dq, dkc, dvc, do, dl]
        seqs = arc.make_seqs(c.q_begin, c.n_q, c.kv_begin, c.n_kv)
        a = arc._decode_args(c.kv_type, dq, dkc, dvc, seqs, len(c.q_begin), c.Hkv, c.n_cells, do, dl, c.scale, 0,
                             None)
        for _ in range(2):
            st = arc.lib().arc_attn_decode_q8_noalloc(ctypes.byref(a), None)
            assert st == arc.ARC_OK, arc.status_string(st)
            (err,) = cu.cuCtxSynchronize()
            assert err == cu.CUresult.CUDA_SUCCESS, err
            compare(torch.from_numpy(do.read()), torch.from_numpy(dl.read()), ro, rl, TOL_O_BF16, TOL_LSE)
    finally:
        for b in bufs:
            b.free()
        cu.cuCtxDestroy(ctx)                        # pops it: torch's context is current again
    o2, lse2 = arc.attn_decode_q8_noalloc(q, kc, vc, **_kw(c))
    torch.cuda.synchronize()
    compare(o2, lse2, ro, rl, TOL_O_BF16, TOL_LSE)
