"""Shared helpers for the GPU tests: upload seeded workloads and compare with the oracle."""
import numpy as np
import torch

import workloads as W

# Parity bars: bf16 inputs (and the quantised decode): max|dO| <= 2e-2, max|dLSE| <= 1e-3;
# fp32 reference mode: max|dO| <= 1e-3.
TOL_O_BF16 = 2e-2
TOL_LSE = 1e-3
TOL_O_F32 = 1e-3


def dev(x, dtype=None):
    """Upload a workloads array: uint16 arrays are bf16 bits."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(x).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, tol_o, tol_lse=TOL_LSE):
    """Element-wise comparison; -inf LSE must match exactly, finite ones within tolerance."""
    o = host(o_gpu)
    lse = host(lse_gpu)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), "non-finite output"
    d_o = float(np.abs(o - o_ref).max()) if o.size else 0.0
    ninf_ref, ninf = np.isneginf(lse_ref), np.isneginf(lse)
    assert np.array_equal(ninf_ref, ninf), "rows with no visible key differ"
    fin = ~ninf_ref
    d_l = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert d_o <= tol_o, f"max|dO| = {d_o:.3e} > {tol_o}"
    assert d_l <= tol_lse, f"max|dLSE| = {d_l:.3e} > {tol_lse}"
    return d_o, d_l


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")
