"""Helpers for the GPU parity tests: tolerances and comparisons against the oracle.

Tolerances (from the problem statement): max|out - oracle| <= 1e-2 * max|oracle|
+ 1e-3 for a bf16 KV cache and 3e-2 * max|oracle| + 1e-3 for FP8; |lse - oracle|
<= 1e-3 absolute.  Rows that see nothing must match exactly (out 0, lse -inf).
"""
import numpy as np
import torch

import mla_workloads as W

LSE_TOL = 1e-3


def out_rel_tol(kv):
    return 1e-2 if kv == W.KV_BF16 else 3e-2


def assert_matches_oracle(out, lse, ref_o, ref_l, kv, what=""):
    """out [n,512] (any float tensor), lse [n]; ref_* fp64 numpy arrays."""
    o = out.detach().to("cpu").to(torch.float64).reshape(-1, 512).numpy()
    l = lse.detach().to("cpu").to(torch.float64).reshape(-1).numpy()
    assert o.shape == ref_o.shape, (o.shape, ref_o.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    bound = out_rel_tol(kv) * np.abs(ref_o).max() + 1e-3
    err = np.abs(o - ref_o).max()
    assert err <= bound, f"{what}: max|out-oracle| = {err:.3e} > {bound:.3e}"
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(l)), f"{what}: lse finiteness differs"
    assert np.array_equal(l[~fin], ref_l[~fin]), f"{what}: infinite lse differs"
    if fin.any():
        lerr = np.abs(l[fin] - ref_l[fin]).max()
        assert lerr <= LSE_TOL, f"{what}: max|lse-oracle| = {lerr:.3e}"
    return err, bound


def require_gpu():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
