"""Comparison helpers for the GPU parity tests.

Tolerances: max |O_gpu - O_ref| <= 2e-2, mean |O_gpu - O_ref| <= 2e-3 and
max |LSE_gpu - LSE_ref| <= 1e-3, for bf16 inputs with fp32 accumulation.
The pages give no numeric tolerance of their own (the Ales Analytics
kernels page defers to a tolerance page that is not among them); these are
the stated targets for this library, against the fp64 oracle.
"""
import numpy as np
import torch

TOL_O_MAX = 2e-2
TOL_O_MEAN = 2e-3
TOL_LSE_MAX = 1e-3


def to64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def compare(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    og = to64(o_gpu)
    assert og.shape == o_ref.shape, (what, og.shape, o_ref.shape)
    assert np.all(np.isfinite(og)), f"{what}: non-finite output"
    err = np.abs(og - o_ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= TOL_O_MAX, f"{what}: max |dO| = {mx:.3e}"
    assert mean <= TOL_O_MEAN, f"{what}: mean |dO| = {mean:.3e}"
    out = {"o_max": mx, "o_mean": mean}
    if lse_ref is not None:
        lg = to64(lse_gpu)
        assert lg.shape == lse_ref.shape, (what, lg.shape, lse_ref.shape)
        inf_ref = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lg), inf_ref), f"{what}: -inf LSE pattern differs"
        fin = ~inf_ref
        le = np.abs(lg[fin] - lse_ref[fin])
        lmx = float(le.max()) if le.size else 0.0
        assert lmx <= TOL_LSE_MAX, f"{what}: max |dLSE| = {lmx:.3e}"
        out["lse_max"] = lmx
    return out
