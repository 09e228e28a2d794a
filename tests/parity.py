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


# FP8 prefill.  The kernel rounds P (at most 2^8 under the conditional
# rescale) to E4M3 before P V: relative error at most 2^-4 for P in E4M3's
# normal range, at most 2^-10 absolute below it (where, for N(0,1)-like
# scores, the weights are small and the errors random).  Against the oracle on
# the same codes, element (i, c) of O may therefore differ by
#   2^-4 * sum_j w_ij |v_jc|   (worst case: every weight rounded the same way)
# plus the output rounding (bf16: 2^-9 relative, 2^-7 allowed) and 1e-3 for
# the sub-normal weights.  sum_j w_ij |v_jc| is the oracle's attention with
# |V| in place of V.  LSE comes from fp32 P: the bf16 tolerance holds.
FP8_P_REL = 2.0 ** -4
FP8_OUT_REL = 2.0 ** -7
FP8_ABS = 1e-3


def compare_fp8(o_gpu, o_ref, abs_v_ref, lse_gpu=None, lse_ref=None, what="", ds=None,
                vmax=0.0):
    """``ds`` [B, Hq, N] (optional): a bound on how far the GPU's scores of each
    row may sit from the oracle's because its operand codes differ (see
    code_flip_score_bound).  LSE is 1-Lipschitz in the max-norm of the scores,
    and the softmax weights move by a factor within exp(+-2 ds), so LSE gets
    ds more room and O (exp(2 ds) - 1) * vmax more."""
    og = to64(o_gpu)
    assert og.shape == o_ref.shape, (what, og.shape, o_ref.shape)
    assert np.all(np.isfinite(og)), f"{what}: non-finite output"
    err = np.abs(og - o_ref)
    bound = FP8_P_REL * abs_v_ref + FP8_OUT_REL * np.abs(o_ref) + FP8_ABS
    if ds is not None:
        bound = bound + (np.expm1(2.0 * ds) * vmax).transpose(0, 2, 1)[..., None]
    worst = float((err / bound).max()) if err.size else 0.0
    assert worst <= 1.0, f"{what}: error {worst:.3f} x the FP8 bound (max |dO| {err.max():.3e})"
    out = {"o_max": float(err.max()) if err.size else 0.0,
           "o_mean": float(err.mean()) if err.size else 0.0, "bound_frac": worst}
    if lse_ref is not None:
        lg = to64(lse_gpu)
        assert lg.shape == lse_ref.shape, (what, lg.shape, lse_ref.shape)
        le = np.abs(lg - lse_ref)
        tol = TOL_LSE_MAX + (ds if ds is not None else 0.0)
        assert np.all(le <= tol), f"{what}: max |dLSE| = {le.max():.3e}"
        out["lse_max"] = float(le.max())
    return out


def code_flip_score_bound(q8_gpu, q8_ref, q_scale, k8_gpu, k8_ref, k_scale, scale, causal,
                          window):
    """Largest |s_gpu - s_ref| over each row's visible keys when the GPU's Q
    and K codes differ from the oracle's (scales equal): per term
    |qg kg - qr kr| <= |qg - qr| |kg| + |qr| |kg - kr|.  -> [B, Hq, N]"""
    t = e4m3_table()

    def deq(codes, sc):
        N = codes.shape[1]
        return t[np.asarray(codes)] * np.repeat(np.asarray(sc).transpose(0, 2, 1), 128,
                                                axis=1)[:, :N, :, None]

    qg, qr = deq(q8_gpu, q_scale), deq(q8_ref, q_scale)
    kg, kr = deq(k8_gpu, k_scale), deq(k8_ref, k_scale)
    g = qg.shape[2] // kg.shape[2]
    kg, kr = np.repeat(kg, g, axis=2), np.repeat(kr, g, axis=2)
    ds = scale * (np.einsum("bihc,bjhc->bhij", np.abs(qg - qr), np.abs(kg)) +
                  np.einsum("bihc,bjhc->bhij", np.abs(qr), np.abs(kg - kr)))
    N = ds.shape[-1]
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    vis = np.ones((N, N), bool)
    if causal:
        vis &= j <= i
        if window > 0:
            vis &= j > i - window
    return np.where(vis, ds, 0.0).max(axis=-1)


def e4m3_table():
    """Values of all 256 E4M3 codes (NaN for the two NaN codes), for comparisons."""
    import oracle
    return np.array([oracle.e4m3_value(c) for c in range(256)])


def compare_codes(gpu, ref, exact, what="", rel_tie=2.0 ** -16, max_frac=1e-3):
    """E4M3 codes from the GPU against the oracle's.  A code may differ only
    where the exact pre-rounding value lies within `rel_tie` (relative) of
    the midpoint between the two codes' values -- fp32 arithmetic on the GPU
    against fp64 in the oracle may round such a value either way -- and then
    only to the neighbouring code."""
    g = np.asarray(gpu, dtype=np.uint8)
    r = np.asarray(ref, dtype=np.uint8)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    diff = g != r
    n = int(diff.sum())
    if n == 0:
        return 0
    assert n <= max_frac * g.size + 1, f"{what}: {n} of {g.size} codes differ"
    t = e4m3_table()
    gv, rv, y = t[g[diff]], t[r[diff]], np.asarray(exact, dtype=np.float64)[diff]
    mid = (gv + rv) / 2.0
    near = np.abs(y - mid) <= rel_tie * np.maximum(np.abs(y), 2.0 ** -9)
    # neighbours on the grid: no representable value strictly between them
    lo, hi = np.minimum(gv, rv), np.maximum(gv, rv)
    fin = t[np.isfinite(t)]
    between = np.array([np.any((fin > a) & (fin < b)) for a, b in zip(lo, hi)])
    assert np.all(near) and not np.any(between), f"{what}: codes differ away from a tie"
    return n
