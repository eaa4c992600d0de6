"""Shared test utilities: tolerances and comparisons (no method arithmetic)."""
import numpy as np

# Tolerances of the parity bar: fp32 outputs rel-L2 <= 1e-5 and max-abs <= 1e-4; bf16
# outputs rel-L2 <= 5e-3 and max-abs <= 2e-2.  The log-domain outputs (lse, b_final, Lambda)
# of a bf16 problem are compared with errors measured against max(1, |ref|) element-wise
# (for the L2 norm too): their magnitude ranges from ~0 (lse of a one-token row) to -O(T)
# (b_final), and an error in them is an error in a logit, i.e. absolute below 1.
TOL = {"f32": (1e-5, 1e-4), "bf16": (5e-3, 2e-2)}
# dalpha and dbeta of a bf16 problem: per-KV-head sums over every causal pair of terms of both
# signs, whose similarity x = <khat_i, khat_j> a bf16 computation forms from bf16 unit keys.
# Feeding the fp64 oracle bf16-rounded unit keys alone moves dalpha by 4e-3..7.3e-3 (rel-L2) on
# the test shapes while every other gradient moves by ~2e-4, so the bar for these two sums is
# rel-L2 <= 2e-2 (about 3x that rounding model), max error 2e-2 of the tensor's scale.
TOL_SUMS = {"f32": TOL["f32"], "bf16": (2e-2, 2e-2)}
SUM_GRADS = ("dalpha", "dbeta")
EVICT_BAND = 1e-3


def rel_l2(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def assert_close(name, got, ref, dtype, relative_max=False, tensor_scale=False, tol=None):
    """relative_max: log-domain outputs, errors measured against max(1, |ref|) elementwise.
    tensor_scale: gradients, whose max error is measured against max(1, max |ref|) of the
    whole tensor (a bf16 output carries ~2^-9 relative rounding whatever its magnitude)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    rl, ma = tol if tol is not None else TOL[dtype]
    if relative_max:
        den = np.linalg.norm(np.maximum(1.0, np.abs(ref)))
        r = float(np.linalg.norm(got - ref) / den) if ref.size else 0.0
    else:
        r = rel_l2(got, ref)
    err = np.abs(got - ref)
    if relative_max:
        err = err / np.maximum(1.0, np.abs(ref))
    elif tensor_scale and ref.size:
        err = err / max(1.0, float(np.abs(ref).max()))
    m = float(err.max()) if err.size else 0.0
    assert r <= rl and m <= ma, f"{name}: rel-L2 {r:.3e} (<= {rl}), max-abs {m:.3e} (<= {ma})"
    return r, m


def assert_grad_close(name, got, ref, dtype):
    """A gradient tensor against the oracle's: rel-L2 and max error against the tensor's own
    scale, with the bar of TOL_SUMS for the per-head sums dalpha, dbeta."""
    return assert_close(name, got, ref, dtype, tensor_scale=True,
                        tol=TOL_SUMS[dtype] if name in SUM_GRADS else None)
