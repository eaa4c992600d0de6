"""Shared test utilities: tolerances and comparisons (no method arithmetic)."""
import numpy as np

# Tolerances of the parity bar: fp32 outputs rel-L2 <= 1e-5 and max-abs <= 1e-4; bf16
# outputs rel-L2 <= 5e-3 and max-abs <= 2e-2.  The log-domain outputs (lse, b_final, Lambda)
# of a bf16 problem are compared with errors measured against max(1, |ref|) element-wise
# (for the L2 norm too): their magnitude ranges from ~0 (lse of a one-token row) to -O(T)
# (b_final), and an error in them is an error in a logit, i.e. absolute below 1.
TOL = {"f32": (1e-5, 1e-4), "bf16": (5e-3, 2e-2)}
# dalpha and dbeta of a bf16 problem: per-KV-head sums over every causal pair of terms of both
# signs.  Two bf16 effects reach them beyond the bars above:
#  * the similarity x = <khat_i, khat_j> formed from bf16 unit keys: feeding the fp64 oracle
#    bf16-rounded unit keys moves dalpha by 4e-3..7.3e-3 (rel-L2) on the test shapes, every
#    other gradient by ~2e-4; hence rel-L2 <= 2e-2 (about 3x), max error 2e-2 of the scale;
#  * the saved forward outputs: a bf16 forward rounds its probabilities before the PV and
#    row-sum products and stores o in bf16, and the backward's delta_i = sum dO o and its
#    recomputed rows (which then sum to 1 + eta_i) inherit that; row i's error eps_i moves the
#    gradients by -sum_i eps_i grad(lse_i), and lse's sensitivity to beta grows with the
#    sequence (Lambda sums D over the rows), so dbeta moves by up to a few 1e-2 absolute.  The
#    oracle's bf16 saved-output model reproduces this; its deviation from the exact gradients is
#    taken as an RMS over softmax-shift scales c (which values round up depends on the shift),
#    and the bar is SUM_MODEL_SIGMAS times it where that exceeds the fixed bar.
TOL_SUMS = {"f32": TOL["f32"], "bf16": (2e-2, 2e-2)}
SUM_GRADS = ("dalpha", "dbeta")
MODEL_SCALES = (1.0, 0.9, 0.8, 0.7, 0.6, 0.55)
SUM_MODEL_SIGMAS = 4.0
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


def sum_model_rms(bwd, ref, **kw):
    """RMS over MODEL_SCALES of the bf16 saved-output model's deviation in dalpha, dbeta.
    bwd: the oracle backward to call (oracle.prefill_bwd or a wrapper passing **kw on), with the
    problem's arguments in kw; ref: its exact result."""
    dev = {n: [] for n in SUM_GRADS}
    for c in MODEL_SCALES:
        m = bwd(**kw, bf16_saved_model=c)
        for n in SUM_GRADS:
            dev[n].append(np.asarray(m[n], np.float64) - np.asarray(ref[n], np.float64))
    return {n: np.sqrt(np.mean(np.square(dev[n]), axis=0)) for n in SUM_GRADS}


def assert_grad_close(name, got, ref, dtype, model_rms=None):
    """A gradient tensor against the oracle's: rel-L2, and the max error absolute for an fp32
    problem, against the tensor's own scale for a bf16 one.  The per-head sums dalpha, dbeta take the bar of TOL_SUMS, widened for a bf16
    problem to SUM_MODEL_SIGMAS x the saved-output model's RMS deviation (model_rms, from
    sum_model_rms) element by element where that is larger."""
    if name not in SUM_GRADS:
        # fp32: the absolute bar as it stands; bf16: the max error against the tensor's scale
        return assert_close(name, got, ref, dtype, tensor_scale=(dtype != "f32"))
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got)), name
    rl, ma = TOL_SUMS[dtype]
    sc = max(1.0, float(np.abs(ref).max())) if ref.size else 1.0
    allow = np.full(ref.shape, ma * sc)
    l2 = rl * np.linalg.norm(ref)
    if model_rms is not None and dtype == "bf16":
        rms = np.asarray(model_rms[name], np.float64)
        allow = np.maximum(allow, SUM_MODEL_SIGMAS * rms)
        l2 = max(l2, SUM_MODEL_SIGMAS * float(np.linalg.norm(rms)))
    err = np.abs(got - ref)
    assert np.all(err <= allow) and np.linalg.norm(got - ref) <= l2, (
        f"{name}: error {err} above {allow} (L2 {np.linalg.norm(got - ref):.3e} > {l2:.3e}?), ref {ref}")


def assert_close_model(name, got, ref, model, dtype, factor=3.0, relative_max=False):
    """assert_close with the bar widened to `factor` times the deviation of an oracle tolerance
    model (the same computation with the implementation's roundings) from the exact result,
    where that is larger: rel-L2 and max error each."""
    rl, ma = TOL[dtype]
    ref64 = np.asarray(ref, np.float64)
    mdl = np.asarray(model, np.float64)
    if relative_max:
        den = np.linalg.norm(np.maximum(1.0, np.abs(ref64)))
        mr = float(np.linalg.norm(mdl - ref64) / den)
        mm = float((np.abs(mdl - ref64) / np.maximum(1.0, np.abs(ref64))).max())
    else:
        mr = rel_l2(mdl, ref64)
        mm = float(np.abs(mdl - ref64).max())
    return assert_close(name, got, ref, dtype, relative_max=relative_max,
                        tol=(max(rl, factor * mr), max(ma, factor * mm)))
