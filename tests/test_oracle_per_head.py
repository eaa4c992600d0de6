"""Per-query-head decay in the oracle (the alternative to decay parameters per KV head).

Pins: rates that are equal across the heads of a group reproduce the per-KV-head results
(prefill and decode); with G = 1 the two readings coincide; the gradients (dk and dv summed over
the group's heads) equal central differences of the per-head forward; distinct per-head rates
give distinct heads."""
import numpy as np
import pytest

import oracle
from kv_cache_compression_ua_b200 import inputs as I


def case(T=24, B=2, H=4, Hkv=2, d=8, seed=3):
    w = I.Workload("ph", B, T, H, Hkv, d, "f32", seed, with_grad=True)
    return w, {k: v.astype(np.float64) for k, v in I.make_prefill_inputs(w).items()}


def per_head(x, G, rng=None):
    """Rates per query head: each KV head's repeated over its group, perturbed if rng is given."""
    y = dict(x)
    for n in ("a_q", "a_k"):
        y[n] = np.repeat(x[n], G, axis=2)
    for n in ("alpha", "beta"):
        y[n] = np.repeat(x[n], G)
    if rng is not None:
        for n in ("a_q", "a_k", "alpha", "beta"):
            y[n] = y[n] + 0.3 * rng.standard_normal(y[n].shape)
    return y


def test_shared_rates_reproduce_the_per_kv_head_decay():
    w, x = case()
    G = w.H // w.Hkv
    xo = {k: v for k, v in x.items() if k != "d_o"}
    ref = oracle.prefill_fwd(**xo, want_lambda=True)
    got = oracle.prefill_fwd_per_head(**{k: v for k, v in per_head(x, G).items() if k != "d_o"}, want_lambda=True)
    np.testing.assert_allclose(got["o"], ref["o"], atol=1e-12, rtol=0)
    np.testing.assert_allclose(got["lse"], ref["lse"], atol=1e-12, rtol=0)
    np.testing.assert_array_equal(got["b_final"], np.repeat(ref["b_final"], G, axis=1))
    np.testing.assert_array_equal(got["lam"], np.repeat(ref["lam"], G, axis=1))


def test_single_head_groups_coincide():
    w, x = case(H=2, Hkv=2)
    xo = {k: v for k, v in x.items() if k != "d_o"}
    a = oracle.prefill_fwd(**xo)
    b = oracle.prefill_fwd_per_head(**xo)
    for n in ("o", "lse", "b_final"):
        np.testing.assert_array_equal(a[n], b[n])


def test_distinct_rates_give_distinct_heads():
    w, x = case()
    G = w.H // w.Hkv
    y = per_head(x, G, np.random.default_rng(1))
    r = oracle.prefill_fwd_per_head(**{k: v for k, v in y.items() if k != "d_o"})
    s = oracle.prefill_fwd_per_head(**{k: v for k, v in per_head(x, G).items() if k != "d_o"})
    assert np.max(np.abs(r["b_final"][:, 0] - r["b_final"][:, 1])) > 1e-3   # heads of one group differ
    assert np.max(np.abs(r["o"] - s["o"])) > 1e-3


def _loss(y, d_o):
    r = oracle.prefill_fwd_per_head(**{k: v for k, v in y.items() if k != "d_o"}, nthreads=1)
    return float(np.sum(r["o"] * d_o))


def test_per_head_backward_matches_central_differences():
    w, x = case(T=7, B=1, H=4, Hkv=2, d=8, seed=9)
    G = w.H // w.Hkv
    y = per_head(x, G, np.random.default_rng(2))
    d_o = y["d_o"]
    gr = oracle.prefill_bwd_per_head(**y, nthreads=1)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "a_q": "da_q", "a_k": "da_k",
             "alpha": "dalpha", "beta": "dbeta"}
    for name, gname in names.items():
        base = y[name]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            h = 1e-6 * max(1.0, abs(base[idx]))
            yp = dict(y); yp[name] = base.copy(); yp[name][idx] += h
            ym = dict(y); ym[name] = base.copy(); ym[name][idx] -= h
            fd[idx] = (_loss(yp, d_o) - _loss(ym, d_o)) / (2 * h)
        assert gr[gname].shape == base.shape, gname
        err = np.max(np.abs(fd - gr[gname]))
        assert err <= 1e-6 * (1.0 + np.max(np.abs(fd))), (name, err)


def test_shared_rates_reproduce_the_per_kv_head_decode():
    """A cache of one head per query head, filled from the keys and values repeated over each
    group and stepped with rates repeated over it, gives the per-KV-head decode: the same
    outputs, and every copy of a group keeps the group's biases and evictions."""
    w, x = case(T=30, B=2, H=4, Hkv=2, d=8, seed=11)
    G = w.H // w.Hkv
    xo = {k: v for k, v in x.items() if k != "d_o"}
    ref_pf = oracle.prefill_fwd(**xo)
    p = 0.2
    logp = np.log(p)
    ref = oracle.DecodeCache(w.B, w.Hkv, w.d, w.T + 8)
    ref.fill_from_prefill(x["k"], x["v"], x["a_k"], ref_pf["b_final"], logp=logp)
    ph = oracle.DecodeCache(w.B, w.H, w.d, w.T + 8)
    ph.fill_from_prefill(np.repeat(x["k"], G, axis=2), np.repeat(x["v"], G, axis=2), np.repeat(x["a_k"], G, axis=2),
                         np.repeat(ref_pf["b_final"], G, axis=1), logp=logp)
    rng = np.random.default_rng(5)
    evicted = 0
    for s in range(6):
        q = rng.standard_normal((w.B, w.H, w.d))
        k = rng.standard_normal((w.B, w.Hkv, w.d))
        v = rng.standard_normal((w.B, w.Hkv, w.d))
        gt = rng.standard_normal((w.B, w.H, w.d))
        aq = rng.standard_normal((w.B, w.Hkv)) + 1.0
        ak = rng.standard_normal((w.B, w.Hkv))
        r1 = oracle.decode_step(ref, q, k, v, gt, aq, ak, x["alpha"], x["beta"], w.T + s, p)
        r2 = oracle.decode_step_per_head(ph, q, k, v, gt, np.repeat(aq, G, axis=1), np.repeat(ak, G, axis=1),
                                         np.repeat(x["alpha"], G), np.repeat(x["beta"], G), w.T + s, p)
        np.testing.assert_allclose(r2["o"], r1["o"], atol=1e-12, rtol=0)
        np.testing.assert_array_equal(ph.n, np.repeat(ref.n, G, axis=1))
        for b in range(w.B):
            for h in range(w.H):
                n = ref.n[b, h // G]
                np.testing.assert_array_equal(ph.pos[b, h, :n], ref.pos[b, h // G, :n])
                np.testing.assert_allclose(ph.b[b, h, :n], ref.b[b, h // G, :n], atol=1e-12, rtol=0)
        evicted += int(r1["evict"].sum())
    assert evicted > 0
