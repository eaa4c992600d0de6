"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin is chosen so that a plausible slip (a dropped term, a sign, an off-by-one in
the causal sum, a transposed operand, a wrong RoPE pairing) fails at least one test:

* prefix-form Lambda equals the O(T^3) direct per-(i,j) sum;
* veto: any single rate at exactly zero gives Lambda == 0 (ai4snews synopsis, veto
  property of the geometric mean);
* all rates zero reduces UA to causal RoPE softmax attention, checked against torch's
  SDPA with RoPE written in complex form (a library routine plus an independent
  formulation of the rotation);
* r_k = r_sim = 1 reduces the decay to FoX's scalar forget gate (paperlayer.ai summary,
  §3), whose accumulated bias has the closed form -(F_i - F_j), F_i = sum_{l<=i} r_q(l)^(1/3);
* a hand-derived worked example with integral Lambda (tests/golden);
* the decode step: p = 0 reproduces the prefill rows and final biases; for p > 0 the
  kept set equals the brute-force set {j : Lambda_tj >= log p}; biases never increase
  and evicted pairs never return (paperlayer.ai summary, §4.2);
* the analytic backward equals fp64 central finite differences on every coordinate.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_case(T=40, B=2, H=4, Hkv=2, d=16, seed=7, dtype="f32"):
    w = I.Workload("small", B, T, H, Hkv, d, dtype, seed)
    return w, {k: v.astype(np.float64) for k, v in I.make_prefill_inputs(w).items()}


def rope_complex(x, theta):
    """RoPE as complex multiplication: z_m = x_m + i x_{m+d/2} times exp(i pos theta^(-2m/d))."""
    B, T, H, d = x.shape
    half = d // 2
    z = torch.complex(x[..., :half], x[..., half:])
    m = torch.arange(half, dtype=torch.float64)
    freq = theta ** (-2.0 * m / d)
    pos = torch.arange(T, dtype=torch.float64)
    rot = torch.polar(torch.ones(T, half, dtype=torch.float64), pos[:, None] * freq[None, :])
    z = z * rot[None, :, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


# --------------------------------------------------------------------------- Lambda


def test_lambda_prefix_equals_bruteforce():
    w, x = small_case(T=48)
    r = oracle.prefill_fwd(**x, want_lambda=True)
    lb = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    assert np.max(np.abs(r["lam"] - lb)) <= 1e-12 * max(1.0, np.max(np.abs(lb)))
    assert np.max(np.abs(lb)) > 1.0   # non-trivial decay


def test_lambda_structure_and_bfinal():
    w, x = small_case(T=64)
    r = oracle.prefill_fwd(**x, want_lambda=True)
    lam = r["lam"]
    T = w.T
    assert np.all(np.diagonal(lam, axis1=2, axis2=3) == 0.0)
    tril = np.tril(np.ones((T, T), bool))
    assert np.all(lam[..., tril] <= 0.0)
    # non-increasing down every column (i increasing, j fixed, i >= j)
    diff = lam[:, :, 1:, :] - lam[:, :, :-1, :]
    assert np.all(diff[..., np.tril(np.ones((T - 1, T), bool), k=0)] <= 0.0)
    np.testing.assert_array_equal(r["b_final"], lam[:, :, -1, :])


@pytest.mark.parametrize("which", ["a_q", "a_k", "sim"])
def test_veto_any_zero_rate_gives_zero_lambda(which):
    w, x = small_case(T=32)
    if which == "sim":
        x["alpha"] = np.zeros_like(x["alpha"])
        x["beta"] = np.full_like(x["beta"], -1e4)
    else:
        x[which] = np.full_like(x[which], -1e4)     # softplus(-1e4) == 0 exactly in fp64
    r = oracle.prefill_fwd(**x, want_lambda=True)
    assert np.all(r["lam"] == 0.0)
    assert np.all(r["b_final"] == 0.0)


def test_fox_closed_form():
    """alpha=0, beta=a_k=log(e-1) makes r_sim = r_k = 1, so D[l,j] = r_q(l)^(1/3) and
    Lambda_ij = -(F_i - F_j) with F the prefix sum of r_q^(1/3)."""
    w, x = small_case(T=50)
    one = math.log(math.e - 1.0)
    x["alpha"] = np.zeros_like(x["alpha"])
    x["beta"] = np.full_like(x["beta"], one)
    x["a_k"] = np.full_like(x["a_k"], one)
    r = oracle.prefill_fwd(**x, want_lambda=True)
    rq = np.log1p(np.exp(x["a_q"]))                    # [B,T,Hkv]
    F = np.cumsum(np.cbrt(rq), axis=1)                 # F_i = sum_{l<=i}
    for b in range(w.B):
        for h in range(w.Hkv):
            Fi = F[b, :, h]
            ref = -(Fi[:, None] - Fi[None, :])
            ref = np.tril(ref)
            np.testing.assert_allclose(r["lam"][b, h], ref, atol=1e-11, rtol=0)


def test_hand_worked_example_prefill():
    ex = json.load(open(os.path.join(GOLDEN, "hand_worked_example.json")))
    x = _worked_inputs(ex, T=4)
    r = oracle.prefill_fwd(**x, want_lambda=True)
    np.testing.assert_allclose(r["lam"][0, 0], np.array(ex["lambda"], float), atol=1e-12)
    np.testing.assert_allclose(r["b_final"][0, 0], np.array(ex["b_final"], float), atol=1e-12)
    v = np.array(ex["values"], float)
    wts = np.exp(np.array(ex["lambda"][3], float))
    o3 = 0.5 * (wts @ v[:4]) / wts.sum()
    np.testing.assert_allclose(r["o"][0, 3, 0], o3, atol=1e-12)


def _worked_inputs(ex, T):
    def logit(rate):
        return math.log(math.expm1(rate))
    keys = np.array(ex["keys"][:T], float)
    vals = np.array(ex["values"][:T], float)
    return {
        "q": np.zeros((1, T, 1, 2)), "k": keys.reshape(1, T, 1, 2), "v": vals.reshape(1, T, 1, 2),
        "g": np.zeros((1, T, 1, 2)),
        "a_q": np.array([logit(r) for r in ex["rates"]["r_q"][:T]]).reshape(1, T, 1),
        "a_k": np.array([logit(r) for r in ex["rates"]["r_k"][:T]]).reshape(1, T, 1),
        "alpha": np.array([logit(ex["r_sim_at_c1"]) - logit(ex["r_sim_at_c0"])]),
        "beta": np.array([logit(ex["r_sim_at_c0"])]),
    }


def test_hand_worked_example_decode():
    ex = json.load(open(os.path.join(GOLDEN, "hand_worked_example.json")))
    x6 = _worked_inputs(ex, T=6)
    x4 = {k: (v[:, :4] if v.ndim >= 2 else v) for k, v in x6.items()}
    r = oracle.prefill_fwd(**x4)
    cache = oracle.DecodeCache(1, 1, 2, 8)
    cache.fill_from_prefill(x4["k"], x4["v"], x4["a_k"], r["b_final"], logp=ex["log_p"])
    assert list(cache.pos[0, 0, :cache.n[0, 0]]) == ex["kept_after_prefill"]
    p = math.exp(ex["log_p"])
    v = np.array(ex["values"], float)
    for step in ex["decode"]:
        t = step["pos"]
        out = oracle.decode_step(cache, np.zeros((1, 1, 2)), x6["k"][:, t], x6["v"][:, t],
                                 np.zeros((1, 1, 2)), x6["a_q"][:, t], x6["a_k"][:, t],
                                 x6["alpha"], x6["beta"], t, p, band=0.0)
        n = cache.n[0, 0]
        pos = [int(a) for a in cache.pos[0, 0, :n]]
        assert pos == step["kept_positions"]
        for ps, bias in step["bias_after"].items():
            ps = int(ps)
            if ps in pos:
                assert abs(cache.b[0, 0, pos.index(ps)] - bias) < 1e-12
        # attention with q = 0: weights exp(b) over survivors + new token (b = 0)
        wts = np.array([math.exp(cache.b[0, 0, i]) for i in range(n)])
        o = 0.5 * (wts @ v[np.array(pos)]) / wts.sum()
        np.testing.assert_allclose(out["o"][0, 0], o, atol=1e-12)


# --------------------------------------------------------------------------- attention


def test_all_rates_zero_is_causal_rope_sdpa():
    w, x = small_case(T=37, H=4, Hkv=2, d=16)
    x["a_q"][:] = -1e4
    x["a_k"][:] = -1e4
    x["alpha"][:] = 0.0
    x["beta"][:] = -1e4
    x["g"][:] = 60.0                      # sigmoid == 1 in fp64
    r = oracle.prefill_fwd(**x)
    q = torch.from_numpy(x["q"])
    k = torch.from_numpy(x["k"])
    k = k / k.norm(dim=-1, keepdim=True)
    qr = rope_complex(q, 500000.0).transpose(1, 2)          # [B,H,T,d]
    kr = rope_complex(k, 500000.0).transpose(1, 2)          # [B,Hkv,T,d]
    v = torch.from_numpy(x["v"]).transpose(1, 2)
    G = w.H // w.Hkv
    kr = kr.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, v, is_causal=True, scale=w.scale)
    np.testing.assert_allclose(r["o"], ref.transpose(1, 2).numpy(), atol=1e-12, rtol=1e-10)
    logits = (qr @ kr.transpose(-1, -2)) * w.scale
    mask = torch.triu(torch.ones(w.T, w.T, dtype=torch.bool), 1)
    lse = torch.logsumexp(logits.masked_fill(mask, -math.inf), dim=-1)
    np.testing.assert_allclose(r["lse"], lse.numpy(), atol=1e-12, rtol=1e-12)


def test_rows_are_convex_combinations():
    """With v == 1 and the gate saturated, every output equals 1 (softmax rows sum to 1)."""
    w, x = small_case(T=33)
    x["v"][:] = 1.0
    x["g"][:] = 60.0
    r = oracle.prefill_fwd(**x)
    np.testing.assert_allclose(r["o"], 1.0, atol=1e-13)


def test_gate_is_elementwise_sigmoid():
    w, x = small_case(T=20)
    r1 = oracle.prefill_fwd(**x)
    x2 = dict(x)
    x2["g"] = np.full_like(x["g"], 60.0)
    r2 = oracle.prefill_fwd(**x2)
    np.testing.assert_allclose(r1["o"], r2["o"] / (1.0 + np.exp(-x["g"])), atol=1e-13)


def test_row_and_unit_masks_select_outputs():
    w, x = small_case(T=24)
    full = oracle.prefill_fwd(**x)
    rm = np.zeros(w.T, np.uint8)
    rm[[0, 5, 23]] = 1
    um = np.zeros(w.B * w.Hkv, np.uint8)
    um[3] = 1
    part = oracle.prefill_fwd(**x, row_mask=rm, unit_mask=um)
    b, kvh = 3 // w.Hkv, 3 % w.Hkv
    G = w.H // w.Hkv
    hs = slice(kvh * G, (kvh + 1) * G)
    np.testing.assert_array_equal(part["o"][b, [0, 5, 23], hs], full["o"][b, [0, 5, 23], hs])
    np.testing.assert_array_equal(part["b_final"][b, kvh], full["b_final"][b, kvh])
    assert np.isnan(part["o"][0, :, :]).all()


# --------------------------------------------------------------------------- decode


def _decode_sequence(T0=20, n_steps=12, p=0.0, seed=11, B=2, H=4, Hkv=2, d=16):
    """Prefill T0 tokens, then decode n_steps tokens drawn as positions T0.. of one
    longer sequence, returning the per-step outputs and the concatenated inputs."""
    w, x = small_case(T=T0 + n_steps, B=B, H=H, Hkv=Hkv, d=d, seed=seed)
    pre = {k: (v[:, :T0] if v.ndim >= 2 else v) for k, v in x.items()}
    r = oracle.prefill_fwd(**pre)
    cache = oracle.DecodeCache(B, Hkv, d, T0 + n_steps + 1)
    logp = math.log(p) if p > 0 else None
    cache.fill_from_prefill(pre["k"], pre["v"], pre["a_k"], r["b_final"], logp=logp)
    steps = []
    for t in range(T0, T0 + n_steps):
        pos_before = cache.pos.copy()
        n_before = cache.n.copy()
        b_before = cache.b.copy()
        out = oracle.decode_step(cache, x["q"][:, t], x["k"][:, t], x["v"][:, t], x["g"][:, t],
                                 x["a_q"][:, t], x["a_k"][:, t], x["alpha"], x["beta"], t, p)
        steps.append({"t": t, "out": out, "pos_before": pos_before, "n_before": n_before,
                      "b_before": b_before, "pos": cache.pos.copy(), "n": cache.n.copy(),
                      "b": cache.b.copy()})
    return w, x, cache, steps


def test_decode_p0_reproduces_prefill_rows_and_biases():
    T0, n = 20, 12
    w, x, cache, steps = _decode_sequence(T0, n, p=0.0)
    full = oracle.prefill_fwd(**x)
    for st in steps:
        np.testing.assert_allclose(st["out"]["o"], full["o"][:, st["t"]], atol=1e-12, rtol=1e-10)
    T = T0 + n
    for b in range(w.B):
        for h in range(w.Hkv):
            assert cache.n[b, h] == T
            np.testing.assert_array_equal(cache.pos[b, h, :T], np.arange(T))
            np.testing.assert_allclose(cache.b[b, h, :T], full["b_final"][b, h], atol=1e-12)


@pytest.mark.parametrize("p", [0.05, 0.15])
def test_decode_kept_set_matches_bruteforce(p):
    T0, n = 16, 20
    w, x, cache, steps = _decode_sequence(T0, n, p=p, seed=5)
    lb = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    logp = math.log(p)
    n_evicted = 0
    for st in steps:
        t = st["t"]
        for b in range(w.B):
            for h in range(w.Hkv):
                kept = set(int(a) for a in st["pos"][b, h, :st["n"][b, h]])
                brute = set(int(j) for j in range(t) if lb[b, h, t, j] >= logp) | {t}
                assert kept == brute
                n_evicted += t + 1 - len(kept)
    assert n_evicted > 0


def test_decode_bias_monotone_and_no_return():
    w, x, cache, steps = _decode_sequence(16, 24, p=0.15, seed=9)
    for st in steps:
        for b in range(w.B):
            for h in range(w.Hkv):
                before = {int(ps): st["b_before"][b, h, i]
                          for i, ps in enumerate(st["pos_before"][b, h, :st["n_before"][b, h]])}
                after = {int(ps): st["b"][b, h, i]
                         for i, ps in enumerate(st["pos"][b, h, :st["n"][b, h]])}
                for ps, bias in after.items():
                    if ps == st["t"]:
                        assert bias == 0.0
                    else:
                        assert ps in before           # evicted pairs never come back
                        assert bias <= before[ps]     # biases only decrease
                order = [int(a) for a in st["pos"][b, h, :st["n"][b, h]]]
                assert order == sorted(order)         # stable compaction


def test_compact_order_is_stable_partition():
    rng = np.random.default_rng(3)
    keep = rng.random(1000) < 0.3
    order = oracle.compact_order(keep)
    ref = sorted(range(len(keep)), key=lambda j: not keep[j])[: int(keep.sum())]
    assert list(order) == ref


# --------------------------------------------------------------------------- backward


def _loss(x, d_o):
    r = oracle.prefill_fwd(**x, nthreads=1)
    return float(np.sum(r["o"] * d_o))


def test_backward_matches_central_differences_everywhere():
    w, x = small_case(T=9, B=1, H=4, Hkv=2, d=8, seed=21)
    rng = np.random.default_rng(0)
    d_o = rng.standard_normal(x["q"].shape)
    gr = oracle.prefill_bwd(**x, d_o=d_o, nthreads=1)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "a_q": "da_q", "a_k": "da_k",
             "alpha": "dalpha", "beta": "dbeta"}
    for name, gname in names.items():
        base = x[name]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            h = 1e-6 * max(1.0, abs(base[idx]))
            xp = dict(x); xp[name] = base.copy(); xp[name][idx] += h
            xm = dict(x); xm[name] = base.copy(); xm[name][idx] -= h
            fd[idx] = (_loss(xp, d_o) - _loss(xm, d_o)) / (2 * h)
        err = np.max(np.abs(fd - gr[gname]))
        assert err <= 1e-6 * (1.0 + np.max(np.abs(fd))), (name, err)
        assert np.max(np.abs(fd)) > 0


def test_backward_vetoed_decay_has_zero_decay_grads():
    w, x = small_case(T=12, B=1, H=2, Hkv=1, d=8, seed=4)
    x["a_q"][:] = -1e4
    rng = np.random.default_rng(1)
    gr = oracle.prefill_bwd(**x, d_o=rng.standard_normal(x["q"].shape))
    assert np.all(gr["da_k"] == 0) and np.all(gr["dalpha"] == 0) and np.all(gr["dbeta"] == 0)
    assert np.all(np.isfinite(gr["dq"])) and np.all(np.isfinite(gr["dk"]))


def test_deferred_compaction_equals_step_by_step():
    """Deferred compaction (pairs left in place, compacted once at the end) attends over the same
    pairs in the same order as step-by-step compaction: an evicted pair's bias never rises back
    above log p (paperlayer.ai summary, §4.2: the bias is monotone), so outputs agree bit for bit
    and the compacted cache is the same."""
    T0, n, p = 16, 20, 0.15
    w, x = small_case(T=T0 + n, B=2, H=4, Hkv=2, d=16, seed=13)
    pre = oracle.prefill_fwd(**{k: (v[:, :T0] if v.ndim >= 3 else v) for k, v in x.items()})
    caches = []
    for _ in range(2):
        c = oracle.DecodeCache(w.B, w.Hkv, w.d, T0 + n + 1)
        c.fill_from_prefill(x["k"][:, :T0], x["v"][:, :T0], x["a_k"][:, :T0], pre["b_final"], logp=math.log(p))
        caches.append(c)
    eager, lazy = caches
    n_evicted = 0
    for t in range(T0, T0 + n):
        args = (x["q"][:, t], x["k"][:, t], x["v"][:, t], x["g"][:, t], x["a_q"][:, t], x["a_k"][:, t],
                x["alpha"], x["beta"], t, p)
        n0 = lazy.n.copy()
        re = oracle.decode_step(eager, *args)
        rl = oracle.decode_step(lazy, *args, defer=True)
        np.testing.assert_array_equal(rl["o"], re["o"])
        assert np.all(lazy.n == n0 + 1)
        for b in range(w.B):
            for h in range(w.Hkv):
                assert list(rl["kept_order"][b, h, :n0[b, h]]) == list(range(n0[b, h]))
        n_evicted += int(re["evict"].sum())
    lazy.compact(p)
    assert n_evicted > 0
    np.testing.assert_array_equal(lazy.n, eager.n)
    for b in range(w.B):
        for h in range(w.Hkv):
            m = eager.n[b, h]
            for name in ("k", "v", "ak", "pos", "b"):
                np.testing.assert_array_equal(getattr(lazy, name)[b, h, :m], getattr(eager, name)[b, h, :m])


@pytest.mark.parametrize("shift", [1, 37, 100000])
def test_rope_relative_position_invariance(shift):
    """RoPE makes a logit depend on the positions only through their difference: moving every
    cached pair and the new token by the same offset leaves every decode output and bias
    unchanged (to fp64 rounding of the rotations).  A rotation applied with opposite senses to
    queries and keys would make the logit depend on the sum instead, and fail this."""
    T0, n, p = 24, 8, 0.15
    w, x = small_case(T=T0 + n, B=2, H=4, Hkv=2, d=16, seed=29)
    pre = {k: (v[:, :T0] if v.ndim >= 2 else v) for k, v in x.items()}
    r = oracle.prefill_fwd(**pre)
    caches = []
    for _ in range(2):
        c = oracle.DecodeCache(w.B, w.Hkv, w.d, T0 + n + 1)
        c.fill_from_prefill(pre["k"], pre["v"], pre["a_k"], r["b_final"], logp=math.log(p))
        caches.append(c)
    base, moved = caches
    moved.pos += shift
    for t in range(T0, T0 + n):
        args = (x["q"][:, t], x["k"][:, t], x["v"][:, t], x["g"][:, t], x["a_q"][:, t], x["a_k"][:, t],
                x["alpha"], x["beta"])
        a = oracle.decode_step(base, *args, t, p)
        b = oracle.decode_step(moved, *args, t + shift, p)
        np.testing.assert_allclose(b["o"], a["o"], atol=1e-9, rtol=0)
        np.testing.assert_array_equal(b["evict"], a["evict"])
    np.testing.assert_array_equal(moved.n, base.n)
    np.testing.assert_array_equal(moved.pos - shift, base.pos)
    np.testing.assert_array_equal(moved.b, base.b)


@pytest.mark.parametrize("c", [1.0, 0.9, 0.55])
def test_bf16_saved_output_model_single_token_closed_form(c):
    """The oracle backward's bf16 saved-output model (a tolerance model, not the method) on one
    token, where every quantity has a closed form: the probability's bf16 rounding of c gives
    the backward P = c / bf16(c), the output A = v, delta = sum dO * bf16(sigmoid(g) v), and at
    position 0 RoPE is the identity, so dq = scale * P * (<dA, v> - delta) * khat,
    dv = P * dA, dg = dO * v * sigmoid'(g); no pair, so dalpha = dbeta = 0.  The rounding is
    torch's bf16 conversion (round to nearest even)."""
    rng = np.random.default_rng(11)
    d, H, Hkv = 64, 2, 1
    x = {"q": rng.standard_normal((1, 1, H, d)), "k": rng.standard_normal((1, 1, Hkv, d)),
         "v": rng.standard_normal((1, 1, Hkv, d)), "g": rng.standard_normal((1, 1, H, d)),
         "a_q": rng.standard_normal((1, 1, Hkv)), "a_k": rng.standard_normal((1, 1, Hkv)),
         "alpha": np.array([2.0]), "beta": np.array([-1.0]), "d_o": rng.standard_normal((1, 1, H, d))}
    scale = d ** -0.5
    ex = oracle.prefill_bwd(**x, scale=scale)
    mo = oracle.prefill_bwd(**x, scale=scale, bf16_saved_model=c)
    bf = lambda a: torch.tensor(np.asarray(a, np.float64)).float().bfloat16().double().numpy()
    v = x["v"][0, 0, 0]
    khat = x["k"][0, 0, 0] / np.linalg.norm(x["k"][0, 0, 0])
    P = c / float(bf(c))
    for h in range(H):
        sg = 1.0 / (1.0 + np.exp(-x["g"][0, 0, h]))
        dA = x["d_o"][0, 0, h] * sg
        delta = float(np.sum(x["d_o"][0, 0, h] * bf(sg * v)))
        dS = P * (float(dA @ v) - delta)
        np.testing.assert_allclose(mo["dq"][0, 0, h], scale * dS * khat, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(mo["dg"][0, 0, h], x["d_o"][0, 0, h] * v * sg * (1 - sg), rtol=1e-12)
        np.testing.assert_allclose(ex["dq"][0, 0, h], 0.0, atol=1e-14)      # exact: dS = 0 at T = 1
    dA_sum = sum(x["d_o"][0, 0, h] / (1.0 + np.exp(-x["g"][0, 0, h])) for h in range(H))
    np.testing.assert_allclose(mo["dv"][0, 0, 0], P * dA_sum, rtol=1e-12)
    np.testing.assert_allclose(ex["dv"][0, 0, 0], dA_sum, rtol=1e-12)
    assert mo["dalpha"][0] == 0.0 and mo["dbeta"][0] == 0.0


def test_bf16_saved_output_model_off_is_the_method():
    w = I.Workload("m0", 1, 40, 4, 2, 64, "bf16", 5, with_grad=True)
    x = I.make_prefill_inputs(w)
    a = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta)
    b = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta, bf16_saved_model=0.0)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n])



def test_bf16_operand_model_single_token_closed_form():
    """The oracle forward's bf16-operand model (a tolerance model, not the method) on one token at
    position 0, where RoPE is the identity and the softmax has one term: o = v * sigmoid(g) as in
    the method, and lse = scale * <bf16(q), bf16(khat)> (torch's bf16 conversion, round to
    nearest even); with the model off, lse = scale * <q, khat>."""
    rng = np.random.default_rng(21)
    d, H = 64, 2
    x = {"q": rng.standard_normal((1, 1, H, d)) * 30, "k": rng.standard_normal((1, 1, 1, d)),
         "v": rng.standard_normal((1, 1, 1, d)), "g": rng.standard_normal((1, 1, H, d)),
         "a_q": rng.standard_normal((1, 1, 1)), "a_k": rng.standard_normal((1, 1, 1)),
         "alpha": np.array([2.0]), "beta": np.array([-1.0])}
    scale = d ** -0.5
    ex = oracle.prefill_fwd(**x, scale=scale)
    mo = oracle.prefill_fwd(**x, scale=scale, bf16_operands=True)
    bf = lambda a: torch.tensor(np.asarray(a, np.float64)).float().bfloat16().double().numpy()
    khat = x["k"][0, 0, 0] / np.linalg.norm(x["k"][0, 0, 0])
    for h in range(H):
        q = x["q"][0, 0, h]
        np.testing.assert_allclose(mo["lse"][0, h, 0], scale * float(bf(q) @ bf(khat)), rtol=1e-12)
        np.testing.assert_allclose(ex["lse"][0, h, 0], scale * float(q @ khat), rtol=1e-12)
        gate = 1.0 / (1.0 + np.exp(-x["g"][0, 0, h]))
        np.testing.assert_allclose(mo["o"][0, 0, h], x["v"][0, 0, 0] * gate, rtol=1e-12)
    assert abs(mo["lse"][0, 0, 0] - ex["lse"][0, 0, 0]) > 0          # the rounding is seen
