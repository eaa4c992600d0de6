"""Pins of the oracle's ablation variants against facts that do not come from the oracle.

The variants are the ablations of "A Self-Pruning Transformer: Extreme KV-Cache Compression
with Universal Attention" (paperlayer.ai summary, §5.4 with Table 3 and App. E with Table 6;
ai4snews synopsis, interpretation paragraph): decay mechanisms dropped from the geometric
mean, and Qwen3-style query normalisation.  With the mechanism set M on,
D = (prod_{m in M} r_m)^(1/|M|).

* every single mechanism and every pair has a closed form for Lambda (alpha = 0 makes the
  similarity rate the constant softplus(beta)); the similarity-only case with alpha != 0 is
  checked against torch's cosine similarity and a cumulative sum;
* a switched-off mechanism is ignored: its veto no longer zeroes Lambda, its logit gets an
  exactly zero gradient, while the veto of a mechanism still on stands;
* the query norm equals plain UA on queries normalised by torch's rms_norm, and makes the
  output invariant (to eps) under rescaling q;
* the analytic backward equals central finite differences for each variant;
* the decode step with p = 0 reproduces the variant's prefill rows and final biases, and for
  p > 0 keeps exactly the pairs the variant's brute-force Lambda keeps.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import VAR_NO_K, VAR_NO_Q, VAR_NO_SIM, VAR_QNORM
from kv_cache_compression_ua_b200 import inputs as I


def small_case(T=40, B=2, H=4, Hkv=2, d=16, seed=7):
    w = I.Workload("small", B, T, H, Hkv, d, "f32", seed)
    return w, {k: v.astype(np.float64) for k, v in I.make_prefill_inputs(w).items()}


def sp(x):
    return np.logaddexp(0.0, x)


def _check_lambda(x, variant, ref_fn, atol=1e-11):
    r = oracle.prefill_fwd(**x, want_lambda=True, variant=variant)
    B, T, Hkv = x["a_q"].shape
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    for b in range(B):
        for h in range(Hkv):
            ref = np.where(i >= j, ref_fn(b, h, i, j), 0.0)
            np.testing.assert_allclose(r["lam"][b, h], ref, atol=atol, rtol=0)
    assert np.max(np.abs(r["lam"])) > 1.0
    return r


def test_query_only_is_prefix_sum_of_query_rates():
    w, x = small_case(T=50)
    C = np.cumsum(sp(x["a_q"]), axis=1)                # C_i = sum_{l<=i} r_q(l)
    _check_lambda(x, VAR_NO_K | VAR_NO_SIM, lambda b, h, i, j: -(C[b, i, h] - C[b, j, h]))


def test_key_only_is_distance_times_key_rate():
    w, x = small_case(T=50)
    rk = sp(x["a_k"])
    _check_lambda(x, VAR_NO_Q | VAR_NO_SIM, lambda b, h, i, j: -(i - j) * rk[b, j, h])


def test_similarity_only_constant_rate():
    w, x = small_case(T=50)
    x["alpha"] = np.zeros_like(x["alpha"])
    x["beta"] = np.array([0.7, -1.3])
    _check_lambda(x, VAR_NO_Q | VAR_NO_K, lambda b, h, i, j: -(i - j) * sp(x["beta"][h]))


def test_similarity_only_matches_torch_cosine_similarity():
    w, x = small_case(T=24)
    x["alpha"] = np.array([2.5, -1.5])
    x["beta"] = np.array([-0.5, 0.25])
    k = torch.from_numpy(x["k"])                       # [B,T,Hkv,d]
    B, T, Hkv, _ = k.shape
    cos = torch.nn.functional.cosine_similarity(k[:, :, None], k[:, None, :], dim=-1)  # [B,l,j,Hkv]
    rsim = sp(x["alpha"][None, None, None, :] * cos.numpy() + x["beta"][None, None, None, :])
    lam = np.zeros((B, Hkv, T, T))
    for i in range(T):
        for j in range(i):
            lam[:, :, i, j] = -np.sum(rsim[:, j + 1:i + 1, j, :], axis=1)
    _check_lambda(x, VAR_NO_Q | VAR_NO_K, lambda b, h, i, j: lam[b, h, i, j], atol=1e-10)


def test_query_key_pair_is_square_root_form():
    w, x = small_case(T=50)
    S = np.cumsum(np.sqrt(sp(x["a_q"])), axis=1)
    rk = sp(x["a_k"])
    _check_lambda(x, VAR_NO_SIM,
                  lambda b, h, i, j: -np.sqrt(rk[b, j, h]) * (S[b, i, h] - S[b, j, h]))


def test_query_similarity_pair_constant_similarity():
    w, x = small_case(T=50)
    x["alpha"] = np.zeros_like(x["alpha"])
    x["beta"] = np.array([1.1, -0.4])
    S = np.cumsum(np.sqrt(sp(x["a_q"])), axis=1)
    _check_lambda(x, VAR_NO_K,
                  lambda b, h, i, j: -np.sqrt(sp(x["beta"][h])) * (S[b, i, h] - S[b, j, h]))


def test_key_similarity_pair_constant_similarity():
    w, x = small_case(T=50)
    x["alpha"] = np.zeros_like(x["alpha"])
    x["beta"] = np.array([1.1, -0.4])
    rk = sp(x["a_k"])
    _check_lambda(x, VAR_NO_Q,
                  lambda b, h, i, j: -(i - j) * np.sqrt(rk[b, j, h] * sp(x["beta"][h])))


@pytest.mark.parametrize("variant", [VAR_NO_Q, VAR_NO_K, VAR_NO_SIM, VAR_NO_Q | VAR_NO_K,
                                     VAR_NO_Q | VAR_NO_SIM, VAR_NO_K | VAR_NO_SIM])
def test_variant_prefix_equals_bruteforce(variant):
    w, x = small_case(T=32)
    r = oracle.prefill_fwd(**x, want_lambda=True, variant=variant)
    lb = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"], variant=variant)
    assert np.max(np.abs(r["lam"] - lb)) <= 1e-12 * max(1.0, np.max(np.abs(lb)))


def test_switched_off_mechanism_is_ignored_and_others_still_veto():
    w, x = small_case(T=32)
    base = oracle.prefill_fwd(**x, want_lambda=True, variant=VAR_NO_Q)
    xq = dict(x)
    xq["a_q"] = np.full_like(x["a_q"], -1e4)           # would veto if the query rate were on
    r = oracle.prefill_fwd(**xq, want_lambda=True, variant=VAR_NO_Q)
    np.testing.assert_array_equal(r["lam"], base["lam"])
    assert np.max(np.abs(r["lam"])) > 1.0
    xk = dict(x)
    xk["a_k"] = np.full_like(x["a_k"], -1e4)           # the key rate is still on: veto
    r = oracle.prefill_fwd(**xk, want_lambda=True, variant=VAR_NO_Q)
    assert np.all(r["lam"] == 0.0)


def test_all_mechanisms_off_is_rejected():
    w, x = small_case(T=8)
    with pytest.raises(ValueError):
        oracle.prefill_fwd(**x, variant=VAR_NO_Q | VAR_NO_K | VAR_NO_SIM)
    with pytest.raises(ValueError):
        oracle.prefill_fwd(**x, variant=16)


def test_query_norm_equals_torch_rms_norm_inputs():
    w, x = small_case(T=40)
    r = oracle.prefill_fwd(**x, variant=VAR_QNORM)
    xn = dict(x)
    d = x["q"].shape[-1]
    xn["q"] = torch.nn.functional.rms_norm(torch.from_numpy(x["q"]), (d,), eps=1e-6).numpy()
    ref = oracle.prefill_fwd(**xn)
    np.testing.assert_allclose(r["o"], ref["o"], atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(r["lse"], ref["lse"], atol=1e-12, rtol=1e-10)
    np.testing.assert_array_equal(r["b_final"], ref["b_final"])   # decay untouched
    plain = oracle.prefill_fwd(**x)
    assert np.max(np.abs(plain["o"] - r["o"])) > 1e-2


def test_query_norm_is_scale_invariant():
    w, x = small_case(T=40)
    r = oracle.prefill_fwd(**x, variant=VAR_QNORM)
    xs = dict(x)
    xs["q"] = 7.3 * x["q"]
    rs = oracle.prefill_fwd(**xs, variant=VAR_QNORM)
    np.testing.assert_allclose(rs["o"], r["o"], atol=2e-6, rtol=0)
    plain = oracle.prefill_fwd(**x)
    plain_s = oracle.prefill_fwd(**xs)
    assert np.max(np.abs(plain_s["o"] - plain["o"])) > 1e-2


# --------------------------------------------------------------------------- backward

def _loss(x, d_o, variant):
    r = oracle.prefill_fwd(**x, variant=variant, nthreads=1)
    return float(np.sum(r["o"] * d_o))


@pytest.mark.parametrize("variant", [VAR_NO_Q, VAR_NO_SIM, VAR_NO_Q | VAR_NO_K,
                                     VAR_NO_K | VAR_NO_SIM, VAR_QNORM | VAR_NO_K, VAR_QNORM])
def test_variant_backward_matches_central_differences(variant):
    w, x = small_case(T=9, B=1, H=4, Hkv=2, d=8, seed=21)
    rng = np.random.default_rng(0)
    d_o = rng.standard_normal(x["q"].shape)
    gr = oracle.prefill_bwd(**x, d_o=d_o, variant=variant, nthreads=1)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "a_q": "da_q", "a_k": "da_k",
             "alpha": "dalpha", "beta": "dbeta"}
    off = set()
    if variant & VAR_NO_Q:
        off.add("a_q")
    if variant & VAR_NO_K:
        off.add("a_k")
    if variant & VAR_NO_SIM:
        off |= {"alpha", "beta"}
    for name, gname in names.items():
        if name in off:
            assert np.all(gr[gname] == 0.0), name    # a switched-off mechanism has no gradient
            continue
        base = x[name]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            h = 1e-6 * max(1.0, abs(base[idx]))
            xp = dict(x); xp[name] = base.copy(); xp[name][idx] += h
            xm = dict(x); xm[name] = base.copy(); xm[name][idx] -= h
            fd[idx] = (_loss(xp, d_o, variant) - _loss(xm, d_o, variant)) / (2 * h)
        err = np.max(np.abs(fd - gr[gname]))
        assert err <= 1e-6 * (1.0 + np.max(np.abs(fd))), (name, err)
        assert np.max(np.abs(fd)) > 0


# --------------------------------------------------------------------------- decode

def _decode_sequence(T0, n, p, variant, seed=11):
    w, x = small_case(T=T0 + n, B=2, H=4, Hkv=2, d=16, seed=seed)
    pre = oracle.prefill_fwd(**{k: (v[:, :T0] if v.ndim >= 3 else v) for k, v in x.items()},
                             variant=variant)
    cache = oracle.DecodeCache(w.B, w.Hkv, w.d, T0 + n + 1)
    logp = math.log(p) if p > 0 else None
    cache.fill_from_prefill(x["k"][:, :T0], x["v"][:, :T0], x["a_k"][:, :T0], pre["b_final"],
                            logp=logp)
    outs = []
    for t in range(T0, T0 + n):
        out = oracle.decode_step(cache, x["q"][:, t], x["k"][:, t], x["v"][:, t], x["g"][:, t],
                                 x["a_q"][:, t], x["a_k"][:, t], x["alpha"], x["beta"], t, p,
                                 variant=variant)
        outs.append((t, out, cache.pos.copy(), cache.n.copy()))
    return w, x, cache, outs


@pytest.mark.parametrize("variant", [VAR_NO_Q, VAR_NO_K | VAR_NO_SIM, VAR_QNORM | VAR_NO_SIM])
def test_variant_decode_p0_reproduces_prefill(variant):
    T0, n = 14, 10
    w, x, cache, outs = _decode_sequence(T0, n, 0.0, variant)
    full = oracle.prefill_fwd(**x, variant=variant)
    for t, out, _, _ in outs:
        np.testing.assert_allclose(out["o"], full["o"][:, t], atol=1e-12, rtol=1e-10)
    T = T0 + n
    for b in range(w.B):
        for h in range(w.Hkv):
            np.testing.assert_allclose(cache.b[b, h, :T], full["b_final"][b, h], atol=1e-12)


@pytest.mark.parametrize("variant", [VAR_NO_Q, VAR_NO_SIM])
def test_variant_decode_kept_set_matches_bruteforce(variant):
    T0, n, p = 16, 20, 0.15
    w, x, cache, outs = _decode_sequence(T0, n, p, variant, seed=5)
    lb = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"], variant=variant)
    logp = math.log(p)
    n_evicted = 0
    for t, out, pos, nk in outs:
        for b in range(w.B):
            for h in range(w.Hkv):
                kept = set(int(a) for a in pos[b, h, :nk[b, h]])
                brute = set(int(j) for j in range(t) if lb[b, h, t, j] >= logp) | {t}
                assert kept == brute
                n_evicted += t + 1 - len(kept)
    assert n_evicted > 0
