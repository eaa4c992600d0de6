"""GPU parity of the split decode step of bf16 caches on the tensor cores (k_decode_tc, through
ua_decode_step_split) against the fp64 oracle in lockstep, compaction deferred.

Long caches (2.2k-4.1k live pairs: 5-8 slices of whole 128-entry tiles, ragged last tiles) and a
130-pair one over 12 steps at p = 0.15 (evictions in every slice) and p = 0; group sizes 1, 2, 3, 4
and 8; head dims 64 and 128.  Both sides start from the oracle prefill's biases.  Eviction
decisions must match the oracle's except within 1e-3 of log p, where the oracle adopts the GPU's
decision; outputs and the live biases are held to the bf16 bars.  A case with large query norms
drives the softmax shift up through the in-TMEM rescale, and a final ua_cache_compact must give
the oracle's compacted cache."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import EVICT_BAND, assert_close

pytestmark = pytest.mark.gpu


def dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt).contiguous()


def unpack_bits(words, n):
    bits = np.unpackbits(np.ascontiguousarray(words, np.uint32).view(np.uint8), bitorder="little")
    return bits[:n].astype(bool)


def run_lockstep(w, T0, steps, p, q_against_key=0.0):
    bf = torch.bfloat16
    x = I.make_prefill_inputs(w, T=T0, names=["q", "k", "v", "g", "a_q", "a_k", "alpha", "beta"])
    dd = {n: dev(a, bf if n in ("k", "v", "q", "g") else torch.float32) for n, a in x.items()}
    # both caches start from the oracle prefill's biases, so the steps are checked on their own
    # (the prefill's b_final is checked elsewhere)
    ob = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, row_mask=np.zeros(T0, np.uint8))["b_final"]
    cap = T0 + steps + 1
    cache = ua.Cache.empty(w.B, w.Hkv, w.d, cap, bf)
    ua.cache_fill(cache, dd["k"], dd["v"], dd["a_k"], dev(ob, torch.float32), theta=w.theta)
    ws = ua.alloc_workspace(ua.decode_workspace_size(cache, w.H), "cuda")
    oc = oracle.DecodeCache(w.B, w.Hkv, w.d, cap)
    oc.fill_from_prefill(x["k"], x["v"], x["a_k"], ob)
    logp = math.log(p) if p > 0 else -math.inf
    words = (cap + 31) // 32
    alpha, beta = dd["alpha"].cpu().numpy(), dd["beta"].cpu().numpy()
    ua.profile_reset()
    ua.profile_enable(True)
    n_evicted = n_adopted = 0
    try:
        for s in range(steps):
            tok = I.make_decode_token(w, s)
            if q_against_key:
                # every query head pointed away from its new key with norm q_against_key: the new
                # token's own logit (where the softmax shift starts) is then ~ -scale*norm while
                # keys at other positions reach well above it
                G = w.H // w.Hkv
                kk = tok["k"].astype(np.float64)
                kdir = kk / np.linalg.norm(kk, axis=-1, keepdims=True)
                q = -q_against_key * np.repeat(kdir, G, axis=1) + 0.3 * tok["q"].astype(np.float64)
                tok["q"] = I.round_bf16(q).astype(np.float32)
            t = {n: dev(a, bf if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
            n_before = cache.n_kept.cpu().numpy()
            ev = torch.full((w.B, w.Hkv, words), -1, dtype=torch.int32, device="cuda")
            kept = torch.full((w.B, w.Hkv, cap), -7, dtype=torch.int32, device="cuda")
            o = ua.decode_step(cache, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], dd["alpha"], dd["beta"],
                               T0 + s, p, scale=w.scale, theta=w.theta, evict_bits=ev, kept_idx=kept, ws=ws)
            torch.cuda.synchronize()
            assert ua.get_device_status() == 0
            ev = ev.cpu().numpy().view(np.uint32)
            kept = kept.cpu().numpy()
            gpu_ev = np.zeros((w.B, w.Hkv, cap), bool)
            for b in range(w.B):
                for h in range(w.Hkv):
                    m = n_before[b, h]
                    gpu_ev[b, h, :m] = unpack_bits(ev[b, h], m)
                    assert not unpack_bits(ev[b, h], words * 32)[m:].any(), "eviction bits past the live pairs"
                    np.testing.assert_array_equal(kept[b, h, :m], np.arange(m))
                    assert kept[b, h, m] == -1
            ro = oracle.decode_step(oc, tok["q"], tok["k"], tok["v"], tok["g"], tok["a_q"], tok["a_k"], alpha,
                                    beta, T0 + s, p, scale=w.scale, theta=w.theta, band=EVICT_BAND,
                                    adopt_keep=(~gpu_ev).astype(np.uint8), defer=True)
            inb = ro["in_band"].astype(bool)
            mism = (ro["evict"].astype(bool) != gpu_ev) & ~inb
            assert not mism.any(), f"step {s}: eviction differs outside the band at {np.argwhere(mism)[:5]}"
            n_adopted += int(inb.sum())
            n_evicted += int(gpu_ev.sum())
            np.testing.assert_array_equal(cache.n_kept.cpu().numpy(), n_before + 1)
            np.testing.assert_array_equal(oc.n, n_before + 1)
            assert_close(f"o step {s}", o.float().cpu().numpy(), ro["o"], "bf16")
            gb = cache.bias.cpu().numpy()
            for b in range(w.B):
                for h in range(w.Hkv):
                    m = n_before[b, h] + 1
                    live = oc.b[b, h, :m] >= logp
                    assert_close(f"bias step {s}", gb[b, h, :m][live], oc.b[b, h, :m][live], "bf16",
                                 relative_max=True)
                    np.testing.assert_array_equal(cache.pos[b, h, :m].cpu().numpy(), oc.pos[b, h, :m])
    finally:
        ua.profile_enable(False)
    names = set(ua.profile_read())
    assert "k_decode_tc" in names, names
    if p > 0:
        assert n_evicted > 0
        kept = torch.full((w.B, w.Hkv, cap), -7, dtype=torch.int32, device="cuda")
        ua.cache_compact(cache, p, kept_idx=kept)
        oc.compact(p)
        np.testing.assert_array_equal(cache.n_kept.cpu().numpy(), oc.n)
        for b in range(w.B):
            for h in range(w.Hkv):
                m = oc.n[b, h]
                np.testing.assert_array_equal(cache.pos[b, h, :m].cpu().numpy(), oc.pos[b, h, :m])
    return n_evicted, n_adopted


@pytest.mark.parametrize("d,H,Hkv,T0,p", [(64, 8, 2, 2600, 0.15), (64, 4, 2, 3001, 0.15), (128, 6, 2, 4095, 0.15),
                                          (64, 8, 1, 2500, 0.0), (64, 16, 2, 2700, 0.15), (128, 2, 2, 2222, 0.0),
                                          (64, 3, 3, 130, 0.15)])
def test_tensor_core_split_decode_lockstep(d, H, Hkv, T0, p):
    w = I.Workload("dec_tc", 2, T0, H, Hkv, d, "bf16", 6100 + T0 + H, bimodal_ak=True)
    run_lockstep(w, T0, 12, p)


def test_tensor_core_split_decode_shift_rescale():
    """Queries anti-aligned with their new key (norm 110, scale*||q|| ~ 14): the own logit, where
    each head's softmax shift starts, sits ~14 below zero while keys elsewhere in the cache reach
    ~+6, beyond the shift's 16-nat headroom, so the shift is raised and the accumulated values
    rescaled in TMEM.  (Larger norms are not used: the bf16 keys put an error of about
    2^-9 * scale*||q|| / sqrt(d) on every logit, so the bf16 bar on o holds up to scale*||q|| of
    about 20; all queries at ~60 measured 6.5e-3.)"""
    w = I.Workload("dec_tc_qn", 1, 2600, 8, 2, 64, "bf16", 6177, bimodal_ak=True)
    run_lockstep(w, 2600, 6, 0.15, q_against_key=110.0)


def _stale_pair(w, T0, fill_nan):
    """A cache filled from a T0-token prefill whose slots past the live pairs hold zeros, or NaN
    keys, values, biases and rates and arbitrary positions."""
    bf = torch.bfloat16
    x = I.make_prefill_inputs(w, T=T0, names=["q", "k", "v", "g", "a_q", "a_k", "alpha", "beta"])
    ob = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, row_mask=np.zeros(T0, np.uint8))["b_final"]
    cap = T0 + 200
    cache = ua.Cache.empty(w.B, w.Hkv, w.d, cap, bf)
    ua.cache_fill(cache, dev(x["k"], bf), dev(x["v"], bf), dev(x["a_k"], torch.float32), dev(ob, torch.float32),
                  theta=w.theta)
    if fill_nan:
        cache.khat[:, :, T0:] = float("nan")
        cache.v[:, :, T0:] = float("nan")
        cache.bias[:, :, T0:] = float("nan")
        cache.rk[:, :, T0:] = float("nan")
        cache.pos[:, :, T0:] = 123456789
    return cache, x


@pytest.mark.parametrize("split", [False, True])
def test_slots_past_the_live_pairs_are_never_read_into_results(split):
    """A ragged cache (300 live pairs: two full 128-entry tiles and 44 more) whose slots past the
    live pairs hold NaN gives bit-identical steps to the same cache with zeros there: those slots'
    values enter the tensor-core product only with zero probabilities, and the kernels zero them
    first (0 x NaN would be NaN)."""
    w = I.Workload("dec_stale", 2, 300, 8, 2, 64, "bf16", 6400, bimodal_ak=True)
    outs = []
    for fill_nan in (False, True):
        cache, x = _stale_pair(w, 300, fill_nan)
        ws = ua.alloc_workspace(ua.decode_workspace_size(cache, w.H), "cuda") if split else None
        bf = torch.bfloat16
        res = []
        for s in range(3):
            tok = I.make_decode_token(w, s)
            t = {n: dev(a, bf if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
            o = ua.decode_step(cache, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], dev(x["alpha"], torch.float32),
                               dev(x["beta"], torch.float32), 300 + s, 0.15, scale=w.scale, theta=w.theta, ws=ws)
            torch.cuda.synchronize()
            assert ua.get_device_status() == 0
            res.append(o.float().cpu().numpy())
        n = cache.n_kept.cpu().numpy()
        live = [cache.bias[b, h, :n[b, h]].cpu().numpy() for b in range(w.B) for h in range(w.Hkv)]
        outs.append((res, n, live))
    (r0, n0, l0), (r1, n1, l1) = outs
    assert all(np.isfinite(a).all() for a in r1)
    for a, b in zip(r0, r1):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(n0, n1)
    for a, b in zip(l0, l1):
        np.testing.assert_array_equal(a, b)


def test_split_step_reports_a_workspace_that_was_not_zeroed():
    """The split step's per-cache arrival counters must start at zero (ua.alloc_workspace zeroes
    them and every step leaves them zero).  Counters found at or past the grid's size raise
    UA_ERR_INVALID_ARG in the device status (and no CTA merges); zeroed again, the workspace
    works."""
    w = I.Workload("dec_ws", 1, 700, 4, 2, 64, "bf16", 6500)
    cache, x = _stale_pair(w, 700, False)
    ws = ua.alloc_workspace(ua.decode_workspace_size(cache, w.H), "cuda")
    bf = torch.bfloat16
    tok = I.make_decode_token(w, 0)
    t = {n: dev(a, bf if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
    args = (t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], dev(x["alpha"], torch.float32),
            dev(x["beta"], torch.float32))
    ua.get_device_status()
    ws[: 4 * w.B * w.Hkv] = 0xFF
    ua.decode_step(cache, *args, 700, 0.15, scale=w.scale, theta=w.theta, ws=ws)
    assert ua.get_device_status() == 1                    # UA_ERR_INVALID_ARG
    np.testing.assert_array_equal(cache.n_kept.cpu().numpy(), 700)   # no merge appended the token
    ws.zero_()
    ua.decode_step(cache, *args, 700, 0.15, scale=w.scale, theta=w.theta, ws=ws)
    assert ua.get_device_status() == 0
    np.testing.assert_array_equal(cache.n_kept.cpu().numpy(), 701)
    assert int(ws[: 4 * w.B * w.Hkv].view(torch.int32).abs().sum().item()) == 0
