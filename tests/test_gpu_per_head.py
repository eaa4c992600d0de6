"""GPU parity of per-query-head decay (UA_VAR_PER_HEAD_DECAY) against the oracle's per-head
forward and backward, through the C ABI.

Every query head gets its own decay logits and similarity parameters (a_q, a_k [B,T,H];
alpha, beta [H]); the library runs the per-KV-head path with one decay unit per query head on
keys and values repeated for each group, and sums dk, dv over the copies.  Checked on the bf16
tensor-core paths (head_dim 64 and 128) and the fp32 SIMT path."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_close, assert_grad_close, sum_model_rms

pytestmark = pytest.mark.gpu
PH = ua.VAR_PER_HEAD_DECAY


def per_head_inputs(w, seed):
    """Rates per query head: each KV head's repeated over its group and perturbed (seeded), then
    rounded like every other input."""
    x = I.make_prefill_inputs(w)
    G = w.H // w.Hkv
    rng = np.random.default_rng(seed)
    for n in ("a_q", "a_k"):
        x[n] = (np.repeat(x[n], G, axis=2) + 0.5 * rng.standard_normal((w.B, w.T, w.H))).astype(np.float32)
    for n in ("alpha", "beta"):
        x[n] = (np.repeat(x[n], G) + 0.5 * rng.standard_normal(w.H)).astype(np.float32)
    return x


def dev(x, dtype):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
        dt if n in ("q", "k", "v", "g", "d_o") else torch.float32).contiguous() for n, a in x.items()}


def kernels_ran(fn):
    ua.profile_reset()
    ua.profile_enable(True)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        ua.profile_enable(False)
    return out, set(ua.profile_read())


CASES = [
    # (B, T, H, Hkv, d, dtype, forward kernel)
    (2, 200, 4, 2, 64, "bf16", "k_fwd_tc"),
    (1, 300, 6, 2, 128, "bf16", "k_fwd_tc128"),
    (1, 150, 4, 1, 64, "f32", "k_fwd_simt"),
]


@pytest.mark.parametrize("B,T,H,Hkv,d,dtype,kernel", CASES)
def test_per_head_forward_matches_oracle(B, T, H, Hkv, d, dtype, kernel):
    w = I.Workload("ph", B, T, H, Hkv, d, dtype, 2600 + T)
    x = per_head_inputs(w, 2600 + T)
    dd = dev(x, dtype)
    r_gpu, names = kernels_ran(lambda: ua.prefill_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["a_q"], dd["a_k"],
                                                        dd["alpha"], dd["beta"], scale=w.scale, theta=w.theta,
                                                        variant=PH))
    assert kernel in names and "k_repeat_kv" in names, names
    assert ua.get_device_status() == 0
    assert r_gpu["b_final"].shape == (B, H, T)
    g = {k: v.float().cpu().numpy() for k, v in r_gpu.items() if v is not None}
    r = oracle.prefill_fwd_per_head(**x, scale=w.scale, theta=w.theta)
    assert_close("o", g["o"], r["o"], dtype)
    assert_close("lse", g["lse"], r["lse"], dtype, relative_max=True)
    assert_close("b_final", g["b_final"], r["b_final"], dtype, relative_max=True)
    # the per-head rates matter: the per-KV-head reading of the same tensors differs
    assert np.max(np.abs(g["b_final"][:, 0] - g["b_final"][:, 1])) > 1e-3


@pytest.mark.parametrize("B,T,H,Hkv,d,dtype,kernel", CASES)
def test_per_head_backward_matches_oracle(B, T, H, Hkv, d, dtype, kernel):
    w = I.Workload("phb", B, T, H, Hkv, d, dtype, 2700 + T, with_grad=True)
    x = per_head_inputs(w, 2700 + T)
    dd = dev(x, dtype)
    f = ua.prefill_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["a_q"], dd["a_k"], dd["alpha"], dd["beta"],
                       scale=w.scale, theta=w.theta, variant=PH)
    gr = ua.prefill_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["a_q"], dd["a_k"], dd["alpha"], dd["beta"], f["o"],
                        f["lse"], f["b_final"], dd["d_o"], scale=w.scale, theta=w.theta, variant=PH)
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    assert gr["da_q"].shape == (B, T, H) and gr["dalpha"].shape == (H,) and gr["dk"].shape == (B, T, Hkv, d)
    g = {k: v.float().cpu().numpy() for k, v in gr.items()}
    r = oracle.prefill_bwd_per_head(**x, scale=w.scale, theta=w.theta)
    rms = sum_model_rms(oracle.prefill_bwd_per_head, r, **x, scale=w.scale, theta=w.theta) if dtype == "bf16" else None
    for n in ("dq", "dk", "dv", "dg", "da_q", "da_k", "dalpha", "dbeta"):
        assert_grad_close(n, g[n], r[n], dtype, rms)


def unpack_bits(words, n):
    bits = np.unpackbits(np.ascontiguousarray(words, np.uint32).view(np.uint8), bitorder="little")
    return bits[:n].astype(bool)


@pytest.mark.parametrize("split", [False, True])
def test_per_head_decode_lockstep(split):
    """Per-query-head decay in decode: a cache of one head per query head (kv_rep = G), filled from
    the prefill's keys and values and stepped with each group's key and value (read by head
    h / G), every head evicting on its own bias; against the oracle's per-head decode in lockstep
    (the eager step with its compaction, and the split step with compaction deferred)."""
    from helpers import EVICT_BAND
    import math
    w = I.Workload("phd", 2, 300, 8, 2, 64, "bf16", 2900 + int(split))
    G = w.H // w.Hkv
    x = per_head_inputs(w, 2900)
    xo = {k: v for k, v in x.items() if k != "d_o"}
    ob = oracle.prefill_fwd_per_head(**xo, scale=w.scale, theta=w.theta, row_mask=np.zeros(w.T, np.uint8))["b_final"]
    p, steps = 0.15, 10
    logp = math.log(p)
    cap = w.T + steps + 1
    dd = dev(xo, "bf16")
    cache = ua.Cache.empty(w.B, w.H, w.d, cap, torch.bfloat16, kv_rep=G)
    ua.cache_fill(cache, dd["k"], dd["v"], dd["a_k"], torch.from_numpy(ob.astype(np.float32)).cuda(), theta=w.theta)
    kept = torch.full((w.B, w.H, cap), -7, dtype=torch.int32, device="cuda")
    ua.cache_compact(cache, p, kept_idx=kept)
    n_g, kept = cache.n_kept.cpu().numpy(), kept.cpu().numpy()
    oc = oracle.DecodeCache(w.B, w.H, w.d, cap)
    gpu_keep = np.zeros((w.B, w.H, w.T), bool)
    for b in range(w.B):
        for h in range(w.H):
            gpu_keep[b, h, kept[b, h, :n_g[b, h]]] = True
    oc.fill_from_prefill(np.repeat(x["k"], G, axis=2), np.repeat(x["v"], G, axis=2), x["a_k"], ob, logp=logp,
                         adopt_keep=gpu_keep)
    np.testing.assert_array_equal(oc.n, n_g)
    ws = ua.alloc_workspace(ua.decode_workspace_size(cache, w.H), "cuda") if split else None
    rng = np.random.default_rng(31)
    words = (cap + 31) // 32
    for s in range(steps):
        tok = I.make_decode_token(w, s)
        for n in ("a_q", "a_k"):
            tok[n] = (np.repeat(tok[n], G, axis=1) + 0.5 * rng.standard_normal((w.B, w.H))).astype(np.float32)
        t = {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
            torch.bfloat16 if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
        n_before = cache.n_kept.cpu().numpy()
        ev = torch.zeros(w.B, w.H, words, dtype=torch.int32, device="cuda")
        o = ua.decode_step(cache, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], dd["alpha"], dd["beta"],
                           w.T + s, p, scale=w.scale, theta=w.theta, evict_bits=ev, variant=PH, ws=ws)
        torch.cuda.synchronize()
        assert ua.get_device_status() == 0
        ev = ev.cpu().numpy().view(np.uint32)
        gev = np.zeros((w.B, w.H, cap), bool)
        for b in range(w.B):
            for h in range(w.H):
                gev[b, h, :n_before[b, h]] = unpack_bits(ev[b, h], n_before[b, h])
        ro = oracle.decode_step_per_head(oc, tok["q"], tok["k"], tok["v"], tok["g"], tok["a_q"], tok["a_k"],
                                         xo["alpha"], xo["beta"], w.T + s, p, scale=w.scale, theta=w.theta,
                                         band=EVICT_BAND, adopt_keep=(~gev).astype(np.uint8), defer=split)
        mism = (ro["evict"].astype(bool) != gev) & ~ro["in_band"].astype(bool)
        assert not mism.any(), f"step {s}: eviction differs outside the band"
        np.testing.assert_array_equal(cache.n_kept.cpu().numpy(), oc.n)
        assert_close(f"o step {s}", o.float().cpu().numpy(), ro["o"], "bf16")
        pos = cache.pos.cpu().numpy()
        for b in range(w.B):
            for h in range(w.H):
                np.testing.assert_array_equal(pos[b, h, :oc.n[b, h]], oc.pos[b, h, :oc.n[b, h]])
    # the heads of a group evict differently (their rates differ)
    n = cache.n_kept.cpu().numpy()
    assert any(len(set(n[b, h * G:(h + 1) * G])) > 1 for b in range(w.B) for h in range(w.Hkv))
