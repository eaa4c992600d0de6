"""Pins of the oracle's chunked pruned prefill against facts that do not come from the oracle.

"A Self-Pruning Transformer: Extreme KV-Cache Compression with Universal Attention"
(paperlayer.ai summary, §5) prunes the prefill in chunks of 128 tokens.  Reading: before the
chunk starting at row c, pairs j < c with Lambda_{c-1,j} < log p are evicted for good; rows of
the chunk attend over the survivors and their own chunk with the usual biases.

* p = 0 is the dense prefill, bit for bit; the first chunk and b_final never change;
* p = 1 (log p = 0) has a closed-form visible set: every earlier pair has a strictly negative
  bias except the last key before the chunk (Lambda_{c-1,c-1} = 0), so a row of chunk c sees its
  own chunk and key c-1 only; checked against torch's scaled_dot_product_attention with that
  mask, the brute-force Lambda as bias and an independently written RoPE;
* for a general p the output equals SDPA with the mask built from the brute-force Lambda at
  the chunk boundaries.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I


def case(T=300, B=1, H=4, Hkv=2, d=16, seed=31):
    w = I.Workload("prune", B, T, H, Hkv, d, "f32", seed)
    return w, {k: v.astype(np.float64) for k, v in I.make_prefill_inputs(w).items() if k != "d_o"}


def rope_t(x, theta):
    """[B,T,h,d] -> RoPE as complex multiplication of (x_m, x_{m+d/2})."""
    B, T, h, d = x.shape
    half = d // 2
    z = torch.complex(x[..., :half], x[..., half:])
    freq = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * freq[None, :]
    z = z * torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def sdpa_reference(w, x, visible, lam):
    """softmax(scale qrot.krot + Lambda, masked by visible[b, kvh, i, j]) V, gated."""
    q = torch.from_numpy(x["q"])
    k = torch.from_numpy(x["k"])
    khat = k / torch.clamp(k.norm(dim=-1, keepdim=True), min=1e-12)
    qr = rope_t(q, w.theta).permute(0, 2, 1, 3)                       # [B,H,T,d]
    kr = rope_t(khat, w.theta).permute(0, 2, 1, 3)                    # [B,Hkv,T,d]
    v = torch.from_numpy(x["v"]).permute(0, 2, 1, 3)
    G = w.H // w.Hkv
    kr = kr.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    bias = torch.from_numpy(np.where(visible, lam, -np.inf)).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qr, kr, v, attn_mask=bias, scale=w.scale)
    o = o.permute(0, 2, 1, 3).numpy()
    return o / (1.0 + np.exp(-x["g"]))


def causal(T):
    return np.tril(np.ones((T, T), bool))


def test_p0_is_dense_bit_for_bit():
    w, x = case()
    a = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta)
    b = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, prune_p=0.0)
    for n in ("o", "lse", "b_final"):
        np.testing.assert_array_equal(a[n], b[n])


def test_first_chunk_and_bfinal_unchanged():
    w, x = case()
    a = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta)
    b = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, prune_p=0.15)
    np.testing.assert_array_equal(a["o"][:, :128], b["o"][:, :128])
    np.testing.assert_array_equal(a["b_final"], b["b_final"])
    assert np.max(np.abs(a["o"][:, 128:] - b["o"][:, 128:])) > 1e-3   # later chunks do change


def test_p1_closed_form_visible_set():
    w, x = case(T=300)
    T = w.T
    lam = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    cs = (i // 128) * 128
    visible = causal(T) & ((j >= cs) | (j == cs - 1))
    r = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, prune_p=1.0)
    ref = sdpa_reference(w, x, np.broadcast_to(visible, lam.shape), lam)
    np.testing.assert_allclose(r["o"], ref, atol=1e-12, rtol=1e-10)


@pytest.mark.parametrize("p", [0.05, 0.15, 0.5])
def test_general_p_matches_masked_sdpa(p):
    w, x = case(T=420, B=2, seed=37)
    T = w.T
    lam = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"])   # [B,Hkv,T,T]
    visible = np.broadcast_to(causal(T), lam.shape).copy()
    for c in range(128, T, 128):
        evicted = lam[:, :, c - 1, :c] < math.log(p)                 # [B,Hkv,c]
        visible[:, :, c:c + 128, :c] &= ~evicted[:, :, None, :]
    assert (~visible & causal(T)).any()                               # something was evicted
    r = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, prune_p=p)
    ref = sdpa_reference(w, x, visible, lam)
    np.testing.assert_allclose(r["o"], ref, atol=1e-12, rtol=1e-10)


def test_invalid_threshold_rejected():
    w, x = case(T=16)
    with pytest.raises(ValueError):
        oracle.prefill_fwd(**x, prune_p=1.5)
