"""GPU parity of the tensor-core backward (bf16, head_dim 64 and 128, 1-4 query heads per KV
head at d=64, 1-3 at d=128) against the analytic fp64 oracle, through the C ABI.

The backward cuts rows into 32-row steps and keys into 128-key tiles; the shapes span a single
token, ragged tails, several key tiles and every group size, and the query-norm variant.  The
kernels that ran are checked too: the fp32 SIMT backward must not be the one that answered."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_grad_close, sum_model_rms

pytestmark = pytest.mark.gpu
GRADS = ("dq", "dk", "dv", "dg", "da_q", "da_k", "dalpha", "dbeta")


def dev(x):
    return {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
        torch.bfloat16 if n in ("q", "k", "v", "g", "d_o") else torch.float32).contiguous() for n, a in x.items()}


def run(w, x, variant=0, ws=None):
    d = dev(x)
    f = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta, variant=variant)
    ua.profile_reset()
    ua.profile_enable(True)
    try:
        gr = ua.prefill_bwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"], f["o"],
                            f["lse"], f["b_final"], d["d_o"], scale=w.scale, theta=w.theta, variant=variant, ws=ws)
        torch.cuda.synchronize()
    finally:
        ua.profile_enable(False)
    names = set(ua.profile_read())
    assert ua.get_device_status() == 0
    return gr, names


SHAPES = [
    # (B, T, H, Hkv, d)
    (1, 1, 4, 1, 64),
    (2, 63, 4, 2, 64),
    (1, 129, 8, 2, 64),
    (1, 300, 6, 2, 64),
    (2, 200, 4, 4, 64),
    (1, 600, 2, 1, 64),
    (1, 257, 6, 2, 128),
    (2, 130, 4, 2, 128),
    (1, 400, 3, 1, 128),
    (1, 1000, 3, 1, 128),
]


@pytest.mark.parametrize("B,T,H,Hkv,d", SHAPES)
def test_tensor_core_backward_matches_analytic_oracle(B, T, H, Hkv, d):
    w = I.Workload("bwdtc", B, T, H, Hkv, d, "bf16", 2300 + T + H + d, with_grad=True)
    x = I.make_prefill_inputs(w)
    gr, names = run(w, x)
    assert "k_bwd_key_tc" in names and "k_bwd_keys" not in names, names
    g = {k: v.float().cpu().numpy() for k, v in gr.items()}
    r = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta)
    rms = sum_model_rms(oracle.prefill_bwd, r, **x, scale=w.scale, theta=w.theta)
    for n in GRADS:
        assert np.all(np.isfinite(g[n])), n
        assert_grad_close(n, g[n], r[n], "bf16", rms)


@pytest.mark.parametrize("d", [64, 128])
def test_tensor_core_backward_with_query_norm(d):
    w = I.Workload("bwdqn", 1, 211, 6, 2, d, "bf16", 2400 + d, with_grad=True)
    x = I.make_prefill_inputs(w)
    x["q"] = x["q"] * 2.0
    gr, names = run(w, x, variant=ua.VAR_QUERY_NORM)
    assert "k_bwd_key_tc" in names, names
    g = {k: v.float().cpu().numpy() for k, v in gr.items()}
    r = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta, variant=ua.VAR_QUERY_NORM)
    rms = sum_model_rms(oracle.prefill_bwd, r, **x, scale=w.scale, theta=w.theta, variant=ua.VAR_QUERY_NORM)
    for n in GRADS:
        assert_grad_close(n, g[n], r[n], "bf16", rms)


def test_tensor_core_backward_is_deterministic():
    w = I.Workload("bwddet", 2, 333, 8, 2, 64, "bf16", 2500, with_grad=True)
    x = I.make_prefill_inputs(w)
    a, _ = run(w, x)
    b, _ = run(w, x)
    for n in GRADS:
        assert torch.equal(a[n], b[n]), n


def test_d128_four_heads_per_kv_head_runs_simt_and_matches():
    """d=128 with 4 query heads per KV head does not fit the key-side kernel's shared memory
    (four dZ/dX step tiles beside the key tile); it runs on the fp32 SIMT backward."""
    w = I.Workload("bwdg4", 1, 150, 4, 1, 128, "bf16", 2600, with_grad=True)
    x = I.make_prefill_inputs(w)
    shape = ua.make_shape(torch.empty(1, 150, 4, 128, dtype=torch.bfloat16),
                          torch.empty(1, 150, 1, 128, dtype=torch.bfloat16), w.scale, w.theta, 0)
    ws = ua.alloc_workspace(ua.prefill_bwd_workspace_size(shape), "cuda")
    gr, names = run(w, x, ws=ws)
    assert "k_bwd_key_tc" not in names and "k_bwd_keys" in names, names
    steps, walked = ua.prefill_bwd_band_stats(shape, ws)
    assert walked == steps == 8 + 4, (steps, walked)   # key tile 0: steps 0..7, key tile 1: steps 4..7
    g = {k: v.float().cpu().numpy() for k, v in gr.items()}
    r = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta)
    rms = sum_model_rms(oracle.prefill_bwd, r, **x, scale=w.scale, theta=w.theta)
    for n in GRADS:
        assert_grad_close(n, g[n], r[n], "bf16", rms)


@pytest.mark.parametrize("T,H,Hkv,d,variant", [(1500, 4, 2, 64, 0), (1200, 3, 1, 128, 0),
                                               (1500, 4, 2, 64, ua.VAR_QUERY_NORM)])
def test_tensor_core_backward_with_underflowing_band(T, H, Hkv, d, variant):
    """Strong decay rates: some hundred rows below a key every probability underflows to exactly 0,
    so the key-major pass walks each key tile only down to its last step with a possibly nonzero
    probability and the GEMMs skip the band below it.  That band contributes exact zeros, so the
    gradients must still match the oracle (with the query norm too: the bound uses the normalised
    queries)."""
    w = I.Workload("bwduf", 1, T, H, Hkv, d, "bf16", 2700 + T + d, with_grad=True)
    x = I.make_prefill_inputs(w)
    x["a_q"] = x["a_q"] + 4.0
    x["a_k"] = x["a_k"] + 4.0
    # the inputs do put the band past the threshold (exp(-88 nats) and the logits' bound of a few
    # nats): Lambda(i, j) for i - j >= 256
    k = x["k"][0, :, 0].astype(np.float64)
    kh = k / np.linalg.norm(k, axis=1, keepdims=True)
    sp = lambda z: np.logaddexp(0.0, z)
    X = x["alpha"][0] * (kh @ kh.T) + x["beta"][0]
    D = np.exp(np.log(sp(x["a_q"][0, :, 0]))[:, None] / 3 + np.log(sp(x["a_k"][0, :, 0]))[None, :] / 3
               + np.log(sp(X)) / 3)
    lam = -np.cumsum(np.tril(D, -1), axis=0)
    far = np.tril(np.ones((T, T), bool), -256)
    assert np.mean(lam[far] < -120.0) > 0.99
    shape = ua.make_shape(torch.empty(1, T, H, d, dtype=torch.bfloat16), torch.empty(1, T, Hkv, d, dtype=torch.bfloat16),
                          w.scale, w.theta, variant)
    ws = ua.alloc_workspace(ua.prefill_bwd_workspace_size(shape), "cuda")
    gr, names = run(w, x, variant=variant, ws=ws)
    assert "k_bwd_key_tc" in names, names
    # the key-major pass stopped early in most key tiles (steps of 32 rows: the band below a
    # few hundred rows underflows)
    steps, walked = ua.prefill_bwd_band_stats(shape, ws)
    nkt = (T + 127) // 128
    assert steps == Hkv * (nkt * 4 * nkt - 2 * nkt * (nkt - 1))
    assert walked < steps // 2, (walked, steps)
    g = {k: v.float().cpu().numpy() for k, v in gr.items()}
    r = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta, variant=variant)
    rms = sum_model_rms(oracle.prefill_bwd, r, **x, scale=w.scale, theta=w.theta, variant=variant)
    for n in GRADS:
        assert np.all(np.isfinite(g[n])), n
        assert_grad_close(n, g[n], r[n], "bf16", rms)
