"""GPU parity of ua_prefill_bwd: against the analytic fp64 oracle on small shapes and on a
1024-token prefix of the 3B workload, and against fp64 central finite differences of the
oracle forward on its 128-token slice (alpha and beta in full; every other tensor through
directional derivatives and sampled coordinates)."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_close, assert_grad_close, sum_model_rms

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}
GRADS = ("dq", "dk", "dv", "dg", "da_q", "da_k", "dalpha", "dbeta")
INPUTS = ("q", "k", "v", "g", "a_q", "a_k", "alpha", "beta")


def gpu_grads(w, x):
    dt = TORCH_DT[w.dtype]
    d = {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt if n in ("q", "k", "v", "g", "d_o") else
                                                                  torch.float32).contiguous() for n, a in x.items()}
    f = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta)
    gr = ua.prefill_bwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"], f["o"], f["lse"],
                        f["b_final"], d["d_o"], scale=w.scale, theta=w.theta)
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    return {k: v.float().cpu().numpy() for k, v in gr.items()}


def check_all(g, r, dtype, x, w):
    rms = sum_model_rms(oracle.prefill_bwd, r, **x, scale=w.scale, theta=w.theta) if dtype == "bf16" else None
    for n in GRADS:
        assert np.all(np.isfinite(g[n])), n
        # every gradient tensor: rel-L2 and max error against the tensor's own scale (sums such
        # as dalpha, dbeta cancel strongly, so a small entry carries the error of the big ones)
        assert_grad_close(n, g[n], r[n], dtype, rms)


SMALL = [
    # (B, T, H, Hkv, d, dtype)
    (1, 70, 4, 2, 64, "f32"),
    (1, 33, 2, 1, 128, "f32"),
    (2, 130, 6, 2, 128, "bf16"),
    (1, 200, 8, 2, 64, "bf16"),
    (2, 97, 4, 4, 64, "bf16"),
]


@pytest.mark.parametrize("B,T,H,Hkv,d,dtype", SMALL)
def test_backward_matches_analytic_oracle(B, T, H, Hkv, d, dtype):
    w = I.Workload("bwd", B, T, H, Hkv, d, dtype, 300 + T, with_grad=True)
    x = I.make_prefill_inputs(w)
    g = gpu_grads(w, x)
    r = oracle.prefill_bwd(**{k: v for k, v in x.items()}, scale=w.scale, theta=w.theta)
    check_all(g, r, dtype, x, w)


def _loss(x, d_o, w):
    r = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta)
    return float(np.sum(r["o"] * d_o))


def test_backward_against_finite_differences_on_3b_slice():
    """3B workload, first 128 tokens of batch 0 (the slice the finite differences run on)."""
    w3 = I.WORKLOADS["fwdbwd_3b"]
    w = w3.resized(B=1, T=128)
    x = I.make_prefill_inputs(w3, T=128, B=1)
    g = gpu_grads(w, x)
    xo = {k: np.asarray(v, np.float64) for k, v in x.items() if k != "d_o"}
    d_o = np.asarray(x["d_o"], np.float64)
    rng = np.random.default_rng(0)
    # alpha and beta: every coordinate (the bar of the per-head sums, with the saved-output
    # model's deviation of the analytic gradients)
    r = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta)
    rms = sum_model_rms(oracle.prefill_bwd, r, **x, scale=w.scale, theta=w.theta)
    for name in ("alpha", "beta"):
        fd = np.zeros(w.Hkv)
        for i in range(w.Hkv):
            h = 1e-6 * max(1.0, abs(xo[name][i]))
            xp = dict(xo); xp[name] = xo[name].copy(); xp[name][i] += h
            xm = dict(xo); xm[name] = xo[name].copy(); xm[name][i] -= h
            fd[i] = (_loss(xp, d_o, w) - _loss(xm, d_o, w)) / (2 * h)
        assert_grad_close("d" + name, g["d" + name], fd, "bf16", rms)
    # every tensor: directional derivative along a random direction, and 4 sampled coordinates
    for name in INPUTS[:6]:
        u = rng.standard_normal(xo[name].shape)
        u /= np.linalg.norm(u)
        h = 1e-6 * max(1.0, float(np.abs(xo[name]).max()))
        xp = dict(xo); xp[name] = xo[name] + h * u
        xm = dict(xo); xm[name] = xo[name] - h * u
        fd = (_loss(xp, d_o, w) - _loss(xm, d_o, w)) / (2 * h)
        an = float(np.sum(g["d" + name].astype(np.float64) * u))
        # |<g_gpu - g, u>| <= ||g_gpu - g|| for a unit u: the rel-L2 bar times ||g||
        assert abs(an - fd) <= 5e-3 * np.linalg.norm(g["d" + name]), (name, an, fd)
        flat = np.argsort(-np.abs(g["d" + name]).ravel())[:2].tolist() + rng.integers(0, u.size, 2).tolist()
        for f_idx in flat:
            idx = np.unravel_index(f_idx, u.shape)
            hh = 1e-6 * max(1.0, abs(xo[name][idx]))
            xp = dict(xo); xp[name] = xo[name].copy(); xp[name][idx] += hh
            xm = dict(xo); xm[name] = xo[name].copy(); xm[name][idx] -= hh
            fdc = (_loss(xp, d_o, w) - _loss(xm, d_o, w)) / (2 * hh)
            # a coordinate far below the tensor's largest carries the accumulation error of the
            # large terms: the floor is 5% of the largest, i.e. an absolute bar of 1e-3 of it (20x
            # tighter than the tensor-scale max-error bar)
            scale_ref = max(abs(fdc), 5e-2 * float(np.abs(g["d" + name]).max()))
            assert abs(g["d" + name][idx] - fdc) <= 2e-2 * scale_ref, (name, idx, g["d" + name][idx], fdc)


@pytest.mark.slow
def test_backward_3b_prefix_1024_matches_oracle():
    w3 = I.WORKLOADS["fwdbwd_3b"]
    w = w3.resized(B=1, T=1024)
    x = I.make_prefill_inputs(w3, T=1024, B=1)
    g = gpu_grads(w, x)
    r = oracle.prefill_bwd(**x, scale=w.scale, theta=w.theta)
    check_all(g, r, "bf16", x, w)


@pytest.mark.slow
def test_backward_3b_full_size_runs_finite():
    """Full 3B workload (B=4, T=8192): the backward completes with finite gradients and the
    value-gradient row sums obey sum_j dv_j = sum_i dA_i (softmax rows sum to 1)."""
    w = I.WORKLOADS["fwdbwd_3b"]
    x = I.make_prefill_inputs_torch(w, "cuda")
    f = ua.prefill_fwd(x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"],
                       scale=w.scale, theta=w.theta)
    gr = ua.prefill_bwd(x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"], f["o"],
                        f["lse"], f["b_final"], x["d_o"], scale=w.scale, theta=w.theta)
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    for n, t in gr.items():
        assert torch.isfinite(t.float()).all(), n
    # sum over keys of dv_j = sum over rows i and the group's heads of dA_i
    dA = (x["d_o"].float() * torch.sigmoid(x["g"].float()))                 # [B,T,H,d]
    G = w.H // w.Hkv
    lhs = gr["dv"].float().sum(dim=1)                                       # [B,Hkv,d]
    rhs = dA.view(w.B, w.T, w.Hkv, G, w.d).sum(dim=(1, 3))
    rel = (lhs - rhs).norm() / rhs.norm()
    assert rel < 1e-2, float(rel)
