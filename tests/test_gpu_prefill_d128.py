"""GPU parity of the head_dim-128 tensor-core forward (the 3B-shaped layer) against the fp64
oracle, through the C ABI.

The kernel cuts 64-row query tiles against 128-key tiles, accumulates O transposed (head dims on
the TMEM lanes) and the row sums of all heads in one accumulator; the shapes below span several
query and key tiles, ragged tails, every group size it takes (1-4), underflow tile skipping, and
heads of very unequal query norm (one shared softmax shift per 16-row quarter)."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_close

pytestmark = pytest.mark.gpu


def to_dev(x):
    return {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
        torch.bfloat16 if n in ("q", "k", "v", "g", "d_o") else torch.float32).contiguous() for n, a in x.items()}


def kernels_ran(fn):
    ua.profile_reset()
    ua.profile_enable(True)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        ua.profile_enable(False)
    return out, set(ua.profile_read())


def run(w, x, want_bfinal=True, ws=None):
    d = to_dev({k: v for k, v in x.items() if k != "d_o"})
    r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta, want_bfinal=want_bfinal, ws=ws)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.float().cpu().numpy()) for k, v in r.items()}


def ora(w, x, **kw):
    return oracle.prefill_fwd(**{k: v for k, v in x.items() if k != "d_o"}, scale=w.scale, theta=w.theta, **kw)


SHAPES = [
    # (B, T, H, Hkv): bf16, d = 128
    (1, 1, 3, 1),
    (2, 63, 6, 2),
    (1, 64, 3, 1),
    (1, 65, 2, 1),
    (2, 129, 6, 2),
    (1, 200, 2, 2),
    (1, 333, 4, 1),
    (2, 517, 8, 2),
    (1, 1000, 3, 1),
]


@pytest.mark.parametrize("B,T,H,Hkv", SHAPES)
def test_d128_tensor_core_full_parity(B, T, H, Hkv):
    w = I.Workload("tc128", B, T, H, Hkv, 128, "bf16", 1700 + T + H)
    x = I.make_prefill_inputs(w)
    g, names = kernels_ran(lambda: run(w, x))
    assert "k_fwd_tc128" in names and "k_fwd_simt" not in names and "k_boundary_simt" not in names, names
    assert ua.get_device_status() == 0
    r = ora(w, x)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)
    assert_close("b_final", g["b_final"], r["b_final"], "bf16", relative_max=True)
    # without b_final (tiles whose probabilities all underflow are then not decayed either)
    g2 = run(w, x, want_bfinal=False)
    assert ua.get_device_status() == 0
    assert_close("o (no b_final)", g2["o"], r["o"], "bf16")
    assert_close("lse (no b_final)", g2["lse"], r["lse"], "bf16", relative_max=True)


@pytest.mark.parametrize("B,T,H,Hkv,shift", [(1, 1000, 3, 1, 4.0), (2, 700, 6, 2, 3.0)])
def test_d128_underflow_tile_skipping_is_exact(B, T, H, Hkv, shift):
    w = I.Workload("skip128", B, T, H, Hkv, 128, "bf16", 1800 + T)
    x = I.make_prefill_inputs(w)
    x["a_q"] = x["a_q"] + shift
    x["a_k"] = x["a_k"] + shift
    d = to_dev({k: v for k, v in x.items() if k != "d_o"})
    shape = ua.make_shape(d["q"], d["k"], w.scale, w.theta)
    ws = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
    r1 = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                        scale=w.scale, theta=w.theta, ws=ws)
    tiles, skipped = ua.prefill_tile_stats(shape, ws)
    assert ua.get_device_status() == 0
    nq = (T + 63) // 64
    assert tiles == B * Hkv * sum(t // 2 + 1 for t in range(nq))
    assert skipped >= max(1, (tiles - B * Hkv * nq) // 8), (skipped, tiles)
    g = {k: v.float().cpu().numpy() for k, v in r1.items() if v is not None}
    r = ora(w, x)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)
    assert_close("b_final", g["b_final"], r["b_final"], "bf16", relative_max=True)
    r2 = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                        scale=w.scale, theta=w.theta, ws=ws, want_bfinal=False)
    _, skipped2 = ua.prefill_tile_stats(shape, ws)
    assert ua.get_device_status() == 0
    assert skipped2 == skipped
    assert torch.equal(r2["o"], r1["o"]) and torch.equal(r2["lse"], r1["lse"])


def test_d128_shared_shift_with_unequal_head_norms():
    w = I.Workload("shift128", 1, 600, 3, 1, 128, "bf16", 78)
    x = I.make_prefill_inputs(w)
    q = x["q"].astype(np.float64)
    q[:, :, 0] *= 5.0
    q[:, :, 2] *= 0.25
    q[:, ::7, :] *= 1e-3
    x["q"] = I.round_bf16(q).astype(np.float32)
    g, names = kernels_ran(lambda: run(w, x))
    assert "k_fwd_tc128" in names
    assert ua.get_device_status() == 0
    r = ora(w, x)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)


def test_d128_veto_gives_plain_attention_and_zero_bias():
    w = I.Workload("veto128", 2, 300, 6, 2, 128, "bf16", 19)
    x = I.make_prefill_inputs(w)
    x["a_k"][:] = -1e4
    g, names = kernels_ran(lambda: run(w, x))
    assert "k_fwd_tc128" in names
    assert np.all(g["b_final"] == 0.0)
    r = ora(w, x)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)


def test_d128_query_norm_stays_on_tensor_cores():
    w = I.Workload("qn128", 1, 400, 6, 2, 128, "bf16", 23)
    x = I.make_prefill_inputs(w)
    x["q"] = x["q"] * 3.0
    d = to_dev({k: v for k, v in x.items() if k != "d_o"})
    (r_gpu, names) = kernels_ran(lambda: ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"],
                                                          d["alpha"], d["beta"], scale=w.scale, theta=w.theta,
                                                          variant=ua.VAR_QUERY_NORM))
    assert "k_fwd_tc128" in names, names
    assert ua.get_device_status() == 0
    r = ora(w, x, variant=ua.VAR_QUERY_NORM)
    assert_close("o", r_gpu["o"].float().cpu().numpy(), r["o"], "bf16")


@pytest.mark.slow
def test_fwdbwd_3b_forward_full_size_sampled():
    """The 3B workload's forward at full size (B=4, T=8192): sampled (batch, KV head) units and
    rows against the oracle, b_final of those units in full."""
    w = I.WORKLOADS["fwdbwd_3b"]
    x = {k: v for k, v in I.make_prefill_inputs(w).items() if k != "d_o"}
    g, names = kernels_ran(lambda: run(w, x))
    assert "k_fwd_tc128" in names
    assert ua.get_device_status() == 0
    rng = np.random.default_rng(5)
    rows = sorted({0, 1, 63, 64, 127, 128, 4095, 4096, w.T - 65, w.T - 64, w.T - 1}
                  | set(int(a) for a in rng.integers(0, w.T, 20)))
    rm = np.zeros(w.T, np.uint8)
    rm[rows] = 1
    units = [(0, 0), (3, 7)]
    um = np.zeros(w.B * w.Hkv, np.uint8)
    for b, h in units:
        um[b * w.Hkv + h] = 1
    r = ora(w, x, unit_mask=um, row_mask=rm)
    G = w.G
    for b, h in units:
        hs = slice(h * G, (h + 1) * G)
        assert_close(f"o[{b},{h}]", g["o"][b][rows][:, hs], r["o"][b][rows][:, hs], "bf16")
        assert_close(f"lse[{b},{h}]", g["lse"][b, hs][:, rows], r["lse"][b, hs][:, rows], "bf16",
                     relative_max=True)
        assert_close(f"b_final[{b},{h}]", g["b_final"][b, h], r["b_final"][b, h], "bf16", relative_max=True)
    assert np.all(np.isfinite(g["o"]))
