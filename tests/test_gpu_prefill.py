"""GPU parity of ua_prefill_fwd against the fp64 oracle (through the C ABI).

Small cases compare every output element; the full-size workloads compare sampled
(batch, KV-head) units and rows, which the oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import TOL, assert_close

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_dev(x, w):
    out = {}
    for n, a in x.items():
        t = torch.from_numpy(np.ascontiguousarray(a))
        dt = TORCH_DT[w.dtype] if n in ("q", "k", "v", "g", "d_o") else torch.float32
        out[n] = t.to("cuda").to(dt).contiguous()
    return out


def run_gpu(w, x, want_lambda=False):
    d = to_dev({k: v for k, v in x.items() if k != "d_o"}, w)
    r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta, want_lambda=want_lambda)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.float().cpu().numpy()) for k, v in r.items()}


def oracle_inputs(x):
    return {k: v for k, v in x.items() if k != "d_o"}


def test_tiny_fp32_full_parity_and_bruteforce_lambda():
    w = I.WORKLOADS["tiny_fp32"]
    x = I.make_prefill_inputs(w)
    g = run_gpu(w, x, want_lambda=True)
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta, want_lambda=True)
    lb = oracle.lambda_bruteforce(x["k"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    assert_close("o", g["o"], r["o"], "f32")
    assert_close("lse", g["lse"], r["lse"], "f32")
    assert_close("b_final", g["b_final"], r["b_final"], "f32")
    assert_close("lambda vs brute force", g["lam"], lb, "f32")


SMALL = [
    # (B, T, H, Hkv, d, dtype)
    (2, 1, 4, 2, 64, "bf16"),
    (2, 63, 4, 2, 64, "bf16"),
    (2, 65, 4, 1, 64, "bf16"),
    (1, 200, 8, 2, 64, "bf16"),
    (2, 333, 4, 4, 64, "bf16"),
    (1, 300, 6, 2, 128, "bf16"),
    (1, 257, 8, 1, 128, "bf16"),
    (1, 130, 2, 2, 64, "f32"),
    (1, 190, 6, 2, 128, "f32"),
]


@pytest.mark.parametrize("B,T,H,Hkv,d,dtype", SMALL)
def test_small_shapes_full_parity(B, T, H, Hkv, d, dtype):
    w = I.Workload("small", B, T, H, Hkv, d, dtype, 77 + T)
    x = I.make_prefill_inputs(w)
    g = run_gpu(w, x, want_lambda=True)
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta, want_lambda=True)
    assert_close("o", g["o"], r["o"], dtype)
    assert_close("lse", g["lse"], r["lse"], dtype, relative_max=True)
    assert_close("b_final", g["b_final"], r["b_final"], dtype, relative_max=True)
    tri = np.tril(np.ones((T, T), bool))
    assert_close("lambda", g["lam"][..., tri], r["lam"][..., tri], dtype, relative_max=True)
    assert np.all(g["lam"][..., ~tri] == 0.0)


TC_SHAPES = [
    # (B, T, H, Hkv): bf16, d = 64 -> tensor-core path
    (1, 1, 4, 1),
    (2, 63, 4, 2),
    (1, 128, 4, 1),
    (2, 129, 8, 2),
    (1, 200, 2, 2),
    (1, 333, 6, 2),
    (2, 517, 4, 4),
    (1, 1000, 4, 1),
]


def kernels_ran(fn):
    ua.profile_reset()
    ua.profile_enable(True)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        ua.profile_enable(False)
    return out, set(ua.profile_read())


@pytest.mark.parametrize("B,T,H,Hkv", TC_SHAPES)
def test_tensor_core_path_full_parity(B, T, H, Hkv):
    w = I.Workload("tc", B, T, H, Hkv, 64, "bf16", 500 + T + H)
    x = I.make_prefill_inputs(w)
    g, names = kernels_ran(lambda: run_gpu(w, x))
    assert "k_fwd_tc" in names and "k_boundary_tc" not in names, names   # boundary prefixes fused
    assert ua.get_device_status() == 0
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)
    assert_close("b_final", g["b_final"], r["b_final"], "bf16", relative_max=True)


SKIP_SHAPES = [
    # (B, T, H, Hkv, rate shift): strong decay, so most off-diagonal tiles underflow
    (1, 1000, 4, 1, 4.0),
    (2, 700, 8, 2, 3.0),
    (1, 1100, 4, 2, 2.0),
]


@pytest.mark.parametrize("B,T,H,Hkv,shift", SKIP_SHAPES)
def test_tensor_core_underflow_tile_skipping_is_exact(B, T, H, Hkv, shift):
    """Rates shifted up (stronger decay): the tensor-core path skips the softmax of tiles whose
    decay prefix underflows every probability.  Skipping must occur, and every output must
    still match the oracle as the dense computation does (b_final included: the decay of a
    skipped tile is still evaluated)."""
    w = I.Workload("skip", B, T, H, Hkv, 64, "bf16", 700 + T)
    x = I.make_prefill_inputs(w)
    x["a_q"] = x["a_q"] + shift
    x["a_k"] = x["a_k"] + shift
    d = to_dev(oracle_inputs(x), w)
    shape = ua.make_shape(d["q"], d["k"], w.scale, w.theta)
    ws = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
    r_gpu = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                           scale=w.scale, theta=w.theta, ws=ws)
    tiles, skipped = ua.prefill_tile_stats(shape, ws)
    assert ua.get_device_status() == 0
    n = (T + 127) // 128
    assert tiles == B * Hkv * n * (n + 1) // 2
    off_diag = B * Hkv * n * (n - 1) // 2
    assert skipped >= max(1, off_diag // 8), (skipped, off_diag)
    g = {k: v.float().cpu().numpy() for k, v in r_gpu.items() if v is not None}
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)
    assert_close("b_final", g["b_final"], r["b_final"], "bf16", relative_max=True)
    # Without b_final the decay of the skipped tiles is skipped as well; o and lse must be
    # bit-identical to the run above (those tiles contribute exactly zero either way).
    r2 = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                        scale=w.scale, theta=w.theta, ws=ws, want_bfinal=False)
    _, skipped2 = ua.prefill_tile_stats(shape, ws)
    assert ua.get_device_status() == 0
    assert skipped2 == skipped
    assert torch.equal(r2["o"], r_gpu["o"])
    assert torch.equal(r2["lse"], r_gpu["lse"])


def test_tensor_core_shared_shift_with_unequal_head_norms():
    """The tensor-core path shifts every row of a 32-row quarter by the largest a-priori bound
    over those rows and the G heads of the group.  Heads with very different query norms (one
    head 6x, one 0.25x) and rows with tiny norms must still match the oracle."""
    w = I.Workload("shift", 1, 600, 4, 1, 64, "bf16", 77)
    x = I.make_prefill_inputs(w)
    q = x["q"].astype(np.float64)
    q[:, :, 0] *= 6.0
    q[:, :, 2] *= 0.25
    q[:, ::7, :] *= 1e-3                                  # some rows with almost no signal
    x["q"] = I.round_bf16(q).astype(np.float32)
    g, names = kernels_ran(lambda: run_gpu(w, x))
    assert "k_fwd_tc" in names
    assert ua.get_device_status() == 0
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta)
    assert_close("o", g["o"], r["o"], "bf16")
    assert_close("lse", g["lse"], r["lse"], "bf16", relative_max=True)


def test_tensor_core_path_veto_and_plain_attention():
    w = I.Workload("tcveto", 1, 300, 4, 1, 64, "bf16", 17)
    x = I.make_prefill_inputs(w)
    x["a_q"][:] = -1e4
    g, names = kernels_ran(lambda: run_gpu(w, x))
    assert "k_fwd_tc" in names
    assert np.all(g["b_final"] == 0.0)
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta)
    assert_close("o", g["o"], r["o"], "bf16")


def test_debug_lambda_runs_exact_path():
    w = I.Workload("dbg", 1, 100, 4, 1, 64, "bf16", 18)
    x = I.make_prefill_inputs(w)
    _, names = kernels_ran(lambda: run_gpu(w, x, want_lambda=True))
    assert "k_fwd_simt" in names and "k_fwd_tc" not in names


def test_veto_gives_plain_attention_and_zero_bias():
    w = I.Workload("veto", 2, 150, 4, 2, 64, "bf16", 5)
    x = I.make_prefill_inputs(w)
    x["a_k"][:] = -1e4
    g = run_gpu(w, x, want_lambda=True)
    assert np.all(g["b_final"] == 0.0) and np.all(g["lam"] == 0.0)
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta)
    assert_close("o", g["o"], r["o"], "bf16")


def sampled_rows(T, n_rand=24, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, 1, 63, 64, 127, 128, 129, T // 2, T - 129, T - 128, T - 65, T - 64, T - 1}
    rows |= set(int(a) for a in rng.integers(0, T, n_rand))
    return sorted(r for r in rows if 0 <= r < T)


def check_sampled(w, units, seed):
    x = I.make_prefill_inputs(w)
    g = run_gpu(w, x)
    T, Hkv, G = w.T, w.Hkv, w.G
    rows = sampled_rows(T, seed=seed)
    rm = np.zeros(T, np.uint8)
    rm[rows] = 1
    um = np.zeros(w.B * Hkv, np.uint8)
    for b, h in units:
        um[b * Hkv + h] = 1
    r = oracle.prefill_fwd(**oracle_inputs(x), scale=w.scale, theta=w.theta, unit_mask=um, row_mask=rm)
    for b, h in units:
        hs = slice(h * G, (h + 1) * G)
        assert_close(f"o[{b},{h}]", g["o"][b][rows][:, hs], r["o"][b][rows][:, hs], w.dtype)
        assert_close(f"lse[{b},{h}]", g["lse"][b, hs][:, rows], r["lse"][b, hs][:, rows], w.dtype,
                     relative_max=True)
        assert_close(f"b_final[{b},{h}]", g["b_final"][b, h], r["b_final"][b, h], w.dtype, relative_max=True)
    assert np.all(np.isfinite(g["o"]))
    return g, r


@pytest.mark.slow
def test_prefill_1b_full_size_sampled():
    w = I.WORKLOADS["prefill_1b"]
    (_, _), names = kernels_ran(lambda: check_sampled(w, [(0, 0), (3, 5), (7, 7)], seed=1))
    assert "k_fwd_tc" in names


@pytest.mark.slow
def test_prefill_1b_16k_full_size_sampled():
    w = I.WORKLOADS["prefill_1b_16k"]
    (_, _), names = kernels_ran(lambda: check_sampled(w, [(0, 0), (0, 7)], seed=2))
    assert "k_fwd_tc" in names
