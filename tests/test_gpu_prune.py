"""GPU parity of the chunked pruned prefill (ua_shape.prune_p) against the fp64 oracle.

"A Self-Pruning Transformer: Extreme KV-Cache Compression with Universal Attention"
(paperlayer.ai summary, §5): prefill pruning proceeds in chunks of 128 tokens.  Before the
chunk starting at row c, pairs j < c with Lambda_{c-1,j} < log p are evicted; later rows attend
over the survivors and their own chunk.

Eviction is a decision taken in floating point: a key whose boundary bias lies within the
bias tolerance of log p (1e-3 on the fp32 path, 2e-2 on the bf16 tensor-core path, the
b_final bars, both relative to max(1, |log p|)) may go either way, and then the rows of that chunk and KV group are not
compared.  Every other row must match; the decisions are re-taken at each boundary from the
monotone prefix, so an in-band key touches its own chunk only."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_close

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}
BAND = {"f32": 1e-3, "bf16": 2e-2}


def kernels_ran(fn):
    ua.profile_reset()
    ua.profile_enable(True)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        ua.profile_enable(False)
    return out, set(ua.profile_read())


def run(w, x, p, want_bfinal=True, want_lambda=False, variant=0):
    d = {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
        TORCH_DT[w.dtype] if n in ("q", "k", "v", "g") else torch.float32).contiguous() for n, a in x.items()}
    r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta, want_bfinal=want_bfinal, want_lambda=want_lambda,
                       prune_p=p, variant=variant)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.float().cpu().numpy()) for k, v in r.items()}


def compared_rows(w, lam, p):
    """[B, H, T] mask of rows whose chunk has no key within the band of log p at its boundary.
    The key just before the chunk is left out of the band check: its bias there,
    Lambda_{c-1,c-1} = 0, is exact on both sides (an empty sum), so it is always kept."""
    G = w.H // w.Hkv
    ok = np.ones((w.B, w.Hkv, w.T), bool)
    for c in range(128, w.T, 128):
        # the b_final bar is relative (errors against max(1, |ref|)), so at the threshold the
        # boundary bias may be off by BAND * max(1, |log p|)
        band = BAND[w.dtype] * max(1.0, abs(math.log(p)))
        near = np.abs(lam[:, :, c - 1, :c - 1] - math.log(p)) < band  # [B,Hkv,c-1]
        ok[:, :, c:c + 128] &= ~near.any(axis=2)[:, :, None]
    return np.repeat(ok, G, axis=1)


def check(w, g, r, lam, p, dense_bfinal=None):
    rows = compared_rows(w, lam, p)                                      # [B,H,T]
    # the relative band leaves 44 % of the rows of the (B=2, T=517, p=0.05) case, 74-100 % elsewhere
    assert rows.mean() > 0.4, "too few rows outside the eviction band"
    o_rows = np.transpose(rows, (0, 2, 1))                               # [B,T,H]
    assert_close("o", g["o"][o_rows], r["o"][o_rows], w.dtype)
    assert_close("lse", g["lse"][rows], r["lse"][rows], w.dtype, relative_max=True)
    if dense_bfinal is not None and g["b_final"] is not None:
        assert_close("b_final", g["b_final"], dense_bfinal, w.dtype, relative_max=True)


def oracle_pair(w, x, p, variant=0):
    xo = {k: v for k, v in x.items() if k != "d_o"}
    r = oracle.prefill_fwd(**xo, scale=w.scale, theta=w.theta, prune_p=p, want_lambda=True, variant=variant)
    dense = oracle.prefill_fwd(**xo, scale=w.scale, theta=w.theta, variant=variant)
    assert np.max(np.abs(dense["o"] - r["o"])) > 1e-3                  # pruning changed something
    return r, dense


@pytest.mark.parametrize("p", [0.05, 0.15, 0.5])
def test_fp32_simt_path(p):
    w = I.Workload("prune", 2, 420, 4, 2, 64, "f32", 1200)
    x = I.make_prefill_inputs(w)
    r, dense = oracle_pair(w, x, p)
    g, names = kernels_ran(lambda: run(w, x, p))
    assert "k_fwd_simt" in names
    check(w, g, r, r["lam"], p, dense["b_final"])


def test_fp32_debug_lambda_is_the_dense_lambda():
    # with the debug Lambda requested no tile is skipped: evicted keys are masked in place
    w = I.Workload("prune", 1, 300, 4, 2, 64, "f32", 1201)
    x = I.make_prefill_inputs(w)
    r, dense = oracle_pair(w, x, 0.15)
    g = run(w, x, 0.15, want_lambda=True)
    check(w, g, r, r["lam"], 0.15, dense["b_final"])
    tri = np.tril(np.ones((w.T, w.T), bool))
    assert_close("lambda", g["lam"][..., tri], r["lam"][..., tri], "f32", relative_max=True)


@pytest.mark.parametrize("B,T,H,Hkv,p", [(1, 1000, 4, 1, 0.15), (2, 517, 8, 2, 0.05), (1, 300, 4, 4, 0.5),
                                         (1, 700, 4, 2, 1.0)])
@pytest.mark.parametrize("want_bfinal", [True, False])
def test_bf16_tensor_core_path(B, T, H, Hkv, p, want_bfinal):
    w = I.Workload("prune_tc", B, T, H, Hkv, 64, "bf16", 1300 + T)
    x = I.make_prefill_inputs(w)
    r, dense = oracle_pair(w, x, p)
    g, names = kernels_ran(lambda: run(w, x, p, want_bfinal=want_bfinal))
    assert "k_fwd_tc" in names and "k_fwd_simt" not in names, names
    assert ua.get_device_status() == 0
    check(w, g, r, r["lam"], p, dense["b_final"])


def test_bf16_pruning_skips_more_tiles():
    w = I.Workload("prune_tc", 1, 1000, 4, 1, 64, "bf16", 1400)
    x = I.make_prefill_inputs(w)
    d = {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
        torch.bfloat16 if n in ("q", "k", "v", "g") else torch.float32).contiguous() for n, a in x.items()}
    skipped = []
    for p in (0.0, 0.15):
        shape = ua.make_shape(d["q"], d["k"], w.scale, w.theta, prune_p=p)
        ws = ua.alloc_workspace(ua.prefill_workspace_size(shape), "cuda")
        ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta, want_bfinal=False, ws=ws, prune_p=p)
        tiles, sk = ua.prefill_tile_stats(shape, ws)
        skipped.append(sk)
    assert skipped[1] > skipped[0], skipped


@pytest.mark.parametrize("B,T,H,Hkv,p", [(1, 400, 6, 2, 0.15), (1, 1000, 3, 1, 0.05), (2, 333, 6, 2, 0.5)])
@pytest.mark.parametrize("want_bfinal", [True, False])
def test_bf16_d128_tensor_core_path(B, T, H, Hkv, p, want_bfinal):
    """head_dim 128: 64-row query tiles, so the second tile of each 128-row chunk takes its
    eviction decisions from the prefix published by the tile two back (the chunk's start)."""
    w = I.Workload("prune", B, T, H, Hkv, 128, "bf16", 1500 + T)
    x = I.make_prefill_inputs(w)
    r, dense = oracle_pair(w, x, p)
    g, names = kernels_ran(lambda: run(w, x, p, want_bfinal=want_bfinal))
    assert "k_fwd_tc128" in names and "k_fwd_simt" not in names, names
    assert ua.get_device_status() == 0
    check(w, g, r, r["lam"], p, dense["b_final"])


@pytest.mark.parametrize("dtype,variant,kernel", [("bf16", ua.VAR_QUERY_NORM, "k_fwd_tc"),
                                                  ("f32", ua.VAR_NO_KEY_DECAY, "k_fwd_simt")])
def test_pruning_with_a_variant(dtype, variant, kernel):
    """The chunked pruning and an ablation variant together: the variant changes the prep and
    the decay, the pruning acts on the resulting prefixes."""
    w = I.Workload("prune_var", 1, 640, 8, 2, 64, dtype, 1600 + variant)
    x = I.make_prefill_inputs(w)
    r, dense = oracle_pair(w, x, 0.15, variant)
    g, names = kernels_ran(lambda: run(w, x, 0.15, variant=variant))
    assert kernel in names, names
    assert ua.get_device_status() == 0
    check(w, g, r, r["lam"], 0.15, dense["b_final"])
