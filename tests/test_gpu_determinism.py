"""Run-to-run bit identity of every GPU path (a race detector where no sanitizer runs).

No kernel accumulates through atomics: the tensor-core forward's CTAs take work tickets in
whatever order they start, but each computes its tile from its own inputs and the prefix its
predecessor published, whose value does not depend on timing; the backward reduces its
partials in a fixed order; the decode's only atomic is an OR of eviction bits.  So repeated
calls on the same inputs must agree bit for bit, and a race (a buffer read before or after
the write it was meant to see) would show as a difference."""
import numpy as np
import pytest
import torch

from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(x, dtype):
    return {n: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(
        TORCH_DT[dtype] if n in ("q", "k", "v", "g", "d_o") else torch.float32).contiguous() for n, a in x.items()}


def same(runs):
    for r in runs[1:]:
        for k in runs[0]:
            if runs[0][k] is not None:
                assert torch.equal(r[k], runs[0][k]), k


@pytest.mark.parametrize("B,T,H,Hkv,d,dtype,want_bfinal", [(2, 2000, 8, 2, 64, "bf16", True),
                                                          (1, 2048, 4, 1, 64, "bf16", False),
                                                          (1, 700, 6, 2, 128, "bf16", True),
                                                          (2, 333, 4, 2, 64, "f32", True)])
def test_prefill_forward_is_deterministic(B, T, H, Hkv, d, dtype, want_bfinal):
    w = I.Workload("det", B, T, H, Hkv, d, dtype, 2100 + T)
    x = dev({k: v for k, v in I.make_prefill_inputs(w).items() if k != "d_o"}, dtype)
    runs = []
    for _ in range(3):
        r = ua.prefill_fwd(x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"],
                           scale=w.scale, theta=w.theta, want_bfinal=want_bfinal)
        torch.cuda.synchronize()
        runs.append({k: (None if v is None else v.clone()) for k, v in r.items()})
    assert ua.get_device_status() == 0
    same(runs)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128)])
def test_backward_is_deterministic(dtype, d):
    w = I.Workload("detb", 1, 300, 4, 2, d, dtype, 2200, with_grad=True)
    x = dev(I.make_prefill_inputs(w), dtype)
    args = (x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"])
    f = ua.prefill_fwd(*args, scale=w.scale, theta=w.theta)
    runs = []
    for _ in range(2):
        g = ua.prefill_bwd(*args, f["o"], f["lse"], f["b_final"], x["d_o"], scale=w.scale, theta=w.theta)
        torch.cuda.synchronize()
        runs.append({k: v.clone() for k, v in g.items()})
    assert ua.get_device_status() == 0
    same(runs)


def test_decode_is_deterministic():
    w = I.Workload("detd", 2, 400, 8, 2, 64, "bf16", 2300, bimodal_ak=True)
    x = dev({k: v for k, v in I.make_prefill_inputs(w).items() if k != "d_o"}, "bf16")
    r = ua.prefill_fwd(x["q"], x["k"], x["v"], x["g"], x["a_q"], x["a_k"], x["alpha"], x["beta"],
                       scale=w.scale, theta=w.theta, want_lse=False)
    outs = []
    for _ in range(2):
        c = ua.Cache.empty(w.B, w.Hkv, w.d, w.T + 20, torch.bfloat16)
        ua.cache_fill(c, x["k"], x["v"], x["a_k"], r["b_final"], theta=w.theta)
        ua.cache_compact(c, 0.15)
        os_ = []
        for s in range(16):
            t = dev(I.make_decode_token(w, s), "bf16")
            o = ua.decode_step(c, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], x["alpha"], x["beta"],
                               w.T + s, 0.15, scale=w.scale, theta=w.theta)
            os_.append(o.clone())
        torch.cuda.synchronize()
        outs.append((os_, {n: getattr(c, n).clone() for n in ("khat", "v", "bias", "rk", "pos", "n_kept")}))
    assert ua.get_device_status() == 0
    for a, b in zip(outs[0][0], outs[1][0]):
        assert torch.equal(a, b)
    for n in outs[0][1]:
        assert torch.equal(outs[0][1][n], outs[1][1][n]), n
