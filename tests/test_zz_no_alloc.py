"""GPU check of ua_prefill_fwd_noalloc, the prefill forward for callers that cannot allocate
device memory (for example a plug-in whose host application owns the whole GPU memory pool,
or a caller that cannot afford cudaMalloc's latency).  It must give the same results as
ua_prefill_fwd with a caller workspace, on two calls in a row (the shared internal scratch
keeps the previous call's contents, which must not leak into the next call).

This file is named to be collected last, so a run that stops at the first failure has run
every other test before it; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_close

pytestmark = pytest.mark.gpu


def _device_inputs(w):
    x = I.make_prefill_inputs(w)
    return {n: torch.from_numpy(a).cuda().to(torch.bfloat16 if n in ("q", "k", "v", "g") else torch.float32)
            for n, a in x.items()}


def _both(d, w):
    args = (d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"])
    ref = ua.prefill_fwd(*args, scale=w.scale, theta=w.theta)
    got = ua.prefill_fwd_noalloc(*args, scale=w.scale, theta=w.theta)
    torch.cuda.synchronize()
    return ref, got


def _compare(ref, got, tag):
    assert_close(f"{tag} o", got["o"].float().cpu().numpy(), ref["o"].float().cpu().numpy(), "bf16")
    assert_close(f"{tag} lse", got["lse"].cpu().numpy(), ref["lse"].cpu().numpy(), "bf16", relative_max=True)
    assert_close(f"{tag} b_final", got["b_final"].cpu().numpy(), ref["b_final"].cpu().numpy(), "bf16",
                 relative_max=True)


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    # a 1B-shaped layer at 2048 tokens, then a different, smaller problem, through the
    # same scratch: the second call must not see the first call's leftovers
    w1 = I.Workload("noalloc_a", 1, 2048, 32, 8, 64, "bf16", 2024)
    w2 = I.Workload("noalloc_b", 2, 333, 8, 2, 64, "bf16", 2025, bimodal_ak=True)
    for w, tag in ((w1, "first call"), (w2, "second call")):
        ref, got = _both(_device_inputs(w), w)
        _compare(ref, got, tag)
    assert ua.get_device_status() == 0


def test_noalloc_simt_layout_twice_in_a_row():
    # problems that run the fp32 SIMT kernels (f32 activations; a decay mechanism switched off)
    # lay the scratch out differently from the tensor-core path: same check on that layout
    w1 = I.Workload("noalloc_c", 1, 300, 4, 2, 128, "f32", 2026)
    w2 = I.Workload("noalloc_d", 2, 200, 8, 2, 64, "bf16", 2027, bimodal_ak=True)
    for w, variant, tag in ((w1, 0, "f32 d=128"), (w2, ua.VAR_NO_SIM_DECAY, "bf16 without the similarity rate")):
        x = I.make_prefill_inputs(w)
        dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        d = {n: torch.from_numpy(a).cuda().to(dt if n in ("q", "k", "v", "g") else torch.float32)
             for n, a in x.items()}
        args = (d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"])
        ref = ua.prefill_fwd(*args, scale=w.scale, theta=w.theta, variant=variant)
        got = ua.prefill_fwd_noalloc(*args, scale=w.scale, theta=w.theta, variant=variant)
        torch.cuda.synchronize()
        assert_close(f"{tag} o", got["o"].float().cpu().numpy(), ref["o"].float().cpu().numpy(), w.dtype)
        assert_close(f"{tag} lse", got["lse"].cpu().numpy(), ref["lse"].cpu().numpy(), w.dtype, relative_max=True)
        assert_close(f"{tag} b_final", got["b_final"].cpu().numpy(), ref["b_final"].cpu().numpy(), w.dtype,
                     relative_max=True)
    assert ua.get_device_status() == 0


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = ua.load_library()
    limit = lib.ua_prefill_noalloc_max_scratch()
    assert limit == 32 << 20
    B, T, H, Hkv, dh = 8, 4096, 32, 8, 64                             # needs far more than 32 MiB
    shape = ua.ua_shape(B, T, H, Hkv, dh, 0.125, 5e5, ua.UA_BF16)
    assert ua.prefill_workspace_size(shape) > limit
    # real device tensors of the full size, so no check order could ever launch on a bad address
    bf, f = torch.bfloat16, torch.float32
    q = torch.zeros(B, T, H, dh, dtype=bf, device="cuda")
    k = torch.zeros(B, T, Hkv, dh, dtype=bf, device="cuda")
    a = torch.zeros(B, T, Hkv, dtype=f, device="cuda")
    ab = torch.zeros(Hkv, dtype=f, device="cuda")
    with pytest.raises(ua.UAError) as e:
        ua.prefill_fwd_noalloc(q, k, k.clone(), q.clone(), a, a.clone(), ab, ab.clone(), scale=0.125, theta=5e5)
    assert e.value.code == 4                                          # UA_ERR_WORKSPACE
    assert ua.get_device_status() == 0
