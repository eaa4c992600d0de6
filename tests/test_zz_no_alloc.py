"""GPU check of ua_prefill_fwd_noalloc, the prefill forward for callers that cannot allocate
device memory (for example a plug-in whose host application owns the whole GPU memory pool,
or a caller that cannot afford cudaMalloc's latency).  It must give the same results as
ua_prefill_fwd with a caller workspace, on two calls in a row (the shared internal scratch
keeps the previous call's contents, which must not leak into the next call).

This file is named to be collected last, so a run that stops at the first failure has run
every other test before it; it also passes on its own in a fresh process."""
import ctypes

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


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = ua.load_library()
    limit = lib.ua_prefill_noalloc_max_scratch()
    assert limit == 32 << 20
    shape = ua.ua_shape(8, 4096, 32, 8, 64, 0.125, 5e5, ua.UA_BF16)   # needs far more than 32 MiB
    need = ua.prefill_workspace_size(shape)
    assert need > limit
    P = ctypes.c_void_p
    fake = P(0x7f0000000000)                                          # never dereferenced: rejected first
    rc = lib.ua_prefill_fwd_noalloc(ctypes.byref(shape), *([fake] * 8), fake, None, None, None)
    assert rc == 4                                                    # UA_ERR_WORKSPACE
