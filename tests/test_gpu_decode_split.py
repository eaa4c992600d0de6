"""GPU check of the split decode step (ua_decode_step_split) of fp32 caches, which runs on the
CUDA cores (bf16 caches take the tensor-core kernel, checked against the oracle in
test_gpu_decode_tc.py): long caches walked by several CTAs at once, compaction deferred.  Against
the one-CTA deferred step on an identical cache: the same biases (the same per-pair arithmetic,
bit for bit), the same eviction bits and appended slots, and outputs within the fp32 bars (the
partial softmax states are summed in another order).  A cache of 2.5k-4k live pairs takes 5-8
slices; the decode threshold evicts inside every slice."""
import numpy as np
import pytest
import torch

from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import assert_close

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt).contiguous()


@pytest.mark.parametrize("dtype,d,H,Hkv,T0", [("f32", 64, 8, 2, 2600), ("f32", 128, 6, 2, 4000),
                                              ("f32", 64, 4, 1, 3000)])
def test_split_decode_matches_single_cta_deferred_step(dtype, d, H, Hkv, T0):
    w = I.Workload("dec_split", 1, T0, H, Hkv, d, dtype, 5100 + T0, bimodal_ak=True)
    steps, p = 12, 0.15
    adt = TORCH_DT[dtype]
    x = I.make_prefill_inputs(w, T=T0)
    dd = {n: dev(a, adt if n in ("k", "v", "q", "g") else torch.float32) for n, a in x.items() if n != "d_o"}
    r = ua.prefill_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["a_q"], dd["a_k"], dd["alpha"], dd["beta"],
                       scale=w.scale, theta=w.theta, want_lse=False)
    cap = T0 + steps + 1
    caches = []
    for _ in range(2):
        c = ua.Cache.empty(w.B, w.Hkv, w.d, cap, adt)
        ua.cache_fill(c, dd["k"], dd["v"], dd["a_k"], r["b_final"], theta=w.theta)
        ua.cache_compact(c, 0.0)              # keep every pair: long caches; the steps evict at p
        caches.append(c)
    one, split = caches
    ws = ua.alloc_workspace(ua.decode_workspace_size(split, H), "cuda")
    words = (cap + 31) // 32
    ua.profile_reset()
    ua.profile_enable(True)
    evicted = 0
    try:
        for s in range(steps):
            tok = I.make_decode_token(w, s)
            t = {n: dev(a, adt if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
            args = (t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], dd["alpha"], dd["beta"], T0 + s, p)
            ev1 = torch.zeros(w.B, w.Hkv, words, dtype=torch.int32, device="cuda")
            ev2 = torch.full_like(ev1, -1)
            k1 = torch.full((w.B, w.Hkv, cap), -7, dtype=torch.int32, device="cuda")
            k2 = torch.full_like(k1, -7)
            o1 = ua.decode_step(one, *args, scale=w.scale, theta=w.theta, evict_bits=ev1, kept_idx=k1,
                                defer_compact=True)
            o2 = ua.decode_step(split, *args, scale=w.scale, theta=w.theta, evict_bits=ev2, kept_idx=k2, ws=ws)
            torch.cuda.synchronize()
            assert ua.get_device_status() == 0
            assert_close(f"o step {s}", o2.float().cpu().numpy(), o1.float().cpu().numpy(), dtype)
            assert torch.equal(ev1, ev2), f"step {s}: eviction bits differ"
            assert torch.equal(k1, k2), f"step {s}: kept_idx differs"
            for name in ("n_kept", "bias", "pos", "rk", "khat", "v"):
                assert torch.equal(getattr(one, name), getattr(split, name)), f"step {s}: cache.{name}"
            evicted += int(sum(bin(int(v) & 0xffffffff).count("1") for v in ev1.cpu().numpy().ravel()))
    finally:
        ua.profile_enable(False)
    assert "k_decode_split" in set(ua.profile_read())
    assert evicted > 0
