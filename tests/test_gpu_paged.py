"""GPU tests of paged cache storage (ua_cache.page_table): a cache set on a pool of pages, with a
caller-owned page table, must give bit-identical results to the same caches stored contiguously
-- fill, compaction, eager and split decode steps -- whatever pages it is given (here shuffled),
while holding pages only for its live pairs; a page id outside the pool is reported, not
followed.  The contiguous caches' own parity with the fp64 oracle is tested elsewhere."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua

pytestmark = pytest.mark.gpu


def dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt).contiguous()


def _setup(w, T0, page_size, steps, dtype):
    x = I.make_prefill_inputs(w, T=T0, names=["q", "k", "v", "g", "a_q", "a_k", "alpha", "beta"])
    ob = oracle.prefill_fwd(**x, scale=w.scale, theta=w.theta, row_mask=np.zeros(T0, np.uint8))["b_final"]
    max_pages = (T0 + steps + page_size - 1) // page_size + 1
    cont = ua.Cache.empty(w.B, w.Hkv, w.d, max_pages * page_size, dtype)
    pool_pages = w.B * w.Hkv * max_pages + 5
    paged = ua.Cache.paged(w.B, w.Hkv, w.d, page_size, max_pages, pool_pages, dtype)
    pool = ua.PagePool(paged)
    rng = np.random.default_rng(w.seed)
    rng.shuffle(pool.free)                                    # pages in no particular order
    pool.ensure(T0)
    k, v, ak, bf = dev(x["k"], dtype), dev(x["v"], dtype), dev(x["a_k"], torch.float32), dev(ob, torch.float32)
    for c in (cont, paged):
        ua.cache_fill(c, k, v, ak, bf, theta=w.theta)
    return x, cont, paged, pool


def _same(cont, paged):
    torch.cuda.synchronize()
    n = cont.n_kept.cpu().numpy()
    np.testing.assert_array_equal(paged.n_kept.cpu().numpy(), n)
    for name in ("khat", "v", "bias", "rk", "pos"):
        a, b = getattr(cont, name), paged.logical(name)
        if name in ("khat", "v"):
            a, b = a.float(), b.float()
        a, b = a.cpu().numpy(), b.cpu().numpy()
        for bb in range(cont.B):
            for h in range(cont.Hkv):
                np.testing.assert_array_equal(b[bb, h, :n[bb, h]], a[bb, h, :n[bb, h]], err_msg=f"{name} {bb} {h}")


@pytest.mark.parametrize("dtype,d,H,Hkv,page_size,split", [(torch.bfloat16, 64, 8, 2, 128, False),
                                                           (torch.bfloat16, 64, 8, 2, 256, True),
                                                           (torch.bfloat16, 128, 6, 2, 128, True),
                                                           (torch.float32, 64, 4, 2, 128, True),
                                                           (torch.float32, 64, 4, 2, 128, False)])
def test_paged_caches_match_contiguous_ones(dtype, d, H, Hkv, page_size, split):
    T0, steps, p = 700, 12, 0.15
    w = I.Workload("paged", 2, T0, H, Hkv, d, "bf16" if dtype == torch.bfloat16 else "f32", 7100 + d + H,
                   bimodal_ak=True)
    x, cont, paged, pool = _setup(w, T0, page_size, steps, dtype)
    _same(cont, paged)
    for c in (cont, paged):
        ua.cache_compact(c, p)
    _same(cont, paged)
    pool.release()                                            # pages past the live pairs go back
    assert pool.pages_in_use() == sum((int(n) + page_size - 1) // page_size for n in paged.n_kept.reshape(-1).tolist())
    ws = {id(c): ua.alloc_workspace(ua.decode_workspace_size(c, H), "cuda") if split else None for c in (cont, paged)}
    al, be = dev(x["alpha"], torch.float32), dev(x["beta"], torch.float32)
    for s in range(steps):
        tok = I.make_decode_token(w, s)
        t = {n: dev(a, dtype if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
        pool.ensure(paged.n_kept.reshape(-1).cpu().numpy() + 1)   # a page for the append slot
        outs = []
        for c in (cont, paged):
            o = ua.decode_step(c, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], al, be, T0 + s, p,
                               scale=w.scale, theta=w.theta, ws=ws[id(c)])
            outs.append(o.float().cpu().numpy())
        assert ua.get_device_status() == 0
        np.testing.assert_array_equal(outs[0], outs[1])
        if split and s % 4 == 3:
            for c in (cont, paged):
                ua.cache_compact(c, p)
            pool.release()
        _same(cont, paged)


def test_a_page_outside_the_pool_is_reported_not_followed():
    """A page id of -1 or past the pool inside a cache's live slots raises UA_ERR_INVALID_ARG in
    the device status; the kernels skip that page's accesses (every address they form stays
    inside the pool), and the context stays usable."""
    w = I.Workload("paged_bad", 1, 300, 4, 2, 64, "bf16", 7300)
    x, cont, paged, pool = _setup(w, 300, 128, 4, torch.bfloat16)
    ua.get_device_status()
    al, be = dev(x["alpha"], torch.float32), dev(x["beta"], torch.float32)
    tok = I.make_decode_token(w, 0)
    t = {n: dev(a, torch.bfloat16 if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
    pool.ensure(301)
    saved = paged.page_table.clone()
    for bad in (-1, paged.pool_pages, 1 << 30):
        for split in (False, True):
            paged.page_table.copy_(saved)
            paged.page_table[1, 1] = bad                          # cache 1's slots 128..255
            ws = ua.alloc_workspace(ua.decode_workspace_size(paged, w.H), "cuda") if split else None
            ua.decode_step(paged, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], al, be, 300, 0.0,
                           scale=w.scale, theta=w.theta, ws=ws, defer_compact=True)
            assert ua.get_device_status() == 1, (bad, split)      # UA_ERR_INVALID_ARG
            paged.n_kept.fill_(300)
        ua.cache_compact(paged, 0.0)
        assert ua.get_device_status() == 1
        paged.n_kept.fill_(300)
    paged.page_table.copy_(saved)
    ua.decode_step(paged, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], al, be, 300, 0.0,
                   scale=w.scale, theta=w.theta)
    assert ua.get_device_status() == 0
