"""GPU parity of the self-pruning cache (ua_cache_fill, ua_cache_compact, ua_decode_step)
against the fp64 oracle, stepped in lockstep.

Eviction decisions and the compacted order must match bit for bit, except for pairs whose
oracle bias lies within 1e-3 of log p; for those the oracle adopts the GPU's decision so
both caches stay in sync (otherwise one disagreement desynchronises every later step)."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ua_b200 import inputs as I
from kv_cache_compression_ua_b200 import ua
from helpers import EVICT_BAND, assert_close

pytestmark = pytest.mark.gpu
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dtype).contiguous()


def unpack_bits(words, n):
    """Bit s of word w is slot 32*w + s."""
    bits = np.unpackbits(np.ascontiguousarray(words, np.uint32).view(np.uint8), bitorder="little")
    return bits[:n].astype(bool)


_ORACLE_BFINAL = {}
_INPUTS = {}


def oracle_bfinal(w, T0, b, variant=0):
    """Oracle b_final of batch b (all KV heads), memoised across thresholds."""
    key = (repr(w), T0, b, variant)
    if key not in _ORACLE_BFINAL:
        xb = I.make_prefill_inputs(w, T=T0, B=1, b0=b)
        rm = np.zeros(T0, np.uint8)          # only b_final is needed
        ro = oracle.prefill_fwd(**{k: v for k, v in xb.items() if k != "d_o"}, scale=w.scale, theta=w.theta,
                                row_mask=rm, variant=variant)
        _ORACLE_BFINAL[key] = (xb, ro["b_final"])
    return _ORACLE_BFINAL[key]


class Lockstep:
    """GPU cache and oracle cache for batches `b_sel` of workload w, prefilled to T0."""

    def __init__(self, w, T0, steps, p, b_sel=None, zero_prefill_q=False, variant=0):
        self.w, self.T0, self.steps, self.p, self.variant = w, T0, steps, p, variant
        self.cap = T0 + steps + 1
        Bg = w.B
        key = (repr(w), T0, zero_prefill_q)
        if key not in _INPUTS:
            _INPUTS.clear()
            _INPUTS[key] = I.make_prefill_inputs(w, T=T0, names=["k", "v", "a_q", "a_k", "alpha", "beta"] +
                                                 ([] if zero_prefill_q else ["q", "g"]))
        x = _INPUTS[key]
        adt = TORCH_DT[w.dtype]
        d = {n: dev(a, adt if n in ("k", "v", "q", "g") else torch.float32) for n, a in x.items()}
        if zero_prefill_q:   # the prefill's queries and gates do not touch the cache
            d["q"] = torch.zeros(Bg, T0, w.H, w.d, dtype=adt, device="cuda")
            d["g"] = torch.zeros(Bg, T0, w.H, w.d, dtype=adt, device="cuda")
        r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                           scale=w.scale, theta=w.theta, want_lse=False, variant=variant)
        self.gb_final = r["b_final"].cpu().numpy()
        self.cache = ua.Cache.empty(Bg, w.Hkv, w.d, self.cap, adt)
        ua.cache_fill(self.cache, d["k"], d["v"], d["a_k"], r["b_final"], theta=w.theta)
        kept = torch.full((Bg, w.Hkv, self.cap), -7, dtype=torch.int32, device="cuda")
        ua.cache_compact(self.cache, p, kept_idx=kept)
        self.alpha, self.beta = d["alpha"], d["beta"]
        n_g = self.cache.n_kept.cpu().numpy()
        kept = kept.cpu().numpy()
        # oracle on the selected batches
        self.b_sel = list(range(Bg)) if b_sel is None else list(b_sel)
        self.ora = []
        for b in self.b_sel:
            xb, ob_final = oracle_bfinal(w, T0, b, variant)
            ro = {"b_final": ob_final}
            assert_close(f"b_final[b={b}]", self.gb_final[b], ro["b_final"][0], w.dtype, relative_max=True)
            gpu_keep = np.zeros((1, w.Hkv, T0), bool)
            for h in range(w.Hkv):
                gpu_keep[0, h, kept[b, h, :n_g[b, h]]] = True
            oc = oracle.DecodeCache(1, w.Hkv, w.d, self.cap)
            logp = math.log(p) if p > 0 else None
            in_band = oc.fill_from_prefill(xb["k"], xb["v"], xb["a_k"], ro["b_final"], logp=logp,
                                           adopt_keep=gpu_keep)
            if logp is not None:
                ora_keep = ro["b_final"] >= logp
                mism = (ora_keep != gpu_keep) & ~in_band
                assert not mism.any(), f"initial compaction differs outside the band: {np.argwhere(mism)[:5]}"
            for h in range(w.Hkv):
                np.testing.assert_array_equal(oc.pos[0, h, :oc.n[0, h]], kept[b, h, :n_g[b, h]])
            self.ora.append(oc)
        self.n_adopted = 0

    def step(self, s):
        w = self.w
        tok = I.make_decode_token(w, s)
        adt = TORCH_DT[w.dtype]
        t = {n: dev(a, adt if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
        pos_t = self.T0 + s
        n_before = self.cache.n_kept.cpu().numpy()
        words = (self.cap + 31) // 32
        ev = torch.zeros(w.B, w.Hkv, words, dtype=torch.int32, device="cuda")
        kept = torch.full((w.B, w.Hkv, self.cap), -7, dtype=torch.int32, device="cuda")
        o = ua.decode_step(self.cache, t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], self.alpha,
                           self.beta, pos_t, self.p, scale=w.scale, theta=w.theta, evict_bits=ev,
                           kept_idx=kept, variant=self.variant)
        assert ua.get_device_status() == 0
        o = o.float().cpu().numpy()
        ev = ev.cpu().numpy().view(np.uint32)
        kept = kept.cpu().numpy()
        n_after = self.cache.n_kept.cpu().numpy()
        pos_g = self.cache.pos.cpu().numpy()
        bias_g = self.cache.bias.cpu().numpy()
        for i, b in enumerate(self.b_sel):
            oc = self.ora[i]
            gpu_keep = np.zeros((1, w.Hkv, self.cap), np.uint8)
            gpu_ev = np.zeros((1, w.Hkv, self.cap), bool)
            for h in range(w.Hkv):
                e = unpack_bits(ev[b, h], n_before[b, h])
                gpu_ev[0, h, :n_before[b, h]] = e
                gpu_keep[0, h, :n_before[b, h]] = ~e
            assert np.array_equal(oc.n[0], n_before[b])
            ro = oracle.decode_step(oc, tok["q"][b:b + 1], tok["k"][b:b + 1], tok["v"][b:b + 1],
                                    tok["g"][b:b + 1], tok["a_q"][b:b + 1], tok["a_k"][b:b + 1],
                                    self.alpha.cpu().numpy(), self.beta.cpu().numpy(), pos_t, self.p,
                                    scale=w.scale, theta=w.theta, band=EVICT_BAND, adopt_keep=gpu_keep,
                                    variant=self.variant)
            inb = ro["in_band"].astype(bool)
            mism = (ro["evict"].astype(bool) != gpu_ev) & ~inb
            assert not mism.any(), f"step {s}: eviction differs outside the band at {np.argwhere(mism)[:5]}"
            self.n_adopted += int((inb & (ro["evict"].astype(bool) == gpu_ev)).sum())
            for h in range(w.Hkv):
                n = oc.n[0, h]
                assert n == n_after[b, h]
                np.testing.assert_array_equal(pos_g[b, h, :n], oc.pos[0, h, :n])
                np.testing.assert_array_equal(kept[b, h, :n - 1], ro["kept_order"][0, h, :n - 1])
                assert kept[b, h, n - 1] == -1
            assert_close(f"o step {s} b {b}", o[b], ro["o"][0], w.dtype)
            live = [(h, j) for h in range(w.Hkv) for j in range(oc.n[0, h])]
            gb = np.array([bias_g[b, h, j] for h, j in live])
            ob = np.array([oc.b[0, h, j] for h, j in live])
            assert_close(f"bias step {s} b {b}", gb, ob, w.dtype, relative_max=True)


@pytest.mark.parametrize("dtype,d,H,Hkv,p", [("bf16", 64, 8, 2, 0.15), ("bf16", 64, 8, 2, 0.05),
                                            ("bf16", 128, 6, 2, 0.15), ("f32", 64, 4, 2, 0.15),
                                            ("bf16", 64, 8, 8, 0.0)])
def test_small_lockstep(dtype, d, H, Hkv, p):
    w = I.Workload("dec_small", 3, 400, H, Hkv, d, dtype, 4242, bimodal_ak=True)
    ls = Lockstep(w, T0=400, steps=40, p=p)
    for s in range(40):
        ls.step(s)


NQ, NK, NS, QN = ua.VAR_NO_QUERY_DECAY, ua.VAR_NO_KEY_DECAY, ua.VAR_NO_SIM_DECAY, ua.VAR_QUERY_NORM


@pytest.mark.parametrize("variant,dtype,d,H,Hkv,p", [(NQ, "bf16", 64, 8, 2, 0.15), (NK | NS, "bf16", 64, 8, 2, 0.05),
                                                    (QN | NS, "f32", 64, 4, 2, 0.15), (QN, "bf16", 128, 6, 2, 0.15),
                                                    (NQ | NK, "f32", 64, 4, 4, 0.15)])
def test_variant_lockstep(variant, dtype, d, H, Hkv, p):
    """Ablation variants (decay mechanisms switched off, query norm) through fill, compaction
    and 24 decode steps, in lockstep with the oracle's variant.

    The similarity-only variant runs in f32: a bf16 cache holds the unit keys rounded to 8
    mantissa bits, and with the similarity rate alone (no cube or square root to divide its
    relative error) that rounding reaches the bias at full strength and accumulates over the
    steps, past the 1e-3 band that eviction decisions are compared within."""
    w = I.Workload("dec_var", 2, 300, H, Hkv, d, dtype, 4300 + variant, bimodal_ak=True)
    ls = Lockstep(w, T0=300, steps=24, p=p, variant=variant)
    for s in range(24):
        ls.step(s)


def test_p0_decode_reproduces_prefill_rows():
    """With p = 0 nothing is evicted, so step t of the decode must give row t of a prefill
    over the whole sequence (an identity between two GPU paths, checked in bf16 tolerance)."""
    w = I.Workload("dec_p0", 2, 96, 8, 2, 64, "bf16", 99)
    T0, steps = 64, 32
    x = I.make_prefill_inputs(w)
    dt = torch.bfloat16
    d = {n: dev(a, dt if n in ("q", "k", "v", "g") else torch.float32) for n, a in x.items()}
    full = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"])
    pre = {n: (t[:, :T0].contiguous() if t.dim() >= 2 else t) for n, t in d.items()}
    r = ua.prefill_fwd(pre["q"], pre["k"], pre["v"], pre["g"], pre["a_q"], pre["a_k"], d["alpha"], d["beta"])
    cache = ua.Cache.empty(w.B, w.Hkv, w.d, T0 + steps, dt)
    ua.cache_fill(cache, pre["k"], pre["v"], pre["a_k"], r["b_final"])
    for s in range(steps):
        t = T0 + s
        o = ua.decode_step(cache, d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                           d["v"][:, t].contiguous(), d["g"][:, t].contiguous(), d["a_q"][:, t].contiguous(),
                           d["a_k"][:, t].contiguous(), d["alpha"], d["beta"], t, 0.0)
        assert_close(f"row {t}", o.float().cpu().numpy(), full["o"][:, t].float().cpu().numpy(), "bf16")
    assert np.all(cache.n_kept.cpu().numpy() == T0 + steps)
    assert_close("bias vs b_final", cache.bias.cpu().numpy(), full["b_final"].cpu().numpy(), "bf16",
                 relative_max=True)


def test_capacity_overflow_sets_device_status():
    w = I.Workload("dec_cap", 1, 32, 4, 2, 64, "bf16", 3)
    x = I.make_prefill_inputs(w)
    dt = torch.bfloat16
    d = {n: dev(a, dt if n in ("q", "k", "v", "g") else torch.float32) for n, a in x.items()}
    r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"])
    cache = ua.Cache.empty(1, 2, 64, 32, dt)           # exactly full after the fill
    ua.cache_fill(cache, d["k"], d["v"], d["a_k"], r["b_final"])
    assert ua.get_device_status() == 0
    ua.decode_step(cache, d["q"][:, 0].contiguous(), d["k"][:, 0].contiguous(), d["v"][:, 0].contiguous(),
                   d["g"][:, 0].contiguous(), d["a_q"][:, 0].contiguous(), d["a_k"][:, 0].contiguous(),
                   d["alpha"], d["beta"], 32, 0.0)
    assert ua.get_device_status() == 5                  # UA_ERR_CAPACITY
    assert ua.get_device_status() == 0                  # cleared by the read
    assert np.all(cache.n_kept.cpu().numpy() == 32)


def test_compact_with_explicit_mask_is_stable_partition():
    w = I.Workload("cmp", 2, 700, 4, 2, 128, "bf16", 8)
    x = I.make_prefill_inputs(w)
    dt = torch.bfloat16
    d = {n: dev(a, dt if n in ("q", "k", "v", "g") else torch.float32) for n, a in x.items()}
    r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"])
    cache = ua.Cache.empty(2, 2, 128, 1000, dt)
    ua.cache_fill(cache, d["k"], d["v"], d["a_k"], r["b_final"])
    before = {n: getattr(cache, n).clone() for n in ("khat", "v", "bias", "rk", "pos")}
    rng = np.random.default_rng(0)
    keep = (rng.random((2, 2, 1000)) < 0.37).astype(np.uint8)
    kept = torch.full((2, 2, 1000), -7, dtype=torch.int32, device="cuda")
    ua.cache_compact(cache, keep=torch.from_numpy(keep).cuda(), kept_idx=kept)
    kept = kept.cpu().numpy()
    n = cache.n_kept.cpu().numpy()
    for b in range(2):
        for h in range(2):
            order = oracle.compact_order(keep[b, h, :700])
            assert n[b, h] == len(order)
            np.testing.assert_array_equal(kept[b, h, :len(order)], order)
            for nm, t0 in before.items():
                got = getattr(cache, nm)[b, h, :len(order)].cpu()
                ref = t0[b, h, torch.from_numpy(order)].cpu()
                assert torch.equal(got, ref), nm          # entries move bit for bit


@pytest.mark.slow
@pytest.mark.parametrize("p", [0.15, 0.05])
def test_decode_1b_full_size_sampled(p):
    """The decode workload at full size (B=32, 16k prefill, 256 steps); the oracle follows
    batches 0 and 31 (all 8 KV heads each) in lockstep."""
    w = I.WORKLOADS["decode_1b"]
    ls = Lockstep(w, T0=w.T, steps=I.DECODE_STEPS, p=p, b_sel=[0, w.B - 1], zero_prefill_q=True)
    for s in range(I.DECODE_STEPS):
        ls.step(s)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_deferred_compaction_matches_step_by_step(dtype):
    """UA_DECODE_DEFER_COMPACT: pairs stay in place (evicted ones excluded by their bias) and one
    ua_cache_compact(p) at the end gives the cache of step-by-step compaction.  Both GPU caches
    take the same decisions; outputs and biases agree within the parity bars (the two kernel
    instantiations may round the decay differently), slots and positions exactly."""
    w = I.Workload("dec_defer", 2, 300, 8, 2, 64, dtype, 4500, bimodal_ak=True)
    T0, steps, p = 300, 24, 0.15
    adt = TORCH_DT[dtype]
    x = I.make_prefill_inputs(w, T=T0)
    d = {n: dev(a, adt if n in ("k", "v", "q", "g") else torch.float32) for n, a in x.items() if n != "d_o"}
    r = ua.prefill_fwd(d["q"], d["k"], d["v"], d["g"], d["a_q"], d["a_k"], d["alpha"], d["beta"],
                       scale=w.scale, theta=w.theta, want_lse=False)
    cap = T0 + steps + 1
    caches = []
    for _ in range(2):
        c = ua.Cache.empty(w.B, w.Hkv, w.d, cap, adt)
        ua.cache_fill(c, d["k"], d["v"], d["a_k"], r["b_final"], theta=w.theta)
        ua.cache_compact(c, p)
        caches.append(c)
    eager, lazy = caches
    words = (cap + 31) // 32
    n_evicted = 0
    for s in range(steps):
        tok = I.make_decode_token(w, s)
        t = {n: dev(a, adt if n in ("q", "k", "v", "g") else torch.float32) for n, a in tok.items()}
        n_lazy = lazy.n_kept.cpu().numpy()
        ev_e = torch.zeros(w.B, w.Hkv, words, dtype=torch.int32, device="cuda")
        ev_l = torch.zeros_like(ev_e)
        kept = torch.full((w.B, w.Hkv, cap), -7, dtype=torch.int32, device="cuda")
        args = (t["q"], t["k"], t["v"], t["g"], t["a_q"], t["a_k"], d["alpha"], d["beta"], T0 + s, p)
        o_e = ua.decode_step(eager, *args, scale=w.scale, theta=w.theta, evict_bits=ev_e)
        o_l = ua.decode_step(lazy, *args, scale=w.scale, theta=w.theta, evict_bits=ev_l, kept_idx=kept,
                             defer_compact=True)
        assert ua.get_device_status() == 0
        assert_close(f"o step {s}", o_l.float().cpu().numpy(), o_e.float().cpu().numpy(), dtype)
        np.testing.assert_array_equal(lazy.n_kept.cpu().numpy(), n_lazy + 1)
        kept = kept.cpu().numpy()
        ev_l = ev_l.cpu().numpy().view(np.uint32)
        ev_e = ev_e.cpu().numpy().view(np.uint32)
        pos_l, pos_e, n_e = lazy.pos.cpu().numpy(), eager.pos.cpu().numpy(), eager.n_kept.cpu().numpy()
        for b in range(w.B):
            for h in range(w.Hkv):
                m = n_lazy[b, h]
                np.testing.assert_array_equal(kept[b, h, :m], np.arange(m))
                assert kept[b, h, m] == -1
                live = ~unpack_bits(ev_l[b, h], m)          # pairs with b >= log p after this step
                np.testing.assert_array_equal(pos_l[b, h, :m][live], pos_e[b, h, :n_e[b, h] - 1])
        n_evicted += int(sum(bin(int(v)).count("1") for v in ev_e.ravel()))
    assert n_evicted > 0
    ua.cache_compact(lazy, p)
    np.testing.assert_array_equal(lazy.n_kept.cpu().numpy(), eager.n_kept.cpu().numpy())
    n_e = eager.n_kept.cpu().numpy()
    for name in ("pos", "bias", "rk", "khat", "v"):
        a, b_ = getattr(lazy, name).float().cpu().numpy(), getattr(eager, name).float().cpu().numpy()
        for b in range(w.B):
            for h in range(w.Hkv):
                m = n_e[b, h]
                if name == "bias":
                    assert_close("bias", a[b, h, :m], b_[b, h, :m], "f32", relative_max=True)
                else:
                    np.testing.assert_array_equal(a[b, h, :m], b_[b, h, :m], err_msg=name)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128)])
def test_cache_fill_layout(dtype, d):
    """ua_cache_fill stores the unit keys pair-interleaved (no rotated copy), the values, the
    biases, softplus(a_k) and the positions, slot t <- token t."""
    w = I.Workload("fill", 2, 37, 2 * 2, 2, d, dtype, 91)
    x = I.make_prefill_inputs(w, names=["k", "v", "a_k"])
    adt = TORCH_DT[dtype]
    k, v, ak = dev(x["k"], adt), dev(x["v"], adt), dev(x["a_k"], torch.float32)
    bf = torch.randn(w.B, w.Hkv, w.T, device="cuda")
    cache = ua.Cache.empty(w.B, w.Hkv, d, 50, adt)
    ua.cache_fill(cache, k, v, ak, bf, theta=w.theta)
    torch.cuda.synchronize()
    assert ua.get_device_status() == 0
    assert cache.nbytes_per_entry() == 2 * d * (2 if dtype == "bf16" else 4) + 12
    np.testing.assert_array_equal(cache.n_kept.cpu().numpy(), np.full((w.B, w.Hkv), w.T))
    kf = k.float()
    khat = (kf / kf.norm(dim=-1, keepdim=True)).permute(0, 2, 1, 3)           # [B,Hkv,T,d]
    got = cache.khat_natural()[:, :, :w.T].float()
    tol = 4e-3 if dtype == "bf16" else 1e-6
    assert float((got - khat).abs().max()) <= tol
    # pair-interleaved: element 2m is component m, element 2m+1 component m + d/2
    h = d // 2
    assert float((cache.khat[:, :, :w.T, 2 * 3].float() - khat[..., 3]).abs().max()) <= tol
    assert float((cache.khat[:, :, :w.T, 2 * 5 + 1].float() - khat[..., h + 5]).abs().max()) <= tol
    assert torch.equal(cache.v[:, :, :w.T], v.permute(0, 2, 1, 3))
    assert torch.equal(cache.bias[:, :, :w.T], bf)
    assert torch.equal(cache.pos[:, :, :w.T].cpu(), torch.arange(w.T, dtype=torch.int32).expand(w.B, w.Hkv, w.T))
    rk = torch.nn.functional.softplus(ak).permute(0, 2, 1)
    assert float((cache.rk[:, :, :w.T] - rk).abs().max()) <= 1e-6
