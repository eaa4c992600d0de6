"""fp64 CPU oracle for Universal Attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  The CUDA library never calls it and shares no
code with it.  The arithmetic lives in ``ua_oracle.c`` (plain C, fp64); this module only
builds it with gcc and marshals numpy arrays through ctypes.

Every function computes straight from the definitions written in the header of
``ua_oracle.c`` (structure from the pages "A Self-Pruning Transformer: Extreme KV-Cache
Compression with Universal Attention" (paperlayer.ai summary, §3, §4, §4.1, §4.2, App. C)
and the ai4snews synopsis of the same paper (Fig. 1 caption, veto property, eviction
paragraph)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ua_oracle.c")
_LIB = os.path.join(_HERE, "libua_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ua_oracle.c into libua_oracle.so next to it (gcc, -O2, IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dd = ctypes.c_double
        lib.ora_prefill_fwd.argtypes = [I, I, I, I, I, Dd, Dd] + [P] * 8 + [P, P] + [P] * 4 + [I, Dd, I, I]
        lib.ora_prefill_fwd.restype = I
        lib.ora_lambda_bruteforce.argtypes = [I, I, I, I, P, P, P, P, P, P, I, I]
        lib.ora_lambda_bruteforce.restype = I
        lib.ora_decode_step.argtypes = ([I, I, I, I, I, Dd, Dd] + [P] * 6 + [P] * 8 +
                                        [Dd, Dd, Dd, P, P, P, P, P, I, I, I])
        lib.ora_decode_step.restype = I
        lib.ora_compact_order.argtypes = [I, P, P]
        lib.ora_compact_order.restype = I
        lib.ora_prefill_bwd.argtypes = [I, I, I, I, I, Dd, Dd] + [P] * 8 + [P, P] + [P] * 8 + [I, Dd, I]
        lib.ora_prefill_bwd.restype = I
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


# Variant bits (the ablations; 0 = the method itself): a set bit 0 / 1 / 2 switches the
# query / key / similarity decay mechanism off; bit 3 RMS-normalises the queries.
VAR_NO_Q, VAR_NO_K, VAR_NO_SIM, VAR_QNORM = 1, 2, 4, 8


def prefill_fwd(q, k, v, g, a_q, a_k, alpha, beta, *, scale=None, theta=500000.0,
                want_lambda=False, unit_mask=None, row_mask=None, variant=0, prune_p=0.0, bf16_operands=False,
                nthreads=None):
    """Prefill forward of UA in fp64.

    Shapes: q, g [B,T,H,d]; k, v [B,T,Hkv,d]; a_q, a_k [B,T,Hkv]; alpha, beta [Hkv].
    prune_p > 0: chunked pruned prefill (128-token chunks, threshold p); 0 = dense.
    bf16_operands: a model for tolerances, not the method: the unit keys, rotated keys and
    rotated queries are rounded to bf16 where they enter the similarity and the logits.
    Returns dict(o [B,T,H,d], lse [B,H,T], b_final [B,Hkv,T], lam [B,Hkv,T,T] or None).
    Entries outside unit_mask / row_mask are left as NaN.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    a_q, a_k, alpha, beta = _f64(a_q), _f64(a_k), _f64(alpha), _f64(beta)
    B, T, H, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.full((B, T, H, d), np.nan)
    lse = np.full((B, H, T), np.nan)
    bfin = np.full((B, Hkv, T), np.nan)
    lam = np.zeros((B, Hkv, T, T)) if want_lambda else None
    um = None if unit_mask is None else np.ascontiguousarray(np.asarray(unit_mask, np.uint8))
    rm = None if row_mask is None else np.ascontiguousarray(np.asarray(row_mask, np.uint8))
    rc = _load().ora_prefill_fwd(B, T, H, Hkv, d, float(scale), float(theta),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q), _ptr(a_k),
                                 _ptr(alpha), _ptr(beta), _ptr(um), _ptr(rm),
                                 _ptr(o), _ptr(lse), _ptr(bfin), _ptr(lam), int(variant),
                                 float(np.log(prune_p)) if prune_p > 0 else -np.inf, int(bool(bf16_operands)),
                                 nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"ora_prefill_fwd rejected the shapes (code {rc})")
    return {"o": o, "lse": lse, "b_final": bfin, "lam": lam}


def lambda_bruteforce(k, a_q, a_k, alpha, beta, variant=0, nthreads=None):
    """Lambda [B,Hkv,T,T] from the O(T^3) direct sum (lower triangle; zeros above)."""
    k, a_q, a_k, alpha, beta = _f64(k), _f64(a_q), _f64(a_k), _f64(alpha), _f64(beta)
    B, T, Hkv, d = k.shape
    lam = np.zeros((B, Hkv, T, T))
    rc = _load().ora_lambda_bruteforce(B, T, Hkv, d, _ptr(k), _ptr(a_q), _ptr(a_k), _ptr(alpha),
                                       _ptr(beta), _ptr(lam), int(variant),
                                       nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"ora_lambda_bruteforce rejected the variant (code {rc})")
    return lam


def prefill_bwd(q, k, v, g, a_q, a_k, alpha, beta, d_o, *, scale=None, theta=500000.0,
                unit_mask=None, variant=0, bf16_saved_model=0.0, nthreads=None):
    """Analytic fp64 gradients of sum(dO * O).  Returns a dict keyed dq, dk, dv, dg,
    da_q, da_k, dalpha, dbeta (same shapes as the inputs).

    bf16_saved_model = c > 0: a model for tolerances, not the method.  The backward is fed what
    a bf16 forward saves: probabilities rounded to bf16 (scaled by c <= 1 first, standing in for
    a softmax shift above the row maximum) in the output and its normaliser, the output itself
    rounded to bf16, and delta_i = sum_x dO_ix o_ix formed from it.  Every gradient then moves
    by about -sum_i eps_i grad(lse_i), eps_i the resulting error of row i's (dP - delta)."""
    q, k, v, g, d_o = _f64(q), _f64(k), _f64(v), _f64(g), _f64(d_o)
    a_q, a_k, alpha, beta = _f64(a_q), _f64(a_k), _f64(alpha), _f64(beta)
    B, T, H, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = {n: np.full(x.shape, np.nan) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("da_q", a_q), ("da_k", a_k))}
    out["dalpha"] = np.zeros(Hkv)
    out["dbeta"] = np.zeros(Hkv)
    um = None if unit_mask is None else np.ascontiguousarray(np.asarray(unit_mask, np.uint8))
    rc = _load().ora_prefill_bwd(B, T, H, Hkv, d, float(scale), float(theta),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q), _ptr(a_k),
                                 _ptr(alpha), _ptr(beta), _ptr(d_o), _ptr(um),
                                 _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                 _ptr(out["dg"]), _ptr(out["da_q"]), _ptr(out["da_k"]),
                                 _ptr(out["dalpha"]), _ptr(out["dbeta"]), int(variant),
                                 float(bf16_saved_model), nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"ora_prefill_bwd rejected the shapes (code {rc})")
    return out


class DecodeCache:
    """fp64 oracle cache: per (b, KV head) slot arrays of raw key, value, a_k logit,
    token position and running bias b, plus the kept count."""

    def __init__(self, B, Hkv, d, cap):
        self.B, self.Hkv, self.d, self.cap = B, Hkv, d, cap
        self.k = np.zeros((B, Hkv, cap, d))
        self.v = np.zeros((B, Hkv, cap, d))
        self.ak = np.zeros((B, Hkv, cap))
        self.pos = np.zeros((B, Hkv, cap))
        self.b = np.zeros((B, Hkv, cap))
        self.n = np.zeros((B, Hkv), dtype=np.int32)

    def fill_from_prefill(self, k, v, a_k, b_final, logp=None, adopt_keep=None, band=1e-3):
        """Load a prefill's keys/values/a_k with their final biases b_final (Lambda's last
        row).  With logp given, keep only pairs with b >= logp (stable order); for pairs whose
        bias lies within `band` of logp, adopt_keep[b, h, t] (if given) decides instead.
        Returns the in-band mask [B,Hkv,T]."""
        k, v, a_k, b_final = _f64(k), _f64(v), _f64(a_k), _f64(b_final)
        B, T, Hkv, d = k.shape
        in_band = np.zeros((B, Hkv, T), bool)
        for b in range(B):
            for h in range(Hkv):
                if logp is None:
                    keep = np.ones(T, bool)
                else:
                    keep = b_final[b, h] >= logp
                    in_band[b, h] = np.abs(b_final[b, h] - logp) < band
                    if adopt_keep is not None:
                        keep = np.where(in_band[b, h], np.asarray(adopt_keep[b, h], bool), keep)
                idx = np.nonzero(keep)[0]
                n = len(idx)
                if n > self.cap:
                    raise ValueError("capacity exceeded")
                self.k[b, h, :n] = k[b, idx, h]
                self.v[b, h, :n] = v[b, idx, h]
                self.ak[b, h, :n] = a_k[b, idx, h]
                self.pos[b, h, :n] = idx
                self.b[b, h, :n] = b_final[b, h, idx]
                self.n[b, h] = n
        return in_band

    def compact(self, p):
        """Stable compaction of every slot list by b >= log p (after deferred decode steps)."""
        logp = float(np.log(p)) if p > 0 else -np.inf
        for b in range(self.B):
            for h in range(self.Hkv):
                n = int(self.n[b, h])
                idx = compact_order(self.b[b, h, :n] >= logp)
                m = len(idx)
                for arr in (self.k, self.v):
                    arr[b, h, :m] = arr[b, h, idx]
                for arr in (self.ak, self.pos, self.b):
                    arr[b, h, :m] = arr[b, h, idx]
                self.n[b, h] = m


def decode_step(cache: DecodeCache, q, k, v, g, a_q, a_k, alpha, beta, pos_t, p, *,
                scale=None, theta=500000.0, band=1e-3, adopt_keep=None, variant=0, defer=False,
                nthreads=None):
    """One decode step on the oracle cache (mutated in place).

    q, g [B,H,d]; k, v [B,Hkv,d]; a_q, a_k [B,Hkv].  Returns dict(o [B,H,d],
    evict [B,Hkv,cap] (over pre-step slots), in_band, kept_order [B,Hkv,cap] (old slot
    index of each survivor in new order, -1 beyond), n_before)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    a_q, a_k, alpha, beta = _f64(a_q), _f64(a_k), _f64(alpha), _f64(beta)
    B, H, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    logp = float(np.log(p)) if p > 0 else -np.inf
    o = np.full((B, H, d), np.nan)
    ev = np.zeros((B, Hkv, cache.cap), np.uint8)
    inb = np.zeros((B, Hkv, cache.cap), np.uint8)
    order = np.full((B, Hkv, cache.cap), -1, np.int64)
    ak_ = None if adopt_keep is None else np.ascontiguousarray(np.asarray(adopt_keep, np.uint8))
    n_before = cache.n.copy()
    rc = _load().ora_decode_step(B, H, Hkv, d, cache.cap, float(scale), float(theta),
                                 _ptr(cache.n), _ptr(cache.k), _ptr(cache.v), _ptr(cache.ak),
                                 _ptr(cache.pos), _ptr(cache.b),
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q), _ptr(a_k),
                                 _ptr(alpha), _ptr(beta), float(pos_t), logp, float(band),
                                 _ptr(ak_), _ptr(o), _ptr(ev), _ptr(inb), _ptr(order),
                                 int(variant), int(bool(defer)), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"ora_decode_step failed (code {rc})")
    return {"o": o, "evict": ev, "in_band": inb, "kept_order": order, "n_before": n_before}


def compact_order(keep):
    """Stable compaction order of a keep mask: kept slot indices, ascending."""
    keep = np.ascontiguousarray(np.asarray(keep, np.uint8))
    order = np.zeros(len(keep), np.int64)
    n = _load().ora_compact_order(len(keep), _ptr(keep), _ptr(order))
    return order[:n]


# ----------------------------------------------------------------------------- per-query-head decay
# The alternative reading of which head the decay parameters belong to (per query head rather
# than per KV head; an ablation direction of "A Self-Pruning Transformer: Extreme KV-Cache
# Compression with Universal Attention", paperlayer.ai summary App. E): a_q, a_k [B,T,H] and
# alpha, beta [H], every query head with its own rates and its own Lambda over its group's
# shared keys, each head evicting for itself.  That is multi-head UA on K and V repeated over
# the G query heads of each group, so these wrappers only repeat the keys and values (and sum
# their gradients back over the copies); all the arithmetic is the functions above.

def _repeat_kv(x, G):
    return np.repeat(_f64(x), G, axis=2)


def prefill_fwd_per_head(q, k, v, g, a_q, a_k, alpha, beta, **kw):
    """Prefill forward with per-query-head decay.  a_q, a_k [B,T,H]; alpha, beta [H].
    Returns as prefill_fwd, with b_final [B,H,T] (and lam [B,H,T,T])."""
    G = np.shape(q)[2] // np.shape(k)[2]
    return prefill_fwd(q, _repeat_kv(k, G), _repeat_kv(v, G), g, a_q, a_k, alpha, beta, **kw)


def prefill_bwd_per_head(q, k, v, g, a_q, a_k, alpha, beta, d_o, **kw):
    """Gradients of the per-query-head forward; dk, dv are summed over each group's heads."""
    B, T, Hkv, d = np.shape(k)
    G = np.shape(q)[2] // Hkv
    r = prefill_bwd(q, _repeat_kv(k, G), _repeat_kv(v, G), g, a_q, a_k, alpha, beta, d_o, **kw)
    r["dk"] = r["dk"].reshape(B, T, Hkv, G, d).sum(axis=3)
    r["dv"] = r["dv"].reshape(B, T, Hkv, G, d).sum(axis=3)
    return r


def decode_step_per_head(cache: DecodeCache, q, k, v, g, a_q, a_k, alpha, beta, pos_t, p, **kw):
    """One decode step with per-query-head decay: cache holds one head per query head (filled from
    the keys and values repeated over each group); q, g [B,H,d]; k, v [B,Hkv,d]; a_q, a_k [B,H];
    alpha, beta [H].  Returns as decode_step."""
    G = np.shape(q)[1] // np.shape(k)[1]
    return decode_step(cache, q, np.repeat(_f64(k), G, axis=1), np.repeat(_f64(v), G, axis=1), g, a_q, a_k,
                       alpha, beta, pos_t, p, **kw)
