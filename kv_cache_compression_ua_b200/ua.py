"""Thin Python binding of libua (include/ua.h): argument marshalling only.

Every step of the Universal Attention hot path runs in libua's CUDA kernels; this module
only turns torch CUDA tensors into device pointers, allocates outputs / workspaces with
torch (device memory plumbing) and checks status codes.  There is no fallback: if libua.so
is missing or a CUDA device is absent, the first call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libua.so")

UA_F32, UA_BF16 = 0, 1
STATUS = {0: "UA_OK", 1: "UA_ERR_INVALID_ARG", 2: "UA_ERR_UNSUPPORTED", 3: "UA_ERR_ALIGNMENT",
          4: "UA_ERR_WORKSPACE", 5: "UA_ERR_CAPACITY", 6: "UA_ERR_CUDA", 7: "UA_ERR_TIMEOUT",
          8: "UA_ERR_RANGE"}


class UAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class ua_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("scale", ctypes.c_float), ("rope_theta", ctypes.c_double),
                ("dtype", ctypes.c_int), ("variant", ctypes.c_int), ("prune_p", ctypes.c_float)]


# ua_shape.variant bits (UA_VAR_* in ua.h); 0 is the method itself.
VAR_NO_QUERY_DECAY, VAR_NO_KEY_DECAY, VAR_NO_SIM_DECAY, VAR_QUERY_NORM = 1, 2, 4, 8
VAR_PER_HEAD_DECAY = 16         # decay logits and parameters per query head: a_q, a_k [B,T,H], alpha, beta [H]
DECODE_DEFER_COMPACT = 256      # ua_decode_step flag: leave evicted pairs in place


class ua_cache(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int), ("capacity", ctypes.c_int),
                ("dtype", ctypes.c_int), ("kv_rep", ctypes.c_int), ("khat", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("rk", ctypes.c_void_p),
                ("pos", ctypes.c_void_p), ("n_kept", ctypes.c_void_p), ("page_size", ctypes.c_int),
                ("max_pages", ctypes.c_int), ("pool_pages", ctypes.c_int), ("page_table", ctypes.c_void_p)]


EXPORTS = ("ua_prefill_workspace_size", "ua_prefill_fwd", "ua_prefill_bwd_workspace_size", "ua_prefill_bwd",
           "ua_cache_fill", "ua_cache_compact", "ua_decode_step", "ua_get_device_status",
           "ua_profile_enable", "ua_profile_reset", "ua_profile_read", "ua_status_string", "ua_version",
           "ua_prefill_fwd_noalloc", "ua_prefill_noalloc_max_scratch", "ua_prefill_tile_stats",
           "ua_set_wait_limit_ns", "ua_decode_workspace_size", "ua_decode_step_split", "ua_prefill_fixed_rows",
           "ua_prefill_bwd_band_stats")


class ua_kernel_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]

_lib = None


def load_library(path: str = LIB_PATH):
    """Load libua.so and declare its signatures.  Raises if the file is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libua.so not found at {path}; build it with "
                           "`python -m kv_cache_compression_ua_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, D, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_size_t
    SP = ctypes.POINTER(ua_shape)
    CP = ctypes.POINTER(ua_cache)
    lib.ua_prefill_workspace_size.argtypes = [SP, ctypes.POINTER(S)]
    lib.ua_prefill_fwd.argtypes = [SP] + [P] * 8 + [P, P, P, P, P, S, P]
    lib.ua_prefill_bwd_workspace_size.argtypes = [SP, ctypes.POINTER(S)]
    lib.ua_prefill_bwd.argtypes = [SP] + [P] * 8 + [P, P, P, P] + [P] * 8 + [P, S, P]
    lib.ua_cache_fill.argtypes = [CP, I, P, P, P, P, D, P]
    lib.ua_cache_compact.argtypes = [CP, P, F, P, P]
    lib.ua_decode_step.argtypes = [CP, I] + [P] * 8 + [I, F, F, D, P, P, P, I, P]
    lib.ua_get_device_status.argtypes = [P, ctypes.POINTER(I)]
    lib.ua_profile_enable.argtypes = [I]
    lib.ua_profile_reset.argtypes = []
    lib.ua_profile_read.argtypes = [ctypes.POINTER(ua_kernel_time), I, ctypes.POINTER(I)]
    lib.ua_prefill_fwd_noalloc.argtypes = [SP] + [P] * 8 + [P, P, P, P]
    lib.ua_prefill_noalloc_max_scratch.argtypes = []
    lib.ua_prefill_tile_stats.argtypes = [SP, P, S, ctypes.POINTER(ctypes.c_ulonglong),
                                          ctypes.POINTER(ctypes.c_ulonglong), P]
    lib.ua_prefill_noalloc_max_scratch.restype = S
    lib.ua_prefill_fixed_rows.argtypes = [SP, P, S, ctypes.POINTER(ctypes.c_ulonglong), P]
    lib.ua_prefill_bwd_band_stats.argtypes = [SP, P, S, ctypes.POINTER(ctypes.c_ulonglong),
                                              ctypes.POINTER(ctypes.c_ulonglong), P]
    lib.ua_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.ua_decode_workspace_size.argtypes = [CP, I, ctypes.POINTER(S)]
    lib.ua_decode_step_split.argtypes = [CP, I] + [P] * 8 + [I, F, F, D, P, P, P, I, P, S, P]
    lib.ua_status_string.argtypes = [I]
    lib.ua_status_string.restype = ctypes.c_char_p
    lib.ua_version.argtypes = []
    for n in EXPORTS:
        if n not in ("ua_status_string", "ua_version", "ua_prefill_noalloc_max_scratch"):
            getattr(lib, n).restype = I
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != 0:
        raise UAError(fn, code)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libua takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libua takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _same_device(dev, **tensors):
    """Every tensor of a call must live on the device the call runs on: the library launches on
    the current device, so a tensor elsewhere would be reached through peer memory or not at all."""
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name}: on {t.device}, the call runs on {dev}")


def _on(dev):
    """Make `dev` current for the call (the library resolves per-device state on the current device).
    A tensor off the GPU is refused by _ptr inside the block."""
    return torch.cuda.device(dev) if dev.type == "cuda" else contextlib.nullcontext()


F32 = (torch.float32,)
I32 = (torch.int32,) + ((torch.uint32,) if hasattr(torch, "uint32") else ())
MASK = (torch.uint8, torch.bool)


def _need(name, t, n, dtypes):
    """Refuse a tensor the library would read or write past its end, or in another element type
    (the C ABI takes bare pointers, so this is the last place such a mistake can be caught)."""
    if t is None:
        return
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if t.numel() < n:
        raise ValueError(f"{name}: {t.numel()} elements, the call needs {n}")


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _rate_heads(H, Hkv, variant):
    """Heads the decay logits and parameters belong to: the KV heads, or (per-query-head decay)
    the query heads."""
    return H if int(variant) & VAR_PER_HEAD_DECAY else Hkv


def _prefill_dims(q, k, v, g, a_q, a_k, alpha, beta, out, variant=0):
    """Checks the prefill arguments against q [B,T,H,d] and k [B,T,Hkv,d]; returns the sizes."""
    B, T, H, d = q.shape
    if k.dim() != 4 or (k.shape[0], k.shape[1], k.shape[3]) != (B, T, d):
        raise ValueError(f"k: shape {tuple(k.shape)}, expected [{B}, {T}, Hkv, {d}]")
    Hkv = k.shape[2]
    Hr = _rate_heads(H, Hkv, variant)
    act = (q.dtype,)
    _need("k", k, B * T * Hkv * d, act)
    _need("v", v, B * T * Hkv * d, act)
    _need("g", g, B * T * H * d, act)
    _need("a_q", a_q, B * T * Hr, F32)
    _need("a_k", a_k, B * T * Hr, F32)
    _need("alpha", alpha, Hr, F32)
    _need("beta", beta, Hr, F32)
    _need("out", out, B * T * H * d, act)
    _same_device(q.device, k=k, v=v, g=g, a_q=a_q, a_k=a_k, alpha=alpha, beta=beta, out=out)
    return B, T, H, Hkv, d


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return UA_F32
    if dt == torch.bfloat16:
        return UA_BF16
    raise ValueError(f"unsupported activation dtype {dt}")


def make_shape(q: torch.Tensor, k: torch.Tensor, scale=None, theta=500000.0, variant=0, prune_p=0.0) -> ua_shape:
    B, T, H, d = q.shape
    Hkv = k.shape[2]
    scale = float(d) ** -0.5 if scale is None else float(scale)
    return ua_shape(B, T, H, Hkv, d, scale, float(theta), _dtype_code(q.dtype), int(variant), float(prune_p))


def prefill_workspace_size(shape: ua_shape) -> int:
    n = ctypes.c_size_t(0)
    _check("ua_prefill_workspace_size", load_library().ua_prefill_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns >= 512-byte aligned blocks; zeroed, as the split decode
    # step's arrival counters must start at zero (the prefill's scratch needs nothing)
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def prefill_fwd(q, k, v, g, a_q, a_k, alpha, beta, *, scale=None, theta=500000.0, want_lse=True,
                want_bfinal=True, want_lambda=False, out=None, lse=None, b_final=None, ws=None, variant=0,
                prune_p=0.0, stream=None):
    """ua_prefill_fwd (variant: VAR_* bits; prune_p > 0: chunked pruned prefill).  out, lse and
    b_final may be given as preallocated outputs.  Returns dict(o, lse, b_final, lam) (absent
    outputs are None)."""
    lib = load_library()
    B, T, H, Hkv, d = _prefill_dims(q, k, v, g, a_q, a_k, alpha, beta, out, variant)
    Hr = _rate_heads(H, Hkv, variant)
    _need("lse", lse, B * H * T, F32)
    _need("b_final", b_final, B * Hr * T, F32)
    shape = make_shape(q, k, scale, theta, variant, prune_p)
    dev = q.device
    _same_device(dev, lse=lse, b_final=b_final)
    o = out if out is not None else torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, T, dtype=torch.float32, device=dev)
    if b_final is None and want_bfinal:
        b_final = torch.empty(B, Hr, T, dtype=torch.float32, device=dev)
    bfin = b_final
    lam = torch.empty(B, Hr, T, T, dtype=torch.float32, device=dev) if want_lambda else None
    need = prefill_workspace_size(shape)
    if ws is None or _nbytes(ws) < need:
        ws = alloc_workspace(need, dev)
    _same_device(dev, ws=ws)
    with _on(dev):
        rc = lib.ua_prefill_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q), _ptr(a_k),
                                _ptr(alpha), _ptr(beta), _ptr(o), _ptr(lse), _ptr(bfin), _ptr(lam),
                                _ptr(ws), ctypes.c_size_t(_nbytes(ws)), _stream(stream))
    _check("ua_prefill_fwd", rc)
    return {"o": o, "lse": lse, "b_final": bfin, "lam": lam}


def prefill_tile_stats(shape: ua_shape, ws: torch.Tensor, stream=None) -> tuple:
    """ua_prefill_tile_stats: (causal tiles, tiles whose softmax was skipped) of the last
    ua_prefill_fwd that used `ws` for `shape`."""
    tiles, skipped = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check("ua_prefill_tile_stats", load_library().ua_prefill_tile_stats(
        ctypes.byref(shape), _ptr(ws), _nbytes(ws), ctypes.byref(tiles), ctypes.byref(skipped), _stream(stream)))
    return tiles.value, skipped.value


def prefill_bwd_band_stats(shape: ua_shape, ws: torch.Tensor, stream=None) -> tuple:
    """ua_prefill_bwd_band_stats: (32-row steps of the causal band, steps the key-major pass
    walked) of the last ua_prefill_bwd that used `ws` for `shape`."""
    steps, walked = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check("ua_prefill_bwd_band_stats", load_library().ua_prefill_bwd_band_stats(
        ctypes.byref(shape), _ptr(ws), _nbytes(ws), ctypes.byref(steps), ctypes.byref(walked), _stream(stream)))
    return steps.value, walked.value


def prefill_fixed_rows(shape: ua_shape, ws: torch.Tensor, stream=None) -> int:
    """ua_prefill_fixed_rows: (row, query head) pairs the last tensor-core ua_prefill_fwd that
    used `ws` for `shape` recomputed exactly (out of its softmax shift's range)."""
    rows = ctypes.c_ulonglong(0)
    _check("ua_prefill_fixed_rows", load_library().ua_prefill_fixed_rows(
        ctypes.byref(shape), _ptr(ws), _nbytes(ws), ctypes.byref(rows), _stream(stream)))
    return rows.value


def prefill_fwd_noalloc(q, k, v, g, a_q, a_k, alpha, beta, *, scale=None, theta=500000.0, want_lse=True,
                        want_bfinal=True, out=None, variant=0, prune_p=0.0, stream=None):
    """ua_prefill_fwd_noalloc: the prefill forward using the library's fixed internal scratch
    instead of a workspace (for callers that cannot allocate device memory)."""
    lib = load_library()
    B, T, H, Hkv, d = _prefill_dims(q, k, v, g, a_q, a_k, alpha, beta, out, variant)
    shape = make_shape(q, k, scale, theta, variant, prune_p)
    dev = q.device
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty(B, H, T, dtype=torch.float32, device=dev) if want_lse else None
    bfin = torch.empty(B, _rate_heads(H, Hkv, variant), T, dtype=torch.float32, device=dev) if want_bfinal else None
    with _on(dev):   # the library's scratch array is resolved on the current device
        rc = lib.ua_prefill_fwd_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q),
                                        _ptr(a_k), _ptr(alpha), _ptr(beta), _ptr(o), _ptr(lse), _ptr(bfin),
                                        _stream(stream))
    _check("ua_prefill_fwd_noalloc", rc)
    return {"o": o, "lse": lse, "b_final": bfin}


def prefill_bwd_workspace_size(shape: ua_shape) -> int:
    n = ctypes.c_size_t(0)
    _check("ua_prefill_bwd_workspace_size",
           load_library().ua_prefill_bwd_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def prefill_bwd(q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final, d_o, *, scale=None, theta=500000.0,
                ws=None, variant=0, stream=None):
    """ua_prefill_bwd (variant: the forward's VAR_* bits).  Returns dict(dq, dk, dv, dg,
    da_q, da_k, dalpha, dbeta)."""
    lib = load_library()
    B, T, H, Hkv, d = _prefill_dims(q, k, v, g, a_q, a_k, alpha, beta, None, variant)
    _need("o", o, B * T * H * d, (q.dtype,))
    _need("d_o", d_o, B * T * H * d, (q.dtype,))
    _need("lse", lse, B * H * T, F32)
    _need("b_final", b_final, B * _rate_heads(H, Hkv, variant) * T, F32)
    shape = make_shape(q, k, scale, theta, variant)
    dev = q.device
    gr = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
          "dg": torch.empty_like(g), "da_q": torch.empty_like(a_q), "da_k": torch.empty_like(a_k),
          "dalpha": torch.empty_like(alpha), "dbeta": torch.empty_like(beta)}
    need = prefill_bwd_workspace_size(shape)
    if ws is None or _nbytes(ws) < need:
        ws = alloc_workspace(need, dev)
    _same_device(dev, o=o, lse=lse, b_final=b_final, d_o=d_o, ws=ws)
    with _on(dev):
        rc = lib.ua_prefill_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q), _ptr(a_k),
                                _ptr(alpha), _ptr(beta), _ptr(o), _ptr(lse), _ptr(b_final), _ptr(d_o),
                                _ptr(gr["dq"]), _ptr(gr["dk"]), _ptr(gr["dv"]), _ptr(gr["dg"]), _ptr(gr["da_q"]),
                                _ptr(gr["da_k"]), _ptr(gr["dalpha"]), _ptr(gr["dbeta"]), _ptr(ws),
                                ctypes.c_size_t(_nbytes(ws)), _stream(stream))
    _check("ua_prefill_bwd", rc)
    return gr


@dataclass
class Cache:
    """Device tensors of one self-pruning cache set (see ua_cache in ua.h).  khat holds the unit
    keys pair-interleaved (element 2m = component m, 2m+1 = component m + d/2); `khat_natural()`
    returns them in the natural order.  kv_rep: cache heads per head of the keys and values the
    cache is filled and stepped with (G for per-query-head decay, where Hkv = H)."""
    B: int
    Hkv: int
    d: int
    capacity: int
    dtype: torch.dtype
    khat: torch.Tensor
    v: torch.Tensor
    bias: torch.Tensor
    rk: torch.Tensor
    pos: torch.Tensor
    n_kept: torch.Tensor
    kv_rep: int = 1
    # paged storage (see ua_cache.page_table): the arrays above are a pool of pool_pages pages of
    # page_size slots, page_table [B*Hkv, max_pages] int32 maps a cache's pages to pool pages
    page_size: int = 0
    pool_pages: int = 0
    page_table: torch.Tensor | None = None

    @staticmethod
    def paged(B, Hkv, d, page_size, max_pages, pool_pages, dtype=torch.bfloat16, device="cuda", kv_rep=1):
        """A cache set on a pool of pool_pages pages of page_size slots; every cache may grow to
        max_pages pages.  The page table starts empty (-1): give the caches pages with a PagePool."""
        if kv_rep < 1 or Hkv % kv_rep:
            raise ValueError(f"kv_rep {kv_rep} must divide Hkv {Hkv}")
        if page_size < 128 or page_size & (page_size - 1):
            raise ValueError(f"page_size {page_size} must be a power of two >= 128")
        kw = dict(device=device)
        slots = pool_pages * page_size
        return Cache(B, Hkv, d, max_pages * page_size, dtype,
                     torch.zeros(slots, d, dtype=dtype, **kw), torch.zeros(slots, d, dtype=dtype, **kw),
                     torch.zeros(slots, dtype=torch.float32, **kw), torch.zeros(slots, dtype=torch.float32, **kw),
                     torch.zeros(slots, dtype=torch.int32, **kw), torch.zeros(B, Hkv, dtype=torch.int32, **kw),
                     kv_rep, page_size, pool_pages,
                     torch.full((B * Hkv, max_pages), -1, dtype=torch.int32, **kw))

    @staticmethod
    def empty(B, Hkv, d, capacity, dtype=torch.bfloat16, device="cuda", kv_rep=1):
        if kv_rep < 1 or Hkv % kv_rep:
            raise ValueError(f"kv_rep {kv_rep} must divide Hkv {Hkv}")
        kw = dict(device=device)
        return Cache(B, Hkv, d, capacity, dtype,
                     torch.zeros(B, Hkv, capacity, d, dtype=dtype, **kw),
                     torch.zeros(B, Hkv, capacity, d, dtype=dtype, **kw),
                     torch.zeros(B, Hkv, capacity, dtype=torch.float32, **kw),
                     torch.zeros(B, Hkv, capacity, dtype=torch.float32, **kw),
                     torch.zeros(B, Hkv, capacity, dtype=torch.int32, **kw),
                     torch.zeros(B, Hkv, dtype=torch.int32, **kw), kv_rep)

    @property
    def Hin(self) -> int:
        """Heads of the keys and values the cache is filled and stepped with."""
        return self.Hkv // self.kv_rep

    def struct(self) -> ua_cache:
        paged = self.page_table is not None
        n = self.pool_pages * self.page_size if paged else self.B * self.Hkv * self.capacity
        for name in ("khat", "v"):
            _need(f"cache.{name}", getattr(self, name), n * self.d, (self.dtype,))
        _need("cache.bias", self.bias, n, F32)
        _need("cache.rk", self.rk, n, F32)
        _need("cache.pos", self.pos, n, I32)
        _need("cache.n_kept", self.n_kept, self.B * self.Hkv, I32)
        names = FIELDS
        dev = self.khat.device
        _same_device(dev, **{f"cache.{n}": getattr(self, n) for n in names})
        ptrs = [_ptr(getattr(self, n)).value for n in names]
        if not paged:
            return ua_cache(self.B, self.Hkv, self.d, self.capacity, _dtype_code(self.dtype), int(self.kv_rep), *ptrs)
        max_pages = self.capacity // self.page_size
        _need("cache.page_table", self.page_table, self.B * self.Hkv * max_pages, I32)
        _same_device(dev, **{"cache.page_table": self.page_table})
        return ua_cache(self.B, self.Hkv, self.d, self.capacity, _dtype_code(self.dtype), int(self.kv_rep), *ptrs,
                        self.page_size, max_pages, self.pool_pages, _ptr(self.page_table).value)

    def logical(self, name: str) -> torch.Tensor:
        """A cache array in the contiguous layout [B, Hkv, capacity(, d)] (a copy for a paged cache,
        slots without a page read as zeros)."""
        t = getattr(self, name)
        if self.page_table is None:
            return t
        ps = self.page_size
        s = torch.arange(self.capacity, device=t.device)
        pg = self.page_table[:, s // ps].long()                     # [B*Hkv, capacity]
        idx = pg * ps + (s % ps)
        out = t[idx.clamp(min=0)]
        out[pg < 0] = 0
        return out.reshape(self.B, self.Hkv, self.capacity, *t.shape[1:])

    def nbytes_per_entry(self) -> int:
        return 2 * self.d * self.khat.element_size() + 12

    def khat_natural(self) -> torch.Tensor:
        """khat with the components in their natural order (a copy)."""
        return torch.cat([self.khat[..., 0::2], self.khat[..., 1::2]], dim=-1)


FIELDS = ("khat", "v", "bias", "rk", "pos", "n_kept")


class PagePool:
    """Host-side page allocator of a paged Cache (argument marshalling: it only edits the page
    table).  ensure(n) gives every cache u pages for its slots [0, n[u]); release() hands the pages
    past each cache's live pairs (ceil(n_kept / page_size)) back to the pool, as a compaction
    leaves them empty.  Both read or write the table with one host<->device copy."""

    def __init__(self, cache: Cache):
        if cache.page_table is None:
            raise ValueError("PagePool needs a paged Cache")
        self.cache = cache
        self.ps = cache.page_size
        self.table = cache.page_table.cpu().numpy().copy()
        used = set(int(x) for x in self.table.ravel() if x >= 0)
        self.free = [pg for pg in range(cache.pool_pages - 1, -1, -1) if pg not in used]

    def pages_in_use(self) -> int:
        return int((self.table >= 0).sum())

    def _upload(self):
        self.cache.page_table.copy_(torch.from_numpy(self.table))

    def ensure(self, n_slots):
        """n_slots: per cache (an int for all, or [B, Hkv] / [B*Hkv]) the slots that need pages."""
        import numpy as np
        want = np.broadcast_to(np.asarray(n_slots, dtype=np.int64).reshape(-1), (self.table.shape[0],))
        for u, n in enumerate(want):
            for pg in range((int(n) + self.ps - 1) // self.ps):
                if self.table[u, pg] < 0:
                    if not self.free:
                        raise RuntimeError("page pool exhausted")
                    self.table[u, pg] = self.free.pop()
        self._upload()

    def release(self):
        """Return the pages past each cache's live pairs (reads n_kept)."""
        n = self.cache.n_kept.reshape(-1).cpu().numpy()
        for u, k in enumerate(n):
            for pg in range((int(k) + self.ps - 1) // self.ps, self.table.shape[1]):
                if self.table[u, pg] >= 0:
                    self.free.append(int(self.table[u, pg]))
                    self.table[u, pg] = -1
        self._upload()


def cache_fill(cache: Cache, k, v, a_k, b_final, *, theta=500000.0, stream=None):
    if k.dim() != 4 or (k.shape[0], k.shape[2], k.shape[3]) != (cache.B, cache.Hin, cache.d):
        raise ValueError(f"k: shape {tuple(k.shape)}, expected [{cache.B}, T, {cache.Hin}, {cache.d}]")
    T = k.shape[1]
    n = cache.B * T * cache.Hkv
    _need("k", k, cache.B * T * cache.Hin * cache.d, (cache.dtype,))
    _need("v", v, cache.B * T * cache.Hin * cache.d, (cache.dtype,))
    _need("a_k", a_k, n, F32)
    _need("b_final", b_final, n, F32)
    c = cache.struct()
    dev = cache.khat.device
    _same_device(dev, k=k, v=v, a_k=a_k, b_final=b_final)
    with _on(dev):
        _check("ua_cache_fill", load_library().ua_cache_fill(ctypes.byref(c), T, _ptr(k), _ptr(v), _ptr(a_k),
                                                             _ptr(b_final), float(theta), _stream(stream)))


def cache_compact(cache: Cache, p: float = 0.0, keep=None, kept_idx=None, stream=None):
    n = cache.B * cache.Hkv * cache.capacity
    _need("keep", keep, n, MASK)
    _need("kept_idx", kept_idx, n, I32)
    c = cache.struct()
    dev = cache.khat.device
    _same_device(dev, keep=keep, kept_idx=kept_idx)
    with _on(dev):
        _check("ua_cache_compact", load_library().ua_cache_compact(ctypes.byref(c), _ptr(keep), float(p),
                                                                   _ptr(kept_idx), _stream(stream)))


def decode_workspace_size(cache: Cache, H: int) -> int:
    """ua_decode_workspace_size: bytes of the split decode step's workspace."""
    n = ctypes.c_size_t(0)
    c = cache.struct()
    _check("ua_decode_workspace_size", load_library().ua_decode_workspace_size(ctypes.byref(c), int(H),
                                                                               ctypes.byref(n)))
    return n.value


def decode_step(cache: Cache, q, k, v, g, a_q, a_k, alpha, beta, pos_t: int, p: float, *, scale=None,
                theta=500000.0, out=None, evict_bits=None, kept_idx=None, variant=0, defer_compact=False,
                ws=None, stream=None):
    """ua_decode_step for one token per sequence (variant: the prefill's VAR_* bits;
    defer_compact: leave evicted pairs in place until cache_compact).  With a workspace `ws`
    (decode_workspace_size bytes) the step runs as ua_decode_step_split: long caches are walked
    by several CTAs each and compaction is deferred.  Returns o [B,H,d]."""
    B, H, d = q.shape
    if (B, d) != (cache.B, cache.d):
        raise ValueError(f"q: shape {tuple(q.shape)}, expected [{cache.B}, H, {cache.d}]")
    Hkv, act = cache.Hkv, (cache.dtype,)
    _need("q", q, B * H * d, act)
    _need("k", k, B * cache.Hin * d, act)
    _need("v", v, B * cache.Hin * d, act)
    _need("g", g, B * H * d, act)
    _need("a_q", a_q, B * Hkv, F32)
    _need("a_k", a_k, B * Hkv, F32)
    _need("alpha", alpha, Hkv, F32)
    _need("beta", beta, Hkv, F32)
    _need("out", out, B * H * d, act)
    _need("evict_bits", evict_bits, B * Hkv * ((cache.capacity + 31) // 32), I32)
    _need("kept_idx", kept_idx, B * Hkv * cache.capacity, I32)
    scale = float(d) ** -0.5 if scale is None else float(scale)
    o = out if out is not None else torch.empty_like(q)
    c = cache.struct()
    dev = cache.khat.device
    _same_device(dev, q=q, k=k, v=v, g=g, a_q=a_q, a_k=a_k, alpha=alpha, beta=beta, out=o,
                 evict_bits=evict_bits, kept_idx=kept_idx)
    flags = int(variant) | (DECODE_DEFER_COMPACT if defer_compact else 0)
    with _on(dev):
        if ws is not None:
            _same_device(dev, ws=ws)
            rc = load_library().ua_decode_step_split(ctypes.byref(c), H, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                                     _ptr(a_q), _ptr(a_k), _ptr(alpha), _ptr(beta), int(pos_t),
                                                     float(p), scale, float(theta), _ptr(o), _ptr(evict_bits),
                                                     _ptr(kept_idx), flags, _ptr(ws), ctypes.c_size_t(_nbytes(ws)),
                                                     _stream(stream))
            _check("ua_decode_step_split", rc)
            return o
        rc = load_library().ua_decode_step(ctypes.byref(c), H, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(a_q),
                                           _ptr(a_k), _ptr(alpha), _ptr(beta), int(pos_t), float(p), scale,
                                           float(theta), _ptr(o), _ptr(evict_bits), _ptr(kept_idx), flags,
                                           _stream(stream))
    _check("ua_decode_step", rc)
    return o


def get_device_status(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("ua_get_device_status", load_library().ua_get_device_status(_stream(stream), ctypes.byref(code)))
    return code.value


WAIT_LIMIT_DEFAULT_NS = 2_000_000_000


def set_wait_limit_ns(ns: int):
    """ua_set_wait_limit_ns: limit of every bounded device-side wait on the current device."""
    _check("ua_set_wait_limit_ns", load_library().ua_set_wait_limit_ns(int(ns)))


def profile_enable(on: bool = True):
    _check("ua_profile_enable", load_library().ua_profile_enable(1 if on else 0))


def profile_reset():
    _check("ua_profile_reset", load_library().ua_profile_reset())


def profile_read() -> dict:
    """{kernel name: (launches, total_ms)} for the launches recorded since the last reset."""
    arr = (ua_kernel_time * 64)()
    n = ctypes.c_int(0)
    _check("ua_profile_read", load_library().ua_profile_read(arr, 64, ctypes.byref(n)))
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n.value)}


def version() -> int:
    return load_library().ua_version()
