"""CPU checks of the C ABI: the library builds, loads, exports every symbol that
include/ua.h declares, and rejects bad arguments on the host (before any launch)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from kv_cache_compression_ua_b200 import build as ua_build
from kv_cache_compression_ua_b200 import ua

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ua_build.build()
    return ua.load_library()


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "ua.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(ua_[a-z_]+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("ua_prefill_fwd", "ua_prefill_bwd", "ua_decode_step", "ua_cache_compact"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ua.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ua_[a-z_]+)\b", out))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    for n in declared_symbols():
        assert hasattr(lib, n)
    assert set(ua.EXPORTS) == set(declared_symbols())


def test_version_and_status_strings(lib):
    assert lib.ua_version() >= 100
    assert lib.ua_status_string(0) == b"UA_OK"
    assert lib.ua_status_string(5) == b"UA_ERR_CAPACITY"


def _shape(**kw):
    s = dict(B=1, T=128, H=4, Hkv=2, d=64, scale=0.125, rope_theta=5e5, dtype=ua.UA_BF16)
    s.update(kw)
    return ua.ua_shape(**s)


FAKE = 0x7f0000000000          # aligned, never dereferenced: validation fails first


def _fwd(lib, shape, ptrs=None, ws=FAKE, ws_bytes=1 << 40):
    P = ctypes.c_void_p
    p = [P(FAKE)] * 8 if ptrs is None else ptrs
    return lib.ua_prefill_fwd(ctypes.byref(shape), *p, P(FAKE), None, None, None, P(ws),
                              ctypes.c_size_t(ws_bytes), None)


@pytest.mark.parametrize("kw,code", [(dict(d=96), 2), (dict(H=6, Hkv=4), 1), (dict(T=0), 1),
                                     (dict(H=12, Hkv=2), 2), (dict(dtype=7), 2), (dict(rope_theta=0.0), 1)])
def test_prefill_rejects_bad_shapes(lib, kw, code):
    assert _fwd(lib, _shape(**kw)) == code


def test_prefill_rejects_null_misaligned_and_small_workspace(lib):
    P = ctypes.c_void_p
    ptrs = [P(FAKE)] * 8
    ptrs[2] = None
    assert _fwd(lib, _shape(), ptrs) == 1
    ptrs = [P(FAKE)] * 8
    ptrs[0] = P(FAKE + 2)
    assert _fwd(lib, _shape(), ptrs) == 3
    assert _fwd(lib, _shape(), ws=FAKE + 16) == 3
    need = ctypes.c_size_t(0)
    assert lib.ua_prefill_workspace_size(ctypes.byref(_shape()), ctypes.byref(need)) == 0
    assert need.value > 0
    assert _fwd(lib, _shape(), ws_bytes=need.value - 1) == 4


@pytest.mark.parametrize("variant,code", [(32, 1), (7, 1), (15, 1), (23, 1), (-8, 1), (1, 0), (6, 0), (8, 0),
                                          (11, 0), (16, 0), (24, 0)])
def test_variant_bits_validated(lib, variant, code):
    need = ctypes.c_size_t(0)
    s = _shape(variant=variant)
    assert lib.ua_prefill_workspace_size(ctypes.byref(s), ctypes.byref(need)) == code
    assert lib.ua_prefill_bwd_workspace_size(ctypes.byref(s), ctypes.byref(need)) == code
    if code:
        assert _fwd(lib, s) == code


@pytest.mark.parametrize("prune_p,code", [(-0.1, 1), (1.5, 1), (float("nan"), 1), (0.0, 0), (0.15, 0), (1.0, 0)])
def test_prune_threshold_validated(lib, prune_p, code):
    need = ctypes.c_size_t(0)
    s = _shape(prune_p=prune_p)
    assert lib.ua_prefill_workspace_size(ctypes.byref(s), ctypes.byref(need)) == code
    if code:
        assert _fwd(lib, s) == code
    # training is dense: the backward refuses any pruning threshold
    bwd_code = 0 if prune_p == 0.0 else 1
    assert lib.ua_prefill_bwd_workspace_size(ctypes.byref(s), ctypes.byref(need)) == bwd_code


def test_mechanism_variants_leave_the_tensor_core_path(lib):
    # a mechanism switched off runs the SIMT path: no tensor-core tile statistics
    tiles, skipped = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    s = _shape(T=512, variant=ua.VAR_NO_SIM_DECAY)
    assert lib.ua_prefill_tile_stats(ctypes.byref(s), None, ctypes.c_size_t(0), ctypes.byref(tiles),
                                     ctypes.byref(skipped), None) == 0
    assert tiles.value == 4 * 5 // 2 * 2 and skipped.value == 0


def test_lambda_debug_limited_to_small_T(lib):
    P = ctypes.c_void_p
    shape = _shape(T=2048)
    rc = lib.ua_prefill_fwd(ctypes.byref(shape), *([P(FAKE)] * 8), P(FAKE), None, None, P(FAKE), P(FAKE),
                            ctypes.c_size_t(1 << 40), None)
    assert rc == 1


def test_cache_calls_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    c = ua.ua_cache(2, 2, 64, 100, ua.UA_BF16, 1, *([FAKE] * 6))
    # capacity too small for the fill
    assert lib.ua_cache_fill(ctypes.byref(c), 101, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 5e5, None) == 5
    # bad p without a mask
    assert lib.ua_cache_compact(ctypes.byref(c), None, ctypes.c_float(1.5), None, None) == 1
    # misaligned cache array
    c2 = ua.ua_cache(2, 2, 64, 100, ua.UA_BF16, 1, *([FAKE] * 5 + [FAKE + 4]))
    assert lib.ua_cache_compact(ctypes.byref(c2), None, ctypes.c_float(0.1), None, None) == 3
    # decode: group size 5 unsupported, flags must be valid variant bits, head_dim 80 unsupported
    args = [P(FAKE)] * 8
    assert lib.ua_decode_step(ctypes.byref(c), 10, *args, 5, ctypes.c_float(0.1), ctypes.c_float(0.125), 5e5,
                              P(FAKE), None, None, 0, None) == 2
    # unknown bits; all three decay mechanisms off; per-query-head decay on a cache that does not
    # hold one head per query head (H = 8 != Hkv = 2)
    for bad in (16, 7, 15, -1, 512, 256 | 7, 256 | 16):
        assert lib.ua_decode_step(ctypes.byref(c), 8, *args, 5, ctypes.c_float(0.1), ctypes.c_float(0.125), 5e5,
                                  P(FAKE), None, None, bad, None) == 1
    # kv_rep must divide Hkv (and not be negative)
    for rep in (3, -1):
        cr = ua.ua_cache(2, 2, 64, 100, ua.UA_BF16, rep, *([FAKE] * 6))
        assert lib.ua_cache_compact(ctypes.byref(cr), None, ctypes.c_float(0.1), None, None) == 1
    # paged storage: page size a power of two >= 128, capacity = max_pages * page_size, a pool,
    # an aligned table
    for ps_, mp, pp, tab, want in ((100, 1, 4, FAKE, 1), (64, 2, 4, FAKE, 1), (128, 2, 4, FAKE, 1),
                                   (128, 1, 0, FAKE, 1), (128, 1, 4, FAKE + 2, 3)):
        cpg = ua.ua_cache(2, 2, 64, 128 if want == 1 and mp == 2 else ps_ * mp, ua.UA_BF16, 1, *([FAKE] * 6),
                          ps_, mp, pp, tab)
        assert lib.ua_cache_compact(ctypes.byref(cpg), None, ctypes.c_float(0.1), None, None) == want, (ps_, mp, pp)
    c3 = ua.ua_cache(2, 2, 80, 100, ua.UA_BF16, 1, *([FAKE] * 6))
    assert lib.ua_decode_step(ctypes.byref(c3), 8, *args, 5, ctypes.c_float(0.1), ctypes.c_float(0.125), 5e5,
                              P(FAKE), None, None, 0, None) == 2


def test_tile_stats_host_logic(lib):
    """ua_prefill_tile_stats: argument checks, and the tile count for problems that run the fp32
    SIMT path (no device access: nothing is skipped there)."""
    import ctypes
    tiles, skipped = ctypes.c_ulonglong(7), ctypes.c_ulonglong(7)
    s = _shape(B=2, T=300, H=4, Hkv=2, d=64, dtype=ua.UA_F32)
    assert lib.ua_prefill_tile_stats(ctypes.byref(s), None, 0, ctypes.byref(tiles), ctypes.byref(skipped),
                                     None) == 0
    n = (300 + 127) // 128
    assert tiles.value == 2 * 2 * n * (n + 1) // 2 and skipped.value == 0
    assert lib.ua_prefill_tile_stats(ctypes.byref(s), None, 0, None, ctypes.byref(skipped), None) == 1
    bad = _shape(B=0)
    assert lib.ua_prefill_tile_stats(ctypes.byref(bad), None, 0, ctypes.byref(tiles), ctypes.byref(skipped),
                                     None) == 1
    # the tensor-core path needs the workspace it ran on
    tc = _shape(B=1, T=300, H=4, Hkv=1, d=64, dtype=ua.UA_BF16)
    assert lib.ua_prefill_tile_stats(ctypes.byref(tc), None, 0, ctypes.byref(tiles), ctypes.byref(skipped),
                                     None) == 1
    assert lib.ua_prefill_tile_stats(ctypes.byref(tc), ctypes.c_void_p(256), 16, ctypes.byref(tiles),
                                     ctypes.byref(skipped), None) == 4


# --------------------------------------------------------------------------- Python binding checks
# The binding refuses, before any CUDA call, tensors the library would read or write past their
# end or in another element type.  CPU tensors with the right sizes get through these checks
# and stop at the device check, which is how the tests tell the two apart.

def _prefill_args(B=1, T=8, H=4, Hkv=2, d=64, act=torch.bfloat16):
    f = torch.float32
    return dict(q=torch.zeros(B, T, H, d, dtype=act), k=torch.zeros(B, T, Hkv, d, dtype=act),
                v=torch.zeros(B, T, Hkv, d, dtype=act), g=torch.zeros(B, T, H, d, dtype=act),
                a_q=torch.zeros(B, T, Hkv, dtype=f), a_k=torch.zeros(B, T, Hkv, dtype=f),
                alpha=torch.zeros(Hkv, dtype=f), beta=torch.zeros(Hkv, dtype=f))


def _call_fwd(**over):
    a = _prefill_args()
    a.update(over)
    return ua.prefill_fwd(a["q"], a["k"], a["v"], a["g"], a["a_q"], a["a_k"], a["alpha"], a["beta"])


def test_binding_passes_well_formed_prefill_arguments(lib):
    with pytest.raises(ValueError, match="CUDA tensors"):
        _call_fwd()


@pytest.mark.parametrize("name,bad,msg", [
    ("a_q", torch.zeros(1, 8, dtype=torch.float32), "a_q"),                   # [B,T] instead of [B,T,Hkv]
    ("alpha", torch.zeros(2, dtype=torch.bfloat16), "alpha"),                 # wrong element type
    ("v", torch.zeros(1, 8, 2, 32, dtype=torch.bfloat16), "v"),               # half the head dim
    ("g", torch.zeros(1, 8, 4, 64, dtype=torch.float32), "g"),                # other activation type
    ("k", torch.zeros(1, 7, 2, 64, dtype=torch.bfloat16), "k: shape"),        # T differs from q
])
def test_binding_refuses_undersized_or_mistyped_prefill_arguments(lib, name, bad, msg):
    with pytest.raises(ValueError, match=msg):
        _call_fwd(**{name: bad})


def test_binding_refuses_bad_cache_and_decode_arguments(lib):
    c = ua.Cache.empty(2, 2, 64, 40, torch.bfloat16, device="cpu")
    f = torch.float32
    q = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    kv = torch.zeros(2, 2, 64, dtype=torch.bfloat16)
    a = torch.zeros(2, 2, dtype=f)
    ab = torch.zeros(2, dtype=f)
    with pytest.raises(ValueError, match="CUDA tensors"):          # well formed
        ua.decode_step(c, q, kv, kv, q, a, a, ab, ab, 40, 0.1)
    with pytest.raises(ValueError, match="evict_bits"):
        ua.decode_step(c, q, kv, kv, q, a, a, ab, ab, 40, 0.1, evict_bits=torch.zeros(2, 2, 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="kept_idx"):
        ua.decode_step(c, q, kv, kv, q, a, a, ab, ab, 40, 0.1, kept_idx=torch.zeros(2, 2, 40, dtype=torch.int64))
    with pytest.raises(ValueError, match="q: shape"):
        ua.decode_step(c, torch.zeros(3, 4, 64, dtype=torch.bfloat16), kv, kv, q, a, a, ab, ab, 40, 0.1)
    with pytest.raises(ValueError, match="a_k"):
        ua.decode_step(c, q, kv, kv, q, a, torch.zeros(2, dtype=f), ab, ab, 40, 0.1)
    with pytest.raises(ValueError, match="keep"):
        ua.cache_compact(c, keep=torch.zeros(2, 2, 40, dtype=torch.int32))
    with pytest.raises(ValueError, match="k: shape"):
        ua.cache_fill(c, torch.zeros(2, 10, 2, 128, dtype=torch.bfloat16), kv, a, a)
    c.bias = torch.zeros(2, 2, 40, dtype=torch.float64)
    with pytest.raises(ValueError, match="cache.bias"):
        ua.cache_compact(c, 0.1)


def test_binding_refuses_cache_tensors_it_cannot_pass_as_device_pointers(lib):
    # every cache field goes through the same device / contiguity check as the other arguments
    c = ua.Cache.empty(2, 2, 64, 40, torch.bfloat16, device="cpu")
    with pytest.raises(ValueError, match="CUDA tensors"):
        c.struct()
    # a field on another device than the rest of the cache (meta stands in for a second GPU)
    c.rk = torch.zeros(2, 2, 40, dtype=torch.float32, device="meta")
    with pytest.raises(ValueError, match="cache.rk: on meta"):
        c.struct()


def test_binding_refuses_arguments_on_another_device(lib):
    a = _prefill_args()
    with pytest.raises(ValueError, match="v: on meta"):
        ua.prefill_fwd(a["q"], a["k"], a["v"].to("meta"), a["g"], a["a_q"], a["a_k"], a["alpha"], a["beta"])


def test_binding_constants_match_the_header():
    txt = open(os.path.join(ROOT, "include", "ua.h")).read()
    defines = {n: int(v) for n, v in re.findall(r"#define\s+(UA_[A-Z_]+)\s+(\d+)", txt)}
    assert defines["UA_VAR_NO_QUERY_DECAY"] == ua.VAR_NO_QUERY_DECAY
    assert defines["UA_VAR_NO_KEY_DECAY"] == ua.VAR_NO_KEY_DECAY
    assert defines["UA_VAR_NO_SIM_DECAY"] == ua.VAR_NO_SIM_DECAY
    assert defines["UA_VAR_QUERY_NORM"] == ua.VAR_QUERY_NORM
    assert defines["UA_VAR_PER_HEAD_DECAY"] == ua.VAR_PER_HEAD_DECAY
    assert defines["UA_DECODE_DEFER_COMPACT"] == ua.DECODE_DEFER_COMPACT
    assert re.search(r"UA_F32\s*=\s*0", txt) and re.search(r"UA_BF16\s*=\s*1", txt)
    assert (ua.UA_F32, ua.UA_BF16) == (0, 1)
    # the shape struct's fields, in order, as the binding lays them out
    body = re.search(r"typedef struct \{([^{}]*)\} ua_shape;", re.sub(r"/\*.*?\*/", "", txt, flags=re.S), re.S).group(1)
    fields = re.findall(r"(\w+)\s*[,;]", body)
    assert fields == [f for f, _ in ua.ua_shape._fields_], fields
    body = re.search(r"typedef struct \{([^{}]*)\} ua_cache;", re.sub(r"/\*.*?\*/", "", txt, flags=re.S), re.S).group(1)
    fields = re.findall(r"(\w+)\s*[,;]", body)
    assert fields == [f for f, _ in ua.ua_cache._fields_], fields


def test_bwd_band_stats_host_logic(lib):
    """ua_prefill_bwd_band_stats: argument checks, and the band's step count for problems that
    run the fp32 SIMT backward (no device access: it walks the whole band)."""
    steps, walked = ctypes.c_ulonglong(7), ctypes.c_ulonglong(7)
    s = _shape(B=2, T=300, H=4, Hkv=2, d=64, dtype=ua.UA_F32)
    assert lib.ua_prefill_bwd_band_stats(ctypes.byref(s), None, 0, ctypes.byref(steps), ctypes.byref(walked),
                                         None) == 0
    nkt = (300 + 127) // 128                   # key tile kt meets 32-row steps 4kt .. 4nkt-1
    assert steps.value == 2 * 2 * sum(4 * nkt - 4 * kt for kt in range(nkt))
    assert walked.value == steps.value
    assert lib.ua_prefill_bwd_band_stats(ctypes.byref(s), None, 0, None, ctypes.byref(walked), None) == 1
    assert lib.ua_prefill_bwd_band_stats(None, None, 0, ctypes.byref(steps), ctypes.byref(walked), None) == 1
    # training is dense: a pruning threshold is refused
    pr = _shape(prune_p=0.15)
    assert lib.ua_prefill_bwd_band_stats(ctypes.byref(pr), None, 0, ctypes.byref(steps), ctypes.byref(walked),
                                         None) == 1
    # the tensor-core backward needs the workspace it ran on, whole
    tc = _shape(B=1, T=300, H=4, Hkv=1, d=64, dtype=ua.UA_BF16)
    assert lib.ua_prefill_bwd_band_stats(ctypes.byref(tc), None, 0, ctypes.byref(steps), ctypes.byref(walked),
                                         None) == 1
    need = ctypes.c_size_t(0)
    assert lib.ua_prefill_bwd_workspace_size(ctypes.byref(tc), ctypes.byref(need)) == 0
    assert lib.ua_prefill_bwd_band_stats(ctypes.byref(tc), ctypes.c_void_p(FAKE), ctypes.c_size_t(need.value - 1),
                                         ctypes.byref(steps), ctypes.byref(walked), None) == 4   # UA_ERR_WORKSPACE
