"""CPU checks of the C-ABI library: it builds for sm_100a, loads, exports every function
include/rolaq.h declares, and rejects bad arguments on the host (no kernel launches)."""
import ctypes
import math
import subprocess

import numpy as np
import pytest

from decode_attention_rotate_b200 import build as B
from decode_attention_rotate_b200 import rolaq as R
from oracle import rolaq_oracle as O


@pytest.fixture(scope="module")
def lib():
    B.build()
    return R.lib()


def test_exports_every_declared_function(lib):
    names = R.header_functions()
    assert "rolaq_decode_attn" in names and "rolaq_quantize_append" in names
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)


def test_version_and_strerror(lib):
    assert R.version() == 100
    assert "workspace" in R.strerror(-2)
    assert R.strerror(12345) == "unknown error"


def test_layer_params_levels_match_oracle(lib):
    for tau in (0.85, 0.9816, 1.1):
        p = R.layer_params_init(tau, 1.16)
        a, b = O.levels(tau)
        assert p.level_a == pytest.approx(a, rel=1e-7)
        assert p.level_b == pytest.approx(b, rel=1e-7)
        assert p.level_a == float(ctypes.c_float(a).value)
    with pytest.raises(R.RolaqError):
        R.layer_params_init(0.0, 1.0)
    with pytest.raises(R.RolaqError):
        R.layer_params_init(1.0, float("nan"))


def _cache(**kw):
    c = R.rolaq_cache()
    c.pages_dev = kw.get("pages", 1 << 20)
    c.num_pages = kw.get("num_pages", 4)
    c.page_table_dev = kw.get("pt", 1 << 21)
    c.batch = kw.get("batch", 2)
    c.max_pages_per_seq = kw.get("max_pages", 2)
    c.prot_dev = kw.get("prot", None)
    c.n_sink = kw.get("n_sink", 0)
    c.n_recent = kw.get("n_recent", 0)
    return c


def test_coupled_gain_matches_oracle(lib):
    """rolaq_coupled_gain against the oracle's coupled gain over the learned threshold
    range 0.85-1.1 (RoLaQ §C.3) and at the Lloyd-Max threshold (gain 1.1331, response at
    gain 1 about 0.88, §B.3); invalid thresholds are refused."""
    for tau in np.linspace(0.85, 1.1, 11):
        tau32 = float(np.float32(tau))
        g, k = R.coupled_gain(tau32)
        assert abs(g - O.coupled_gain(tau32)) < 1e-12
        assert abs(k - O.response(tau32, 1.0)) < 1e-12
    g, k = R.coupled_gain(0.9816)
    assert abs(g - 1.1331) < 1e-4 and abs(k - 0.8825) < 1e-4
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(R.RolaqError):
            R.coupled_gain(bad)


def test_decode_argument_errors(lib):
    p = R.rolaq_layer_params(0.9, 1.0, 0.45, 1.5)
    ptr = 1 << 22
    def call(cache, heads=16, batch=2, ws=1 << 30, q=ptr):
        return lib.rolaq_decode_attn(ctypes.byref(cache), ctypes.byref(p), q, ptr, ptr, batch, heads,
                                     0.07, ptr, ptr, ptr, ws, None)
    assert call(_cache(pages=None)) == -1
    assert call(_cache(pages=(1 << 20) + 8)) == -1          # misaligned pool
    assert call(_cache(), heads=24) == -4
    assert call(_cache(), heads=0) == -4
    assert call(_cache(), batch=3) == -1                     # more requests than the cache
    assert call(_cache(), ws=16) == -2
    assert call(_cache(), q=None) == -1
    assert call(_cache(n_sink=4)) == -1                      # protection without a side store
    bad = R.rolaq_layer_params(0.9, 1.0, 1.5, 0.45)          # levels out of order
    assert lib.rolaq_decode_attn(ctypes.byref(_cache()), ctypes.byref(bad), ptr, ptr, ptr, 2, 16, 0.07,
                                 ptr, ptr, ptr, 1 << 30, None) == -1


def test_quantize_argument_errors(lib):
    p = R.rolaq_layer_params(0.9, 1.0, 0.45, 1.5)
    ptr = 1 << 22
    def call(cache, n=10, c=ptr, seq=ptr):
        return lib.rolaq_quantize_append(ctypes.byref(cache), ctypes.byref(p), ptr, c, ptr, ptr, ptr, seq, n, None)
    assert call(_cache(), n=-1) == -1
    assert call(_cache(), n=0) == 0
    assert call(_cache(), c=None) == -1
    assert call(_cache(), c=ptr + 2) == -1
    assert call(_cache(n_recent=8, prot=ptr), seq=None) == -1


def test_workspace_bytes_shape_rules(lib):
    assert lib.rolaq_decode_workspace_bytes(4, 24) == 0
    assert lib.rolaq_decode_workspace_bytes(0, 16) == 0
    n16 = lib.rolaq_decode_workspace_bytes(4, 16)
    assert n16 > 0 and n16 % 16 == 0
    # (one work item per SM + one per request) x heads x (512 fp32 partial + (m, l))
    per_item_head = 512 * 4 + 8
    assert n16 % (16 * per_item_head) == 0
    sms = n16 // (16 * per_item_head) - 4
    assert sms >= 1
    for b, h in [(1, 16), (32, 128), (7, 48), (1000, 32)]:
        assert lib.rolaq_decode_workspace_bytes(b, h) == (sms + b) * h * per_item_head


def test_projection_argument_errors(lib):
    """Bad pointers and sizes are rejected before any launch; batch == 0 is a no-op."""
    ptr = 1 << 22
    fw = lambda a=ptr, b=ptr, r=ptr, h=16, q=ptr, o=ptr: lib.rolaq_fold_weights(a, b, r, h, q, o, None)
    assert fw(a=None) == -1 and fw(r=None) == -1 and fw(o=None) == -1
    assert fw(h=0) == -1 and fw(h=-3) == -1
    assert fw(b=ptr + 2) == -1                                 # fp32 operand not 4-byte aligned
    fq = lambda q=ptr, w=ptr, b=2, h=16, o=ptr: lib.rolaq_fold_query(q, w, b, h, o, None)
    assert fq(q=None) == -1 and fq(o=None) == -1 and fq(b=-1) == -1 and fq(h=0) == -1
    assert fq(q=ptr + 1) == -1                                 # bf16 operand not 2-byte aligned
    assert fq(b=0) == 0 and fq(b=0, q=None, o=None) == 0
    uo = lambda o=ptr, w=ptr, b=2, h=16, v=ptr: lib.rolaq_unfold_output(o, w, b, h, v, None)
    assert uo(o=None) == -1 and uo(v=None) == -1 and uo(b=-1) == -1 and uo(h=0) == -1
    assert uo(w=ptr + 2) == -1
    assert uo(b=0) == 0 and uo(b=0, o=None, v=None) == 0


def test_static_decode_rejects_before_any_launch(lib):
    """The static-scratch decode sizes its plan on the host: shapes it cannot hold fail
    with ROLAQ_ENOSPACE (and unsupported shapes with their own codes) before any CUDA call."""
    p = R.rolaq_layer_params(0.9, 1.0, 0.45, 1.5)
    ptr = 1 << 22
    def call(batch, heads):
        c = _cache(batch=max(batch, 1))
        return lib.rolaq_decode_attn_static(ctypes.byref(c), ctypes.byref(p), ptr, ptr, ptr, batch, heads,
                                            0.07, ptr, ptr, None)
    assert call(2, 24) == -4                  # heads not a multiple of 16
    assert call(2, 0) == -4
    assert call(0, 16) == -1
    # 32 MiB / (128 heads x 2,056 B) = 127 items: 127 requests leave no room for a split
    assert call(127, 128) == -2
    assert call(5000, 16) == -2               # 1,020 items at 16 heads
    # the shared argument checks come first: a batch beyond the cache, a null cache or a
    # null output give ROLAQ_EINVAL even where the scratch could not hold the plan
    c = _cache(batch=4)
    assert lib.rolaq_decode_attn_static(ctypes.byref(c), ctypes.byref(p), ptr, ptr, ptr, 5000, 16,
                                        0.07, ptr, ptr, None) == -1
    assert lib.rolaq_decode_attn_static(None, ctypes.byref(p), ptr, ptr, ptr, 5000, 16,
                                        0.07, ptr, ptr, None) == -1
    c = _cache(batch=5000)
    assert lib.rolaq_decode_attn_static(ctypes.byref(c), ctypes.byref(p), ptr, ptr, ptr, 5000, 16,
                                        0.07, None, ptr, None) == -1


def test_append_decode_rejects_before_any_launch(lib):
    """The fused append + decode checks its extra pointers and its larger workspace on the
    host, after the decode's own checks, before any CUDA call."""
    p = R.rolaq_layer_params(0.9, 1.0, 0.45, 1.5)
    ptr = 1 << 22
    need = lib.rolaq_decode_append_workspace_bytes(2, 16)
    assert need == lib.rolaq_decode_workspace_bytes(2, 16) + 2 * 512 * 4
    assert lib.rolaq_decode_append_workspace_bytes(2, 24) == 0
    assert lib.rolaq_decode_append_workspace_bytes(0, 16) == 0

    def call(Rs=ptr, c=ptr, k=ptr, ws=ptr, nbytes=need, batch=2, heads=16, cache=None):
        cd = cache if cache is not None else _cache(batch=2)
        return lib.rolaq_decode_attn_append(ctypes.byref(cd), ctypes.byref(p), Rs, c, k, ptr, ptr, ptr, batch,
                                            heads, 0.07, ptr, ptr, ws, nbytes, None)
    assert call(Rs=None) == -1 and call(c=None) == -1 and call(k=None) == -1
    assert call(c=ptr + 2) == -1 and call(k=ptr + 8) == -1 and call(Rs=ptr + 4) == -1
    assert call(heads=24) == -4
    assert call(batch=3) == -1                                  # beyond the cache's batch
    assert call(ws=None) == -1
    # enough for the plain decode but not for the new tokens' coordinates
    assert call(nbytes=lib.rolaq_decode_workspace_bytes(2, 16)) == -2


def test_bf16_decode_rejects_before_any_launch(lib):
    """The BF16 decode needs a side store whose windows are multiples of 64 tokens."""
    p = R.rolaq_layer_params(0.9, 1.0, 0.45, 1.5)
    ptr = 1 << 22
    need = lib.rolaq_decode_workspace_bytes(2, 16)

    def call(**kw):
        c = _cache(batch=2, **kw)
        return lib.rolaq_decode_attn_bf16(ctypes.byref(c), ctypes.byref(p), ptr, ptr, ptr, 2, 16, 0.07, ptr, ptr,
                                          ptr, need, None)
    assert call() == -1                                      # no side store
    assert call(prot=ptr, n_sink=4, n_recent=128) == -4      # sink window not a multiple of 64
    assert call(prot=ptr, n_sink=0, n_recent=100) == -4
    c = _cache(batch=2, prot=ptr, n_recent=128)
    assert lib.rolaq_decode_attn_bf16(ctypes.byref(c), ctypes.byref(p), ptr, ptr, ptr, 2, 24, 0.07, ptr, ptr,
                                      ptr, need, None) == -4     # heads not a multiple of 16
    assert lib.rolaq_decode_attn_bf16(ctypes.byref(c), ctypes.byref(p), ptr, ptr, ptr, 2, 16, 0.07, ptr, ptr,
                                      ptr, need - 16, None) == -2
