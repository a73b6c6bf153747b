"""The C ABI without a GPU: libzha.so loads, exports every function include/zha.h declares,
and its host-only paths (validation, layouts, sizes) behave as documented."""
import ctypes
import os
import re
import subprocess

import pytest

import tree_indexed_sparse_03_b200 as z
from tree_indexed_sparse_03_b200 import zha as zb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zha.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"ZHA_API\s+[\w\s\*]+?\b(zha_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def built():
    from tree_indexed_sparse_03_b200 import build_lib
    build_lib.build()
    return z.lib()


def test_header_declares_the_boundary():
    fns = declared_functions()
    for name in ["zha_tree_bytes", "zha_tree_create", "zha_tree_build", "zha_tree_append", "zha_decode",
                 "zha_dense_decode", "zha_last_error", "zha_tree_destroy"]:
        assert name in fns


def test_every_declared_symbol_is_exported(built):
    out = subprocess.run(["nm", "-D", "--defined-only", z.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (zha_\w+)", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(built, f)
    assert set(zb._SIGS) == set(declared_functions())


def cfg(**kw):
    base = dict(d=128, n_q_heads=32, n_kv_heads=4, block=4, levels=6, n_refs=16, p=0.95, dtype="bf16",
                capacity=262144, max_batch=1)
    base.update(kw)
    return z.make_config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), zb.ZHA_ERR_UNSUPPORTED),
    (dict(n_q_heads=30), zb.ZHA_ERR_UNSUPPORTED),
    (dict(block=1), zb.ZHA_ERR_UNSUPPORTED),
    (dict(levels=0), zb.ZHA_ERR_UNSUPPORTED),
    (dict(n_refs=33), zb.ZHA_ERR_UNSUPPORTED),
    (dict(n_refs=0), zb.ZHA_ERR_UNSUPPORTED),
    (dict(p=0.0), zb.ZHA_ERR_INVALID),
    (dict(p=1.5), zb.ZHA_ERR_INVALID),
    (dict(p=float("nan")), zb.ZHA_ERR_INVALID),
    (dict(capacity=0), zb.ZHA_ERR_INVALID),
    (dict(capacity=2 ** 31), zb.ZHA_ERR_INVALID),
    (dict(max_batch=0), zb.ZHA_ERR_INVALID),
    (dict(block=1024), zb.ZHA_ERR_UNSUPPORTED),
])
def test_invalid_configs(built, kw, code):
    with pytest.raises(z.ZhaError) as e:
        z.tree_bytes(cfg(**kw))
    assert e.value.code == code
    assert z.lib().zha_last_error().decode()


def test_sizes_and_layout(built):
    c = cfg()
    nb, sb = z.tree_bytes(c)
    rb = 16 * 128 * 2 + 64
    prev_end = 0
    total_nodes = 0
    for level in range(1, 7):
        lay = z.tree_layout(c, level)
        assert lay.rec_bytes == rb
        assert lay.cap_nodes == 262144 // 4 ** level
        assert lay.rec_offset % 256 == 0 and lay.f_offset % 256 == 0
        assert lay.rec_offset >= prev_end
        assert lay.f_offset >= lay.rec_offset + 4 * lay.cap_nodes * rb
        prev_end = lay.f_offset + 4 * lay.cap_nodes * 16 * 4
        total_nodes += lay.cap_nodes
    assert nb >= prev_end
    assert sb > 0
    with pytest.raises(z.ZhaError):
        z.tree_layout(c, 7)
    # fp32 records: R*d*4 bytes of slopes then R floats padded to 16 bytes
    lay = z.tree_layout(cfg(dtype="f32", d=64, n_refs=3), 1)
    assert lay.rec_bytes == 3 * 64 * 4 + 16


def test_fp4_router_layout(built):
    """FP4 router records: R*(d/2 + d/16) bytes of codes and scales, then R floats padded to 16 bytes,
    after the key planes; bf16 only; a key-plane configuration has none."""
    c = cfg(planes="fp4")
    nb_fp4, _ = z.tree_bytes(c)
    nb_key, _ = z.tree_bytes(cfg())
    total = 0
    for level in range(1, 7):
        off, rb = z.zha.tree_layout_fp4(c, level)
        assert rb == 16 * (64 + 8) + 64 == 1216
        assert off % 256 == 0 and off >= nb_key
        total += 4 * (262144 // 4 ** level) * rb
    assert nb_fp4 >= nb_key + total
    with pytest.raises(z.ZhaError) as e:
        z.zha.tree_layout_fp4(cfg(), 1)
    assert e.value.code == zb.ZHA_ERR_INVALID
    with pytest.raises(z.ZhaError) as e:
        z.tree_bytes(cfg(planes="fp4", dtype="f32"))
    assert e.value.code == zb.ZHA_ERR_UNSUPPORTED
    bad = cfg()
    bad.planes = 7
    with pytest.raises(z.ZhaError) as e:
        z.tree_bytes(bad)
    assert e.value.code == zb.ZHA_ERR_INVALID


def test_dense_scratch_bytes(built):
    c = cfg()
    assert z.dense_scratch_bytes(c, 1, 262144) > 0
    assert z.dense_scratch_bytes(c, 1, 0) == 0
    assert z.dense_scratch_bytes(cfg(d=96), 1, 10) == 0


def test_null_arguments_fail_before_any_device_work(built):
    L = z.lib()
    c = cfg()
    h = ctypes.c_void_p()
    assert L.zha_tree_create(ctypes.byref(c), None, None, None, None, None, ctypes.byref(h)) == zb.ZHA_ERR_INVALID
    assert L.zha_tree_create(ctypes.byref(c), 16, 16, 16, 256, 256, None) == zb.ZHA_ERR_INVALID
    assert L.zha_tree_build(None, 10, None) == zb.ZHA_ERR_INVALID
    assert L.zha_tree_append(None, None, None, 1, None) == zb.ZHA_ERR_INVALID
    assert L.zha_decode(None, None, None, 1, None, None, None, None, 0, None) == zb.ZHA_ERR_INVALID
    assert L.zha_launch_count() == 0
    assert L.zha_tree_status(None, None) == zb.ZHA_ERR_INVALID
    assert L.zha_tree_set_step_p(None, None, 0) == zb.ZHA_ERR_INVALID
    assert L.zha_tree_size(None) == -1
    assert L.zha_dense_decode(ctypes.byref(c), None, None, 1, 1, None, None, 1, None, None) == zb.ZHA_ERR_INVALID
    L.zha_tree_destroy(None)


def test_binding_refuses_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(zb, "_lib", None)
    monkeypatch.setattr(zb, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        zb.lib()


def _dense_plan(B, hkv, n):
    """The dense decode's split plan (zha_dense.cu, dense_plan): about four CTAs per SM of 148, splits of a
    multiple of 64 keys."""
    s = (148 * 4 + B * hkv - 1) // (B * hkv)
    s = max(1, min(s, (n + 63) // 64))
    per = max(64, ((n + s - 1) // s + 63) // 64 * 64)
    return max(1, (n + per - 1) // per)


@pytest.mark.parametrize("hkv,hq,d,B,n", [(1, 8, 128, 1, 37915), (4, 32, 128, 1, 262144), (2, 16, 64, 3, 5003),
                                          (1, 1, 64, 1, 130)])
def test_dense_scratch_covers_every_smaller_call(built, hkv, hq, d, B, n):
    """One scratch of zha_dense_scratch_bytes(B, n) holds the split partials of every call with B' <= B and
    n' <= n, although the split count itself is not monotone in n."""
    c = cfg(d=d, n_q_heads=hq, n_kv_heads=hkv, levels=1, n_refs=1, capacity=max(n, 64), max_batch=B)
    have = z.dense_scratch_bytes(c, B, n)
    assert have > 0
    worst = 0
    for b in range(1, B + 1):
        for m in list(range(1, min(n, 2048) + 1)) + list(range(max(1, n - 4096), n + 1)):
            worst = max(worst, b * hq * _dense_plan(b, hkv, m) * (d + 2) * 4)
    assert worst <= have, (worst, have)
    # the advisor's case: the plan at n is smaller than at a shorter length
    if (hkv, B, n) == (1, 1, 37915):
        assert _dense_plan(1, 1, 37915) < _dense_plan(1, 1, 37851)
