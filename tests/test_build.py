"""The in-tree build reuses an object only when it is newer than its source and
every header and was compiled with the current flags, so that a self-checking
build (KV4_DEBUG_CHECKS=1) never leaves its objects in the product library."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_module():
    spec = importlib.util.spec_from_file_location("kv4_build", os.path.join(ROOT, "int4_kv_cache_paged_b200",
                                                                             "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_object_reuse_needs_newer_mtime_and_same_flags(tmp_path):
    b = _build_module()
    src, hdr, obj = tmp_path / "a.cu", tmp_path / "a.cuh", tmp_path / "a.o"
    for p in (src, hdr, obj):
        p.write_text("x")
    os.utime(src, (100, 100))
    os.utime(hdr, (200, 200))
    os.utime(obj, (300, 300))
    assert b.up_to_date(str(obj), [str(src), str(hdr)], True)
    assert not b.up_to_date(str(obj), [str(src), str(hdr)], False)       # other flags
    os.utime(hdr, (400, 400))
    assert not b.up_to_date(str(obj), [str(src), str(hdr)], True)        # a header changed after it
    assert not b.up_to_date(str(tmp_path / "missing.o"), [str(src)], True)


def test_self_checking_build_has_other_flags(monkeypatch):
    b = _build_module()
    monkeypatch.delenv("KV4_DEBUG_CHECKS", raising=False)
    normal = b.flags()
    monkeypatch.setenv("KV4_DEBUG_CHECKS", "1")
    checking = b.flags()
    assert "-DKV4_DEBUG_CHECKS" in checking and "-DKV4_DEBUG_CHECKS" not in normal
    assert " ".join(normal) != " ".join(checking)
    assert "arch=compute_100a,code=sm_100a" in normal
