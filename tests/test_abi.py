"""The C-ABI library builds, loads and exports every entry point include/arl2.h declares.

No compute calls: these run on machines without a GPU.
"""
import ctypes
import os
import re

import pytest

from softmax_attention_ar_b200 import arl2, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "arl2.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(arl2_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return arl2.load_library()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["arl2_create", "arl2_set_feature_maps", "arl2_frame_query", "arl2_frame_commit", "arl2_reset",
              "arl2_get_state", "arl2_set_state", "arl2_get_status", "arl2_memory_bytes", "arl2_destroy"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    assert sorted(arl2.SIGNATURES) == _declared()


def test_argument_checks_need_no_gpu(lib):
    # These fail in the argument checks, before any CUDA call.
    assert lib.arl2_create(12, 1560, 128, 128, 1, None) == arl2.ARL2_ERR_INVALID_ARG
    out = ctypes.c_void_p()
    assert lib.arl2_create(0, 1560, 128, 128, 1, ctypes.byref(out)) == arl2.ARL2_ERR_INVALID_ARG
    assert not out.value
    assert lib.arl2_create(12, 1560, 128, 64, 1, ctypes.byref(out)) == arl2.ARL2_ERR_UNSUPPORTED
    assert lib.arl2_create(12, 4097, 128, 128, 1, ctypes.byref(out)) == arl2.ARL2_ERR_UNSUPPORTED
    assert lib.arl2_create(12, 1560, 96, 96, 1, ctypes.byref(out)) == arl2.ARL2_ERR_UNSUPPORTED
    assert lib.arl2_frame_query(None, None, None, None, None, None) == arl2.ARL2_ERR_INVALID_ARG
    assert lib.arl2_frame_commit(None, None, None, None, None, None) == arl2.ARL2_ERR_INVALID_ARG
    assert lib.arl2_reset(None, None) == arl2.ARL2_ERR_INVALID_ARG
    assert lib.arl2_get_status(None) == arl2.ARL2_ERR_INVALID_ARG
    assert lib.arl2_memory_bytes(None) == 0
    assert lib.arl2_frame_index(None) == -1
    lib.arl2_destroy(None)
    assert lib.arl2_kvcache_create(12, 1560, 128, 1, 0, ctypes.byref(out)) == arl2.ARL2_ERR_INVALID_ARG
    lib.arl2_kvcache_destroy(None)
    # The allocation-free commit has no context to report a time-out through, so its status
    # word is required; a missing one is refused before any CUDA call.
    p = 1 << 20   # an aligned address; never dereferenced by the argument checks
    assert lib.arl2_frame_commit_noalloc(1, 12, 1560, 128, p, p, p, p, p, p, p, p, None, None) == \
        arl2.ARL2_ERR_INVALID_ARG


def test_built_for_sm100a_only():
    log = open(os.path.join(build.BUILD_DIR, "ptxas.log")).read()
    assert "arch=compute_100a,code=sm_100a" in log
    assert "for 'sm_100a'" in log
    assert "spill stores" in log and not re.search(r"[1-9]\d* bytes spill stores", log)


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "softmax_attention_ar_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), f
                assert "arl2_oracle" not in src, f


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(arl2, "_lib", None)
    with pytest.raises(ImportError):
        arl2.load_library(str(tmp_path / "libarl2.so"))
