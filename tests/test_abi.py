"""The C-ABI library builds, loads and exports every symbol include/duolm.h
declares; host-side validation needs no GPU.  No compute calls here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(duolm_[a-z_0-9]+)\s*\(", txt))
    return names


@pytest.fixture(scope="module")
def so():
    from shared_prefix_item_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for required in ["duolm_model_load", "duolm_vid_table_load", "duolm_score", "duolm_last_error",
                     "duolm_destroy"]:
        assert required in names


def test_every_declared_symbol_is_exported(so):
    missing = [n for n in sorted(_declared()) if not hasattr(so, n)]
    assert not missing, missing


def test_binding_loads_and_matches_header():
    import shared_prefix_item_b200 as S
    from shared_prefix_item_b200 import _lib
    src = open(_lib.__file__).read()
    bound = set(re.findall(r'"(duolm_[a-z_0-9]+)"', src))
    assert bound == _declared()
    assert os.path.exists(S.lib_path)


def test_weight_count_and_null_arguments(so):
    from shared_prefix_item_b200._lib import ModelDesc, lib
    d = ModelDesc(28, 1024, 16, 8, 128, 3072, 151936, 1e6, 1e-6, 1)
    assert lib.duolm_weight_count(ctypes.byref(d)) == 1 + 11 * 28 + 2
    assert lib.duolm_weight_count(None) == -1
    out = ctypes.c_void_p(123)
    # invalid descriptor (head_dim 64 on the bf16 path) is rejected before any CUDA call
    bad = ModelDesc(2, 1024, 16, 8, 64, 3072, 151936, 1e6, 1e-6, 1)
    assert lib.duolm_model_load(ctypes.byref(bad), (ctypes.c_void_p * 25)(*([1] * 25)), 0, None,
                                ctypes.byref(out)) == -1
    assert out.value is None
    assert lib.duolm_model_load(None, None, 0, None, ctypes.byref(out)) == -1
    for fn in ["duolm_execute", "duolm_sync", "duolm_debug_wait_timeout"]:
        assert getattr(lib, fn)(None) == -1
    assert lib.duolm_prepare(None, 1, None, None, None, None, 1, 0) == -1
    assert lib.duolm_scores_device(None) is None
    lib.duolm_destroy(None)
