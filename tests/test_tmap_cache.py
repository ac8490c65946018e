"""Host checks of the tensor-map cache the C ABI keeps in front of the TMA descriptor encoder
(csrc/tmap_cache.h), compiled for the CPU with a fake encoder.  A stale or mixed-up entry would
hand a kernel the descriptor of another tensor, so the tests check that every field of the key
separates entries, that repeated lookups skip the encoder, that replacement keeps the table
correct, that a failed encode is reported and not cached, and that concurrent host threads get
correct values."""
import ctypes
import os
import shutil
import subprocess

import pytest

import causal_attention_sdpa_b200 as ga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc")


@pytest.fixture()
def C(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("tmap") / "libtmap_host.so")
    subprocess.run([cxx, "-std=c++17", "-O1", "-shared", "-fPIC", "-pthread", "-I", CSRC,
                    os.path.join(ROOT, "tests", "tmap_cache_host.cpp"), "-o", out], check=True)
    lib = ctypes.CDLL(out)
    lib.tc_get.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.POINTER(ctypes.c_longlong)]
    lib.tc_expected_word.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.tc_expected_word.restype = ctypes.c_longlong
    lib.tc_clear()
    return lib


def get(C, *key):
    w = ctypes.c_longlong()
    ok = C.tc_get(*key, ctypes.byref(w))
    return w.value if ok else None


def stats(C):
    h, m, u = ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_int()
    C.tc_stats(ctypes.byref(h), ctypes.byref(m), ctypes.byref(u))
    return h.value, m.value, u.value


def test_repeated_lookups_hit(C):
    key = (0x10000, 1, 64, 1024, 768)
    for _ in range(5):
        assert get(C, *key) == C.tc_expected_word(*key)
    assert C.tc_encodes() == 1
    assert stats(C) == (4, 1, 1)


@pytest.mark.parametrize("field", range(5))
def test_every_key_field_separates_entries(C, field):
    a = [0x10000, 1, 64, 1024, 768]
    b = list(a)
    b[field] += 16 if field == 0 else 1
    assert get(C, *a) == C.tc_expected_word(*a)
    assert get(C, *b) == C.tc_expected_word(*b)
    assert C.tc_encodes() == 2
    assert get(C, *a) == C.tc_expected_word(*a) and get(C, *b) == C.tc_expected_word(*b)
    assert C.tc_encodes() == 2


@pytest.mark.parametrize("which", range(3))
def test_every_stride_separates_entries(C, which):
    w0, w1 = ctypes.c_longlong(), ctypes.c_longlong()
    C.tc_get_stride.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_longlong, ctypes.POINTER(ctypes.c_longlong)]
    assert C.tc_get_stride(0x1000, which, 0, ctypes.byref(w0))
    assert C.tc_get_stride(0x1000, which, 8, ctypes.byref(w1))
    assert w0.value != w1.value and C.tc_encodes() == 2


def test_replacement_keeps_values_correct(C):
    keys = [(0x1000 * (i + 1), 1, 64, 128 * (i + 1), 3) for i in range(7)]   # more keys than slots
    for _ in range(3):
        for k in keys:
            assert get(C, *k) == C.tc_expected_word(*k)
    assert stats(C)[2] == 4


def test_failed_encode_is_reported_and_not_cached(C):
    key = (0x20000, 2, 64, 300, 2)
    C.tc_set_fail(1)
    assert get(C, *key) is None
    C.tc_set_fail(0)
    assert stats(C)[2] == 0
    assert get(C, *key) == C.tc_expected_word(*key)
    assert C.tc_encodes() == 1


def test_concurrent_threads_get_correct_values(C):
    assert C.tc_threads(8, 2000) == 0


def test_library_exports_cache_counters():
    from causal_attention_sdpa_b200 import build
    build.build()
    h, m, u = ga.gpt_attn_tmap_cache_stats()
    assert h >= 0 and m >= 0 and 0 <= u <= 64
