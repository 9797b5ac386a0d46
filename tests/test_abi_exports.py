"""The C ABI library loads and exports every symbol include/sigattn.h declares; argument
checks answer without touching a GPU (CPU only: no compute call is made)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sigattn.h")
LIB = os.path.join(ROOT, "padded_variable_length_b200", "libsigattn.so")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SIGATTN_API\s+(?:const\s+)?\w+\**\s+\**(sigattn_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from padded_variable_length_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in sigattn.h but not exported"


def test_error_strings_and_version(lib):
    lib.sigattn_error_string.restype = ctypes.c_char_p
    for code in range(0, -9, -1):
        s = lib.sigattn_error_string(code)
        assert s and s != b"unknown error code"
    assert lib.sigattn_error_string(-99) == b"unknown error code"
    assert lib.sigattn_version() >= 100


def test_argument_checks_without_device(lib):
    P = ctypes.c_void_p
    out = P()
    # null inputs / out pointers are rejected before any CUDA call
    assert lib.sigattn_plan_from_lengths(None, 4, 128, None, ctypes.byref(out)) == -1
    assert lib.sigattn_plan_from_lengths(P(16), 4, 128, None, None) == -1
    assert lib.sigattn_plan_from_lengths(P(16), 0, 128, None, ctypes.byref(out)) == -1
    assert lib.sigattn_plan_from_mask(None, 1, 8, 8, 64, 8, None, ctypes.byref(out)) == -1
    assert lib.sigattn_plan_from_mask(P(16), 1, 8, 8, -1, 8, None, ctypes.byref(out)) == -1
    strides = (ctypes.c_int64 * 3)(0, 0, 0)
    lib.sigattn_fwd.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                P, P, P, P, P, P, P, ctypes.c_int64, P, P, P, P]
    assert lib.sigattn_fwd(None, 0, 1, 64, 0.125, P(16), strides, P(16), strides, P(16), strides,
                           None, 0, P(16), strides, None, None) == -1
    lib.sigattn_plan_get_sizes.argtypes = [P, P]
    assert lib.sigattn_plan_get_sizes(None, None) == -1
    lib.sigattn_plan_destroy.argtypes = [P]
    lib.sigattn_plan_destroy(None)  # safe on NULL
    lib.sigattn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    assert lib.sigattn_set_wait_limit_ns(0) == -1
    assert lib.sigattn_set_wait_limit_ns(2_000_000_000) == 0
    lib.sigattn_bias_from_counts.argtypes = [P, ctypes.c_int64, P, P]
    assert lib.sigattn_bias_from_counts(None, 5, None, None) == -1
    assert lib.sigattn_bias_from_counts(None, 0, None, None) == 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The Python binding raises at import when the library is absent (no CPU fallback)."""
    import importlib.util
    src = os.path.join(ROOT, "padded_variable_length_b200", "binding.py")
    pkg = tmp_path / "fakepkg"
    pkg.mkdir()
    (pkg / "binding.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("fakepkg.binding", pkg / "binding.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_more_argument_checks_without_device(lib):
    P = ctypes.c_void_p
    strides = (ctypes.c_int64 * 3)(0, 0, 0)
    lib.sigattn_last_cuda_error.restype = ctypes.c_char_p
    assert lib.sigattn_last_cuda_error() == b"no CUDA error"
    bwd_args = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float] + [P, P] * 5 + \
        [P, ctypes.c_int64, P, P] + [P, P] * 3
    lib.sigattn_bwd.argtypes = bwd_args + [P]
    lib.sigattn_bwd_ex.argtypes = bwd_args + [ctypes.c_int, P]
    t = [P(16), strides] * 5
    tail = [None, 0, None, None] + [P(16), strides] * 3
    # no plan
    assert lib.sigattn_bwd(None, 0, 1, 64, 0.125, *t, *tail, None) == -1
    # a plan pointer that is never dereferenced: the part mask and the epilogue are checked
    # first, the head dimension next
    assert lib.sigattn_bwd_ex(P(16), 0, 1, 64, 0.125, *t, *tail, 0, None) == -1
    assert lib.sigattn_bwd_ex(P(16), 0, 1, 64, 0.125, *t, *tail, 8, None) == -1
    assert lib.sigattn_bwd_ex(P(16), 3, 1, 64, 0.125, *t, *tail, 7, None) == -1
    assert lib.sigattn_bwd_ex(P(16), 0, 1, 96, 0.125, *t, *tail, 7, None) == -2
    # softmax modes need LSE and the D workspace
    assert lib.sigattn_bwd_ex(P(16), 1, 1, 64, 0.125, *t, *tail, 7, None) == -1
    # the allocation-free form rejects a missing plan the same way
    lib.sigattn_bwd_noalloc.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_float] + [P, P] * 5 + [P, ctypes.c_int64, P] + \
        [P, P] * 3 + [P]
    assert lib.sigattn_bwd_noalloc(None, 0, 1, 64, 0.125, *t, None, 0, None,
                                   *([P(16), strides] * 3), None) == -1
