"""Host-only checks of the C-ABI library (no GPU needed).

* libdq.so builds, loads and exports every entry point include/dq.h declares;
* argument validation rejects bad input before touching any device;
* the layer's host plumbing (status strings, version).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dq.h")


@pytest.fixture(scope="module")
def libdq():
    from quantized_gemm_token_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def _declared():
    text = open(HEADER).read()
    return re.findall(r"^DQ_API\s+[\w\s\*]+?\b(dq_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_layer():
    names = set(_declared())
    for n in ("dq_quantize_rows", "dq_int8_linear", "dq_bsr_int8_linear", "dq_sync_status",
              "dq_quantize_weight", "dq_bsr_pack", "dq_bsr_validate", "dq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(libdq):
    missing = [n for n in _declared() if not hasattr(libdq, n)]
    assert not missing, missing


def test_status_strings(libdq):
    libdq.dq_status_string.restype = ctypes.c_char_p
    for s in range(5):
        assert libdq.dq_status_string(s).startswith(b"DQ_")
    assert libdq.dq_status_string(99) == b"unknown dq_status"
    assert libdq.dq_version() == 100


def _i64(*v):
    return [ctypes.c_int64(x) for x in v]


def test_argument_validation_without_device(libdq):
    P = ctypes.c_void_p
    fake = P(0x1000)   # never dereferenced: validation fails first
    # bad out dtype
    assert libdq.dq_int8_linear(fake, fake, *_i64(4, 64), fake, fake, ctypes.c_int64(64), None, fake,
                                ctypes.c_int(7), None, ctypes.c_size_t(0), None) == 1
    # negative M
    assert libdq.dq_int8_linear(fake, fake, *_i64(-1, 64), fake, fake, ctypes.c_int64(64), None, fake,
                                ctypes.c_int(0), None, ctypes.c_size_t(0), None) == 1
    # K not a multiple of 16, N not a multiple of 8, K above the int32 bound
    for M, K, N in ((4, 40, 64), (4, 64, 60), (4, 133152, 64)):
        assert libdq.dq_int8_linear(fake, fake, *_i64(M, K), fake, fake, ctypes.c_int64(N), None, fake,
                                    ctypes.c_int(0), None, ctypes.c_size_t(0), None) == 2
    # null pointers
    assert libdq.dq_int8_linear(None, fake, *_i64(4, 64), fake, fake, ctypes.c_int64(64), None, fake,
                                ctypes.c_int(0), None, ctypes.c_size_t(0), None) == 1
    # misaligned A
    assert libdq.dq_int8_linear(P(0x1001), fake, *_i64(4, 64), fake, fake, ctypes.c_int64(64), None, fake,
                                ctypes.c_int(0), None, ctypes.c_size_t(0), None) == 2
    # quantize: ldx < K, K < 1
    assert libdq.dq_quantize_rows(fake, *_i64(4, 64, 32), fake, ctypes.c_int64(64), fake, None) == 1
    assert libdq.dq_quantize_rows(fake, *_i64(4, 0, 0), fake, ctypes.c_int64(0), fake, None) == 1
    # BSR: N, K not multiples of 64; negative nnzb
    assert libdq.dq_bsr_int8_linear(fake, fake, *_i64(4, 96, 64), fake, fake, fake, ctypes.c_int64(1),
                                    fake, None, fake, ctypes.c_int(0), None) == 2
    assert libdq.dq_bsr_int8_linear(fake, fake, *_i64(4, 64, 64), fake, fake, fake, ctypes.c_int64(-1),
                                    fake, None, fake, ctypes.c_int(0), None) == 1
    assert libdq.dq_bsr_pack(fake, *_i64(64, 100), fake, fake, ctypes.c_int64(1), fake, None) == 2


def test_binding_refuses_to_run_without_library(tmp_path, monkeypatch):
    # The binding has no fallback: with the library missing every call raises.
    import quantized_gemm_token_b200 as pkg
    monkeypatch.setattr(pkg, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        pkg._load()
    try:
        pkg._load()
    except ImportError as e:
        missing = pkg._MissingLibrary(e)
    monkeypatch.setattr(pkg, "lib", missing)
    with pytest.raises(ImportError):
        pkg.dq_version()
    with pytest.raises(ImportError):
        pkg.dq_sync_status(0)
