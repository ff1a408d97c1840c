"""The C-ABI library loads and exports every entry point include/hca.h declares; host-side
argument checks reject bad calls before any launch.  CPU only (no CUDA call reaches a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from compressed_long_context_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "hca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return sorted(set(re.findall(r"\b(hca_[a-z_]+)\s*\(", text)))


def test_header_lists_the_binding_exports():
    assert declared_functions() == sorted(_lib.EXPORTS)


def declared_param_counts():
    text = open(os.path.join(ROOT, "include", "hca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(hca_[a-z_]+)\s*\(([^)]*)\)\s*;", text):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_header(libhca):
    counts = declared_param_counts()
    assert set(counts) == set(_lib.EXPORTS)
    for name, n in counts.items():
        assert len(getattr(libhca, name).argtypes) == n, name


def test_library_exports_every_declared_symbol(libhca):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name
        assert getattr(libhca, name) is not None


def test_status_strings(libhca):
    for code in range(7):
        s = libhca.hca_status_string(code).decode()
        assert s.startswith("HCA_")
    assert b"unknown" in libhca.hca_status_string(99)


def test_compress_rejects_before_launch(libhca):
    p = ctypes.c_void_p(16)
    # unsupported head dim
    assert libhca.hca_compress(p, p, None, p, p, 1, 256, 1, 96, 64, 128, None) == _lib.HCA_ERR_UNSUPPORTED
    # block larger than 128
    assert libhca.hca_compress(p, p, None, p, p, 1, 256, 1, 64, 64, 129, None) == _lib.HCA_ERR_UNSUPPORTED
    # null pointers / bad sizes
    assert libhca.hca_compress(None, p, None, p, p, 1, 256, 1, 64, 64, 128, None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_compress(p, p, None, p, p, -1, 256, 1, 64, 64, 128, None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_compress(p, p, None, p, p, 1, 256, 0, 64, 64, 128, None) == _lib.HCA_ERR_INVALID_ARG
    # misaligned pointer
    q = ctypes.c_void_p(18)
    assert libhca.hca_compress(q, p, None, p, p, 1, 256, 1, 64, 64, 128, None) == _lib.HCA_ERR_INVALID_ARG
    # nothing to do: no launch, OK
    assert libhca.hca_compress(None, None, None, None, None, 1, 100, 1, 64, 64, 128, None) == _lib.HCA_OK


def test_prefill_rejects_before_launch(libhca):
    p = ctypes.c_void_p(16)
    # (q, k, v, kc, vc, out, lse, B, T, Hq, Hkv, d, dv, blk, W, scale, flags, stream)
    # unsupported head dims, block, group size, flags
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 96, 96, 128, 128, 0.1, 0,
                              None) == _lib.HCA_ERR_UNSUPPORTED
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 64, 512, 128, 128, 0.1, 0,
                              None) == _lib.HCA_ERR_UNSUPPORTED
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 64, 64, 129, 128, 0.1, 0,
                              None) == _lib.HCA_ERR_UNSUPPORTED
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 6, 2, 64, 64, 128, 128, 0.1, 0,
                              None) == _lib.HCA_ERR_UNSUPPORTED
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 64, 64, 128, 128, 0.1, 1 << 8,
                              None) == _lib.HCA_ERR_UNSUPPORTED
    # null pointers, bad sizes, NaN scale, LSE requested without a buffer
    assert libhca.hca_prefill(None, p, p, p, p, p, None, 1, 256, 4, 1, 64, 64, 128, 128, 0.1, 0,
                              None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 64, 64, 128, 0, 0.1, 0,
                              None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 64, 64, 128, 128, float("nan"), 0,
                              None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_prefill(p, p, p, p, p, p, None, 1, 256, 4, 1, 64, 64, 128, 128, 0.1,
                              _lib.HCA_WRITE_LSE, None) == _lib.HCA_ERR_INVALID_ARG
    # nothing to do: no launch, OK
    assert libhca.hca_prefill(None, None, None, None, None, None, None, 0, 256, 4, 1, 512, 512, 128, 128,
                              0.1, 0, None) == _lib.HCA_OK
