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


def test_decode_rejects_before_launch(libhca):
    p = ctypes.c_void_p(16)
    f = ctypes.c_void_p(32)

    def call(q=p, kc=p, vc=p, table=None, ps=0, maxp=0, npages=0, kw=p, vw=p, seq=p, gq=None, gk=None,
             eps=1e-6, gate=None, out=p, ws=p, ws_bytes=1 << 20, B=1, Hq=64, Hkv=1, d=512, dv=512, blk=128,
             W=128, Nmax=8, scale=0.05, flags=0):
        return libhca.hca_decode(q, kc, vc, table, ps, maxp, npages, kw, vw, seq, gq, gk, eps, gate, out, ws,
                                 ws_bytes, B, Hq, Hkv, d, dv, blk, W, Nmax, scale, flags, None)

    # unsupported head dim, group larger than 64, block larger than 128, unknown flag
    assert call(d=64, dv=64) == _lib.HCA_ERR_UNSUPPORTED
    assert call(Hq=128) == _lib.HCA_ERR_UNSUPPORTED
    assert call(blk=129) == _lib.HCA_ERR_UNSUPPORTED
    assert call(flags=1 << 8) == _lib.HCA_ERR_UNSUPPORTED
    # null or misaligned pointers, bad sizes
    assert call(q=None) == _lib.HCA_ERR_INVALID_ARG
    assert call(kw=ctypes.c_void_p(24)) == _lib.HCA_ERR_INVALID_ARG
    assert call(B=-1) == _lib.HCA_ERR_INVALID_ARG
    assert call(W=0) == _lib.HCA_ERR_INVALID_ARG
    assert call(eps=-1.0) == _lib.HCA_ERR_INVALID_ARG
    # QK normalisation without gains; a gate that is NULL or not 16-byte aligned (read 8 bytes
    # at a time on the device, so a 4-byte-aligned gate must be refused, not faulted on)
    assert call(flags=_lib.HCA_QK_NORM) == _lib.HCA_ERR_INVALID_ARG
    assert call(flags=_lib.HCA_OUT_GATE) == _lib.HCA_ERR_INVALID_ARG
    assert call(flags=_lib.HCA_OUT_GATE, gate=ctypes.c_void_p(20)) == _lib.HCA_ERR_INVALID_ARG
    assert call(flags=_lib.HCA_OUT_GATE, gate=ctypes.c_void_p(24)) == _lib.HCA_ERR_INVALID_ARG
    # paged without a table, a page size that is not a multiple of 64
    assert call(flags=_lib.HCA_PAGED) == _lib.HCA_ERR_INVALID_ARG
    assert call(flags=_lib.HCA_PAGED, table=f, ps=100, maxp=4, npages=4) == _lib.HCA_ERR_INVALID_ARG
    # nothing to do: no launch, OK
    assert call(q=None, kc=None, vc=None, kw=None, vw=None, seq=None, out=None, ws=None, B=0) == _lib.HCA_OK


def test_append_rejects_before_launch(libhca):
    p = ctypes.c_void_p(16)

    def call(k=p, v=p, w=None, seq=p, kw=p, vw=p, kc=p, vc=p, table=None, ps=0, maxp=0, npages=0, state=p,
             B=1, Hkv=1, d=512, dv=512, blk=128, W=128, Nmax=8, flags=0):
        return libhca.hca_append(k, v, w, seq, kw, vw, kc, vc, table, ps, maxp, npages, state, B, Hkv, d, dv,
                                 blk, W, Nmax, flags, None)

    assert libhca.hca_append_state_size(2, 3, 512, 512) == 2 * 3 * (4 + 1024) * 4
    assert libhca.hca_append_state_size(-1, 1, 64, 64) == 0
    # unsupported head dims, block, flags
    assert call(d=96) == _lib.HCA_ERR_UNSUPPORTED
    assert call(blk=129) == _lib.HCA_ERR_UNSUPPORTED
    assert call(flags=_lib.HCA_QK_NORM) == _lib.HCA_ERR_UNSUPPORTED
    # null / misaligned pointers, bad sizes, no cache rows
    assert call(k=None) == _lib.HCA_ERR_INVALID_ARG
    assert call(state=ctypes.c_void_p(24)) == _lib.HCA_ERR_INVALID_ARG
    assert call(seq=ctypes.c_void_p(18)) == _lib.HCA_ERR_INVALID_ARG
    assert call(W=0) == _lib.HCA_ERR_INVALID_ARG
    assert call(Nmax=0) == _lib.HCA_ERR_INVALID_ARG
    assert call(flags=_lib.HCA_PAGED) == _lib.HCA_ERR_INVALID_ARG
    assert call(flags=_lib.HCA_PAGED, table=p, ps=96, maxp=2, npages=2) == _lib.HCA_ERR_INVALID_ARG
    # nothing to do: no launch, OK
    assert call(k=None, v=None, seq=None, kw=None, vw=None, kc=None, vc=None, state=None, B=0) == _lib.HCA_OK


def test_vha_rejects_before_launch(libhca):
    p = ctypes.c_void_p(16)
    # (out, U, V, n, Hq, dv, r, flags, stream)
    assert libhca.hca_vha(p, p, p, 4, 65, 512, 4, 0, None) == _lib.HCA_ERR_UNSUPPORTED     # more than 64 heads
    assert libhca.hca_vha(p, p, p, 4, 64, 512, 33, 0, None) == _lib.HCA_ERR_UNSUPPORTED    # rank above 32
    assert libhca.hca_vha(p, p, p, 4, 64, 96, 4, 0, None) == _lib.HCA_ERR_UNSUPPORTED      # dv not a multiple of 64
    assert libhca.hca_vha(p, p, p, 4, 64, 512, 4, 1 << 8, None) == _lib.HCA_ERR_UNSUPPORTED
    assert libhca.hca_vha(None, p, p, 4, 64, 512, 4, 0, None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_vha(ctypes.c_void_p(24), p, p, 4, 64, 512, 4, 0, None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_vha(p, p, p, 4, 64, 512, 0, 0, None) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_vha(None, None, None, 0, 64, 512, 4, 0, None) == _lib.HCA_OK          # nothing to do


def test_prefill_backward_rejects_before_launch(libhca):
    p = ctypes.c_void_p(256)
    big = 1 << 30

    def call(q=p, k=p, v=p, w=None, kc=p, vc=p, out=p, lse=p, dout=p, dq=p, dk=p, dv=p, dw=None, ws=p,
             ws_bytes=big, B=1, T=256, Hq=64, Hkv=1, d=512, dvd=512, blk=128, W=128, scale=0.05, flags=0):
        return libhca.hca_prefill_backward(q, k, v, w, kc, vc, out, lse, dout, dq, dk, dv, dw, ws, ws_bytes,
                                           B, T, Hq, Hkv, d, dvd, blk, W, scale, flags, None)

    # workspace: per-row terms, the entries' fp32 gradients, then 64 KB P / dS records for
    # every (row tile, key tile slot) of a segment: 512 row tiles of 2 tokens, one entry tile and
    # up to three 128-aligned raw tiles each
    assert libhca.hca_prefill_backward_workspace_size(1, 1024, 64, 1, 512, 128, 128) == (
        1024 * 64 * 4 + 2 * 8 * 512 * 4 + 512 * 4 * 65536)
    assert libhca.hca_prefill_backward_workspace_size(1, 1024, 64, 1, 64, 128, 128) == 0
    assert libhca.hca_prefill_backward_workspace_size(-1, 1024, 64, 1, 512, 128, 128) == 0
    assert libhca.hca_prefill_backward_workspace_size(1, 1024, 48, 1, 512, 128, 128) == 0
    # a forced segment of 7 row tiles bounds the records to 7 row tiles
    assert libhca.hca_debug_set_backward_segment(7) == _lib.HCA_OK
    try:
        assert libhca.hca_prefill_backward_workspace_size(1, 1024, 64, 1, 512, 128, 128) == (
            1024 * 64 * 4 + 2 * 8 * 512 * 4 + 7 * 4 * 65536)
    finally:
        assert libhca.hca_debug_set_backward_segment(0) == _lib.HCA_OK
    assert libhca.hca_debug_set_backward_segment(-1) == _lib.HCA_ERR_INVALID_ARG
    assert libhca.hca_debug_set_dsa_rows_limit(1 << 20) == _lib.HCA_OK
    assert libhca.hca_debug_set_dsa_rows_limit(0) == _lib.HCA_OK
    assert libhca.hca_debug_set_dsa_rows_limit(-1) == _lib.HCA_ERR_INVALID_ARG
    # unsupported head dims, block, group size, flags
    assert call(d=64, dvd=64) == _lib.HCA_ERR_UNSUPPORTED
    assert call(blk=129) == _lib.HCA_ERR_UNSUPPORTED
    assert call(Hq=6, Hkv=2) == _lib.HCA_ERR_UNSUPPORTED
    assert call(flags=_lib.HCA_WRITE_LSE) == _lib.HCA_ERR_UNSUPPORTED
    # null or misaligned pointers, bad sizes, NaN scale, a workspace too small or misaligned
    assert call(lse=None) == _lib.HCA_ERR_INVALID_ARG
    assert call(dout=None) == _lib.HCA_ERR_INVALID_ARG
    assert call(dq=ctypes.c_void_p(264)) == _lib.HCA_ERR_INVALID_ARG
    assert call(dw=ctypes.c_void_p(258)) == _lib.HCA_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(272)) == _lib.HCA_ERR_INVALID_ARG
    assert call(ws_bytes=1024) == _lib.HCA_ERR_INVALID_ARG
    assert call(W=0) == _lib.HCA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == _lib.HCA_ERR_INVALID_ARG
    # nothing to do: no launch, OK
    assert call(q=None, k=None, v=None, kc=None, vc=None, out=None, lse=None, dout=None, dq=None, dk=None,
                dv=None, ws=None, B=0) == _lib.HCA_OK


def test_header_compiles_as_c_and_links(tmp_path, libhca):
    """include/hca.h is a plain C header: a C99 translation unit that includes it and takes the
    address of every entry point compiles warning-free and links against libhca.so."""
    import shutil
    import subprocess
    from compressed_long_context_b200 import _lib as L
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_hca.c"
    names = sorted(L.EXPORTS)
    body = "\n".join("    (void)&%s;" % n for n in names)
    src.write_text('#include "hca.h"\n#include <stddef.h>\nint main(void) {\n%s\n    return 0;\n}\n' % body)
    exe = tmp_path / "use_hca"
    lib_dir = os.path.dirname(L.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", lib_dir, "-l:libhca.so", "-Wl,--unresolved-symbols=ignore-in-shared-libs",
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
