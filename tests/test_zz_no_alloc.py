"""hca_decode_noalloc: decode for callers that cannot allocate device memory when they
decode (engine plugins that must not allocate while enqueuing, servers that forbid
allocation after warm-up, hosts that only hold pre-allocated buffers).

Called through the C ABI and checked against the workspace-taking hca_decode on the same
inputs, and against the fp64 oracle, with the decode tolerances (max abs 1e-2, mean abs
1e-3), on two calls in a row (the library-owned scratch keeps the first call's contents).
The device's free memory must be the same before and after the two calls: the entry point
allocates nothing.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle
from compressed_long_context_b200 import _lib

pytestmark = pytest.mark.gpu
MAX_TOL, MEAN_TOL = 1e-2, 1e-3


def _case(dev, seed, lengths, W=128, paged_ps=0, extras=False):
    g = torch.Generator(device=dev).manual_seed(seed)
    B, Hq, d = len(lengths), 64, 512
    nc = max(max(0, (L - W) // 128) for L in lengths)
    Nmax = max(1, nc)
    r = lambda *s: torch.randn(s, generator=g, device=dev).to(torch.bfloat16)  # noqa: E731
    c = dict(q=r(B, Hq, d), kw=r(B, W, 1, d), vw=r(B, W, 1, d),
             seqlens=torch.tensor(lengths, dtype=torch.int32, device=dev), W=W, page_size=0, page_table=None,
             gq=None, gk=None, gate=None)
    if paged_ps:
        npg = (Nmax + paged_ps - 1) // paged_ps
        c["kc"], c["vc"] = r(B * npg, paged_ps, 1, d), r(B * npg, paged_ps, 1, d)
        perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
        c["page_table"], c["page_size"] = perm.view(B, npg).to(dev), paged_ps
    else:
        c["kc"], c["vc"] = r(B, Nmax, 1, d), r(B, Nmax, 1, d)
    if extras:
        c["gq"] = torch.rand((d,), generator=g, device=dev) + 0.5
        c["gk"] = torch.rand((d,), generator=g, device=dev) + 0.5
        c["gate"] = r(B, Hq, d)
    return c


def _noalloc(lib, c, out, scale):
    B, Hq, d = c["q"].shape
    flags = ((_lib.HCA_PAGED if c["page_table"] is not None else 0)
             | (_lib.HCA_QK_NORM if c["gq"] is not None else 0)
             | (_lib.HCA_OUT_GATE if c["gate"] is not None else 0))
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    paged = c["page_table"] is not None
    return lib.hca_decode_noalloc(
        p(c["q"]), p(c["kc"]), p(c["vc"]), p(c["page_table"]), c["page_size"],
        c["page_table"].shape[1] if paged else 0, c["kc"].shape[0] if paged else 0,
        p(c["kw"]), p(c["vw"]), p(c["seqlens"]), p(c["gq"]), p(c["gk"]), 1e-6, p(c["gate"]), p(out),
        B, Hq, 1, d, d, 128, c["W"], 0 if paged else c["kc"].shape[1], scale, flags,
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("kind", ["contiguous", "paged_norm_gate"])
def test_decode_noalloc_matches_decode(cuda_device, libhca, kind):
    if kind == "contiguous":
        c = _case(cuda_device, 7, [131072, 5000, 129, 1, 70000])
    else:
        c = _case(cuda_device, 8, [9000, 4096 + 17, 300, 12345], W=256, paged_ps=64, extras=True)
    scale = 1.0 / np.sqrt(512)
    ref = hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], 128, c["W"], scale,
                     page_table=c["page_table"], page_size=c["page_size"], gq=c["gq"], gk=c["gk"],
                     gate=c["gate"])
    torch.cuda.synchronize()
    hca.get_device_error()
    b = oracle.bf16_bits
    exact = oracle.decode(b(c["q"]), b(c["kc"]), b(c["vc"]), b(c["kw"]), b(c["vw"]), c["seqlens"].cpu().numpy(),
                          128, c["W"], scale,
                          page_table=None if c["page_table"] is None else c["page_table"].cpu().numpy(),
                          page_size=c["page_size"], gq=None if c["gq"] is None else c["gq"].cpu().numpy(),
                          gk=None if c["gk"] is None else c["gk"].cpu().numpy(), eps=1e-6,
                          gate=None if c["gate"] is None else b(c["gate"]))
    outs = [torch.full_like(ref, float("nan")) for _ in range(2)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for out in outs:
        assert _noalloc(libhca, c, out, scale) == _lib.HCA_OK
        torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    hca.get_device_error()
    assert free_after == free_before
    for out in outs:
        err = (out - ref).abs()
        assert torch.isfinite(out).all()
        assert err.max().item() <= MAX_TOL and err.mean().item() <= MEAN_TOL
        e64 = np.abs(out.cpu().numpy().astype(np.float64) - exact)
        assert e64.max() <= MAX_TOL and e64.mean() <= MEAN_TOL


def test_decode_noalloc_rejects_batches_beyond_the_scratch(cuda_device, libhca):
    B = 4096    # 4096 units need far more than the fixed scratch holds
    need = libhca.hca_decode_workspace_size(B, 64, 1, 512)
    assert need > libhca_limit()
    dummy = ctypes.c_void_p(256)
    rc = libhca.hca_decode_noalloc(dummy, dummy, dummy, None, 0, 0, 0, dummy, dummy, dummy, None, None, 1e-6,
                                   None, dummy, B, 64, 1, 512, 512, 128, 128, 1024, 0.05, 0,
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.HCA_ERR_INVALID_ARG


def libhca_limit():
    import os
    import re
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                             "hca.h")).read()
    m = re.search(r"#define HCA_DECODE_NOALLOC_MAX_BYTES \((\d+)u << (\d+)\)", text)
    return int(m.group(1)) << int(m.group(2))
