"""The bounded-wait path on the GPU, made to run out on purpose without any fault: the wait
limit is shortened to milliseconds through the test hooks, then (1) a one-CTA probe waits on
a barrier that cannot complete, and (2) a real decode launch whose producer never requests
its first key slab.  Both must report HCA_ERR_TIMEOUT through hca_get_device_error, the
decode must mark its outputs NaN rather than merge incomplete records, and the next normal
decode on the same device must match the oracle (the GPU still answers; tensor memory was
freed)."""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle
from compressed_long_context_b200 import _lib

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _case(dev):
    g = torch.Generator(device=dev).manual_seed(17)
    lengths = [9000, 300, 20000]
    B, Hq, d, W = len(lengths), 64, 512, 128
    Nmax = max((L - W) // 128 for L in lengths)
    r = lambda *s: torch.randn(s, generator=g, device=dev).to(torch.bfloat16)  # noqa: E731
    return dict(q=r(B, Hq, d), kc=r(B, Nmax, 1, d), vc=r(B, Nmax, 1, d), kw=r(B, W, 1, d), vw=r(B, W, 1, d),
                seqlens=torch.tensor(lengths, dtype=torch.int32, device=dev), W=W)


def _decode(c):
    return hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], 128, c["W"], 1.0 / np.sqrt(512))


def test_wait_probe_times_out(cuda_device, libhca):
    hca.get_device_error()
    try:
        assert libhca.hca_debug_set_wait_limit(1_000_000, _stream()) == _lib.HCA_OK      # 1 ms
        assert libhca.hca_debug_wait_probe(_stream()) == _lib.HCA_OK
        assert libhca.hca_get_device_error(_stream()) == _lib.HCA_ERR_TIMEOUT
        assert libhca.hca_get_device_error(_stream()) == _lib.HCA_OK                    # cleared
    finally:
        libhca.hca_debug_set_wait_limit(0, _stream())


def test_decode_unwinds_after_a_missing_slab(cuda_device, libhca):
    c = _case(cuda_device)
    hca.get_device_error()
    try:
        assert libhca.hca_debug_set_wait_limit(2_000_000, _stream()) == _lib.HCA_OK      # 2 ms
        assert libhca.hca_debug_set_drop_slab(1, _stream()) == _lib.HCA_OK
        bad = _decode(c)
        torch.cuda.synchronize()
        assert libhca.hca_get_device_error(_stream()) == _lib.HCA_ERR_TIMEOUT
        assert torch.isnan(bad).all()
    finally:
        libhca.hca_debug_set_drop_slab(0, _stream())
        libhca.hca_debug_set_wait_limit(0, _stream())
    hca.get_device_error()
    good = _decode(c)
    torch.cuda.synchronize()
    hca.get_device_error()
    b = oracle.bf16_bits
    ref = oracle.decode(b(c["q"]), b(c["kc"]), b(c["vc"]), b(c["kw"]), b(c["vw"]), c["seqlens"].cpu().numpy(),
                        128, c["W"], 1.0 / np.sqrt(512))
    err = np.abs(good.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3
