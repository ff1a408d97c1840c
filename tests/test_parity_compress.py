"""GPU parity of hca_compress against the fp64 oracle.

Tolerance on the bf16 cache: 4e-3 absolute, widened to the bf16 rounding bound
2^-8 * |ref| (+1e-5 for fp32 accumulation) where |ref| >= 1, since no bf16 value can be
closer than half a unit in the last place to a reference of that size.
"""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle
from compressed_long_context_b200 import workloads as wl

pytestmark = pytest.mark.gpu
TOL = 4e-3


def cache_tol(ref):
    return np.maximum(TOL, np.abs(ref) * 2.0 ** -8 + 1e-5)


def _ref(k, v, w, blk):
    kc, vc = oracle.compress(oracle.bf16_bits(k), oracle.bf16_bits(v),
                             None if w is None else w.cpu().numpy(), blk)
    return kc, vc


def _cmp(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    assert np.all(err <= cache_tol(ref)), (err.max(), np.abs(ref).max())


@pytest.mark.parametrize("B,T,Hkv,d,dv,blk,wmode", [
    (2, 1000, 1, 512, 512, 128, "rand"),
    (1, 1024, 1, 64, 64, 128, "zero"),
    (2, 333, 2, 64, 512, 128, "none"),
    (1, 700, 2, 256, 128, 100, "rand"),
    (3, 130, 1, 512, 64, 1, "rand"),
    (1, 257, 3, 128, 256, 2, "rand"),
    (1, 127, 1, 512, 512, 128, "rand"),     # no complete block
])
def test_compress_small(cuda_device, libhca, B, T, Hkv, d, dv, blk, wmode):
    g = torch.Generator(device=cuda_device).manual_seed(B * 1000 + T + d)
    k = torch.randn((B, T, Hkv, d), generator=g, device=cuda_device).to(torch.bfloat16)
    v = torch.randn((B, T, Hkv, dv), generator=g, device=cuda_device).to(torch.bfloat16)
    w = {"rand": torch.randn((B, T), generator=g, device=cuda_device) * 2.0,
         "zero": torch.zeros((B, T), device=cuda_device), "none": None}[wmode]
    kc, vc = hca.compress(k, v, w, blk)
    torch.cuda.synchronize()
    rk, rv = _ref(k, v, w, blk)
    assert kc.shape == (B, T // blk, Hkv, d)
    _cmp(kc, rk)
    _cmp(vc, rv)
    hca.get_device_error()


def test_compress_dominant_weight(cuda_device, libhca):
    k = torch.randn((1, 256, 1, 512), device=cuda_device).to(torch.bfloat16)
    w = torch.zeros((1, 256), device=cuda_device)
    w[0, 5] = 90.0
    w[0, 200] = 90.0
    kc, _ = hca.compress(k, k, w, 128)
    torch.cuda.synchronize()
    assert torch.equal(kc[0, 0, 0], k[0, 5, 0])
    assert torch.equal(kc[0, 1, 0], k[0, 200, 0])


@pytest.mark.parametrize("cfg", [wl.DECODE_128K, wl.DECODE_1M], ids=lambda c: c.name)
def test_compress_full_size_sampled(cuda_device, libhca, cfg):
    """Full-size raw K/V, compressed in the launch configuration the benchmark times;
    a sample of entries (first, last, random) is checked against the oracle."""
    inp = wl.decode_inputs(cfg, cuda_device)
    k, v, w = inp["k"], inp["v"], inp["w"]
    kc, vc = hca.compress(k, v, w, cfg.blk)
    torch.cuda.synchronize()
    hca.get_device_error()
    Nc = cfg.T // cfg.blk
    rs = np.random.RandomState(0)
    picks = [(0, 0), (cfg.B - 1, Nc - 1)] + [(int(rs.randint(cfg.B)), int(rs.randint(Nc))) for _ in range(30)]
    kb = torch.stack([k[b, j * cfg.blk:(j + 1) * cfg.blk] for b, j in picks])
    vb = torch.stack([v[b, j * cfg.blk:(j + 1) * cfg.blk] for b, j in picks])
    wb = torch.stack([w[b, j * cfg.blk:(j + 1) * cfg.blk] for b, j in picks])
    rk, rv = _ref(kb, vb, wb, cfg.blk)
    got_k = torch.stack([kc[b, j] for b, j in picks]).unsqueeze(1)
    got_v = torch.stack([vc[b, j] for b, j in picks]).unsqueeze(1)
    _cmp(got_k, rk)
    _cmp(got_v, rv)
    del inp, k, v, kc, vc
    torch.cuda.empty_cache()
