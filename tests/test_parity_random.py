"""Seeded randomized parity sweep (GPU) over combinations of the supported options.

Each case draws its shape and options from its own seed, so a failure names a case that
can be replayed alone.  Decode: batch size, lengths, GQA group, block and window sizes,
contiguous or paged cache (page size a multiple of 64), QK normalisation and gate.  Prefill:
head dim 64 or 512, GQA group (a power of two), block and window sizes, sequence length,
fp32 or bf16 output.  Sizes stay small enough for the fp64 oracle to finish in seconds;
the bar is the one of the other parity tests.
"""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle

pytestmark = pytest.mark.gpu
MAX_TOL, MEAN_TOL = 1e-2, 1e-3


def bits(t):
    return oracle.bf16_bits(t)


def check(got, ref):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape
    assert np.isfinite(g).all()
    err = np.abs(g - ref)
    assert err.max() <= MAX_TOL, ("max", err.max())
    assert err.mean() <= MEAN_TOL, ("mean", err.mean())


def _bf16(shape, g, dev, std=1.0):
    return (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16)


@pytest.mark.parametrize("seed", range(40))
def test_decode_random(cuda_device, libhca, seed):
    rs = np.random.RandomState(1000 + seed)
    dev = cuda_device
    Hkv = int(rs.choice([1, 1, 2, 4]))
    G = int(rs.choice([1, 8, 16, 48, 64]))
    Hq = Hkv * G
    blk = int(rs.choice([1, 16, 100, 128, 128]))
    W = int(rs.randint(1, 300))
    B = int(rs.randint(1, 9))
    lengths = [int(x) for x in rs.randint(1, 40000 if blk >= 64 else 3000, size=B)]
    paged = bool(rs.randint(2))
    ps = int(rs.choice([64, 128, 192])) if paged else 0
    norm, gate = bool(rs.randint(2)), bool(rs.randint(2))
    g = torch.Generator(device=dev).manual_seed(2000 + seed)
    nc = [oracle.visible_entries(L - 1, W, blk) for L in lengths]
    Nmax = max(1, max(nc))
    q = _bf16((B, Hq, 512), g, dev)
    kw = _bf16((B, W, Hkv, 512), g, dev)
    vw = _bf16((B, W, Hkv, 512), g, dev)
    if paged:
        npg = (Nmax + ps - 1) // ps
        P = B * npg + 2
        kc = _bf16((P, ps, Hkv, 512), g, dev)
        vc = _bf16((P, ps, Hkv, 512), g, dev)
        perm = torch.randperm(P, generator=torch.Generator().manual_seed(seed))[:B * npg]
        table = perm.view(B, npg).to(torch.int32).to(dev)
    else:
        kc = _bf16((B, Nmax, Hkv, 512), g, dev)
        vc = _bf16((B, Nmax, Hkv, 512), g, dev)
        table = None
    gq = (torch.rand((512,), generator=g, device=dev) + 0.5) if norm else None
    gk = (torch.rand((512,), generator=g, device=dev) + 0.5) if norm else None
    gt = _bf16((B, Hq, 512), g, dev) if gate else None
    seq = torch.tensor(lengths, dtype=torch.int32, device=dev)
    scale = 1.0 / np.sqrt(512)
    out = hca.decode(q, kc, vc, kw, vw, seq, blk, W, scale, page_table=table, page_size=ps, gq=gq, gk=gk,
                     gate=gt)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = oracle.decode(bits(q), bits(kc), bits(vc), bits(kw), bits(vw), seq.cpu().numpy(), blk, W, scale,
                        page_table=None if table is None else table.cpu().numpy(), page_size=ps,
                        gq=None if gq is None else gq.cpu().numpy(), gk=None if gk is None else gk.cpu().numpy(),
                        eps=1e-6, gate=None if gt is None else bits(gt))
    check(out, ref)


@pytest.mark.parametrize("seed", range(30))
def test_prefill_random(cuda_device, libhca, seed):
    rs = np.random.RandomState(3000 + seed)
    dev = cuda_device
    d = int(rs.choice([64, 512]))
    Hkv = int(rs.choice([1, 1, 2]))
    G = int(rs.choice([1, 2, 8, 32, 64, 128]))
    Hq = Hkv * G
    blk = int(rs.choice([1, 8, 64, 128]))
    W = int(rs.randint(1, 400))
    B = int(rs.randint(1, 3))
    Tmax = 700 if d == 512 else 1500
    T = int(rs.randint(1, max(2, Tmax * 64 // max(Hq, 64))))
    out_f32 = bool(rs.randint(2))
    g = torch.Generator(device=dev).manual_seed(4000 + seed)
    q = _bf16((B, T, Hq, d), g, dev)
    k = _bf16((B, T, Hkv, d), g, dev)
    v = _bf16((B, T, Hkv, d), g, dev)
    w = torch.randn((B, T), generator=g, device=dev) * float(rs.choice([0.0, 0.5, 2.0]))
    scale = 1.0 / np.sqrt(d)
    kc, vc = hca.compress(k, v, w, blk)
    out = hca.prefill(q, k, v, kc, vc, blk, W, scale, out_f32=True)
    if not out_f32:
        assert torch.equal(hca.prefill(q, k, v, kc, vc, blk, W, scale), out.to(torch.bfloat16))
    torch.cuda.synchronize()
    hca.get_device_error()
    okc, ovc = oracle.compress(bits(k), bits(v), w.cpu().numpy(), blk)
    rows = [(b, t) for b in range(B) for t in range(T)]
    ref = oracle.prefill_rows(bits(q), bits(k), bits(v), oracle.round_bf16(okc), oracle.round_bf16(ovc), blk, W,
                              scale, rows)
    check(out.cpu().reshape(B * T, Hq, d), ref)
