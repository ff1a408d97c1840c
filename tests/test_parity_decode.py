"""GPU parity of hca_decode (through the C ABI) against the fp64 oracle.

Bar: max abs error <= 1e-2 and mean abs error <= 1e-3 on the fp32 output.
"""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle
from compressed_long_context_b200 import workloads as wl

pytestmark = pytest.mark.gpu
MAX_TOL, MEAN_TOL = 1e-2, 1e-3


def check(got, ref):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape
    err = np.abs(g - ref)
    assert np.isfinite(g).all()
    assert err.max() <= MAX_TOL, ("max", err.max())
    assert err.mean() <= MEAN_TOL, ("mean", err.mean())
    return err.max(), err.mean()


def bits(t):
    return oracle.bf16_bits(t)


def rand_bf16(shape, g, dev, std=1.0):
    return (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16)


def direct_case(dev, seed, lengths, Hq=64, Hkv=1, W=128, blk=128, Nmax=None, paged_ps=0, norm=False,
                gate=False):
    """Cache entries drawn directly (both sides read the same bf16 cache)."""
    g = torch.Generator(device=dev).manual_seed(seed)
    B = len(lengths)
    seq = torch.tensor(lengths, dtype=torch.int32, device=dev)
    nc_max = max(oracle.visible_entries(L - 1, W, blk) for L in lengths)
    if Nmax is None:
        Nmax = max(1, nc_max)
    q = rand_bf16((B, Hq, 512), g, dev)
    kw = rand_bf16((B, W, Hkv, 512), g, dev)
    vw = rand_bf16((B, W, Hkv, 512), g, dev)
    gq = gk = gt = None
    if norm:
        gq = torch.rand((512,), generator=g, device=dev) + 0.5
        gk = torch.rand((512,), generator=g, device=dev) + 0.5
    if gate:
        gt = rand_bf16((B, Hq, 512), g, dev)
    if paged_ps:
        npg = (Nmax + paged_ps - 1) // paged_ps
        P = B * npg + 3
        kc = rand_bf16((P, paged_ps, Hkv, 512), g, dev)
        vc = rand_bf16((P, paged_ps, Hkv, 512), g, dev)
        perm = torch.randperm(P, generator=torch.Generator().manual_seed(seed))[:B * npg]
        table = perm.view(B, npg).to(torch.int32).to(dev)
    else:
        kc = rand_bf16((B, Nmax, Hkv, 512), g, dev)
        vc = rand_bf16((B, Nmax, Hkv, 512), g, dev)
        table = None
    return dict(q=q, kc=kc, vc=vc, kw=kw, vw=vw, seqlens=seq, gq=gq, gk=gk, gate=gt, page_table=table,
                page_size=paged_ps, W=W, blk=blk)


def run_both(c, scale=None):
    scale = scale if scale is not None else 1.0 / np.sqrt(512)
    out = hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], c["blk"], c["W"], scale,
                     page_table=c["page_table"], page_size=c["page_size"], gq=c["gq"], gk=c["gk"],
                     gate=c["gate"])
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = oracle.decode(bits(c["q"]), bits(c["kc"]), bits(c["vc"]), bits(c["kw"]), bits(c["vw"]),
                        c["seqlens"].cpu().numpy(), c["blk"], c["W"], scale,
                        page_table=None if c["page_table"] is None else c["page_table"].cpu().numpy(),
                        page_size=c["page_size"],
                        gq=None if c["gq"] is None else c["gq"].cpu().numpy(),
                        gk=None if c["gk"] is None else c["gk"].cpu().numpy(), eps=1e-6,
                        gate=None if c["gate"] is None else bits(c["gate"]))
    return out, ref


@pytest.mark.parametrize("lengths,W", [
    ([131072 // 16], 128),                       # one sequence, 63 entries + window
    ([1000, 129, 5000, 300, 1], 128),            # ragged, incl. L=1 and L<W
    ([128 * 9 + 77] * 7, 128),
    ([4096 + 5, 70, 20000], 256),                # two window tiles
    ([60000, 3], 200),
    ([128, 129, 255, 256, 257, 2], 128),   # around the window size and the first complete block
])
def test_decode_contiguous(cuda_device, libhca, lengths, W):
    c = direct_case(cuda_device, 11 + len(lengths), lengths, W=W)
    check(*run_both(c))


@pytest.mark.parametrize("ps", [64, 128])
def test_decode_paged(cuda_device, libhca, ps):
    lengths = [9000, 4096 + 17, 130, 30000, 777]
    c = direct_case(cuda_device, 21 + ps, lengths, paged_ps=ps)
    check(*run_both(c))


def test_decode_norm_gate(cuda_device, libhca):
    lengths = [9000, 4096 + 17, 300, 12345]
    c = direct_case(cuda_device, 31, lengths, W=256, paged_ps=64, norm=True, gate=True)
    check(*run_both(c))


def test_decode_norm_contiguous(cuda_device, libhca):
    c = direct_case(cuda_device, 32, [5000, 900], norm=True)
    check(*run_both(c))


@pytest.mark.parametrize("Hq,Hkv", [(64, 2), (8, 1), (48, 3)])
def test_decode_groups(cuda_device, libhca, Hq, Hkv):
    c = direct_case(cuda_device, 41 + Hq, [3000, 777, 129], Hq=Hq, Hkv=Hkv)
    check(*run_both(c))


@pytest.mark.parametrize("blk,W", [(1, 1), (2, 5), (100, 50)])
def test_decode_block_and_window(cuda_device, libhca, blk, W):
    c = direct_case(cuda_device, 51 + blk, [700, 333, 64], W=W, blk=blk)
    check(*run_both(c))


def test_decode_many_short_sequences(cuda_device, libhca):
    rs = np.random.RandomState(5)
    lengths = [int(x) for x in rs.randint(1, 3000, size=300)]
    c = direct_case(cuda_device, 61, lengths, Hq=16)
    check(*run_both(c))


def test_decode_large_logits_rescale(cuda_device, libhca):
    """Keys scaled so the running max keeps growing across tiles (exercises the O^T rescale)."""
    c = direct_case(cuda_device, 71, [40000, 20000])
    ramp = torch.linspace(0.2, 6.0, c["kc"].shape[1], device=cuda_device).view(1, -1, 1, 1)
    c["kc"] = (c["kc"].float() * ramp).to(torch.bfloat16)
    check(*run_both(c))


@pytest.mark.parametrize("boost", [12.0, 40.0])
def test_decode_first_key_far_below(cuda_device, libhca, boost):
    """Entry 0 (the first key of every piece that starts a sequence) is zero and the other
    entries are scaled up, so the reference seeded from the first key lies far below the
    tile maximum and must be raised inside the first tile; with the larger scale the logits
    span hundreds of binary orders of magnitude."""
    c = direct_case(cuda_device, 73, [40000, 20000, 9000])
    kc = c["kc"].float() * boost
    kc[:, 0] = 0.0
    c["kc"] = kc.to(torch.bfloat16)
    check(*run_both(c))


def test_decode_repeatable_and_workspace_reuse(cuda_device, libhca):
    c = direct_case(cuda_device, 81, [20000, 100, 7000])
    ws = torch.empty(hca.decode_workspace_size(3, 64, 1, 512), dtype=torch.uint8, device=cuda_device)
    a = hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], 128, 128, 0.05, workspace=ws)
    b = hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], 128, 128, 0.05, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_decode_device_input_error(cuda_device, libhca):
    """A sequence whose visible entries exceed Nmax is reported, not read out of bounds."""
    c = direct_case(cuda_device, 91, [5000], Nmax=4)
    hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], 128, 128, 0.05)
    with pytest.raises(hca.HCAError) as e:
        hca.get_device_error()
    assert e.value.code == 5
    hca.get_device_error()     # cleared


def test_decode_bad_page_id_reported(cuda_device, libhca):
    """A page id outside the pool is reported as a device-input error; the loads are
    clamped into the pool, so nothing is read outside it."""
    c = direct_case(cuda_device, 95, [9000, 3000], paged_ps=64)
    c["page_table"][0, 1] = c["kc"].shape[0]          # one past the last page (entries 64..68)
    hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], 128, 128, 0.05,
               page_table=c["page_table"], page_size=64)
    with pytest.raises(hca.HCAError) as e:
        hca.get_device_error()
    assert e.value.code == 5
    hca.get_device_error()     # cleared


def test_decode_ragged_long_and_short(cuda_device, libhca):
    """Few long sequences among many short ones: the per-sequence CTA counts cannot hold
    every CTA near the even share of tiles, so the batch is cut into equal ranges that
    cross sequence boundaries."""
    lengths = [60000 if i % 2 == 0 else 1000 for i in range(100)]    # 350 tiles over 148 CTAs
    out, ref = run_both(direct_case(cuda_device, 96, lengths, paged_ps=128, norm=True))
    check(out, ref)


# ------------------------------------------------------------ full-size workloads (every output)

@pytest.mark.parametrize("cfg", [wl.DECODE_128K, wl.DECODE_1M], ids=lambda c: c.name)
def test_decode_full_size_from_raw(cuda_device, libhca, cfg):
    """Compress + decode at full size in the benchmark's launch configuration; every sequence,
    head and channel checked end to end against oracle compress + oracle decode."""
    inp = wl.decode_inputs(cfg, cuda_device)
    kc, vc = hca.compress(inp["k"], inp["v"], inp["w"], cfg.blk)
    scale = 1.0 / np.sqrt(cfg.d)
    out = hca.decode(inp["q"], kc, vc, inp["kw"], inp["vw"], inp["seqlens"], cfg.blk, cfg.W, scale)
    torch.cuda.synchronize()
    hca.get_device_error()
    rk, rv = oracle.compress(bits(inp["k"]), bits(inp["v"]), inp["w"].cpu().numpy(), cfg.blk)
    for got, ref in ((kc, rk), (vc, rv)):
        assert np.abs(got.float().cpu().numpy() - ref).max() <= 4e-3
    ref = oracle.decode(bits(inp["q"]), oracle.round_bf16(rk), oracle.round_bf16(rv), bits(inp["kw"]),
                        bits(inp["vw"]), inp["seqlens"].cpu().numpy(), cfg.blk, cfg.W, scale)
    check(out, ref)
    del inp, kc, vc, rk, rv
    torch.cuda.empty_cache()


def test_decode_full_size_ragged_paged(cuda_device, libhca):
    """The ragged paged batch with QK RMSNorm and the output gate: every output."""
    cfg = wl.RAGGED_PAGED
    inp = wl.paged_decode_inputs(cfg, cuda_device)
    scale = 1.0 / np.sqrt(cfg.d)
    out = hca.decode(inp["q"], inp["kc"], inp["vc"], inp["kw"], inp["vw"], inp["seqlens"], cfg.blk, cfg.W,
                     scale, page_table=inp["page_table"], page_size=cfg.page_size, gq=inp["gq"],
                     gk=inp["gk"], gate=inp["gate"])
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = oracle.decode(bits(inp["q"]), bits(inp["kc"]), bits(inp["vc"]), bits(inp["kw"]), bits(inp["vw"]),
                        inp["seqlens"].cpu().numpy(), cfg.blk, cfg.W, scale,
                        page_table=inp["page_table"].cpu().numpy(), page_size=cfg.page_size,
                        gq=inp["gq"].cpu().numpy(), gk=inp["gk"].cpu().numpy(), eps=1e-6, gate=bits(inp["gate"]))
    check(out, ref)
