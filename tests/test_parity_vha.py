"""GPU parity of hca_vha (Virtual Head Attention on an attention output) against the fp64
oracle.

 - After attention: the oracle's attention output (prefill rows or decode, gate included)
   followed by the oracle's cross-head mixing; fp32 outputs, bar max abs 1e-2 and mean abs
   1e-3.
 - The bf16 path on its own: seeded bf16 inputs (not from the CUDA path), each result
   within one bf16 rounding of the fp64 mixing of the same values.
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
    assert g.shape == ref.shape and np.isfinite(g).all()
    err = np.abs(g - ref)
    assert err.max() <= MAX_TOL, ("max", err.max())
    assert err.mean() <= MEAN_TOL, ("mean", err.mean())


def factors(dev, Hq, r, seed, std=0.1):
    g = torch.Generator(device=dev).manual_seed(seed)
    U = torch.randn((Hq, r), generator=g, device=dev) * std
    V = torch.randn((Hq, r), generator=g, device=dev) * std
    return U, V


@pytest.mark.parametrize("r", [1, 8, 32])
def test_vha_after_gated_decode(cuda_device, libhca, r):
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(40 + r)
    B, Hq, W, blk = 4, 64, 128, 128
    lengths = [9000, 130, 20000, 700]
    Nmax = max(oracle.visible_entries(L - 1, W, blk) for L in lengths)
    q = torch.randn((B, Hq, 512), generator=g, device=dev).to(torch.bfloat16)
    kc = torch.randn((B, Nmax, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn((B, Nmax, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    kw = torch.randn((B, W, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    vw = torch.randn((B, W, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    gate = torch.randn((B, Hq, 512), generator=g, device=dev).to(torch.bfloat16)
    seq = torch.tensor(lengths, dtype=torch.int32, device=dev)
    U, V = factors(dev, Hq, r, 50 + r)
    scale = 1.0 / np.sqrt(512)
    out = hca.decode(q, kc, vc, kw, vw, seq, blk, W, scale, gate=gate)
    hca.vha(out, U, V)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = oracle.decode(bits(q), bits(kc), bits(vc), bits(kw), bits(vw), seq.cpu().numpy(), blk, W, scale,
                        gate=bits(gate))
    check(out, oracle.vha(ref, U.cpu().numpy(), V.cpu().numpy()))


@pytest.mark.parametrize("d,Hq,r", [(512, 64, 4), (512, 64, 16), (64, 8, 2), (64, 32, 32)])
def test_vha_after_prefill(cuda_device, libhca, d, Hq, r):
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(60 + d + Hq + r)
    B, T, blk, W = 1, 400, 128, 128
    q = torch.randn((B, T, Hq, d), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((B, T, 1, d), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((B, T, 1, d), generator=g, device=dev).to(torch.bfloat16)
    w = torch.randn((B, T), generator=g, device=dev) * 0.5
    U, V = factors(dev, Hq, r, 70 + r)
    scale = 1.0 / np.sqrt(d)
    kc, vc = hca.compress(k, v, w, blk)
    out = hca.prefill(q, k, v, kc, vc, blk, W, scale, out_f32=True)
    hca.vha(out, U, V)
    torch.cuda.synchronize()
    hca.get_device_error()
    okc, ovc = oracle.compress(bits(k), bits(v), w.cpu().numpy(), blk)
    rows = [(0, t) for t in range(T)]
    ref = oracle.prefill_rows(bits(q), bits(k), bits(v), oracle.round_bf16(okc), oracle.round_bf16(ovc), blk, W,
                              scale, rows)
    check(out[0], oracle.vha(ref, U.cpu().numpy(), V.cpu().numpy()))


@pytest.mark.parametrize("n,Hq,dv,r", [(300, 64, 512, 8), (7, 16, 64, 32), (50, 64, 128, 1)])
def test_vha_bf16_within_one_rounding(cuda_device, libhca, n, Hq, dv, r):
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(80 + n + r)
    x = (torch.randn((n, Hq, dv), generator=g, device=dev) * 2.0).to(torch.bfloat16)
    U, V = factors(dev, Hq, r, 90 + r, std=0.2)
    ref = oracle.vha(oracle.bits_to_f64(bits(x)), U.cpu().numpy(), V.cpu().numpy())
    y = x.clone()
    hca.vha(y, U, V)
    torch.cuda.synchronize()
    hca.get_device_error()
    got = y.float().cpu().numpy().astype(np.float64)
    # bf16 keeps 8 significant bits: a correctly rounded value is within 2^-9 |ref| (plus the
    # fp32 arithmetic's own error, far smaller), so 2^-8 |ref| + 1e-6 allows one ulp
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def test_vha_zero_factor_leaves_output_unchanged(cuda_device, libhca):
    dev = cuda_device
    x = torch.randn((5, 16, 128), device=dev).to(torch.bfloat16)
    y = x.clone()
    U = torch.randn((16, 3), device=dev)
    hca.vha(y, U, torch.zeros_like(U))
    torch.cuda.synchronize()
    assert torch.equal(x, y)


@pytest.mark.parametrize("n,Hq,dv,r,f32", [
    (33, 3, 64, 5, False),     # odd head count (factor rows not a multiple of 16 bytes apart), rank padded 5 -> 8
    (33, 3, 64, 5, True),      # fp32: two 32-channel slices per token
    (10, 1, 128, 1, False),    # one head: the mixing is a scalar 1 + u v per channel
    (3, 64, 512, 32, True),    # every head, the largest rank, fp32
    (257, 8, 192, 2, True),    # rank padded 2 -> 4, three slices per 64-wide channel block
])
def test_vha_odd_shapes(cuda_device, libhca, n, Hq, dv, r, f32):
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(100 + n + Hq + r)
    x = torch.randn((n, Hq, dv), generator=g, device=dev)
    if not f32:
        x = x.to(torch.bfloat16)
    U, V = factors(dev, Hq, r, 110 + r, std=0.3)
    ref = oracle.vha((oracle.bits_to_f64(bits(x)) if not f32 else x.double().cpu().numpy()), U.cpu().numpy(),
                     V.cpu().numpy())
    y = x.clone()
    hca.vha(y, U, V)
    torch.cuda.synchronize()
    hca.get_device_error()
    got = y.double().cpu().numpy()
    if f32:
        # fp32 arithmetic over at most 2 Hq r products per value: far inside 1e-4 at these magnitudes
        assert np.abs(got - ref).max() <= 1e-4
    else:
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def _decode_case(dev, seed, lengths, Hq=64, W=128, blk=128, paged_ps=0, norm=False, gate=True):
    g = torch.Generator(device=dev).manual_seed(seed)
    B = len(lengths)
    Nmax = max(1, max(oracle.visible_entries(L - 1, W, blk) for L in lengths))
    r = lambda *s: torch.randn(s, generator=g, device=dev).to(torch.bfloat16)  # noqa: E731
    c = dict(q=r(B, Hq, 512), kw=r(B, W, 1, 512), vw=r(B, W, 1, 512),
             seqlens=torch.tensor(lengths, dtype=torch.int32, device=dev), gate=r(B, Hq, 512) if gate else None,
             gq=None, gk=None, page_table=None, page_size=0, W=W, blk=blk)
    if paged_ps:
        npg = (Nmax + paged_ps - 1) // paged_ps
        c["kc"], c["vc"] = r(B * npg, paged_ps, 1, 512), r(B * npg, paged_ps, 1, 512)
        perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
        c["page_table"], c["page_size"] = perm.view(B, npg).to(dev), paged_ps
    else:
        c["kc"], c["vc"] = r(B, Nmax, 1, 512), r(B, Nmax, 1, 512)
    if norm:
        c["gq"] = torch.rand((512,), generator=g, device=dev) + 0.5
        c["gk"] = torch.rand((512,), generator=g, device=dev) + 0.5
    return c


def _oracle_decode(c, scale):
    n = lambda t: None if t is None else t.cpu().numpy()  # noqa: E731
    return oracle.decode(bits(c["q"]), bits(c["kc"]), bits(c["vc"]), bits(c["kw"]), bits(c["vw"]),
                         c["seqlens"].cpu().numpy(), c["blk"], c["W"], scale, page_table=n(c["page_table"]),
                         page_size=c["page_size"], gq=n(c["gq"]), gk=n(c["gk"]), eps=1e-6,
                         gate=None if c["gate"] is None else bits(c["gate"]))


@pytest.mark.parametrize("r,lengths,gate,paged,norm", [
    (1, [9000, 130, 20000, 700], True, 0, False),
    (8, [131072, 5000, 1, 129, 70000], True, 0, False),
    (32, [4096 + 17, 300, 12345], True, 64, True),
    (5, [3000] * 40, False, 0, False),            # odd rank, no gate, many sequences (one piece each)
    (8, [1048576], True, 0, False),               # one long sequence: many pieces merged
])
def test_decode_vha_fused(cuda_device, libhca, r, lengths, gate, paged, norm):
    """Decode with the gate and Virtual Head Attention fused into the merge, against the oracle's
    gated decode followed by the oracle's mixing; and against the unfused hca_decode + hca_vha."""
    dev = cuda_device
    W = 256 if paged else 128
    c = _decode_case(dev, 120 + r + len(lengths), lengths, W=W, paged_ps=paged, norm=norm, gate=gate)
    U, V = factors(dev, 64, r, 130 + r)
    scale = 1.0 / np.sqrt(512)
    kw = dict(page_table=c["page_table"], page_size=c["page_size"], gq=c["gq"], gk=c["gk"], gate=c["gate"])
    fused = hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], c["blk"], W, scale,
                       vha_u=U, vha_v=V, **kw)
    plain = hca.decode(c["q"], c["kc"], c["vc"], c["kw"], c["vw"], c["seqlens"], c["blk"], W, scale, **kw)
    hca.vha(plain, U, V)
    torch.cuda.synchronize()
    hca.get_device_error()
    check(fused, oracle.vha(_oracle_decode(c, scale), U.cpu().numpy(), V.cpu().numpy()))
    # same arithmetic up to the order of a few fp32 sums
    assert (fused - plain).abs().max().item() <= 1e-5


def test_decode_vha_rejects_grouped_heads(cuda_device, libhca):
    c = _decode_case(cuda_device, 140, [3000, 700], Hq=64)
    U, V = factors(cuda_device, 64, 4, 141)
    kv2 = c["kc"].repeat(1, 1, 2, 1).contiguous()
    with pytest.raises(hca.HCAError):
        hca.decode(c["q"], kv2, kv2, c["kw"].repeat(1, 1, 2, 1).contiguous(), c["vw"].repeat(1, 1, 2, 1).contiguous(),
                   c["seqlens"], 128, 128, 0.05, vha_u=U, vha_v=V)
