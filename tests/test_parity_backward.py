"""GPU parity of hca_prefill_backward (through the C ABI) against the fp64 oracle.

The forward is hca_compress + hca_prefill (with the log-sum-exp); the oracle differentiates
the same layer in fp64 (oracle.backward): attend_backward_f64 over its own compressed cache,
rounded to bf16 as the stored cache is, then pool_backward_f64 through the pooling.  Nothing
the oracle reads comes from the CUDA path.

Bar, per gradient tensor X in (dq, dk, dv, dw): normwise ||X - ref||_2 <= 2^-7 ||ref||_2 and
elementwise max |X - ref| <= 2^-5 max |ref|.  Reading: the kernels round P (for dv) and
dS = P (dP - D) (for dq and dk) once to bf16 (relative 2^-9) before contractions over
hundreds of keys or queries; those roundings add up like a random walk, so the normwise error
is a small multiple of 2^-9, and single elements where the sum cancels are bounded against
the tensor's largest value instead of their own.  Where the exact gradient is zero everywhere
(a sequence of one token), the bar is 2^-13 absolute: fp32 rounding of two cancelling sums.
"""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle
from oracle import backward as ob

pytestmark = pytest.mark.gpu
NORM_TOL, MAX_TOL = 2.0 ** -7, 2.0 ** -5
ZERO_TOL = 2.0 ** -13


def bits(t):
    return oracle.bf16_bits(t)


def f64(t):
    """Exact fp64 values of a bf16 tensor."""
    return oracle.bits_to_f64(oracle.bf16_bits(t))


def check(got, ref, what):
    g = got.detach().double().cpu().numpy()
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    scale = np.abs(ref).max()
    if scale == 0:
        # an exactly zero gradient (a token that sees only itself: dP and D are the same sum)
        # comes out as the difference of two fp32 sums of 512 terms formed along different paths
        assert err.max() <= ZERO_TOL, (what, err.max())
        return
    rel = np.sqrt((err ** 2).sum() / (ref ** 2).sum())
    assert rel <= NORM_TOL, (what, "normwise", rel)
    assert err.max() <= MAX_TOL * scale, (what, "max", err.max(), scale)


def inputs(dev, B, T, Hq, Hkv, seed, wstd=0.5, zero_w=False, boost=0):
    g = torch.Generator(device=dev).manual_seed(seed)
    d = 512
    q = torch.randn((B, T, Hq, d), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((B, T, Hkv, d), generator=g, device=dev).to(torch.bfloat16)
    if boost:
        # every boost-th raw key row times 8 (exact in bf16): softmax rows dominated by one key
        k[:, ::boost] = (k[:, ::boost].float() * 8).to(torch.bfloat16)
    v = torch.randn((B, T, Hkv, d), generator=g, device=dev).to(torch.bfloat16)
    w = None if zero_w else torch.randn((B, T), generator=g, device=dev) * wstd
    dout = torch.randn((B, T, Hq, d), generator=g, device=dev).to(torch.bfloat16)
    return q, k, v, w, dout


def gpu_grads(q, k, v, w, dout, blk, W, scale, out_f32=True):
    kc, vc = hca.compress(k, v, w, blk)
    out, lse = hca.prefill(q, k, v, kc, vc, blk, W, scale, want_lse=True, out_f32=out_f32)
    dq, dk, dv, dw = hca.prefill_backward(q, k, v, w, kc, vc, out, lse, dout, blk, W, scale)
    torch.cuda.synchronize()
    hca.get_device_error()
    return dq, dk, dv, dw


def oracle_grads(q, k, v, w, dout, blk, W, scale):
    wn = None if w is None else w.cpu().numpy()
    kc, vc = oracle.compress(bits(k), bits(v), wn, blk)
    kcb, vcb = oracle.bits_to_f64(oracle.round_bf16(kc)), oracle.bits_to_f64(oracle.round_bf16(vc))
    qb, kb, vb = f64(q), f64(k), f64(v)
    dq, dk_w, dv_w, dkc, dvc = ob.attend_backward_f64(qb, kb, vb, kcb, vcb, blk, W, scale, f64(dout))
    dk_p, dv_p, dw = ob.pool_backward_f64(kb, vb, wn, blk, dkc, dvc)
    return dq, dk_w + dk_p, dv_w + dv_p, dw


def run_case(dev, B, T, Hq, Hkv, blk, W, seed, out_f32=True, wstd=0.5, zero_w=False, boost=0):
    q, k, v, w, dout = inputs(dev, B, T, Hq, Hkv, seed, wstd, zero_w, boost)
    scale = 1.0 / np.sqrt(512)
    got = gpu_grads(q, k, v, w, dout, blk, W, scale, out_f32)
    ref = oracle_grads(q, k, v, w, dout, blk, W, scale)
    for name, g_, r_ in zip(("dq", "dk", "dv", "dw"), got, ref):
        check(g_, r_, name)


@pytest.mark.parametrize("B,T,Hq,Hkv,blk,W", [
    (1, 640, 64, 1, 128, 128),    # the model's head layout: 64 query heads on one KV head
    (2, 1000, 16, 2, 32, 200),    # two KV groups, window over two key tiles, ragged tail
    (1, 700, 4, 1, 1, 64),        # one entry per token: six tiles of compressed keys
    (1, 300, 2, 2, 16, 200),      # one head per group: 128 tokens per row tile
    (1, 131, 128, 1, 8, 17),      # 128 heads per group: one token per row tile
])
def test_backward_d512(cuda_device, libhca, B, T, Hq, Hkv, blk, W):
    run_case(cuda_device, B, T, Hq, Hkv, blk, W, seed=3 * T + Hq, out_f32=(T % 2 == 0))


def test_backward_boosted_keys(cuda_device, libhca):
    """One raw key in 97 scaled by 8 (the prefill workload's boosted keys): rows whose softmax
    one key dominates, where dS = P (dP - D) cancels; fp32 forward output."""
    run_case(cuda_device, 1, 1000, 64, 1, 128, 128, seed=41, out_f32=True, boost=97)


@pytest.mark.parametrize("B,T,Hq,Hkv,blk,W,zero_w", [
    (1, 1, 64, 1, 128, 128, False),    # a single token: it sees only itself
    (1, 100, 64, 1, 128, 50, False),   # shorter than a block: no entry, dw = 0
    (1, 256, 64, 1, 128, 128, False),  # the last row sees exactly one entry
    (2, 384, 32, 1, 128, 128, True),   # mean pooling (w = NULL)
])
def test_backward_edges(cuda_device, libhca, B, T, Hq, Hkv, blk, W, zero_w):
    run_case(cuda_device, B, T, Hq, Hkv, blk, W, seed=5 * T + B, zero_w=zero_w)


def test_backward_long_sampled(cuda_device, libhca):
    """T = 20000, 64 heads on one KV head: two tiles of compressed keys and 10000 row tiles;
    dq of sampled rows, and dk / dv / dw of raw rows in the ragged tail (window path only) and
    in a late complete block (window + pooling path), from oracle.backward.backward_sampled."""
    B, T, Hq, Hkv, blk, W = 1, 20000, 64, 1, 128, 128
    q, k, v, w, dout = inputs(cuda_device, B, T, Hq, Hkv, seed=17)
    scale = 1.0 / np.sqrt(512)
    dq, dk, dv, dw = gpu_grads(q, k, v, w, dout, blk, W, scale)
    rows = [0, 127, 128, 255, 16511, 16512, 19999]
    Nc = T // blk
    raw = [19970, 19999, blk * (Nc - 3), blk * (Nc - 3) + 77]
    qn, kn, vn, don = f64(q), f64(k), f64(v), f64(dout)
    ref = ob.backward_sampled(qn, kn, vn, w.cpu().numpy(), blk, W, scale, don, 0, rows=rows, raw=raw)
    check(dq[0, rows], np.stack([ref["dq"][t] for t in rows]), "dq")
    check(dk[0, raw], np.stack([ref["dk"][u] for u in raw]), "dk")
    check(dv[0, raw], np.stack([ref["dv"][u] for u in raw]), "dv")
    got_dw = dw[0, raw].double().cpu().numpy()
    ref_dw = np.array([ref["dw"][u] for u in raw])
    assert np.abs(got_dw - ref_dw).max() <= MAX_TOL * max(np.abs(ref_dw).max(), 1e-30) + 1e-6


def test_backward_rejects_unsupported(cuda_device, libhca):
    q, k, v, w, dout = inputs(cuda_device, 1, 256, 64, 1, seed=1)
    kc, vc = hca.compress(k, v, w, 128)
    out, lse = hca.prefill(q, k, v, kc, vc, 128, 128, 0.05, want_lse=True)
    with pytest.raises(hca.HCAError):
        hca.prefill_backward(q, k, v, w, kc, vc, out, lse, dout, 256, 128, 0.05)   # blk > 128


@pytest.mark.parametrize("seg,B,T,Hq,Hkv,blk,W", [
    (5, 1, 640, 64, 1, 128, 128),
    (3, 2, 1000, 16, 2, 32, 200),
])
def test_backward_segments(cuda_device, libhca, seg, B, T, Hq, Hkv, blk, W):
    """Long sequences are processed in segments of row tiles (the P / dS records of one segment
    at a time); forcing a few row tiles per segment walks the same path on a short sequence."""
    assert libhca.hca_debug_set_backward_segment(seg) == 0
    try:
        run_case(cuda_device, B, T, Hq, Hkv, blk, W, seed=7 * T + seg)
    finally:
        assert libhca.hca_debug_set_backward_segment(0) == 0
