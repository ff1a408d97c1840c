"""Pins of the fp64 backward oracle (oracle/backward.py), CPU only.

The backward is checked against things other than itself:
 - central finite differences of the fp64 forward, for every input (q, k, v, w) on tiny
   shapes, with and without grouped KV heads;
 - torch autograd of plain causal attention (fp64) in the two cases where the layer reduces
   to it: blocks of one token with zero weights (each past token is seen exactly once, as an
   entry or as a raw key), and a window covering the whole sequence (no entry is visible);
 - invariants: a block's weight gradients sum to zero (a common shift of the weights does not
   change the pooling); the value gradients sum to the output gradients of the heads reading
   that KV head (probabilities and pooling coefficients each sum to one); a query that sees
   only itself has zero query gradient.
The dense forward it differentiates is pinned to the C oracle's forward and pooling.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def rand(rs, *shape):
    return rs.standard_normal(shape)


def case(seed, B=1, T=11, Hq=2, Hkv=1, d=3, dv=2, wstd=1.0):
    rs = np.random.RandomState(seed)
    return (rand(rs, B, T, Hq, d), rand(rs, B, T, Hkv, d), rand(rs, B, T, Hkv, dv),
            rand(rs, B, T) * wstd, rand(rs, B, T, Hq, dv))


def loss(q, k, v, w, blk, W, scale, dout):
    return float((ob.forward(q, k, v, w, blk, W, scale) * dout).sum())


def finite_diff(f, x, eps=1e-6):
    g = np.zeros_like(x)
    for i in np.ndindex(*x.shape):
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("T,Hq,Hkv,blk,W", [(11, 2, 1, 2, 3), (13, 4, 2, 3, 4), (9, 2, 2, 4, 1), (8, 1, 1, 2, 8)])
def test_backward_matches_finite_differences(T, Hq, Hkv, blk, W):
    q, k, v, w, dout = case(T + 10 * Hq + blk, T=T, Hq=Hq, Hkv=Hkv)
    scale = 0.7
    dq, dk, dv, dw = ob.backward(q, k, v, w, blk, W, scale, dout)
    f = lambda: loss(q, k, v, w, blk, W, scale, dout)
    for got, x in ((dq, q), (dk, k), (dv, v), (dw, w)):
        np.testing.assert_allclose(got, finite_diff(f, x), rtol=1e-6, atol=1e-8)


def test_pool_backward_matches_finite_differences():
    rs = np.random.RandomState(3)
    k, v, w = rand(rs, 2, 10, 2, 3), rand(rs, 2, 10, 2, 4), rand(rs, 2, 10)
    dkc, dvc = rand(rs, 2, 3, 2, 3), rand(rs, 2, 3, 2, 4)     # blk 3: three blocks, one tail row
    f = lambda: float((ob.pool_f64(k, v, w, 3)[0] * dkc).sum() + (ob.pool_f64(k, v, w, 3)[1] * dvc).sum())
    dk, dv, dw = ob.pool_backward_f64(k, v, w, 3, dkc, dvc)
    for got, x in ((dk, k), (dv, v), (dw, w)):
        np.testing.assert_allclose(got, finite_diff(f, x), rtol=1e-6, atol=1e-8)
    assert np.all(dk[:, 9:] == 0) and np.all(dw[:, 9:] == 0)      # the tail row is never pooled


def causal_attention_grads(q, k, v, scale, dout):
    """torch autograd of causal softmax attention, fp64, KV heads shared by consecutive
    query heads."""
    Hq, Hkv = q.shape[2], k.shape[2]
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    rep = Hq // Hkv
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(1, 2), tk.repeat_interleave(rep, dim=2).transpose(1, 2),
        tv.repeat_interleave(rep, dim=2).transpose(1, 2), is_causal=True, scale=scale)
    (o.transpose(1, 2) * torch.tensor(dout)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("Hq,Hkv", [(2, 1), (4, 2)])
def test_one_token_blocks_are_causal_attention(Hq, Hkv):
    q, k, v, _, dout = case(21 + Hq, B=2, T=17, Hq=Hq, Hkv=Hkv, d=5, dv=4)
    dq, dk, dv, dw = ob.backward(q, k, v, None, 1, 3, 0.45, dout)
    tq, tk, tv = causal_attention_grads(q, k, v, 0.45, dout)
    for got, want in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    assert np.all(dw == 0)


def test_window_covering_the_sequence_is_causal_attention():
    q, k, v, w, dout = case(31, B=1, T=15, Hq=3, Hkv=1, d=4, dv=3)
    dq, dk, dv, dw = ob.backward(q, k, v, w, 4, 15, 0.5, dout)
    tq, tk, tv = causal_attention_grads(q, k, v, 0.5, dout)
    for got, want in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    assert np.all(dw == 0)     # no entry is ever visible


def test_weight_gradients_sum_to_zero_per_block():
    q, k, v, w, dout = case(41, B=2, T=20, Hq=2, Hkv=1, d=3, dv=3)
    _, _, _, dw = ob.backward(q, k, v, w, 4, 3, 0.6, dout)
    sums = dw.reshape(2, 5, 4).sum(axis=2)
    assert np.abs(sums).max() < 1e-13
    assert np.abs(dw).max() > 1e-3       # and the gradients themselves are not all zero


def test_value_gradients_sum_to_output_gradients():
    q, k, v, w, dout = case(51, B=1, T=19, Hq=4, Hkv=2, d=3, dv=5)
    _, _, dv, _ = ob.backward(q, k, v, w, 3, 4, 0.8, dout)
    for g in range(2):
        want = dout[:, :, 2 * g:2 * g + 2].sum(axis=(0, 1, 2))
        np.testing.assert_allclose(dv[:, :, g].sum(axis=(0, 1)), want, rtol=0, atol=1e-12)


def test_query_with_only_itself_has_zero_gradient():
    q, k, v, w, dout = case(61, T=6, Hq=2)
    dq, _, _, _ = ob.backward(q, k, v, w, 2, 3, 0.9, dout)
    # t = 0 sees one key: its output is v_0 for any q (zero up to the rounding of dO.v_0
    # computed two ways)
    assert np.abs(dq[:, 0]).max() < 1e-15
    assert np.abs(dq[:, 1:]).max() > 1e-3


def test_dense_forward_matches_c_oracle():
    """The dense mask forward equals the C oracle's row loop on bf16 inputs (entries pooled by
    the C oracle and rounded to bf16, as the cache stores them)."""
    g = torch.Generator().manual_seed(7)
    B, T, Hq, Hkv, d, dv, blk, W = 2, 70, 4, 2, 8, 6, 8, 10
    q = torch.randn((B, T, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, T, Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, T, Hkv, dv), generator=g).to(torch.bfloat16)
    w = torch.randn((B, T), generator=g) * 0.5
    kc, vc = oracle.compress(oracle.bf16_bits(k), oracle.bf16_bits(v), w.numpy(), blk)
    kcb, vcb = oracle.round_bf16(kc), oracle.round_bf16(vc)
    rows = [(b, t) for b in range(B) for t in range(T)]
    want = oracle.prefill_rows(oracle.bf16_bits(q), oracle.bf16_bits(k), oracle.bf16_bits(v), kcb, vcb, blk, W,
                               0.35, rows)
    got = ob.attend_f64(q.double().numpy(), k.double().numpy(), v.double().numpy(), oracle.bits_to_f64(kcb),
                        oracle.bits_to_f64(vcb), blk, W, 0.35)
    np.testing.assert_allclose(got.reshape(B * T, Hq, dv), want, rtol=0, atol=1e-12)
    # and the dense pooling equals the C oracle's
    pk, pv, _ = ob.pool_f64(k.double().numpy(), v.double().numpy(), w.double().numpy(), blk)
    np.testing.assert_allclose(pk, kc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(pv, vc, rtol=0, atol=1e-13)


@pytest.mark.parametrize("T,Hq,Hkv,blk,W", [(40, 4, 2, 4, 6), (37, 2, 1, 8, 3), (25, 3, 1, 1, 2)])
def test_sampled_backward_equals_dense(T, Hq, Hkv, blk, W):
    """The sampled form (only the queries that matter) gives the dense backward's values."""
    q, k, v, w, dout = case(70 + T, B=2, T=T, Hq=Hq, Hkv=Hkv, d=5, dv=3)
    scale = 0.6
    dq, dk, dv, dw = ob.backward(q, k, v, w, blk, W, scale, dout)
    kc, vc, _ = ob.pool_f64(k, v, w, blk)
    _, _, _, dkc, dvc = ob.attend_backward_f64(q, k, v, kc, vc, blk, W, scale, dout)
    Nc = T // blk
    rows = [0, 1, T // 2, T - 1]
    raw = sorted({0, blk - 1, blk, T // 2, T - 2, T - 1})
    entries = sorted({0, Nc // 2, Nc - 1}) if Nc else []
    for b in range(2):
        got = ob.backward_sampled(q, k, v, w, blk, W, scale, dout, b, rows=rows, raw=raw, entries=entries)
        for t in rows:
            np.testing.assert_allclose(got["dq"][t], dq[b, t], rtol=1e-12, atol=1e-13)
        for u in raw:
            np.testing.assert_allclose(got["dk"][u], dk[b, u], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(got["dv"][u], dv[b, u], rtol=1e-12, atol=1e-13)
            assert abs(got["dw"][u] - dw[b, u]) <= 1e-12 + 1e-12 * abs(dw[b, u])
        for j in entries:
            np.testing.assert_allclose(got["dkc"][j], dkc[b, j], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(got["dvc"][j], dvc[b, j], rtol=1e-12, atol=1e-13)
