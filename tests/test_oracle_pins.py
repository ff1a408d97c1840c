"""Pins for the fp64 CPU oracle: closed forms, invariants, a hand-worked example,
library special cases and an independent dense brute force.  CPU only.

Each check is chosen so that a plausible slip in the oracle (a dropped segment,
an off-by-one in the visible-entry count, a wrong softmax sign, a transposed
operand, a wrong norm constant) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.oracle_bruteforce import (bits_to_f64, hca_prefill_bruteforce, pool_numpy, to_bf16_f64,
                                     visibility)


def rand_bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(shape, generator=g) * std).to(torch.bfloat16)
    return oracle.bf16_bits(x)


def rand_w(shape, seed, std=0.5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).numpy().astype(np.float32)


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_float32_rounding():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(100000, generator=g) * torch.exp(torch.randn(100000, generator=g) * 8)
    ref = oracle.bf16_bits(x.to(torch.bfloat16))
    got = oracle.round_bf16(x.double().numpy())
    assert np.array_equal(ref, got)


def test_round_bf16_ties_and_double_rounding():
    one = 1.0
    cases = {
        one + 2.0 ** -8: one,                       # tie -> even (1.0)
        one + 3 * 2.0 ** -8: one + 2.0 ** -6,       # tie -> even (1 + 2^-6)
        one + 2.0 ** -8 + 2.0 ** -40: one + 2.0 ** -7,   # just above the tie: direct rounding goes up
        -(one + 2.0 ** -8 + 2.0 ** -40): -(one + 2.0 ** -7),
        0.0: 0.0,
    }
    xs = np.array(list(cases.keys()))
    want = np.array(list(cases.values()))
    got = bits_to_f64(oracle.round_bf16(xs))
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- visible entries

@pytest.mark.parametrize("t,W,blk,want", [
    (131071, 128, 128, 1023),     # 128K decode: 1023 entries
    (1048575, 128, 128, 8191),    # 1M decode: 8191 entries
    (126, 128, 128, 0), (127, 128, 128, 0), (254, 128, 128, 0), (255, 128, 128, 1),
    (0, 1, 1, 0), (9, 1, 1, 9), (9, 3, 1, 7), (5, 2, 2, 2), (4, 2, 2, 1), (2, 2, 2, 0),
])
def test_visible_entries_closed_form(t, W, blk, want):
    assert oracle.visible_entries(t, W, blk) == want


# ---------------------------------------------------------------- compression

def test_compress_zero_weights_is_mean():
    k = rand_bf16((2, 384 + 50, 2, 64), 1)
    v = rand_bf16((2, 384 + 50, 2, 32), 2)
    kc, vc = oracle.compress(k, v, None, 128)
    kf, vf = bits_to_f64(k), bits_to_f64(v)
    assert kc.shape == (2, 3, 2, 64) and vc.shape == (2, 3, 2, 32)
    np.testing.assert_allclose(kc, kf[:, :384].reshape(2, 3, 128, 2, 64).mean(axis=2), rtol=0, atol=1e-14)
    np.testing.assert_allclose(vc, vf[:, :384].reshape(2, 3, 128, 2, 32).mean(axis=2), rtol=0, atol=1e-14)
    # explicit zero weights == NULL weights
    kc2, _ = oracle.compress(k, v, np.zeros((2, 434), np.float32), 128)
    assert np.array_equal(kc, kc2)


def test_compress_cache_ratio_and_partial_tail_unused():
    T = 1024 + 77
    k = rand_bf16((1, T, 1, 64), 3)
    v = rand_bf16((1, T, 1, 64), 4)
    w = rand_w((1, T), 5)
    kc, vc = oracle.compress(k, v, w, 128)
    assert kc.shape[1] == 1024 // 128 == 8
    # a compressed entry per 128 raw tokens: 1/128 of the rows
    assert kc.shape[1] * 128 == 1024
    # changing the partial tail (and its weights) changes nothing
    k2, v2, w2 = k.copy(), v.copy(), w.copy()
    k2[:, 1024:] = rand_bf16((1, 77, 1, 64), 6)
    w2[:, 1024:] = 9.0
    kc2, vc2 = oracle.compress(k2, v2, w2, 128)
    assert np.array_equal(kc, kc2) and np.array_equal(vc, vc2)


def test_compress_constant_rows_give_the_constant():
    T = 256
    row = rand_bf16((64,), 7)
    k = np.tile(row, (1, T, 1, 1)).reshape(1, T, 1, 64)
    w = rand_w((1, T), 8, std=3.0)
    kc, vc = oracle.compress(k, k, w, 128)
    np.testing.assert_allclose(kc, np.broadcast_to(bits_to_f64(row), kc.shape), rtol=1e-15, atol=0)


def test_compress_weight_shift_invariance():
    T = 512
    k = rand_bf16((1, T, 1, 64), 9)
    w = rand_w((1, T), 10)
    kc, _ = oracle.compress(k, k, w, 128)
    shift = np.repeat(np.array([3.0, -7.0, 0.5, 11.0], np.float32), 128)[None]
    kc2, _ = oracle.compress(k, k, (w.astype(np.float64) + shift).astype(np.float32), 128)
    # fp32 shifted weights carry their own rounding; the pooled result must agree closely
    np.testing.assert_allclose(kc, kc2, rtol=0, atol=5e-6)
    kc3, _ = oracle.compress(k, k, w + np.float32(0.0), 128)
    assert np.array_equal(kc, kc3)


def test_compress_permutation_invariance():
    T = 256
    k = rand_bf16((1, T, 1, 64), 11)
    w = rand_w((1, T), 12)
    perm = np.concatenate([np.random.RandomState(0).permutation(128), 128 + np.random.RandomState(1).permutation(128)])
    kc, _ = oracle.compress(k, k, w, 128)
    kc2, _ = oracle.compress(np.ascontiguousarray(k[:, perm]), np.ascontiguousarray(k[:, perm]),
                             np.ascontiguousarray(w[:, perm]), 128)
    np.testing.assert_allclose(kc, kc2, rtol=0, atol=1e-13)


def test_compress_dominant_weight_selects_row():
    T = 256
    k = rand_bf16((1, T, 1, 64), 13)
    w = rand_w((1, T), 14, std=1.0)
    w[0, 37] = 80.0
    w[0, 128 + 100] = 75.0
    kc, _ = oracle.compress(k, k, w, 128)
    kf = bits_to_f64(k)
    np.testing.assert_allclose(kc[0, 0, 0], kf[0, 37, 0], rtol=0, atol=1e-20)
    np.testing.assert_allclose(kc[0, 1, 0], kf[0, 228, 0], rtol=0, atol=1e-20)


def test_compress_two_row_closed_form():
    # blk = 2, weights (0, ln 3): alpha = (1/4, 3/4)
    k = oracle.round_bf16(np.array([[[[1.0, 4.0]], [[5.0, -8.0]]]]))
    w = np.array([[0.0, math.log(3.0)]], np.float32)
    kc, _ = oracle.compress(k, k, w, 2)
    a1 = 3.0 * math.exp(float(np.float32(math.log(3.0))) - math.log(3.0))
    want = np.array([(1.0 + a1 * 5.0) / (1 + a1), (4.0 - a1 * 8.0) / (1 + a1)])
    np.testing.assert_allclose(kc[0, 0, 0], want, rtol=1e-14)
    np.testing.assert_allclose(kc[0, 0, 0], [4.0, -5.0], rtol=1e-7)


def test_compress_block_one_is_copy():
    k = rand_bf16((2, 33, 2, 64), 15)
    kc, _ = oracle.compress(k, k, rand_w((2, 33), 16), 1)
    assert np.array_equal(kc, bits_to_f64(k))


def test_compress_matches_numpy_pooling():
    k = rand_bf16((2, 640, 2, 64), 17)
    w = rand_w((2, 640), 18, std=2.0)
    kc, _ = oracle.compress(k, k, w, 128)
    np.testing.assert_allclose(kc, pool_numpy(bits_to_f64(k), w, 128), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- attention helpers

def make_prefill(B, T, Hq, Hkv, d, dv, seed, w_zero=False):
    q = rand_bf16((B, T, Hq, d), seed)
    k = rand_bf16((B, T, Hkv, d), seed + 1)
    v = rand_bf16((B, T, Hkv, dv), seed + 2)
    w = np.zeros((B, T), np.float32) if w_zero else rand_w((B, T), seed + 3)
    return q, k, v, w


def oracle_prefill_all(q, k, v, w, blk, W, scale, want_lse=False):
    B, T = q.shape[:2]
    kc, vc = oracle.compress(k, v, w, blk)
    kcb, vcb = oracle.round_bf16(kc), oracle.round_bf16(vc)
    rows = [(b, t) for b in range(B) for t in range(T)]
    res = oracle.prefill_rows(q, k, v, kcb, vcb, blk, W, scale, rows, want_lse=want_lse)
    if want_lse:
        out, lse = res
        return out.reshape(B, T, *out.shape[1:]), lse.reshape(B, T, -1)
    return res.reshape(B, T, *res.shape[1:])


def sdpa_causal(q, k, v, scale):
    """torch's scaled_dot_product_attention in fp64 (library special case), GQA by repeat."""
    qt = torch.from_numpy(bits_to_f64(q)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(bits_to_f64(k)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(bits_to_f64(v)).permute(0, 2, 1, 3)
    rep = qt.shape[1] // kt.shape[1]
    kt = kt.repeat_interleave(rep, dim=1)
    vt = vt.repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- attention pins

def test_window_covers_everything_is_full_causal_attention():
    B, T, Hq, Hkv, d = 2, 200, 4, 2, 64
    q, k, v, w = make_prefill(B, T, Hq, Hkv, d, d, 20)
    out = oracle_prefill_all(q, k, v, w, 128, W=T, scale=0.125)
    np.testing.assert_allclose(out, sdpa_causal(q, k, v, 0.125), rtol=0, atol=1e-12)


@pytest.mark.parametrize("W", [1, 3, 17])
def test_block_one_zero_weights_is_full_causal_attention(W):
    B, T, Hq, Hkv, d = 1, 96, 2, 1, 64
    q, k, v, w = make_prefill(B, T, Hq, Hkv, d, d, 30, w_zero=True)
    out = oracle_prefill_all(q, k, v, w, 1, W=W, scale=0.125)
    np.testing.assert_allclose(out, sdpa_causal(q, k, v, 0.125), rtol=0, atol=1e-12)


def test_all_ones_values_give_ones():
    # softmax rows sum to one: with V = 1 (so every pooled entry is 1) the output is exactly 1
    B, T, Hq, Hkv, d = 1, 700, 4, 1, 64
    q, k, _, w = make_prefill(B, T, Hq, Hkv, d, d, 40)
    v = oracle.round_bf16(np.ones((B, T, Hkv, 32)))
    out = oracle_prefill_all(q, k, v, w, 128, W=128, scale=0.125)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)


@pytest.mark.parametrize("T,W,blk,Hq,Hkv", [(512, 128, 128, 4, 1), (300, 40, 16, 4, 2), (257, 1, 2, 2, 1),
                                            (130, 200, 128, 2, 1), (64, 5, 3, 3, 1)])
def test_matches_dense_bruteforce(T, W, blk, Hq, Hkv):
    B, d, dv = 2, 64, 48
    q, k, v, w = make_prefill(B, T, Hq, Hkv, d, dv, 50 + T)
    out, lse = oracle_prefill_all(q, k, v, w, blk, W, scale=0.11, want_lse=True)
    bo, bl = hca_prefill_bruteforce(bits_to_f64(q), bits_to_f64(k), bits_to_f64(v), w, blk, W, 0.11)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-11)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-11)


def test_hand_worked_example():
    """T=6, blk=2, W=2, d=dv=1-dim keys, scale 1.  Key sets enumerated by hand:
      t=0: raw {0}            t=1: raw {0,1}          t=2: raw {1,2} (pos 0 in the gap)
      t=3: entry0 + raw {2,3} t=4: entry0 + raw {3,4} (pos 2 in the gap)
      t=5: entry0, entry1 + raw {4,5}
    with q = 1, k_u in {0, 1} so logits are 0 or 1, v_u = u, zero pooling weights.
    """
    kv = [0.0, 1.0, 1.0, 0.0, 1.0, 0.0]
    k = oracle.round_bf16(np.array(kv).reshape(1, 6, 1, 1))
    v = oracle.round_bf16(np.arange(6.0).reshape(1, 6, 1, 1))
    q = oracle.round_bf16(np.ones((1, 6, 1, 1)))
    out = oracle_prefill_all(q, k, v, np.zeros((1, 6), np.float32), 2, 2, 1.0)[0, :, 0, 0]
    e = math.e
    # entry0 = mean of positions 0,1: k = 0.5, v = 0.5; entry1 = positions 2,3: k = 0.5, v = 2.5
    es = math.exp(0.5)
    want = [
        0.0,
        (1 * 0 + e * 1) / (1 + e),
        (e * 1 + e * 2) / (2 * e),
        (es * 0.5 + e * 2 + 1 * 3) / (es + e + 1),
        (es * 0.5 + 1 * 3 + e * 4) / (es + 1 + e),
        (es * 0.5 + es * 2.5 + e * 4 + 1 * 5) / (2 * es + e + 1),
    ]
    np.testing.assert_allclose(out, want, rtol=1e-14)


def test_visibility_mask_entry_count_agrees_with_closed_form():
    # the brute force's semantic mask and the oracle's closed form count the same entries
    for (T, W, blk) in [(700, 128, 128), (300, 1, 7), (50, 60, 4)]:
        m = visibility(T, W, blk)
        Nc = T // blk
        for t in range(T):
            assert m[t, :Nc].sum() == oracle.visible_entries(t, W, blk)
            assert m[t, Nc:].sum() == min(W, t + 1)


# ---------------------------------------------------------------- decode pins

def decode_from_raw(q_last, k, v, w, blk, W, L, scale, **opts):
    """Decode of one query per sequence at position L-1 with the cache pooled by the oracle."""
    B = k.shape[0]
    kc, vc = oracle.compress(k[:, :L], v[:, :L], w[:, :L], blk)
    kcb, vcb = oracle.round_bf16(kc), oracle.round_bf16(vc)
    kw = np.zeros((B, W) + k.shape[2:], np.uint16)
    vw = np.zeros((B, W) + v.shape[2:], np.uint16)
    n = min(W, L)
    kw[:, W - n:] = k[:, L - n:L]
    vw[:, W - n:] = v[:, L - n:L]
    seq = np.full((B,), L, np.int32)
    return oracle.decode(q_last, kcb, vcb, kw, vw, seq, blk, W, scale, **opts), (kcb, vcb, kw, vw, seq)


@pytest.mark.parametrize("L,W", [(1000, 128), (700, 256), (90, 128), (129, 1), (256, 128)])
def test_decode_equals_last_prefill_row(L, W):
    B, Hq, Hkv, d, dv = 2, 4, 2, 64, 32
    q, k, v, w = make_prefill(B, L, Hq, Hkv, d, dv, 60 + L)
    pre = oracle_prefill_all(q, k, v, w, 128, W, 0.1)
    dec, _ = decode_from_raw(np.ascontiguousarray(q[:, L - 1]), k, v, w, 128, W, L, 0.1)
    np.testing.assert_allclose(dec, pre[:, L - 1], rtol=0, atol=1e-13)


def test_paged_equals_contiguous():
    B, Hq, Hkv, d, dv, W, L = 3, 4, 1, 64, 64, 128, 5000
    q, k, v, w = make_prefill(B, L, Hq, Hkv, d, dv, 70)
    ql = np.ascontiguousarray(q[:, L - 1])
    ref, (kcb, vcb, kw, vw, seq) = decode_from_raw(ql, k, v, w, 128, W, L, 0.1)
    Nmax, ps = kcb.shape[1], 8
    npg = (Nmax + ps - 1) // ps
    perm = np.random.RandomState(3).permutation(B * npg)
    pool_k = np.zeros((B * npg, ps, Hkv, d), np.uint16)
    pool_v = np.zeros((B * npg, ps, Hkv, dv), np.uint16)
    table = np.zeros((B, npg), np.int32)
    for b in range(B):
        for p in range(npg):
            pg = perm[b * npg + p]
            table[b, p] = pg
            n = min(ps, Nmax - p * ps)
            pool_k[pg, :n] = kcb[b, p * ps:p * ps + n]
            pool_v[pg, :n] = vcb[b, p * ps:p * ps + n]
    got = oracle.decode(ql, pool_k, pool_v, kw, vw, seq, 128, W, 0.1, page_table=table, page_size=ps)
    np.testing.assert_array_equal(got, ref)


def _small_decode_case(seed, L=900, W=64, B=2, Hq=4, d=64, dv=32):
    q = rand_bf16((B, Hq, d), seed)
    kc = rand_bf16((B, L // 128, 1, d), seed + 1)
    vc = rand_bf16((B, L // 128, 1, dv), seed + 2)
    kw = rand_bf16((B, W, 1, d), seed + 3)
    vw = rand_bf16((B, W, 1, dv), seed + 4)
    seq = np.full((B,), L, np.int32)
    return q, kc, vc, kw, vw, seq


def test_qk_norm_scale_invariance():
    q, kc, vc, kw, vw, seq = _small_decode_case(80)
    gq = np.random.RandomState(0).uniform(0.5, 1.5, 64).astype(np.float32)
    gk = np.random.RandomState(1).uniform(0.5, 1.5, 64).astype(np.float32)
    base = oracle.decode(q, kc, vc, kw, vw, seq, 128, 64, 0.125, gq=gq, gk=gk, eps=0.0)
    # scale every key by its own power of two and every query head too (exact in bf16)
    rs = np.random.RandomState(2)
    kc2 = oracle.round_bf16(bits_to_f64(kc) * 2.0 ** rs.randint(-3, 4, size=kc.shape[:3] + (1,)))
    kw2 = oracle.round_bf16(bits_to_f64(kw) * 2.0 ** rs.randint(-3, 4, size=kw.shape[:3] + (1,)))
    q2 = oracle.round_bf16(bits_to_f64(q) * 2.0 ** rs.randint(-3, 4, size=q.shape[:2] + (1,)))
    got = oracle.decode(q2, kc2, vc, kw2, vw, seq, 128, 64, 0.125, gq=gq, gk=gk, eps=0.0)
    np.testing.assert_allclose(got, base, rtol=0, atol=1e-13)
    # the gains enter symmetrically
    swp = oracle.decode(q, kc, vc, kw, vw, seq, 128, 64, 0.125, gq=gk, gk=gq, eps=0.0)
    np.testing.assert_allclose(swp, base, rtol=0, atol=1e-13)
    # and without the norm, the scaling does change the result
    a = oracle.decode(q, kc, vc, kw, vw, seq, 128, 64, 0.125)
    b = oracle.decode(q2, kc2, vc, kw2, vw, seq, 128, 64, 0.125)
    assert np.abs(a - b).max() > 1e-3


def test_qk_norm_two_key_closed_form():
    """Two raw keys k1 = 4 q and k2 = -q/2 (exact in bf16), unit gains, eps 0: after RMSNorm the
    logits are +-scale*d, so p1 = 1 / (1 + exp(-2*scale*d))."""
    d = 64
    qv = bits_to_f64(rand_bf16((d,), 90))
    q = oracle.round_bf16(qv.reshape(1, 1, d))
    kw = oracle.round_bf16(np.stack([4.0 * qv, -0.5 * qv]).reshape(1, 2, 1, d))
    vw = oracle.round_bf16(np.array([1.0, -2.0]).reshape(1, 2, 1, 1))
    kc = np.zeros((1, 1, 1, d), np.uint16)
    vc = np.zeros((1, 1, 1, 1), np.uint16)
    ones = np.ones(d, np.float32)
    scale = 0.01
    out = oracle.decode(q, kc, vc, kw, vw, np.array([2], np.int32), 128, 2, scale, gq=ones, gk=ones, eps=0.0)
    p1 = 1.0 / (1.0 + math.exp(-2 * scale * d))
    np.testing.assert_allclose(out[0, 0, 0], p1 * 1.0 + (1 - p1) * -2.0, rtol=1e-13)


def test_gate_limits():
    q, kc, vc, kw, vw, seq = _small_decode_case(100)
    base = oracle.decode(q, kc, vc, kw, vw, seq, 128, 64, 0.125)
    zero = np.zeros((2, 4, 32), np.uint16)
    half = oracle.decode(q, kc, vc, kw, vw, seq, 128, 64, 0.125, gate=zero)
    np.testing.assert_allclose(half, 0.5 * base, rtol=0, atol=1e-15)
    big = oracle.round_bf16(np.full((2, 4, 32), 40.0))
    open_ = oracle.decode(q, kc, vc, kw, vw, seq, 128, 64, 0.125, gate=big)
    np.testing.assert_allclose(open_, base, rtol=1e-15, atol=1e-15)


def test_decode_lse_matches_bruteforce():
    B, L, Hq, Hkv, d, dv, W = 1, 400, 4, 1, 64, 64, 100
    q, k, v, w = make_prefill(B, L, Hq, Hkv, d, dv, 110)
    (out, lse), _ = decode_from_raw(np.ascontiguousarray(q[:, L - 1]), k, v, w, 128, W, L, 0.1,
                                    want_lse=True)
    bo, bl = hca_prefill_bruteforce(bits_to_f64(q), bits_to_f64(k), bits_to_f64(v), w, 128, W, 0.1)
    np.testing.assert_allclose(out, bo[:, L - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl[:, L - 1], rtol=0, atol=1e-12)


def test_decode_rejects_short_cache():
    q, kc, vc, kw, vw, seq = _small_decode_case(120)
    with pytest.raises(ValueError):
        oracle.decode(q, kc[:, :3], vc[:, :3], kw, vw, seq, 128, 64, 0.125)


# ------------------------------------------------------------------ VHA (cross-head mixing)

def test_vha_zero_factor_is_identity():
    rs = np.random.RandomState(0)
    o = rs.randn(3, 8, 16)
    U = rs.randn(8, 2).astype(np.float32)
    np.testing.assert_array_equal(oracle.vha(o, U, np.zeros_like(U)), o)
    np.testing.assert_array_equal(oracle.vha(o, np.zeros_like(U), U), o)


def test_vha_rank_one_closed_form():
    """U = e_i, V = e_j: head i gains head j's output, every other head is unchanged."""
    rs = np.random.RandomState(1)
    o = rs.randn(2, 6, 5)
    U = np.zeros((6, 1), np.float32)
    V = np.zeros((6, 1), np.float32)
    U[4, 0] = 1.0
    V[1, 0] = 1.0
    got = oracle.vha(o, U, V)
    want = o.copy()
    want[:, 4] += o[:, 1]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_vha_factor_gauge_invariance():
    """(U A, V A^-T) is the same mixing matrix as (U, V) for any invertible A."""
    rs = np.random.RandomState(2)
    o = rs.randn(4, 16, 7)
    U = rs.randn(16, 3)
    V = rs.randn(16, 3)
    A = rs.randn(3, 3) + 3 * np.eye(3)
    got = oracle.vha(o, U @ A, V @ np.linalg.inv(A).T)
    np.testing.assert_allclose(got, oracle.vha(o, U, V), rtol=1e-11, atol=1e-11)


def test_vha_equals_dense_mixing_matrix():
    """Channel by channel, the result is the dense (I + U V^T) applied to the head vector."""
    rs = np.random.RandomState(3)
    o = rs.randn(2, 12, 9)
    U = rs.randn(12, 4).astype(np.float32)
    V = rs.randn(12, 4).astype(np.float32)
    M = np.eye(12) + U.astype(np.float64) @ V.astype(np.float64).T
    want = np.stack([np.stack([M @ o[n, :, c] for c in range(9)], axis=1) for n in range(2)])
    np.testing.assert_allclose(oracle.vha(o, U, V), want, rtol=1e-12, atol=1e-12)



def test_prefill_rows_rejects_rows_outside_the_batch():
    z = np.zeros((1, 8, 1, 4), np.uint16)
    zc = np.zeros((1, 2, 1, 4), np.uint16)
    for bad in ([(1, 0)], [(0, 8)], [(-1, 3)], [(0, -1)]):
        with pytest.raises(ValueError):
            oracle.prefill_rows(z, z, z, zc, zc, 4, 2, 1.0, bad)
    oracle.prefill_rows(z, z, z, zc, zc, 4, 2, 1.0, [(0, 7)])
