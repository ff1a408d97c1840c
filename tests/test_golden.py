"""The oracle against the hand-worked fixtures under tests/golden/ (CPU).

visibility_T12_blk4_W3.txt: which keys every query sees.  The C oracle is probed with K = 0
(every visible logit equal) and one-hot values (value channel c marks key c), so each output
row is uniform exactly over the keys that query attends to; the support is compared with the
hand enumeration, for prefill rows and for decode at L = t + 1.
compress_two_rows.txt: the pooled entry of a two-row block with weights 0 and ln 3.
"""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rows_of(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def parse_set(s):
    s = s.strip()
    return [] if s == "-" else [int(x) for x in s.split()]


def visibility_fixture():
    out = {}
    for ln in rows_of("visibility_T12_blk4_W3.txt"):
        t, ent, raw = ln.split("|")
        out[int(t)] = (parse_set(ent), parse_set(raw))
    return out


T, BLK, W, D = 12, 4, 3, 8
NC = T // BLK


def one_hot_bits(n_keys, offset, count):
    """[1, count, 1, n_keys] bf16 bits: row i is the unit vector e_(offset + i)."""
    x = np.zeros((1, count, 1, n_keys))
    for i in range(count):
        x[0, i, 0, offset + i] = 1.0
    return oracle.round_bf16(x)


def support(row):
    ent = [c for c in range(NC) if row[c] > 0]
    raw = [c - NC for c in range(NC, NC + T) if row[c] > 0]
    return ent, raw


def test_visibility_fixture_prefill():
    want = visibility_fixture()
    assert sorted(want) == list(range(T))
    nk = NC + T
    zeros = lambda *s: np.zeros(s, np.uint16)
    v = one_hot_bits(nk, NC, T)
    vc = one_hot_bits(nk, 0, NC)
    out = oracle.prefill_rows(zeros(1, T, 1, D), zeros(1, T, 1, D), v, zeros(1, NC, 1, D), vc, BLK, W, 1.0,
                              [(0, t) for t in range(T)])
    for t in range(T):
        row = out[t, 0]
        ent, raw = support(row)
        assert (ent, raw) == want[t], t
        n = len(ent) + len(raw)
        np.testing.assert_allclose(row[row > 0], 1.0 / n, rtol=0, atol=1e-15)
        assert oracle.visible_entries(t, W, BLK) == len(want[t][0])


def test_visibility_fixture_decode():
    """Decode at length L = t + 1 sees the same keys; its window is the last W slots of the
    raw ring, oldest first."""
    want = visibility_fixture()
    nk = NC + T
    for t in range(T):
        L = t + 1
        kw = np.zeros((1, W, 1, D), np.uint16)
        vw = np.zeros((1, W, 1, nk))
        for i in range(W):                   # slot i holds position L - W + i (negative: unused)
            p = L - W + i
            if p >= 0:
                vw[0, i, 0, NC + p] = 1.0
        vc = one_hot_bits(nk, 0, NC)
        out = oracle.decode(np.zeros((1, 1, D), np.uint16), np.zeros((1, NC, 1, D), np.uint16), vc, kw,
                            oracle.round_bf16(vw), np.array([L], np.int32), BLK, W, 1.0)
        assert support(out[0, 0]) == want[t], t


def test_compress_two_rows_fixture():
    vals = {}
    for ln in rows_of("compress_two_rows.txt"):
        key, rest = ln.split(":")
        vals[key] = rest.split()
    w = np.array([[0.0 if x == "0" else np.log(3.0) for x in vals["w"]]], np.float32)
    k = np.array([[[[float(x) for x in vals["k0"]]], [[float(x) for x in vals["k1"]]]]])
    v = np.array([[[[float(x) for x in vals["v0"]]], [[float(x) for x in vals["v1"]]]]])
    kc, vc = oracle.compress(oracle.round_bf16(k), oracle.round_bf16(v), w, 2)
    # the weight ln 3 is rounded to fp32; alpha moves by at most ~1e-7 from 3/4
    np.testing.assert_allclose(kc[0, 0, 0], [float(x) for x in vals["kc"]], rtol=0, atol=1e-6)
    np.testing.assert_allclose(vc[0, 0, 0], [float(x) for x in vals["vc"]], rtol=0, atol=1e-6)


def test_low_rank_gate_fixture():
    """The gate projection maps the query latent (not the hidden state) to one logit per head
    and channel; with the pages' dimensions that is 75% fewer weights."""
    dims = {}
    for ln in rows_of("low_rank_gate_dims.txt"):
        key, val = ln.split(":")
        dims[key] = int(val)
    out_width = dims["heads"] * dims["head_dim"]
    full = dims["hidden"] * out_width                 # a gate projected from the hidden state
    low = dims["query_latent"] * out_width            # the low-rank gate
    assert 100 * (full - low) // full == dims["fewer_weights_percent"]
    # the oracle's gate has exactly the low-rank projection's shape and is linear in the latent:
    # a one-hot latent selects one row of the projection
    rs = np.random.RandomState(5)
    Wg = rs.standard_normal((8, 4, 6))               # a small stand-in: r_q 8, 4 heads, 6 channels
    cq = np.zeros((2, 8))
    cq[0, 3] = 1.0
    cq[1, 5] = -2.0
    g = oracle.gate_logits(cq, Wg)
    assert g.shape == (2, 4, 6)
    np.testing.assert_array_equal(g[0], Wg[3])
    np.testing.assert_array_equal(g[1], -2.0 * Wg[5])
