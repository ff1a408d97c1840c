"""Pins of the sparse-attention oracle (oracle/dsa.py), CPU only.

Checked against things other than itself: a pure-Python brute force of the indexer on tiny
inputs; closed forms (all dot products positive: the ReLU is the identity and the score is one
dot product with the weighted sum of the indexer queries; all negative: every score is zero);
the hand-worked selection fixture tests/golden/dsa_topk_ties.txt; order properties of the
selection on random scores; PyTorch's scaled_dot_product_attention (float64) with a boolean
mask for the core attention; and planted mistakes, each caught by one of these.
"""
import os

import numpy as np
import pytest
import torch

from oracle import dsa

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "dsa_topk_ties.txt")


def _rand(rs, *shape):
    return rs.standard_normal(shape)


def _brute_scores(q, w, k, L):
    out = []
    for s in range(L):
        tot = 0.0
        for j in range(q.shape[0]):
            dot = 0.0
            for c in range(q.shape[1]):
                dot += float(q[j, c]) * float(k[s, c])
            tot += float(w[j]) * (dot if dot > 0 else 0.0)
        out.append(tot)
    return out


def test_index_scores_bruteforce():
    rs = np.random.RandomState(0)
    B, L, HI, dI = 2, 7, 3, 4
    q, w, k = _rand(rs, B, HI, dI), _rand(rs, B, HI), _rand(rs, B, L, dI)
    lens = np.array([7, 5])
    got = dsa.index_scores(q, w, k, lens)
    for b in range(B):
        ref = _brute_scores(q[b], w[b], k[b], lens[b])
        assert np.allclose(got[b, :lens[b]], ref, rtol=0, atol=1e-12)
        assert np.all(np.isneginf(got[b, lens[b]:]))


def test_index_scores_closed_forms():
    rs = np.random.RandomState(1)
    q = np.abs(_rand(rs, 1, 4, 8)) + 0.1
    k = np.abs(_rand(rs, 1, 9, 8)) + 0.1
    w = _rand(rs, 1, 4)
    # positive dot products: ReLU is the identity, so I(s) = k_s . (sum_j w_j q_j)
    got = dsa.index_scores(q, w, k, np.array([9]))
    assert np.allclose(got[0], k[0] @ (w[0] @ q[0]), rtol=1e-12)
    # negative dot products: every score is exactly zero, whatever the weights
    got = dsa.index_scores(-q, w, k, np.array([9]))
    assert np.all(got[0] == 0.0)


def _golden():
    rows = [l.strip() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    scores = np.array([float(x) for x in rows[0].split("|")[1].split()])
    cases = []
    for r in rows[1:]:
        kk, kept = r.split("|")
        cases.append((int(kk), [int(x) for x in kept.split()]))
    return scores, cases


def test_topk_golden_ties():
    scores, cases = _golden()
    L = len(scores)
    for k, kept in cases:
        got = dsa.select_topk(scores[None, :], np.array([L]), k)[0]
        assert list(got[got >= 0]) == kept, (k, list(got))
        assert np.all(got[len(kept):] == -1)


@pytest.mark.parametrize("seed", range(5))
def test_topk_order_properties(seed):
    rs = np.random.RandomState(seed)
    L, k = 300, 37
    # coarse values so that ties occur
    s = np.round(rs.standard_normal(L) * 3) / 2
    sel = dsa.select_topk(s[None, :], np.array([L]), k)[0]
    assert len(sel) == k and np.all(np.diff(sel) > 0)
    chosen = np.zeros(L, bool)
    chosen[sel] = True
    assert s[chosen].min() >= s[~chosen].max()
    thr = s[chosen].min()
    tied_in = np.where(chosen & (s == thr))[0]
    tied_out = np.where(~chosen & (s == thr))[0]
    if len(tied_out):
        assert tied_in.max() < tied_out.min()


def test_topk_bruteforce_small():
    rs = np.random.RandomState(7)
    for L in (1, 2, 5, 9):
        s = rs.randint(-2, 3, size=L).astype(float)
        for k in (1, 3, 10):
            ref = sorted(sorted(range(L), key=lambda i: (-s[i], i))[:k])
            got = dsa.select_topk(s[None, :], np.array([L]), k)[0]
            assert list(got[got >= 0]) == ref


def test_topk_signed_zeros_tie():
    """-0.0 and +0.0 compare equal, so they are one score and tie by position."""
    s = np.array([[-0.0, 0.0, -0.0, 1.0, 0.0, -0.0]])
    got = dsa.select_topk(s, np.array([6]), 3)[0]
    assert list(got) == [0, 1, 3]
    ref = sorted(sorted(range(6), key=lambda i: (-s[0, i], i))[:3])     # brute force
    assert list(got) == ref


def _sdpa(q, kk, vv, sel, scale):
    """torch SDPA (float64) of one sequence over the positions in sel (a boolean mask)."""
    Hq = q.shape[0]
    qt = torch.tensor(q)[None, :, None, :]                       # [1, Hq, 1, d]
    kt = torch.tensor(kk)[None, None].expand(1, Hq, -1, -1)      # shared key rows
    vt = torch.tensor(vv)[None, None].expand(1, Hq, -1, -1)
    mask = torch.tensor(sel)[None, None, None, :].expand(1, Hq, 1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)[0, :, 0].numpy()


def test_sparse_attend_matches_sdpa():
    rs = np.random.RandomState(3)
    B, Hq, d, Lmax, k = 2, 4, 16, 40, 11
    q, kk, vv = _rand(rs, B, Hq, d), _rand(rs, B, Lmax, d), _rand(rs, B, Lmax, d)
    idx = np.full((B, k), -1, np.int32)
    idx[0] = np.sort(rs.choice(Lmax, k, replace=False))
    idx[1, :5] = np.sort(rs.choice(30, 5, replace=False))
    got = dsa.sparse_attend(q, kk, vv, idx, 0.3)
    for b in range(B):
        sel = np.zeros(Lmax, bool)
        sel[idx[b][idx[b] >= 0]] = True
        assert np.allclose(got[b], _sdpa(q[b], kk[b], vv[b], sel, 0.3), rtol=0, atol=1e-12)


def test_all_positions_kept_is_dense_attention():
    """k at least the length: the selection keeps every position and the step is dense
    attention of the query over the whole sequence."""
    rs = np.random.RandomState(4)
    L, Hq, d = 23, 3, 8
    q_idx, w_idx, k_idx = _rand(rs, 1, 2, 4), _rand(rs, 1, 2), _rand(rs, 1, L, 4)
    q, kk, vv = _rand(rs, 1, Hq, d), _rand(rs, 1, L, d), _rand(rs, 1, L, d)
    out, idx, _ = dsa.decode(q_idx, w_idx, k_idx, q, kk, vv, np.array([L]), 64, 0.5)
    assert list(idx[0][idx[0] >= 0]) == list(range(L))
    assert np.allclose(out[0], _sdpa(q[0], kk[0], vv[0], np.ones(L, bool), 0.5), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- planted mistakes

def _mutant(fn_name, new_fn):
    old = getattr(dsa, fn_name)
    setattr(dsa, fn_name, new_fn)
    return old


CHECKS = [test_index_scores_bruteforce, test_index_scores_closed_forms, test_topk_golden_ties,
          lambda: test_topk_order_properties(0), test_topk_bruteforce_small, test_sparse_attend_matches_sdpa,
          test_all_positions_kept_is_dense_attention]


def _no_relu(q_idx, w_idx, k_idx, seqlens):
    q, w, k = (np.asarray(x, dtype=np.float64) for x in (q_idx, w_idx, k_idx))
    out = np.full(k.shape[:2], -np.inf)
    for b in range(k.shape[0]):
        L = int(seqlens[b])
        out[b, :L] = (k[b, :L] @ q[b].T) @ w[b]
    return out


def _relu_after_sum(q_idx, w_idx, k_idx, seqlens):
    q, w, k = (np.asarray(x, dtype=np.float64) for x in (q_idx, w_idx, k_idx))
    out = np.full(k.shape[:2], -np.inf)
    for b in range(k.shape[0]):
        L = int(seqlens[b])
        out[b, :L] = np.maximum((k[b, :L] @ q[b].T) @ w[b], 0.0)
    return out


def _ties_high_first(scores, seqlens, k):
    out = np.full((scores.shape[0], k), -1, dtype=np.int32)
    for b in range(scores.shape[0]):
        L = int(seqlens[b])
        s = np.asarray(scores[b, :L], dtype=np.float64)
        order = np.lexsort((-np.arange(L), -s))
        keep = np.sort(order[:min(k, L)])
        out[b, :len(keep)] = keep
    return out


def _no_scale(q, kk, vv, idx, scale):
    return _ORIG_ATTEND(q, kk, vv, idx, 1.0)


def _all_positions(q, kk, vv, idx, scale):
    full = np.tile(np.arange(kk.shape[1], dtype=np.int32), (q.shape[0], 1))
    return _ORIG_ATTEND(q, kk, vv, full, scale)


_ORIG_ATTEND = dsa.sparse_attend

MUTANTS = {
    "indexer without ReLU": ("index_scores", _no_relu),
    "ReLU after the weighted sum": ("index_scores", _relu_after_sum),
    "ties taken from the highest position": ("select_topk", _ties_high_first),
    "logit scale dropped": ("sparse_attend", _no_scale),
    "attention over every position": ("sparse_attend", _all_positions),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    fn_name, new_fn = MUTANTS[name]
    old = _mutant(fn_name, new_fn)
    try:
        caught = False
        for check in CHECKS:
            try:
                check()
            except AssertionError:
                caught = True
                break
        assert caught, name
    finally:
        setattr(dsa, fn_name, old)
