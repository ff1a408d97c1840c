"""GPU parity of the sparse-attention decode step (hca_dsa_index, hca_dsa_topk, hca_dsa_attend,
through the C ABI) against the fp64 oracle (oracle/dsa.py).

Bars:
  - indexer scores: exact when the inputs are small integers (every product and partial sum is
    an integer below 2^24, so fp32 sums in any order are exact); otherwise within
    2^-20 * sum_j |w_j| |q_j . k_s| (fp32 rounding of a sum of H_I * d_I terms).
  - selection (an integer result): bit-exact on exact scores; on rounded scores every kept
    position's oracle score is within the scores' bound of the oracle's k-th largest.
  - attention: max abs error <= 1e-2 and mean abs error <= 1e-3 (P rounded to bf16 once,
    fp32 accumulation; the HCA decode's bar).
"""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle
from oracle import dsa as od
from compressed_long_context_b200 import _lib

pytestmark = pytest.mark.gpu
MAX_TOL, MEAN_TOL = 1e-2, 1e-3


def f64(t):
    return oracle.bits_to_f64(oracle.bf16_bits(t))


def int_inputs(dev, B, HI, Lmax, seed):
    g = torch.Generator(device=dev).manual_seed(seed)
    q = torch.randint(-3, 4, (B, HI, 64), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randint(-3, 4, (B, Lmax, 64), generator=g, device=dev).to(torch.bfloat16)
    w = torch.randint(0, 5, (B, HI), generator=g, device=dev).to(torch.float32) * 0.5
    return q, w, k


@pytest.mark.parametrize("HI,lengths,topk", [
    (16, [1000, 513, 1], 64),
    (64, [1000, 513, 1], 700),
    (32, [300, 299, 128], 1),
    (16, [2000, 1500], 2048),      # k above every length: all positions kept
    (48, [4096, 257], 300),
])
def test_index_and_topk_exact(cuda_device, libhca, HI, lengths, topk):
    B, Lmax = len(lengths), max(lengths)
    q, w, k = int_inputs(cuda_device, B, HI, Lmax, seed=HI + Lmax)
    seq = torch.tensor(lengths, dtype=torch.int32, device=cuda_device)
    sc = hca.dsa_index(q, w, k, seq)
    idx = hca.dsa_topk(sc, seq, topk)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = od.index_scores(f64(q), w.cpu().numpy(), f64(k), np.array(lengths))
    got = sc.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])                         # exact
    ridx = od.select_topk(ref, np.array(lengths), topk)
    assert np.array_equal(idx.cpu().numpy(), ridx)                    # bit-exact, ties included


@pytest.mark.parametrize("topk,lengths", [
    (100, [5000, 3000, 7]), (1000, [5000, 1001, 999]), (4096, [3000, 5000]),
    (70000, [300001, 150000, 70001, 69999]),    # quarters of 75K positions, k far above 2^16
])
def test_topk_exact_on_given_scores(cuda_device, libhca, topk, lengths):
    """Scores drawn by the test (coarse values: many ties, some -inf), the same array for both."""
    rs = np.random.RandomState(topk)
    B, Lmax = len(lengths), max(lengths)
    s = np.round(rs.standard_normal((B, Lmax)) * 4) / 4
    s[rs.rand(B, Lmax) < 0.01] = -np.inf
    s = s.astype(np.float32)
    seq = np.array(lengths, dtype=np.int32)
    idx = hca.dsa_topk(torch.tensor(s, device=cuda_device), torch.tensor(seq, device=cuda_device), topk)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = od.select_topk(s.astype(np.float64), seq, topk)
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_topk_all_equal_scores(cuda_device, libhca):
    """Every score equal (one digit in every pass): the first k positions are kept, and with
    more than 2^16 equal keys in a quarter the counts still place each quarter's output."""
    lengths = np.array([280000, 5, 4097], dtype=np.int32)
    s = torch.full((3, 280000), 0.75, device=cuda_device)
    idx = hca.dsa_topk(s, torch.tensor(lengths, device=cuda_device), 100000)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = od.select_topk(s.cpu().numpy().astype(np.float64), lengths, 100000)
    assert np.array_equal(idx.cpu().numpy(), ref)
    assert np.array_equal(ref[0], np.arange(100000))


def test_topk_signed_zeros_are_equal(cuda_device, libhca):
    """-0.0 and +0.0 are the same score: with the threshold at zero, the zeros are kept in
    position order whatever their sign."""
    rs = np.random.RandomState(5)
    s = np.where(rs.rand(2, 20000) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    s[:, ::7] = 1.0
    lengths = np.array([20000, 9999], dtype=np.int32)
    idx = hca.dsa_topk(torch.tensor(s, device=cuda_device), torch.tensor(lengths, device=cuda_device), 5000)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = od.select_topk(s.astype(np.float64), lengths, 5000)
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_index_rounding_bound(cuda_device, libhca):
    B, HI, Lmax = 2, 16, 3000
    g = torch.Generator(device=cuda_device).manual_seed(5)
    q = torch.randn((B, HI, 64), generator=g, device=cuda_device).to(torch.bfloat16)
    k = torch.randn((B, Lmax, 64), generator=g, device=cuda_device).to(torch.bfloat16)
    w = torch.rand((B, HI), generator=g, device=cuda_device) + 0.5
    lengths = [3000, 1234]
    seq = torch.tensor(lengths, dtype=torch.int32, device=cuda_device)
    sc = hca.dsa_index(q, w, k, seq)
    idx = hca.dsa_topk(sc, seq, 256)
    torch.cuda.synchronize()
    hca.get_device_error()
    qn, kn, wn = f64(q), f64(k), w.cpu().numpy().astype(np.float64)
    ref = od.index_scores(qn, wn, kn, np.array(lengths))
    got = sc.cpu().numpy().astype(np.float64)
    for b in range(B):
        L = lengths[b]
        bound = 2.0 ** -20 * (np.abs(kn[b, :L] @ qn[b].T) @ np.abs(wn[b])) + 1e-6
        assert np.all(np.abs(got[b, :L] - ref[b, :L]) <= bound)
        # the kept positions are a top-k of the oracle's scores up to that bound
        kth = np.sort(ref[b, :L])[::-1][255]
        kept = idx[b].cpu().numpy()
        assert np.all(ref[b, kept] >= kth - 2 * bound.max())
        assert np.all(np.diff(kept) > 0)


def attend_case(dev, B, Hq, Lmax, lengths, kmax, seed, boost=False):
    g = torch.Generator(device=dev).manual_seed(seed)
    q = torch.randn((B, Hq, 256), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((B, Lmax, 256), generator=g, device=dev)
    if boost:
        k[:, ::37] *= 8
    k = k.to(torch.bfloat16)
    v = torch.randn((B, Lmax, 256), generator=g, device=dev).to(torch.bfloat16)
    rs = np.random.RandomState(seed)
    idx = np.full((B, kmax), -1, np.int32)
    for b, L in enumerate(lengths):
        n = min(kmax, L)
        idx[b, :n] = np.sort(rs.choice(L, n, replace=False))
    return q, k, v, idx


@pytest.mark.parametrize("Hq,lengths,kmax,boost", [
    (64, [5000, 3000, 100], 2048, False),
    (64, [5000, 5000], 300, True),
    (16, [1000, 7, 129], 128, False),
    (64, [10, 1], 1, False),
    (33, [4000, 2500, 2049], 2048, True),
])
def test_attend_matches_oracle(cuda_device, libhca, Hq, lengths, kmax, boost):
    B, Lmax = len(lengths), max(lengths)
    q, k, v, idx = attend_case(cuda_device, B, Hq, Lmax, lengths, kmax, seed=kmax + Hq, boost=boost)
    scale = 1.0 / np.sqrt(256)
    seq = torch.tensor(lengths, dtype=torch.int32, device=cuda_device)
    out = hca.dsa_attend(q, k, v, torch.tensor(idx, device=cuda_device), seq, scale)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = od.sparse_attend(f64(q), f64(k), f64(v), idx, scale)
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert np.isfinite(out.cpu().numpy()).all()
    assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, (err.max(), err.mean())


def test_attend_grouped_launches_match_one_launch(cuda_device, libhca):
    """Sequences launched in groups (forced small row bound on the key / value maps): the
    output equals the single launch's bit for bit, and the oracle's within the bar."""
    lengths = [3000, 700, 2049, 1, 2500, 130, 3000]
    B, Lmax, kmax = len(lengths), max(lengths), 1024
    q, k, v, idx = attend_case(cuda_device, B, 64, Lmax, lengths, kmax, seed=41)
    seq = torch.tensor(lengths, dtype=torch.int32, device=cuda_device)
    idx_t = torch.tensor(idx, device=cuda_device)
    one = hca.dsa_attend(q, k, v, idx_t, seq, 0.0625)
    assert libhca.hca_debug_set_dsa_rows_limit(3 * Lmax) == 0      # two sequences per launch
    try:
        grouped = hca.dsa_attend(q, k, v, idx_t, seq, 0.0625)
        torch.cuda.synchronize()
    finally:
        assert libhca.hca_debug_set_dsa_rows_limit(0) == 0
    hca.get_device_error()
    assert torch.equal(one, grouped)
    ref = od.sparse_attend(f64(q), f64(k), f64(v), idx, 0.0625)
    err = np.abs(grouped.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL, (err.max(), err.mean())


def test_whole_step_matches_oracle(cuda_device, libhca):
    """Indexer inputs exact (small integers), attention inputs normal: the selection is
    bit-exact and the output within the attention bar."""
    lengths = [6000, 2500, 2048, 300]
    B, Lmax, HI, topk = len(lengths), max(lengths), 16, 2048
    qi, wi, ki = int_inputs(cuda_device, B, HI, Lmax, seed=31)
    q, k, v, _ = attend_case(cuda_device, B, 64, Lmax, lengths, topk, seed=32)
    seq = torch.tensor(lengths, dtype=torch.int32, device=cuda_device)
    scale = 1.0 / np.sqrt(256)
    out, idx, _ = hca.dsa_decode(qi, wi, ki, q, k, v, seq, topk, scale)
    torch.cuda.synchronize()
    hca.get_device_error()
    rout, ridx, _ = od.decode(f64(qi), wi.cpu().numpy(), f64(ki), f64(q), f64(k), f64(v), np.array(lengths), topk, scale)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    err = np.abs(out.cpu().numpy().astype(np.float64) - rout)
    assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL


def test_attend_reports_positions_past_the_buffer(cuda_device, libhca):
    q, k, v, idx = attend_case(cuda_device, 1, 64, 500, [500], 128, seed=3)
    idx[0, 5] = 10_000
    seq = torch.tensor([500], dtype=torch.int32, device=cuda_device)
    hca.dsa_attend(q, k, v, torch.tensor(idx, device=cuda_device), seq, 0.0625)
    with pytest.raises(hca.HCAError) as e:
        hca.get_device_error()
    assert e.value.code == _lib.HCA_ERR_DEVICE_INPUT
    hca.get_device_error()


def test_dsa_rejects_unsupported(cuda_device, libhca):
    q, w, k = int_inputs(cuda_device, 1, 24, 100, seed=1)     # 24 indexer heads: not a multiple of 16
    with pytest.raises(hca.HCAError):
        hca.dsa_index(q, w, k, torch.tensor([100], dtype=torch.int32, device=cuda_device))


def test_dsa_128k_sequences_sampled(cuda_device, libhca):
    """Four sequences of the bench's 128K sparse-attention workload shape (H_I = 16, d_I = 64,
    top-2048, 64 heads of 256), two of them checked in full against the oracle: scores within
    the rounding bound, the kept positions a top-k of the oracle's scores within it, and the
    attention over the kept positions within the attention bar."""
    from compressed_long_context_b200 import workloads as wl
    cfg = wl.DsaWorkload("dsa_test", B=4, L=131072, HI=16, dI=64, topk=2048, Hq=64, d=256, seed=12)
    inp = wl.dsa_inputs(cfg, cuda_device)
    scale = 1.0 / np.sqrt(cfg.d)
    out, idx, sc = hca.dsa_decode(inp["q_idx"], inp["w_idx"], inp["k_idx"], inp["q"], inp["k"], inp["v"],
                                  inp["seqlens"], cfg.topk, scale)
    torch.cuda.synchronize()
    hca.get_device_error()
    for b in (0, 3):
        qi, ki = f64(inp["q_idx"][b:b + 1]), f64(inp["k_idx"][b:b + 1])
        wi = inp["w_idx"][b:b + 1].cpu().numpy().astype(np.float64)
        ref = od.index_scores(qi, wi, ki, np.array([cfg.L]))[0]
        got = sc[b].double().cpu().numpy()
        bound = 2.0 ** -20 * (np.abs(ki[0] @ qi[0].T) @ np.abs(wi[0])) + 1e-6
        assert np.all(np.abs(got - ref) <= bound)
        kept = idx[b].cpu().numpy()
        kth = np.sort(ref)[::-1][cfg.topk - 1]
        assert np.all(kept >= 0) and np.all(np.diff(kept) > 0)
        assert np.all(ref[kept] >= kth - 2 * bound.max())
        ro = od.sparse_attend(f64(inp["q"][b:b + 1]), f64(inp["k"][b:b + 1]), f64(inp["v"][b:b + 1]), kept[None], scale)[0]
        err = np.abs(out[b].double().cpu().numpy() - ro)
        assert err.max() <= MAX_TOL and err.mean() <= MEAN_TOL
