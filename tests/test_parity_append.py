"""GPU parity of hca_append (one decode step's cache update) and of hca_decode reading the
window ring it maintains, against the fp64 oracle on the same raw history.

A serving loop is simulated: sequences start at different lengths, and each step appends
one token to every sequence.  Checked:
 - the ring holds the raw tokens, bit for bit (slot p % W = position p);
 - every entry written equals the oracle's compression of the same raw block (cache bar:
   4e-3 abs, or the bf16 rounding bound where |ref| >= 1, as for hca_compress);
 - hca_decode with HCA_WINDOW_RING over the appended cache equals the oracle's decode of
   the history (max abs 1e-2, mean abs 1e-3), including while L < W;
 - an entry beyond the cache and a length < 1 are reported as device-input errors.
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


def check_out(got, ref):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape and np.isfinite(g).all()
    err = np.abs(g - ref)
    assert err.max() <= MAX_TOL, ("max", err.max())
    assert err.mean() <= MEAN_TOL, ("mean", err.mean())


def check_cache(got_bf16, ref_f64):
    g = got_bf16.float().cpu().numpy().astype(np.float64)
    tol = np.maximum(4e-3, 2.0 ** -8 * np.abs(ref_f64) + 1e-5)
    err = np.abs(g - ref_f64)
    assert np.all(err <= tol), (err.max(), np.abs(ref_f64).max())


class Loop:
    """Raw history + the device state that hca_append maintains for it."""

    def __init__(self, dev, seed, B, Hkv, d, dv, T, blk, W, paged_ps=0, wstd=0.5):
        g = torch.Generator(device=dev).manual_seed(seed)
        self.dev, self.B, self.Hkv, self.d, self.dv, self.T, self.blk, self.W = dev, B, Hkv, d, dv, T, blk, W
        self.k = torch.randn((B, T, Hkv, d), generator=g, device=dev).to(torch.bfloat16)
        self.v = torch.randn((B, T, Hkv, dv), generator=g, device=dev).to(torch.bfloat16)
        self.w = torch.randn((B, T), generator=g, device=dev) * wstd
        self.q = torch.randn((B, 64 * Hkv, d), generator=g, device=dev).to(torch.bfloat16)
        self.kw = torch.zeros((B, W, Hkv, d), dtype=torch.bfloat16, device=dev)
        self.vw = torch.zeros((B, W, Hkv, dv), dtype=torch.bfloat16, device=dev)
        Nmax = T // blk + 1
        if paged_ps:
            npg = (Nmax + paged_ps - 1) // paged_ps
            P = B * npg + 3
            self.kc = torch.zeros((P, paged_ps, Hkv, d), dtype=torch.bfloat16, device=dev)
            self.vc = torch.zeros((P, paged_ps, Hkv, dv), dtype=torch.bfloat16, device=dev)
            perm = torch.randperm(P, generator=torch.Generator().manual_seed(seed))[:B * npg]
            self.table = perm.view(B, npg).to(torch.int32).to(dev)
        else:
            self.kc = torch.zeros((B, Nmax, Hkv, d), dtype=torch.bfloat16, device=dev)
            self.vc = torch.zeros((B, Nmax, Hkv, dv), dtype=torch.bfloat16, device=dev)
            self.table = None
        self.ps = paged_ps
        self.state = torch.zeros(hca.append_state_size(B, Hkv, d, dv) // 4, dtype=torch.float32, device=dev)
        self.L = [0] * B

    def append(self, idx):
        """Append the next token of the sequences in idx (a contiguous range of the batch)."""
        b0, b1 = idx[0], idx[-1] + 1
        assert list(idx) == list(range(b0, b1))
        pos = [self.L[b] for b in idx]
        kn = torch.stack([self.k[b, p] for b, p in zip(idx, pos)])
        vn = torch.stack([self.v[b, p] for b, p in zip(idx, pos)])
        wn = torch.stack([self.w[b, p] for b, p in zip(idx, pos)]).contiguous()
        seq = torch.tensor([p + 1 for p in pos], dtype=torch.int32, device=self.dev)
        per = self.state.numel() // self.B
        st = self.state[b0 * per:b1 * per]
        tbl = None if self.table is None else self.table[b0:b1]
        kc, vc = (self.kc, self.vc) if self.table is not None else (self.kc[b0:b1], self.vc[b0:b1])
        hca.append(kn, vn, wn, seq, self.kw[b0:b1], self.vw[b0:b1], kc, vc, st, self.blk, page_table=tbl)
        for b in idx:
            self.L[b] += 1

    def entry(self, b, j):
        if self.table is None:
            return self.kc[b, j], self.vc[b, j]
        pg = int(self.table[b, j // self.ps])
        return self.kc[pg, j % self.ps], self.vc[pg, j % self.ps]

    def check_state(self):
        torch.cuda.synchronize()
        hca.get_device_error()
        for b in range(self.B):
            L = self.L[b]
            # the ring: slot p % W holds position p for the last min(L, W) positions (bit exact)
            for p in range(max(0, L - self.W), L):
                assert torch.equal(self.kw[b, p % self.W], self.k[b, p])
                assert torch.equal(self.vw[b, p % self.W], self.v[b, p])
            # every complete block's entry, against the oracle's compression of the raw block
            nb = L // self.blk
            if nb:
                ok, ov = oracle.compress(bits(self.k[b:b + 1, :nb * self.blk]), bits(self.v[b:b + 1, :nb * self.blk]),
                                         self.w[b:b + 1, :nb * self.blk].cpu().numpy(), self.blk)
                for j in range(nb):
                    ek, ev = self.entry(b, j)
                    check_cache(ek, ok[0, j])
                    check_cache(ev, ov[0, j])

    def check_decode(self, norm=False):
        """hca_decode over the ring against the oracle's decode of the history."""
        seq = torch.tensor(self.L, dtype=torch.int32, device=self.dev)
        scale = 1.0 / np.sqrt(self.d)
        out = hca.decode(self.q, self.kc, self.vc, self.kw, self.vw, seq, self.blk, self.W, scale,
                         page_table=self.table, page_size=self.ps, window_ring=True)
        torch.cuda.synchronize()
        hca.get_device_error()
        for b in range(self.B):
            L = self.L[b]
            nb = L // self.blk
            Nc = max(nb, 1)
            kc = np.zeros((1, Nc, self.Hkv, self.d), np.uint16)
            vc = np.zeros((1, Nc, self.Hkv, self.dv), np.uint16)
            if nb:
                ok, ov = oracle.compress(bits(self.k[b:b + 1, :nb * self.blk]), bits(self.v[b:b + 1, :nb * self.blk]),
                                         self.w[b:b + 1, :nb * self.blk].cpu().numpy(), self.blk)
                kc[:, :nb], vc[:, :nb] = oracle.round_bf16(ok), oracle.round_bf16(ov)
            # oldest-first window of the oracle: slot i = position L - W + i (negative ignored)
            kw = torch.zeros((1, self.W, self.Hkv, self.d), dtype=torch.bfloat16)
            vw = torch.zeros((1, self.W, self.Hkv, self.dv), dtype=torch.bfloat16)
            n = min(L, self.W)
            kw[0, self.W - n:] = self.k[b, L - n:L].cpu()
            vw[0, self.W - n:] = self.v[b, L - n:L].cpu()
            ref = oracle.decode(bits(self.q[b:b + 1]), kc, vc, bits(kw), bits(vw), np.array([L], np.int32),
                                self.blk, self.W, scale)
            check_out(out[b:b + 1], ref)


def run_loop(lp, starts, steps, decode_every):
    # bring each sequence to its own starting length, one sequence at a time
    for b, s in enumerate(starts):
        for _ in range(s):
            lp.append([b])
    lp.check_state()
    if min(lp.L) >= 1:      # a decode query needs at least its own token
        lp.check_decode()
    for step in range(steps):
        lp.append(list(range(lp.B)))
        if (step + 1) % decode_every == 0:
            lp.check_decode()
    lp.check_state()
    lp.check_decode()


def test_append_contiguous(cuda_device, libhca):
    lp = Loop(cuda_device, 11, B=3, Hkv=1, d=512, dv=512, T=700, blk=128, W=128)
    run_loop(lp, starts=[0, 37, 300], steps=390, decode_every=97)


def test_append_paged_two_kv_heads(cuda_device, libhca):
    lp = Loop(cuda_device, 12, B=2, Hkv=2, d=512, dv=512, T=600, blk=128, W=200, paged_ps=64)
    run_loop(lp, starts=[5, 130], steps=300, decode_every=75)


def test_append_small_block_mean_pooling(cuda_device, libhca):
    """Blocks of 16 tokens, zero weights (the mean), a window shorter than a block."""
    lp = Loop(cuda_device, 13, B=2, Hkv=1, d=512, dv=512, T=200, blk=16, W=7, wstd=0.0)
    run_loop(lp, starts=[0, 9], steps=150, decode_every=50)


def test_append_device_input_errors(cuda_device, libhca):
    dev = cuda_device
    kn = torch.zeros((1, 1, 512), dtype=torch.bfloat16, device=dev)
    kw = torch.zeros((1, 128, 1, 512), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((1, 1, 1, 512), dtype=torch.bfloat16, device=dev)      # room for entry 0 only
    st = torch.zeros(hca.append_state_size(1, 1, 512, 512) // 4, dtype=torch.float32, device=dev)
    # completing block 1 (L = 256) would write entry 1: outside the cache
    hca.append(kn, kn, None, torch.tensor([256], dtype=torch.int32, device=dev), kw, kw.clone(), kc, kc.clone(),
               st, 128)
    with pytest.raises(hca.HCAError) as e:
        hca.get_device_error()
    assert e.value.code == 5
    hca.append(kn, kn, None, torch.tensor([0], dtype=torch.int32, device=dev), kw, kw.clone(), kc, kc.clone(),
               st, 128)
    with pytest.raises(hca.HCAError) as e:
        hca.get_device_error()
    assert e.value.code == 5
    hca.get_device_error()     # cleared
