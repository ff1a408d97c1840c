"""GPU parity of hca_gate_logits (Low-Rank Gated Attention's gate projection, through the C
ABI) against the fp64 oracle, and of the whole gated path: the projection feeding the decode
gate, with Virtual Head Attention fused into the merge, against the oracle's projection ->
decode -> mixing.

Bar for the logits: they are stored in bf16, so each is within half a bf16 ulp of the fp32
sum, which is within ~2^-20 |sum of |terms|| of the exact value: |got - ref| <= 2^-8 |ref| +
1e-3.  Bar for the decode outputs: max abs 1e-2, mean abs 1e-3.
"""
import numpy as np
import pytest
import torch

import compressed_long_context_b200 as hca
import oracle

pytestmark = pytest.mark.gpu


def bits(t):
    return oracle.bf16_bits(t)


def latent_and_weights(dev, n, rq, Hq, dv, seed):
    g = torch.Generator(device=dev).manual_seed(seed)
    cq = torch.randn((n, rq), generator=g, device=dev).to(torch.bfloat16)
    wg = (torch.randn((rq, Hq, dv), generator=g, device=dev) / np.sqrt(rq)).to(torch.bfloat16)
    return cq, wg


@pytest.mark.parametrize("n,rq,Hq,dv", [(64, 1024, 64, 512), (1, 64, 4, 64), (130, 256, 8, 512), (7, 128, 64, 64)])
def test_gate_logits_against_oracle(cuda_device, libhca, n, rq, Hq, dv):
    cq, wg = latent_and_weights(cuda_device, n, rq, Hq, dv, 7 + n + rq)
    got = hca.gate_logits(cq, wg)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref = oracle.gate_logits(oracle.bits_to_f64(bits(cq)), oracle.bits_to_f64(bits(wg)))
    g = got.float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape
    assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3)


def test_gate_logits_rejects_unsupported(cuda_device, libhca):
    cq, wg = latent_and_weights(cuda_device, 4, 96, 64, 512, 3)    # rq not a multiple of 64
    with pytest.raises(hca.HCAError):
        hca.gate_logits(cq, wg)


def test_low_rank_gated_decode_with_vha(cuda_device, libhca):
    """The pages' gated layer at decode: gate logits from the query latent (rq = 1024, a quarter
    of the 4096 hidden size), the decode over entries + window with that gate, then the cross-head
    mixing -- GPU path hca_gate_logits -> hca_decode_vha against oracle.gate_logits (rounded to
    bf16 by the oracle, as the stored logits are) -> oracle.decode -> oracle.vha."""
    dev = cuda_device
    B, Hq, W, blk, r = 16, 64, 128, 128, 8
    lengths = [131072, 9000, 300, 70000] * 4
    g = torch.Generator(device=dev).manual_seed(23)
    Nmax = max(oracle.visible_entries(L - 1, W, blk) for L in lengths)
    q = torch.randn((B, Hq, 512), generator=g, device=dev).to(torch.bfloat16)
    kc = torch.randn((B, Nmax, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn((B, Nmax, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    kw = torch.randn((B, W, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    vw = torch.randn((B, W, 1, 512), generator=g, device=dev).to(torch.bfloat16)
    seq = torch.tensor(lengths, dtype=torch.int32, device=dev)
    cq, wg = latent_and_weights(dev, B, 1024, Hq, 512, 29)
    U = torch.randn((Hq, r), generator=g, device=dev) * 0.1
    V = torch.randn((Hq, r), generator=g, device=dev) * 0.1
    scale = 1.0 / np.sqrt(512)
    gate = hca.gate_logits(cq, wg)
    out = hca.decode(q, kc, vc, kw, vw, seq, blk, W, scale, gate=gate, vha_u=U, vha_v=V)
    torch.cuda.synchronize()
    hca.get_device_error()
    ref_g = oracle.round_bf16(oracle.gate_logits(oracle.bits_to_f64(bits(cq)), oracle.bits_to_f64(bits(wg))))
    ref = oracle.decode(bits(q), bits(kc), bits(vc), bits(kw), bits(vw), seq.cpu().numpy(), blk, W, scale,
                        gate=ref_g)
    ref = oracle.vha(ref, U.cpu().numpy(), V.cpu().numpy())
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert np.isfinite(out.cpu().numpy()).all()
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
