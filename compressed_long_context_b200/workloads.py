"""Seeded synthetic inputs for the HCA hot path.

This module only draws random numbers and lays them out; it holds none of the
attention or pooling arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.  Shapes and distributions follow the workloads described for
ERNIE 5.5 Flash Base: 64 query heads sharing one KV head, 512-dim HCA heads,
128-token compression blocks and 128K to 1M-token contexts (model-card page
"ERNIE 5.5 Flash Base", architecture paragraph; official blog, section 2.1).

Draw order inside one generator: Q, K, V, pooling weights, gains, gate logits.
Values are drawn in fp32 and rounded to bf16 by torch (round to nearest even).
"""
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "prefill", "decode" (cache built from raw K/V) or "paged_decode"
    B: int
    T: int             # prefill length, or context length L for decode with a raw history
    Hq: int
    Hkv: int
    d: int
    dv: int
    blk: int
    W: int
    seed: int
    zero_weights: bool = False      # pooling weights all zero (plain mean)
    w_std: float = 0.5              # std of the pooling weights when drawn
    boost_frac: float = 0.0         # fraction of raw K rows multiplied by boost
    boost: float = 8.0
    out_f32: bool = False
    # ragged paged decode only
    L_min: int = 0
    L_max: int = 0
    page_size: int = 64
    qk_norm: bool = False
    gate: bool = False

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_PREFILL = Workload("tiny_prefill_T1024_d64", "prefill", B=1, T=1024, Hq=4, Hkv=1, d=64, dv=64,
                        blk=128, W=128, seed=0, zero_weights=True, out_f32=True)
DECODE_128K = Workload("decode_B64_L131072_d512", "decode", B=64, T=131072, Hq=64, Hkv=1, d=512,
                       dv=512, blk=128, W=128, seed=1)
PREFILL_128K = Workload("prefill_T131072_d512", "prefill", B=1, T=131072, Hq=64, Hkv=1, d=512, dv=512,
                        blk=128, W=128, seed=2, boost_frac=0.01)
DECODE_1M = Workload("compress_decode_B8_L1048576_d512", "decode", B=8, T=1048576, Hq=64, Hkv=1,
                     d=512, dv=512, blk=128, W=128, seed=3)
RAGGED_PAGED = Workload("ragged_paged_decode_B128_W256", "paged_decode", B=128, T=0, Hq=64, Hkv=1,
                        d=512, dv=512, blk=128, W=256, seed=4, L_min=4096, L_max=1048576,
                        qk_norm=True, gate=True)

WORKLOADS = [TINY_PREFILL, DECODE_128K, PREFILL_128K, DECODE_1M, RAGGED_PAGED]


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, g, device, std=1.0):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def _normal_bf16_chunked(shape, g, device):
    """Large bf16 normal tensors drawn in slices to bound the fp32 temporary."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def prefill_inputs(wl: Workload, device="cpu"):
    """q [B,T,Hq,d], k [B,T,Hkv,d], v [B,T,Hkv,dv] bf16; w [B,T] fp32."""
    g = _gen(device, wl.seed)
    B, T = wl.B, wl.T
    q = _normal_bf16_chunked((B, T, wl.Hq, wl.d), g, device)
    k = _normal_bf16_chunked((B, T, wl.Hkv, wl.d), g, device)
    v = _normal_bf16_chunked((B, T, wl.Hkv, wl.dv), g, device)
    if wl.zero_weights:
        w = torch.zeros((B, T), dtype=torch.float32, device=device)
    else:
        w = torch.randn((B, T), generator=g, device=device, dtype=torch.float32) * wl.w_std
    if wl.boost_frac > 0:
        # exactly round(frac * T) raw K rows per sequence, chosen by a seeded permutation,
        # multiplied after the bf16 rounding (x8 is exact in bf16)
        n = int(round(wl.boost_frac * T))
        for b in range(B):
            idx = torch.randperm(T, generator=g, device=device)[:n]
            k[b, idx] = (k[b, idx].float() * wl.boost).to(torch.bfloat16)
    return {"q": q, "k": k, "v": v, "w": w}


def decode_inputs(wl: Workload, device="cpu"):
    """Raw history + one query per sequence, all sequences of context L = wl.T.

    k, v [B,L,Hkv,d|dv] bf16 (the raw history, compressed by the caller),
    w [B,L] fp32, q [B,Hq,d] bf16, kw/vw [B,W,Hkv,d|dv] = the last W raw rows,
    seqlens [B] int32 (= L).
    """
    g = _gen(device, wl.seed)
    B, L = wl.B, wl.T
    q = _normal_bf16((B, wl.Hq, wl.d), g, device)
    k = _normal_bf16_chunked((B, L, wl.Hkv, wl.d), g, device)
    v = _normal_bf16_chunked((B, L, wl.Hkv, wl.dv), g, device)
    if wl.zero_weights:
        w = torch.zeros((B, L), dtype=torch.float32, device=device)
    else:
        w = torch.randn((B, L), generator=g, device=device, dtype=torch.float32) * wl.w_std
    Wn = min(wl.W, L)
    kw = torch.zeros((B, wl.W, wl.Hkv, wl.d), dtype=torch.bfloat16, device=device)
    vw = torch.zeros((B, wl.W, wl.Hkv, wl.dv), dtype=torch.bfloat16, device=device)
    kw[:, wl.W - Wn:] = k[:, L - Wn:]
    vw[:, wl.W - Wn:] = v[:, L - Wn:]
    seqlens = torch.full((B,), L, dtype=torch.int32, device=device)
    return {"q": q, "k": k, "v": v, "w": w, "kw": kw, "vw": vw, "seqlens": seqlens}


def ragged_lengths(wl: Workload):
    """Context lengths L_b ~ U{L_min..L_max}, redrawn while L_b is a multiple of blk (CPU, seeded)."""
    g = _gen("cpu", wl.seed)
    out = []
    while len(out) < wl.B:
        x = int(torch.randint(wl.L_min, wl.L_max + 1, (1,), generator=g).item())
        if x % wl.blk:
            out.append(x)
    return torch.tensor(out, dtype=torch.int32)


def paged_decode_inputs(wl: Workload, device="cpu", seqlens=None):
    """Ragged batch over a paged compressed cache whose entries are drawn directly.

    Sequence b holds floor(L_b / blk) complete-block entries in pages of wl.page_size
    entries; pages are handed out in a seeded shuffled order.
    Returns q [B,Hq,d], kc/vc pools [P,page,Hkv,d|dv], page_table [B,max_pages] int32,
    kw/vw [B,W,Hkv,d|dv], seqlens [B] int32, gq/gk [d] fp32 (or None), gate [B,Hq,dv] bf16
    (or None).
    """
    if seqlens is None:
        seqlens = ragged_lengths(wl)
    seqlens = seqlens.to(torch.int32).cpu()
    B, ps = wl.B, wl.page_size
    entries = [int(L) // wl.blk for L in seqlens.tolist()]
    pages = [(n + ps - 1) // ps for n in entries]
    P = max(1, sum(pages))
    maxp = max(1, max(pages))
    gm = _gen("cpu", wl.seed + 1000)
    perm = torch.randperm(P, generator=gm)
    table = torch.zeros((B, maxp), dtype=torch.int32)
    at = 0
    for b in range(B):
        table[b, :pages[b]] = perm[at:at + pages[b]].to(torch.int32)
        at += pages[b]
    g = _gen(device, wl.seed)
    q = _normal_bf16((B, wl.Hq, wl.d), g, device)
    kc = _normal_bf16_chunked((P, ps, wl.Hkv, wl.d), g, device)
    vc = _normal_bf16_chunked((P, ps, wl.Hkv, wl.dv), g, device)
    kw = _normal_bf16((B, wl.W, wl.Hkv, wl.d), g, device)
    vw = _normal_bf16((B, wl.W, wl.Hkv, wl.dv), g, device)
    gq = gk = gate = None
    if wl.qk_norm:
        gq = (torch.rand((wl.d,), generator=g, device=device, dtype=torch.float32) + 0.5)
        gk = (torch.rand((wl.d,), generator=g, device=device, dtype=torch.float32) + 0.5)
    if wl.gate:
        gate = _normal_bf16((B, wl.Hq, wl.dv), g, device)
    return {"q": q, "kc": kc, "vc": vc, "page_table": table.to(device), "kw": kw, "vw": vw,
            "seqlens": seqlens.to(device), "gq": gq, "gk": gk, "gate": gate,
            "page_size": ps, "max_pages": maxp}


@dataclass(frozen=True)
class DsaWorkload:
    """The sparse-attention layers' decode step: B sequences of context L, an indexer of H_I
    heads of d_I dims, the top-k positions kept, Hq query heads of d dims over one key and one
    value row per position (the pages' MLA layers use 256-dim heads)."""
    name: str
    B: int
    L: int
    HI: int
    dI: int
    topk: int
    Hq: int
    d: int
    seed: int


DSA_DECODE_128K = DsaWorkload("dsa_decode_B64_L131072_topk2048_d256", B=64, L=131072, HI=16, dI=64, topk=2048,
                              Hq=64, d=256, seed=6)


def dsa_inputs(wl: DsaWorkload, device="cpu"):
    """Draw order: indexer queries, indexer weights, indexer keys, queries, keys, values.

    q_idx [B,H_I,d_I] ~ N(0,1) bf16, w_idx [B,H_I] ~ U(0.5,1.5) fp32, k_idx [B,L,d_I] ~ N(0,1)
    bf16, q [B,Hq,d], k, v [B,L,d] ~ N(0,1) bf16, seqlens [B] int32 (= L).
    """
    g = _gen(device, wl.seed)
    B, L = wl.B, wl.L
    q_idx = _normal_bf16((B, wl.HI, wl.dI), g, device)
    w_idx = torch.rand((B, wl.HI), generator=g, device=device, dtype=torch.float32) + 0.5
    k_idx = _normal_bf16_chunked((B, L, wl.dI), g, device)
    q = _normal_bf16((B, wl.Hq, wl.d), g, device)
    k = _normal_bf16_chunked((B, L, wl.d), g, device)
    v = _normal_bf16_chunked((B, L, wl.d), g, device)
    seqlens = torch.full((B,), L, dtype=torch.int32, device=device)
    return {"q_idx": q_idx, "w_idx": w_idx, "k_idx": k_idx, "q": q, "k": k, "v": v, "seqlens": seqlens}
