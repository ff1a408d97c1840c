"""Small, self-contained launches of one HCA kernel for profiling (ncu) and quick timing.

    python -m compressed_long_context_b200.profile_cases compress [--reps N]
    python -m compressed_long_context_b200.profile_cases decode   [--reps N]
    python -m compressed_long_context_b200.profile_cases prefill  [--reps N]
    python -m compressed_long_context_b200.profile_cases paged    [--reps N]
    python -m compressed_long_context_b200.profile_cases vha      [--reps N]
    python -m compressed_long_context_b200.profile_cases append   [--reps N]
    python -m compressed_long_context_b200.profile_cases gate     [--reps N]
    python -m compressed_long_context_b200.profile_cases backward [--reps N] [--T tokens]
    python -m compressed_long_context_b200.profile_cases dsa      [--reps N]   (index + topk + attend)

Each case keeps its working set larger than the 126 MB L2 (so DRAM counters mean
something) but a few GB at most, and launches the kernel `--reps` times after one
warm-up launch.  The size options (--B, --L, --T) are for timing and for one-pass launch
lists; multi-metric captures use the default sizes and scale.  Prints the per-launch time from CUDA events (not meaningful under a
profiler).
"""
import argparse
import json
import math

import torch

from . import (append, append_state_size, compress, decode, decode_workspace_size, dsa_attend, dsa_index, dsa_topk,
               gate_logits, get_device_error, prefill, prefill_backward, vha)
from . import workloads as wl


_last_fn = [None]


def _events():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def run(case: str, reps: int, B_override: int = 0, L_override: int = 0, T_override: int = 0) -> dict:
    dev = torch.device("cuda", torch.cuda.current_device())
    g = torch.Generator(device=dev).manual_seed(123)
    if case == "compress":
        # 8 sequences x 131072 tokens x 512: 2.1 GB of raw K/V
        B, T, d = 8, 131072, 512
        k = torch.randn((B, T, 1, d), generator=g, device=dev).to(torch.bfloat16)
        v = torch.randn((B, T, 1, d), generator=g, device=dev).to(torch.bfloat16)
        w = torch.randn((B, T), generator=g, device=dev) * 0.5
        kc = torch.empty((B, T // 128, 1, d), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        fn = lambda: compress(k, v, w, 128, kc=kc, vc=vc)  # noqa: E731
        nbytes = B * (T // 128) * (128 * 2 * d * 2 + 2 * d * 2) + B * T * 4
    elif case in ("decode", "paged"):
        # the 128K decode batch with its cache drawn directly (134 MB of entries)
        B, L, Hq, d, W = 64, 131072, 64, 512, 128
        B = B_override or B
        L = L_override or L
        nc = (L - W) // 128
        q = torch.randn((B, Hq, d), generator=g, device=dev).to(torch.bfloat16)
        kw = torch.randn((B, W, 1, d), generator=g, device=dev).to(torch.bfloat16)
        vw = torch.randn((B, W, 1, d), generator=g, device=dev).to(torch.bfloat16)
        seq = torch.full((B,), L, dtype=torch.int32, device=dev)
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
        ws = torch.empty(decode_workspace_size(B, Hq, 1, d), dtype=torch.uint8, device=dev)
        if case == "decode":
            kc = torch.randn((B, L // 128, 1, d), generator=g, device=dev).to(torch.bfloat16)
            vc = torch.randn((B, L // 128, 1, d), generator=g, device=dev).to(torch.bfloat16)
            fn = lambda: decode(q, kc, vc, kw, vw, seq, 128, W, 1 / math.sqrt(d), out=out,  # noqa: E731
                                workspace=ws)
        else:
            ps = 64
            npg = (L // 128 + ps - 1) // ps
            kc = torch.randn((B * npg, ps, 1, d), generator=g, device=dev).to(torch.bfloat16)
            vc = torch.randn((B * npg, ps, 1, d), generator=g, device=dev).to(torch.bfloat16)
            perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(5)).to(torch.int32)
            table = perm.view(B, npg).to(dev)
            gq = torch.rand((d,), generator=g, device=dev) + 0.5
            gk = torch.rand((d,), generator=g, device=dev) + 0.5
            gate = torch.randn((B, Hq, d), generator=g, device=dev).to(torch.bfloat16)
            fn = lambda: decode(q, kc, vc, kw, vw, seq, 128, W, 1 / math.sqrt(d), page_table=table,  # noqa: E731
                                page_size=ps, gq=gq, gk=gk, gate=gate, out=out, workspace=ws)
        nbytes = B * (Hq * d * 2 + (nc + W) * 2 * d * 2 + Hq * d * 4)
    elif case == "prefill":
        # default T = 16384 tokens, 64 heads of 512: 1 GB of Q, 1 GB of output
        cfg = wl.PREFILL_128K.scaled(T=T_override or 16384)
        inp = wl.prefill_inputs(cfg, dev)
        kc, vc = compress(inp["k"], inp["v"], inp["w"], 128)
        out = torch.empty((1, cfg.T, cfg.Hq, cfg.dv), dtype=torch.bfloat16, device=dev)
        fn = lambda: prefill(inp["q"], inp["k"], inp["v"], kc, vc, 128, cfg.W, 1 / math.sqrt(cfg.d),  # noqa: E731
                             out=out)
        keys = sum(max(0, (t - cfg.W + 1) // 128) + min(cfg.W, t + 1) for t in range(cfg.T))
        nbytes = None
        flops = 2.0 * cfg.Hq * keys * (cfg.d + cfg.dv)
    elif case == "vha":
        # 8192 tokens x 64 heads x 512 bf16 (512 MB, mixed in place), rank 8
        n, Hq, d = 8192, 64, 512
        x = torch.randn((n, Hq, d), generator=g, device=dev).to(torch.bfloat16)
        U = torch.randn((Hq, 8), generator=g, device=dev) * 0.1
        V = torch.randn((Hq, 8), generator=g, device=dev) * 0.1
        fn = lambda: vha(x, U, V)  # noqa: E731
        nbytes = 2 * x.numel() * 2
    elif case == "append":
        # 64 sequences of 131072 tokens appending their newest token (each completes a block)
        B, L, d, W = 64, 131072, 512, 128
        kn = torch.randn((B, 1, d), generator=g, device=dev).to(torch.bfloat16)
        vn = torch.randn((B, 1, d), generator=g, device=dev).to(torch.bfloat16)
        wn = torch.randn((B,), generator=g, device=dev)
        seq = torch.full((B,), L, dtype=torch.int32, device=dev)
        kw = torch.zeros((B, W, 1, d), dtype=torch.bfloat16, device=dev)
        vw = torch.zeros_like(kw)
        kc = torch.zeros((B, L // 128, 1, d), dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        state = torch.zeros(append_state_size(B, 1, d, d), dtype=torch.uint8, device=dev)
        fn = lambda: append(kn, vn, wn, seq, kw, vw, kc, vc, state, 128)  # noqa: E731
        nbytes = B * (4 * d * 2 + 2 * (4 + 2 * d) * 4) + B * 8
    elif case == "gate":
        # the low-rank gate projection: 64 latents of 1024 -> 64 x 512 logits (64 MB of weights)
        B, rq, Hq, d = 64, 1024, 64, 512
        cq = torch.randn((B, rq), generator=g, device=dev).to(torch.bfloat16)
        wg = (torch.randn((rq, Hq, d), generator=g, device=dev) / 32.0).to(torch.bfloat16)
        gate = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
        fn = lambda: gate_logits(cq, wg, out=gate)  # noqa: E731
        nbytes = (cq.numel() + wg.numel() + gate.numel()) * 2
    elif case == "backward":
        # default T = 8192 tokens, 64 heads of 512: 512 MB each of Q, dO and the bf16 output
        cfg = wl.PREFILL_128K.scaled(T=T_override or 8192)
        inp = wl.prefill_inputs(cfg, dev)
        kc, vc = compress(inp["k"], inp["v"], inp["w"], 128)
        sc = 1 / math.sqrt(cfg.d)
        out, lse = prefill(inp["q"], inp["k"], inp["v"], kc, vc, 128, cfg.W, sc, want_lse=True)
        dout = torch.randn(inp["q"].shape, generator=g, device=dev).to(torch.bfloat16)
        fn = lambda: prefill_backward(inp["q"], inp["k"], inp["v"], inp["w"], kc, vc, out, lse,  # noqa: E731
                                      dout, 128, cfg.W, sc)
        keys = sum(max(0, (t - cfg.W + 1) // 128) + min(cfg.W, t + 1) for t in range(cfg.T))
        nbytes = None
        flops = 5 * 2.0 * cfg.Hq * keys * cfg.d
    elif case == "dsa":
        # the sparse-attention decode step at 16 sequences of 32768 positions (64 MB of indexer
        # keys, 512 MB of key / value rows)
        cfg = wl.DSA_DECODE_128K
        cfg = wl.DsaWorkload(cfg.name, B=B_override or 16, L=L_override or 32768, HI=cfg.HI, dI=cfg.dI, topk=cfg.topk,
                             Hq=cfg.Hq, d=cfg.d, seed=cfg.seed)
        inp = wl.dsa_inputs(cfg, dev)
        scores = torch.empty((cfg.B, cfg.L), dtype=torch.float32, device=dev)
        idx = torch.empty((cfg.B, cfg.topk), dtype=torch.int32, device=dev)
        out = torch.empty((cfg.B, cfg.Hq, cfg.d), dtype=torch.float32, device=dev)

        def fn():
            dsa_index(inp["q_idx"], inp["w_idx"], inp["k_idx"], inp["seqlens"], scores=scores)
            dsa_topk(scores, inp["seqlens"], cfg.topk, idx=idx)
            dsa_attend(inp["q"], inp["k"], inp["v"], idx, inp["seqlens"], 1 / math.sqrt(cfg.d), out=out)
        nbytes = cfg.B * cfg.L * (cfg.dI * 2 + 8) + cfg.B * cfg.topk * (4 * cfg.d + 8)
    else:
        raise ValueError(case)
    _last_fn[0] = fn
    fn()
    torch.cuda.synchronize()
    get_device_error()
    a, b = _events()
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    get_device_error()
    ms = a.elapsed_time(b) / reps
    res = {"case": case, "reps": reps, "ms_per_launch": ms}
    if case in ("decode", "paged"):
        res["B"], res["L"] = B, L
    if nbytes:
        res["bytes"] = nbytes
        res["GB_per_s"] = nbytes / (ms / 1e3) / 1e9
    if case in ("prefill", "backward"):
        res["T"] = cfg.T
        res["TFLOP_per_s"] = flops / (ms / 1e3) / 1e12
    return res


def run_flushed(args) -> dict:
    """Per-launch device time with L2 flushed before every launch (a GPU spin is queued first
    so that launches are enqueued ahead of the GPU)."""
    import statistics
    res = run(args.case, 1, args.B, args.L, args.T)
    fn = _last_fn[0]
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    buf = torch.empty(2 * l2, dtype=torch.uint8, device="cuda")
    evs = [_events() for _ in range(args.reps)]
    torch.cuda._sleep(int(2e8))
    for a, b in evs:
        buf.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    res["ms_per_launch"] = statistics.median(ms)
    res["flushed"] = True
    if "bytes" in res:
        res["GB_per_s"] = res["bytes"] / (res["ms_per_launch"] / 1e3) / 1e9
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["compress", "decode", "paged", "prefill", "vha", "append", "gate", "backward", "dsa"])
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--B", type=int, default=0, help="decode batch (default 64)")
    ap.add_argument("--L", type=int, default=0, help="decode context length (default 131072)")
    ap.add_argument("--T", type=int, default=0, help="prefill tokens (default 16384; backward 8192)")
    ap.add_argument("--flush", action="store_true", help="flush L2 before every launch (events per launch)")
    args = ap.parse_args()
    print(json.dumps(run(args.case, args.reps, args.B, args.L, args.T) if not args.flush else run_flushed(args)))


if __name__ == "__main__":
    main()
