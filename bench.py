"""Benchmark of the HCA hot path on B200 (one JSON line on stdout).

Headline (`value`): HCA decode queries/s on the 128K decode workload -- 64 sequences of
131072 tokens, Hq=64 query heads sharing one 512-dim KV head, blocks of 128, a raw window
of 128 tokens (1023 compressed entries + 128 raw tokens per query); pooling weights
~N(0, 0.5); bf16 inputs ~N(0, 1); seed 1.  One step = one `hca_decode` call (split kernel +
combine kernel) over the whole batch, the compressed cache resident in HBM, L2 flushed
before every timed call.  value = queries of all ranks / device time (max over ranks).

Every workload of the hot path is measured in the same run, one at a time (memory freed in
between), under `configs`: its GPU time and rate, its roofline fraction, the algorithmic
bytes or flops per unit, the fp64 CPU oracle's time on this host's cores and the max/mean
absolute error of the GPU result against that oracle:
  tiny_prefill       T=1024, Hq=4, d=64, mean pooling, fp32 output (compress + prefill)
  decode_128k        the headline batch; compress of its raw K/V reported as its own GB/s
  prefill_128k       T=131072, Hq=64, d=512, 1% of raw keys x8 (compress + prefill TFLOP/s,
                     fraction of the burst bf16 peak); oracle on sampled rows
  decode_1m          8 sequences of 1048576 tokens: compress GB/s + decode queries/s
  ragged_paged       128 ragged sequences (4K..1M), paged cache, QK RMSNorm + sigmoid gate

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: torchrun, one rank per GPU, each rank a full batch (weak scaling); the oracle
checks run at N=1 only.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "HCA decode queries/s, prefill TFLOP/s, % of HBM/TC roofline (1 B200)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CONFIG_KEYS = ("tiny_prefill", "decode_128k", "prefill_128k", "decode_1m", "ragged_paged", "dsa_decode_128k")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-oracle", action="store_true", help="skip the per-config oracle checks")
    ap.add_argument("--configs", default=",".join(CONFIG_KEYS),
                    help="comma-separated subset of %s (the headline config always runs)" % ",".join(CONFIG_KEYS))
    return ap.parse_args(argv)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- algorithmic work

def compress_bytes(B, T, Hkv, d, dv, blk):
    """Raw K/V and weights read, entries written."""
    Nc = T // blk
    return B * Nc * Hkv * (blk * (d + dv) * 2 + 2 * (d + dv)) + B * Nc * blk * 4


def decode_seq_bytes(L, Hq, Hkv, d, dv, blk, W, gate=False):
    """One query: q read, visible entries + window keys/values read, fp32 output written,
    the length read (+ the gate logits read)."""
    nc = max(0, (L - W) // blk)
    nw = min(W, L)
    return Hq * d * 2 + (nc + nw) * Hkv * (d + dv) * 2 + Hq * dv * 4 + 4 + (Hq * dv * 2 if gate else 0)


def decode_bytes(B, L, Hq, Hkv, d, dv, blk, W):
    return B * decode_seq_bytes(L, Hq, Hkv, d, dv, blk, W)


def append_bytes(B, Hkv, d, dv):
    """hca_append when every sequence completes a block: new token read, pooling state read and
    written, ring slot written, entry written (bytes per call)."""
    state = (4 + d + dv) * 4
    return B * Hkv * ((d + dv) * 2 + 2 * state + (d + dv) * 2 + (d + dv) * 2) + B * 8


def vha_bytes(numel, esize, Hq, r):
    """hca_vha in place: the output read and written once, plus the two fp32 factors."""
    return 2 * numel * esize + 2 * Hq * r * 4


def prefill_flops(B, T, Hq, d, dv, blk, W):
    """2 * Hq * (d + dv) flops per (query row, visible key)."""
    t = np.arange(T, dtype=np.int64)
    a = t - W + 1
    nc = np.where(a > 0, a // blk, 0)
    keys = int((nc + np.minimum(W, t + 1)).sum())
    return 2.0 * B * Hq * keys * (d + dv), keys


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled every 20 ms while the
    timed regions run (NVML; nvidia-smi at 200 ms if NVML is unavailable).  Reads only."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.device_index = device_index
        self.samples = []          # (sm_mhz, max_mhz, reason bits)
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            prop = torch.cuda.get_device_properties(device_index)
            bus = "%08X:%02X:%02X.0" % (getattr(prop, "pci_domain_id", 0), prop.pci_bus_id, prop.pci_device_id)
            self._handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nvml = pynvml
        except Exception:
            self._nvml = None

    def _sample_nvml(self):
        n = self._nvml
        sm = n.nvmlDeviceGetClockInfo(self._handle, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(self._handle, n.NVML_CLOCK_SM)
        try:
            bits = n.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
        except Exception:
            bits = n.nvmlDeviceGetCurrentClocksThrottleReasons(self._handle)
        return float(sm), float(mx), int(bits)

    def _sample_smi(self):
        out = subprocess.run(["nvidia-smi", "-i", str(self.device_index), "--query-gpu=clocks.sm,clocks.max.sm,"
                              "clocks_event_reasons.active", "--format=csv,noheader,nounits"],
                             capture_output=True, text=True, timeout=5).stdout.strip().split(",")
        return float(out[0]), float(out[1]), int(out[2].strip(), 16)

    def _run(self):
        period = 0.02 if self._nvml else 0.2
        while not self._stop.is_set():
            try:
                self.samples.append(self._sample_nvml() if self._nvml else self._sample_smi())
            except Exception:
                pass
            self._stop.wait(period)

    def __enter__(self):
        self._stop.clear()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        sm = [x[0] for x in self.samples]
        mx = [x[1] for x in self.samples]
        reasons = sorted({name for _, _, bits in self.samples for b, name in self.REASONS.items() if bits & b})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml" if self._nvml else "nvidia-smi"}


# ---------------------------------------------------------------- helpers

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    """Max of a host scalar over all ranks (timing only; not on the data path)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(per_rank_units, world, seconds):
    """Whole-job throughput: units processed by all ranks / max-over-ranks device time."""
    return per_rank_units * world / seconds


def l2_flush_buffer():
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    return torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")


def traffic_for(kernel_key, source_files):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent:
        return None
    h = hashlib.sha256()
    for rel in source_files:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if ent.get("source_sha256") != h.hexdigest():
        return None
    return ent.get("dram_bytes_per_launch")


def timed_calls(fn, n, stream, sampler, flush=None, spin=True):
    """n calls of fn on `stream`, each bracketed by CUDA events (an L2 flush before each when
    `flush` is given).  A GPU-side spin queued first keeps every timed call enqueued before the
    GPU reaches it, so the events bracket device work only.  Returns the per-call ms."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    with sampler:
        if spin:
            torch.cuda._sleep(int(2e8))
        for a, b in ev:
            if flush is not None:
                flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def err_stats(got, ref):
    """Max and mean absolute error of a GPU result against an fp64 oracle array."""
    g = got.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    e = np.abs(g - ref)
    return {"max_abs_err": float(e.max()), "mean_abs_err": float(e.mean()), "finite": bool(np.isfinite(g).all()),
            "outputs_compared": int(e.size)}


def within(stats, max_tol=1e-2, mean_tol=1e-3):
    return bool(stats["finite"] and stats["max_abs_err"] <= max_tol and stats["mean_abs_err"] <= mean_tol)


class OracleTimer:
    def __init__(self):
        self.s = 0.0

    def __call__(self, f, *a, **k):
        t0 = time.perf_counter()
        r = f(*a, **k)
        self.s += time.perf_counter() - t0
        return r


# ---------------------------------------------------------------- reference arm (the CPU oracle)

def reference_decode_inputs(cfg):
    """Inputs of one decode step of `cfg` for the oracle: the query, a compressed cache with
    the workload's shape and the raw window, drawn on the host with a seeded generator.  The
    decode's work does not depend on the cache's values, so its entries are drawn directly
    (N(0, 0.1^2), the spread of pooled N(0, 1) rows) instead of pooling 17 GB of raw history."""
    import oracle
    g = torch.Generator().manual_seed(cfg.seed)
    B, Hkv, d = cfg.B, cfg.Hkv, cfg.d
    Nc = cfg.T // cfg.blk
    q = torch.randn((B, cfg.Hq, d), generator=g).to(torch.bfloat16)
    kc = (torch.randn((B, Nc, Hkv, d), generator=g) * 0.1).to(torch.bfloat16)
    vc = (torch.randn((B, Nc, Hkv, cfg.dv), generator=g) * 0.1).to(torch.bfloat16)
    kw = torch.randn((B, cfg.W, Hkv, d), generator=g).to(torch.bfloat16)
    vw = torch.randn((B, cfg.W, Hkv, cfg.dv), generator=g).to(torch.bfloat16)
    seq = np.full((B,), cfg.T, np.int32)
    return [oracle.bf16_bits(x) for x in (q, kc, vc, kw, vw)] + [seq]


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sys.path.insert(0, ROOT)
    import oracle
    from compressed_long_context_b200 import workloads as wl
    cfg = wl.DECODE_128K
    qb, kcb, vcb, kwb, vwb, seq = reference_decode_inputs(cfg)
    scale = 1.0 / np.sqrt(cfg.d)

    def step():
        return oracle.decode(qb, kcb, vcb, kwb, vwb, seq, cfg.blk, cfg.W, scale)

    for _ in range(max(1, args.warmup)):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    qps = cfg.B / dt
    cores = oracle.num_threads()
    sample = ("oracle fp64 decode of the whole batch per step: %d queries (64 heads each) over 1023 cached "
              "entries + 128 window tokens; cache entries drawn directly with the workload's shape" % cfg.B)
    line = {"metric": METRIC, "value": qps, "unit": "queries/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "L": cfg.T, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                       "blk": cfg.blk, "W": cfg.W, "step": "oracle decode of the batch (cache resident)"},
            "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm: one function per workload

class Ctx:
    def __init__(self, args, world, rank, local):
        import compressed_long_context_b200 as hca
        from compressed_long_context_b200 import workloads as wl
        self.args, self.world, self.rank = args, world, rank
        self.hca, self.wl = hca, wl
        self.pk, self.pk_kind = peaks()
        self.dev = torch.device("cuda", torch.cuda.current_device())
        self.stream = torch.cuda.current_stream()
        self.flush = l2_flush_buffer()
        self.sampler = ClockSampler(local)
        self.oracle_on = world == 1 and not args.no_oracle
        self.launches = 0

    def hbm_roof(self, kernel, nbytes, seconds, traffic=None):
        gbs = nbytes / seconds / 1e9
        return {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": self.pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / self.pk["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes, "traffic": traffic,
                "peak_kind": self.pk_kind + " (hbm_gbs)"}

    def median_s(self, ms):
        return max_over_ranks(statistics.median(ms) / 1e3, self.world)

    def mean_s(self, ms):
        return max_over_ranks(sum(ms) / len(ms) / 1e3, self.world)


def oracle_cache_of(oracle, k, v, w, blk, timer):
    kc, vc = timer(oracle.compress, oracle.bf16_bits(k), oracle.bf16_bits(v),
                   None if w is None else w.cpu().numpy(), blk)
    return kc, vc, timer(oracle.round_bf16, kc), timer(oracle.round_bf16, vc)


def bench_tiny_prefill(c):
    hca, wl = c.hca, c.wl
    cfg = wl.TINY_PREFILL
    inp = wl.prefill_inputs(cfg, c.dev)
    scale = 1.0 / np.sqrt(cfg.d)
    kc = torch.empty((1, cfg.T // cfg.blk, 1, cfg.d), dtype=torch.bfloat16, device=c.dev)
    vc = torch.empty_like(kc)
    out = torch.empty((1, cfg.T, cfg.Hq, cfg.dv), dtype=torch.float32, device=c.dev)

    def step():
        hca.compress(inp["k"], inp["v"], inp["w"], cfg.blk, kc=kc, vc=vc)
        hca.prefill(inp["q"], inp["k"], inp["v"], kc, vc, cfg.blk, cfg.W, scale, out=out, out_f32=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    hca.get_device_error()
    ms = timed_calls(step, c.args.steps, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    flops, keys = prefill_flops(1, cfg.T, cfg.Hq, cfg.d, cfg.dv, cfg.blk, cfg.W)
    t = c.median_s(ms)
    res = {"workload": cfg.name, "us": t * 1e6, "what": "hca_compress + hca_prefill (fp32 output)",
           "algorithmic_flops": flops, "keys_per_head": keys, "tflops": flops / t / 1e12,
           "bound": "launch latency (4 row tiles)"}
    if c.oracle_on:
        import oracle
        tm = OracleTimer()
        rk, rv, kcb, vcb = oracle_cache_of(oracle, inp["k"], inp["v"], inp["w"], cfg.blk, tm)
        rows = [(0, t) for t in range(cfg.T)]
        ro = tm(oracle.prefill_rows, oracle.bf16_bits(inp["q"]), oracle.bf16_bits(inp["k"]),
                oracle.bf16_bits(inp["v"]), kcb, vcb, cfg.blk, cfg.W, scale, rows)
        e = err_stats(out[0], ro)
        ek = err_stats(kc, rk)
        res["oracle"] = {"seconds": tm.s, "cores": oracle.num_threads(), "scope": "full (every row and head)"}
        res["parity"] = dict(e, cache_max_abs_err=ek["max_abs_err"],
                             within_tolerance=within(e) and ek["max_abs_err"] <= 4e-3)
    return res


def bench_decode_128k(c):
    """The headline: decode alone (cache resident, L2 flushed before each call); compress of the
    raw K/V timed separately (GB/s); serving step; e2e through host buffers; oracle parity."""
    hca, wl = c.hca, c.wl
    cfg = wl.DECODE_128K
    scale = 1.0 / np.sqrt(cfg.d)
    inp = wl.decode_inputs(cfg, c.dev)
    k, v, w, q, kw, vw, seq = (inp[x] for x in ("k", "v", "w", "q", "kw", "vw", "seqlens"))
    B, L = cfg.B, cfg.T
    Nc = L // cfg.blk
    kc = torch.empty((B, Nc, 1, cfg.d), dtype=torch.bfloat16, device=c.dev)
    vc = torch.empty((B, Nc, 1, cfg.dv), dtype=torch.bfloat16, device=c.dev)
    out = torch.empty((B, cfg.Hq, cfg.dv), dtype=torch.float32, device=c.dev)
    ws = torch.empty(hca.decode_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.dv), dtype=torch.uint8, device=c.dev)

    def comp():
        hca.compress(k, v, w, cfg.blk, kc=kc, vc=vc)

    def dec():
        hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws)

    for _ in range(max(3, c.args.warmup)):
        comp()
        dec()
    torch.cuda.synchronize()
    hca.get_device_error()

    # ---- the headline: K timed decode calls
    barrier(c.world)
    torch.cuda.synchronize()
    d_ms = timed_calls(dec, c.args.steps, c.stream, c.sampler, flush=c.flush)
    barrier(c.world)
    hca.get_device_error()
    c.launches += 2 * c.args.steps
    t_dec = c.mean_s(d_ms)
    dbytes = decode_bytes(B, L, cfg.Hq, 1, cfg.d, cfg.dv, cfg.blk, cfg.W)
    head = {"value": weak_scaling_value(B, c.world, t_dec), "ms_per_step": t_dec * 1e3,
            "roofline": c.hbm_roof("decode_split_kernel + decode_combine_kernel", dbytes, t_dec,
                                   traffic_for("decode_B64_L131072", ["compressed_long_context_b200/csrc/decode.cuh"]))}

    # ---- compress of the raw history (17.35 GB), its own GB/s
    c_ms = timed_calls(comp, max(3, min(c.args.steps, 10)), c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    cbytes = compress_bytes(B, L, 1, cfg.d, cfg.dv, cfg.blk)
    t_c = c.mean_s(c_ms)
    res = {"workload": cfg.name, "what": "hca_decode (split + combine), cache resident; compress separately",
           "decode": {"us": t_dec * 1e6, "median_us": statistics.median(d_ms) * 1e3,
                      "queries_per_s": B / t_dec, "algorithmic_bytes": dbytes,
                      "bytes_per_query": dbytes // B, "roofline": head["roofline"]},
           "compress": {"ms": t_c * 1e3, "gbs": cbytes / t_c / 1e9, "algorithmic_bytes": cbytes,
                        "bytes_per_entry": cbytes // (B * Nc),
                        "roofline": c.hbm_roof("compress_kernel<512,512>", cbytes, t_c,
                                               traffic_for("compress_decode_B64_L131072",
                                                           ["compressed_long_context_b200/csrc/compress.cuh"]))}}

    # ---- one serving step: hca_append of every sequence's newest token, then hca_decode over the
    # window ring (at L = 131072 every sequence completes a block, so an entry is written too)
    kn, vn = k[:, L - 1].contiguous(), v[:, L - 1].contiguous()
    wn = w[:, L - 1].contiguous()
    state = torch.zeros(hca.append_state_size(B, 1, cfg.d, cfg.dv), dtype=torch.uint8, device=c.dev)
    kc_s, vc_s = kc.clone(), vc.clone()
    kw_s, vw_s = kw.clone(), vw.clone()

    def serve(decode_too):
        hca.append(kn, vn, wn, seq, kw_s, vw_s, kc_s, vc_s, state, cfg.blk)
        if decode_too:
            hca.decode(q, kc_s, vc_s, kw_s, vw_s, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws,
                       window_ring=True)

    serve_part = {}
    for name, dflag in (("append_us", False), ("append_plus_decode_us", True)):
        for _ in range(3):
            serve(dflag)
        sm = timed_calls(lambda: serve(dflag), c.args.steps, c.stream, c.sampler, flush=c.flush)
        serve_part[name] = c.median_s(sm) * 1e6
    hca.get_device_error()
    abytes = append_bytes(B, 1, cfg.d, cfg.dv)
    serve_part.update({"append_algorithmic_bytes": abytes,
                       "append_frac_of_hbm": abytes / (serve_part["append_us"] / 1e6) / 1e9 / c.pk["hbm_gbs"],
                       "append_bound": "latency (one small CTA per sequence; %d KB moved)" % (abytes // 1024)})
    res["serving_step"] = serve_part
    del state, kc_s, vc_s, kw_s, vw_s

    # ---- the gated layer's extras on the same batch: the low-rank gate projection (query latent
    # 1024 -> 64 x 512 logits; 64 MB of weights read once) and the decode with the gate and
    # Virtual Head Attention (rank 8) fused into its merge
    gg = torch.Generator(device=c.dev).manual_seed(6)
    cq = torch.randn((B, 1024), generator=gg, device=c.dev).to(torch.bfloat16)
    wg = (torch.randn((1024, cfg.Hq, cfg.dv), generator=gg, device=c.dev) / 32.0).to(torch.bfloat16)
    gate = torch.empty((B, cfg.Hq, cfg.dv), dtype=torch.bfloat16, device=c.dev)
    vu = torch.randn((cfg.Hq, 8), generator=gg, device=c.dev) * 0.1
    vv = torch.randn((cfg.Hq, 8), generator=gg, device=c.dev) * 0.1

    def gate_proj():
        hca.gate_logits(cq, wg, out=gate)

    def dec_gated_vha():
        hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, gate=gate, vha_u=vu, vha_v=vv, out=out,
                   workspace=ws)

    for _ in range(3):
        gate_proj()
        dec_gated_vha()
    torch.cuda.synchronize()
    hca.get_device_error()
    g_ms = timed_calls(gate_proj, c.args.steps, c.stream, c.sampler, flush=c.flush)
    v_ms = timed_calls(dec_gated_vha, c.args.steps, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    t_g, t_v = c.mean_s(g_ms), c.mean_s(v_ms)
    gbytes = (cq.numel() + wg.numel() + gate.numel()) * 2
    vbytes = dbytes + B * cfg.Hq * cfg.dv * 2
    res["gated_layer"] = {
        "gate_projection": {"us": t_g * 1e6, "algorithmic_bytes": gbytes,
                            "roofline": c.hbm_roof("gate_logits_kernel", gbytes, t_g)},
        "decode_gate_vha_fused": {"us": t_v * 1e6, "rank": 8, "queries_per_s": B / t_v, "algorithmic_bytes": vbytes,
                                  "roofline": c.hbm_roof("decode_split_kernel + decode_combine_kernel<.., vha>",
                                                         vbytes, t_v)}}
    del cq, wg, gate, vu, vv

    # ---- parity of the benchmarked decode (and compress) against the oracle, every output
    dec()
    torch.cuda.synchronize()
    hca.get_device_error()
    ref_cache = None
    if c.oracle_on:
        import oracle
        tm = OracleTimer()
        rk, rv, kcb, vcb = oracle_cache_of(oracle, k, v, w, cfg.blk, tm)
        t_comp = tm.s
        ro = tm(oracle.decode, oracle.bf16_bits(q), kcb, vcb, oracle.bf16_bits(kw), oracle.bf16_bits(vw),
                seq.cpu().numpy(), cfg.blk, cfg.W, scale)
        e = err_stats(out, ro)
        ek = err_stats(kc, rk)
        ev = err_stats(vc, rv)
        res["oracle"] = {"seconds": tm.s, "compress_seconds": t_comp, "decode_seconds": tm.s - t_comp,
                         "cores": oracle.num_threads(), "scope": "full (every sequence, head and channel)"}
        res["parity"] = dict(e, cache_max_abs_err=max(ek["max_abs_err"], ev["max_abs_err"]),
                             within_tolerance=within(e) and max(ek["max_abs_err"], ev["max_abs_err"]) <= 4e-3)
        ref_cache = (oracle.bf16_bits(q), kcb, vcb, oracle.bf16_bits(kw), oracle.bf16_bits(vw),
                     seq.cpu().numpy(), cfg.blk, cfg.W, scale)
        del rk, rv
    del k, v, w, inp
    torch.cuda.empty_cache()

    # ---- e2e through the public API: the step's inputs copied from pinned host buffers, the
    # result read back, both inside the timed region
    e2e = None
    if not c.args.no_e2e:
        srcs = (q, kc, vc, kw, vw, seq)
        hsrc = [x.cpu().pin_memory() for x in srcs]
        dsts = [torch.empty_like(x) for x in srcs]
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h2d = sum(x.numel() * x.element_size() for x in hsrc)
        d2h = hout.numel() * hout.element_size()

        def e2e_step():
            for hs, dd in zip(hsrc, dsts):
                dd.copy_(hs, non_blocking=True)
            hca.decode(dsts[0], dsts[1], dsts[2], dsts[3], dsts[4], dsts[5], cfg.blk, cfg.W, scale, out=out,
                       workspace=ws)
            hout.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        ne = max(3, min(c.args.steps, 10))
        barrier(c.world)
        e_ms = timed_calls(e2e_step, ne, c.stream, c.sampler, flush=None, spin=False)
        barrier(c.world)
        hca.get_device_error()
        te = c.mean_s(e_ms)
        e2e = {"value": weak_scaling_value(B, c.world, te), "unit": "queries/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": ne,
               "step": "pinned host -> device copies of q, cache, window and lengths; hca_decode; output read back"}
        del hsrc, dsts, hout
    del kc, vc, out, ws
    torch.cuda.empty_cache()
    return head, res, e2e, ref_cache


def bench_prefill_128k(c):
    hca, wl = c.hca, c.wl
    pc = wl.PREFILL_128K
    scale = 1.0 / np.sqrt(pc.d)
    pin = wl.prefill_inputs(pc, c.dev)
    pkc, pvc = hca.compress(pin["k"], pin["v"], pin["w"], pc.blk)
    pout = torch.empty((1, pc.T, pc.Hq, pc.dv), dtype=torch.bfloat16, device=c.dev)

    def pre():
        hca.prefill(pin["q"], pin["k"], pin["v"], pkc, pvc, pc.blk, pc.W, scale, out=pout)

    def comp():
        hca.compress(pin["k"], pin["v"], pin["w"], pc.blk, kc=pkc, vc=pvc)

    for _ in range(2):
        comp()
        pre()
    torch.cuda.synchronize()
    hca.get_device_error()
    n = max(3, min(c.args.steps, 6))
    p_ms = timed_calls(pre, n, c.stream, c.sampler, flush=c.flush)
    c_ms = timed_calls(comp, n, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    flops, keys = prefill_flops(1, pc.T, pc.Hq, pc.d, pc.dv, pc.blk, pc.W)
    tp = c.median_s(p_ms)
    tf = flops / tp / 1e12
    burst = c.pk["bf16_tflops"]
    sust = c.pk.get("bf16_tflops_sustained", burst)
    res = {"workload": pc.name, "what": "hca_prefill (bf16 output) after hca_compress of the raw K/V",
           "ms": tp * 1e3, "compress_ms": c.median_s(c_ms) * 1e3, "tflops": tf, "algorithmic_flops": flops,
           "flops_per_row_key": 2 * pc.Hq * (pc.d + pc.dv), "keys_per_head": keys,
           "roofline": {"bound": "tensor", "kernel": "prefill_pair_kernel", "achieved": tf, "peak": burst,
                        "unit": "TFLOP/s", "frac": tf / burst,
                        "peak_kind": c.pk_kind + " (bf16_tflops, burst: each call is an isolated ~15 ms launch)",
                        "frac_of_sustained": tf / sust,
                        "traffic": traffic_for("prefill_T131072",
                                               ["compressed_long_context_b200/csrc/prefill.cuh",
                                                "compressed_long_context_b200/csrc/prefill_pair.cuh"])}}
    # Virtual Head Attention on the prefill output (in place, bf16), synthetic rank-8 factors
    gv = torch.Generator(device=c.dev).manual_seed(5)
    vu = torch.randn((pc.Hq, 8), generator=gv, device=c.dev) * 0.1
    vv = torch.randn((pc.Hq, 8), generator=gv, device=c.dev) * 0.1
    vout = pout.clone()
    hca.vha(vout, vu, vv)
    v_ms = timed_calls(lambda: hca.vha(vout, vu, vv), n, c.stream, c.sampler)
    hca.get_device_error()
    tv = c.median_s(v_ms)
    vbytes = vha_bytes(vout.numel(), vout.element_size(), pc.Hq, vu.shape[1])
    res["vha"] = {"ms": tv * 1e3, "rank": 8, "algorithmic_bytes": vbytes,
                  "roofline": c.hbm_roof("vha_kernel<false,8>", vbytes, tv)}
    del vout
    res["backward"] = bench_backward_128k(c, pc, pin, pkc, pvc, scale, flops, keys, n)
    if c.oracle_on:
        import oracle
        T = pc.T
        kmax = pin["k"][0, :, 0].float().abs().amax(dim=1)
        boosted = torch.nonzero(kmax > 6.0).flatten().tolist()[:8]
        rs = np.random.RandomState(2)
        ts = set([0, 1, 127, 128, 129, 255, 256, T - 2, T - 1])
        ts |= set(int(x) for x in rs.randint(0, T, 40))
        ts |= set(min(T - 1, b + o) for b in boosted for o in (0, 127))
        rows = [(0, t) for t in sorted(ts)]
        tm = OracleTimer()
        rk, rv, kcb, vcb = oracle_cache_of(oracle, pin["k"], pin["v"], pin["w"], pc.blk, tm)
        t_comp = tm.s
        qsel = oracle.bf16_bits(pin["q"][0, [t for _, t in rows]])
        ro = tm(oracle.prefill_rows, qsel, oracle.bf16_bits(pin["k"]), oracle.bf16_bits(pin["v"]), kcb, vcb,
                pc.blk, pc.W, scale, rows, q_rows=True)
        t_rows = tm.s - t_comp
        idx = torch.tensor([t for _, t in rows], device=c.dev)
        got = pout[0, idx]
        e = err_stats(got, ro)
        # the bf16 output is the stored result: within the bar plus half a bf16 ulp of the reference
        half_ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(ro), 2.0 ** -126))).astype(np.int64) - 8)
        g64 = got.float().cpu().numpy().astype(np.float64)
        ok_bf16 = bool(np.all(np.abs(g64 - ro) <= 1e-2 + half_ulp))
        ek = err_stats(pkc, rk)
        sel_keys = sum(oracle.visible_entries(t, pc.W, pc.blk) + min(pc.W, t + 1) for _, t in rows)
        res["oracle"] = {"seconds_sampled_rows": t_rows, "compress_seconds": t_comp, "rows": len(rows),
                         "cores": oracle.num_threads(),
                         "seconds_full_extrapolated": t_comp + t_rows * keys / sel_keys,
                         "scope": "compress in full; %d sampled query rows x all 64 heads (the full fp64 "
                                  "prefill is ~1.1e13 flop), extrapolated by visible keys" % len(rows)}
        res["parity"] = dict(e, cache_max_abs_err=ek["max_abs_err"], bf16_within_bar_plus_half_ulp=ok_bf16,
                             within_tolerance=ok_bf16 and e["mean_abs_err"] <= 1e-3 and ek["max_abs_err"] <= 4e-3)
    del pin, pkc, pvc, pout
    torch.cuda.empty_cache()
    return res


class RowsF64:
    """Read-only fp64 view of a bf16 device tensor, converted on indexing, so that the oracle's
    row-by-row reads of a 128K-token input need no host copy of the whole tensor."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        import oracle
        return oracle.bits_to_f64(oracle.bf16_bits(self.t[idx]))


def backward_segments(B, T, Hq, Hkv, blk, W, cap=2 << 30):
    """Segments of row tiles hca_prefill_backward walks (each one dq and one dk/dv launch)."""
    tpt = 128 // (Hq // Hkv)
    ntile = (T + tpt - 1) // tpt
    nkc, nkw = (T // blk + 127) // 128, (T + 127) // 128
    nt_max = nkc + min((tpt + W - 2) // 128 + 2, nkw)
    seg = max(1, min(ntile, cap // (B * Hkv * nt_max * 65536)))
    return (ntile + seg - 1) // seg


def bench_backward_128k(c, pc, pin, pkc, pvc, scale, fwd_flops, keys, n):
    """Training step of the prefill workload: hca_prefill with the log-sum-exp, then
    hca_prefill_backward (dq, dk, dv, dw) for a synthetic dout."""
    hca = c.hca
    g = torch.Generator(device=c.dev).manual_seed(9)
    dout = torch.empty_like(pin["q"])
    flat = dout.view(-1)
    for i in range(0, flat.numel(), 1 << 28):
        m = min(1 << 28, flat.numel() - i)
        flat[i:i + m] = torch.randn(m, generator=g, device=c.dev).to(torch.bfloat16)
    # the forward output in fp32: D = rowsum(dout * out) then carries no bf16 rounding of out, which
    # rows dominated by one key (the boosted ones) would turn into a large relative error of dS
    out, lse = hca.prefill(pin["q"], pin["k"], pin["v"], pkc, pvc, pc.blk, pc.W, scale, want_lse=True,
                           out_f32=True)
    grads = {}

    def bwd():
        grads["g"] = hca.prefill_backward(pin["q"], pin["k"], pin["v"], pin["w"], pkc, pvc, out, lse, dout,
                                          pc.blk, pc.W, scale)

    for _ in range(2):
        bwd()
    torch.cuda.synchronize()
    hca.get_device_error()
    b_ms = timed_calls(bwd, n, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    tb = c.median_s(b_ms)
    # five contractions of the forward's size: S, dP, dq, dk, dv (2.5x the forward's flops)
    flops = 2.5 * fwd_flops
    tf = flops / tb / 1e12
    burst = c.pk["bf16_tflops"]
    res = {"what": "hca_prefill_backward: dq, dk, dv, dw of the prefill workload (forward output fp32, "
                   "its LSE, synthetic bf16 dout)",
           "ms": tb * 1e3, "tflops": tf, "algorithmic_flops": flops,
           "flops_per_row_key": 5 * 2 * pc.Hq * pc.d,
           "roofline": {"bound": "tensor", "kernel": "bwd_dq_kernel + bwd_dkv_kernel", "achieved": tf,
                        "peak": burst, "unit": "TFLOP/s", "frac": tf / burst,
                        "peak_kind": c.pk_kind + " (bf16_tflops, burst)", "traffic": None}}
    from compressed_long_context_b200 import _lib
    res["workspace_bytes"] = int(_lib.load().hca_prefill_backward_workspace_size(1, pc.T, pc.Hq, pc.Hkv, pc.dv,
                                                                                  pc.blk, pc.W))
    res["launches_per_call"] = 2 + 2 * backward_segments(1, pc.T, pc.Hq, pc.Hkv, pc.blk, pc.W)
    if c.oracle_on:
        from oracle import backward as ob
        import oracle
        T, blk, W = pc.T, pc.blk, pc.W
        Nc = T // blk
        rows = [0, 127, 128, 255, 16511, 16512, 65537, T - 2, T - 1]
        raw = [blk * (Nc - 3), blk * (Nc - 3) + 77, T - 128, T - 1]
        tm = OracleTimer()
        f64 = lambda t: oracle.bits_to_f64(oracle.bf16_bits(t))  # noqa: E731
        # q and dout are widened row by row on access (the oracle reads one (t, h) row at a time)
        qn, don = RowsF64(pin["q"]), RowsF64(dout)
        kn, vn = f64(pin["k"]), f64(pin["v"])
        ref = tm(ob.backward_sampled, qn, kn, vn, pin["w"].cpu().numpy(), blk, W, scale, don, 0, rows=rows, raw=raw)
        dq, dk, dv, dw = grads["g"]

        def rel(got, r):
            g64 = got.double().cpu().numpy()
            return float(np.sqrt(((g64 - r) ** 2).sum() / max((r ** 2).sum(), 1e-300))), \
                float(np.abs(g64 - r).max() / max(np.abs(r).max(), 1e-300))

        out_rel = {}
        for name, got, r in (("dq", dq[0, rows], np.stack([ref["dq"][t] for t in rows])),
                             ("dk", dk[0, raw], np.stack([ref["dk"][u] for u in raw])),
                             ("dv", dv[0, raw], np.stack([ref["dv"][u] for u in raw]))):
            nr, mr = rel(got, r)
            out_rel[name] = {"normwise_rel_err": nr, "max_err_over_max_ref": mr}
        ok = all(v["normwise_rel_err"] <= 2 ** -7 and v["max_err_over_max_ref"] <= 2 ** -5 for v in out_rel.values())
        res["oracle"] = {"seconds": tm.s, "rows": len(rows), "raw_positions": len(raw), "cores": oracle.num_threads(),
                         "scope": "oracle.backward.backward_sampled: dq of %d query positions, dk/dv of %d raw "
                                  "positions (window path, and the pooling path of a late block)" % (len(rows), len(raw))}
        res["parity"] = dict(out_rel, within_tolerance=ok,
                             bar="normwise <= 2^-7 and max <= 2^-5 of the largest reference value")
        del qn, kn, vn, don
    del dout, out, lse, grads
    torch.cuda.empty_cache()
    return res


def bench_decode_1m(c):
    hca, wl = c.hca, c.wl
    cfg = wl.DECODE_1M
    scale = 1.0 / np.sqrt(cfg.d)
    inp = wl.decode_inputs(cfg, c.dev)
    k, v, w, q, kw, vw, seq = (inp[x] for x in ("k", "v", "w", "q", "kw", "vw", "seqlens"))
    B, L = cfg.B, cfg.T
    Nc = L // cfg.blk
    kc = torch.empty((B, Nc, 1, cfg.d), dtype=torch.bfloat16, device=c.dev)
    vc = torch.empty((B, Nc, 1, cfg.dv), dtype=torch.bfloat16, device=c.dev)
    out = torch.empty((B, cfg.Hq, cfg.dv), dtype=torch.float32, device=c.dev)
    ws = torch.empty(hca.decode_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.dv), dtype=torch.uint8, device=c.dev)

    def comp():
        hca.compress(k, v, w, cfg.blk, kc=kc, vc=vc)

    def dec():
        hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws)

    for _ in range(3):
        comp()
        dec()
    torch.cuda.synchronize()
    hca.get_device_error()
    c_ms = timed_calls(comp, max(3, min(c.args.steps, 10)), c.stream, c.sampler, flush=c.flush)
    d_ms = timed_calls(dec, c.args.steps, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    t_c, t_d = c.mean_s(c_ms), c.mean_s(d_ms)
    cbytes = compress_bytes(B, L, 1, cfg.d, cfg.dv, cfg.blk)
    dbytes = decode_bytes(B, L, cfg.Hq, 1, cfg.d, cfg.dv, cfg.blk, cfg.W)
    res = {"workload": cfg.name, "what": "hca_compress (timed alone) then hca_decode (cache resident)",
           "compress": {"ms": t_c * 1e3, "gbs": cbytes / t_c / 1e9, "algorithmic_bytes": cbytes,
                        "roofline": c.hbm_roof("compress_kernel<512,512>", cbytes, t_c)},
           "decode": {"us": t_d * 1e6, "median_us": statistics.median(d_ms) * 1e3, "queries_per_s": B / t_d,
                      "algorithmic_bytes": dbytes, "bytes_per_query": dbytes // B,
                      "roofline": c.hbm_roof("decode_split_kernel + decode_combine_kernel", dbytes, t_d)}}
    dec()
    torch.cuda.synchronize()
    hca.get_device_error()
    if c.oracle_on:
        import oracle
        tm = OracleTimer()
        rk, rv, kcb, vcb = oracle_cache_of(oracle, k, v, w, cfg.blk, tm)
        t_comp = tm.s
        ro = tm(oracle.decode, oracle.bf16_bits(q), kcb, vcb, oracle.bf16_bits(kw), oracle.bf16_bits(vw),
                seq.cpu().numpy(), cfg.blk, cfg.W, scale)
        e = err_stats(out, ro)
        ek = max(err_stats(kc, rk)["max_abs_err"], err_stats(vc, rv)["max_abs_err"])
        res["oracle"] = {"seconds": tm.s, "compress_seconds": t_comp, "decode_seconds": tm.s - t_comp,
                         "cores": oracle.num_threads(), "scope": "full (every sequence, head and channel)"}
        res["parity"] = dict(e, cache_max_abs_err=ek, within_tolerance=within(e) and ek <= 4e-3)
        del rk, rv, kcb, vcb
    del inp, k, v, w, kc, vc, out, ws
    torch.cuda.empty_cache()
    return res


def bench_ragged_paged(c):
    hca, wl = c.hca, c.wl
    cfg = wl.RAGGED_PAGED
    scale = 1.0 / np.sqrt(cfg.d)
    inp = wl.paged_decode_inputs(cfg, c.dev)
    B = cfg.B
    out = torch.empty((B, cfg.Hq, cfg.dv), dtype=torch.float32, device=c.dev)
    ws = torch.empty(hca.decode_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.dv), dtype=torch.uint8, device=c.dev)

    def dec():
        hca.decode(inp["q"], inp["kc"], inp["vc"], inp["kw"], inp["vw"], inp["seqlens"], cfg.blk, cfg.W, scale,
                   page_table=inp["page_table"], page_size=cfg.page_size, gq=inp["gq"], gk=inp["gk"],
                   gate=inp["gate"], out=out, workspace=ws)

    for _ in range(3):
        dec()
    torch.cuda.synchronize()
    hca.get_device_error()
    d_ms = timed_calls(dec, c.args.steps, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    t = c.mean_s(d_ms)
    lens = inp["seqlens"].cpu().tolist()
    dbytes = sum(decode_seq_bytes(L, cfg.Hq, cfg.Hkv, cfg.d, cfg.dv, cfg.blk, cfg.W, gate=True) for L in lens)
    res = {"workload": cfg.name, "what": "hca_decode, paged cache, QK RMSNorm + sigmoid gate",
           "us": t * 1e6, "median_us": statistics.median(d_ms) * 1e3, "queries_per_s": B / t,
           "algorithmic_bytes": dbytes, "mean_context": float(np.mean(lens)),
           "roofline": c.hbm_roof("decode_split_kernel + decode_combine_kernel", dbytes, t)}
    dec()
    torch.cuda.synchronize()
    hca.get_device_error()
    if c.oracle_on:
        import oracle
        tm = OracleTimer()
        b = oracle.bf16_bits
        ro = tm(oracle.decode, b(inp["q"]), b(inp["kc"]), b(inp["vc"]), b(inp["kw"]), b(inp["vw"]),
                inp["seqlens"].cpu().numpy(), cfg.blk, cfg.W, scale, page_table=inp["page_table"].cpu().numpy(),
                page_size=cfg.page_size, gq=inp["gq"].cpu().numpy(), gk=inp["gk"].cpu().numpy(), eps=1e-6,
                gate=b(inp["gate"]))
        e = err_stats(out, ro)
        res["oracle"] = {"seconds": tm.s, "cores": oracle.num_threads(),
                         "scope": "full (every sequence, head and channel)"}
        res["parity"] = dict(e, within_tolerance=within(e))
    del inp, out, ws
    torch.cuda.empty_cache()
    return res


def bench_dsa_decode_128k(c):
    """The sparse-attention decode step: indexer scores, top-k selection, core attention."""
    hca, wl = c.hca, c.wl
    cfg = wl.DSA_DECODE_128K
    inp = wl.dsa_inputs(cfg, c.dev)
    B, L = cfg.B, cfg.L
    scale = 1.0 / np.sqrt(cfg.d)
    scores = torch.empty((B, L), dtype=torch.float32, device=c.dev)
    idx = torch.empty((B, cfg.topk), dtype=torch.int32, device=c.dev)
    out = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.float32, device=c.dev)

    def index():
        hca.dsa_index(inp["q_idx"], inp["w_idx"], inp["k_idx"], inp["seqlens"], scores=scores)

    def topk():
        hca.dsa_topk(scores, inp["seqlens"], cfg.topk, idx=idx)

    def attend():
        hca.dsa_attend(inp["q"], inp["k"], inp["v"], idx, inp["seqlens"], scale, out=out)

    def step():
        index()
        topk()
        attend()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    hca.get_device_error()
    n = max(5, min(c.args.steps, 20))
    s_ms = timed_calls(step, n, c.stream, c.sampler, flush=c.flush)
    i_ms = timed_calls(index, n, c.stream, c.sampler, flush=c.flush)
    k_ms = timed_calls(topk, n, c.stream, c.sampler, flush=c.flush)
    a_ms = timed_calls(attend, n, c.stream, c.sampler, flush=c.flush)
    hca.get_device_error()
    ts, ti, tk, ta = (c.median_s(x) for x in (s_ms, i_ms, k_ms, a_ms))
    # algorithmic bytes: the indexer reads every indexer key once and writes the scores; the
    # selection reads the scores; the attention reads the kept key and value rows, q, writes out
    i_bytes = B * L * cfg.dI * 2 + B * cfg.HI * (cfg.dI * 2 + 4) + B * L * 4
    k_bytes = B * L * 4 + B * cfg.topk * 4
    a_bytes = B * cfg.topk * (2 * cfg.d * 2 + 4) + B * cfg.Hq * cfg.d * (2 + 4)
    res = {"workload": cfg.name, "what": "hca_dsa_index + hca_dsa_topk + hca_dsa_attend, inputs resident",
           "B": B, "L": L, "HI": cfg.HI, "dI": cfg.dI, "topk": cfg.topk, "Hq": cfg.Hq, "d": cfg.d,
           "us": ts * 1e6, "queries_per_s": B / ts,
           "algorithmic_bytes": i_bytes + k_bytes + a_bytes,
           "index": {"us": ti * 1e6, "algorithmic_bytes": i_bytes, "roofline": c.hbm_roof("dsa_index_kernel", i_bytes, ti)},
           "topk": {"us": tk * 1e6, "algorithmic_bytes": k_bytes, "roofline": c.hbm_roof("dsa_topk_kernel", k_bytes, tk)},
           "attend": {"us": ta * 1e6, "algorithmic_bytes": a_bytes, "roofline": c.hbm_roof("dsa_attend_kernel", a_bytes, ta)},
           "roofline": c.hbm_roof("dsa_index_kernel + dsa_topk_kernel + dsa_attend_kernel",
                                  i_bytes + k_bytes + a_bytes, ts)}
    if c.oracle_on:
        import oracle
        from oracle import dsa as od
        f64 = lambda t: oracle.bits_to_f64(oracle.bf16_bits(t))  # noqa: E731
        tm = OracleTimer()
        sel_b = [0, 31, 63]
        worst = {"scores_rel": 0.0, "out_max_abs": 0.0, "out_mean_abs": 0.0, "kept_outside_bound": 0}
        for b in sel_b:
            qi, ki, wi = f64(inp["q_idx"][b:b + 1]), f64(inp["k_idx"][b:b + 1]), inp["w_idx"][b:b + 1].cpu().numpy()
            lens = np.array([L])
            ref_s = tm(od.index_scores, qi, wi, ki, lens)[0]
            got_s = scores[b].double().cpu().numpy()
            bound = 2.0 ** -20 * (np.abs(ki[0] @ qi[0].T) @ np.abs(wi[0].astype(np.float64))) + 1e-6
            rel = np.abs(got_s - ref_s) / bound
            worst["scores_rel"] = max(worst["scores_rel"], float(np.max(rel)) if np.all(np.isfinite(rel)) else float("inf"))
            ridx = tm(od.select_topk, ref_s[None], lens, cfg.topk)[0]
            kept = idx[b].cpu().numpy()
            kth = np.sort(ref_s)[::-1][cfg.topk - 1]
            worst["kept_outside_bound"] += int(np.sum(ref_s[kept] < kth - 2 * bound.max()))
            # the attention over the GPU's kept positions (its selection is checked just above)
            ro = tm(od.sparse_attend, f64(inp["q"][b:b + 1]), f64(inp["k"][b:b + 1]), f64(inp["v"][b:b + 1]),
                    kept[None], scale)[0]
            e = np.abs(out[b].double().cpu().numpy() - ro)
            worst["out_max_abs"] = max(worst["out_max_abs"], float(e.max()))
            worst["out_mean_abs"] = max(worst["out_mean_abs"], float(e.mean()))
            worst["same_selection_as_oracle"] = worst.get("same_selection_as_oracle", True) and bool(np.array_equal(kept, ridx))
        res["oracle"] = {"seconds": tm.s, "sequences": len(sel_b), "cores": oracle.num_threads(),
                         "seconds_full_extrapolated": tm.s * B / len(sel_b),
                         "scope": "oracle.dsa on 3 of the 64 sequences (scores, selection, attention)"}
        res["parity"] = dict(worst, within_tolerance=bool(worst["scores_rel"] <= 1.0 and worst["kept_outside_bound"] == 0
                                                          and worst["out_max_abs"] <= 1e-2
                                                          and worst["out_mean_abs"] <= 1e-3),
                             bar="scores within 2^-20 sum|w||q.k|; kept positions a top-k within that bound; "
                                 "attention max abs 1e-2, mean abs 1e-3")
    del inp, scores, idx, out
    torch.cuda.empty_cache()
    return res


def cpu_baseline_sample(ref_cache, target_s=10.0):
    """The oracle as it stands, on this host, for a bounded sample of the headline workload: the
    oracle's decode of the whole 64-query batch over its own compressed cache, repeated for about
    ``target_s`` seconds."""
    import oracle
    B = ref_cache[0].shape[0]
    reps = 0
    t0 = time.perf_counter()
    while True:
        oracle.decode(*ref_cache)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            break
    return {"value": B * reps / dt, "unit": "queries/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d oracle fp64 decodes of the whole batch (%d queries, 64 heads, 1023 entries + 128 window "
                      "tokens each, over the oracle's own compressed cache), %.1f s" % (reps, B, dt)}


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        run_reference(args)
        return
    world, rank, local = dist_setup(args)
    sys.path.insert(0, ROOT)
    from compressed_long_context_b200 import _lib
    c = Ctx(args, world, rank, local)
    want = set(x.strip() for x in args.configs.split(",") if x.strip())
    unknown = want - set(CONFIG_KEYS)
    if unknown:
        raise SystemExit("unknown configs: %s" % ",".join(sorted(unknown)))

    configs = {}
    head, configs["decode_128k"], e2e, ref_cache = bench_decode_128k(c)
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and ref_cache is not None:
        cpu_base = cpu_baseline_sample(ref_cache)
    del ref_cache
    runners = {"tiny_prefill": bench_tiny_prefill, "prefill_128k": bench_prefill_128k,
               "decode_1m": bench_decode_1m, "ragged_paged": bench_ragged_paged,
               "dsa_decode_128k": bench_dsa_decode_128k}
    for key in CONFIG_KEYS:
        if key in runners and key in want:
            configs[key] = runners[key](c)
            barrier(world)

    clocks = c.sampler.summary()
    if rank == 0:
        cfg = c.wl.DECODE_128K
        line = {"metric": METRIC, "value": head["value"], "unit": "queries/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded; no dataset)",
                "config": {"workload": cfg.name, "B": cfg.B, "L": cfg.T, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                           "blk": cfg.blk, "W": cfg.W,
                           "step": "hca_decode of the batch (split + combine kernels), compressed cache resident",
                           "l2": "flushed (2x L2 memset) before every timed call",
                           "parallelism": "dp%d (independent batches, no collective)" % world},
                "roofline": head["roofline"], "configs": configs, "cpu_baseline": cpu_base, "e2e": e2e,
                "gpu_launches": 2 * args.steps, "clocks": clocks,
                "libhca": os.path.relpath(_lib.LIB_PATH, ROOT)}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
