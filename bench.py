"""Benchmark of the HCA hot path on B200 (one JSON line on stdout).

Workload (the decode configuration the headline metric is quoted on): 64 sequences of
131072 tokens, Hq=64 query heads sharing one 512-dim KV head, blocks of 128, a raw
window of 128 tokens; pooling weights ~N(0, 0.5); bf16 inputs ~N(0, 1); seed 1.

One step = the whole path for one batch:
    hca_compress  (raw K/V [64, 131072, 1, 512] -> 1024 cached entries per sequence)
    hca_decode    (one query per sequence over 1023 entries + 128 raw tokens;
                   split kernel + combine kernel)
value = queries of all ranks / device time of the step (max over ranks).

Also reported, measured in the same run: the decode kernels alone (cache resident,
L2 flushed before each call) and the 128K prefill (T=131072, Hq=64, d=512, W=128,
1% of raw keys x8; seed 2) in TFLOP/s.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: torchrun, one rank per GPU, each rank a full batch (weak scaling).
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- algorithmic work

def compress_bytes(B, T, Hkv, d, dv, blk):
    Nc = T // blk
    return B * Nc * Hkv * (blk * (d + dv) * 2 + 2 * (d + dv)) + B * Nc * blk * 4


def decode_bytes(B, L, Hq, Hkv, d, dv, blk, W):
    nc = max(0, (L - W) // blk)
    nw = min(W, L)
    per = Hq * d * 2 + (nc + nw) * Hkv * (d + dv) * 2 + Hq * dv * 4 + 4
    return B * per


def append_bytes(B, Hkv, d, dv):
    """hca_append when every sequence completes a block: new token read, pooling state read and
    written, ring slot written, entry written (bytes per call)."""
    state = (4 + d + dv) * 4
    return B * Hkv * ((d + dv) * 2 + 2 * state + (d + dv) * 2 + (d + dv) * 2) + B * 8


def vha_bytes(numel, esize, Hq, r):
    """hca_vha in place: the output read and written once, plus the two fp32 factors."""
    return 2 * numel * esize + 2 * Hq * r * 4


def prefill_flops(B, T, Hq, d, dv, blk, W):
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


# ---------------------------------------------------------------- reference arm (the CPU oracle)

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sys.path.insert(0, ROOT)
    import oracle
    from compressed_long_context_b200 import workloads as wl
    cfg = wl.DECODE_128K
    one = cfg.scaled(B=1)
    inp = wl.decode_inputs(one, "cpu")
    kb, vb = oracle.bf16_bits(inp["k"]), oracle.bf16_bits(inp["v"])
    wn, qb = inp["w"].numpy(), oracle.bf16_bits(inp["q"])
    kwb, vwb = oracle.bf16_bits(inp["kw"]), oracle.bf16_bits(inp["vw"])
    seq = inp["seqlens"].numpy()
    scale = 1.0 / np.sqrt(cfg.d)

    def step():
        kc, vc = oracle.compress(kb, vb, wn, cfg.blk)
        out = oracle.decode(qb, oracle.round_bf16(kc), oracle.round_bf16(vc), kwb, vwb, seq, cfg.blk, cfg.W,
                            scale)
        return out

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    qps = 1.0 / dt
    cores = oracle.num_threads()
    sample = ("oracle fp64 compress of one 131072-token sequence (K and V, d=512) + decode of its query "
              "(64 heads, 1023 entries + 128 window), per step")
    line = {"metric": METRIC, "value": qps, "unit": "queries/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "L": cfg.T, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                       "blk": cfg.blk, "W": cfg.W, "step": "oracle compress(raw K/V) + oracle decode",
                       "sample_sequences_per_step": 1},
            "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(target_s=10.0):
    """The oracle as it stands, on this host, for a bounded sample of the workload: batches of
    2 sequences (compress of their raw K/V + decode of their queries), repeated for about
    ``target_s`` seconds."""
    import oracle
    from compressed_long_context_b200 import workloads as wl
    cfg = wl.DECODE_128K
    n = 2
    inp = wl.decode_inputs(cfg.scaled(B=n), "cpu")
    kb, vb = oracle.bf16_bits(inp["k"]), oracle.bf16_bits(inp["v"])
    w = inp["w"].numpy()
    qb, kwb, vwb = oracle.bf16_bits(inp["q"]), oracle.bf16_bits(inp["kw"]), oracle.bf16_bits(inp["vw"])
    seq = inp["seqlens"].numpy()
    scale = 1.0 / np.sqrt(cfg.d)
    reps = 0
    t0 = time.perf_counter()
    while True:
        kc, vc = oracle.compress(kb, vb, w, cfg.blk)
        oracle.decode(qb, oracle.round_bf16(kc), oracle.round_bf16(vc), kwb, vwb, seq, cfg.blk, cfg.W, scale)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            break
    return {"value": n * reps / dt, "unit": "queries/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d passes over 2 sequences of the workload (oracle fp64 compress of 131072 raw tokens, K and "
                      "V, + decode of 64 heads over 1023 entries + 128 window tokens), %.1f s" % (reps, dt)}


# ---------------------------------------------------------------- our arm

def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    world, rank, local = dist_setup(args)
    sys.path.insert(0, ROOT)
    import compressed_long_context_b200 as hca
    from compressed_long_context_b200 import _lib, workloads as wl

    pk, pk_kind = peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = wl.DECODE_128K
    scale = 1.0 / np.sqrt(cfg.d)
    inp = wl.decode_inputs(cfg, dev)
    k, v, w, q, kw, vw, seq = (inp[x] for x in ("k", "v", "w", "q", "kw", "vw", "seqlens"))
    B, L = cfg.B, cfg.T
    Nc = L // cfg.blk
    kc = torch.empty((B, Nc, 1, cfg.d), dtype=torch.bfloat16, device=dev)
    vc = torch.empty((B, Nc, 1, cfg.dv), dtype=torch.bfloat16, device=dev)
    out = torch.empty((B, cfg.Hq, cfg.dv), dtype=torch.float32, device=dev)
    ws = torch.empty(hca.decode_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.dv), dtype=torch.uint8, device=dev)
    flush = l2_flush_buffer()
    stream = torch.cuda.current_stream()

    def step():
        hca.compress(k, v, w, cfg.blk, kc=kc, vc=vc)
        hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    hca.get_device_error()

    # ---- timed region: K steps, each bracketed by events; L2 flushed between steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        torch.cuda._sleep(int(2e8))
        for i in range(args.steps):
            flush.zero_()
            a, m, b = ev[i]
            a.record(stream)
            hca.compress(k, v, w, cfg.blk, kc=kc, vc=vc)
            m.record(stream)
            hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws)
            b.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, _, b in ev]
    comp_ms = [a.elapsed_time(m) for a, m, _ in ev]
    dec_in_step_ms = [m.elapsed_time(b) for _, m, b in ev]
    hca.get_device_error()
    t_step = max_over_ranks(sum(step_ms) / 1e3, world)
    ms_per_step = t_step * 1e3 / args.steps
    value = weak_scaling_value(B * args.steps, world, t_step)

    # compress roofline (dominant kernel of the step)
    cbytes = compress_bytes(B, L, 1, cfg.d, cfg.dv, cfg.blk)
    c_avg = sum(comp_ms) / len(comp_ms) / 1e3
    c_gbs = cbytes / c_avg / 1e9
    roof = {"bound": "hbm", "kernel": "compress_kernel<512,512>", "achieved": c_gbs, "peak": pk["hbm_gbs"],
            "unit": "GB/s", "frac": c_gbs / pk["hbm_gbs"],
            "traffic": traffic_for("compress_decode_B64_L131072",
                                   ["compressed_long_context_b200/csrc/compress.cuh"]),
            "algorithmic_bytes_per_launch": cbytes, "peak_kind": pk_kind + " (hbm_gbs)"}

    # ---- decode alone: cache resident, L2 flushed before each call.  A GPU-side spin is
    # queued first so that every timed call is already enqueued when the GPU reaches it:
    # the events then bracket device work only, not host launch overhead.
    dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    with sampler:
        torch.cuda._sleep(int(2e8))
        for i in range(args.steps):
            flush.zero_()
            a, b = dev_ev[i]
            a.record(stream)
            hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws)
            b.record(stream)
        torch.cuda.synchronize()
    d_ms = [a.elapsed_time(b) for a, b in dev_ev]
    d_avg = max_over_ranks(sum(d_ms) / len(d_ms) / 1e3, world)
    dbytes = decode_bytes(B, L, cfg.Hq, 1, cfg.d, cfg.dv, cfg.blk, cfg.W)
    d_gbs = dbytes / d_avg / 1e9
    decode_part = {"queries_per_s": world * B / d_avg, "us_per_call": d_avg * 1e6,
                   "roofline": {"bound": "hbm", "kernel": "decode_split_kernel + decode_combine_kernel",
                                "achieved": d_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                "frac": d_gbs / pk["hbm_gbs"], "algorithmic_bytes_per_call": dbytes,
                                "traffic": traffic_for("decode_B64_L131072",
                                                       ["compressed_long_context_b200/csrc/decode.cuh"])},
                   "median_us_per_call": statistics.median(d_ms) * 1e3,
                   "decode_in_step_us": statistics.median(dec_in_step_ms) * 1e3}

    # ---- one serving step: hca_append of every sequence's newest token (window ring write +
    # online pooling; at L = 131072 every sequence completes a block, so an entry is written
    # too), then hca_decode over the ring.  L2 flushed before each step.
    kn, vn = k[:, L - 1].contiguous(), v[:, L - 1].contiguous()
    wn = w[:, L - 1].contiguous()
    state = torch.zeros(hca.append_state_size(B, 1, cfg.d, cfg.dv), dtype=torch.uint8, device=dev)

    def serve(decode_too):
        hca.append(kn, vn, wn, seq, kw, vw, kc, vc, state, cfg.blk)
        if decode_too:
            hca.decode(q, kc, vc, kw, vw, seq, cfg.blk, cfg.W, scale, out=out, workspace=ws, window_ring=True)

    serve_part = {}
    for name, dec in (("append_us", False), ("append_plus_decode_us", True)):
        for _ in range(3):
            serve(dec)
        sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        with sampler:
            torch.cuda._sleep(int(2e8))
            for i in range(args.steps):
                flush.zero_()
                a, b = sev[i]
                a.record(stream)
                serve(dec)
                b.record(stream)
            torch.cuda.synchronize()
        serve_part[name] = max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in sev]) / 1e3,
                                          world) * 1e6
    hca.get_device_error()
    abytes = append_bytes(B, 1, cfg.d, cfg.dv)
    serve_part.update({"workload": "append + ring decode, %s" % cfg.name,
                       "append_algorithmic_bytes": abytes,
                       "append_frac_of_hbm": abytes / (serve_part["append_us"] / 1e6) / 1e9 / pk["hbm_gbs"],
                       "append_bound": "latency (one small CTA per sequence; %d KB moved)" % (abytes // 1024)})
    del state

    # ---- e2e through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        hk.copy_(k)
        hv.copy_(v)
        hw, hq, hkw, hvw, hs = (x.cpu().pin_memory() for x in (w, q, kw, vw, seq))
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dk, dvv = torch.empty_like(k), torch.empty_like(v)
        dw, dq, dkw, dvw, ds = (torch.empty_like(x) for x in (w, q, kw, vw, seq))
        h2d = sum(x.numel() * x.element_size() for x in (hk, hv, hw, hq, hkw, hvw, hs))
        d2h = hout.numel() * hout.element_size()
        del k, v
        torch.cuda.empty_cache()

        def e2e_step():
            for hsrc, ddst in ((hk, dk), (hv, dvv), (hw, dw), (hq, dq), (hkw, dkw), (hvw, dvw), (hs, ds)):
                ddst.copy_(hsrc, non_blocking=True)
            hca.compress(dk, dvv, dw, cfg.blk, kc=kc, vc=vc)
            hca.decode(dq, kc, vc, dkw, dvw, ds, cfg.blk, cfg.W, scale, out=out, workspace=ws)
            hout.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        ne = max(2, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(ne):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        te = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
        e2e = {"value": world * B * ne / te, "unit": "queries/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": ne}
        del hk, hv, dk, dvv
        torch.cuda.empty_cache()
    else:
        del k, v
        torch.cuda.empty_cache()

    # ---- prefill 128K (TFLOP/s)
    prefill_part = None
    if not args.no_prefill:
        pc = wl.PREFILL_128K
        pin = wl.prefill_inputs(pc, dev)
        pkc, pvc = hca.compress(pin["k"], pin["v"], pin["w"], pc.blk)
        pout = torch.empty((1, pc.T, pc.Hq, pc.dv), dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            hca.prefill(pin["q"], pin["k"], pin["v"], pkc, pvc, pc.blk, pc.W, 1.0 / np.sqrt(pc.d), out=pout)
        torch.cuda.synchronize()
        hca.get_device_error()
        np_steps = max(2, min(args.steps, 5))
        pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True)) for _ in range(np_steps)]
        with sampler:
            for i in range(np_steps):
                flush.zero_()
                a, m, b = pev[i]
                a.record(stream)
                hca.compress(pin["k"], pin["v"], pin["w"], pc.blk, kc=pkc, vc=pvc)
                m.record(stream)
                hca.prefill(pin["q"], pin["k"], pin["v"], pkc, pvc, pc.blk, pc.W, 1.0 / np.sqrt(pc.d), out=pout)
                b.record(stream)
            torch.cuda.synchronize()
        hca.get_device_error()
        p_ms = max_over_ranks(statistics.median([m.elapsed_time(b) for _, m, b in pev]), world)
        c3_ms = statistics.median([a.elapsed_time(m) for a, m, _ in pev])
        flops, keys = prefill_flops(1, pc.T, pc.Hq, pc.d, pc.dv, pc.blk, pc.W)
        tf = flops / (p_ms / 1e3) / 1e12
        peak_tf = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        prefill_part = {"workload": pc.name, "tflops": tf, "ms": p_ms, "compress_ms": c3_ms,
                        "algorithmic_flops": flops, "keys_per_head": keys,
                        "roofline": {"bound": "tensor", "kernel": "prefill_pair_kernel", "achieved": tf,
                                     "peak": peak_tf, "unit": "TFLOP/s", "frac": tf / peak_tf,
                                     "peak_kind": pk_kind + " (bf16_tflops_sustained)",
                                     "frac_of_burst": tf / pk["bf16_tflops"],
                                     "traffic": traffic_for("prefill_T131072",
                                                            ["compressed_long_context_b200/csrc/prefill.cuh",
                                                             "compressed_long_context_b200/csrc/prefill_pair.cuh"])}}
        # Virtual Head Attention on the prefill output (in place, bf16): one read and one write
        # of the 8.6 GB output, HBM-bound; synthetic rank-8 factors
        gv = torch.Generator(device=dev).manual_seed(5)
        vu = torch.randn((pc.Hq, 8), generator=gv, device=dev) * 0.1
        vv = torch.randn((pc.Hq, 8), generator=gv, device=dev) * 0.1
        hca.vha(pout, vu, vv)
        vev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(np_steps)]
        with sampler:
            for i in range(np_steps):
                a, b = vev[i]
                a.record(stream)
                hca.vha(pout, vu, vv)
                b.record(stream)
            torch.cuda.synchronize()
        hca.get_device_error()
        v_ms = max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in vev]), world)
        vbytes = vha_bytes(pout.numel(), pout.element_size(), pc.Hq, vu.shape[1])
        prefill_part["vha"] = {"ms": v_ms, "rank": 8, "algorithmic_bytes": vbytes, "bound": "hbm",
                               "achieved_gbs": vbytes / (v_ms / 1e3) / 1e9,
                               "frac": vbytes / (v_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                               "peak_kind": pk_kind + " (hbm_gbs)"}
        del pin, pkc, pvc, pout
        torch.cuda.empty_cache()

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_base = cpu_baseline_sample()

    clocks = sampler.summary()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded; no dataset)",
                "config": {"workload": cfg.name, "B": B, "L": L, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                           "blk": cfg.blk, "W": cfg.W, "step": "hca_compress(raw K/V) + hca_decode",
                           "l2": "flushed (2x L2 memset) before every timed step; raw K/V 17.2 GB > L2",
                           "parallelism": "dp%d (independent batches, no collective)" % world},
                "roofline": roof, "decode": decode_part, "serving_step": serve_part, "prefill": prefill_part,
                "cpu_baseline": cpu_base, "e2e": e2e,
                "gpu_launches": 3 * args.steps, "clocks": clocks,
                "libhca": os.path.relpath(_lib.LIB_PATH, ROOT)}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
