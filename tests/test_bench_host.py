"""Host-side logic of bench.py on CPU: algorithmic work counts and the multi-rank timing
reduction over a world-size-2 gloo group (no GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_decode_bytes_128k():
    # q 64 KB + (1023 entries + 128 window) x 2 KB + out 128 KB (+ 4 B length) per query
    per = 64 * 512 * 2 + (1023 + 128) * 1 * 1024 * 2 + 64 * 512 * 4 + 4
    assert bench.decode_bytes(64, 131072, 64, 1, 512, 512, 128, 128) == 64 * per
    assert abs(64 * per - 163.4e6) < 0.1e6


def test_compress_bytes_128k():
    b = bench.compress_bytes(64, 131072, 1, 512, 512, 128)
    assert b == 64 * 1024 * (128 * 1024 * 2 + 2048) + 64 * 131072 * 4
    assert abs(b - 17.35e9) < 0.01e9


def test_prefill_flops_128k():
    flops, keys = bench.prefill_flops(1, 131072, 64, 512, 512, 128, 128)
    brute = 0
    for t in range(131072):
        a = t - 128 + 1
        brute += (a // 128 if a > 0 else 0) + min(128, t + 1)
    assert keys == brute == 83682495
    assert flops == 2.0 * 64 * keys * 1024


def test_append_bytes_block_completing_step():
    # per (sequence, KV head): the new token (2 KB), the pooling state read and written
    # (2 x 4,112 B), the ring slot (2 KB) and the entry (2 KB); plus length and weight
    per = 2048 + 2 * (4 + 1024) * 4 + 2048 + 2048
    assert bench.append_bytes(64, 1, 512, 512) == 64 * per + 64 * 8 == 920064


def test_vha_bytes_prefill_output():
    # the 128K prefill output, bf16, read and written once; rank-8 factors
    n = 131072 * 64 * 512
    assert bench.vha_bytes(n, 2, 64, 8) == 2 * n * 2 + 2 * 64 * 8 * 4
    assert abs(bench.vha_bytes(n, 2, 64, 8) - 17.18e9) < 0.01e9


def test_weak_scaling_value():
    assert bench.weak_scaling_value(64 * 10, 4, 2.0) == 64 * 10 * 4 / 2.0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + rank, world, device="cpu")
        bench.barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


def test_decode_seq_bytes_gate_and_short():
    # the gate logits add Hq * dv bf16 per query; a sequence shorter than the window has no entries
    base = bench.decode_seq_bytes(131072, 64, 1, 512, 512, 128, 128)
    assert bench.decode_seq_bytes(131072, 64, 1, 512, 512, 128, 128, gate=True) == base + 64 * 512 * 2
    assert bench.decode_seq_bytes(100, 64, 1, 512, 512, 128, 128) == 64 * 1024 + 100 * 2048 + 64 * 2048 + 4


def test_err_stats_and_within():
    ref = np.array([[0.0, 1.0], [2.0, -1.0]])
    got = torch.tensor([[0.0, 1.002], [2.0, -1.0]])
    s = bench.err_stats(got, ref)
    assert abs(s["max_abs_err"] - 0.002) < 1e-6 and s["outputs_compared"] == 4 and s["finite"]
    assert bench.within(s)                       # max 2e-3 <= 1e-2, mean 5e-4 <= 1e-3
    assert not bench.within(bench.err_stats(torch.tensor([[0.0, 1.02], [2.0, -1.0]]), ref))


def test_parse_config_subset():
    a = bench.parse(["--configs", "decode_128k,ragged_paged", "--steps", "5"])
    assert a.steps == 5 and a.configs == "decode_128k,ragged_paged" and a.impl == "ours"
