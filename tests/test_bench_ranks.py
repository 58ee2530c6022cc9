"""The benchmark's whole-job reduction over ranks (max of the timings, sum of the
byte counts), run as two gloo processes on the CPU, and its helpers."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [1.0 + rank, 10.0 - 3.0 * rank]
        counts = [100.0 * (rank + 1), 7.0]
        t, c = bench.reduce_over_ranks(times, counts, torch.device("cpu"), world)
        out[rank] = (t, c)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world_2():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        t, c = res[rank]
        assert t == [2.0, 10.0]            # max over ranks of each timing
        assert c == [300.0, 14.0]          # sum over ranks of each count


def test_reduce_over_ranks_single_process():
    assert bench.reduce_over_ranks([1.5], [2.0], torch.device("cpu"), 1) == ([1.5], [2.0])


def test_kv_bytes_counts_int4_and_int8_positions():
    # D = 128: 136 B per INT4 token-head, 264 B per INT8 token-head; protected = min(L, S + W)
    L = np.array([10, 200])
    got = bench.kv_bytes(L, Hkv=8, D=128, S=4, W=128)
    prot = np.minimum(L, 132)
    assert got == int(np.sum(8 * ((L - prot) * 136 + prot * 264)))
    assert bench.kv_bytes(L, 8, 128, 4, 128, int4_only=True) == int(np.sum(8 * L * 136))
    assert bench.bf16_bytes(L, 8, 128) == int(np.sum(L * 8 * 512))
