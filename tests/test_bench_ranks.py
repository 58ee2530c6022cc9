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


def test_side_bytes_match_the_copies_of_the_end_to_end_leg():
    # the e2e leg copies per layer 2 * B*Hkv*D + B*Hq*D bf16 elements in and B*Hq*D out
    w = {"Hq": 32, "Hkv": 8, "D": 128, "P": 16, "S": 4, "W": 128}
    L = np.array([1, 16, 17, 5000])
    B, layers = len(L), 3
    sb = bench.side_bytes(L, w, layers)
    assert sb["q_read"] + sb["new_kv_read"] == layers * (2 * B * 8 * 128 + B * 32 * 128) * 2
    assert sb["out_written"] == layers * B * 32 * 128 * 2
    assert sb["new_kv_written"] == layers * B * 8 * (136 + 264)          # INT4 page and INT8 store
    assert sb["block_table_read"] == layers * (1 + 1 + 2 + 313) * 2 * 4  # pages x 2 groups of 4 heads x int32
    assert sb["total"] == sum(v for k, v in sb.items() if k not in ("total", "kv_stream"))
    assert sb["kv_stream"] == layers * bench.kv_bytes(L, 8, 128, 4, 128)


@pytest.mark.parametrize("Hkv,groups", [(8, 2), (6, 3), (2, 1), (3, 3), (1, 1)])
def test_side_bytes_count_table_reads_per_head_group(Hkv, groups):
    w = {"Hq": Hkv, "Hkv": Hkv, "D": 64, "P": 64, "S": 4, "W": 32}
    assert bench.side_bytes(np.array([64, 65]), w, 1)["block_table_read"] == (1 + 2) * groups * 4
