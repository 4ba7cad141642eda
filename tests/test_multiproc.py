"""Multi-process logic of the benchmark on CPU (gloo, world size 2).

The decode path has no exchange step: every rank runs its own replica and only the timing
is reduced (max over ranks) together with the query counts (sum).
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import lowram_synth as S


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        ms = [40.0, 55.0][rank]
        value, ms_max = bench.aggregate_rate(128.0 * 10, ms, ws)
        cfg = bench.replica_config(S.TINY_F32, rank)
        cache = S.make_cache(cfg)
        out[rank] = (value, ms_max, cfg.seed, float(cache.coeff.double().sum()))
    finally:
        dist.destroy_process_group()


def test_replicas_and_max_over_ranks_gloo():
    ws = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(ws, port, out), nprocs=ws, join=True, start_method="spawn")
    v0, ms0, seed0, c0 = out[0]
    v1, ms1, seed1, c1 = out[1]
    assert ms0 == ms1 == 55.0                       # the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 1280 / 0.055)
    assert seed0 != seed1 and c0 != c1              # independent replicas


def test_single_rank_aggregate_is_local():
    value, ms = bench.aggregate_rate(1280.0, 40.0, 1)
    assert ms == 40.0 and value == pytest.approx(1280 / 0.04)
