"""The context-sharded decode protocol across two processes on CPU (gloo, world size 2).

Each rank holds one shard of the same cache and runs ``sharded.decode_step``, the protocol the
GPU path runs, with its gathers over the process group.  The local steps here are the fp64
oracle's (``oracle.shard``), since the CUDA kernels need a GPU; the test checks the exchange:
every rank must end with the unsharded oracle's output and selection.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import lowram_synth as S
import oracle as O
import oracle.shard as SH
from kv_cache_compression_lowram_b200.sharded import all_gather, decode_step

CFG = S.MISTRAL_GROUP.replace(name="gloo_shard", batch=2, n_ctx=1024, top_k=4, tail_cap=64)
BOUNDS = [0, 9, 16]


class OracleShard:
    """The three local steps of one shard, computed by the oracle, as torch tensors."""

    def __init__(self, oc, offset):
        self.oc, self.offset = oc, offset

    def candidates(self, q, layer0):
        oc = self.oc
        n, g = q.shape[0], oc.g
        cs = torch.zeros(n, oc.B, oc.Hkv, oc.k, dtype=torch.float64)
        ci = torch.zeros(n, oc.B, oc.Hkv, oc.k, dtype=torch.int64)
        for li in range(n):
            for b in range(oc.B):
                for h in range(oc.Hkv):
                    s, i = SH.shard_candidates(oc, b, layer0 + li, h, q[li, b, h * g:(h + 1) * g].numpy(), self.offset)
                    cs[li, b, h] = torch.from_numpy(s)
                    ci[li, b, h] = torch.from_numpy(i)
        self.q = q
        return cs, ci

    def partial(self, cs_all, ci_all, layer0):
        oc, q = self.oc, self.q
        n, g, d = q.shape[0], oc.g, oc.d
        part = torch.zeros(n, oc.B, oc.Hq, d + 2, dtype=torch.float64)
        sel = torch.zeros(n, oc.B, oc.Hkv, oc.k, dtype=torch.int64)
        for li in range(n):
            for b in range(oc.B):
                for h in range(oc.Hkv):
                    gs = SH.global_top_k(cs_all[:, li, b, h].reshape(-1).numpy(), ci_all[:, li, b, h].reshape(-1).numpy(),
                                         oc.k)
                    m, l, y = SH.shard_partial(oc, b, layer0 + li, h, q[li, b, h * g:(h + 1) * g].numpy(), gs,
                                               self.offset)
                    part[li, b, h * g:(h + 1) * g, 0] = torch.from_numpy(m)
                    part[li, b, h * g:(h + 1) * g, 1] = torch.from_numpy(l)
                    part[li, b, h * g:(h + 1) * g, 2:] = torch.from_numpy(y)
                    sel[li, b, h] = torch.from_numpy(gs)
        return part, sel

    def merge(self, parts_all):
        P, n, B, Hq, w = parts_all.shape
        out = torch.zeros(n, B, Hq, w - 2, dtype=torch.float64)
        for li in range(n):
            for b in range(B):
                p = parts_all[:, li, b].numpy()          # [P][Hq][w]
                out[li, b] = torch.from_numpy(SH.merge_partials(list(p[:, :, 0]), list(p[:, :, 1]), list(p[:, :, 2:])))
        return out


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
        cache = S.make_cache(CFG, tail_len=[64, 31])
        q = S.make_queries(cache).double()
        lo, hi = BOUNDS[rank], BOUNDS[rank + 1]
        shard = S.shard_chunks(cache, lo, hi, keep_tail=(rank == ws - 1))
        local = OracleShard(O.OracleCache(S.cache_to_numpy(shard)), lo)
        got, sel = decode_step(local, q, all_gather())
        out[rank] = (got.numpy(), sel.numpy())
    finally:
        dist.destroy_process_group()


def test_sharded_protocol_two_ranks_gloo():
    ws = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(ws, port, out), nprocs=ws, join=True, start_method="spawn")
    cache = S.make_cache(CFG, tail_len=[64, 31])
    ref = O.decode(O.OracleCache(S.cache_to_numpy(cache)), S.make_queries(cache).double().numpy())
    for rank in range(ws):
        got, sel = out[rank]
        assert np.array_equal(sel, ref["sel"])
        err = np.abs(got - ref["out"]).max(axis=-1) / np.abs(ref["out"]).max(axis=-1)
        assert err.max() <= 1e-12


def test_shard_decoder_checks_the_gathered_shard_count():
    """Phase 2 is refused on the host when the gather returned another number of shards than
    the decoder was built for (no library call is made)."""
    from types import SimpleNamespace

    from kv_cache_compression_lowram_b200.sharded import ShardDecoder

    cfg = dict(batch=1, n_kv_heads=2, n_q_heads=8, head_dim=128, top_k=4, dtype="bf16")
    dec = ShardDecoder(SimpleNamespace(cfg=cfg, handle=None), 0, 2)
    dec._n = 1
    cs = torch.zeros(3, 1, 1, 2, 4)
    with pytest.raises(ValueError):
        dec.partial(cs, torch.zeros(3, 1, 1, 2, 4, dtype=torch.int32))
    with pytest.raises(ValueError):
        dec.partial(cs[:2], torch.zeros(2, 1, 1, 2, 3, dtype=torch.int32))
