"""Context-sharded decode: one sequence's chunks split by chunk id over several shards.

Each shard is an ordinary cache over a contiguous chunk range (usually one shard per GPU);
the step's four parts are the library's entry points (``lowram.h``, "context-sharded decode"):
the shard's own top k (phase 1), the gather of every shard's candidates, the shard's part of
the global top k as unnormalised partials (phase 2), the gather of the partials and their
merge.  The gathers are torch.distributed all-gathers into local buffers (NCCL over NVLink /
NVSwitch between GPUs): no kernel reads another GPU's memory.

``decode_step`` is the protocol itself, written once over its three local operations and a
gather; ``ShardDecoder`` binds the operations to the CUDA library for one shard.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch

from . import (LowramCache, lowram_merge_partials, lowram_shard_candidates, lowram_shard_partial, _get)


def decode_step(local, q, gather: Callable[[torch.Tensor], torch.Tensor], layer0: int = 0):
    """One decode step of the sharded protocol on this shard.

    local: the shard's operations -- ``candidates(q, layer0) -> (scores, ids)``,
    ``partial(scores_all, ids_all, layer0) -> (partial, sel)`` and ``merge(partials_all) -> out``;
    gather(t): every shard's t stacked in shard order (ascending chunk offset) on this shard.
    Returns (out, sel): this step's attention output and the global selection."""
    cs, ci = local.candidates(q, layer0)
    part, sel = local.partial(gather(cs), gather(ci), layer0)
    return local.merge(gather(part)), sel


def all_gather(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """A gather over a torch.distributed process group (all ranks, rank order)."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        ws = dist.get_world_size(group)
        parts = [torch.empty_like(t) for _ in range(ws)]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)

    return gather


class ShardDecoder:
    """The local operations of one shard: a cache over chunk ids [chunk_offset, ...) of every
    unit, one of n_shards."""

    def __init__(self, cache: LowramCache, chunk_offset: int, n_shards: int):
        self.cache = cache
        self.offset = int(chunk_offset)
        self.n_shards = int(n_shards)
        c = cache.cfg
        self.B, self.Hkv, self.Hq = _get(c, "batch"), _get(c, "n_kv_heads"), _get(c, "n_q_heads")
        self.d, self.k = _get(c, "head_dim"), _get(c, "top_k")
        self.dtype = torch.float32 if _get(c, "dtype") in (0, "f32") else torch.bfloat16

    def candidates(self, q, layer0: int = 0):
        n = int(q.shape[0])
        cs = torch.empty(n, self.B, self.Hkv, self.k, dtype=torch.float32, device=q.device)
        ci = torch.empty(n, self.B, self.Hkv, self.k, dtype=torch.int32, device=q.device)
        lowram_shard_candidates(self.cache.handle, layer0, n, q, self.offset, cs, ci)
        self._n = n
        return cs, ci

    def partial(self, cs_all, ci_all, layer0: int = 0):
        if int(cs_all.shape[0]) != self.n_shards or tuple(ci_all.shape) != tuple(cs_all.shape):
            raise ValueError(f"expected the candidates of {self.n_shards} shards, got {tuple(cs_all.shape)} "
                             f"scores and {tuple(ci_all.shape)} ids")
        n = self._n
        part = torch.empty(n, self.B, self.Hq, self.d + 2, dtype=torch.float32, device=cs_all.device)
        sel = torch.empty(n, self.B, self.Hkv, self.k, dtype=torch.int32, device=cs_all.device)
        lowram_shard_partial(self.cache.handle, layer0, n, self.offset, int(cs_all.shape[0]), cs_all, ci_all,
                             part, sel)
        return part, sel

    def merge(self, parts_all):
        P, n, B, Hq, w = parts_all.shape
        out = torch.empty(n, B, Hq, w - 2, dtype=self.dtype, device=parts_all.device)
        lowram_merge_partials(parts_all.view(P, n * B * Hq, w), out)
        return out

    def decode(self, q, layer0: int = 0, gather: Optional[Callable] = None):
        """One step with every other shard running the same call (gather: a process-group
        all-gather by default)."""
        return decode_step(self, q, gather or all_gather(), layer0)
