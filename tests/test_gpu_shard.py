"""Context-sharded decode on one GPU: P virtual shards of one cache (each an ordinary cache over
a chunk range, only the last with the raw tail), the protocol's gathers done by stacking the
shards' tensors.  Checked against the unsharded GPU decode (the global selection must equal its
selection exactly) and against the fp64 oracle on the whole cache (the parity rules of
``parity_utils``).  The multi-GPU path runs the same kernels with NCCL all-gathers between
them; it is covered on CPU by ``test_multiproc_shard.py``.
"""

import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
from kv_cache_compression_lowram_b200.sharded import ShardDecoder
from parity_utils import check, sample_units

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_shards(cache, bounds, q):
    decs = []
    for s, (lo, hi) in enumerate(zip(bounds[:-1], bounds[1:])):
        sh = S.shard_chunks(cache, lo, hi, keep_tail=(s == len(bounds) - 2))
        decs.append(ShardDecoder(K.LowramCache.from_synth(sh), lo, len(bounds) - 1))
    cands = [d.candidates(q) for d in decs]
    cs_all = torch.stack([c[0] for c in cands])
    ci_all = torch.stack([c[1] for c in cands])
    parts = [d.partial(cs_all, ci_all) for d in decs]
    out = decs[0].merge(torch.stack([p[0] for p in parts]))
    torch.cuda.synchronize()
    for d in decs:
        assert d.cache.validate() == 0
        d.cache.close()
    sels = [p[1] for p in parts]
    for s in sels[1:]:
        assert torch.equal(s, sels[0])
    return out, sels[0], ci_all


CASES = [
    # (config, shard boundaries in chunks, tail lengths)
    (S.LLAMA_32K.replace(name="shard_llama", batch=2, n_layers=4, n_ctx=8192, top_k=8), [0, 20, 41, 64], [128, 77]),
    (S.LLAMA_32K.replace(name="shard_llama1", batch=2, n_layers=4, n_ctx=8192, top_k=8), [0, 64], [5, 128]),
    (S.MISTRAL_GROUP.replace(name="shard_mistral", batch=2), [0, 16, 32, 48, 64], [64, 0]),
    (S.LLAMA_64K_INT8.replace(name="shard_int8", batch=2, n_layers=4, n_kv_heads=2, n_q_heads=8, n_ctx=8192,
                              top_k=8, evict_frac=0.0), [0, 33, 64], [128, 3]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}_p{len(c[1]) - 1}")
def test_virtual_shards_match_unsharded_and_oracle(case):
    cfg, bounds, tail_len = case
    cache = S.make_cache(cfg, device=DEV, tail_len=tail_len)
    q = S.make_queries(cache)
    out, sel, ci_all = _run_shards(cache, bounds, q)
    # every shard exported its own top k with global ids inside its range
    for s, (lo, hi) in enumerate(zip(bounds[:-1], bounds[1:])):
        assert bool(((ci_all[s] >= lo) & (ci_all[s] < hi)).all())
    lc = K.LowramCache.from_synth(cache)
    ref, ref_sel = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    lc.close()
    assert torch.equal(sel, ref_sel)
    check(cfg, O.OracleCache(S.cache_to_numpy(cache)), q, out, sel)


def test_two_shards_of_the_32k_workload_sampled():
    """The bench workload (B=4, 32 layers, 256 chunks) split into two shards of 128 chunks."""
    cfg = S.LLAMA_32K
    cache = S.make_cache(cfg, device=DEV)
    q = S.make_queries(cache)
    out, sel, _ = _run_shards(cache, [0, 128, 256], q)
    lc = K.LowramCache.from_synth(cache)
    ref, ref_sel = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    lc.close()
    assert torch.equal(sel, ref_sel)
    check(cfg, O.OracleCache(S.cache_to_numpy(cache)), q, out, sel, units=sample_units(cfg, cfg.n_layers, 64, seed=7))


def test_shards_reused_across_steps():
    """The same shard decoders over consecutive steps with different queries: every step must
    match the unsharded decode (a shard's tile list is shorter than the grid here, so this
    also checks that no stale piece record of an earlier step is merged)."""
    cfg = S.MISTRAL_GROUP.replace(name="shard_steps", batch=2)
    cache = S.make_cache(cfg, device=DEV, tail_len=[64, 9])
    bounds = [0, 16, 32, 48, 64]
    decs = []
    for s, (lo, hi) in enumerate(zip(bounds[:-1], bounds[1:])):
        sh = S.shard_chunks(cache, lo, hi, keep_tail=(s == len(bounds) - 2))
        decs.append(ShardDecoder(K.LowramCache.from_synth(sh), lo, len(bounds) - 1))
    lc = K.LowramCache.from_synth(cache)
    for t, q in enumerate(S.make_query_steps(cache, 3, 0.0, 1.0)):
        cands = [d.candidates(q) for d in decs]
        cs_all = torch.stack([c[0] for c in cands])
        ci_all = torch.stack([c[1] for c in cands])
        parts = [d.partial(cs_all, ci_all) for d in decs]
        out = decs[0].merge(torch.stack([p[0] for p in parts]))
        ref, ref_sel = lc.decode(q, sel=True)
        torch.cuda.synchronize()
        assert torch.equal(parts[0][1], ref_sel), t
        err = ((out.float() - ref.float()).norm(dim=-1) / ref.float().norm(dim=-1)).max().item()
        assert err <= 1e-2, (t, err)
    for d in decs:
        d.cache.close()
    lc.close()


def test_phase_two_requires_phase_one():
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg).to(DEV)
    lc = K.LowramCache.from_synth(cache)
    d = ShardDecoder(lc, 0, 1)
    q = S.make_queries(cache)
    cs, ci = d.candidates(q)
    lc.decode(q)                          # overwrites the scratch phase 1 prepared
    with pytest.raises(K.LowramError) as ei:
        d.partial(cs[None], ci[None])
    assert ei.value.status == 1
    lc.close()
