"""Pins of the context-sharded decode oracle (``oracle.shard``), CPU only.

* Sharded = unsharded: for 1 to 4 shards with uneven chunk boundaries, bf16 and int8
  stores and ragged tails, the merged outputs equal ``oracle.decode`` on the whole cache to
  1e-12 and the global selection equals the unsharded one exactly.
* The candidate lemma by brute force: on random integer scores with many ties, the k best of
  the union of every shard's own top k are the k best overall (ties to the lower id).
* Ties across a shard boundary are resolved toward the lower global id.
* Planted mistakes (unweighted merge, local ids taken as global, the tail counted in every
  shard, only the top k/P of each shard exchanged) each break the equality.
"""

import numpy as np
import pytest

import lowram_synth as S
import oracle as O
import oracle.shard as SH

BF16 = S.MISTRAL_GROUP.replace(name="shard_bf16", batch=2, n_ctx=1024, top_k=4, tail_cap=64)
INT8 = S.LLAMA_64K_INT8.replace(name="shard_int8", batch=1, n_layers=4, n_kv_heads=2, n_q_heads=8,
                                n_ctx=2048, top_k=4, evict_frac=0.0)
SPLITS = {1: [0, 16], 2: [0, 7, 16], 3: [0, 5, 11, 16], 4: [0, 4, 8, 12, 16]}


def _shards(cache, bounds):
    out = []
    for s, (lo, hi) in enumerate(zip(bounds[:-1], bounds[1:])):
        sh = S.shard_chunks(cache, lo, hi, keep_tail=(s == len(bounds) - 2))
        out.append(O.OracleCache(S.cache_to_numpy(sh)))
    return out


def _cache(cfg, tail_len):
    cache = S.make_cache(cfg, tail_len=tail_len)
    return cache, S.make_queries(cache).double().numpy()


@pytest.mark.parametrize("n_shards", [1, 2, 3, 4])
@pytest.mark.parametrize("cfg,tail_len", [(BF16, [64, 23]), (INT8, [77])], ids=["bf16", "int8"])
def test_sharded_decode_equals_unsharded(cfg, tail_len, n_shards):
    cache, q = _cache(cfg, tail_len)
    full = O.decode(O.OracleCache(S.cache_to_numpy(cache)), q)
    bounds = SPLITS[n_shards]
    res = SH.decode_sharded(_shards(cache, bounds), bounds[:-1], q)
    assert np.array_equal(res["sel"], full["sel"])
    err = np.abs(res["out"] - full["out"]).max(axis=-1) / np.abs(full["out"]).max(axis=-1)
    assert err.max() <= 1e-12


def test_candidate_lemma_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(400):
        n = int(rng.integers(6, 40))
        k = int(rng.integers(1, 5))
        scores = rng.integers(0, 6, size=n).astype(np.float64)   # many exact ties
        scores[rng.random(n) < 0.15] = -np.inf                   # evicted chunks
        if np.isfinite(scores).sum() < 3 * k:
            continue
        want, _ = O.select_top_k(scores, k)
        cuts = np.sort(rng.choice(np.arange(1, n), size=2, replace=False))
        bounds = [0, int(cuts[0]), int(cuts[1]), n]
        cs, ci = [], []
        for lo, hi in zip(bounds[:-1], bounds[1:]):
            part = scores[lo:hi]
            kk = min(k, int(np.isfinite(part).sum()))
            if kk == 0:
                continue
            sel, _ = O.select_top_k(part, kk)
            cs.append(part[sel])
            ci.append(sel + lo)
        got = SH.global_top_k(np.concatenate(cs), np.concatenate(ci), k)
        assert np.array_equal(got, want), (scores, bounds, k)


def test_ties_across_the_shard_boundary_go_to_the_lower_id():
    cache, q = _cache(BF16, [64, 64])
    # chunks 3 (shard 0) and 12 (shard 1) get the same summary: equal scores everywhere
    cache.summary[:, :, :, 12] = cache.summary[:, :, :, 3]
    oc = O.OracleCache(S.cache_to_numpy(cache))
    bounds = [0, 8, 16]
    shards = _shards(cache, bounds)
    b, l, h, g = 0, 1, 2, BF16.q_per_kv
    qh = q[l, b, h * g:(h + 1) * g]
    s = O.chunk_scores(qh, oc.summary[b, 0, h], oc.basis[l, h], oc.slot[b, 0, h])
    assert s[3] == s[12]
    # force the tie onto the selection boundary: the query prefers exactly the k-1 chunks
    # above both and then the tied pair
    order = sorted(range(16), key=lambda c: (-s[c], c))
    res = SH.decode_sharded(shards, bounds[:-1], q)
    want = O.decode(oc, q)
    assert np.array_equal(res["sel"], want["sel"])
    if order.index(3) == BF16.top_k - 1 or order.index(12) == BF16.top_k - 1:
        assert 3 in res["sel"][l, b, h]


def _planted(kind, shards, offsets, q, k):
    """decode_sharded with one planted mistake (for the pins' power)."""
    oc0 = shards[0]
    g = oc0.g
    out = np.zeros((q.shape[0], oc0.B, oc0.Hq, oc0.d))
    for li in range(q.shape[0]):
        for b in range(oc0.B):
            for h in range(oc0.Hkv):
                qh = q[li, b, h * g:(h + 1) * g]
                cands = []
                for oc, off in zip(shards, offsets):
                    cs, ci = SH.shard_candidates(oc, b, li, h, qh, off)
                    if kind == "local_ids":
                        ci = ci - off
                    if kind == "top_k_over_p":
                        keep = np.argsort(-cs, kind="stable")[:max(1, k // len(shards))]
                        cs, ci = cs[keep], ci[keep]
                    cands.append((cs, ci))
                gs = SH.global_top_k(np.concatenate([c[0] for c in cands]), np.concatenate([c[1] for c in cands]), k)
                parts = [SH.shard_partial(oc, b, li, h, qh, gs, off) for oc, off in zip(shards, offsets)]
                ms, ls, ys = [p[0] for p in parts], [p[1] for p in parts], [p[2] for p in parts]
                if kind == "unweighted":
                    o = sum(ys) / sum(ls)[:, None]
                else:
                    o = SH.merge_partials(ms, ls, ys)
                out[li, b, h * g:(h + 1) * g] = o
    return out


@pytest.mark.parametrize("kind", ["unweighted", "local_ids", "tail_everywhere", "top_k_over_p"])
def test_planted_mistakes_fail(kind):
    cfg = BF16.replace(top_k=8)
    cache, q = _cache(cfg, [64, 40])
    full = O.decode(O.OracleCache(S.cache_to_numpy(cache)), q)["out"]
    bounds = SPLITS[2]
    if kind == "tail_everywhere":
        shards = [O.OracleCache(S.cache_to_numpy(S.shard_chunks(cache, lo, hi, keep_tail=True)))
                  for lo, hi in zip(bounds[:-1], bounds[1:])]
        got = SH.decode_sharded(shards, bounds[:-1], q)["out"]
    else:
        got = _planted(kind, _shards(cache, bounds), bounds[:-1], q, cfg.top_k)
    err = np.abs(got - full).max(axis=-1) / np.abs(full).max(axis=-1)
    assert err.max() > 1e-6
