"""Reuse of rebuilt chunks across decode steps, on the GPU, against the oracle's model.

Each case runs a few consecutive decode steps (``make_query_steps``: queries whose selections
persist from step to step, at a chosen drift) through a reuse store and checks, step by step:

* the selection equals the plain decode's exactly, and the output matches the plain decode
  (tight: the stored values differ from rebuilt ones by one bf16 rounding) and the fp64 oracle
  (the parity rules of ``parity_utils``);
* the hit / miss / fill counts and the whole table (which entry holds which chunk) equal
  ``oracle.reuse.ReuseModel`` fed the same selections;
* the values in filled entries match ``oracle.reuse.stored_values``.
"""

import numpy as np
import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
from oracle.reuse import ReuseModel, stored_values
from parity_utils import check, sample_units

pytestmark = pytest.mark.gpu
DEV = "cuda"

BASE = S.LLAMA_32K.replace(name="reuse_llama", batch=2, n_layers=4, n_ctx=8192, top_k=8)
# (config, steps, rho, drift, capacity, fill_cap)
CASES = [
    (BASE, 4, 0.9, 0.1, 4096, 4096),                                       # no evictions, high reuse
    (BASE, 4, 0.0, 1.0, 4096, 4096),                                       # independent steps
    (BASE, 5, 0.9, 0.2, 48, 40),                                           # small store: evictions, capped fills
    (BASE.replace(name="reuse_r64", rank=64), 3, 0.9, 0.1, 4096, 64),
    (BASE.replace(name="reuse_g8", n_kv_heads=2, n_q_heads=16), 3, 0.9, 0.1, 4096, 4096),
    (BASE.replace(name="reuse_evict", evict_frac=0.25), 4, 0.9, 0.2, 100, 100),
    (BASE, 3, 0.9, 0.1, 4096, 0),                                          # never fills: all misses
]
TIGHT = 5e-3   # max |o_reuse - o_plain| per output vector, relative to its 2-norm


def _unit_selections(sel: np.ndarray, layer0: int = 0):
    """Selections in the store's unit order ((layer, KV head, sequence), sequence fastest)."""
    n_layers, B, H, _ = sel.shape
    return [((b, layer0 + li, h), sel[li, b, h].tolist()) for li in range(n_layers) for h in range(H)
            for b in range(B)]


def _expected_table(model: ReuseModel, oc, shape):
    B, L, H, stride = shape
    table = np.full(shape, -1, dtype=np.int64)
    owner = np.full(model.E, -1, dtype=np.int64)
    for (b, l, h, c), e in model.table.items():
        s = int(oc.slot[b, l // oc.G, h, c])
        table[b, l, h, s] = e
        owner[e] = ((b * L + l) * H + h) * stride + s
    return table, owner


def _check_entries(store, model: ReuseModel, oc, n_sample: int, seed: int):
    v = store.view()
    entries = v["entries"].float().cpu().numpy()
    held = sorted(model.table.items(), key=lambda kv: kv[1])
    rng = np.random.default_rng(seed)
    pick = rng.choice(len(held), size=min(n_sample, len(held)), replace=False) if held else []
    for i in pick:
        (b, l, h, c), e = held[int(i)]
        ref = stored_values(oc, b, l, h, c)
        err = np.abs(entries[e] - ref).max()
        assert err <= 1e-2 * np.abs(ref).max(), ((b, l, h, c), e, err)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}_r{c[2]}_d{c[3]}_E{c[4]}_f{c[5]}")
def test_reuse_steps_match_plain_decode_model_and_oracle(case):
    cfg, n_steps, rho, drift, cap, fill_cap = case
    cache = S.make_cache(cfg, device=DEV)
    steps = S.make_query_steps(cache, n_steps, rho, drift)
    oc = O.OracleCache(S.cache_to_numpy(cache))
    lc = K.LowramCache.from_synth(cache)
    store = K.LowramReuse(lc, cap, fill_cap)
    model = ReuseModel(cap, fill_cap)
    try:
        for t, q in enumerate(steps):
            out, sel = store.decode(q, sel=True)
            ref, ref_sel = lc.decode(q, sel=True)
            torch.cuda.synchronize()
            assert lc.validate() == 0
            assert torch.equal(sel, ref_sel), t
            err = ((out.float() - ref.float()).norm(dim=-1) / ref.float().norm(dim=-1)).max().item()
            assert err <= TIGHT, (t, err)
            check(cfg, oc, q, out, sel, units=sample_units(cfg, cfg.n_layers, 24, seed=t))
            hits, misses, fills = model.call(_unit_selections(sel.cpu().numpy()))
            got = store.counts()
            assert got == {"hits": model.hits, "misses": model.misses, "fills": model.fills}, (t, got)
            v = store.view()
            exp_table, exp_owner = _expected_table(model, oc, tuple(v["table"].shape))
            assert np.array_equal(v["table"].cpu().numpy(), exp_table), t
            assert np.array_equal(v["owner"].cpu().numpy(), exp_owner), t
        model.check()
        if drift < 1.0 and fill_cap > 0:
            assert model.hits > 0
        _check_entries(store, model, oc, 12, seed=n_steps)
    finally:
        store.close()
        lc.close()


def test_repeated_query_is_all_hits():
    """The same query twice: the second call's chunks all come from the store (no tile for the
    chunk-attention kernel) and its output is the first call's up to the stored rounding."""
    cfg = BASE
    cache = S.make_cache(cfg, device=DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    store = K.LowramReuse(lc, 4096, 4096)
    try:
        o1, s1 = store.decode(q, sel=True)
        o2, s2 = store.decode(q, sel=True)
        torch.cuda.synchronize()
        assert torch.equal(s1, s2)
        n = cfg.n_layers * cfg.batch * cfg.n_kv_heads * cfg.top_k
        assert store.counts() == {"hits": n, "misses": n, "fills": n}
        err = ((o2.float() - o1.float()).norm(dim=-1) / o1.float().norm(dim=-1)).max().item()
        assert err <= TIGHT
        check(cfg, O.OracleCache(S.cache_to_numpy(cache)), q, o2, s2)
        assert lc.validate() == 0
    finally:
        store.close()
        lc.close()


def test_layer_window_and_bench_sized_store():
    """A window of layers of the 32K workload (B = 4, 256 chunks) through a store, sampled."""
    cfg = S.LLAMA_32K
    cache = S.make_cache(cfg, device=DEV)
    steps = S.make_query_steps(cache, 2, 0.9, 0.1, layer0=8, n_layers=8)
    lc = K.LowramCache.from_synth(cache)
    store = K.LowramReuse(lc, 2048, 1024)
    model = ReuseModel(2048, 1024)
    oc = O.OracleCache(S.cache_to_numpy(cache))
    try:
        for t, q in enumerate(steps):
            out, sel = store.decode(q, sel=True, layer0=8)
            ref, ref_sel = lc.decode(q, sel=True, layer0=8)
            torch.cuda.synchronize()
            assert torch.equal(sel, ref_sel)
            err = ((out.float() - ref.float()).norm(dim=-1) / ref.float().norm(dim=-1)).max().item()
            assert err <= TIGHT, (t, err)
            check(cfg, oc, q, out, sel, layer0=8, units=sample_units(cfg, 8, 16, seed=t))
            model.call(_unit_selections(sel.cpu().numpy(), layer0=8))
            assert store.counts() == {"hits": model.hits, "misses": model.misses, "fills": model.fills}
    finally:
        store.close()
        lc.close()


def test_store_refuses_after_repack_and_unsupported_shapes():
    cfg = BASE.replace(name="reuse_repack", tail_cap=128)
    cache = S.make_cache(cfg, device=DEV, tail_len=[128, 128])
    lc = K.LowramCache.from_synth(cache)
    store = K.LowramReuse(lc, 64, 64)
    q = S.make_queries(cache)
    store.decode(q)
    lc.repack(16)
    with pytest.raises(K.LowramError) as ei:
        store.decode(q)
    assert ei.value.status == 1
    store.close()
    fresh = K.LowramReuse(lc, 64, 64)     # a new store serves the re-packed cache
    out, sel = fresh.decode(q, sel=True)
    ref, ref_sel = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    assert torch.equal(sel, ref_sel)
    fresh.close()
    lc.close()
    other = K.LowramCache.from_synth(S.make_cache(S.MISTRAL_GROUP, device=DEV))   # chunk 64
    with pytest.raises(K.LowramError) as ei:
        K.LowramReuse(other, 16, 16)
    assert ei.value.status == 4
    for cap, fill in ((16, 17), (0, 0), ((1 << 30) + 1, 1), (16, -1)):
        with pytest.raises(K.LowramError) as ei:
            K.LowramReuse(other, cap, fill)
        assert ei.value.status == 1, (cap, fill)
    other.close()
