"""Pins of the reuse model (``oracle.reuse``), CPU only.

* Bookkeeping against sequences worked out by hand: hits decided before the call's fills,
  admission of the misses in unit order up to the fill cap, first-in first-out eviction.
* Its invariants on random sequences (table and owners agree, counts add up).
* The stored values are ``rebuild_values`` of the chunk: attending over them reproduces the
  decode of the whole cache (a decode whose selected chunks are all hits).
* The temporal query recipe: consecutive selections overlap when the targets persist, and
  barely when every step is independent.
"""

import numpy as np

import lowram_synth as S
import oracle as O
from oracle.reuse import ReuseModel, stored_values


def test_bookkeeping_worked_example():
    m = ReuseModel(capacity=3, fill_cap=2)
    u0, u1 = (0, 0, 0), (1, 0, 0)
    h, mi, f = m.call([(u0, [5, 2]), (u1, [7])])
    assert h == [] and mi == [(0, 0, 0, 2), (0, 0, 0, 5), (1, 0, 0, 7)]
    assert f == [(0, 0, 0, 2), (0, 0, 0, 5)]                # unit order, ids ascending, cap 2
    assert m.table == {(0, 0, 0, 2): 0, (0, 0, 0, 5): 1}
    h, mi, f = m.call([(u0, [2, 5]), (u1, [7, 8])])
    assert h == [(0, 0, 0, 2), (0, 0, 0, 5)] and f == [(1, 0, 0, 7), (1, 0, 0, 8)]
    # entry 2 then entry 0 (the oldest): chunk 2 of unit 0 is evicted by chunk 8 of unit 1
    assert m.table == {(0, 0, 0, 5): 1, (1, 0, 0, 7): 2, (1, 0, 0, 8): 0}
    h, mi, f = m.call([(u0, [2])])
    assert h == [] and f == [(0, 0, 0, 2)] and m.table[(0, 0, 0, 2)] == 1   # evicts chunk 5
    assert (m.hits, m.misses, m.fills) == (2, 6, 5)
    m.check()


def test_bookkeeping_invariants_random():
    rng = np.random.default_rng(3)
    for _ in range(50):
        E = int(rng.integers(1, 12))
        m = ReuseModel(E, int(rng.integers(0, E + 1)))
        for _ in range(20):
            sel = [((b, 0, 0), rng.choice(16, size=3, replace=False).tolist()) for b in range(3)]
            before = dict(m.table)
            h, mi, f = m.call(sel)
            assert len(h) + len(mi) == 9 and len(f) == min(len(mi), m.fill_cap)
            assert all(k in before for k in h) and not any(k in before for k in mi)
            m.check()


def test_stored_values_reproduce_the_decode():
    """A unit's output from its selected chunks' stored values (and the tail) equals decode."""
    cfg = S.MISTRAL_GROUP.replace(name="reuse_pin", batch=1, n_ctx=1024, top_k=4)
    cache = S.make_cache(cfg, tail_len=[23])
    q = S.make_queries(cache).double().numpy()
    oc = O.OracleCache(S.cache_to_numpy(cache))
    ref = O.decode(oc, q)
    g = oc.g
    for (l, h) in [(0, 0), (1, 5)]:
        keys, vals = [], []
        for c in ref["sel"][l, 0, h]:
            s = int(oc.slot[0, 0, h, c])
            rows = oc.coeff[0, 0, h, s * oc.C:(s + 1) * oc.C]
            keys.append(O.rebuild_keys(rows, np.ones(oc.C), oc.basis[l, h]))
            vals.append(stored_values(oc, 0, l, h, int(c)))
        keys.append(oc.tail_k[0, l, h, :23])
        vals.append(oc.tail_v[0, l, h, :23])
        out = O.attend(q[l, 0, h * g:(h + 1) * g], np.concatenate(keys), np.concatenate(vals))
        assert np.abs(out - ref["out"][l, 0, h * g:(h + 1) * g]).max() <= 1e-12 * np.abs(out).max()


def _overlap(cfg, rho, drift):
    cache = S.make_cache(cfg)
    oc = O.OracleCache(S.cache_to_numpy(cache))
    steps = S.make_query_steps(cache, 4, rho=rho, drift=drift)
    sels = [O.decode(oc, s.double().numpy())["sel"] for s in steps]
    same = [np.mean([len(set(a.tolist()) & set(b.tolist())) / cfg.top_k
                     for a, b in zip(x.reshape(-1, cfg.top_k), y.reshape(-1, cfg.top_k))])
            for x, y in zip(sels[:-1], sels[1:])]
    return float(np.mean(same))


def test_query_steps_control_the_overlap():
    cfg = S.MISTRAL_GROUP.replace(name="reuse_q", batch=1, n_kv_heads=2, n_q_heads=8, n_ctx=2048, top_k=8)
    sticky = _overlap(cfg, rho=0.95, drift=0.0)
    fresh = _overlap(cfg, rho=0.0, drift=1.0)
    assert sticky > 0.6 and fresh < sticky - 0.3
