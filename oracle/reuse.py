"""Plain CPU model of reusing rebuilt chunks across decode steps.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may import this module.  It shares no code with the CUDA library.

Page: rit.work "lowram-kv-cache-compression", section "Значения предсказывают, ключи
раскладывают по общему базису": each step picks the fragments that fit the query and reuses
data it has already reconstructed.  The pages give no store, size or policy; this library's
reading (names as in ``oracle/__init__.py``):

* The store keeps, per (sequence, layer, KV head, chunk), the chunk's rebuilt values
  vhat_t = f(khat_t) + rho_t delta_t ([Asym] "Core Mechanism"), the part of a chunk whose
  rebuild costs the predictor; its keys are scored from the stored coefficients as usual.
* E entries, filled first-in first-out: the n-th chunk ever admitted takes entry n mod E and
  evicts whatever that entry held.  Admission, per decode call: the call's misses in unit
  order ((layer, KV head, sequence), sequence fastest), each unit's in ascending chunk id, at
  most ``fill_cap`` of them.  Hits are decided against the store as it was before the call.
* Reuse changes no result: a hit attends over the stored values, which are the values a miss
  rebuilds, so the output is ``oracle.decode``'s.

Parity pins: ``tests/test_reuse_pins.py`` (the bookkeeping against scripted sequences worked
out by hand, its invariants on random sequences, and the stored values against
``rebuild_values``).
"""

from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

from . import OracleCache, rebuild_keys, rebuild_values

__all__ = ["ReuseModel", "stored_values"]

Key = Tuple[int, int, int, int]   # (b, l, hkv, chunk id)


class ReuseModel:
    """The store's bookkeeping: which chunks it holds, where, and each call's hits and fills."""

    def __init__(self, capacity: int, fill_cap: int):
        assert capacity >= 1 and 0 <= fill_cap <= capacity
        self.E = capacity
        self.fill_cap = fill_cap
        self.table: Dict[Key, int] = {}
        self.owner: List = [None] * capacity
        self.ring = 0          # entries ever filled (the next entry is ring % E)
        self.hits = self.misses = self.fills = 0

    def call(self, selections: Sequence[Tuple[Tuple[int, int, int], Sequence[int]]]):
        """One decode call.  selections: ((b, l, hkv), chunk ids) per unit, in unit order.
        Returns (hits, misses, fills) as lists of keys."""
        hits, misses = [], []
        for (b, l, h), ids in selections:
            for c in sorted(int(x) for x in ids):
                (hits if (b, l, h, c) in self.table else misses).append((b, l, h, c))
        fills = misses[:self.fill_cap]
        for key in fills:
            e = self.ring % self.E
            self.ring += 1
            old = self.owner[e]
            if old is not None:
                del self.table[old]
            self.owner[e] = key
            self.table[key] = e
        self.hits += len(hits)
        self.misses += len(misses)
        self.fills += len(fills)
        return hits, misses, fills

    def check(self):
        """The table and the owners describe the same map, one entry per chunk."""
        for e, key in enumerate(self.owner):
            if key is not None:
                assert self.table[key] == e
        assert len(self.table) == sum(k is not None for k in self.owner)


def stored_values(oc: OracleCache, b: int, l: int, hkv: int, chunk: int) -> np.ndarray:
    """The values a store entry holds for a chunk: vhat_t = f(khat_t) + rho_t delta_t, [C][d]."""
    grp = l // oc.G
    s = int(oc.slot[b, grp, hkv, chunk])
    assert s >= 0
    rows = oc.coeff[b, grp, hkv, s * oc.C:(s + 1) * oc.C]
    sigma = oc.coeff_scale[b, grp, hkv, s * oc.C:(s + 1) * oc.C] if oc.coeff_scale is not None else np.ones(oc.C)
    khat = rebuild_keys(rows, sigma, oc.basis[l, hkv])
    ptr = oc.res_ptr[b, l, hkv]
    r0, r1 = int(ptr[s]), int(ptr[s + 1])
    rho = oc.res_scale[r0:r1] if oc.res_scale is not None else np.ones(r1 - r0)
    return rebuild_values(khat, oc.w1[l, hkv], oc.w2[l, hkv], oc.res_pos[r0:r1], oc.res_val[r0:r1], rho)
