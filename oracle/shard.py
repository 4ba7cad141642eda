"""Plain CPU oracle of context-sharded decode: one sequence's chunks split over P shards.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may import this module.  It shares no code with the CUDA library.

Page: "LowRAM Compresses KV Cache Asymmetrically", section "Why Peak Throughput Can Improve
by 5x": decode throughput is bounded by moving the KV cache, including across GPUs.  The
pages describe no sharding protocol; this library's reading, written out literally here in
float64 (page names as in ``oracle/__init__.py``):

* Shard s holds the chunk ids [off_s, off_s + nC_s) of every unit (sequence, layer, KV head)
  as a compressed cache of its own, chunk ids local (global id = off_s + local id); only the
  shard with the newest tokens holds a non-empty raw tail.
* Step 1, per shard: score its chunks (``chunk_scores``) and take its own top k: candidates
  (score, global id).
* Step 2, on the union of all shards' candidates: the k best by (descending score, ascending
  global id), i.e. the unsharded selection (``select_top_k`` on all scores): a chunk among the
  k best overall has fewer than k better chunks anywhere, so fewer than k in its own shard,
  so it is among its shard's candidates.
* Step 3, per shard: attention of each query head over the selected chunks the shard holds
  plus its tail, kept unnormalised: m_j = the largest logit, l_j = sum_t exp(logit_t - m_j),
  y_j = sum_t exp(logit_t - m_j) v_t, with the rebuilt values of ``decode_unit``.
* Step 4: o_j = sum_s w_s y_{s,j} / sum_s w_s l_{s,j}, w_s = exp(m_{s,j} - max_s m_{s,j}):
  the softmax over the union of the shards' tokens, regrouped by shard ([OjaKV] section 3,
  the attention equations).

Parity pins: ``tests/test_shard_pins.py`` (sharded = unsharded ``oracle.decode`` to 1e-12 for
1 to 4 shards, int8 stores and ragged tails; the candidate lemma against brute force with
ties; planted mistakes that the pins catch).
"""

from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np

from . import OracleCache, chunk_scores, rebuild_keys, rebuild_values, select_top_k

__all__ = ["shard_candidates", "global_top_k", "shard_partial", "merge_partials", "decode_sharded"]


def shard_candidates(oc: OracleCache, b: int, l: int, hkv: int, q_heads: np.ndarray, offset: int):
    """Step 1: the shard's own top k as (scores, global ids), ids ascending."""
    grp = l // oc.G
    s = chunk_scores(q_heads, oc.summary[b, grp, hkv], oc.basis[l, hkv], oc.slot[b, grp, hkv])
    sel, _ = select_top_k(s, oc.k)
    return s[sel], sel + offset


def global_top_k(cand_scores: np.ndarray, cand_ids: np.ndarray, k: int) -> np.ndarray:
    """Step 2: the k best candidates by (descending score, ascending global id), ascending."""
    order = sorted(range(cand_ids.shape[0]), key=lambda i: (-cand_scores[i], int(cand_ids[i])))
    return np.array(sorted(int(cand_ids[i]) for i in order[:k]), dtype=np.int64)


def shard_partial(oc: OracleCache, b: int, l: int, hkv: int, q_heads: np.ndarray,
                  global_sel: Sequence[int], offset: int):
    """Step 3: (m [g], l [g], y [g][d]) of the shard's selected chunks plus its raw tail.

    m = -inf, l = 0, y = 0 for a head that sees no token in this shard."""
    grp = l // oc.G
    basis_l, w1, w2 = oc.basis[l, hkv], oc.w1[l, hkv], oc.w2[l, hkv]
    slot = oc.slot[b, grp, hkv]
    ptr = oc.res_ptr[b, l, hkv]
    keys, vals = [], []
    for c in global_sel:
        lc = int(c) - offset
        if not (0 <= lc < oc.nC):
            continue
        s = int(slot[lc])
        assert s >= 0, "selected an evicted chunk"
        rows = oc.coeff[b, grp, hkv, s * oc.C:(s + 1) * oc.C]
        sigma = (oc.coeff_scale[b, grp, hkv, s * oc.C:(s + 1) * oc.C]
                 if oc.coeff_scale is not None else np.ones(oc.C))
        khat = rebuild_keys(rows, sigma, basis_l)
        r0, r1 = int(ptr[s]), int(ptr[s + 1])
        rho = oc.res_scale[r0:r1] if oc.res_scale is not None else np.ones(r1 - r0)
        keys.append(khat)
        vals.append(rebuild_values(khat, w1, w2, oc.res_pos[r0:r1], oc.res_val[r0:r1], rho))
    tl = int(oc.tail_len[b])
    keys.append(oc.tail_k[b, l, hkv, :tl])
    vals.append(oc.tail_v[b, l, hkv, :tl])
    K, V = np.concatenate(keys), np.concatenate(vals)
    g, d = q_heads.shape
    if K.shape[0] == 0:
        return np.full(g, -np.inf), np.zeros(g), np.zeros((g, d))
    logits = q_heads @ K.T / math.sqrt(d)
    m = logits.max(axis=1)
    p = np.exp(logits - m[:, None])
    return m, p.sum(axis=1), p @ V


def merge_partials(ms: List[np.ndarray], ls: List[np.ndarray], ys: List[np.ndarray]) -> np.ndarray:
    """Step 4: o_j = sum_s w_s y_s / sum_s w_s l_s with w_s = exp(m_s - max_s m_s)."""
    M = np.max(np.stack(ms), axis=0)
    num = np.zeros_like(ys[0])
    den = np.zeros_like(ls[0])
    for m, l, y in zip(ms, ls, ys):
        w = np.where(np.isfinite(m), np.exp(m - M), 0.0)
        num += w[:, None] * y
        den += w * l
    return num / den[:, None]


def decode_sharded(shards: List[OracleCache], offsets: List[int], q: np.ndarray, layer0: int = 0,
                   n_layers=None, units=None) -> dict:
    """Steps 1-4 for every unit of layers [layer0, layer0 + n_layers): out [n_layers][B][Hq][d],
    sel [n_layers][B][Hkv][k] (global ids), and per shard the candidates and partials."""
    q = np.asarray(q, dtype=np.float64)
    oc0 = shards[0]
    if n_layers is None:
        n_layers = q.shape[0]
    k, g = oc0.k, oc0.g
    out = np.full((n_layers, oc0.B, oc0.Hq, oc0.d), np.nan)
    sel = np.full((n_layers, oc0.B, oc0.Hkv, k), -1, dtype=np.int64)
    if units is None:
        units = [(li, b, h) for li in range(n_layers) for b in range(oc0.B) for h in range(oc0.Hkv)]
    for (li, b, h) in units:
        l = layer0 + li
        qh = q[li, b, h * g:(h + 1) * g]
        cands = [shard_candidates(oc, b, l, h, qh, off) for oc, off in zip(shards, offsets)]
        gs = global_top_k(np.concatenate([c[0] for c in cands]), np.concatenate([c[1] for c in cands]), k)
        parts = [shard_partial(oc, b, l, h, qh, gs, off) for oc, off in zip(shards, offsets)]
        out[li, b, h * g:(h + 1) * g] = merge_partials([p[0] for p in parts], [p[1] for p in parts],
                                                       [p[2] for p in parts])
        sel[li, b, h] = gs
    return {"out": out, "sel": sel}
