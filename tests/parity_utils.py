"""Comparison of the CUDA path with the fp64 oracle (used by the GPU tests).

Rules (tolerances written here, per output vector o of one (layer, sequence, query head)):
* fp32 caches: max_i |o_gpu_i - o_ref_i| <= 1e-4 * max_i |o_ref_i|;
* bf16 caches: max_i |o_gpu_i - o_ref_i| <= 2e-2 * ||o_ref||_2;
* chunk selection: where the oracle's margin between its k-th and (k+1)-th best score is
  above 1e-3, the GPU must select exactly the oracle's chunks; everywhere the GPU's chunks
  must be a valid top-k of the oracle's scores up to the score tolerance below, and the
  output is compared with the oracle run on the GPU's selection.
* chunk scores: |s_gpu - s_ref| <= 1e-4 * (1 + |s_ref|) (fp32 accumulation of exact inputs).
"""

from __future__ import annotations

import math

import numpy as np
import torch

import lowram_synth as S
import oracle as O

MARGIN = 1e-3
SCORE_TOL = 1e-4


def out_tol(cfg) -> float:
    return 1e-4 if cfg.dtype == "f32" else 2e-2


def q_to_f64(q: torch.Tensor) -> np.ndarray:
    return q.detach().cpu().double().numpy()


def sample_units(cfg, n_layers: int, n: int, seed: int = 0):
    all_units = [(li, b, h) for li in range(n_layers) for b in range(cfg.batch)
                 for h in range(cfg.n_kv_heads)]
    if len(all_units) <= n:
        return all_units
    rng = np.random.default_rng(seed)
    idx = set(rng.choice(len(all_units), size=n - 2, replace=False).tolist())
    idx |= {0, len(all_units) - 1}
    return [all_units[i] for i in sorted(idx)]


def check(cfg, oc: O.OracleCache, q: torch.Tensor, out: torch.Tensor, sel: torch.Tensor,
          layer0: int = 0, units=None, scores: torch.Tensor = None) -> dict:
    """Compare one decode call; raises AssertionError with a description on a mismatch."""
    n_layers = q.shape[0]
    qf = q_to_f64(q)
    sel_np = sel.detach().cpu().numpy().astype(np.int64)
    out_np = out.detach().cpu().double().numpy()
    if units is None:
        units = [(li, b, h) for li in range(n_layers) for b in range(cfg.batch)
                 for h in range(cfg.n_kv_heads)]
    ref = O.decode(oc, qf, layer0, n_layers, forced_sel=sel_np, units=units)
    tol = out_tol(cfg)
    g = cfg.q_per_kv
    worst = 0.0
    n_strict = 0
    for (li, b, h) in units:
        l = layer0 + li
        grp = l // cfg.group
        qh = qf[li, b, h * g:(h + 1) * g]
        s = O.chunk_scores(qh, oc.summary[b, grp, h], oc.basis[l, h], oc.slot[b, grp, h])
        own, margin = O.select_top_k(s, cfg.top_k)
        gs = sel_np[li, b, h]
        assert len(set(gs.tolist())) == cfg.top_k and list(gs) == sorted(gs), (li, b, h, gs)
        assert all(np.isfinite(s[c]) for c in gs), f"evicted chunk selected at {(li, b, h)}"
        kth = np.sort(s[np.isfinite(s)])[::-1][cfg.top_k - 1]
        assert min(s[c] for c in gs) >= kth - SCORE_TOL * (1 + abs(kth)), (li, b, h)
        if margin > MARGIN:
            n_strict += 1
            assert list(gs) == list(own), f"selection differs at {(li, b, h)}: {gs} vs {own}"
        if scores is not None:
            gsc = scores[li, b, h].detach().cpu().double().numpy()
            fin = np.isfinite(s)
            assert np.array_equal(np.isfinite(gsc), fin)
            err = np.abs(gsc[fin] - s[fin]) / (1 + np.abs(s[fin]))
            assert err.max() <= SCORE_TOL, (li, b, h, err.max())
        for j in range(h * g, (h + 1) * g):
            o_ref = ref["out"][li, b, j]
            o_gpu = out_np[li, b, j]
            denom = np.abs(o_ref).max() if cfg.dtype == "f32" else np.linalg.norm(o_ref)
            e = float(np.abs(o_gpu - o_ref).max() / denom)
            worst = max(worst, e)
            assert e <= tol, f"output mismatch at {(li, b, j)}: {e:.3e} > {tol}"
    return {"worst": worst, "units": len(units), "strict_selection_units": n_strict}
