"""Plain, slow fp64 CPU oracle of LowRAM decode-time attention over a compressed KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this package.  It shares no code with
the CUDA library and does not import it.

Every function cites the passage it follows.  Page names used below:

* [OjaKV] "OjaKV: 上下文感知的在线低秩KV缓存压缩" (zh translation of arXiv 2509.21623),
  section 3 "预备知识：低秩注意力" (the attention equations) and 3.1 (orthonormal bases).
* [Asym] "LowRAM Compresses KV Cache Asymmetrically for Up to 5x Faster Decoding",
  sections "Core Mechanism: Predict Values and Keep Difficult Residuals" (M_KV formula,
  Vhat = f(K), delta = V - Vhat) and "Cross-Layer Low-Rank Key Compression".
* [Abstract] "LowRAM: Low-Rank Keys and Amortised Values for Composable KV Cache
  Compression at Test-Time" (arXiv 2611.07025): per-head predictor, residuals for the worst
  tokens, cross-layer low-rank keys, reconstruction of a selected subset per step,
  composition with quantisation and eviction.
* [Rit] rit.work "lowram-kv-cache-compression", section "Значения предсказывают, ключи
  раскладывают по общему базису": xKV keys with a common basis for adjacent layers; the
  context split into fragments, the ones that fit the current query chosen; tokens
  generated after prefill kept uncompressed.

Readings where the pages are silent (each a reading this library takes, not a page's rule):
the chunk summary is the mean of the chunk's coefficient rows, so the chunk's mean key at
layer l is abar_c . B_l, and a chunk's score is sum_j q_j . kbar_c / sqrt(d); selection is
per (b, l, KV head) and ties go to the lower chunk id; the predictor is
W2 . silu(W1 . k) without biases; the int8 scale multiplies the whole row.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` except the
chunk score's definition itself (the pages give none), which is "parity unpinned" against
the pages; it is pinned only against brute force over its own definition.
"""

from __future__ import annotations

import itertools
import math
from typing import Optional

import numpy as np

__all__ = [
    "dense_kv_bytes", "silu", "predict_values", "chunk_scores", "select_top_k",
    "rebuild_keys", "rebuild_values", "attend", "OracleCache", "decode", "decode_unit",
    "decode_unit_rewritten", "compressed_bytes",
]


# ------------------------------------------------------------------ stored value decoding

def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f64(arr: Optional[np.ndarray], is_bf16: bool) -> Optional[np.ndarray]:
    if arr is None:
        return None
    if is_bf16:
        return _bf16_bits_to_f64(arr)
    return arr.astype(np.float64)


# ----------------------------------------------------------------------------- formulas

def dense_kv_bytes(n_layers: int, n_kv_heads: int, head_dim: int, n_ctx: int,
                   bytes_per_scalar: int, batch: int) -> int:
    """Dense KV-cache bytes M_KV * B with M_KV = 2 * L * H_kv * d_h * N * s.

    [Asym] "Core Mechanism", the M_KV formula (per sequence); times the batch.
    """
    return 2 * n_layers * n_kv_heads * head_dim * n_ctx * bytes_per_scalar * batch


def silu(x: np.ndarray) -> np.ndarray:
    """silu(x) = x * sigmoid(x) = x / (1 + exp(-x)), the predictor's activation."""
    return x / (1.0 + np.exp(-x))


def predict_values(w1: np.ndarray, w2: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Per-head value predictor Vhat = f(K) = W2 . silu(W1 . k) for each key row.

    [Asym] "Core Mechanism" (Vhat = f(K)); [Abstract] (lightweight per-head predictor).
    keys [n][d], w1 [h][d], w2 [d][h] -> [n][d].
    """
    hidden = silu(keys @ w1.T)
    return hidden @ w2.T


def rebuild_keys(coeff_rows: np.ndarray, sigma: np.ndarray, basis_l: np.ndarray) -> np.ndarray:
    """Key rebuild from the cross-layer low-rank form: khat_t = sigma_t * (a_t . B_l).

    [Asym] "Cross-Layer Low-Rank Key Compression"; [Rit] (xKV, common basis of adjacent
    layers).  coeff_rows [n][r], sigma [n] (int8 row scale, or ones), basis_l [r][d].
    """
    return sigma[:, None] * (coeff_rows @ basis_l)


def rebuild_values(keys: np.ndarray, w1: np.ndarray, w2: np.ndarray,
                   res_pos: np.ndarray, res_val: np.ndarray, res_scale: np.ndarray) -> np.ndarray:
    """Vhat_t = f(khat_t), plus rho_i * delta_i for every stored residual record i.

    [Asym] "Core Mechanism": delta = V - Vhat is kept only for the selected (worst) tokens,
    so Vhat + delta restores V on those tokens.  res_pos are token offsets inside ``keys``.
    """
    vals = predict_values(w1, w2, keys)
    for i in range(res_pos.shape[0]):
        vals[int(res_pos[i])] += res_scale[i] * res_val[i]
    return vals


def attend(q_heads: np.ndarray, keys: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Scaled dot-product attention o_j = softmax(q_j K^T / sqrt(d)) V, one row per head.

    [OjaKV] section 3, A = softmax(Q K^T / sqrt(d_h)), O = A V.  The maximum is subtracted
    before exponentiation, which leaves the softmax unchanged.
    """
    d = q_heads.shape[-1]
    logits = q_heads @ keys.T / math.sqrt(d)               # [g][n]
    logits = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    return (p @ values) / p.sum(axis=1, keepdims=True)


def chunk_scores(q_heads: np.ndarray, summary: np.ndarray, basis_l: np.ndarray,
                 slot: np.ndarray) -> np.ndarray:
    """s_c = sum_j q_j . kbar_c / sqrt(d), kbar_c = abar_c . B_l; -inf for evicted chunks.

    Reading of [Rit] (fragments chosen by the current query) and [Abstract] (a selected
    subset is reconstructed): the chunk is represented by its mean rebuilt key.
    q_heads [g][d], summary [nL][r] (abar per live slot), slot [nC].
    """
    d = q_heads.shape[-1]
    qsum = q_heads.sum(axis=0)
    s = np.full(slot.shape[0], -np.inf)
    for c in range(slot.shape[0]):
        if slot[c] >= 0:
            kbar = summary[int(slot[c])] @ basis_l
            s[c] = float(qsum @ kbar) / math.sqrt(d)
    return s


def select_top_k(scores: np.ndarray, k: int):
    """The k chunks with the highest score (ties to the lower id), returned ascending.

    Also returns the margin s_(k) - s_(k+1) between the k-th and (k+1)-th best live scores
    (+inf when every live chunk is selected).
    """
    live = [c for c in range(scores.shape[0]) if np.isfinite(scores[c])]
    order = sorted(live, key=lambda c: (-scores[c], c))
    chosen = sorted(order[:k])
    margin = (scores[order[k - 1]] - scores[order[k]]) if len(order) > k else math.inf
    return np.array(chosen, dtype=np.int64), float(margin)


# ------------------------------------------------------------------------------- cache

class OracleCache:
    """Stored arrays of a compressed cache as exact float64 values (plus index tables).

    ``npc`` is the dict ``lowram_synth.cache_to_numpy`` returns (or the same layout built
    by hand): bf16 arrays as uint16 bit patterns, fp16 scales as float16.
    """

    def __init__(self, npc: dict):
        c = npc["cfg"]
        self.B, self.L, self.G = c["batch"], c["n_layers"], c["group"]
        self.Hkv, self.Hq, self.d = c["n_kv_heads"], c["n_q_heads"], c["head_dim"]
        self.r, self.h, self.N, self.C = c["rank"], c["mlp_hidden"], c["n_ctx"], c["chunk"]
        self.k, self.T = c["top_k"], c["tail_cap"]
        self.g = self.Hq // self.Hkv
        self.nC = self.N // self.C
        self.int8 = c["store"] == "int8"
        bf = lambda n: npc.get(n + "_is_bf16", False)
        self.coeff = _f64(npc["coeff"], bf("coeff"))
        self.coeff_scale = (npc["coeff_scale"].astype(np.float64)
                            if npc.get("coeff_scale") is not None else None)
        self.basis = _f64(npc["basis"], bf("basis"))
        self.w1 = _f64(npc["w1"], bf("w1"))
        self.w2 = _f64(npc["w2"], bf("w2"))
        self.summary = _f64(npc["summary"], bf("summary"))
        self.slot = npc["slot"].astype(np.int64)
        self.res_ptr = npc["res_ptr"].astype(np.int64)
        self.res_pos = npc["res_pos"].astype(np.int64)
        self.res_val = _f64(npc["res_val"], bf("res_val"))
        self.res_scale = (npc["res_scale"].astype(np.float64)
                          if npc.get("res_scale") is not None else None)
        self.tail_k = _f64(npc["tail_k"], bf("tail_k"))
        self.tail_v = _f64(npc["tail_v"], bf("tail_v"))
        self.tail_len = npc["tail_len"].astype(np.int64)


def _q_f64(q) -> np.ndarray:
    if isinstance(q, tuple):        # (bits, is_bf16)
        return _f64(q[0], q[1])
    return np.asarray(q, dtype=np.float64)


def decode_unit(oc: OracleCache, b: int, l: int, hkv: int, q_heads: np.ndarray,
                forced_sel: Optional[np.ndarray] = None) -> dict:
    """Decode-time attention of one unit (sequence b, layer l, KV head hkv), literal form.

    Steps in the order of [Rit] (chunks chosen by the query, selected chunks rebuilt, raw
    tail attended) with the rebuild of [Asym] / [Abstract] and attention of [OjaKV]:
      1. score every live chunk; 2. take the top k (or ``forced_sel``);
      3. rebuild khat for every token of the selected chunks;
      4. rebuild vhat = f(khat) and add the stored residuals;
      5. attend over those tokens plus the raw tail.
    """
    grp = l // oc.G
    basis_l, w1, w2 = oc.basis[l, hkv], oc.w1[l, hkv], oc.w2[l, hkv]
    slot = oc.slot[b, grp, hkv]
    scores = chunk_scores(q_heads, oc.summary[b, grp, hkv], basis_l, slot)
    if forced_sel is None:
        sel, margin = select_top_k(scores, oc.k)
    else:
        sel, margin = np.sort(np.asarray(forced_sel, dtype=np.int64)), math.nan

    keys, vals = [], []
    ptr = oc.res_ptr[b, l, hkv]
    for c in sel:
        s = int(slot[c])
        assert s >= 0, "selected an evicted chunk"
        rows = oc.coeff[b, grp, hkv, s * oc.C:(s + 1) * oc.C]
        sigma = (oc.coeff_scale[b, grp, hkv, s * oc.C:(s + 1) * oc.C]
                 if oc.coeff_scale is not None else np.ones(oc.C))
        khat = rebuild_keys(rows, sigma, basis_l)
        r0, r1 = int(ptr[s]), int(ptr[s + 1])
        rho = oc.res_scale[r0:r1] if oc.res_scale is not None else np.ones(r1 - r0)
        vhat = rebuild_values(khat, w1, w2, oc.res_pos[r0:r1], oc.res_val[r0:r1], rho)
        keys.append(khat)
        vals.append(vhat)
    tl = int(oc.tail_len[b])
    keys.append(oc.tail_k[b, l, hkv, :tl])
    vals.append(oc.tail_v[b, l, hkv, :tl])
    out = attend(q_heads, np.concatenate(keys), np.concatenate(vals))
    return {"out": out, "sel": sel, "scores": scores, "margin": margin}


def decode(oc: OracleCache, q, layer0: int = 0, n_layers: Optional[int] = None,
           forced_sel: Optional[np.ndarray] = None, units=None) -> dict:
    """Decode every unit of layers [layer0, layer0 + n_layers).

    q: [n_layers][B][Hq][d] float array, or (bf16 bits, True).  forced_sel, if given, is
    [n_layers][B][Hkv][k].  ``units`` restricts the work to a list of (li, b, hkv); the
    other outputs stay NaN.  Returns out [n_layers][B][Hq][d], sel, scores, margin.
    """
    qf = _q_f64(q)
    if n_layers is None:
        n_layers = qf.shape[0]
    out = np.full((n_layers, oc.B, oc.Hq, oc.d), np.nan)
    sel = np.full((n_layers, oc.B, oc.Hkv, oc.k), -1, dtype=np.int64)
    scores = np.full((n_layers, oc.B, oc.Hkv, oc.nC), np.nan)
    margin = np.full((n_layers, oc.B, oc.Hkv), np.nan)
    if units is None:
        units = [(li, b, h) for li in range(n_layers) for b in range(oc.B) for h in range(oc.Hkv)]
    for (li, b, h) in units:
        j0 = h * oc.g
        fs = None if forced_sel is None else forced_sel[li, b, h]
        res = decode_unit(oc, b, layer0 + li, h, qf[li, b, j0:j0 + oc.g], fs)
        out[li, b, j0:j0 + oc.g] = res["out"]
        sel[li, b, h] = res["sel"]
        scores[li, b, h] = res["scores"]
        margin[li, b, h] = res["margin"]
    return {"out": out, "sel": sel, "scores": scores, "margin": margin}


def decode_unit_rewritten(oc: OracleCache, b: int, l: int, hkv: int, q_heads: np.ndarray,
                          forced_sel: Optional[np.ndarray] = None) -> dict:
    """The same result through three exact rewrites (checked against ``decode_unit``):

    R3  q . khat_t = sigma_t * (B_l q) . a_t (scores in the coefficient space; [OjaKV] 3.1
        projects queries into the key basis) and s_c = (B_l sum_j q_j) . abar_c / sqrt(d);
    R2  W1 . khat_t = sigma_t * (W1 B_l^T) a_t (predictor folded onto the coefficients);
    R1  sum_t p_t (W2 silu_t + delta_t) = W2 (sum_t p_t silu_t) + sum_t p_t delta_t
        (the second predictor layer applied once, after the softmax-weighted sum).
    """
    grp = l // oc.G
    d = oc.d
    basis_l, w1, w2 = oc.basis[l, hkv], oc.w1[l, hkv], oc.w2[l, hkv]
    slot = oc.slot[b, grp, hkv]
    qt = q_heads @ basis_l.T                       # [g][r]  (R3)
    w1f = w1 @ basis_l.T                           # [h][r]  (R2)
    s = np.full(slot.shape[0], -np.inf)
    qt_sum = qt.sum(axis=0)
    for c in range(slot.shape[0]):
        if slot[c] >= 0:
            s[c] = float(qt_sum @ oc.summary[b, grp, hkv, int(slot[c])]) / math.sqrt(d)
    if forced_sel is None:
        sel, _ = select_top_k(s, oc.k)
    else:
        sel = np.sort(np.asarray(forced_sel, dtype=np.int64))
    logits, hid, dl = [], [], []
    ptr = oc.res_ptr[b, l, hkv]
    for c in sel:
        si = int(slot[c])
        rows = oc.coeff[b, grp, hkv, si * oc.C:(si + 1) * oc.C]
        sigma = (oc.coeff_scale[b, grp, hkv, si * oc.C:(si + 1) * oc.C]
                 if oc.coeff_scale is not None else np.ones(oc.C))
        logits.append(sigma[None, :] * (qt @ rows.T) / math.sqrt(d))      # [g][C]
        hid.append(silu(sigma[:, None] * (rows @ w1f.T)))                  # [C][h]
        dd = np.zeros((oc.C, d))
        r0, r1 = int(ptr[si]), int(ptr[si + 1])
        for i in range(r0, r1):
            rho = oc.res_scale[i] if oc.res_scale is not None else 1.0
            dd[int(oc.res_pos[i])] += rho * oc.res_val[i]
        dl.append(dd)
    tl = int(oc.tail_len[b])
    tk, tv = oc.tail_k[b, l, hkv, :tl], oc.tail_v[b, l, hkv, :tl]
    lg = np.concatenate(logits + [q_heads @ tk.T / math.sqrt(d)], axis=1)
    m = lg.max(axis=1, keepdims=True)
    p = np.exp(lg - m)
    n_sel = len(sel) * oc.C
    H = np.concatenate(hid) if hid else np.zeros((0, oc.h))
    D = np.concatenate(dl + [tv]) if dl else tv
    acc_h = p[:, :n_sel] @ H                                   # [g][h]
    acc_d = p[:, :n_sel] @ D[:n_sel] + p[:, n_sel:] @ D[n_sel:]
    out = (acc_h @ w2.T + acc_d) / p.sum(axis=1, keepdims=True)
    return {"out": out, "sel": sel, "scores": s}


# ---------------------------------------------------------------------- byte accounting

def compressed_bytes(cfg: dict, n_records: int) -> dict:
    """Closed-form byte counts of the compressed cache (layouts of ``lowram.h``).

    dense_equiv = M_KV * B ([Asym] "Core Mechanism") at the element size of the dense
    cache the compressed one replaces (4 B for fp32, 2 B otherwise) plus the raw tail.
    """
    B, L, G, Hkv = cfg["batch"], cfg["n_layers"], cfg["group"], cfg["n_kv_heads"]
    d, r, h, N, C, T = (cfg["head_dim"], cfg["rank"], cfg["mlp_hidden"], cfg["n_ctx"],
                        cfg["chunk"], cfg["tail_cap"])
    nC = N // C
    nL = nC - int(math.floor(cfg.get("evict_frac", 0.0) * nC))
    s = 4 if cfg["dtype"] == "f32" else 2
    int8 = cfg["store"] == "int8"
    NG = L // G
    sa = 1 if int8 else s
    coeff = B * NG * Hkv * nL * C * (r * sa + (2 if int8 else 0))
    basis = L * Hkv * r * d * s
    predictor = 2 * L * Hkv * h * d * s
    summary = B * NG * Hkv * nL * r * s
    residual = n_records * (d * sa + 2 + (2 if int8 else 0)) + B * L * Hkv * (nL + 1) * 4
    index = B * NG * Hkv * nC * 2 if nL < nC else 0
    st = 2 if int8 else s
    tail = 2 * B * L * Hkv * T * d * st + 4 * B
    total = coeff + basis + predictor + summary + residual + index + tail
    dense = dense_kv_bytes(L, Hkv, d, N, s, B) + 2 * B * L * Hkv * T * d * s
    return {"coeff": coeff, "basis": basis, "predictor": predictor, "summary": summary,
            "residual": residual, "index": index, "tail": tail, "total": total,
            "dense_equiv": dense}


def brute_force_top_k(scores: np.ndarray, k: int) -> np.ndarray:
    """Exhaustive search over every k-subset of live chunks: the subset with the largest
    score sum, ties broken toward the lexicographically smallest id list (tiny cases only).
    """
    live = [c for c in range(scores.shape[0]) if np.isfinite(scores[c])]
    best, best_key = None, None
    for sub in itertools.combinations(live, k):
        key = (sum(scores[c] for c in sub), [-c for c in sub])
        if best_key is None or key > best_key:
            best, best_key = sub, key
    return np.array(sorted(best), dtype=np.int64)
