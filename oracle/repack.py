"""Plain CPU oracle of the decode loop's cache upkeep: appending a decode step's keys and
values to the raw tail, and re-packing the tail's oldest chunk into the compressed store.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may import this module.  It shares no code with the CUDA library.

Pages (names as in ``oracle/__init__.py``): [Rit] keeps the tokens generated after prefill
uncompressed (the raw tail); [Abstract] and [Asym] compress a context with a given basis
and predictor (coefficients on the group basis, Vhat = f(K), residuals kept for the worst
tokens).  The pages name no moment at which new tokens join the compressed store; this
library's reading (no page fixes it; it is the plainest one): once every sequence's tail holds
at least C tokens, the oldest C tail tokens of every (sequence, layer, KV head) are encoded
by the encoder's steps (``oracle.encode``) as one new chunk, appended after the existing
chunks (a new live chunk when the cache evicts), and removed from the tail.

Both functions take and return the cache dict ``OracleCache`` reads (storage form: bf16 as
uint16 bit patterns).  The returned dict is a new one; the input is not modified.

Parity pins: ``tests/test_repack_pins.py`` (appended rows by brute force, the record set
before and after, the tail shift, and a decode round trip over a tail the basis and
predictor represent to bf16 rounding, with planted mistakes that the round trip catches).
"""

from __future__ import annotations

from typing import Optional

import numpy as np

from . import _f64
from . import encode as E

__all__ = ["append", "repack"]


def _copy(npc: dict) -> dict:
    out = {}
    for k, v in npc.items():
        out[k] = v.copy() if isinstance(v, np.ndarray) else (dict(v) if isinstance(v, dict) else v)
    return out


def append(npc: dict, k_new: np.ndarray, v_new: np.ndarray):
    """Write one decode step's key and value of every (layer, sequence, KV head) after the
    sequence's tail, and count the token: tail[b][l][h][tail_len[b]] = new, tail_len[b] += 1.

    k_new, v_new [L][B][Hkv][d] in the tail's storage form.  A sequence whose tail is full
    (tail_len[b] == T) is left unchanged.  Returns (new dict, list of the sequences whose
    token was dropped)."""
    out = _copy(npc)
    T = npc["cfg"]["tail_cap"]
    dropped = []
    for b in range(out["tail_len"].shape[0]):
        t = int(out["tail_len"][b])
        if t >= T:
            dropped.append(b)
            continue
        out["tail_k"][b, :, :, t] = k_new[:, b]
        out["tail_v"][b, :, :, t] = v_new[:, b]
        out["tail_len"][b] = t + 1
    return out, dropped


def repack(npc: dict, n_res: int, given: Optional[tuple] = None) -> dict:
    """Encode the oldest C tail tokens of every unit into one new chunk and append it.

    n_res residual records are kept for the new chunk of each (sequence, layer, KV head)
    (its n_res worst-predicted tokens).  ``given`` is passed to ``oracle.encode`` (the new
    chunk's stored coefficients from another implementation).  Records of the result are in
    unit order (b, l, KV head): a unit's old records, then its new chunk's.  Tail rows at or
    past the new tail length are zero."""
    cfg = npc["cfg"]
    B, L, G, Hkv = cfg["batch"], cfg["n_layers"], cfg["group"], cfg["n_kv_heads"]
    C, T, d = cfg["chunk"], cfg["tail_cap"], cfg["head_dim"]
    NG = L // G
    tl = npc["tail_len"].astype(np.int64)
    if np.any(tl < C):
        raise ValueError("every sequence's tail must hold at least one chunk")
    bf = lambda n: npc.get(n + "_is_bf16", False)
    keys = _f64(npc["tail_k"][:, :, :, :C], bf("tail_k"))
    values = _f64(npc["tail_v"][:, :, :, :C], bf("tail_v"))
    basis = _f64(npc["basis"], bf("basis"))
    w1 = _f64(npc["w1"], bf("w1"))
    w2 = _f64(npc["w2"], bf("w2"))
    enc = E.encode(dict(cfg, n_ctx=C), keys, values, basis, w1, w2, n_res, given=given)

    out = _copy(npc)
    int8 = cfg["store"] == "int8"
    nL = npc["summary"].shape[3]
    out["coeff"] = np.concatenate([npc["coeff"], enc["coeff"]], axis=3)
    if int8:
        out["coeff_scale"] = np.concatenate([npc["coeff_scale"], enc["coeff_scale"]], axis=3)
    out["summary"] = np.concatenate([npc["summary"], enc["summary"]], axis=3)
    out["slot"] = np.concatenate([npc["slot"], np.full((B, NG, Hkv, 1), nL, dtype=npc["slot"].dtype)],
                                 axis=3)

    rp, erp = npc["res_ptr"].astype(np.int64), enc["res_ptr"].astype(np.int64)
    new_ptr = np.zeros((B, L, Hkv, nL + 2), dtype=np.int64)
    pos, val, scl = [], [], []
    base = 0
    for b in range(B):
        for l in range(L):
            for h in range(Hkv):
                r0, r1 = rp[b, l, h, 0], rp[b, l, h, nL]
                e0, e1 = erp[b, l, h, 0], erp[b, l, h, 1]
                new_ptr[b, l, h, :nL + 1] = base + (rp[b, l, h] - r0)
                new_ptr[b, l, h, nL + 1] = base + (r1 - r0) + (e1 - e0)
                base += (r1 - r0) + (e1 - e0)
                pos += [npc["res_pos"][r0:r1], enc["res_pos"][e0:e1]]
                val += [npc["res_val"][r0:r1], enc["res_val"][e0:e1]]
                if int8:
                    scl += [npc["res_scale"][r0:r1], enc["res_scale"][e0:e1]]
    out["res_ptr"] = new_ptr.astype(np.int32)
    out["res_pos"] = np.concatenate(pos).astype(npc["res_pos"].dtype)
    out["res_val"] = np.concatenate(val).astype(npc["res_val"].dtype).reshape(-1, d)
    if int8:
        out["res_scale"] = np.concatenate(scl).astype(npc["res_scale"].dtype)

    for name in ("tail_k", "tail_v"):
        t_old, t_new = npc[name], np.zeros_like(npc[name])
        for b in range(B):
            n = int(tl[b]) - C
            t_new[b, :, :, :n] = t_old[b, :, :, C:C + n]
        out[name] = t_new
    out["tail_len"] = (tl - C).astype(npc["tail_len"].dtype)
    out["cfg"] = dict(cfg, n_ctx=cfg["n_ctx"] + C)
    return out
