"""Plain fp64 CPU oracle of the prefill-side encoder: dense keys and values -> the
compressed cache that the decode oracle (and the CUDA library) reads.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may import this module.  It shares no code with the CUDA library.

The encoder uses a GIVEN basis and predictor (no fitting).  Its steps, in the order the
pages describe the stored form (page names as in ``oracle/__init__.py``):

1. Keys -> coefficients shared by the G layers of a group ([Asym] "Cross-Layer Low-Rank Key
   Compression"; [Rit] xKV: keys of adjacent layers on one common basis): the
   least-squares coefficients a_t = argmin_a sum_{l in group} |k_{l,t} - a B_l|^2, i.e. the
   normal equations a (sum_l B_l B_l^T) = sum_l k_{l,t} B_l^T.
2. Coefficient storage: bf16, or int8 with a per-row fp16 scale ([Asym] "Composition with
   Quantization and Eviction"; the encoding itself is this library's reading: scale =
   max|x| / 127 rounded to fp16, code = round-half-even(x / scale) clamped to +-127).
3. Chunk summaries: the mean of each chunk's stored (dequantised) coefficient rows (reading;
   no page defines a summary).
4. Values: vhat_t = W2 silu(W1 khat_t) from the rebuilt key khat_t = stored a_t . B_l, and
   the residual delta_t = v_t - vhat_t ([Asym] "Core Mechanism: Predict Values and Keep
   Difficult Residuals": Vhat = f(K), delta = V - Vhat).
5. Residual flags: the n_res tokens of each (sequence, layer, KV head) with the largest
   |delta_t|_2, ties to the lower token index ([Asym] "Core Mechanism": residuals are kept
   for the worst-predicted tokens; the count per unit is the caller's).
6. Records: per unit, chunk by chunk, ascending token offset, as offsets into one record
   array (the layout ``lowram.h`` documents for ``lowram_cache_src``).

Parity pins: ``tests/test_encode_pins.py`` (exact recovery of planted coefficients, the
normal equations, the predictor against torch, brute-force flags, decode round trip).
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np

from . import silu

__all__ = ["lstsq_coefficients", "round_bf16_bits", "quantize_rows_int8", "flag_worst",
           "encode"]


def lstsq_coefficients(keys: np.ndarray, bases: np.ndarray) -> np.ndarray:
    """Least-squares coefficients of a group's keys on its stacked basis.

    keys [G][N][d], bases [G][r][d] (the group's layer slices B_l) -> a [N][r] with
    a (sum_l B_l B_l^T) = sum_l k_l B_l^T ([Asym] "Cross-Layer Low-Rank Key Compression").
    """
    gram = np.zeros((bases.shape[1], bases.shape[1]))
    rhs = np.zeros((keys.shape[1], bases.shape[1]))
    for k_l, b_l in zip(keys, bases):
        gram += b_l @ b_l.T
        rhs += k_l @ b_l.T
    return np.linalg.solve(gram, rhs.T).T


def round_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns (uint16): round to float32, then to bf16, each to nearest
    even (the order in which a float32 computation is stored as bf16)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _bits_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def quantize_rows_int8(x: np.ndarray):
    """Per-row int8 codes and fp16 scales: scale = fp16(max|x| / 127), code =
    round-half-even(x / scale) clamped to +-127; an all-zero row has scale 0 and codes 0.
    The division is taken in float32, the precision the CUDA encoder uses for it."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.abs(x32).max(axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float16)
    s = scale.astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0))
    q = np.clip(np.rint(x32 / safe[..., None]), -127, 127)
    q = np.where((s > 0)[..., None], q, 0)
    return q.astype(np.int8), scale


def flag_worst(norms: np.ndarray, n_res: int) -> np.ndarray:
    """Boolean mask of the n_res largest entries of a 1-D array, ties to the lower index."""
    order = np.lexsort((np.arange(norms.shape[0]), -norms))
    mask = np.zeros(norms.shape[0], dtype=bool)
    mask[order[:n_res]] = True
    return mask


def encode(cfg: dict, keys: np.ndarray, values: np.ndarray, basis: np.ndarray,
           w1: np.ndarray, w2: np.ndarray, n_res: int,
           tail_k: Optional[np.ndarray] = None, tail_v: Optional[np.ndarray] = None,
           tail_len: Optional[np.ndarray] = None, given: Optional[tuple] = None) -> dict:
    """Encode dense keys/values [B][L][Hkv][N][d] (float64) with the given basis [L][Hkv][r][d],
    predictor w1 [L][Hkv][h][d], w2 [L][Hkv][d][h] (float64) into the storage layout of
    ``lowram.h`` (no eviction: every chunk live).  Returns the dict ``OracleCache`` reads,
    with bf16 arrays as uint16 bit patterns (storage dtype bf16; int8 + fp16 scales when
    cfg["store"] == "int8").  The tail arrays are passed through (zero-length tails if
    omitted).  Also returns, under "extra", the float64 intermediates the tests compare:
    coefficients before storage, residual norms and flags.

    ``given`` = (codes, scales) replaces the result of steps 1-2 with given stored
    coefficients (bf16 bit patterns and None, or int8 codes and fp16 scales, layout of
    ``coeff`` / ``coeff_scale``), so that steps 3-6 can be checked on exactly the stored
    values another implementation produced."""
    B, L, Hkv, N, d = keys.shape
    G, C = cfg["group"], cfg["chunk"]
    r = basis.shape[2]
    NG, nC = L // G, N // C
    int8 = cfg["store"] == "int8"

    coeff_full = np.zeros((B, NG, Hkv, N, r))
    stored = np.zeros((B, NG, Hkv, N, r))           # dequantised stored coefficients
    coeff_store = np.zeros((B, NG, Hkv, N, r), dtype=np.int8 if int8 else np.uint16)
    coeff_scale = np.zeros((B, NG, Hkv, N), dtype=np.float16) if int8 else None
    summary = np.zeros((B, NG, Hkv, nC, r), dtype=np.uint16)
    for b in range(B):
        for grp in range(NG):
            ls = slice(grp * G, (grp + 1) * G)
            for h in range(Hkv):
                a = lstsq_coefficients(keys[b, ls, h], basis[ls, h])       # step 1
                coeff_full[b, grp, h] = a
                if given is not None:
                    q = given[0][b, grp, h]
                    s = given[1][b, grp, h] if int8 else None
                elif int8:                                                  # step 2
                    q, s = quantize_rows_int8(a)
                else:
                    q, s = round_bf16_bits(a), None
                if int8:
                    coeff_store[b, grp, h] = q
                    coeff_scale[b, grp, h] = s
                    deq = q.astype(np.float64) * s.astype(np.float64)[:, None]
                else:
                    coeff_store[b, grp, h] = q
                    deq = _bits_f64(q)
                stored[b, grp, h] = deq
                summary[b, grp, h] = round_bf16_bits(deq.reshape(nC, C, r).mean(axis=1))   # step 3

    norms = np.zeros((B, L, Hkv, N))
    flags = np.zeros((B, L, Hkv, N), dtype=bool)
    res_ptr = np.zeros((B, L, Hkv, nC + 1), dtype=np.int64)
    pos_list, val_list = [], []
    base = 0
    for b in range(B):
        for l in range(L):
            grp = l // G
            for h in range(Hkv):
                khat = stored[b, grp, h] @ basis[l, h]                      # step 4
                vhat = silu(khat @ w1[l, h].T) @ w2[l, h].T
                delta = values[b, l, h] - vhat
                nrm = np.sqrt((delta * delta).sum(axis=1))
                norms[b, l, h] = nrm
                f = flag_worst(nrm, n_res)                                  # step 5
                flags[b, l, h] = f
                idx = np.nonzero(f)[0]                                      # step 6
                counts = np.bincount(idx // C, minlength=nC)
                res_ptr[b, l, h, 0] = base
                res_ptr[b, l, h, 1:] = base + np.cumsum(counts)
                base += idx.size
                pos_list.append((idx % C).astype(np.uint16))
                val_list.append(delta[idx])
    res_pos = np.concatenate(pos_list) if pos_list else np.zeros(0, dtype=np.uint16)
    vals = np.concatenate(val_list) if val_list else np.zeros((0, d))
    if int8:
        res_val, res_scale = quantize_rows_int8(vals)
    else:
        res_val, res_scale = round_bf16_bits(vals), None

    T = cfg["tail_cap"]
    if tail_k is None:
        tail_k = np.zeros((B, L, Hkv, T, d))
        tail_v = np.zeros((B, L, Hkv, T, d))
        tail_len = np.zeros(B, dtype=np.int32)
    out_cfg = dict(cfg)
    out_cfg["n_ctx"] = N
    npc = {
        "cfg": out_cfg,
        "coeff": coeff_store, "coeff_is_bf16": not int8,
        "coeff_scale": coeff_scale, "coeff_scale_is_bf16": False,
        "basis": round_bf16_bits(basis), "basis_is_bf16": True,
        "w1": round_bf16_bits(w1), "w1_is_bf16": True,
        "w2": round_bf16_bits(w2), "w2_is_bf16": True,
        "summary": summary, "summary_is_bf16": True,
        "slot": np.broadcast_to(np.arange(nC, dtype=np.int16), (B, NG, Hkv, nC)).copy(),
        "slot_is_bf16": False,
        "res_ptr": res_ptr.astype(np.int32), "res_ptr_is_bf16": False,
        "res_pos": res_pos, "res_pos_is_bf16": False,
        "res_val": res_val, "res_val_is_bf16": not int8,
        "res_scale": res_scale, "res_scale_is_bf16": False,
        "tail_k": round_bf16_bits(tail_k), "tail_k_is_bf16": True,
        "tail_v": round_bf16_bits(tail_v), "tail_v_is_bf16": True,
        "tail_len": np.asarray(tail_len, dtype=np.int32), "tail_len_is_bf16": False,
        "extra": {"coeff_full": coeff_full, "stored_coeff": stored, "norms": norms,
                  "flags": flags},
    }
    return npc
