"""Pins of the tail append / re-pack oracle (``oracle.repack``).

CPU only.  Append is checked by brute force.  Re-pack is checked by (1) the record set of
every unit before and after (old records unchanged, the new chunk's records exactly the
tokens whose residuals were planted), (2) a reconstruction round trip: over a tail that the
basis and predictor represent up to bf16 rounding, the new chunk rebuilt by the decode
oracle gives back the tail's keys and values, and decoding with every chunk selected gives
the same attention before and after; and (3) planted mistakes in the re-packed cache (records
moved to another unit, the new chunk's rows in the wrong place, the tail not shifted) that
the round trip must catch.
"""

import numpy as np
import pytest

import lowram_synth as S
import oracle as O
import oracle.encode as E
import oracle.repack as RP

TINY = S.LowramConfig(
    name="repack_pin", batch=2, n_layers=4, group=2, n_kv_heads=2, n_q_heads=4, head_dim=16,
    rank=8, mlp_hidden=12, n_ctx=32, chunk=8, top_k=2, tail_cap=12, resid_frac=0.25,
    dtype="bf16", seed=77)
N_RES = 2          # residual records kept per unit for the new chunk


def _npc(cfg, tail_len):
    return S.cache_to_numpy(S.make_cache(cfg, tail_len=tail_len))


def _bits(x):
    return E.round_bf16_bits(x)


def _representable_tail(npc, seed=5):
    """Overwrite the first C tail tokens: keys bf16(a B_l) with a shared by the layers of a
    group; values bf16(W2 silu(W1 k)) except N_RES planted tokens per unit, whose values get
    +-2 added.  Returns the planted token sets {(b, l, h): set of offsets}."""
    cfg = npc["cfg"]
    B, L, G, H, C, r = cfg["batch"], cfg["n_layers"], cfg["group"], cfg["n_kv_heads"], cfg["chunk"], cfg["rank"]
    rng = np.random.default_rng(seed)
    basis = O._bf16_bits_to_f64(npc["basis"])
    w1 = O._bf16_bits_to_f64(npc["w1"])
    w2 = O._bf16_bits_to_f64(npc["w2"])
    planted = {}
    for b in range(B):
        for grp in range(L // G):
            for h in range(H):
                a = rng.standard_normal((C, r)) / np.sqrt(np.arange(1, r + 1))
                for l in range(grp * G, (grp + 1) * G):
                    kb = _bits(a @ basis[l, h])
                    k = O._bf16_bits_to_f64(kb)
                    v = O.predict_values(w1[l, h], w2[l, h], k)
                    toks = rng.choice(C, size=N_RES, replace=False)
                    v[toks] += 2.0 * rng.choice([-1.0, 1.0], size=(N_RES, v.shape[1]))
                    npc["tail_k"][b, l, h, :C] = kb
                    npc["tail_v"][b, l, h, :C] = _bits(v)
                    planted[(b, l, h)] = set(int(t) for t in toks)
    return planted


def _records(npc):
    """{(b, l, h): {(chunk id, offset, value bytes)}} by walking the CSR through the slot map."""
    cfg = npc["cfg"]
    B, L, H, C = cfg["batch"], cfg["n_layers"], cfg["n_kv_heads"], cfg["chunk"]
    G = cfg["group"]
    rp = npc["res_ptr"].astype(np.int64)
    out = {}
    for b in range(B):
        for l in range(L):
            for h in range(H):
                slot = npc["slot"][b, l // G, h].astype(np.int64)
                recs = set()
                for c in np.nonzero(slot >= 0)[0]:
                    s = slot[c]
                    for i in range(rp[b, l, h, s], rp[b, l, h, s + 1]):
                        sc = npc["res_scale"][i].tobytes() if npc.get("res_scale") is not None else b""
                        recs.add((int(c), int(npc["res_pos"][i]), npc["res_val"][i].tobytes() + sc))
                out[(b, l, h)] = recs
    return out


def test_append_brute_force():
    npc = _npc(TINY, tail_len=[5, 12])
    rng = np.random.default_rng(1)
    L, B, H, d = TINY.n_layers, TINY.batch, TINY.n_kv_heads, TINY.head_dim
    kn = _bits(rng.standard_normal((L, B, H, d)))
    vn = _bits(rng.standard_normal((L, B, H, d)))
    out, dropped = RP.append(npc, kn, vn)
    assert dropped == [1]                                    # sequence 1's tail is full
    assert list(out["tail_len"]) == [6, 12]
    for l in range(L):
        for h in range(H):
            assert np.array_equal(out["tail_k"][0, l, h, 5], kn[l, 0, h])
            assert np.array_equal(out["tail_v"][0, l, h, 5], vn[l, 0, h])
    assert np.array_equal(np.delete(out["tail_k"][0], 5, axis=2), np.delete(npc["tail_k"][0], 5, axis=2))
    assert np.array_equal(out["tail_k"][1], npc["tail_k"][1])
    assert np.array_equal(npc["tail_len"], [5, 12])          # the input is not modified


def test_repack_refuses_short_tail():
    npc = _npc(TINY, tail_len=[7, 12])
    with pytest.raises(ValueError):
        RP.repack(npc, N_RES)


def _repacked(cfg=TINY, tail_len=(10, 12)):
    npc = _npc(cfg, tail_len=list(tail_len))
    planted = _representable_tail(npc)
    return npc, RP.repack(npc, N_RES), planted


def test_repack_record_sets_and_shapes():
    npc, out, planted = _repacked()
    C, nC = TINY.chunk, TINY.n_chunks
    assert out["cfg"]["n_ctx"] == TINY.n_ctx + C
    assert out["coeff"].shape[3] == npc["coeff"].shape[3] + C
    assert np.array_equal(out["coeff"][:, :, :, :TINY.n_ctx], npc["coeff"])
    assert np.array_equal(out["summary"][:, :, :, :nC], npc["summary"])
    before, after = _records(npc), _records(out)
    for u, recs in before.items():
        old = {x for x in after[u] if x[0] < nC}
        new = {x for x in after[u] if x[0] == nC}
        assert old == recs
        assert {x[1] for x in new} == planted[u]             # the planted tokens, nothing else
    # CSR: non-decreasing within a unit, units back to back
    rp = out["res_ptr"].astype(np.int64).reshape(-1, nC + 2)
    assert np.all(np.diff(rp, axis=1) >= 0)
    assert np.array_equal(rp[1:, 0], rp[:-1, -1]) and rp[0, 0] == 0
    assert rp[-1, -1] == out["res_pos"].shape[0] == npc["res_pos"].shape[0] + rp.shape[0] * N_RES


def test_repack_tail_shift():
    npc, out, _ = _repacked()
    C = TINY.chunk
    assert list(out["tail_len"]) == [2, 4]
    for b, n in ((0, 2), (1, 4)):
        assert np.array_equal(out["tail_k"][b, :, :, :n], npc["tail_k"][b, :, :, C:C + n])
        assert np.array_equal(out["tail_v"][b, :, :, :n], npc["tail_v"][b, :, :, C:C + n])
        assert not out["tail_k"][b, :, :, n:].any()


def _roundtrip_errors(npc, out):
    """Max errors of the new chunk's rebuilt keys and values against the tail they came from."""
    cfg, oc = npc["cfg"], O.OracleCache(out)
    C, G, nL = cfg["chunk"], cfg["group"], npc["summary"].shape[3]
    ek = ev = 0.0
    for b in range(cfg["batch"]):
        for l in range(cfg["n_layers"]):
            for h in range(cfg["n_kv_heads"]):
                rows = oc.coeff[b, l // G, h, nL * C:(nL + 1) * C]
                sig = oc.coeff_scale[b, l // G, h, nL * C:(nL + 1) * C] if oc.coeff_scale is not None else np.ones(C)
                kh = O.rebuild_keys(rows, sig, oc.basis[l, h])
                r0, r1 = oc.res_ptr[b, l, h, nL], oc.res_ptr[b, l, h, nL + 1]
                rho = oc.res_scale[r0:r1] if oc.res_scale is not None else np.ones(r1 - r0)
                vh = O.rebuild_values(kh, oc.w1[l, h], oc.w2[l, h], oc.res_pos[r0:r1], oc.res_val[r0:r1], rho)
                k = O._bf16_bits_to_f64(npc["tail_k"][b, l, h, :C])
                v = O._bf16_bits_to_f64(npc["tail_v"][b, l, h, :C])
                ek = max(ek, np.abs(kh - k).max() / np.abs(k).max())
                ev = max(ev, np.abs(vh - v).max() / np.abs(v).max())
    return ek, ev


def _decode_all_chunks(npc, q):
    cfg, oc = npc["cfg"], O.OracleCache(npc)
    g = cfg["n_q_heads"] // cfg["n_kv_heads"]
    out = np.zeros((cfg["n_layers"], cfg["batch"], cfg["n_q_heads"], cfg["head_dim"]))
    for l in range(cfg["n_layers"]):
        for b in range(cfg["batch"]):
            for h in range(cfg["n_kv_heads"]):
                live = np.nonzero(oc.slot[b, l // cfg["group"], h] >= 0)[0]
                out[l, b, h * g:(h + 1) * g] = O.decode_unit(oc, b, l, h, q[l, b, h * g:(h + 1) * g],
                                                             forced_sel=live)["out"]
    return out


def _decode_gap(npc, out, seed=3):
    rng = np.random.default_rng(seed)
    cfg = npc["cfg"]
    q = rng.standard_normal((cfg["n_layers"], cfg["batch"], cfg["n_q_heads"], cfg["head_dim"]))
    o0, o1 = _decode_all_chunks(npc, q), _decode_all_chunks(out, q)
    return (np.abs(o1 - o0).max(axis=-1) / np.linalg.norm(o0, axis=-1)).max()


# The new chunk's keys come back to the bf16 rounding of the stored coefficients and of the
# raw keys (a few 2^-9 of the largest entry); values to the bf16 rounding of the raw values,
# of the residual rows and of the predictor's input (2^-6 of the largest entry covers them).
K_TOL, V_TOL, DECODE_TOL = 2 ** -6, 2 ** -6, 2e-2


def test_repack_reconstruction_round_trip():
    npc, out, _ = _repacked()
    ek, ev = _roundtrip_errors(npc, out)
    assert ek <= K_TOL and ev <= V_TOL, (ek, ev)
    assert _decode_gap(npc, out) <= DECODE_TOL


def test_repack_round_trip_catches_planted_mistakes():
    npc, out, _ = _repacked()
    nC, C = TINY.n_chunks, TINY.chunk
    # (1) the new chunk's records attached to the next unit (CSR offsets shifted by a unit)
    bad = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in out.items()}
    rp = bad["res_ptr"].reshape(-1, nC + 2)
    nrec = rp[:, nC + 1] - rp[:, nC]
    rp[1:, nC], rp[1:, nC + 1] = rp[:-1, nC], rp[:-1, nC + 1]
    assert np.all(nrec == N_RES)
    assert _roundtrip_errors(npc, bad)[1] > 10 * V_TOL
    # (2) the new chunk's rows written over the first chunk instead of after the last
    bad = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in out.items()}
    bad["coeff"][:, :, :, nC * C:] = out["coeff"][:, :, :, :C]
    assert _roundtrip_errors(npc, bad)[0] > 10 * K_TOL
    # (3) the tail not shifted: its first chunk is attended twice
    bad = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in out.items()}
    bad["tail_k"], bad["tail_v"], bad["tail_len"] = npc["tail_k"], npc["tail_v"], npc["tail_len"]
    assert _decode_gap(npc, bad) > 5 * DECODE_TOL


@pytest.mark.parametrize("store,evict", [("native", 0.5), ("int8", 0.0), ("int8", 0.5)])
def test_repack_int8_and_eviction(store, evict):
    cfg = TINY.replace(name="repack_pin_var", store=store, evict_frac=evict, n_ctx=64)
    npc, out, planted = _repacked(cfg)
    nC, nL, C = cfg.n_chunks, cfg.n_live, cfg.chunk
    # the new chunk is live, in the slot after the last live one
    assert np.all(out["slot"][..., nC] == nL)
    assert np.array_equal(out["slot"][..., :nC], npc["slot"])
    assert np.array_equal(out["coeff"][:, :, :, :nL * C], npc["coeff"])
    if store == "int8":
        assert np.array_equal(out["coeff_scale"][:, :, :, :nL * C], npc["coeff_scale"])
    before, after = _records(npc), _records(out)
    for u, recs in before.items():
        assert {x for x in after[u] if x[0] < nC} == recs
        assert {x[1] for x in after[u] if x[0] == nC} == planted[u]
    ek, ev = _roundtrip_errors(npc, out)
    # int8 rows: one code step of the row maximum (2^-7) on top of the bf16 terms
    tol = 2 ** -5 if store == "int8" else K_TOL
    assert ek <= tol and ev <= 2 * tol, (ek, ev)
    assert _decode_gap(npc, out) <= (4e-2 if store == "int8" else DECODE_TOL)
