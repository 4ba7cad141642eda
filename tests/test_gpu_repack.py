"""Parity of the decode-loop upkeep (tail append, chunk re-pack) with ``oracle.repack``.

Append is compared bit for bit.  Re-pack: the old chunks' arrays and records must come
through bit for bit, the tail shift likewise; the new chunk is the encoder's work on the
tail's oldest chunk and is compared with the encoder oracle under the encoder's rules
(``test_gpu_encode._check_encode``); then the re-packed cache validates and decodes on the
GPU in parity with the decode oracle run on the same arrays.
"""

import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
import oracle.repack as RP
from parity_utils import check
from test_gpu_encode import _check_encode

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np_arrays(arrays, cfg):
    """torch views of a cache's arrays -> the oracle's dict layout."""
    out = {"cfg": dataclasses.asdict(cfg)}
    for n, t in arrays.items():
        out[n] = S._np_storage(t)
        if n == "res_pos" and out[n] is not None:
            out[n] = out[n].view("uint16")
        out[n + "_is_bf16"] = bool(t is not None and t.dtype == torch.bfloat16)
    if out["slot"] is None:
        B, NG, H = cfg.batch, cfg.n_layers // cfg.group, cfg.n_kv_heads
        out["slot"] = np.broadcast_to(np.arange(cfg.n_chunks, dtype=np.int16), (B, NG, H, cfg.n_chunks)).copy()
    return out


def _unit_records(npc, cfg, u_slots):
    """{unit: [(slot, pos, value bytes, scale bytes)]} for the slots in u_slots."""
    rp = npc["res_ptr"].astype(np.int64).reshape(-1, npc["res_ptr"].shape[-1])
    out = {}
    for u in range(rp.shape[0]):
        recs = []
        for s in u_slots:
            for i in range(rp[u, s], rp[u, s + 1]):
                sc = npc["res_scale"][i].tobytes() if npc.get("res_scale") is not None else b""
                recs.append((s, int(npc["res_pos"][i]), npc["res_val"][i].tobytes(), sc))
        out[u] = recs
    return out


def _check_layout(rp, arrays, n_live_records, spare_records):
    """Units in unit order, each unit's records followed by its spare rows, inside the array."""
    assert rp[0, 0] == 0
    assert np.all(rp[:-1, -1] + spare_records == rp[1:, 0])
    assert rp[-1, -1] + spare_records == arrays["res_pos"].shape[0]
    assert int((rp[:, -1] - rp[:, 0]).sum()) == n_live_records


def _new_chunk(arrays, cfg, s, n_res):
    """The arrays of live slot s (a re-packed chunk) in the encoder's output form."""
    B, L, H, C = cfg.batch, cfg.n_layers, cfg.n_kv_heads, cfg.chunk
    U = B * L * H
    int8 = cfg.store == "int8"
    rp = arrays["res_ptr"].cpu().numpy().astype(np.int64).reshape(U, -1)
    idx = torch.as_tensor(np.concatenate([np.arange(rp[u, s], rp[u, s + 1]) for u in range(U)]), device=DEV)
    assert np.all(rp[:, s + 1] - rp[:, s] == n_res)
    return {
        "coeff": arrays["coeff"][:, :, :, s * C:(s + 1) * C].contiguous(),
        "coeff_scale": arrays["coeff_scale"][:, :, :, s * C:(s + 1) * C].contiguous() if int8 else None,
        "summary": arrays["summary"][:, :, :, s:s + 1].contiguous(),
        "res_ptr": torch.tensor(np.stack([np.arange(U) * n_res, np.arange(1, U + 1) * n_res], -1)
                                .reshape(B, L, H, 2), dtype=torch.int32),
        "res_pos": arrays["res_pos"][idx], "res_val": arrays["res_val"][idx],
        "res_scale": arrays["res_scale"][idx] if int8 else None,
    }


def _codes(g, int8):
    if int8:
        return (g["coeff"].cpu().numpy(), g["coeff_scale"].cpu().numpy())
    return (g["coeff"].cpu().view(torch.int16).numpy().view(np.uint16), None)


def _decode_check(lc, cfg2, arrays):
    got = _np_arrays(arrays, cfg2)
    gpu_cache = S.SynthCache(cfg=cfg2, **{n: (t.clone() if t is not None else None) for n, t in arrays.items()})
    gpu_cache.slot = torch.as_tensor(got["slot"], device=DEV)
    q = S.make_queries(gpu_cache).to(DEV)
    out, sel = lc.decode(q, sel=True)
    scores, _ = lc.select(q)
    torch.cuda.synchronize()
    check(cfg2, O.OracleCache(got), q, out, sel, scores=scores)


@pytest.mark.parametrize("store,evict", [("native", 0.0), ("int8", 0.5)])
def test_repeated_repacks_in_place_and_relaid(store, evict):
    """Six re-packs from one long tail: the first re-lays the cache with room for 4 more
    chunks, the next four write in place, the sixth re-lays again; the residual count per
    chunk changes from call to call (the re-pack scratch, with the encoder's kept copy of
    W2, is laid out again each time).  Every new chunk is the encoder's work on its tail
    segment; old chunks stay bit for bit; the cache decodes in parity after an in-place
    re-pack and at the end."""
    import oracle.encode as E
    C = 128
    cfg = S.LLAMA_32K.replace(name="repack6", batch=2, n_layers=4, n_kv_heads=2, n_ctx=512, top_k=2,
                              tail_cap=6 * C, store=store, evict_frac=evict)
    n_res_seq = [16, 8, 16, 8, 8, 16]
    cache = S.make_cache(cfg, tail_len=[6 * C, 6 * C])
    npc = S.cache_to_numpy(cache)
    lc = K.LowramCache.from_synth(cache.to(DEV))
    nL0 = cfg.n_live
    spares = []
    for i in range(6):
        lc.repack(n_res_seq[i])
        cfg2d, arrays = lc.view()
        spares.append(cfg2d["spare_chunks"])
        if i == 2:
            cfg2 = cfg.replace(n_ctx=cfg.n_ctx + 3 * C)
            _decode_check(lc, cfg2, arrays)
    assert spares == [4, 3, 2, 1, 0, 4]
    cfg2d, arrays = lc.view()
    cfg2 = cfg.replace(n_ctx=cfg.n_ctx + 6 * C)
    assert cfg2d["n_live"] == nL0 + 6 and arrays["tail_len"].cpu().tolist() == [0, 0]
    int8 = store == "int8"
    assert np.array_equal(S._np_storage(arrays["coeff"][:, :, :, :nL0 * C]), npc["coeff"])
    assert np.array_equal(S._np_storage(arrays["summary"][:, :, :, :nL0]), npc["summary"])
    U = cfg.batch * cfg.n_layers * cfg.n_kv_heads
    rp = arrays["res_ptr"].cpu().numpy().astype(np.int64).reshape(U, -1)
    _check_layout(rp, arrays, npc["res_pos"].shape[0] + U * sum(n_res_seq), 4 * n_res_seq[-1])
    cfg_c = cfg.replace(name="repack_chunk", n_ctx=C, evict_frac=0.0)
    f64 = O._bf16_bits_to_f64
    for i in range(6):
        n_res = n_res_seq[i]
        g_new = _new_chunk(arrays, cfg, nL0 + i, n_res)
        seg = slice(i * C, (i + 1) * C)
        args = (dataclasses.asdict(cfg_c), f64(npc["tail_k"][:, :, :, seg]), f64(npc["tail_v"][:, :, :, seg]),
                f64(npc["basis"]), f64(npc["w1"]), f64(npc["w2"]), n_res)
        _check_encode(cfg_c, g_new, E.encode(*args), E.encode(*args, given=_codes(g_new, int8)), n_res)
    assert lc.validate() == 0
    _decode_check(lc, cfg2, arrays)
    lc.close()


def test_append_matches_oracle():
    cfg = S.MISTRAL_GROUP.replace(name="append", batch=3, n_ctx=1024)
    cache = S.make_cache(cfg, tail_len=[5, cfg.tail_cap, 0])
    npc = S.cache_to_numpy(cache)
    lc = K.LowramCache.from_synth(cache.to(DEV))
    g = torch.Generator().manual_seed(3)
    shape = (cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.head_dim)
    for step in range(3):
        kn = torch.randn(shape, generator=g).to(torch.bfloat16)
        vn = torch.randn(shape, generator=g).to(torch.bfloat16)
        lc.append(kn.to(DEV), vn.to(DEV))
        npc, dropped = RP.append(npc, S._np_storage(kn), S._np_storage(vn))
        assert dropped == [1]
    torch.cuda.synchronize()
    _, arrays = lc.view()
    assert arrays["tail_len"].cpu().tolist() == [8, cfg.tail_cap, 3] == list(npc["tail_len"])
    for name in ("tail_k", "tail_v"):
        assert np.array_equal(S._np_storage(arrays[name]), npc[name])
    assert lc.validate() == 1          # the full tail's tokens were dropped
    assert lc.validate() == 0          # ... and the word is cleared
    lc.close()


# (config, overrides, store, evict fraction, tail_cap in chunks, tail lengths in chunks + extra)
REPACK_CASES = [
    ("llama8b_32k_bf16", dict(n_layers=4, n_kv_heads=2, n_ctx=512), "native", 0.0, 1, (0, 0)),
    ("llama8b_32k_bf16", dict(n_layers=4, n_kv_heads=2, n_ctx=512), "native", 0.0, 2, (5, 128)),
    ("llama8b_32k_bf16", dict(n_layers=4, n_kv_heads=2, n_ctx=1024, rank=64), "int8", 0.5, 2, (1, 0)),
    ("llama8b_32k_bf16", dict(n_layers=4, n_kv_heads=1, n_q_heads=4, n_ctx=512), "native", 0.5, 1, (0, 0)),
    ("mistral7b_group_bf16", dict(n_layers=4, n_kv_heads=2, n_ctx=512), "int8", 0.0, 3, (70, 3)),
]


@pytest.mark.parametrize("case", REPACK_CASES, ids=lambda c: f"{c[0][:7]}-{c[2]}-e{c[3]}-t{c[4]}")
def test_repack_matches_oracle(case):
    name, kw, store, evict, tcap, extra = case
    base = S.CONFIGS[name]
    C = base.chunk
    cfg = base.replace(name="repack", batch=2, store=store, evict_frac=evict, tail_cap=tcap * C, top_k=2, **kw)
    n_res = max(1, int(round(cfg.resid_frac * C)))
    tl = [C + extra[0], C + extra[1]]
    cache = S.make_cache(cfg, tail_len=tl)
    npc = S.cache_to_numpy(cache)
    lc = K.LowramCache.from_synth(cache.to(DEV))
    lc.repack(n_res)
    cfg2d, arrays = lc.view()
    nC, nL = cfg.n_chunks, cfg.n_live
    assert cfg2d["n_ctx"] == cfg.n_ctx + C and cfg2d["n_live"] == nL + 1
    cfg2 = cfg.replace(n_ctx=cfg.n_ctx + C, evict_frac=0.0 if evict == 0 else cfg.evict_frac)
    got = _np_arrays(arrays, cfg2)
    int8 = store == "int8"

    # the new chunk: the encoder's work on the tail's oldest C tokens, encoder rules
    cfg_c = cfg.replace(name="repack_chunk", n_ctx=C, evict_frac=0.0)
    B, NG, H = cfg.batch, cfg.n_layers // cfg.group, cfg.n_kv_heads
    U = B * cfg.n_layers * H
    rp = got["res_ptr"].astype(np.int64).reshape(U, nL + 2)
    new_idx = np.concatenate([np.arange(rp[u, nL], rp[u, nL + 1]) for u in range(U)])
    assert np.all(rp[:, nL + 1] - rp[:, nL] == n_res)
    g_new = {
        "coeff": arrays["coeff"][:, :, :, nL * C:].contiguous(),
        "coeff_scale": arrays["coeff_scale"][:, :, :, nL * C:].contiguous() if int8 else None,
        "summary": arrays["summary"][:, :, :, nL:].contiguous(),
        "res_ptr": torch.tensor(np.stack([np.arange(U) * n_res, np.arange(1, U + 1) * n_res], -1)
                                .reshape(B, cfg.n_layers, H, 2), dtype=torch.int32),
        "res_pos": arrays["res_pos"][torch.as_tensor(new_idx, device=DEV)],
        "res_val": arrays["res_val"][torch.as_tensor(new_idx, device=DEV)],
        "res_scale": arrays["res_scale"][torch.as_tensor(new_idx, device=DEV)] if int8 else None,
    }
    codes = (g_new["coeff"].cpu().numpy(), g_new["coeff_scale"].cpu().numpy()) if int8 else \
        (g_new["coeff"].cpu().view(torch.int16).numpy().view(np.uint16), None)
    ref = RP.repack(npc, n_res)
    ref_g = RP.repack(npc, n_res, given=codes)
    tk = lambda t: O._bf16_bits_to_f64(t[:, :, :, :C])
    E_args = (dataclasses.asdict(cfg_c), tk(npc["tail_k"]), tk(npc["tail_v"]), O._bf16_bits_to_f64(npc["basis"]),
              O._bf16_bits_to_f64(npc["w1"]), O._bf16_bits_to_f64(npc["w2"]), n_res)
    import oracle.encode as E
    _check_encode(cfg_c, g_new, E.encode(*E_args), E.encode(*E_args, given=codes), n_res)

    # the old chunks: bit for bit
    assert np.array_equal(got["coeff"][:, :, :, :nL * C], npc["coeff"])
    if int8:
        assert np.array_equal(got["coeff_scale"][:, :, :, :nL * C], npc["coeff_scale"])
    assert np.array_equal(got["summary"][:, :, :, :nL], npc["summary"])
    assert np.array_equal(got["slot"], ref["slot"])
    old_g, old_o = _unit_records(got, cfg2, range(nL)), _unit_records(npc, cfg, range(nL))
    assert old_g == old_o
    _check_layout(rp, arrays, npc["res_pos"].shape[0] + U * n_res, cfg2d["spare_chunks"] * n_res)
    # where the flags agree, each unit's records are laid as the oracle lays them
    rp_o = ref_g["res_ptr"].astype(np.int64).reshape(U, nL + 2)
    live_pos = np.concatenate([got["res_pos"][rp[u, 0]:rp[u, -1]] for u in range(U)])
    if np.array_equal(live_pos, ref_g["res_pos"]):
        assert np.array_equal(rp - rp[:, :1], rp_o - rp_o[:, :1])
    # the tail: shifted by C, lengths down by C
    assert list(got["tail_len"]) == list(ref["tail_len"]) == [extra[0], extra[1]]
    for name in ("tail_k", "tail_v"):
        for b in range(B):
            n = int(ref["tail_len"][b])
            assert np.array_equal(got[name][b, :, :, :n], ref[name][b, :, :, :n])

    # the re-packed cache validates and decodes in parity with the oracle on its arrays
    assert lc.validate() == 0
    gpu_cache = S.SynthCache(cfg=cfg2, **{n: (t.clone() if t is not None else None) for n, t in arrays.items()})
    if gpu_cache.slot is None:
        gpu_cache.slot = torch.as_tensor(got["slot"], device=DEV)
    q = S.make_queries(gpu_cache).to(DEV)
    out, sel = lc.decode(q, sel=True)
    scores, _ = lc.select(q)
    torch.cuda.synchronize()
    check(cfg2, O.OracleCache(got), q, out, sel, scores=scores)
    lc.close()


def test_repack_refuses_short_tail_and_keeps_cache():
    cfg = S.LLAMA_32K.replace(name="repack_short", batch=2, n_layers=4, n_kv_heads=1, n_q_heads=4, n_ctx=512,
                              top_k=2)
    cache = S.make_cache(cfg, tail_len=[cfg.chunk, cfg.chunk - 1])
    lc = K.LowramCache.from_synth(cache.to(DEV))
    with pytest.raises(K.LowramError) as ei:
        lc.repack(8)
    assert ei.value.status == 1
    cfg2, arrays = lc.view()
    assert cfg2["n_ctx"] == cfg.n_ctx and arrays["tail_len"].cpu().tolist() == [cfg.chunk, cfg.chunk - 1]
    with pytest.raises(K.LowramError) as ei:
        lc.repack(cfg.chunk + 1)                       # more records than tokens
    assert ei.value.status == 1
    lc.close()


def test_decode_loop_append_repack_decode():
    """C decode steps appended to a tail of length 0, a re-pack, then a decode: the cache
    holds one more chunk and the decode matches the oracle on the GPU's arrays."""
    cfg = S.LLAMA_32K.replace(name="decode_loop", batch=2, n_layers=4, n_kv_heads=2, n_ctx=512, top_k=2)
    C = cfg.chunk
    cache = S.make_cache(cfg, tail_len=[0, 0])
    lc = K.LowramCache.from_synth(cache.to(DEV))
    g = torch.Generator(device=DEV).manual_seed(9)
    shape = (cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.head_dim)
    for _ in range(C):
        lc.append((torch.randn(shape, generator=g, device=DEV) * 0.3).to(torch.bfloat16),
                  (torch.randn(shape, generator=g, device=DEV) * 0.1).to(torch.bfloat16))
    lc.repack(16)
    cfg2d, arrays = lc.view()
    assert cfg2d["n_ctx"] == cfg.n_ctx + C and arrays["tail_len"].cpu().tolist() == [0, 0]
    cfg2 = cfg.replace(n_ctx=cfg.n_ctx + C)
    got = _np_arrays(arrays, cfg2)
    gpu_cache = S.SynthCache(cfg=cfg2, **{n: (t.clone() if t is not None else None) for n, t in arrays.items()})
    gpu_cache.slot = torch.as_tensor(got["slot"], device=DEV)
    q = S.make_queries(gpu_cache).to(DEV)
    out, sel = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    assert lc.validate() == 0
    check(cfg2, O.OracleCache(got), q, out, sel)
    lc.close()


def test_host_entry_graph_follows_the_repack():
    """lowram_decode_attn_host replays a captured decode; after a re-pack it must decode the
    longer cache (the captured graph is dropped), matching the device entry point."""
    cfg = S.LLAMA_32K.replace(name="host_graph", batch=2, n_layers=4, n_kv_heads=2, n_ctx=512, top_k=2)
    cache = S.make_cache(cfg, tail_len=[cfg.chunk, cfg.chunk])
    lc = K.LowramCache.from_synth(cache.to(DEV))
    q = S.make_queries(cache).to(DEV)
    q_h = q.cpu().pin_memory()
    out_h = torch.empty_like(q_h).pin_memory()
    for step in range(2):
        out_d = lc.decode(q)
        torch.cuda.synchronize()
        for _ in range(3):   # the first call captures, the others replay
            out_h.zero_()
            K.lowram_decode_attn_host(lc.handle, 0, cfg.n_layers, q_h, out_h)
            assert torch.equal(out_h, out_d.cpu())
        if step == 0:
            lc.repack(16)
    assert lc.view()[0]["n_ctx"] == cfg.n_ctx + cfg.chunk
    lc.close()
