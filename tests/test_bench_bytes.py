"""The roofline numerator of bench.py (algorithmic bytes of one decode call) against the
per-unit byte count written out here: per unit, the chunk summaries it scores (coefficient
space, r per chunk), the coefficient rows of its k selected chunks, their residual records
(row + position) and k+1 CSR offsets, its raw tail, q and out; per (layer, KV head), the
basis, the folded W1' and W2.  Every unit's rows count, also when several layers of one group
select the same chunk (the formula counts per unit); the once-per-group count is reported
beside it.  CPU only."""

import numpy as np

import bench
import lowram_synth as S

CFG = S.MISTRAL_GROUP.replace(name="bytes", batch=2, n_layers=2, n_kv_heads=2, n_ctx=1024, top_k=4)


def _host(cfg, seed=0):
    B, L, H, nC = cfg.batch, cfg.n_layers, cfg.n_kv_heads, cfg.n_chunks
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 6, size=(B, L, H, nC))
    res_ptr = np.zeros((B, L, H, nC + 1), dtype=np.int64)
    res_ptr[..., 1:] = np.cumsum(counts, axis=-1)
    slot = np.broadcast_to(np.arange(nC), (B, L // cfg.group, H, nC)).copy()
    tail_len = np.array([cfg.tail_cap, cfg.tail_cap // 2])
    return {"res_ptr": res_ptr, "slot": slot, "tail_len": tail_len}, counts


def _expected(cfg, counts, sel, tail_len, shared_rows):
    B, L, H, k, C = cfg.batch, cfg.n_layers, cfg.n_kv_heads, cfg.top_k, cfg.chunk
    d, r, h, g, s = cfg.head_dim, cfg.rank, cfg.mlp_hidden, cfg.q_per_kv, 2
    per_unit = 0
    for l in range(L):
        for b in range(B):
            for hk in range(H):
                per_unit += sum(int(counts[b, l, hk, c]) for c in sel[l, b, hk]) * (d * s + 2)
                per_unit += (k + 1) * 4 + 2 * int(tail_len[b]) * d * s + 2 * g * d * s
    units = B * L * H
    rows = units * k * C * r * s
    summaries = units * cfg.n_live * r * s
    weights = L * H * (r * d + h * r + d * h) * s
    return per_unit + rows + summaries + weights


def test_disjoint_selections_match_the_per_unit_count():
    cfg = CFG
    host, counts = _host(cfg)
    k, L, B, H = cfg.top_k, cfg.n_layers, cfg.batch, cfg.n_kv_heads
    sel = np.zeros((L, B, H, k), dtype=np.int64)
    for l in range(L):
        sel[l] = np.arange(l * k, (l + 1) * k)          # the group's two layers pick disjoint chunks
    ab = bench.algorithmic_bytes(cfg, host, sel, 0, L)
    assert ab["total"] == _expected(cfg, counts, sel, host["tail_len"], shared_rows=False)


def test_rows_chosen_by_a_whole_group_count_per_unit():
    cfg = CFG
    host, counts = _host(cfg, seed=1)
    k, L, B, H = cfg.top_k, cfg.n_layers, cfg.batch, cfg.n_kv_heads
    sel = np.broadcast_to(np.arange(k), (L, B, H, k)).copy()
    ab = bench.algorithmic_bytes(cfg, host, sel, 0, L)
    assert ab["total"] == _expected(cfg, counts, sel, host["tail_len"], shared_rows=True)
    groups = B * (L // cfg.group) * H
    assert ab["unique_coeff"] == groups * k * cfg.chunk * cfg.rank * 2
    assert ab["coeff"] == cfg.group * ab["unique_coeff"]
    # the attend kernel's share: rows, records and offsets, and the folded W1' it reads
    rows = L * B * H * k * cfg.chunk * cfg.rank * 2
    recs = sum(int(counts[b, l, hk, c]) for l in range(L) for b in range(B) for hk in range(H)
               for c in sel[l, b, hk]) * (cfg.head_dim * 2 + 2)
    ptrs = L * B * H * (k + 1) * 4
    w1f = L * H * cfg.mlp_hidden * cfg.rank * 2
    assert ab["attend"] == rows + recs + ptrs + w1f
