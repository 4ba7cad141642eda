"""Invariants of the seeded input generator (host only)."""

import math

import numpy as np
import pytest
import torch

import lowram_synth as S


def test_basis_rows_orthonormal():
    """B_l B_l^T = I_r ("OjaKV", section 3.1: orthonormal bases)."""
    for name in ("tiny_f32", "mistral7b_group_bf16"):
        cfg = S.CONFIGS[name]
        basis, _, _ = S.make_weights(cfg)
        eye = torch.eye(cfg.rank, dtype=torch.float64)
        gram = basis @ basis.transpose(-1, -2)
        assert (gram - eye).abs().max() < 1e-12


def test_identity_basis_slices():
    cfg = S.TINY_F32.replace(rank=128)
    basis, _, _ = S.make_weights(cfg, identity_basis=True)
    full = torch.cat([basis[0, 0], basis[1, 0]], dim=1)
    assert torch.equal(full, torch.eye(128, dtype=torch.float64))


def test_deterministic():
    a = S.make_cache(S.TINY_F32)
    b = S.make_cache(S.TINY_F32)
    for k, v in a.tensors().items():
        if v is not None:
            assert torch.equal(v, b.tensors()[k]), k


@pytest.mark.parametrize("name", ["tiny_f32", "mistral7b_group_bf16"])
def test_residual_records(name):
    cfg = S.CONFIGS[name]
    c = S.make_cache(cfg)
    ptr = c.res_ptr.long()
    assert (ptr[..., 1:] >= ptr[..., :-1]).all()
    flat = ptr.reshape(-1, cfg.n_live + 1)
    assert (flat[1:, 0] == flat[:-1, -1]).all()           # units are contiguous
    assert int(flat[0, 0]) == 0 and int(flat[-1, -1]) == c.n_records
    per_unit = flat[:, -1] - flat[:, 0]
    assert (per_unit == cfg.n_resid).all()                 # no eviction: ceil(rho*N) each
    pos = c.res_pos.long()
    assert (pos >= 0).all() and (pos < cfg.chunk).all()
    for u in range(flat.shape[0]):
        for s in range(cfg.n_live):
            p = pos[flat[u, s]:flat[u, s + 1]]
            assert (p[1:] > p[:-1]).all()


def test_flags_are_worst_noise_tokens():
    cfg = S.TINY_F32
    c = S.make_cache(cfg)
    for l in range(cfg.n_layers):
        eps = S._draw_eps(cfg, 0, l, "cpu")[0]                 # [N][d]
        nrm = eps.norm(dim=-1)
        p0, p1 = int(c.res_ptr[0, l, 0, 0]), int(c.res_ptr[0, l, 0, -1])
        tok = []
        for s in range(cfg.n_live):
            a, b = int(c.res_ptr[0, l, 0, s]), int(c.res_ptr[0, l, 0, s + 1])
            tok += [s * cfg.chunk + int(x) for x in c.res_pos[a:b]]
        flagged = torch.zeros(cfg.n_ctx, dtype=torch.bool)
        flagged[tok] = True
        assert int(flagged.sum()) == cfg.n_resid
        assert nrm[flagged].min() >= nrm[~flagged].max()
        assert torch.equal(c.res_val[p0:p1], eps[tok].float())


def test_summaries_are_chunk_means():
    cfg = S.MISTRAL_GROUP
    c = S.make_cache(cfg)
    rows = c.coeff.double().view(cfg.batch, cfg.n_groups, cfg.n_kv_heads, cfg.n_live, cfg.chunk, cfg.rank)
    want = rows.mean(dim=4).to(torch.bfloat16)
    assert torch.equal(c.summary, want)


def test_int8_rows_and_eviction():
    cfg = S.LLAMA_64K_INT8.replace(name="x", batch=2, n_layers=4, n_kv_heads=2, n_q_heads=8,
                                   n_ctx=4096, top_k=8)
    c = S.make_cache(cfg)
    slot = c.slot.long()
    assert ((slot >= 0).sum(-1) == cfg.n_live).all()
    for row in slot.reshape(-1, cfg.n_chunks):
        live = row[row >= 0]
        assert torch.equal(live, torch.arange(cfg.n_live))
    assert c.coeff.dtype == torch.int8 and c.coeff.abs().max() <= 127
    assert c.coeff_scale.dtype == torch.float16
    # every row's largest entry quantises to +-127 (scale = max|x|/127)
    assert (c.coeff.abs().amax(-1) >= 126).all()
    flat = c.res_ptr.long().reshape(-1, cfg.n_live + 1)
    assert int(flat[-1, -1]) == c.n_records == c.res_val.shape[0] == c.res_scale.shape[0]
    assert (flat[:, -1] - flat[:, 0] <= cfg.n_resid).all()


def test_quantize_rows_round_trip_bound():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(100, 64, generator=g) * torch.rand(100, 1, generator=g) * 10
    x[3] = 0
    q, s = S.quantize_rows_int8(x)
    deq = q.float() * s.float()[:, None]
    assert (deq - x).abs().max() <= (s.float()[:, None] / 2 * 1.02 + 1e-7).max()
    assert torch.equal(q[3], torch.zeros(64, dtype=torch.int8)) and float(s[3]) == 0


def test_queries_target_chunks():
    cfg = S.MISTRAL_GROUP
    c = S.make_cache(cfg)
    q = S.make_queries(c)
    assert q.shape == (cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.head_dim)
    assert q.dtype == torch.bfloat16
    q2 = S.make_queries(c, layer0=1, n_layers=1)
    assert torch.equal(q2[0], q[1])


def test_select_sequences_keeps_the_oracle_result_of_those_sequences():
    """Slicing a batch down to a few sequences (used to check large batches on sampled
    sequences) changes nothing about those sequences' decode results."""
    import oracle as O
    cfg = S.MISTRAL_GROUP.replace(name="m3", batch=3, n_ctx=1024, top_k=4)
    cache = S.make_cache(cfg, tail_len=[64, 10, 33])
    q = S.make_queries(cache)
    sub = S.select_sequences(cache, [2, 0])
    assert sub.cfg.batch == 2 and sub.n_records == int(sub.res_ptr.max())
    full = O.decode(O.OracleCache(S.cache_to_numpy(cache)), q.double().numpy())["out"]
    part = O.decode(O.OracleCache(S.cache_to_numpy(sub)), q[:, [2, 0]].double().numpy())["out"]
    assert np.array_equal(full[:, [2, 0]], part)
