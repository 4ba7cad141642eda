"""Parity of the CUDA path (called through the C ABI) with the fp64 oracle.

Small workloads are generated on the CPU and checked on every unit; the full-size
workloads are generated on the GPU and checked on a seeded sample of units.
"""

import numpy as np
import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
from parity_utils import check, sample_units

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(cache, q, path=K.PATH_AUTO, layer0=0):
    lc = K.LowramCache.from_synth(cache.to(DEV))
    qd = q.to(DEV)
    out, sel = lc.decode(qd, sel=True, layer0=layer0, path=path)
    scores, sel2 = lc.select(qd, layer0=layer0)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel2)
    assert lc.validate() == 0
    launched_path = lc.last_path
    lc.close()
    return out, sel, scores, launched_path


def _oracle(cache):
    return O.OracleCache(S.cache_to_numpy(cache))


def _small(name, **kw):
    return S.CONFIGS[name].replace(name=name + "_edge", **kw)


# ------------------------------------------------------------------ small, every unit

@pytest.mark.parametrize("path", [K.PATH_AUTO, K.PATH_SIMT])
def test_tiny_f32_every_unit(path):
    cfg = S.TINY_F32
    cache = S.make_cache(cfg)
    q = S.make_queries(cache)
    out, sel, scores, p = _run(cache, q, path)
    assert p == K.PATH_SIMT
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


ALL_PATHS = [K.PATH_AUTO, K.PATH_SIMT, K.PATH_TC]


@pytest.mark.parametrize("path", ALL_PATHS)
def test_mistral_group_bf16_every_unit(path):
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg)
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q, path)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


@pytest.mark.parametrize("path", ALL_PATHS)
def test_sharp_queries_strict_selection(path):
    """Peaky softmax and well-separated chunk scores: the exact-selection rule applies."""
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg)
    q = S.make_queries(cache, q_scale=40.0)
    out, sel, scores, _ = _run(cache, q, path)
    res = check(cfg, _oracle(cache), q, out, sel, scores=scores)
    assert res["strict_selection_units"] >= res["units"] // 2


@pytest.mark.parametrize("path", ALL_PATHS)
def test_ragged_tail_select_all_full_residuals(path):
    cfg = _small("mistral7b_group_bf16", batch=3, n_ctx=1024, top_k=16, resid_frac=1.0,
                 tail_cap=64)
    cache = S.make_cache(cfg, tail_len=[0, 37, 64])
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q, path)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)
    assert (sel.cpu() == torch.arange(16, dtype=torch.int32)).all()


@pytest.mark.parametrize("path", ALL_PATHS)
def test_top1_and_no_residuals(path):
    cfg = _small("mistral7b_group_bf16", n_ctx=2048, top_k=1, resid_frac=0.0)
    cache = S.make_cache(cfg)
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q, path)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


@pytest.mark.parametrize("path", ALL_PATHS)
def test_tail_longer_than_block_and_many_units(path):
    """Four sequences with the 32K shape cut to 8K context: 64 units x 32 chunks spread over
    every SM, units straddling CTA ranges, tails of 128, 0, 1 and 77 tokens."""
    cfg = S.LLAMA_32K.replace(name="llama_8k", n_ctx=8192, n_layers=4, top_k=32)
    cache = S.make_cache(cfg, tail_len=[128, 0, 1, 77])
    q = S.make_queries(cache)
    out, sel, scores, p = _run(cache, q, path)
    if path == K.PATH_TC:
        assert p == K.PATH_TC
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


def test_auto_picks_tensor_cores_for_bf16():
    cache = S.make_cache(S.MISTRAL_GROUP)
    q = S.make_queries(cache)
    _, _, _, p = _run(cache, q, K.PATH_AUTO)
    assert p == K.PATH_TC


def test_odd_shapes_f32():
    cfg = S.LowramConfig(name="odd", batch=2, n_layers=3, group=3, n_kv_heads=2, n_q_heads=6,
                         head_dim=40, rank=24, mlp_hidden=96, n_ctx=480, chunk=48, top_k=3,
                         tail_cap=19, resid_frac=0.3, dtype="f32", seed=77)
    cache = S.make_cache(cfg, tail_len=[19, 5])
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


@pytest.mark.parametrize("path", [K.PATH_AUTO, K.PATH_SIMT])
def test_int8_eviction_small_every_unit(path):
    cfg = S.LLAMA_64K_INT8.replace(name="int8_small", batch=2, n_layers=4, n_kv_heads=2,
                                   n_q_heads=8, n_ctx=8192, top_k=8)
    cache = S.make_cache(cfg, tail_len=[128, 77])
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q, path)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


@pytest.mark.parametrize("rank,resid_frac", [(64, 0.125), (128, 0.4)])
def test_int8_rank_and_residual_overflow(rank, resid_frac):
    """int8 rows at both ranks; at 40 % flagged tokens most chunks hold more residual
    records than one residual tile, so the records past it take the overflow route."""
    cfg = S.LLAMA_64K_INT8.replace(name=f"int8_r{rank}", batch=1, n_layers=4, n_kv_heads=2,
                                   n_q_heads=8, n_ctx=8192, rank=rank, resid_frac=resid_frac,
                                   top_k=16)
    cache = S.make_cache(cfg, tail_len=[33])
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


def test_int8_eviction_select_all_live():
    cfg = S.LLAMA_64K_INT8.replace(name="int8_all", batch=1, n_layers=4, n_kv_heads=2,
                                   n_q_heads=8, n_ctx=4096, top_k=16)
    cache = S.make_cache(cfg)
    q = S.make_queries(cache)
    out, sel, scores, _ = _run(cache, q)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)


def test_identity_basis_dense_attention_on_gpu():
    """GPU version of the dense special case: rank = G*d identity basis, residuals on every
    token, every chunk selected; compared with textbook attention computed by torch."""
    cfg = S.LowramConfig(name="dense", batch=1, n_layers=2, group=2, n_kv_heads=1, n_q_heads=2,
                         head_dim=32, rank=64, mlp_hidden=48, n_ctx=256, chunk=32, top_k=8,
                         tail_cap=16, resid_frac=1.0, dtype="f32", seed=5)
    g = torch.Generator().manual_seed(0)
    B, L, N, d, T = 1, 2, 256, 32, 16
    Kd = torch.randn(B, L, 1, N, d, generator=g, dtype=torch.float64)
    Vd = torch.randn(B, L, 1, N, d, generator=g, dtype=torch.float64)
    basis, w1, w2 = S.make_weights(cfg, identity_basis=True)
    coeff = torch.cat([Kd[:, 0], Kd[:, 1]], dim=-1)[:, None]
    pred = torch.stack([torch.nn.functional.linear(torch.nn.functional.silu(
        torch.nn.functional.linear(Kd[:, l, 0], w1[l, 0])), w2[l, 0]) for l in range(L)], dim=1)
    delta = (Vd[:, :, 0] - pred)[:, :, None]
    tk = torch.randn(B, L, 1, T, d, generator=g, dtype=torch.float64)
    tv = torch.randn(B, L, 1, T, d, generator=g, dtype=torch.float64)
    cache = S.pack_cache(cfg, coeff, basis, w1, w2, torch.ones(B, L, 1, N, dtype=torch.bool),
                         delta, tk, tv, torch.tensor([T]))
    q = torch.randn(L, B, 2, d, generator=g).float()
    out, sel, scores, _ = _run(cache, q)
    check(cfg, _oracle(cache), q, out, sel, scores=scores)
    # and directly against attention over the fp32-stored dense keys/values
    for l in range(L):
        keys = torch.cat([Kd[0, l, 0], tk[0, l, 0]]).float().double()
        vals = torch.cat([Vd[0, l, 0], tv[0, l, 0]]).float().double()
        att = torch.softmax(q[l, 0].double() @ keys.T / d ** 0.5, dim=-1) @ vals
        err = (out[l, 0].cpu().double() - att).abs().max() / att.abs().max()
        assert err < 1e-3   # fp32 storage of delta = V - f(K) rounds V by ~1e-7 relative


# ------------------------------------------------------------- full size, sampled units

@pytest.fixture(scope="module")
def llama32k():
    cfg = S.LLAMA_32K
    cache = S.make_cache(cfg, device=DEV)
    return cfg, cache


@pytest.mark.parametrize("path", ALL_PATHS)
def test_llama_32k_all_layers_sampled(llama32k, path):
    cfg, cache = llama32k
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    out, sel = lc.decode(q, sel=True, path=path)
    scores, _ = lc.select(q)
    torch.cuda.synchronize()
    assert lc.validate() == 0
    lc.close()
    oc = _oracle(cache)
    units = sample_units(cfg, cfg.n_layers, 64, seed=1)
    res = check(cfg, oc, q, out, sel, units=units, scores=scores)
    assert res["units"] >= 64


def test_llama_32k_single_layer_call(llama32k):
    cfg, cache = llama32k
    q = S.make_queries(cache, layer0=21, n_layers=1, seed_offset=3)
    lc = K.LowramCache.from_synth(cache)
    out, sel = lc.decode(q, sel=True, layer0=21)
    torch.cuda.synchronize()
    lc.close()
    check(cfg, _oracle(cache), q, out, sel, layer0=21)


def test_llama_32k_batch1_sampled():
    cfg = S.CONFIGS["llama8b_32k_bf16_b1"]
    cache = S.make_cache(cfg, device=DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    out, sel = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    lc.close()
    check(cfg, _oracle(cache), q, out, sel, units=sample_units(cfg, cfg.n_layers, 64, seed=2))


def test_int8_evict_64k_sampled():
    cfg = S.LLAMA_64K_INT8
    cache = S.make_cache(cfg, device=DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    out, sel = lc.decode(q, sel=True)
    scores, _ = lc.select(q)
    torch.cuda.synchronize()
    assert lc.validate() == 0
    lc.close()
    check(cfg, _oracle(cache), q, out, sel, units=sample_units(cfg, cfg.n_layers, 64, seed=3),
          scores=scores)


# ------------------------------------------------------------------------ entry points

def test_host_entry_point_matches_device_call():
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg).to(DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    out_d, sel_d = lc.decode(q, sel=True)
    q_h = q.cpu().pin_memory()
    out_h = torch.empty_like(q_h).pin_memory()
    sel_h = torch.empty(sel_d.shape, dtype=torch.int32).pin_memory()
    K.lowram_decode_attn_host(lc.handle, 0, cfg.n_layers, q_h, out_h, sel_h)
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(sel_h, sel_d.cpu())
    lc.close()


def test_host_entry_point_pinned_and_pageable_across_steps():
    """Consecutive steps through the host entry point, alternating a pinned buffer refilled in
    place and a fresh pageable one: every call matches the device entry point."""
    cfg = S.LLAMA_32K.replace(name="host_q", batch=2, n_layers=4, n_kv_heads=2, n_ctx=1024, top_k=4)
    cache = S.make_cache(cfg, device=DEV)
    steps = S.make_query_steps(cache, 3, 0.0, 1.0)
    lc = K.LowramCache.from_synth(cache)
    q_pin = steps[0].cpu().pin_memory()
    out_h = torch.empty_like(q_pin).pin_memory()
    for t, q in enumerate(steps):
        ref = lc.decode(q)
        torch.cuda.synchronize()
        q_pin.copy_(q.cpu())                   # same pinned buffer, new contents
        K.lowram_decode_attn_host(lc.handle, 0, cfg.n_layers, q_pin, out_h)
        assert torch.equal(out_h, ref.cpu()), t
        q_page = q.cpu().clone()               # pageable
        out_p = torch.empty_like(q_page)
        K.lowram_decode_attn_host(lc.handle, 0, cfg.n_layers, q_page, out_p)
        assert torch.equal(out_p, ref.cpu()), t
    lc.close()


def test_validate_detects_corrupt_tables():
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg)
    bad = cache.to(DEV)
    rp = bad.res_ptr.clone()
    rp[0, 0, 0, 3] = rp[0, 0, 0, 2] - 1       # offsets decreasing
    bad.res_ptr = rp
    lc = K.LowramCache.from_synth(bad)
    assert lc.validate() == 5
    assert lc.validate() == 5                 # tables stay corrupt; the word is re-derived
    lc.close()
    bad = cache.to(DEV)
    tl = bad.tail_len.clone()
    tl[0] = cfg.tail_cap + 1
    bad.tail_len = tl
    lc = K.LowramCache.from_synth(bad)
    assert lc.validate() == 5
    lc.close()


def test_stage_events_and_launch_count():
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg).to(DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    K.lowram_cache_set_stage_events(lc.handle, ev)
    lc.decode(q)
    torch.cuda.synchronize()
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]
    assert all(t >= 0 for t in times)
    assert lc.last_launches == 3
    K.lowram_cache_set_stage_events(lc.handle, None)
    lc.close()


def test_tensor_core_path_rejects_fp32():
    cache = S.make_cache(S.TINY_F32).to(DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    with pytest.raises(K.LowramError) as ei:
        lc.decode(q, path=K.PATH_TC)
    assert ei.value.status == 4
    lc.close()


def test_bad_layer_range_rejected():
    cache = S.make_cache(S.TINY_F32).to(DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    with pytest.raises(K.LowramError) as ei:
        lc.decode(q, layer0=1)          # 2 layers from layer 1 exceeds the cache
    assert ei.value.status == 1
    lc.close()


# (B, L, Hkv, Hq, S, d, q scale): the tensor-core kernel for d = 128 and g in {1,2,4,8,16}
# (ragged last tile, a single partial tile, exact tiles, several trips round the three-stage
# ring, peaked softmax), the CUDA-core kernel otherwise (d = 64, g = 3)
DENSE_CASES = [
    (2, 2, 2, 8, 1000, 128, 0.3),
    (1, 1, 1, 8, 128, 128, 0.3),
    (1, 2, 2, 2, 129, 128, 0.3),
    (1, 1, 1, 16, 517, 128, 0.3),
    (1, 1, 2, 4, 5, 128, 0.3),
    (1, 1, 1, 4, 3000, 128, 0.3),
    (1, 1, 1, 4, 700, 128, 3.0),
    (2, 1, 2, 6, 300, 64, 0.3),
]


@pytest.mark.parametrize("case", DENSE_CASES, ids=lambda c: "x".join(map(str, c[:6])))
def test_dense_baseline_matches_textbook_attention(case):
    """The uncompressed baseline kernel against the oracle's textbook attention."""
    B, L, Hkv, Hq, S_, d, qs = case
    g = torch.Generator().manual_seed(11 + S_)
    k = torch.randn(B, L, Hkv, S_, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, S_, d, generator=g).to(torch.bfloat16)
    q = (torch.randn(L, B, Hq, d, generator=g) * qs).to(torch.bfloat16)
    out = torch.full((L, B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    K.lowram_dense_decode_attn(k.to(DEV), v.to(DEV), q.to(DEV), out)
    torch.cuda.synchronize()
    gq = Hq // Hkv
    for l in range(L):
        for b in range(B):
            for h in range(Hkv):
                ref = O.attend(q[l, b, h * gq:(h + 1) * gq].double().numpy(),
                               k[b, l, h].double().numpy(), v[b, l, h].double().numpy())
                got = out[l, b, h * gq:(h + 1) * gq].cpu().double().numpy()
                # bf16 probabilities and a bf16 output: a few units of 2^-9 relative
                err = np.abs(got - ref).max(axis=1) / np.linalg.norm(ref, axis=1)
                assert np.isfinite(got).all() and err.max() <= 2e-2
