"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every check is written independently of the oracle's code (torch library routines, closed
forms, brute force, the dense ingredients the test itself packed).  The mutation tests at
the end plant plausible mistakes in the oracle (on the CPU) and show that a pin fails.
"""

import dataclasses
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import lowram_synth as S
import oracle as O

F64 = torch.float64
GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden",
                                     "worked_examples.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        lhs, rhs = line.split("->")
        parts = lhs.split()
        args = dict(p.split("=") for p in parts[1:])
        out[parts[0]] = ({k: int(v) for k, v in args.items()}, float(rhs) if "." in rhs else int(rhs))
    return out


def _mlp_torch(w1, w2, k):
    """Reference predictor with torch's own linear and silu."""
    return F.linear(F.silu(F.linear(k, w1)), w2)


def _attn_torch(q, k, v):
    """Reference attention: torch's scaled_dot_product_attention (math backend, fp64)."""
    return F.scaled_dot_product_attention(q[None, :, None, :].transpose(1, 2),
                                          k[None, None], v[None, None])[0, 0]


def _small_cfg(**kw):
    base = dict(name="pin", batch=2, n_layers=4, group=2, n_kv_heads=2, n_q_heads=4,
                head_dim=8, rank=16, mlp_hidden=12, n_ctx=24, chunk=4, top_k=6, tail_cap=3,
                resid_frac=1.0, dtype="f32", seed=11)
    base.update(kw)
    return S.LowramConfig(**base)


# --------------------------------------------------------------------------- P1 + P3

def check_dense_equivalence(seed=0):
    """Identity basis (r = G*d), coefficients = the G layers' keys side by side, residuals
    on every token (delta = V - f(K)), every chunk selected: the result must be textbook
    attention over the original K, V and the raw tail.  Returns max relative error."""
    cfg = _small_cfg()
    B, L, G, Hkv, N, d, T = cfg.batch, cfg.n_layers, cfg.group, cfg.n_kv_heads, cfg.n_ctx, cfg.head_dim, cfg.tail_cap
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(B, L, Hkv, N, d, dtype=F64, generator=g)
    V = torch.randn(B, L, Hkv, N, d, dtype=F64, generator=g)
    basis, w1, w2 = S.make_weights(cfg, identity_basis=True)
    coeff = torch.stack([torch.cat([K[:, grp * G + li] for li in range(G)], dim=-1)
                         for grp in range(L // G)], dim=1)           # [B][L/G][Hkv][N][G*d]
    pred = torch.stack([torch.stack([_mlp_torch(w1[l, h], w2[l, h], K[:, l, h])
                                     for h in range(Hkv)], dim=1) for l in range(L)], dim=1)
    delta = V - pred
    flags = torch.ones(B, L, Hkv, N, dtype=torch.bool)
    tk = torch.randn(B, L, Hkv, T, d, dtype=F64, generator=g)
    tv = torch.randn(B, L, Hkv, T, d, dtype=F64, generator=g)
    tail_len = torch.tensor([T, 1])
    cache = S.pack_cache(cfg, coeff, basis, w1, w2, flags, delta, tk, tv, tail_len,
                         store_dtype=F64)
    oc = O.OracleCache(S.cache_to_numpy(cache))
    q = torch.randn(L, B, cfg.n_q_heads, d, dtype=F64, generator=g)
    res = O.decode(oc, q.numpy())
    worst = 0.0
    gq = cfg.q_per_kv
    for l in range(L):
        for b in range(B):
            tl = int(tail_len[b])
            for h in range(Hkv):
                keys = torch.cat([K[b, l, h], tk[b, l, h, :tl]])
                vals = torch.cat([V[b, l, h], tv[b, l, h, :tl]])
                ref = _attn_torch(q[l, b, h * gq:(h + 1) * gq], keys, vals)
                got = torch.from_numpy(res["out"][l, b, h * gq:(h + 1) * gq])
                worst = max(worst, float((got - ref).abs().max() / ref.abs().max()))
            assert list(res["sel"][l, b, 0]) == list(range(cfg.n_chunks))
    return worst


def test_p1_identity_basis_reproduces_dense_attention():
    assert check_dense_equivalence() < 1e-12


def check_residuals_restore_values(seed=1):
    """With a residual on every token (delta = V - f(khat)), vhat + delta = V."""
    cfg = _small_cfg(rank=8)
    g = torch.Generator().manual_seed(seed)
    basis, w1, w2 = S.make_weights(cfg)
    a = torch.randn(16, cfg.rank, dtype=F64, generator=g)
    khat = a @ basis[1, 0]                          # torch's own matmul
    V = torch.randn(16, cfg.head_dim, dtype=F64, generator=g)
    delta = V - _mlp_torch(w1[1, 0], w2[1, 0], khat)
    got = O.rebuild_values(O.rebuild_keys(a.numpy(), np.ones(16), basis[1, 0].numpy()),
                           w1[1, 0].numpy(), w2[1, 0].numpy(), np.arange(16),
                           delta.numpy(), np.ones(16))
    return float(np.abs(got - V.numpy()).max())


def test_p3_residuals_on_every_token_restore_values():
    assert check_residuals_restore_values() < 1e-12


# ------------------------------------------------------------------------------- P2

def _random_cache(cfg, seed, store_dtype=F64):
    """Dense ingredients drawn here (the reference below uses them directly) and packed."""
    B, L, G, Hkv, N, d, r, T = (cfg.batch, cfg.n_layers, cfg.group, cfg.n_kv_heads, cfg.n_ctx,
                                cfg.head_dim, cfg.rank, cfg.tail_cap)
    g = torch.Generator().manual_seed(seed)
    basis, w1, w2 = S.make_weights(cfg)
    coeff = torch.randn(B, L // G, Hkv, N, r, dtype=F64, generator=g) / math.sqrt(r) * 3
    flags = torch.rand(B, L, Hkv, N, generator=g) < 0.4
    delta = 0.3 * torch.randn(B, L, Hkv, N, d, dtype=F64, generator=g)
    tk = torch.randn(B, L, Hkv, T, d, dtype=F64, generator=g)
    tv = torch.randn(B, L, Hkv, T, d, dtype=F64, generator=g)
    tail_len = torch.randint(0, T + 1, (B,), generator=g)
    slot = None
    if cfg.evict_frac > 0:
        nC = cfg.n_chunks
        slot = torch.empty(B, L // G, Hkv, nC, dtype=torch.int16)
        for b in range(B):
            for grp in range(L // G):
                for h in range(Hkv):
                    perm = torch.randperm(nC, generator=g)
                    dead = torch.zeros(nC, dtype=torch.bool)
                    dead[perm[:cfg.n_evicted]] = True
                    sl = torch.cumsum((~dead).long(), 0) - 1
                    sl[dead] = -1
                    slot[b, grp, h] = sl.to(torch.int16)
    cache = S.pack_cache(cfg, coeff, basis, w1, w2, flags, delta, tk, tv, tail_len, slot=slot,
                         store_dtype=store_dtype)
    return cache, dict(coeff=coeff, basis=basis, w1=w1, w2=w2, flags=flags, delta=delta,
                       tk=tk, tv=tv, tail_len=tail_len)


def check_select_all_is_full_attention(cfg, seed=2):
    """k = number of live chunks: the output must equal attention over every live rebuilt
    token (no selection step) plus the tail, computed here from the dense ingredients."""
    cache, ing = _random_cache(cfg, seed, store_dtype=F64 if cfg.store == "native" else None)
    oc = O.OracleCache(S.cache_to_numpy(cache))
    g = torch.Generator().manual_seed(seed + 100)
    q = torch.randn(cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.head_dim, dtype=F64, generator=g)
    res = O.decode(oc, q.numpy())
    C, gq = cfg.chunk, cfg.q_per_kv
    worst = 0.0
    for l in range(cfg.n_layers):
        grp = l // cfg.group
        for b in range(cfg.batch):
            tl = int(ing["tail_len"][b])
            for h in range(cfg.n_kv_heads):
                slot = cache.slot[b, grp, h].long()
                live = torch.nonzero(slot >= 0).flatten()
                tok = (live[:, None] * C + torch.arange(C)).flatten()
                if cfg.store == "int8":   # dequantise the stored rows here
                    rows = cache.coeff[b, grp, h].double() * cache.coeff_scale[b, grp, h].double()[:, None]
                    delta = None
                else:
                    rows = ing["coeff"][b, grp, h, tok]
                khat = rows @ cache.basis[l, h].double()
                vhat = _mlp_torch(cache.w1[l, h].double(), cache.w2[l, h].double(), khat)
                fl = ing["flags"][b, l, h, tok]
                if cfg.store == "int8":
                    p0 = int(cache.res_ptr[b, l, h, 0])
                    p1 = int(cache.res_ptr[b, l, h, -1])
                    dq = cache.res_val[p0:p1].double() * cache.res_scale[p0:p1].double()[:, None]
                    vhat[fl] += dq
                else:
                    vhat[fl] += ing["delta"][b, l, h, tok][fl]
                keys = torch.cat([khat, cache.tail_k[b, l, h, :tl].double()])
                vals = torch.cat([vhat, cache.tail_v[b, l, h, :tl].double()])
                ref = _attn_torch(q[l, b, h * gq:(h + 1) * gq], keys, vals)
                got = torch.from_numpy(res["out"][l, b, h * gq:(h + 1) * gq])
                worst = max(worst, float((got - ref).abs().max() / ref.abs().max()))
                assert list(res["sel"][l, b, h]) == live.tolist()
    return worst


def test_p2_select_all_equals_full_attention():
    cfg = _small_cfg(rank=8, resid_frac=0.4, top_k=6)
    assert check_select_all_is_full_attention(cfg) < 1e-12


def test_p2_select_all_with_eviction_and_int8():
    cfg = _small_cfg(rank=8, resid_frac=0.4, dtype="bf16", store="int8", evict_frac=0.5,
                     n_ctx=32, top_k=4)
    assert check_select_all_is_full_attention(cfg, seed=5) < 1e-12


# ------------------------------------------------------------------------------- P4

def test_p4_dense_kv_bytes_worked_example():
    args, want = _golden()["dense_kv_bytes"]
    got = O.dense_kv_bytes(args["L"], args["Hkv"], args["d"], args["N"], args["s"], args["B"])
    assert got == want == 16 * 2**30


def test_p4_low_rank_saving_worked_example():
    args, want = _golden()["low_rank_saving"]
    cfg = dict(batch=1, n_layers=1, group=1, n_kv_heads=1, head_dim=args["d"], rank=args["r"],
               mlp_hidden=1, n_ctx=1024, chunk=128, tail_cap=0, dtype="bf16", store="native")
    nb = O.compressed_bytes(cfg, 0)
    key_dense = nb["dense_equiv"] / 2          # keys are half of M_KV
    assert 1 - nb["coeff"] / key_dense == pytest.approx(want, abs=0)


@pytest.mark.parametrize("name", ["tiny_f32", "mistral7b_group_bf16"])
def test_p7_compressed_bytes_match_storage(name):
    cfg = S.CONFIGS[name]
    c = S.make_cache(cfg)
    nb = O.compressed_bytes(dataclasses.asdict(cfg), c.n_records)
    t = c.tensors()
    nbytes = lambda *ks: sum(t[k].numel() * t[k].element_size() for k in ks if t[k] is not None)
    assert nb["coeff"] == nbytes("coeff", "coeff_scale")
    assert nb["basis"] == nbytes("basis")
    assert nb["predictor"] == nbytes("w1", "w2")
    assert nb["summary"] == nbytes("summary")
    assert nb["residual"] == nbytes("res_val", "res_pos", "res_scale", "res_ptr")
    assert nb["tail"] == nbytes("tail_k", "tail_v", "tail_len")
    assert nb["dense_equiv"] > nb["total"]


def test_p7_compressed_bytes_int8_evict():
    cfg = S.LLAMA_64K_INT8.replace(name="x", batch=1, n_layers=4, n_kv_heads=2, n_q_heads=8,
                                   n_ctx=4096, top_k=8)
    c = S.make_cache(cfg)
    nb = O.compressed_bytes(dataclasses.asdict(cfg), c.n_records)
    t = c.tensors()
    nbytes = lambda *ks: sum(t[k].numel() * t[k].element_size() for k in ks if t[k] is not None)
    assert nb["coeff"] == nbytes("coeff", "coeff_scale")
    assert nb["residual"] == nbytes("res_val", "res_pos", "res_scale", "res_ptr")
    assert nb["index"] == nbytes("slot")
    assert nb["summary"] == nbytes("summary")
    assert nb["tail"] == nbytes("tail_k", "tail_v", "tail_len")


# ------------------------------------------------------------------------------- P5

def test_p5_top_k_matches_brute_force_with_ties():
    rng = np.random.default_rng(0)
    for trial in range(200):
        nC = int(rng.integers(2, 9))
        s = rng.integers(-3, 4, size=nC).astype(np.float64)      # many exact ties
        dead = rng.random(nC) < 0.3
        s[dead] = -np.inf
        live = int(np.isfinite(s).sum())
        if live == 0:
            continue
        k = int(rng.integers(1, live + 1))
        got, margin = O.select_top_k(s, k)
        assert list(got) == list(O.brute_force_top_k(s, k))
        srt = np.sort(s[np.isfinite(s)])[::-1]
        want_margin = srt[k - 1] - srt[k] if k < live else math.inf
        assert margin == want_margin


def test_p5_softmax_without_max_shift_agrees():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(3, 16, dtype=F64, generator=g)
    k = torch.randn(40, 16, dtype=F64, generator=g)
    v = torch.randn(40, 16, dtype=F64, generator=g)
    got = O.attend(q.numpy(), k.numpy(), v.numpy())
    # naive: exponentiate the raw logits, no shift
    e = [[math.exp(sum(q[j, i].item() * k[t, i].item() for i in range(16)) / 4.0)
          for t in range(40)] for j in range(3)]
    for j in range(3):
        z = sum(e[j])
        for i in range(16):
            ref = sum(e[j][t] * v[t, i].item() for t in range(40)) / z
            assert abs(got[j, i] - ref) < 1e-13


def test_attention_matches_torch_sdpa():
    g = torch.Generator().manual_seed(4)
    q = torch.randn(4, 32, dtype=F64, generator=g) * 3
    k = torch.randn(77, 32, dtype=F64, generator=g)
    v = torch.randn(77, 32, dtype=F64, generator=g)
    got = torch.from_numpy(O.attend(q.numpy(), k.numpy(), v.numpy()))
    assert (got - _attn_torch(q, k, v)).abs().max() < 1e-13


def test_predictor_matches_torch_linear_silu():
    g = torch.Generator().manual_seed(5)
    w1 = torch.randn(24, 16, dtype=F64, generator=g)
    w2 = torch.randn(16, 24, dtype=F64, generator=g)
    k = torch.randn(50, 16, dtype=F64, generator=g) * 2
    got = torch.from_numpy(O.predict_values(w1.numpy(), w2.numpy(), k.numpy()))
    assert (got - _mlp_torch(w1, w2, k)).abs().max() < 1e-12
    x = torch.linspace(-30, 30, 121, dtype=F64)
    assert (torch.from_numpy(O.silu(x.numpy())) - F.silu(x)).abs().max() < 1e-14


def test_key_rebuild_identity_basis_and_scale():
    g = torch.Generator().manual_seed(6)
    a = torch.randn(10, 12, dtype=F64, generator=g)
    eye = torch.eye(12, dtype=F64)
    # identity basis slices return the coefficient columns of the layer
    for li in range(3):
        bl = eye[:, li * 4:(li + 1) * 4]
        got = O.rebuild_keys(a.numpy(), np.ones(10), bl.numpy())
        assert np.array_equal(got, a[:, li * 4:(li + 1) * 4].numpy())
    sig = torch.rand(10, dtype=F64, generator=g)
    bl = torch.randn(12, 5, dtype=F64, generator=g)
    got = torch.from_numpy(O.rebuild_keys(a.numpy(), sig.numpy(), bl.numpy()))
    assert (got - torch.diag(sig) @ torch.matmul(a, bl)).abs().max() < 1e-13


def test_chunk_score_is_mean_rebuilt_key_score():
    """Internal pin of the score reading (parity unpinned against the pages): scoring with
    the stored mean coefficient row equals scoring with the mean of the chunk's rebuilt
    keys computed here."""
    cfg = _small_cfg(rank=8, resid_frac=0.4)
    cache, ing = _random_cache(cfg, seed=7)
    oc = O.OracleCache(S.cache_to_numpy(cache))
    g = torch.Generator().manual_seed(8)
    for l in range(cfg.n_layers):
        q = torch.randn(cfg.q_per_kv, cfg.head_dim, dtype=F64, generator=g)
        b, h, grp = 1, 1, l // cfg.group
        s = O.chunk_scores(q.numpy(), oc.summary[b, grp, h], oc.basis[l, h], oc.slot[b, grp, h])
        for c in range(cfg.n_chunks):
            khat = ing["coeff"][b, grp, h, c * cfg.chunk:(c + 1) * cfg.chunk] @ ing["basis"][l, h]
            want = float(q.sum(0) @ khat.mean(0)) / math.sqrt(cfg.head_dim)
            assert abs(s[c] - want) < 1e-12


# ------------------------------------------------------------------------------- P8

@pytest.mark.parametrize("name", ["tiny_f32", "int8_evict"])
def test_p8_rewrites_equal_literal_form(name):
    if name == "tiny_f32":
        cfg = S.TINY_F32
    else:
        cfg = S.LLAMA_64K_INT8.replace(name="x", batch=1, n_layers=4, n_kv_heads=2, n_q_heads=8,
                                       n_ctx=2048, top_k=6, chunk=64)
    c = S.make_cache(cfg)
    q = S.make_queries(c).float().double().numpy()
    oc = O.OracleCache(S.cache_to_numpy(c))
    for l in range(cfg.n_layers):
        for h in range(cfg.n_kv_heads):
            qh = q[l, 0, h * cfg.q_per_kv:(h + 1) * cfg.q_per_kv]
            a = O.decode_unit(oc, 0, l, h, qh)
            b = O.decode_unit_rewritten(oc, 0, l, h, qh)
            assert list(a["sel"]) == list(b["sel"])
            fin = np.isfinite(a["scores"])
            assert np.abs(a["scores"][fin] - b["scores"][fin]).max() < 1e-14
            assert np.abs(a["out"] - b["out"]).max() <= 1e-12 * np.abs(a["out"]).max()


# ------------------------------------------------------------- planted-mistake checks

def test_mutation_dropped_residuals_fail_p1(monkeypatch):
    orig = O.rebuild_values
    monkeypatch.setattr(O, "rebuild_values",
                        lambda k, w1, w2, pos, val, sc: orig(k, w1, w2, pos[:0], val[:0], sc[:0]))
    assert check_dense_equivalence() > 1e-3


def test_mutation_wrong_softmax_scale_fails_sdpa_pin(monkeypatch):
    def bad_attend(q, k, v):
        lg = q @ k.T / q.shape[-1]
        p = np.exp(lg - lg.max(axis=1, keepdims=True))
        return (p @ v) / p.sum(axis=1, keepdims=True)
    monkeypatch.setattr(O, "attend", bad_attend)
    assert check_dense_equivalence() > 1e-3


def test_mutation_transposed_basis_fails_p2(monkeypatch):
    orig = O.rebuild_keys
    monkeypatch.setattr(O, "rebuild_keys", lambda a, s, bl: orig(a, s, bl.T.copy()))
    cfg = _small_cfg(rank=8, head_dim=8, resid_frac=0.4)
    assert check_select_all_is_full_attention(cfg) > 1e-3


def test_mutation_silu_sign_fails_p3(monkeypatch):
    monkeypatch.setattr(O, "silu", lambda x: x / (1.0 + np.exp(x)))
    assert check_residuals_restore_values() > 1e-3


def test_mutation_tie_to_higher_id_fails_p5(monkeypatch):
    def bad(scores, k):
        live = [c for c in range(scores.shape[0]) if np.isfinite(scores[c])]
        order = sorted(live, key=lambda c: (-scores[c], -c))
        return np.array(sorted(order[:k])), 0.0
    s = np.array([1.0, 2.0, 1.0, 0.0])
    assert list(bad(s, 2)[0]) != list(O.brute_force_top_k(s, 2))
