"""Pins of the encoder oracle (``oracle.encode``) against closed forms, torch and brute force.

CPU only.  Each pin fixes one step of the encoder as ``oracle/encode.py`` lists them; the
planted-mistake tests check that a plausible error in the oracle fails its pin.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
import oracle.encode as E

CFG = dict(name="enc_pin", batch=1, n_layers=4, group=2, n_kv_heads=2, n_q_heads=4,
           head_dim=32, rank=16, mlp_hidden=32, n_ctx=256, chunk=32, top_k=8, tail_cap=8,
           resid_frac=0.125, dtype="bf16", store="native", evict_frac=0.0, seed=1)


def _orthonormal_rows(rng, r, d):
    q, _ = np.linalg.qr(rng.standard_normal((d, r)))
    return q.T                                    # [r][d], rows orthonormal


def _weights(rng, cfg):
    L, H, d, r, h = cfg["n_layers"], cfg["n_kv_heads"], cfg["head_dim"], cfg["rank"], cfg["mlp_hidden"]
    basis = np.stack([np.stack([_orthonormal_rows(rng, r, d) for _ in range(H)]) for _ in range(L)])
    w1 = rng.standard_normal((L, H, h, d)) / np.sqrt(d)
    w2 = rng.standard_normal((L, H, d, h)) / np.sqrt(h)
    return basis, w1, w2


def _planted(rng, cfg, basis, noise=0.0):
    """keys K_l = A B_l (+ noise) with A shared by the layers of a group; values random."""
    B, L, G, H, N = cfg["batch"], cfg["n_layers"], cfg["group"], cfg["n_kv_heads"], cfg["n_ctx"]
    r, d = cfg["rank"], cfg["head_dim"]
    A = rng.standard_normal((B, L // G, H, N, r))
    K = np.zeros((B, L, H, N, d))
    for l in range(L):
        K[:, l] = np.einsum("bhnr,hrd->bhnd", A[:, l // G], basis[l])
    K += noise * rng.standard_normal(K.shape)
    V = 0.3 * rng.standard_normal((B, L, H, N, d))
    return A, K, V


# ------------------------------------------------------------------ step 1: coefficients

def test_planted_coefficients_recovered_exactly():
    rng = np.random.default_rng(0)
    basis, _, _ = _weights(rng, CFG)
    A, K, _ = _planted(rng, CFG, basis)
    for grp in range(CFG["n_layers"] // CFG["group"]):
        ls = slice(grp * CFG["group"], (grp + 1) * CFG["group"])
        for h in range(CFG["n_kv_heads"]):
            a = E.lstsq_coefficients(K[0, ls, h], basis[ls, h])
            np.testing.assert_allclose(a, A[0, grp, h], atol=1e-11)


def test_non_orthonormal_basis_still_least_squares():
    """The normal equations hold for any full-rank stacked basis (not only orthonormal)."""
    rng = np.random.default_rng(1)
    G, N, r, d = 3, 64, 8, 16
    bases = rng.standard_normal((G, r, d))
    keys = rng.standard_normal((G, N, d))
    a = E.lstsq_coefficients(keys, bases)
    stacked_k = np.concatenate(list(keys), axis=1)            # [N][G*d]
    stacked_b = np.concatenate(list(bases), axis=1)           # [r][G*d]
    ref, *_ = np.linalg.lstsq(stacked_b.T, stacked_k.T, rcond=None)   # library least squares
    np.testing.assert_allclose(a, ref.T, atol=1e-10)


def test_orthonormal_rows_reduce_to_group_average_of_projections():
    """With B_l B_l^T = I the solution is the closed form (1/G) sum_l k_l B_l^T."""
    rng = np.random.default_rng(2)
    basis, _, _ = _weights(rng, CFG)
    _, K, _ = _planted(rng, CFG, basis, noise=0.05)
    ls = slice(0, CFG["group"])
    a = E.lstsq_coefficients(K[0, ls, 0], basis[ls, 0])
    closed = sum(K[0, l, 0] @ basis[l, 0].T for l in range(CFG["group"])) / CFG["group"]
    np.testing.assert_allclose(a, closed, atol=1e-12)
    # residual of the fit is orthogonal to the stacked basis (normal equations)
    res = sum((K[0, l, 0] - a @ basis[l, 0]) @ basis[l, 0].T for l in range(CFG["group"]))
    assert np.abs(res).max() < 1e-10


# --------------------------------------------------------------- step 2: storage rounding

def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 3.14159, 0.0])
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view("uint16")
    np.testing.assert_array_equal(E.round_bf16_bits(x), ref)


def test_int8_rows():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((50, 24))
    x[7] = 0.0
    q, s = E.quantize_rows_int8(x)
    sf = s.astype(np.float64)
    assert sf[7] == 0 and np.all(q[7] == 0)
    live = sf > 0
    err = np.abs(x - q.astype(np.float64) * sf[:, None])[live]
    assert np.all(err <= (sf[live, None] * 0.5 + 1e-3 * sf[live, None]))
    amax_idx = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(q[live, amax_idx[live]]) >= 126)   # the largest element maps to ~127


# ------------------------------------------------------------------- step 5: residual flags

def test_flags_are_brute_force_top_n_with_low_index_ties():
    norms = np.array([0.5, 2.0, 2.0, 1.0, 2.0, 0.1, 1.0, 3.0])
    got = E.flag_worst(norms, 4)
    order = torch.sort(torch.tensor(norms), descending=True, stable=True).indices[:4]
    ref = np.zeros(8, dtype=bool)
    ref[order.numpy()] = True
    np.testing.assert_array_equal(got, ref)
    assert got[1] and got[2] and got[4] and got[7] and not got[3]


# ------------------------------------------------------------------ full encoder vs torch

def _encode(cfg, seed=4, noise=0.02, n_res=None):
    rng = np.random.default_rng(seed)
    basis, w1, w2 = _weights(rng, cfg)
    _, K, V = _planted(rng, cfg, basis, noise=noise)
    n_res = cfg["n_ctx"] // 8 if n_res is None else n_res
    return E.encode(cfg, K, V, basis, w1, w2, n_res), K, V, basis, w1, w2


def test_residuals_match_torch_predictor():
    npc, K, V, basis, w1, w2 = _encode(CFG)
    stored = npc["extra"]["stored_coeff"]
    for l in range(CFG["n_layers"]):
        for h in range(CFG["n_kv_heads"]):
            khat = torch.tensor(stored[0, l // CFG["group"], h]) @ torch.tensor(basis[l, h])
            vhat = F.linear(F.silu(F.linear(khat, torch.tensor(w1[l, h]))), torch.tensor(w2[l, h]))
            delta = torch.tensor(V[0, l, h]) - vhat
            np.testing.assert_allclose(npc["extra"]["norms"][0, l, h], delta.norm(dim=1).numpy(), atol=1e-10)


def test_summaries_are_chunk_means_of_stored_rows():
    npc, *_ = _encode(CFG)
    stored = torch.tensor(npc["extra"]["stored_coeff"])
    C = CFG["chunk"]
    mean = stored.view(*stored.shape[:3], -1, C, stored.shape[-1]).mean(dim=4)
    got = O._bf16_bits_to_f64(npc["summary"])
    np.testing.assert_allclose(got, mean.numpy(), rtol=2 ** -8, atol=1e-6)


def test_records_are_csr_of_flags():
    npc, *_ = _encode(CFG)
    C, nC = CFG["chunk"], CFG["n_ctx"] // CFG["chunk"]
    flags = npc["extra"]["flags"]
    rp, pos = npc["res_ptr"].astype(np.int64), npc["res_pos"].astype(np.int64)
    for l in range(CFG["n_layers"]):
        for h in range(CFG["n_kv_heads"]):
            f = flags[0, l, h]
            for c in range(nC):
                seg = pos[rp[0, l, h, c]:rp[0, l, h, c + 1]]
                np.testing.assert_array_equal(seg, np.nonzero(f[c * C:(c + 1) * C])[0])
    assert rp.ravel()[-1] == pos.shape[0] == flags.sum()


def test_round_trip_all_residuals_is_dense_attention():
    """Every token flagged: decode(encode(K, V)) = attention over (Khat, V), up to the bf16
    rounding of the stored residuals (|err| <= 2^-9 |delta| per element)."""
    cfg = dict(CFG, top_k=CFG["n_ctx"] // CFG["chunk"])
    npc, K, V, basis, w1, w2 = _encode(cfg, n_res=cfg["n_ctx"])
    oc = O.OracleCache(npc)
    rng = np.random.default_rng(9)
    L, B, Hq, d, G = cfg["n_layers"], cfg["batch"], cfg["n_q_heads"], cfg["head_dim"], cfg["group"]
    q = rng.standard_normal((L, B, Hq, d)) / np.sqrt(d)
    out = O.decode(oc, q)["out"]
    g = Hq // cfg["n_kv_heads"]
    stored = npc["extra"]["stored_coeff"]
    for l in range(L):
        for h in range(cfg["n_kv_heads"]):
            khat = torch.tensor(stored[0, l // G, h] @ basis[l, h])
            qq = torch.tensor(q[l, 0, h * g:(h + 1) * g])
            ref = F.scaled_dot_product_attention(qq[None], khat[None], torch.tensor(V[0, l, h])[None])[0]
            bound = 2 ** -8 * np.abs(V[0, l, h]).max() + 1e-9
            assert np.abs(out[l, 0, h * g:(h + 1) * g] - ref.numpy()).max() <= bound


# ------------------------------------------------------------------- planted mistakes

def test_planted_mistake_single_layer_basis_fails_recovery(monkeypatch):
    def wrong(keys, bases):                      # fits layer 0 only
        return keys[0] @ bases[0].T
    rng = np.random.default_rng(5)
    basis, _, _ = _weights(rng, CFG)
    A, K, _ = _planted(rng, CFG, basis, noise=0.1)
    ls = slice(0, CFG["group"])
    good = E.lstsq_coefficients(K[0, ls, 0], basis[ls, 0])
    bad = wrong(K[0, ls, 0], basis[ls, 0])
    # the pin's tolerance separates them: the right fit averages the noise of G layers
    assert np.abs(good - A[0, 0, 0]).max() < np.abs(bad - A[0, 0, 0]).max()
    with pytest.raises(AssertionError):
        np.testing.assert_allclose(bad, sum(K[0, l, 0] @ basis[l, 0].T for l in range(CFG["group"])) / CFG["group"],
                                   atol=1e-12)


def test_planted_mistake_high_index_ties_fails_flags(monkeypatch):
    def wrong(norms, n_res):                     # ties to the higher index
        order = np.lexsort((-np.arange(norms.shape[0]), -norms))
        m = np.zeros(norms.shape[0], dtype=bool)
        m[order[:n_res]] = True
        return m
    norms = np.array([0.5, 2.0, 2.0, 1.0, 2.0, 0.1])
    order = torch.sort(torch.tensor(norms), descending=True, stable=True).indices[:2]
    ref = np.zeros(6, dtype=bool)
    ref[order.numpy()] = True
    assert not np.array_equal(wrong(norms, 2), ref)
    np.testing.assert_array_equal(E.flag_worst(norms, 2), ref)


@pytest.mark.parametrize("store", ["native", "int8"])
def test_given_stored_coefficients_reproduce_steps_3_to_6(store):
    """Feeding the encoder's own stored coefficients back reproduces every later output."""
    cfg = dict(CFG, store=store)
    rng = np.random.default_rng(11)
    basis, w1, w2 = _weights(rng, cfg)
    _, K, V = _planted(rng, cfg, basis, noise=0.02)
    a = E.encode(cfg, K, V, basis, w1, w2, 32)
    b = E.encode(cfg, K, V, basis, w1, w2, 32, given=(a["coeff"], a["coeff_scale"]))
    for k in ("coeff", "summary", "res_ptr", "res_pos", "res_val"):
        np.testing.assert_array_equal(a[k], b[k])
    np.testing.assert_array_equal(a["extra"]["flags"], b["extra"]["flags"])
