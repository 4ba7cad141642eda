"""Parity of the CUDA encoder (through the C ABI) with the fp64 encoder oracle.

Stored coefficients agree to the tolerance the bf16-rounded basis implies, with no
systematic bias (see _check_encode); summaries to one bf16 unit.  Residual norms: each
token's norm, read back from the kernel's workspace, must lie within NORM_RTOL of the
oracle's (the roundings behind that bound are listed at NORM_RTOL).  Flags then agree except
on tokens whose norm is within the two tokens' bounds of the oracle's threshold, the only
ones a norm error of that size can move across it.  Residual rows agree to their bf16
(int8) rounding.
The encoded cache then decodes on the GPU in parity with the decode oracle.
"""

import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
import oracle.encode as E
from parity_utils import check

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _weights_bf16(cfg):
    basis, w1, w2 = S.make_weights(cfg)
    return [t.to(torch.bfloat16) for t in (basis, w1, w2)]


def _f64(t):
    return t.float().double().cpu().numpy()


def _gpu_codes(g, cfg):
    """The GPU's stored coefficients in the oracle's storage form (bits / codes, scales)."""
    if cfg.store == "int8":
        return (g["coeff"].cpu().numpy(), g["coeff_scale"].cpu().numpy())
    return (g["coeff"].cpu().view(torch.int16).numpy().view(np.uint16), None)


# Residual norms: the kernels fold W1' = W1 B_l^T once and round it (bf16 for the tensor-core
# predictor: unit roundoff 2^-9), and the tensor-core predictor also rounds u = pre/2 and H
# to fp16 (2^-11) around the hardware tanh.  Each pre-activation is then off by a sum of 128
# independent roundings, and a residual norm by a sum over 128 dimensions of those, so the
# relative norm error concentrates far below the 2^-9 of a single rounding: a numpy model of
# exactly these roundings on the 32K workload's weights puts it at 8e-5 (median) and 5.8e-4
# (largest of 8192 tokens), with the W1' rounding alone at 5.8e-4 and the fp16 H alone at
# 1.2e-4.  For int8 stores with C = 128 the tensor-core predictor takes W1'/2 and the
# dequantised rows sigma*a in fp16 (unit roundoff 2^-11, four times finer); with C = 64 the
# CUDA-core predictor keeps everything in fp32.  The bound asserted token by token, where the
# kernel's norms can be read back:
NORM_RTOL = 1e-3
NORM_ATOL = 1e-6


def _gpu_norms(g, cfg):
    """The kernel's residual norms [B][L][Hkv][N] (fp32), read from the workspace that
    ``lowram_encode`` was given (pieces 256-byte aligned: fp32 W1', bf16 W1'/2, fp16 W2,
    norms, flags, error word)."""
    al = lambda x: (x + 255) // 256 * 256
    lh = cfg.n_layers * cfg.n_kv_heads
    units = cfg.batch * lh
    off = al(lh * cfg.rank * cfg.mlp_hidden * 4) + al(lh * cfg.mlp_hidden * cfg.rank * 2) \
        + al(lh * cfg.head_dim * cfg.mlp_hidden * 2)
    ws = g["_workspace"]
    n = ws[off:off + units * cfg.n_ctx * 4].view(torch.float32)
    return n.view(cfg.batch, cfg.n_layers, cfg.n_kv_heads, cfg.n_ctx).double().cpu().numpy()


def _encode_both(cfg, n_res, device_kv="cpu"):
    """GPU encode, the oracle's own encode, and the oracle's steps 3-6 on the GPU's stored
    coefficients."""
    Kd, Vd = S.make_dense_kv(cfg, device=device_kv)
    basis, w1, w2 = _weights_bf16(cfg)
    g = K.lowram_encode(cfg, n_res, Kd.to(DEV).contiguous(), Vd.to(DEV).contiguous(),
                        basis.to(DEV).contiguous(), w1.to(DEV).contiguous(), w2.to(DEV).contiguous())
    torch.cuda.synchronize()
    args = (dataclasses.asdict(cfg), _f64(Kd), _f64(Vd), _f64(basis), _f64(w1), _f64(w2), n_res)
    o = E.encode(*args)
    og = E.encode(*args, given=_gpu_codes(g, cfg))
    return g, o, og


def _stored_coeff(g, cfg):
    if cfg.store == "int8":
        return g["coeff"].double() * g["coeff_scale"].double().unsqueeze(-1)
    return g["coeff"].double()


def _flags_from_records(g, cfg):
    B, L, H, N, C = cfg.batch, cfg.n_layers, cfg.n_kv_heads, cfg.n_ctx, cfg.chunk
    rp = g["res_ptr"].cpu().numpy().astype(np.int64)
    pos = g["res_pos"].cpu().numpy().astype(np.int64) & 0xFFFF
    flags = np.zeros((B, L, H, N), dtype=bool)
    rec_tok = np.full(pos.shape[0], -1, dtype=np.int64)
    for b in range(B):
        for l in range(L):
            for h in range(H):
                for c in range(N // C):
                    seg = slice(rp[b, l, h, c], rp[b, l, h, c + 1])
                    p = pos[seg]
                    assert np.all(np.diff(p) > 0) and np.all(p < C)
                    flags[b, l, h, c * C + p] = True
                    rec_tok[seg] = c * C + p
    return flags, rec_tok


def _check_encode(cfg, g, o, og, n_res, norms_gpu=None):
    """o: the oracle's encode; og: the oracle's steps 3-6 on the GPU's stored coefficients;
    norms_gpu: the kernel's residual norms [B][L][Hkv][N] when they can be read back (the
    re-pack keeps its workspace inside the cache)."""
    int8 = cfg.store == "int8"
    # coefficients.  The GPU projects, (1/G) sum_l k_l B_l^T; the oracle solves the normal
    # equations of the stored (bf16-rounded) basis, whose rows are orthonormal only to about
    # 2^-8 per Gram entry, so the two differ by up to ~2^-7 of the row's largest entry, plus
    # one unit of the rounding of each result.
    ag = _stored_coeff(g, cfg).cpu().numpy()
    ao = o["extra"]["stored_coeff"]
    rowmax = np.abs(ao).max(axis=-1, keepdims=True)
    if int8:
        unit = o["coeff_scale"].astype(np.float64)[..., None]
        assert np.all(np.abs(ag - ao) <= 2 ** -6 * rowmax + unit + 1e-9)
    else:
        assert np.all(np.abs(ag - ao) <= 2 ** -6 * rowmax + 2 ** -7 * np.abs(ao) + 1e-9)
    # no systematic bias: rounding to nearest and the basis' departure from orthonormality
    # both scatter around zero, so the mean signed difference stays far below one unit of
    # the storage rounding (2^-8 relative for bf16), which a biased rounding would reach
    scale = np.abs(ao).mean()
    assert abs(float((ag - ao).mean())) <= 2 ** -11 * scale
    for idx in np.ndindex(*ag.shape[:3]):
        assert abs(float((ag[idx] - ao[idx]).mean())) <= 2 ** -9 * np.abs(ao[idx]).mean() + 1e-12, idx
    o = og   # from here on, everything is a function of the stored coefficients
    # summaries: fp32 vs fp64 sums of the same stored rows, rounded to bf16
    sg = g["summary"].double().cpu().numpy()
    so = O._bf16_bits_to_f64(o["summary"])
    cmax = np.abs(o["extra"]["stored_coeff"]).max(axis=-1).reshape(*so.shape[:3], so.shape[3], -1).max(-1)
    assert np.all(np.abs(sg - so) <= 2 ** -7 * np.abs(so) + 2 ** -12 * cmax[..., None] + 1e-9)
    # CSR offsets: unit u's records are [u * n_res, (u + 1) * n_res)
    rp = g["res_ptr"].cpu().numpy().astype(np.int64)
    units = cfg.batch * cfg.n_layers * cfg.n_kv_heads
    np.testing.assert_array_equal(rp.reshape(units, -1)[:, 0], np.arange(units) * n_res)
    np.testing.assert_array_equal(rp.reshape(units, -1)[:, -1], (np.arange(units) + 1) * n_res)
    # flags
    fg, rec_tok = _flags_from_records(g, cfg)
    fo = o["extra"]["flags"]
    norms = o["extra"]["norms"]
    bound = NORM_RTOL * norms + NORM_ATOL
    if norms_gpu is not None:
        assert np.all(np.abs(norms_gpu - norms) <= bound), float((np.abs(norms_gpu - norms) / norms).max())
    for idx in np.ndindex(*fo.shape[:3]):
        if np.array_equal(fg[idx], fo[idx]) or n_res in (0, cfg.n_ctx):
            assert np.array_equal(fg[idx], fo[idx])
            continue
        order = np.lexsort((np.arange(cfg.n_ctx), -norms[idx]))
        t_thr = order[n_res - 1]
        thr = norms[idx][t_thr]
        diff = fg[idx] != fo[idx]
        assert np.all(np.abs(norms[idx][diff] - thr) <= bound[idx][diff] + bound[idx][t_thr]), idx
    # residual rows of tokens both sides flagged
    d = cfg.head_dim
    if n_res > 0:
        if int8:
            vg = g["res_val"].double() * g["res_scale"].double().unsqueeze(-1)
            vo = o["res_val"].astype(np.float64) * o["res_scale"].astype(np.float64)[:, None]
        else:
            vg = g["res_val"].double()
            vo = O._bf16_bits_to_f64(o["res_val"])
        vg = vg.cpu().numpy()
        fo_flat = fo.reshape(-1, cfg.n_ctx)
        _, o_tok = _flags_from_records({"res_ptr": torch.tensor(o["res_ptr"]),
                                        "res_pos": torch.tensor(o["res_pos"].astype(np.int16))}, cfg)
        o_index = {}
        for i, t in enumerate(o_tok):
            o_index[(i // n_res, t)] = i
        worst = 0.0
        for i, t in enumerate(rec_tok):
            j = o_index.get((i // n_res, t))
            if j is None:
                continue
            scale = np.abs(vo[j]).max() + 1e-6
            err = np.abs(vg[i] - vo[j]).max() / scale
            worst = max(worst, err)
        assert worst <= (2 ** -6 if int8 else 2 ** -7) + 1e-3, worst
        assert fo_flat.sum() == vg.shape[0] == units * n_res


ENC_CASES = [
    ("mistral7b_group_bf16", dict(n_layers=4, n_kv_heads=2, n_ctx=1024)),              # r 64, C 64
    ("llama8b_32k_bf16", dict(batch=1, n_layers=4, n_kv_heads=2, n_ctx=1024)),        # r 128, C 128
    ("llama8b_32k_bf16", dict(batch=2, n_layers=4, n_kv_heads=1, n_ctx=512, rank=64)),  # r 64, C 128
    ("llama8b_32k_bf16", dict(batch=1, n_layers=4, n_kv_heads=2, n_ctx=512, chunk=64)),  # r 128, C 64
    ("llama8b_32k_bf16", dict(batch=2, n_layers=4, n_kv_heads=2, n_ctx=768, group=2)),   # G 2: two bases resident
    ("llama8b_32k_bf16", dict(batch=1, n_layers=8, n_kv_heads=1, n_ctx=512, group=8)),   # G 8: the one-tile form
    # 512 tiles over the 148 persistent CTAs: each tile group takes a second tile into the stage
    # its first one used
    ("llama8b_32k_bf16", dict(batch=2, n_layers=4, n_kv_heads=2, n_ctx=4096)),
]


@pytest.mark.parametrize("store", ["native", "int8"])
@pytest.mark.parametrize("name,kw", ENC_CASES)
def test_encode_matches_oracle(name, kw, store):
    cfg = S.CONFIGS[name].replace(name="enc_" + name, store=store, evict_frac=0.0, **kw)
    n_res = cfg.n_resid
    g, o, og = _encode_both(cfg, n_res)
    _check_encode(cfg, g, o, og, n_res, norms_gpu=_gpu_norms(g, cfg))


@pytest.mark.parametrize("n_res", [64, 128])
def test_encode_int8_records_with_sparse_flags(n_res):
    """int8 records from the tensor-core passes (r = C = 128) when few tokens are flagged: most
    warps of a tile then have no flagged token and finish its records long before the others,
    while the tile group's next tile (several per CTA here) is converted into the stage where
    the others' values rows sit."""
    cfg = S.CONFIGS["llama8b_32k_bf16"].replace(name="enc_sparse", store="int8", evict_frac=0.0, batch=2,
                                                n_layers=4, n_kv_heads=2, n_ctx=4096)
    g, o, og = _encode_both(cfg, n_res)
    _check_encode(cfg, g, o, og, n_res, norms_gpu=_gpu_norms(g, cfg))


@pytest.mark.parametrize("n_res", [0, 1, 512])
def test_encode_residual_count_edges(n_res):
    cfg = S.MISTRAL_GROUP.replace(name="enc_edges", n_layers=2, n_kv_heads=1, n_ctx=512)
    g, o, og = _encode_both(cfg, n_res)
    _check_encode(cfg, g, o, og, n_res, norms_gpu=_gpu_norms(g, cfg))


def _as_cache(cfg, g, weights):
    B, L, H, T, d = cfg.batch, cfg.n_layers, cfg.n_kv_heads, cfg.tail_cap, cfg.head_dim
    nC = cfg.n_ctx // cfg.chunk
    basis, w1, w2 = (t.to(DEV).contiguous() for t in weights)
    tk = torch.zeros(B, L, H, T, d, dtype=torch.bfloat16, device=DEV)
    return S.SynthCache(
        cfg=cfg, coeff=g["coeff"], coeff_scale=g["coeff_scale"], basis=basis, w1=w1, w2=w2,
        summary=g["summary"],
        slot=torch.arange(nC, dtype=torch.int16, device=DEV).expand(B, L // cfg.group, H, nC).contiguous(),
        res_ptr=g["res_ptr"], res_pos=g["res_pos"], res_val=g["res_val"], res_scale=g["res_scale"],
        tail_k=tk, tail_v=tk.clone(), tail_len=torch.zeros(B, dtype=torch.int32, device=DEV))


@pytest.mark.parametrize("store", ["native", "int8"])
def test_encoded_cache_decodes_in_parity(store):
    cfg = S.LLAMA_32K.replace(name="enc_decode", batch=2, n_layers=4, n_kv_heads=2, n_ctx=2048,
                              top_k=8, store=store)
    Kd, Vd = S.make_dense_kv(cfg, device=DEV)
    weights = _weights_bf16(cfg)
    g = K.lowram_encode(cfg, cfg.n_resid, Kd, Vd, *(t.to(DEV).contiguous() for t in weights))
    cache = _as_cache(cfg, g, weights)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    out, sel = lc.decode(q.to(DEV), sel=True)
    scores, _ = lc.select(q.to(DEV))
    torch.cuda.synchronize()
    assert lc.validate() == 0
    lc.close()
    check(cfg, O.OracleCache(S.cache_to_numpy(cache)), q, out, sel, scores=scores)


def _slice_ptr(res_ptr, b, ls, h, units, n_res):
    """CSR offsets of the slice's units rebased as if their records were contiguous."""
    rp = res_ptr[b, ls, h].clone().long()
    for li, u in enumerate(units):
        rp[li] -= (u - li) * n_res
    return rp.view(1, rp.shape[0], 1, rp.shape[1]).int()


def test_encode_full_size_sampled_units():
    """The 32K workload (B=4) encoded on the GPU; two (b, group, KV head) slices checked
    against the oracle run on just those slices."""
    cfg = S.LLAMA_32K
    Kd, Vd = S.make_dense_kv(cfg, device=DEV)
    weights = _weights_bf16(cfg)
    g = K.lowram_encode(cfg, cfg.n_resid, Kd, Vd, *(t.to(DEV).contiguous() for t in weights))
    torch.cuda.synchronize()
    norms_full = _gpu_norms(g, cfg)
    G = cfg.group
    for (b, grp, h) in [(1, 3, 5), (3, 7, 0)]:
        sub = cfg.replace(name="enc_slice", batch=1, n_layers=G, n_kv_heads=1)
        ls = slice(grp * G, (grp + 1) * G)
        basis, w1, w2 = weights
        args = (dataclasses.asdict(sub), _f64(Kd[b:b + 1, ls, h:h + 1]), _f64(Vd[b:b + 1, ls, h:h + 1]),
                _f64(basis[ls, h:h + 1]), _f64(w1[ls, h:h + 1]), _f64(w2[ls, h:h + 1]), cfg.n_resid)
        o = E.encode(*args)
        units = [(b * cfg.n_layers + l) * cfg.n_kv_heads + h for l in range(grp * G, (grp + 1) * G)]
        n_res, nC = cfg.n_resid, cfg.n_ctx // cfg.chunk
        rec = np.concatenate([np.arange(u * n_res, (u + 1) * n_res) for u in units])
        gs = {
            "coeff": g["coeff"][b:b + 1, grp:grp + 1, h:h + 1],
            "coeff_scale": None,
            "summary": g["summary"][b:b + 1, grp:grp + 1, h:h + 1],
            "res_ptr": _slice_ptr(g["res_ptr"], b, ls, h, units, n_res),
            "res_pos": g["res_pos"][torch.tensor(rec, device=DEV)],
            "res_val": g["res_val"][torch.tensor(rec, device=DEV)],
            "res_scale": None,
        }
        og = E.encode(*args, given=_gpu_codes(gs, sub))
        ng = norms_full[b:b + 1, ls, h:h + 1]
        _check_encode(sub, gs, o, og, n_res, norms_gpu=ng)
