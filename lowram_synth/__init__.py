"""Seeded synthetic LowRAM-compressed KV caches and decode queries.

This module defines the workloads and draws their inputs.  It is shared by the tests,
the benchmark and the CUDA library's Python binding users, and it deliberately holds
none of the decode-time arithmetic (no key rebuild of cached tokens, no value predictor,
no scoring, selection or attention): it only draws random ingredients and packs them into
the storage layout that ``include/lowram.h`` documents.

The synthetic cache is written directly in compressed form (compression fitting is not
part of the decode path):

* coefficients ``a_t`` (per token, shared by the G layers of a group): entry i (1-based)
  ~ N(0, 1) * i**-0.5;
* basis ``B_l`` (r x d per layer and KV head): orthonormal rows, the transposed Q of a QR
  factorisation of a Gaussian d x r matrix (the orthonormal bases of "OjaKV", section 3.1);
* predictor weights W1 (h x d) ~ N(0,1)/sqrt(d), W2 (d x h) ~ N(0,1)/sqrt(h), no biases;
* residuals: the synthetic true values are V = Vhat + eps, so the residual of a token is
  delta_t = eps_t, eps ~ N(0, 0.02**2) per element, except a seeded 5 % of tokens whose
  eps is 0.2 * t3 per element (Student-t with 3 degrees of freedom, Z / sqrt(chi2_3 / 3)).
  The ceil(rho * N) tokens with the largest ||eps_t||_2 per (b, l, KV head) are flagged
  and keep delta_t (the error-driven choice of "LowRAM Compresses KV Cache
  Asymmetrically", section "Core Mechanism"); ties go to the lower token index;
* eviction (optional): floor(evict_frac * nC) chunks per (b, group, KV head), chosen by a
  seeded permutation; storage is compacted to the live chunks;
* int8 store (optional): per row, scale = max|x| / 127 rounded to fp16,
  q = round-half-even(x / scale) clamped to +-127;
* chunk summaries: the mean of the chunk's stored (dequantised) coefficient rows;
* raw tail: keys a . B_l + N(0, 0.01**2) with a drawn by the coefficient law, values
  ~ N(0, 0.1**2), tail_len[b] = T unless given;
* queries: q_j = q_scale * (z_j / sqrt(d) + beta * (kbar_c1/|kbar_c1| + kbar_c2/|kbar_c2|)),
  z ~ N(0, I), beta = 1, c1 != c2 two seeded live chunks per (b, l, KV head) shared by the
  g query heads of the KV head, kbar_c = abar_c . B_l the layer's mean key of chunk c.

Big tensors are drawn on the requested device in slices; small ones (bases, weights) are
always drawn on the CPU, so a cache generated on the CPU and one generated on a GPU
share their weights but not their coefficient draws.
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import torch

__all__ = [
    "LowramConfig",
    "CONFIGS",
    "get_config",
    "SynthCache",
    "make_cache",
    "make_queries",
    "pack_cache",
    "cache_to_numpy",
    "quantize_rows_int8",
]

SIGMA_V = 0.02          # value noise std
OUTLIER_FRAC = 0.05     # share of tokens with Student-t(3) value noise
OUTLIER_SCALE = 0.2     # scale of the Student-t(3) noise (10 * SIGMA_V)
KEY_NOISE = 0.01        # std of the raw tail keys' noise around a . B_l
TAIL_V_STD = 0.1        # std of the raw tail values
QUERY_BETA = 1.0        # weight of the two target chunks in a query


@dataclass(frozen=True)
class LowramConfig:
    """Shapes and storage of one synthetic workload (symbols as in ``lowram.h``)."""

    name: str
    batch: int
    n_layers: int
    group: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    rank: int
    mlp_hidden: int
    n_ctx: int
    chunk: int
    top_k: int
    tail_cap: int
    resid_frac: float
    dtype: str = "bf16"       # "f32" | "bf16"
    store: str = "native"     # "native" | "int8"
    evict_frac: float = 0.0
    seed: int = 1234

    @property
    def n_chunks(self) -> int:
        return self.n_ctx // self.chunk

    @property
    def n_evicted(self) -> int:
        return int(math.floor(self.evict_frac * self.n_chunks))

    @property
    def n_live(self) -> int:
        return self.n_chunks - self.n_evicted

    @property
    def n_groups(self) -> int:
        return self.n_layers // self.group

    @property
    def q_per_kv(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_resid(self) -> int:
        """Flagged tokens per (b, l, KV head) before eviction: ceil(rho * N)."""
        return int(math.ceil(self.resid_frac * self.n_ctx - 1e-9))

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "LowramConfig":
        return dataclasses.replace(self, **kw)

    def validate(self) -> None:
        assert self.n_layers % self.group == 0
        assert self.n_q_heads % self.n_kv_heads == 0
        assert self.n_ctx % self.chunk == 0
        assert 1 <= self.top_k <= self.n_live
        assert self.dtype in ("f32", "bf16") and self.store in ("native", "int8")
        assert not (self.store == "int8" and self.dtype != "bf16")


CONFIGS: Dict[str, LowramConfig] = {}


def _reg(cfg: LowramConfig) -> LowramConfig:
    CONFIGS[cfg.name] = cfg
    return cfg


# Tiny fp32 case: one layer group of 2, one KV head, one query head, d=64, N=256.
TINY_F32 = _reg(LowramConfig(
    name="tiny_f32", batch=1, n_layers=2, group=2, n_kv_heads=1, n_q_heads=1, head_dim=64,
    rank=16, mlp_hidden=64, n_ctx=256, chunk=32, top_k=4, tail_cap=8, resid_frac=0.25,
    dtype="f32", seed=1000))
# Mistral-7B-shaped single layer group, bf16.
MISTRAL_GROUP = _reg(LowramConfig(
    name="mistral7b_group_bf16", batch=1, n_layers=2, group=2, n_kv_heads=8, n_q_heads=32,
    head_dim=128, rank=64, mlp_hidden=256, n_ctx=4096, chunk=64, top_k=16, tail_cap=64,
    resid_frac=0.10, dtype="bf16", seed=2000))
# Llama-3.1-8B-shaped full model at 32K context, batch 4, bf16.
LLAMA_32K = _reg(LowramConfig(
    name="llama8b_32k_bf16", batch=4, n_layers=32, group=4, n_kv_heads=8, n_q_heads=32,
    head_dim=128, rank=128, mlp_hidden=256, n_ctx=32768, chunk=128, top_k=32, tail_cap=128,
    resid_frac=0.125, dtype="bf16", seed=3000))
# Batch sweep of the 32K Llama shape.
for _b in (1, 4, 16, 32, 64):
    _reg(LLAMA_32K.replace(name=f"llama8b_32k_bf16_b{_b}", batch=_b))
# One sequence, 8 layers: a profiling case above L2 size but only ~1 GB of dense K, V.
_reg(LLAMA_32K.replace(name="llama8b_32k_bf16_b1_l8", batch=1, n_layers=8))
# Composition with int8 quantisation and 50 % chunk eviction at 64K context, batch 8.
LLAMA_64K_INT8 = _reg(LowramConfig(
    name="llama8b_64k_int8_evict", batch=8, n_layers=32, group=4, n_kv_heads=8,
    n_q_heads=32, head_dim=128, rank=128, mlp_hidden=256, n_ctx=65536, chunk=128, top_k=32,
    tail_cap=128, resid_frac=0.125, dtype="bf16", store="int8", evict_frac=0.5, seed=4000))
# Its small profiling case (2 sequences, 8 layers: 0.13 GB of int8 coefficients).
_reg(LLAMA_64K_INT8.replace(name="llama8b_64k_int8_evict_b2_l8", batch=2, n_layers=8))


def get_config(name: str) -> LowramConfig:
    return CONFIGS[name]


# ----------------------------------------------------------------------------- seeding

_MASK64 = (1 << 64) - 1


def _mix(*keys: int) -> int:
    """splitmix64 over a tuple of integers (S. Vigna's finaliser), 63-bit result."""
    x = 0x9E3779B97F4A7C15
    for k in keys:
        x = (x + (int(k) & _MASK64) + 0x9E3779B97F4A7C15) & _MASK64
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        x = z ^ (z >> 31)
    return x & ((1 << 63) - 1)


def _gen(device, *keys: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_mix(*keys))
    return g


# tensor tags for seeding
_T_COEFF, _T_BASIS, _T_W1, _T_W2, _T_EPS, _T_EVICT, _T_TAILA, _T_TAILK, _T_TAILV, _T_Q = range(10)
_T_DKA, _T_DKN, _T_DV = 10, 11, 12


# --------------------------------------------------------------------------- container

@dataclass
class SynthCache:
    """Storage arrays of one compressed cache (torch tensors, layouts of ``lowram.h``)."""

    cfg: LowramConfig
    coeff: torch.Tensor
    coeff_scale: Optional[torch.Tensor]
    basis: torch.Tensor
    w1: torch.Tensor
    w2: torch.Tensor
    summary: torch.Tensor
    slot: torch.Tensor
    res_ptr: torch.Tensor
    res_pos: torch.Tensor
    res_val: torch.Tensor
    res_scale: Optional[torch.Tensor]
    tail_k: torch.Tensor
    tail_v: torch.Tensor
    tail_len: torch.Tensor
    extra: dict = field(default_factory=dict)

    @property
    def n_records(self) -> int:
        return int(self.res_pos.shape[0])

    def to(self, device) -> "SynthCache":
        kw = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            kw[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return SynthCache(**kw)

    def tensors(self) -> Dict[str, Optional[torch.Tensor]]:
        return {f.name: getattr(self, f.name) for f in dataclasses.fields(self)
                if f.name not in ("cfg", "extra")}


# ----------------------------------------------------------------------------- helpers

def quantize_rows_int8(x: torch.Tensor):
    """Per-row int8 encoding: scale = max|x|/127 rounded to fp16; q = RNE(x/scale), |q|<=127.

    Returns (q int8, scale fp16).  A zero row gets scale 0 and q = 0.
    """
    x32 = x.float()
    amax = x32.abs().amax(dim=-1)
    scale = (amax / 127.0).to(torch.float16)
    s = scale.float()
    s_div = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.round(x32 / s_div.unsqueeze(-1)).clamp_(-127, 127)
    q = torch.where((s > 0).unsqueeze(-1), q, torch.zeros_like(q))
    return q.to(torch.int8), scale


def _coeff_law(n: int, r: int, gen: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(n, r, generator=gen, device=device, dtype=torch.float32)
    col = torch.arange(1, r + 1, device=device, dtype=torch.float32).rsqrt()
    return z * col


def _orthonormal_rows(r: int, d: int, gen: torch.Generator) -> torch.Tensor:
    g = torch.randn(d, r, generator=gen, dtype=torch.float64)
    qm, rm = torch.linalg.qr(g)  # d x r, orthonormal columns
    # fix signs so the factorisation is unique
    sgn = torch.sign(torch.diagonal(rm))
    sgn[sgn == 0] = 1
    return (qm * sgn).t().contiguous()  # r x d


def _slot_map(cfg: LowramConfig, b: int, grp: int, hkv: int) -> torch.Tensor:
    nC = cfg.n_chunks
    slot = torch.arange(nC, dtype=torch.int64)
    if cfg.n_evicted > 0:
        perm = torch.randperm(nC, generator=_gen("cpu", cfg.seed, _T_EVICT, b, grp, hkv))
        dead = torch.zeros(nC, dtype=torch.bool)
        dead[perm[: cfg.n_evicted]] = True
        live = (~dead).to(torch.int64)
        slot = torch.cumsum(live, 0) - 1
        slot[dead] = -1
    return slot.to(torch.int16)


def _draw_eps(cfg: LowramConfig, b: int, l: int, device) -> torch.Tensor:
    """Value noise eps [Hkv][N][d] of one (b, l): Gaussian, Student-t(3) on 5 % of tokens."""
    Hkv, N, d = cfg.n_kv_heads, cfg.n_ctx, cfg.head_dim
    gen = _gen(device, cfg.seed, _T_EPS, b, l)
    eps = torch.randn(Hkv, N, d, generator=gen, device=device) * SIGMA_V
    is_out = torch.rand(Hkv, N, generator=gen, device=device) < OUTLIER_FRAC
    z = torch.randn(Hkv, N, d, generator=gen, device=device)
    chi = torch.randn(Hkv, N, d, 3, generator=gen, device=device).square().sum(-1)
    t3 = z / torch.sqrt(chi / 3.0)
    return torch.where(is_out.unsqueeze(-1), OUTLIER_SCALE * t3, eps)


def _flag_worst(err_norm: torch.Tensor, n_res: int) -> torch.Tensor:
    """Boolean mask of the n_res largest entries per row (ties to the lower index)."""
    order = torch.sort(err_norm, dim=-1, descending=True, stable=True).indices
    mask = torch.zeros_like(err_norm, dtype=torch.bool)
    mask.scatter_(-1, order[..., :n_res], True)
    return mask


# ------------------------------------------------------------------------------ packing

def pack_cache(cfg: LowramConfig, coeff_full: torch.Tensor, basis: torch.Tensor,
               w1: torch.Tensor, w2: torch.Tensor, flags: torch.Tensor, delta: torch.Tensor,
               tail_k: torch.Tensor, tail_v: torch.Tensor, tail_len: torch.Tensor,
               slot: Optional[torch.Tensor] = None,
               store_dtype: Optional[torch.dtype] = None) -> SynthCache:
    """Pack dense per-token ingredients into the storage layout.

    coeff_full [B][L/G][Hkv][N][r] (float), basis [L][Hkv][r][d], w1 [L][Hkv][h][d],
    w2 [L][Hkv][d][h], flags [B][L][Hkv][N] bool, delta [B][L][Hkv][N][d] (rows of
    unflagged tokens are ignored), tail_k/v [B][L][Hkv][T][d], tail_len [B],
    slot [B][L/G][Hkv][nC] int16 or None (no eviction).  ``store_dtype`` overrides the
    storage dtype of the native arrays (torch.float64 builds exact caches for the oracle's
    pins; such caches are not accepted by the CUDA library).
    """
    B, NG, Hkv, N, r = coeff_full.shape
    L, d, C = cfg.n_layers, cfg.head_dim, cfg.chunk
    nC = N // C
    dev = coeff_full.device
    if slot is None:
        slot = torch.arange(nC, dtype=torch.int16).expand(B, NG, Hkv, nC).contiguous()
    slot = slot.to(dev)
    nL = int((slot[0, 0, 0] >= 0).sum())
    sd = store_dtype if store_dtype is not None else cfg.torch_dtype
    int8 = cfg.store == "int8"

    coeff = torch.empty(B, NG, Hkv, nL * C, r, device=dev,
                        dtype=torch.int8 if int8 else sd)
    coeff_scale = torch.empty(B, NG, Hkv, nL * C, device=dev, dtype=torch.float16) if int8 else None
    summary = torch.empty(B, NG, Hkv, nL, r, device=dev, dtype=sd)
    for b in range(B):
        for grp in range(NG):
            live_tok = (slot[b, grp] >= 0).repeat_interleave(C, dim=-1)  # [Hkv][N]
            rows = coeff_full[b, grp][live_tok].view(Hkv, nL * C, r)
            if int8:
                q, s = quantize_rows_int8(rows)
                coeff[b, grp] = q
                coeff_scale[b, grp] = s
                deq = q.double() * s.double().unsqueeze(-1)
            else:
                stored = rows.to(sd)
                coeff[b, grp] = stored
                deq = stored.double()
            summary[b, grp] = deq.view(Hkv, nL, C, r).mean(dim=2).to(sd)

    # residual records, unit order (b, l, hkv), inside a unit ascending token index
    res_ptr = torch.empty(B, L, Hkv, nL + 1, dtype=torch.int64)
    pos_list, val_list = [], []
    base = 0
    for b in range(B):
        for l in range(L):
            grp = l // cfg.group
            for h in range(Hkv):
                sl = slot[b, grp, h].to(torch.int64)
                live_tok = (sl >= 0).repeat_interleave(C)
                f = flags[b, l, h].to(dev) & live_tok
                idx = torch.nonzero(f).flatten()
                chunk_slot = sl[(idx // C)]
                counts = torch.bincount(chunk_slot, minlength=nL)[:nL].cpu()
                res_ptr[b, l, h, 0] = base
                res_ptr[b, l, h, 1:] = base + torch.cumsum(counts, 0)
                base += int(idx.numel())
                pos_list.append((idx % C).to(torch.int16))
                val_list.append(delta[b, l, h][idx])
    res_pos = torch.cat(pos_list) if pos_list else torch.empty(0, dtype=torch.int16, device=dev)
    vals = torch.cat(val_list) if val_list else torch.empty(0, d, device=dev)
    if int8:
        res_val, res_scale = quantize_rows_int8(vals)
    else:
        res_val, res_scale = vals.to(sd), None
    assert base < 2**31
    return SynthCache(
        cfg=cfg, coeff=coeff, coeff_scale=coeff_scale,
        basis=basis.to(dev).to(sd).contiguous(), w1=w1.to(dev).to(sd).contiguous(),
        w2=w2.to(dev).to(sd).contiguous(), summary=summary, slot=slot.contiguous(),
        res_ptr=res_ptr.to(torch.int32).to(dev), res_pos=res_pos.contiguous(),
        res_val=res_val.contiguous(), res_scale=res_scale,
        tail_k=tail_k.to(dev).to(torch.bfloat16 if int8 else sd).contiguous(),
        tail_v=tail_v.to(dev).to(torch.bfloat16 if int8 else sd).contiguous(),
        tail_len=tail_len.to(torch.int32).to(dev).contiguous())


# ---------------------------------------------------------------------------- generator

def make_weights(cfg: LowramConfig, identity_basis: bool = False):
    """Basis B_l, W1, W2 (fp64, CPU) for every (layer, KV head)."""
    L, Hkv, r, d, h = cfg.n_layers, cfg.n_kv_heads, cfg.rank, cfg.head_dim, cfg.mlp_hidden
    basis = torch.empty(L, Hkv, r, d, dtype=torch.float64)
    w1 = torch.empty(L, Hkv, h, d, dtype=torch.float64)
    w2 = torch.empty(L, Hkv, d, h, dtype=torch.float64)
    for l in range(L):
        for hk in range(Hkv):
            if identity_basis:
                assert r == cfg.group * d, "identity basis needs rank = group * head_dim"
                eye = torch.eye(r, dtype=torch.float64)
                li = l % cfg.group
                basis[l, hk] = eye[:, li * d:(li + 1) * d]
            else:
                assert r <= d, "orthonormal basis rows need rank <= head_dim"
                basis[l, hk] = _orthonormal_rows(r, d, _gen("cpu", cfg.seed, _T_BASIS, l, hk))
            w1[l, hk] = torch.randn(h, d, generator=_gen("cpu", cfg.seed, _T_W1, l, hk),
                                    dtype=torch.float64) / math.sqrt(d)
            w2[l, hk] = torch.randn(d, h, generator=_gen("cpu", cfg.seed, _T_W2, l, hk),
                                    dtype=torch.float64) / math.sqrt(h)
    return basis, w1, w2


def make_dense_kv(cfg: LowramConfig, device="cpu"):
    """Dense prefill keys and values [B][L][Hkv][N][d] (bf16) for the encoder.

    Keys follow the cache's law: K_l = A B_l + N(0, 0.01^2) with A (coefficient law, shared
    by the layers of a group) and B_l from ``make_weights``; values are N(0, 0.1^2) with a
    seeded 5 % of tokens scaled by 4 (so that residual norms spread out).  Returns (K, V).
    """
    B, L, G, Hkv, N, d, r = (cfg.batch, cfg.n_layers, cfg.group, cfg.n_kv_heads, cfg.n_ctx,
                             cfg.head_dim, cfg.rank)
    basis, _, _ = make_weights(cfg)
    K = torch.empty(B, L, Hkv, N, d, dtype=torch.bfloat16, device=device)
    V = torch.empty(B, L, Hkv, N, d, dtype=torch.bfloat16, device=device)
    bdev = basis.to(device=device, dtype=torch.float32)
    for b in range(B):
        for grp in range(L // G):
            for h in range(Hkv):
                a = _coeff_law(N, r, _gen(device, cfg.seed, _T_DKA, b, grp, h), device).float()
                for li in range(G):
                    l = grp * G + li
                    noise = torch.randn(N, d, generator=_gen(device, cfg.seed, _T_DKN, b, l, h),
                                        device=device) * 0.01
                    K[b, l, h] = (a @ bdev[l, h] + noise).to(torch.bfloat16)
        for l in range(L):
            gen = _gen(device, cfg.seed, _T_DV, b, l)
            v = torch.randn(Hkv, N, d, generator=gen, device=device) * 0.1
            big = torch.rand(Hkv, N, generator=gen, device=device) < 0.05
            V[b, l] = torch.where(big.unsqueeze(-1), 4.0 * v, v).to(torch.bfloat16)
    return K, V


def make_cache(cfg: LowramConfig, device="cpu", tail_len=None) -> SynthCache:
    """Draw and pack the synthetic compressed cache of ``cfg`` on ``device``.

    Works slice by slice (one (b, layer group) or (b, layer) at a time) so that the
    full-size workloads fit in device memory; the result is identical to what
    ``pack_cache`` gives for the same ingredients.
    """
    cfg.validate()
    dev = torch.device(device)
    B, L, G, Hkv = cfg.batch, cfg.n_layers, cfg.group, cfg.n_kv_heads
    NG, N, r, d, C, T = cfg.n_groups, cfg.n_ctx, cfg.rank, cfg.head_dim, cfg.chunk, cfg.tail_cap
    nC, nL = cfg.n_chunks, cfg.n_live
    sd = cfg.torch_dtype
    int8 = cfg.store == "int8"

    basis64, w1_64, w2_64 = make_weights(cfg)
    basis_dev = basis64.to(dev, torch.float32)

    slot = torch.empty(B, NG, Hkv, nC, dtype=torch.int16)
    for b in range(B):
        for grp in range(NG):
            for h in range(Hkv):
                slot[b, grp, h] = _slot_map(cfg, b, grp, h)
    slot_dev = slot.to(dev)

    coeff = torch.empty(B, NG, Hkv, nL * C, r, device=dev, dtype=torch.int8 if int8 else sd)
    coeff_scale = torch.empty(B, NG, Hkv, nL * C, device=dev, dtype=torch.float16) if int8 else None
    summary = torch.empty(B, NG, Hkv, nL, r, device=dev, dtype=sd)
    for b in range(B):
        for grp in range(NG):
            full = torch.empty(Hkv, N, r, device=dev)
            for h in range(Hkv):
                full[h] = _coeff_law(N, r, _gen(dev, cfg.seed, _T_COEFF, b, grp, h), dev)
            live_tok = (slot_dev[b, grp] >= 0).repeat_interleave(C, dim=-1)
            rows = full[live_tok].view(Hkv, nL * C, r)
            if int8:
                q, s = quantize_rows_int8(rows)
                coeff[b, grp] = q
                coeff_scale[b, grp] = s
                deq = q.double() * s.double().unsqueeze(-1)
            else:
                stored = rows.to(sd)
                coeff[b, grp] = stored
                deq = stored.double()
            summary[b, grp] = deq.view(Hkv, nL, C, r).mean(dim=2).to(sd)
            del full, rows, deq

    # residuals: exact record counts are known only after flagging; allocate the no-eviction
    # upper bound and trim at the end.
    n_res = cfg.n_resid
    cap = B * L * Hkv * n_res
    res_pos = torch.empty(cap, dtype=torch.int16, device=dev)
    res_val = torch.empty(cap, d, dtype=torch.int8 if int8 else sd, device=dev)
    res_scale = torch.empty(cap, dtype=torch.float16, device=dev) if int8 else None
    res_ptr = torch.empty(B, L, Hkv, nL + 1, dtype=torch.int64, device=dev)
    base = 0
    for b in range(B):
        for l in range(L):
            grp = l // G
            eps = _draw_eps(cfg, b, l, dev)                      # [Hkv][N][d]
            flags = _flag_worst(eps.norm(dim=-1), n_res)         # [Hkv][N]
            sl = slot_dev[b, grp].to(torch.int64)                # [Hkv][nC]
            live_tok = (sl >= 0).repeat_interleave(C, dim=-1)
            flags &= live_tok
            counts = flags.view(Hkv, nC, C).sum(-1)              # per chunk id
            # per slot counts: live chunks in ascending id order == slot order
            live_counts = counts[sl >= 0].view(Hkv, nL)
            per_head = flags.sum(-1)                              # [Hkv]
            head_base = base + torch.cumsum(per_head, 0) - per_head
            res_ptr[b, l, :, 0] = head_base
            res_ptr[b, l, :, 1:] = head_base.unsqueeze(-1) + torch.cumsum(live_counts, -1)
            hh, tt = torch.nonzero(flags, as_tuple=True)          # row-major: head, token
            nrec = int(tt.numel())
            rows = eps[hh, tt]
            res_pos[base:base + nrec] = (tt % C).to(torch.int16)
            if int8:
                q, s = quantize_rows_int8(rows)
                res_val[base:base + nrec] = q
                res_scale[base:base + nrec] = s
            else:
                res_val[base:base + nrec] = rows.to(sd)
            base += nrec
            del eps, flags, rows
    assert base < 2**31
    res_pos = res_pos[:base].clone()
    res_val = res_val[:base].clone()
    if int8:
        res_scale = res_scale[:base].clone()

    tail_dt = torch.bfloat16 if int8 else sd
    tail_k = torch.empty(B, L, Hkv, T, d, device=dev, dtype=tail_dt)
    tail_v = torch.empty(B, L, Hkv, T, d, device=dev, dtype=tail_dt)
    for b in range(B):
        for l in range(L):
            ga = _gen(dev, cfg.seed, _T_TAILA, b, l)
            a = torch.randn(Hkv, T, r, generator=ga, device=dev)
            a = a * torch.arange(1, r + 1, device=dev, dtype=torch.float32).rsqrt()
            k = torch.bmm(a, basis_dev[l])
            k += KEY_NOISE * torch.randn(Hkv, T, d, generator=_gen(dev, cfg.seed, _T_TAILK, b, l),
                                         device=dev)
            v = TAIL_V_STD * torch.randn(Hkv, T, d, generator=_gen(dev, cfg.seed, _T_TAILV, b, l),
                                         device=dev)
            tail_k[b, l] = k.to(tail_dt)
            tail_v[b, l] = v.to(tail_dt)
    if tail_len is None:
        tl = torch.full((B,), T, dtype=torch.int32)
    else:
        tl = torch.as_tensor(tail_len, dtype=torch.int32).reshape(B)
    return SynthCache(
        cfg=cfg, coeff=coeff, coeff_scale=coeff_scale,
        basis=basis64.to(dev).to(sd), w1=w1_64.to(dev).to(sd), w2=w2_64.to(dev).to(sd),
        summary=summary, slot=slot_dev, res_ptr=res_ptr.to(torch.int32), res_pos=res_pos,
        res_val=res_val, res_scale=res_scale, tail_k=tail_k, tail_v=tail_v,
        tail_len=tl.to(dev))


def make_queries(cache: SynthCache, layer0: int = 0, n_layers: Optional[int] = None,
                 q_scale: float = 1.0, seed_offset: int = 0, device=None) -> torch.Tensor:
    """Decode queries [n_layers][B][Hq][d] biased toward two live chunks per KV head."""
    cfg = cache.cfg
    if n_layers is None:
        n_layers = cfg.n_layers - layer0
    dev = torch.device(device) if device is not None else cache.summary.device
    B, Hkv, g, d, r = cfg.batch, cfg.n_kv_heads, cfg.q_per_kv, cfg.head_dim, cfg.rank
    nL = cfg.n_live
    out = torch.empty(n_layers, B, cfg.n_q_heads, d, dtype=torch.float32, device=dev)
    summ = cache.summary.to(dev).float()
    basis = cache.basis.to(dev).float()
    for li in range(n_layers):
        l = layer0 + li
        grp = l // cfg.group
        gz = _gen(dev, cfg.seed, _T_Q, seed_offset, l)
        z = torch.randn(B, cfg.n_q_heads, d, generator=gz, device=dev)
        gc = _gen("cpu", cfg.seed, _T_Q, seed_offset, l, 7)
        for b in range(B):
            for h in range(Hkv):
                if nL >= 2:
                    pair = torch.randperm(nL, generator=gc)[:2]
                else:
                    pair = torch.zeros(1, dtype=torch.int64)
                kbar = summ[b, grp, h, pair.to(dev)] @ basis[l, h]     # [2][d]
                bias = (kbar / kbar.norm(dim=-1, keepdim=True).clamp_min(1e-30)).sum(0)
                j0 = h * g
                out[li, b, j0:j0 + g] = z[b, j0:j0 + g] / math.sqrt(d) + QUERY_BETA * bias
    out *= q_scale
    return out.to(cfg.torch_dtype)


def make_query_steps(cache: SynthCache, n_steps: int, rho: float, drift: float, layer0: int = 0,
                     n_layers: Optional[int] = None, seed_offset: int = 0):
    """Decode queries of n_steps consecutive steps, each [n_layers][B][Hq][d], whose selections
    persist: per unit the query is z_t / sqrt(d) + beta (kbar_c1 / |kbar_c1| + kbar_c2 /
    |kbar_c2|) as in ``make_queries``, with AR(1) noise z_t = rho z_{t-1} + sqrt(1 - rho^2) eps_t
    and two target chunks that each jump to a random live chunk with probability ``drift`` per
    step (else stay).  rho = 0, drift = 1 gives independent steps."""
    cfg = cache.cfg
    if n_layers is None:
        n_layers = cfg.n_layers - layer0
    dev = cache.summary.device
    B, Hkv, g, d = cfg.batch, cfg.n_kv_heads, cfg.q_per_kv, cfg.head_dim
    nL = cfg.n_live
    summ = cache.summary.float()
    basis = cache.basis.float()
    gsel = _gen("cpu", cfg.seed, _T_Q, seed_offset, 11)
    targets = torch.randint(0, nL, (n_layers, B, Hkv, 2), generator=gsel)
    z = torch.randn(n_layers, B, cfg.n_q_heads, d, generator=_gen(dev, cfg.seed, _T_Q, seed_offset, 12, 0), device=dev)
    steps = []
    for t in range(n_steps):
        if t > 0:
            eps = torch.randn(z.shape, generator=_gen(dev, cfg.seed, _T_Q, seed_offset, 12, t), device=dev)
            z = rho * z + math.sqrt(max(0.0, 1.0 - rho * rho)) * eps
            jump = torch.rand(targets.shape, generator=gsel) < drift
            targets = torch.where(jump, torch.randint(0, nL, targets.shape, generator=gsel), targets)
        out = torch.empty(n_layers, B, cfg.n_q_heads, d, dtype=torch.float32, device=dev)
        for li in range(n_layers):
            l = layer0 + li
            grp = l // cfg.group
            for b in range(B):
                for h in range(Hkv):
                    kbar = summ[b, grp, h, targets[li, b, h].to(dev)] @ basis[l, h]      # [2][d]
                    bias = (kbar / kbar.norm(dim=-1, keepdim=True).clamp_min(1e-30)).sum(0)
                    j0 = h * g
                    out[li, b, j0:j0 + g] = z[li, b, j0:j0 + g] / math.sqrt(d) + QUERY_BETA * bias
        steps.append(out.to(cfg.torch_dtype))
    return steps


def select_sequences(cache: SynthCache, seqs, device="cpu") -> SynthCache:
    """The cache of sequences ``seqs`` alone (in that order), on ``device``.

    Every per-sequence array keeps only those sequences; the residual records of each kept
    sequence (a contiguous range: records are laid out sequence by sequence) are gathered
    and the CSR offsets rebased.  Used to check a large batch against the oracle on a few
    sequences without copying the whole cache to the host.
    """
    seqs = [int(b) for b in seqs]
    idx = torch.as_tensor(seqs, device=cache.coeff.device)
    rp = cache.res_ptr.to(torch.int64)
    spans = [(int(rp[b].min()), int(rp[b].max())) for b in seqs]
    rec_idx = torch.cat([torch.arange(a, e, device=cache.res_pos.device) for a, e in spans]) \
        if spans else torch.empty(0, dtype=torch.int64, device=cache.res_pos.device)
    new_rp = []
    base = 0
    for b, (a, e) in zip(seqs, spans):
        new_rp.append(rp[b] - a + base)
        base += e - a
    res_ptr = torch.stack(new_rp).to(torch.int32)

    def rows(t):
        return None if t is None else t.index_select(0, idx).to(device)

    def recs(t):
        return None if t is None else t.index_select(0, rec_idx).to(device)

    return SynthCache(
        cfg=cache.cfg.replace(name=cache.cfg.name + "_seqs", batch=len(seqs)),
        coeff=rows(cache.coeff), coeff_scale=rows(cache.coeff_scale), basis=cache.basis.to(device),
        w1=cache.w1.to(device), w2=cache.w2.to(device), summary=rows(cache.summary),
        slot=rows(cache.slot), res_ptr=res_ptr.to(device), res_pos=recs(cache.res_pos),
        res_val=recs(cache.res_val), res_scale=recs(cache.res_scale), tail_k=rows(cache.tail_k),
        tail_v=rows(cache.tail_v), tail_len=rows(cache.tail_len))


def shard_chunks(cache: SynthCache, c_lo: int, c_hi: int, keep_tail: bool) -> SynthCache:
    """The cache of chunk ids [c_lo, c_hi) of every unit, as a cache of its own (local ids).

    Every unit keeps those chunks' coefficient rows, scales and summaries and the residual
    records of those chunks (gathered unit by unit, CSR offsets rebased).  The raw tail is
    kept (keep_tail) or emptied (tail_len = 0, arrays kept).  Caches with evicted chunks are
    not split (their live chunks per range differ between units).  Used to build the shards
    of a context-sharded decode from one generated cache.
    """
    cfg = cache.cfg
    assert cfg.n_live == cfg.n_chunks, "no eviction in a split cache"
    assert 0 <= c_lo < c_hi <= cfg.n_chunks
    C = cfg.chunk
    n = c_hi - c_lo
    dev = cache.coeff.device
    rp = cache.res_ptr.to(torch.int64)
    lo, hi = rp[..., c_lo], rp[..., c_hi]                      # [B][L][Hkv]
    counts = (hi - lo).reshape(-1)
    starts = lo.reshape(-1)
    idx = torch.cat([torch.arange(int(a), int(a) + int(c), device=dev) for a, c in zip(starts.tolist(), counts.tolist())]) \
        if counts.numel() else torch.empty(0, dtype=torch.int64, device=dev)
    base = (torch.cumsum(counts, 0) - counts).reshape(lo.shape)
    res_ptr = (rp[..., c_lo:c_hi + 1] - lo.unsqueeze(-1) + base.unsqueeze(-1)).to(torch.int32)

    def recs(t):
        return None if t is None else t.index_select(0, idx).contiguous()

    tl = cache.tail_len.clone() if keep_tail else torch.zeros_like(cache.tail_len)
    B, NG, H = cfg.batch, cfg.n_groups, cfg.n_kv_heads
    return SynthCache(
        cfg=cfg.replace(name=f"{cfg.name}_c{c_lo}_{c_hi}", n_ctx=n * C),
        coeff=cache.coeff[:, :, :, c_lo * C:c_hi * C].contiguous(),
        coeff_scale=None if cache.coeff_scale is None else cache.coeff_scale[:, :, :, c_lo * C:c_hi * C].contiguous(),
        basis=cache.basis, w1=cache.w1, w2=cache.w2,
        summary=cache.summary[:, :, :, c_lo:c_hi].contiguous(),
        slot=torch.arange(n, dtype=torch.int16, device=dev).expand(B, NG, H, n).contiguous(),
        res_ptr=res_ptr, res_pos=recs(cache.res_pos), res_val=recs(cache.res_val),
        res_scale=recs(cache.res_scale), tail_k=cache.tail_k, tail_v=cache.tail_v, tail_len=tl)


# ------------------------------------------------------------------------ numpy export

def _np_storage(t: Optional[torch.Tensor]):
    """Tensor -> numpy array holding the same bits (bf16 as uint16 bit patterns)."""
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


def cache_to_numpy(cache: SynthCache) -> dict:
    """Host copies of every storage array, plus the config fields as plain values.

    bf16 arrays come back as uint16 bit patterns (key ``<name>_is_bf16`` True); fp16 as
    numpy float16; res_pos as uint16.
    """
    out = {"cfg": dataclasses.asdict(cache.cfg)}
    for name, t in cache.tensors().items():
        arr = _np_storage(t)
        if name == "res_pos" and arr is not None:
            arr = arr.view("uint16")
        out[name] = arr
        out[name + "_is_bf16"] = bool(t is not None and t.dtype == torch.bfloat16)
    return out
