"""The allocation-free decode entry point against the regular one (through the C ABI).

Some callers cannot allocate device memory on their decode path: an engine that reserves
all device memory for its own pool, a runtime that forbids allocation after start-up, a
thread capturing a CUDA graph in a mode that rejects allocation calls.  They call
lowram_decode_attn_static, which reads the compressed cache straight from their arrays and
keeps all scratch in a static device array inside the library.  Its results must match
lowram_decode_attn on the same cache and the fp64 oracle, on two calls in a row, because the
static array keeps whatever the previous call left in it, and the calls must leave free device
memory where it was.

This file is collected last so that a run stopping at the first failure has already run
every other test.
"""

import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
from parity_utils import check

pytestmark = pytest.mark.gpu


def _vector_error(cfg, got, ref):
    g, r = got.double(), ref.double()
    diff = (g - r).abs().amax(dim=-1)
    if cfg.dtype == "f32":
        return float((diff / r.abs().amax(dim=-1)).max())
    return float((diff / r.norm(dim=-1)).max())


CASES = [
    ("tiny_f32", dict(), 0, 2, 1e-4),
    ("mistral7b_group_bf16", dict(), 0, 2, 2e-2),
    ("mistral7b_group_bf16", dict(), 1, 1, 2e-2),
    ("llama8b_64k_int8_evict", dict(batch=2, n_layers=8, n_kv_heads=2, n_q_heads=8,
                                    n_ctx=8192, top_k=8), 4, 2, 2e-2),
]


@pytest.mark.parametrize("name,kw,layer0,n_layers,tol", CASES)
def test_static_entry_point_matches_regular_one(name, kw, layer0, n_layers, tol):
    cfg = S.CONFIGS[name].replace(**kw) if kw else S.CONFIGS[name]
    cache = S.make_cache(cfg).to("cuda")
    q = S.make_queries(cache, layer0=layer0, n_layers=n_layers)
    lc = K.LowramCache.from_synth(cache)
    ref, ref_sel = lc.decode(q, sel=True, layer0=layer0, path=K.PATH_SIMT)
    torch.cuda.synchronize()
    lc.close()
    outs = [torch.full_like(q, float("nan")) for _ in range(3)]
    sels = [torch.full_like(ref_sel, -1) for _ in range(3)]
    # the first call on this device sets up the static array's address (it may also be
    # where the driver loads the module that holds the array); then free device memory must
    # not move across two more calls: they allocate nothing
    K.lowram_decode_attn_static(cfg, cache, layer0, n_layers, q, outs[2], sels[2])
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for i in range(2):
        K.lowram_decode_attn_static(cfg, cache, layer0, n_layers, q, outs[i], sels[i])
        torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    for out, sel in zip(outs[:2], sels[:2]):
        assert torch.equal(sel, ref_sel)
        assert _vector_error(cfg, out, ref) <= tol
        # and against the fp64 oracle, under the same parity rules as the regular path
        check(cfg, O.OracleCache(S.cache_to_numpy(cache)), q, out, sel, layer0=layer0)


def test_static_entry_point_rejects_calls_above_its_scratch():
    """All 32 layers of the 32K Llama-shaped cache need more than the 16 MiB static array;
    the call is refused on the host before anything is launched."""
    cfg = S.LLAMA_32K
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    arrays = {n: dummy for n in ("coeff", "basis", "w1", "w2", "summary", "res_ptr", "tail_k",
                                 "tail_v", "tail_len")}
    arrays.update(coeff_scale=None, slot=None, res_pos=dummy[:0], res_val=None, res_scale=None)
    q = torch.zeros(cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.head_dim, dtype=torch.bfloat16,
                    device="cuda")
    with pytest.raises(K.LowramError) as ei:
        K.lowram_decode_attn_static(cfg, arrays, 0, cfg.n_layers, q, torch.empty_like(q))
    assert ei.value.status == 1 and "static maximum" in str(ei.value)
