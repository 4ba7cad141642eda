"""Failure paths that can be exercised without faulting, trapping or hanging the GPU.

* A bounded wait that runs out: the test hook ``lowram_debug_set_wait_limit`` shortens the
  tensor-core kernel's main-loop waits to a few cycles, so the first wait that is not already
  satisfied gives up.  The kernel must report it (``lowram_cache_validate`` returns
  LOWRAM_ETIMEOUT), leave the context usable, and the next call with the normal limit must be
  in parity with the oracle again.  Every wait in the kernel stays bounded throughout: the
  waits that drain a CTA's own copies and MMAs after an abort keep the full limit.
* A device allocation that fails: the host-side hook ``lowram_debug_fail_alloc`` makes one
  allocation of ``lowram_cache_create`` / ``lowram_cache_repack`` report out-of-memory.
  Both must return LOWRAM_ENOMEM and leave nothing behind; a failed re-pack must leave the
  cache exactly as it was.
"""

import gc

import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
from parity_utils import check

pytestmark = pytest.mark.gpu
DEV = "cuda"
ETIMEOUT, ENOMEM = 6, 2


def _oracle(cache):
    return O.OracleCache(S.cache_to_numpy(cache))


CASES = {
    "bf16": S.MISTRAL_GROUP,
    "int8_evict": S.LLAMA_64K_INT8.replace(name="int8_fail", batch=1, n_layers=4, n_kv_heads=2,
                                           n_q_heads=8, n_ctx=8192, top_k=8),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_wait_timeout_is_reported_and_the_next_call_recovers(name):
    cfg = CASES[name]
    cache = S.make_cache(cfg).to(DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    ref, ref_sel = lc.decode(q, sel=True, path=K.PATH_TC)
    torch.cuda.synchronize()
    assert lc.validate() == 0
    # a few cycles: the first wait that is not already satisfied runs out
    K.lowram_debug_set_wait_limit(lc.handle, 4)
    out = torch.full_like(q, float("nan"))
    lc.decode(q, out=out, path=K.PATH_TC)
    torch.cuda.synchronize()               # the kernel returned: the context is usable
    assert lc.validate() == ETIMEOUT
    assert lc.validate() == 0              # validate clears the error word
    # the normal limit again: the same results as before the timeout, in parity
    K.lowram_debug_set_wait_limit(lc.handle, 0)
    out2, sel2 = lc.decode(q, sel=True, path=K.PATH_TC)
    torch.cuda.synchronize()
    assert lc.validate() == 0
    assert torch.equal(sel2, ref_sel) and torch.equal(out2, ref)
    lc.close()
    check(cfg, _oracle(cache), q, out2, sel2)


def _free_bytes():
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return torch.cuda.mem_get_info()[0]


@pytest.mark.parametrize("after", [0, 1, 7, 14])
def test_create_allocation_failure_returns_enomem_and_frees_everything(after):
    cache = S.make_cache(S.MISTRAL_GROUP).to(DEV)
    free0 = _free_bytes()
    K.lowram_debug_fail_alloc(after)
    try:
        with pytest.raises(K.LowramError) as ei:
            K.LowramCache.from_synth(cache)
    finally:
        K.lowram_debug_fail_alloc(-1)
    assert ei.value.status == ENOMEM
    assert abs(_free_bytes() - free0) <= (4 << 20)
    # the library works normally afterwards
    lc = K.LowramCache.from_synth(cache)
    q = S.make_queries(cache)
    out, sel = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    lc.close()
    check(S.MISTRAL_GROUP, _oracle(cache), q, out, sel)


@pytest.mark.parametrize("after", [0, 1, 4])
def test_repack_allocation_failure_leaves_the_cache_unchanged(after):
    """The first re-pack of a created cache allocates its scratch and re-lays the arrays;
    a failed allocation at any of those steps must leave every array, count and result as
    they were."""
    cfg = S.MISTRAL_GROUP
    cache = S.make_cache(cfg, tail_len=[cfg.tail_cap]).to(DEV)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    before, sel_before = lc.decode(q, sel=True)
    cfg0, arr0 = lc.view()
    snap = {n: (t.clone() if isinstance(t, torch.Tensor) else t) for n, t in arr0.items()}
    K.lowram_debug_fail_alloc(after)
    try:
        with pytest.raises(K.LowramError) as ei:
            lc.repack(n_resid=6)
    finally:
        K.lowram_debug_fail_alloc(-1)
    assert ei.value.status == ENOMEM
    cfg1, arr1 = lc.view()
    assert cfg1 == cfg0
    for n, t in snap.items():
        if isinstance(t, torch.Tensor):
            assert torch.equal(arr1[n], t), n
        else:
            assert arr1[n] is None, n
    after_out, sel_after = lc.decode(q, sel=True)
    torch.cuda.synchronize()
    assert lc.validate() == 0
    assert torch.equal(sel_after, sel_before) and torch.equal(after_out, before)
    # and the re-pack goes through once allocations succeed
    lc.repack(n_resid=6)
    assert lc.validate() == 0
    lc.close()
