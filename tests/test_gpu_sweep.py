"""Parity at the batch sweep's larger batches (32K Llama shape, B = 16 and B = 64).

The sweep's throughput numbers come from these launch configurations (16384 units and
524288 chunk tiles at B = 64), so the same calls are checked here: the workload is generated
on the GPU, decoded in one all-layer call, and 64 seeded units of a few sampled sequences are
compared with the fp64 oracle (selection, scores and outputs under the rules of
``parity_utils``).  At B = 16 every path is checked; at B = 64 (about 87 GB of compressed
cache, which the cache object then copies) the product path only.
"""

import gc

import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O
from parity_utils import check, sample_units

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _release():
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("batch,paths", [(16, (K.PATH_AUTO, K.PATH_TC, K.PATH_SIMT)), (64, (K.PATH_AUTO,))])
def test_sweep_batch_sampled_units(batch, paths):
    cfg = S.CONFIGS[f"llama8b_32k_bf16_b{batch}"]
    _release()
    cache = S.make_cache(cfg, device=DEV)
    q = S.make_queries(cache)
    _release()
    seqs = sorted({0, batch // 2 + 1, batch - 1})
    sub = S.select_sequences(cache, seqs)          # host copy of the sampled sequences
    lc = K.LowramCache.from_synth(cache)
    del cache
    _release()
    results = []
    for path in paths:
        out, sel = lc.decode(q, sel=True, path=path)
        scores, _ = lc.select(q)
        torch.cuda.synchronize()
        assert lc.validate() == 0
        if path == K.PATH_TC:
            assert lc.last_path == K.PATH_TC
        results.append((out[:, seqs].cpu(), sel[:, seqs].cpu(), scores[:, seqs].cpu()))
        del out, sel, scores
    lc.close()
    _release()
    oc = O.OracleCache(S.cache_to_numpy(sub))
    units = sample_units(sub.cfg, cfg.n_layers, 64, seed=batch)
    for out, sel, scores in results:
        res = check(sub.cfg, oc, q[:, seqs].cpu(), out, sel, units=units, scores=scores)
        assert res["units"] >= 64
