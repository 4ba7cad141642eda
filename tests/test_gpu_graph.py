"""The decode call captured in a CUDA graph: the library launches only on the caller's
stream, with no synchronisation and no allocation, so an all-layer call can be captured once
and replayed; the replays must reproduce the eager call bit for bit, also after the queries
are overwritten in place."""

import pytest
import torch

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,path", [("mistral7b_group_bf16", K.PATH_TC), ("mistral7b_group_bf16", K.PATH_SIMT),
                                       ("tiny_f32", K.PATH_AUTO)])
def test_decode_replays_from_a_cuda_graph(name, path):
    cfg = S.CONFIGS[name]
    cache = S.make_cache(cfg)
    lc = K.LowramCache.from_synth(cache.to(DEV))
    q = S.make_queries(cache).to(DEV)
    out_e = torch.empty_like(q)
    out_g = torch.empty_like(q)
    lc.decode(q, out=out_e, path=path)          # warm-up and the eager reference
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lc.decode(q, out=out_g, path=path)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e)
    # new queries written into the captured buffer, then replay vs eager again
    q.copy_(S.make_queries(cache, seed_offset=3).to(DEV))
    g.replay()
    lc.decode(q, out=out_e, path=path)
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e)
    assert lc.validate() == 0
    del g
    lc.close()
