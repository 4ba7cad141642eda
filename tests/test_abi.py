"""The C-ABI library loads, exports every declared symbol and validates on the host.

No compute call here needs a GPU: only host-only entry points and argument checks that
return before any CUDA call.
"""

import ctypes
import dataclasses
import glob
import os
import re

import pytest

import kv_cache_compression_lowram_b200 as K
import lowram_synth as S
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(lowram_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = K.lib()
    names = _declared_functions()
    assert len(names) >= 14
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_dense_kv_bytes_worked_example():
    # Llama-3.1-8B, 32K prompt, batch 4, fp16: 16 GiB ("OjaKV" abstract; M_KV formula of
    # "LowRAM Compresses KV Cache Asymmetrically", section "Core Mechanism")
    assert K.lowram_dense_kv_bytes(32, 8, 128, 32768, 2, 4) == 17179869184
    assert K.lowram_dense_kv_bytes(32, 8, 128, 32768, 2, 4) == O.dense_kv_bytes(32, 8, 128, 32768, 2, 4)
    assert K.lowram_dense_kv_bytes(-1, 8, 128, 32768, 2, 4) == 0


@pytest.mark.parametrize("name", ["tiny_f32", "mistral7b_group_bf16", "llama8b_32k_bf16",
                                  "llama8b_64k_int8_evict", "llama8b_32k_bf16_b64"])
def test_config_bytes_match_oracle_closed_form(name):
    cfg = S.CONFIGS[name]
    n_rec = cfg.batch * cfg.n_layers * cfg.n_kv_heads * cfg.n_resid // 3
    got = K.lowram_config_bytes(cfg, n_rec, has_slot=True)
    want = O.compressed_bytes(dataclasses.asdict(cfg), n_rec)
    assert got == want


def test_bad_configs_rejected_on_host():
    bad = [
        dict(top_k=10_000),
        dict(n_ctx=1000),            # not a multiple of chunk
        dict(n_q_heads=30),          # not a multiple of n_kv_heads
        dict(n_layers=30),           # not a multiple of group
        dict(rank=10_000),
        dict(dtype="f32", store="int8"),
        dict(batch=0),
        dict(batch=70_000),          # coefficient rows above 2^31 (32-bit row indices)
    ]
    for kw in bad:
        cfg = S.LLAMA_32K.replace(**kw)
        with pytest.raises(K.LowramError) as ei:
            K.lowram_config_bytes(cfg, 0)
        assert ei.value.status == 1


def test_create_rejects_null_sources_without_touching_cuda():
    lib = K.lib()
    c = K.config_struct(S.TINY_F32)
    src = K.LowramSrcC()
    h = ctypes.c_void_p()
    st = lib.lowram_cache_create(ctypes.byref(c), ctypes.byref(src), ctypes.byref(h), None)
    assert st == 1 and not h.value
    assert b"NULL" in lib.lowram_last_error_string()
    # NULL cache handles are rejected, not dereferenced
    assert lib.lowram_decode_attn(None, 0, 1, None, None, None, 0, None) == 1
    assert lib.lowram_cache_validate(None, None) == 1
    assert lib.lowram_cache_last_launches(None) == 0
    lib.lowram_cache_destroy(None)


def test_status_strings():
    lib = K.lib()
    for s in range(7):
        assert lib.lowram_status_string(s)


def test_encode_host_checks():
    """Workspace size and the argument checks that return before any CUDA call."""
    cfg = S.MISTRAL_GROUP
    c = K.config_struct(cfg)
    c.n_live = c.n_ctx // c.chunk
    al = lambda x: (x + 255) // 256 * 256
    units = cfg.batch * cfg.n_layers * cfg.n_kv_heads
    lh = cfg.n_layers * cfg.n_kv_heads
    want = (al(lh * cfg.rank * cfg.mlp_hidden * 4) + al(lh * cfg.mlp_hidden * cfg.rank * 2)
            + al(lh * cfg.head_dim * cfg.mlp_hidden * 2) + al(units * cfg.n_ctx * 4) + al(units * cfg.n_ctx)
            + al(4))
    assert K.lib().lowram_encode_workspace_bytes(ctypes.byref(c)) == want
    f32 = K.config_struct(S.TINY_F32)
    assert K.lib().lowram_encode_workspace_bytes(ctypes.byref(f32)) == 0
    dst = K.LowramEncodeDstC()
    st = K.lib().lowram_encode(ctypes.byref(f32), 1, None, None, None, None, None, ctypes.byref(dst),
                               None, 0, None)
    assert st == 4   # LOWRAM_EUNSUPPORTED
    st = K.lib().lowram_encode(ctypes.byref(c), -1, None, None, None, None, None, ctypes.byref(dst),
                               None, 0, None)
    assert st == 1   # LOWRAM_EINVAL
    st = K.lib().lowram_encode(ctypes.byref(c), 4, None, None, None, None, None, ctypes.byref(dst),
                               None, 0, None)
    assert st == 1


def test_upkeep_host_checks():
    """Cache view, append and re-pack reject a NULL cache before touching the device."""
    lib = K.lib()
    cfg, src = K.LowramConfigC(), K.LowramSrcC()
    spare = ctypes.c_int32()
    assert lib.lowram_cache_view(None, ctypes.byref(cfg), ctypes.byref(src), ctypes.byref(spare)) == 1
    assert lib.lowram_cache_append(None, None, None, None) == 1
    assert lib.lowram_cache_repack(None, 4, None) == 1


def test_test_hooks_host_side():
    """The failure-path hooks: NULL caches are rejected and the allocation hook can be armed
    and disarmed without a device (it only counts allocations)."""
    lib = K.lib()
    assert lib.lowram_debug_set_wait_limit(None, 5) == 1
    K.lowram_debug_fail_alloc(3)
    K.lowram_debug_fail_alloc(-1)


def test_shard_and_merge_host_checks():
    """Context-sharded decode: NULL caches and impossible merge shapes are rejected before any
    CUDA call."""
    lib = K.lib()
    assert lib.lowram_shard_candidates(None, 0, 1, None, 0, None, None, None) == 1
    assert lib.lowram_shard_partial(None, 0, 1, 0, 2, None, None, None, None, None) == 1
    bad = [
        (0, 4, 128, 1),      # no parts
        (2, -1, 128, 1),     # negative row count
        (2, 1 << 31, 128, 1),
        (2, 4, 0, 1),        # head_dim outside 1..256
        (2, 4, 257, 1),
        (2, 4, 128, 7),      # unknown output dtype
        (2, 4, 128, 1),      # rows but NULL buffers
    ]
    for n_parts, n_rows, d, dt in bad:
        assert lib.lowram_merge_partials(n_parts, n_rows, d, None, dt, None, None) == 1, (n_parts, n_rows, d, dt)
        assert lib.lowram_last_error_string()


def test_reuse_host_checks():
    """The reuse store's entry points reject NULL handles and outputs on the host; destroying
    NULL is a no-op."""
    lib = K.lib()
    h = ctypes.c_void_p(1234)
    assert lib.lowram_reuse_create(None, 16, 16, ctypes.byref(h), None) == 1
    assert not h.value   # the output handle is cleared on every error
    assert lib.lowram_decode_attn_reuse(None, 0, 1, None, None, None, None) == 1
    counts = K.LowramReuseCountsC()
    assert lib.lowram_reuse_counts_get(None, ctypes.byref(counts), None) == 1
    t, o, e = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    stride = ctypes.c_int64()
    assert lib.lowram_reuse_view(None, ctypes.byref(t), ctypes.byref(o), ctypes.byref(e), ctypes.byref(stride)) == 1
    lib.lowram_reuse_destroy(None)


def test_reuse_wrapper_refuses_a_closed_cache():
    """A store whose cache was closed is refused before the library follows the freed cache."""
    from types import SimpleNamespace

    store = K.LowramReuse.__new__(K.LowramReuse)
    store.cache, store.capacity, store.handle = SimpleNamespace(cfg=None, handle=0), 16, 0
    with pytest.raises(K.LowramError) as ei:
        store.decode(None)
    assert ei.value.status == 1
