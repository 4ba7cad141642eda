"""Python binding of liblowram.so: decode-time attention over a LowRAM-compressed KV cache.

This module only marshals arguments (torch tensors -> device pointers, config objects ->
C structs) for the C ABI declared in ``include/lowram.h``; every step of the computation
runs in the library's CUDA kernels.  The library must be built first
(``python -m kv_cache_compression_lowram_b200.build``); if it is missing, every call raises.

Entry points keep the C names: ``lowram_cache_create``, ``lowram_decode_attn``,
``lowram_select_chunks``, ``lowram_decode_attn_host``, ``lowram_cache_bytes``,
``lowram_config_bytes``, ``lowram_cache_validate``, ``lowram_cache_destroy``,
``lowram_dense_kv_bytes``, ``lowram_cache_set_stage_events``,
``lowram_cache_last_launches``, ``lowram_cache_last_path``.  ``LowramCache`` wraps a handle.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "LowramError", "LIB_PATH", "PATH_AUTO", "PATH_SIMT", "PATH_TC", "lib",
    "lowram_dense_kv_bytes", "lowram_config_bytes", "lowram_cache_create",
    "lowram_cache_destroy", "lowram_decode_attn", "lowram_select_chunks",
    "lowram_decode_attn_host", "lowram_cache_bytes", "lowram_cache_validate",
    "lowram_cache_set_stage_events", "lowram_cache_last_launches", "lowram_cache_last_path",
    "LowramCache", "config_struct", "lowram_decode_attn_static", "lowram_dense_decode_attn",
    "lowram_cache_view", "lowram_cache_append", "lowram_cache_repack",
    "lowram_encode", "LowramReuse", "lowram_reuse_create", "lowram_reuse_destroy",
    "lowram_decode_attn_reuse", "lowram_reuse_counts_get", "lowram_reuse_view",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblowram.so")
PATH_AUTO, PATH_SIMT, PATH_TC = 0, 1, 2
STATUS = {0: "LOWRAM_OK", 1: "LOWRAM_EINVAL", 2: "LOWRAM_ENOMEM", 3: "LOWRAM_ECUDA",
          4: "LOWRAM_EUNSUPPORTED", 5: "LOWRAM_ECORRUPT", 6: "LOWRAM_ETIMEOUT"}


class LowramError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")
        self.status = status


class LowramConfigC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_layers", "group", "n_kv_heads", "n_q_heads", "head_dim", "rank",
        "mlp_hidden", "n_ctx", "chunk", "top_k", "tail_cap", "n_live", "dtype", "store")]


class LowramSrcC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "coeff", "coeff_scale", "basis", "w1", "w2", "summary", "slot", "res_ptr", "res_pos",
        "res_val", "res_scale", "tail_k", "tail_v", "tail_len")] + [("n_records", ctypes.c_int64)]


class LowramEncodeDstC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "coeff", "coeff_scale", "summary", "res_ptr", "res_pos", "res_val", "res_scale")]


class LowramBytesC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "coeff", "basis", "predictor", "summary", "residual", "index", "tail", "total",
        "dense_equiv")]


_LIB = None


class LowramReuseCountsC(ctypes.Structure):
    _fields_ = [("hits", ctypes.c_uint64), ("misses", ctypes.c_uint64), ("fills", ctypes.c_uint64)]


def lib() -> ctypes.CDLL:
    """The loaded library (raises if liblowram.so was not built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m kv_cache_compression_lowram_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    sig = {
        "lowram_dense_kv_bytes": (U64, [I32, I32, I32, I64, I32, I32]),
        "lowram_config_bytes": (I32, [ctypes.POINTER(LowramConfigC), I64, I32,
                                      ctypes.POINTER(LowramBytesC)]),
        "lowram_cache_create": (I32, [ctypes.POINTER(LowramConfigC), ctypes.POINTER(LowramSrcC),
                                      ctypes.POINTER(P), P]),
        "lowram_cache_destroy": (None, [P]),
        "lowram_decode_attn": (I32, [P, I32, I32, P, P, P, I32, P]),
        "lowram_select_chunks": (I32, [P, I32, I32, P, P, P, P]),
        "lowram_decode_attn_host": (I32, [P, I32, I32, P, P, P, P]),
        "lowram_cache_bytes": (I32, [P, ctypes.POINTER(LowramBytesC)]),
        "lowram_cache_validate": (I32, [P, P]),
        "lowram_cache_set_stage_events": (I32, [P, P]),
        "lowram_cache_last_launches": (I32, [P]),
        "lowram_cache_last_path": (I32, [P]),
        "lowram_cache_view": (I32, [P, ctypes.POINTER(LowramConfigC), ctypes.POINTER(LowramSrcC),
                                    ctypes.POINTER(I32)]),
        "lowram_cache_append": (I32, [P, P, P, P]),
        "lowram_cache_repack": (I32, [P, I32, P]),
        "lowram_decode_attn_static": (I32, [ctypes.POINTER(LowramConfigC), ctypes.POINTER(LowramSrcC),
                                            I32, I32, P, P, P, P]),
        "lowram_dense_decode_attn": (I32, [I32, I32, I32, I32, I32, I64, P, P, P, P, P]),
        "lowram_encode_workspace_bytes": (U64, [ctypes.POINTER(LowramConfigC)]),
        "lowram_encode": (I32, [ctypes.POINTER(LowramConfigC), I32, P, P, P, P, P,
                                ctypes.POINTER(LowramEncodeDstC), P, U64, P]),
        "lowram_shard_candidates": (I32, [P, I32, I32, P, I32, P, P, P]),
        "lowram_shard_partial": (I32, [P, I32, I32, I32, I32, P, P, P, P, P]),
        "lowram_merge_partials": (I32, [I32, I64, I32, P, I32, P, P]),
        "lowram_reuse_create": (I32, [P, I32, I32, ctypes.POINTER(P), P]),
        "lowram_reuse_destroy": (None, [P]),
        "lowram_decode_attn_reuse": (I32, [P, I32, I32, P, P, P, P]),
        "lowram_reuse_counts_get": (I32, [P, ctypes.POINTER(LowramReuseCountsC), P]),
        "lowram_reuse_view": (I32, [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                                    ctypes.POINTER(I64)]),
        "lowram_debug_set_wait_limit": (I32, [P, I64]),
        "lowram_debug_fail_alloc": (None, [I32]),
        "lowram_status_string": (ctypes.c_char_p, [I32]),
        "lowram_last_error_string": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L


def _check(status: int, where: str) -> None:
    if status != 0:
        raise LowramError(status, where, lib().lowram_last_error_string().decode())


# --------------------------------------------------------------------------- marshalling

def _get(cfg, name):
    return cfg[name] if isinstance(cfg, dict) else getattr(cfg, name)


def config_struct(cfg) -> LowramConfigC:
    """C config from an object or dict with the ``lowram.h`` field names.

    ``dtype`` may be "f32"/"bf16" or 0/1, ``store`` "native"/"int8" or 0/1.  ``n_live``
    defaults to n_ctx // chunk (no eviction).
    """
    c = LowramConfigC()
    for n in ("batch", "n_layers", "group", "n_kv_heads", "n_q_heads", "head_dim", "rank",
              "mlp_hidden", "n_ctx", "chunk", "top_k", "tail_cap"):
        setattr(c, n, int(_get(cfg, n)))
    try:
        n_live = int(_get(cfg, "n_live"))
    except (AttributeError, KeyError):
        n_live = c.n_ctx // c.chunk
    c.n_live = n_live
    dt = _get(cfg, "dtype")
    c.dtype = {"f32": 0, "bf16": 1}.get(dt, dt) if isinstance(dt, str) else int(dt)
    stv = _get(cfg, "store")
    c.store = {"native": 0, "int8": 1}.get(stv, stv) if isinstance(stv, str) else int(stv)
    return c


def _ptr(t) -> int:
    if t is None:
        return 0
    if not t.is_contiguous():
        raise ValueError("tensors passed to liblowram must be contiguous")
    return int(t.data_ptr())


def _stream(stream) -> int:
    if stream is not None:
        return int(stream) if isinstance(stream, int) else int(stream.cuda_stream)
    import torch
    if torch.cuda.is_available():
        return int(torch.cuda.current_stream().cuda_stream)
    return 0


def _bytes_dict(b: LowramBytesC) -> dict:
    return {n: int(getattr(b, n)) for n, _ in LowramBytesC._fields_}


def lowram_dense_kv_bytes(n_layers: int, n_kv_heads: int, head_dim: int, n_ctx: int,
                          bytes_per_scalar: int, batch: int) -> int:
    return int(lib().lowram_dense_kv_bytes(n_layers, n_kv_heads, head_dim, n_ctx,
                                           bytes_per_scalar, batch))


def lowram_config_bytes(cfg, n_records: int, has_slot: bool = True) -> dict:
    out = LowramBytesC()
    c = config_struct(cfg)
    _check(lib().lowram_config_bytes(ctypes.byref(c), int(n_records), int(has_slot),
                                     ctypes.byref(out)), "lowram_config_bytes")
    return _bytes_dict(out)


def _src_struct(arrays):
    src = LowramSrcC()
    names = ("coeff", "coeff_scale", "basis", "w1", "w2", "summary", "slot", "res_ptr",
             "res_pos", "res_val", "res_scale", "tail_k", "tail_v", "tail_len")
    keep = []
    for n in names:
        try:
            t = _get(arrays, n)
        except (AttributeError, KeyError):
            t = None
        if t is not None and not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
        keep.append(t)
        setattr(src, n, _ptr(t))
    rp = _get(arrays, "res_pos")
    src.n_records = int(rp.shape[0]) if rp is not None else 0
    return src, keep


def lowram_cache_create(cfg, arrays, stream=None) -> int:
    """Create a cache from device tensors.  ``arrays`` is a mapping (or an object with
    attributes) holding coeff, coeff_scale, basis, w1, w2, summary, slot, res_ptr, res_pos,
    res_val, res_scale, tail_k, tail_v, tail_len (layouts of ``lowram.h``)."""
    src, keep = _src_struct(arrays)
    c = config_struct(cfg)
    h = ctypes.c_void_p()
    _check(lib().lowram_cache_create(ctypes.byref(c), ctypes.byref(src), ctypes.byref(h),
                                     _stream(stream)), "lowram_cache_create")
    return int(h.value)


def lowram_cache_destroy(handle: int) -> None:
    if handle:
        lib().lowram_cache_destroy(handle)


def lowram_decode_attn(handle: int, layer0: int, n_layers: int, q, out, sel=None,
                       path: int = PATH_AUTO, stream=None) -> None:
    _check(lib().lowram_decode_attn(handle, layer0, n_layers, _ptr(q), _ptr(out), _ptr(sel),
                                    path, _stream(stream)), "lowram_decode_attn")


def lowram_select_chunks(handle: int, layer0: int, n_layers: int, q, scores=None, sel=None,
                         stream=None) -> None:
    _check(lib().lowram_select_chunks(handle, layer0, n_layers, _ptr(q), _ptr(scores), _ptr(sel),
                                      _stream(stream)), "lowram_select_chunks")


def lowram_decode_attn_host(handle: int, layer0: int, n_layers: int, q_host, out_host,
                            sel_host=None, stream=None) -> None:
    _check(lib().lowram_decode_attn_host(handle, layer0, n_layers, _ptr(q_host), _ptr(out_host),
                                         _ptr(sel_host), _stream(stream)),
           "lowram_decode_attn_host")


def lowram_decode_attn_static(cfg, arrays, layer0: int, n_layers: int, q, out, sel=None,
                              stream=None) -> None:
    """Decode straight from the caller's device arrays with no device allocation (the
    library's static scratch; see ``lowram.h``)."""
    src, keep = _src_struct(arrays)
    c = config_struct(cfg)
    _check(lib().lowram_decode_attn_static(ctypes.byref(c), ctypes.byref(src), layer0, n_layers,
                                           _ptr(q), _ptr(out), _ptr(sel), _stream(stream)),
           "lowram_decode_attn_static")


def lowram_dense_decode_attn(k, v, q, out, stream=None) -> None:
    """Dense baseline: k, v [B][L][Hkv][S][d] bf16, q/out [L][B][Hq][d] bf16 (device)."""
    B, L, Hkv, S_, d = (int(x) for x in k.shape)
    Hq = int(q.shape[2])
    _check(lib().lowram_dense_decode_attn(B, L, Hkv, Hq, d, S_, _ptr(k), _ptr(v), _ptr(q), _ptr(out),
                                          _stream(stream)), "lowram_dense_decode_attn")


def lowram_cache_bytes(handle: int) -> dict:
    out = LowramBytesC()
    _check(lib().lowram_cache_bytes(handle, ctypes.byref(out)), "lowram_cache_bytes")
    return _bytes_dict(out)


def lowram_cache_validate(handle: int, stream=None) -> int:
    """Returns the lowram_status (0 = consistent, 1 = an append found a full tail, 5 = corrupt
    tables, 6 = a wait timed out)."""
    st = int(lib().lowram_cache_validate(handle, _stream(stream)))
    if st not in (0, 1, 5, 6):
        _check(st, "lowram_cache_validate")
    return st


def lowram_cache_set_stage_events(handle: int, events=None) -> None:
    if events is None:
        _check(lib().lowram_cache_set_stage_events(handle, None), "set_stage_events")
        return
    for e in events:
        if int(e.cuda_event) == 0:   # torch creates the CUDA event on its first record
            e.record()
    arr = (ctypes.c_void_p * 4)(*[int(e.cuda_event) for e in events])
    _check(lib().lowram_cache_set_stage_events(handle, ctypes.cast(arr, ctypes.c_void_p)),
           "set_stage_events")


def lowram_cache_last_launches(handle: int) -> int:
    return int(lib().lowram_cache_last_launches(handle))


def lowram_cache_last_path(handle: int) -> int:
    return int(lib().lowram_cache_last_path(handle))


def lowram_shard_candidates(handle: int, layer0: int, n_layers: int, q, chunk_offset: int, cand_score, cand_id,
                            stream=None) -> None:
    """Phase 1 of a context-sharded decode step on one shard (see lowram.h)."""
    _check(lib().lowram_shard_candidates(handle, layer0, n_layers, _ptr(q), int(chunk_offset), _ptr(cand_score),
                                         _ptr(cand_id), _stream(stream)), "lowram_shard_candidates")


def lowram_shard_partial(handle: int, layer0: int, n_layers: int, chunk_offset: int, n_shards: int, cand_score,
                         cand_id, partial, sel=None, stream=None) -> None:
    """Phase 2 on one shard, from every shard's gathered candidates (see lowram.h)."""
    _check(lib().lowram_shard_partial(handle, layer0, n_layers, int(chunk_offset), int(n_shards), _ptr(cand_score),
                                      _ptr(cand_id), _ptr(partial), _ptr(sel), _stream(stream)),
           "lowram_shard_partial")


def lowram_merge_partials(partials, out, stream=None) -> None:
    """partials [n_parts][n_rows][d + 2] fp32 -> out [n_rows][d] (fp32 or bf16), CUDA tensors."""
    import torch
    n_parts, n_rows, w = (int(x) for x in partials.shape)
    dt = 0 if out.dtype == torch.float32 else 1
    _check(lib().lowram_merge_partials(n_parts, n_rows, w - 2, _ptr(partials), dt, _ptr(out), _stream(stream)),
           "lowram_merge_partials")


def lowram_reuse_create(handle: int, capacity: int, fill_cap: int, stream=None) -> int:
    """A store of rebuilt chunk values for cache ``handle`` (see lowram.h); returns its handle."""
    out = ctypes.c_void_p()
    _check(lib().lowram_reuse_create(handle, int(capacity), int(fill_cap), ctypes.byref(out), _stream(stream)),
           "lowram_reuse_create")
    return int(out.value)


def lowram_reuse_destroy(store: int) -> None:
    lib().lowram_reuse_destroy(store)


def lowram_decode_attn_reuse(store: int, layer0: int, n_layers: int, q, out, sel=None, stream=None) -> None:
    """lowram_decode_attn through a reuse store (CUDA tensors as there)."""
    _check(lib().lowram_decode_attn_reuse(store, layer0, n_layers, _ptr(q), _ptr(out), _ptr(sel), _stream(stream)),
           "lowram_decode_attn_reuse")


def lowram_reuse_counts_get(store: int, stream=None) -> dict:
    c = LowramReuseCountsC()
    _check(lib().lowram_reuse_counts_get(store, ctypes.byref(c), _stream(stream)), "lowram_reuse_counts_get")
    return {"hits": int(c.hits), "misses": int(c.misses), "fills": int(c.fills)}


def lowram_reuse_view(store: int, cfg, capacity: int) -> dict:
    """Zero-copy torch views of the store's table, owner and entries (device memory it owns)."""
    import torch
    table, owner, entries = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    stride = ctypes.c_int64()
    _check(lib().lowram_reuse_view(store, ctypes.byref(table), ctypes.byref(owner), ctypes.byref(entries),
                                   ctypes.byref(stride)), "lowram_reuse_view")
    B, L, H = _get(cfg, "batch"), _get(cfg, "n_layers"), _get(cfg, "n_kv_heads")
    C, d = _get(cfg, "chunk"), _get(cfg, "head_dim")

    def wrap(ptr, shape, typestr):
        return torch.as_tensor(_DeviceArray(ptr.value, shape, typestr), device="cuda")

    return {"table": wrap(table, (B, L, H, int(stride.value)), "<i4"),
            "owner": wrap(owner, (int(capacity),), "<i8"),
            "entries": wrap(entries, (int(capacity), C, d), "<i2").view(torch.bfloat16)}


class LowramReuse:
    """Owning wrapper of a reuse store (destroy it before its cache)."""

    def __init__(self, cache: "LowramCache", capacity: int, fill_cap: int, stream=None):
        self.cache, self.capacity = cache, int(capacity)
        self.handle = lowram_reuse_create(cache.handle, capacity, fill_cap, stream)

    def decode(self, q, out=None, sel: bool = False, layer0: int = 0, n_layers: Optional[int] = None, stream=None):
        import torch
        if not getattr(self.cache, "handle", 0):   # the library would follow a freed cache
            raise LowramError(1, "LowramReuse.decode", "the store's cache was closed")
        if n_layers is None:
            n_layers = int(q.shape[0])
        if out is None:
            out = torch.empty_like(q)
        s = None
        if sel:
            c = self.cache.cfg
            s = torch.empty(n_layers, _get(c, "batch"), _get(c, "n_kv_heads"), _get(c, "top_k"),
                            dtype=torch.int32, device=q.device)
        lowram_decode_attn_reuse(self.handle, layer0, n_layers, q, out, s, stream)
        return (out, s) if sel else out

    def counts(self, stream=None) -> dict:
        return lowram_reuse_counts_get(self.handle, stream)

    def view(self) -> dict:
        return lowram_reuse_view(self.handle, self.cache.cfg, self.capacity)

    def close(self) -> None:
        if getattr(self, "handle", 0):
            lowram_reuse_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lowram_debug_set_wait_limit(handle: int, cycles: int) -> None:
    """Test hook: limit of the tensor-core kernel's main-loop waits (cycles <= 0: default)."""
    _check(lib().lowram_debug_set_wait_limit(handle, int(cycles)), "lowram_debug_set_wait_limit")


def lowram_debug_fail_alloc(after: int) -> None:
    """Test hook: the device allocation after the next ``after`` ones fails (-1: off)."""
    lib().lowram_debug_fail_alloc(int(after))


def lowram_cache_append(handle: int, k_new, v_new, stream=None) -> None:
    """Append one decode step's k, v [L][B][Hkv][d] (the tail's dtype, CUDA) to every tail."""
    _check(lib().lowram_cache_append(handle, _ptr(k_new), _ptr(v_new), _stream(stream)),
           "lowram_cache_append")


def lowram_cache_repack(handle: int, n_resid: int, stream=None) -> None:
    """Compress the oldest chunk of every tail into a new chunk (synchronous; see lowram.h)."""
    _check(lib().lowram_cache_repack(handle, int(n_resid), _stream(stream)), "lowram_cache_repack")


class _DeviceArray:
    """A device pointer with a shape, for torch.as_tensor (CUDA array interface, no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(int(x) for x in shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def lowram_cache_view(handle: int):
    """(config dict, arrays dict): the cache's current config and torch tensors aliasing the
    device arrays it owns (read-only use; valid until the next re-pack or destroy).  The
    chunk arrays are strided views of their live part (the cache keeps room for more chunks
    after a re-pack: ``cfg["spare_chunks"]``); records may have spare rows between units."""
    import torch
    c, src, spare = LowramConfigC(), LowramSrcC(), ctypes.c_int32()
    _check(lib().lowram_cache_view(handle, ctypes.byref(c), ctypes.byref(src), ctypes.byref(spare)),
           "lowram_cache_view")
    cfg = {n: int(getattr(c, n)) for n, _ in LowramConfigC._fields_}
    cfg["spare_chunks"] = S_ = int(spare.value)
    B, L, G, H, d, r = c.batch, c.n_layers, c.group, c.n_kv_heads, c.head_dim, c.rank
    h, C, T, nL, nC = c.mlp_hidden, c.chunk, c.tail_cap, c.n_live, c.n_ctx // c.chunk
    R = int(src.n_records)
    int8 = c.store == 1
    dt = torch.float32 if c.dtype == 0 else torch.bfloat16
    tail_dt = torch.bfloat16 if int8 else dt
    codes = {torch.int8: "|i1", torch.int16: "<i2", torch.int32: "<i4", torch.float16: "<f2",
             torch.float32: "<f4"}

    def wrap(ptr, shape, dtype):
        if not ptr:
            return None
        base = torch.int16 if dtype == torch.bfloat16 else dtype
        t = torch.as_tensor(_DeviceArray(ptr, shape, codes[base]), device="cuda")
        return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t

    def live(t, n):   # the first n entries along the unit's axis
        return None if t is None else t[:, :, :, :n]

    arrays = {
        "coeff": live(wrap(src.coeff, (B, L // G, H, (nL + S_) * C, r), torch.int8 if int8 else dt), nL * C),
        "coeff_scale": live(wrap(src.coeff_scale, (B, L // G, H, (nL + S_) * C), torch.float16), nL * C)
        if int8 else None,
        "basis": wrap(src.basis, (L, H, r, d), dt),
        "w1": wrap(src.w1, (L, H, h, d), dt),
        "w2": wrap(src.w2, (L, H, d, h), dt),
        "summary": live(wrap(src.summary, (B, L // G, H, nL + S_, r), dt), nL),
        "slot": live(wrap(src.slot, (B, L // G, H, nC + S_), torch.int16), nC),
        "res_ptr": live(wrap(src.res_ptr, (B, L, H, nL + S_ + 1), torch.int32), nL + 1),
        "res_pos": wrap(src.res_pos, (R,), torch.int16) if R else torch.empty(0, dtype=torch.int16, device="cuda"),
        "res_val": wrap(src.res_val, (R, d), torch.int8 if int8 else dt),
        "res_scale": wrap(src.res_scale, (R,), torch.float16) if (int8 and R) else None,
        "tail_k": wrap(src.tail_k, (B, L, H, T, d), tail_dt),
        "tail_v": wrap(src.tail_v, (B, L, H, T, d), tail_dt),
        "tail_len": wrap(src.tail_len, (B,), torch.int32),
    }
    return cfg, arrays


def lowram_encode(cfg, n_resid: int, keys, values, basis, w1, w2, stream=None, out=None) -> dict:
    """Encode dense keys/values [B][L][Hkv][N][d] (bf16, CUDA) with the given basis, w1, w2
    (bf16, CUDA; layouts of ``lowram.h``) into the compressed storage arrays.  Allocates the
    outputs and the workspace with torch on the keys' device (or reuses ``out``, the dict a
    previous call with the same shapes returned) and returns the arrays by their
    ``lowram_cache_src`` names (no ``slot``: nothing is evicted)."""
    import torch
    c = config_struct(cfg)
    c.n_live = c.n_ctx // c.chunk
    if out is not None:
        return _encode_into(c, int(n_resid), keys, values, basis, w1, w2, out, stream)
    B, L, G, H, N, C = c.batch, c.n_layers, c.group, c.n_kv_heads, c.n_ctx, c.chunk
    r, d = c.rank, c.head_dim
    int8 = c.store == 1
    dev = keys.device
    n = B * L * H * int(n_resid)
    out = {
        "coeff": torch.empty(B, L // G, H, N, r, dtype=torch.int8 if int8 else torch.bfloat16, device=dev),
        "coeff_scale": torch.empty(B, L // G, H, N, dtype=torch.float16, device=dev) if int8 else None,
        "summary": torch.empty(B, L // G, H, N // C, r, dtype=torch.bfloat16, device=dev),
        "res_ptr": torch.empty(B, L, H, N // C + 1, dtype=torch.int32, device=dev),
        "res_pos": torch.empty(n, dtype=torch.int16, device=dev),
        "res_val": torch.empty(n, d, dtype=torch.int8 if int8 else torch.bfloat16, device=dev),
        "res_scale": torch.empty(n, dtype=torch.float16, device=dev) if int8 else None,
    }
    ws_bytes = int(lib().lowram_encode_workspace_bytes(ctypes.byref(c)))
    if ws_bytes == 0:
        raise LowramError(1, "lowram_encode_workspace_bytes", "invalid config for the encoder")
    out["_workspace"] = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    return _encode_into(c, int(n_resid), keys, values, basis, w1, w2, out, stream)


def _encode_into(c, n_resid, keys, values, basis, w1, w2, out, stream):
    ws = out["_workspace"]
    dst = LowramEncodeDstC()
    for k in LowramEncodeDstC._fields_:
        t = out[k[0]]
        setattr(dst, k[0], _ptr(t) if (t is not None and t.numel()) else None)
    _check(lib().lowram_encode(ctypes.byref(c), n_resid, _ptr(keys), _ptr(values), _ptr(basis),
                               _ptr(w1), _ptr(w2), ctypes.byref(dst), _ptr(ws), int(ws.numel()),
                               _stream(stream)),
           "lowram_encode")
    return out


class LowramCache:
    """Owning wrapper of a cache handle (destroys it on ``close``/garbage collection)."""

    def __init__(self, cfg, arrays, stream=None):
        self.cfg = cfg
        self.handle = lowram_cache_create(cfg, arrays, stream)

    @classmethod
    def from_synth(cls, cache, stream=None):
        """From an object with ``.cfg`` and the storage tensors as attributes."""
        cfg = cache.cfg
        cs = config_struct(cfg)
        try:
            cs.n_live = int(cfg.n_live)
        except AttributeError:
            pass
        return cls({n: getattr(cs, n) for n, _ in LowramConfigC._fields_}, cache, stream)

    def decode(self, q, out=None, sel: bool = False, layer0: int = 0,
               n_layers: Optional[int] = None, path: int = PATH_AUTO, stream=None):
        import torch
        if n_layers is None:
            n_layers = int(q.shape[0])
        if out is None:
            out = torch.empty_like(q)
        s = None
        if sel:
            c = self.cfg
            s = torch.empty(n_layers, _get(c, "batch"), _get(c, "n_kv_heads"), _get(c, "top_k"),
                            dtype=torch.int32, device=q.device)
        lowram_decode_attn(self.handle, layer0, n_layers, q, out, s, path, stream)
        return (out, s) if sel else out

    def select(self, q, layer0: int = 0, n_layers: Optional[int] = None, stream=None):
        import torch
        c = self.cfg
        if n_layers is None:
            n_layers = int(q.shape[0])
        nC = _get(c, "n_ctx") // _get(c, "chunk")
        scores = torch.empty(n_layers, _get(c, "batch"), _get(c, "n_kv_heads"), nC,
                             dtype=torch.float32, device=q.device)
        sel = torch.empty(n_layers, _get(c, "batch"), _get(c, "n_kv_heads"), _get(c, "top_k"),
                          dtype=torch.int32, device=q.device)
        lowram_select_chunks(self.handle, layer0, n_layers, q, scores, sel, stream)
        return scores, sel

    def append(self, k_new, v_new, stream=None) -> None:
        """Append one decode step's k, v [L][B][Hkv][d] to every sequence's raw tail."""
        lowram_cache_append(self.handle, k_new, v_new, stream)

    def repack(self, n_resid: int, stream=None) -> None:
        """Compress the oldest chunk of every tail (synchronous); the config grows by a chunk."""
        lowram_cache_repack(self.handle, n_resid, stream)
        cfg, _ = lowram_cache_view(self.handle)
        if isinstance(self.cfg, dict):
            self.cfg = dict(self.cfg, n_ctx=cfg["n_ctx"], n_live=cfg["n_live"])
        else:
            self.cfg = cfg

    def view(self):
        """(config dict, arrays dict) of the cache's own device arrays (see lowram_cache_view)."""
        return lowram_cache_view(self.handle)

    def bytes(self) -> dict:
        return lowram_cache_bytes(self.handle)

    def validate(self, stream=None) -> int:
        return lowram_cache_validate(self.handle, stream)

    @property
    def last_path(self) -> int:
        return lowram_cache_last_path(self.handle)

    @property
    def last_launches(self) -> int:
        return lowram_cache_last_launches(self.handle)

    def close(self) -> None:
        if getattr(self, "handle", 0):
            lowram_cache_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
