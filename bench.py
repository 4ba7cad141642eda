"""Benchmark: decode-time attention over a LowRAM-compressed KV cache on B200.

One step = one all-layer decode call (steps 1-5 for every layer and sequence) of the
32K-context Llama-3.1-8B-shaped workload (batch 4, bf16), inputs resident in HBM.  The
metric is queries/s, one query = one (sequence, layer) decode-attention evaluation over all
32 query heads.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lowram|reference]
                  [--config NAME] [--path auto|simt|tc] [--sweep]

Multi-GPU: one process per GPU (torchrun); every rank holds its own replica of the
workload (different seeds) and no collective runs on the data path ("weak" scaling);
the reported time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import lowram_synth as S  # noqa: E402

METRIC = "decode-attn queries/s over compressed KV at 32K ctx; achieved % of HBM roofline"
NOMINAL_HBM_GBS = 8000.0   # the metric's roofline denominator (B200 HBM3e, nominal)
DEFAULT_CONFIG = "llama8b_32k_bf16"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lowram", choices=["lowram", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--sweep", action="store_true",
                    help="also run the batch sweep 1,4,16,32,64 (extra JSON lines)")
    ap.add_argument("--dense", action="store_true",
                    help="only the uncompressed bf16 dense-KV baseline at its largest batch")
    ap.add_argument("--encode", action="store_true",
                    help="only the prefill-side encoder (dense K, V -> compressed cache) of the workload")
    ap.add_argument("--dense-batch", type=int, default=0,
                    help="with --dense: this batch instead of the largest that fits (profiling)")
    ap.add_argument("--repack", action="store_true",
                    help="only the decode-loop upkeep: C tail appends and one chunk re-pack per step")
    ap.add_argument("--shards", type=int, default=0,
                    help="context-sharded decode of the workload over this many chunk shards: one shard "
                         "per rank under torchrun (NCCL gathers), else every shard on this one GPU")
    ap.add_argument("--reuse", action="store_true",
                    help="decode steps whose selections persist, through a store of rebuilt chunks, at "
                         "several drift rates (one JSON line each) next to the plain decode of the same steps")
    ap.add_argument("--reuse-drift", type=float, action="append", default=None,
                    help="with --reuse: this drift rate only (repeatable)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ------------------------------------------------------------------------ environment

def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(x: float, ws: int, op: str) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, ws: int) -> float:
    """The slowest rank's time (every multi-GPU number is timed as the max over ranks)."""
    return _reduce(x, ws, "max")


def replica_config(cfg, rank: int):
    """Each rank decodes its own replica of the workload (own seed): no data-path exchange."""
    return cfg if rank == 0 else cfg.replace(seed=cfg.seed + 7919 * rank)


def aggregate_rate(queries_per_rank: float, ms_total: float, ws: int):
    """Whole-job throughput: all ranks' queries over the slowest rank's time."""
    ms = max_over_ranks(ms_total, ws)
    total_q = _reduce(queries_per_rank, ws, "sum")
    return total_q / (ms / 1e3), ms


# DRAM traffic of the tensor-core attend kernel per launch (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture:
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum \
#       --clock-control none -k regex:attend_tc -s 1 -c 1 --csv --log-file dram_b1.csv \
#       python bench.py --config llama8b_32k_bf16_b1 --steps 1 --warmup 1 --no-cpu-baseline
# 343.92 MB on that 256-unit case, scaled by the units of the named workload: 1024, x4).
# The figure stands only while the kernel's sources are the captured ones, so it carries
# their hash.
ATTEND_TC_SOURCES = ("attend_tc.cu", "tc_ptx.cuh", "lowram_internal.cuh")
# The int8 + eviction workload's figure: 78.39 MB on its 128-unit case
#   ncu --set full --clock-control none -k regex:attend_tc -s 3 -c 1 -o prof_i8 \
#       python bench.py --config llama8b_64k_int8_evict_b2_l8 --steps 3 --warmup 3 --no-cpu-baseline
# scaled by its 2048 units (x16).
MEASURED_TRAFFIC = {
    "llama8b_32k_bf16": {"bytes": 1375687680, "sources_sha1": "44abd08d2b474f45a6bc2b362f1604ef429b0fe0"},
    "llama8b_64k_int8_evict": {"bytes": 1254232064, "sources_sha1": "44abd08d2b474f45a6bc2b362f1604ef429b0fe0"},
}


def measured_traffic(workload: str, path: str):
    """ncu DRAM bytes per attend launch, or None (other path, workload or kernel version)."""
    rec = MEASURED_TRAFFIC.get(workload)
    if rec is None or path != "tc":
        return None
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kv_cache_compression_lowram_b200", "csrc")
    for f in ATTEND_TC_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return rec["bytes"] if h.hexdigest() == rec["sources_sha1"] else None


def tensor_peak_sustained() -> float:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops_sustained"])
    return 1400.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for _, _, flags in rows:
            for n, v in zip(names, flags):
                if v.lower() == "active":
                    seen.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "reasons": sorted(seen), "samples": len(rows)}


# ------------------------------------------------------------------- byte accounting

def algorithmic_bytes(cfg, cache_host: dict, sel: np.ndarray, layer0: int, n_layers: int) -> dict:
    """Bytes the method must move for one decode call, counted per unit (sequence, layer, KV
    head) by the hot path's byte formula, from the call's actual selection.

    Per unit: the chunk summaries it scores (n_live rows of r) and, with eviction, its slot
    map; the coefficient rows of its k selected chunks (+ int8 row scales); the residual
    records of those chunks (values, positions, int8 scales) and k+1 CSR offsets; its raw
    tail (actual length); q and out.  Once per (layer, KV head): the basis, the folded W1'
    (h x r, what the kernels read in place of W1) and W2.  "attend" is the chunk-attention
    kernel's share: coefficient rows, records, offsets and W1'.  "unique_coeff" is for
    reference only: the coefficient bytes if rows that several layers of one group select
    were read once per group (the rows are shared by the group's layers).
    """
    B, Hkv, g, d, r, h = cfg.batch, cfg.n_kv_heads, cfg.q_per_kv, cfg.head_dim, cfg.rank, cfg.mlp_hidden
    C, k, T = cfg.chunk, cfg.top_k, cfg.tail_cap
    s = 4 if cfg.dtype == "f32" else 2
    i8 = cfg.store == "int8"
    sa = 1 if i8 else s
    row_bytes = C * (r * sa + (2 if i8 else 0))
    res_ptr = cache_host["res_ptr"]
    slot = cache_host["slot"]
    tail_len = cache_host["tail_len"]
    coeff = 0
    resid = 0
    groups_seen = {}
    for li in range(n_layers):
        l = layer0 + li
        grp = l // cfg.group
        for b in range(B):
            for hk in range(Hkv):
                chosen = groups_seen.setdefault((b, grp, hk), set())
                for c in sel[li, b, hk]:
                    sl = int(slot[b, grp, hk, c])
                    chosen.add(sl)
                    n = int(res_ptr[b, l, hk, sl + 1] - res_ptr[b, l, hk, sl])
                    resid += n * (d * sa + 2 + (2 if i8 else 0))
                coeff += k * row_bytes
    n_units = n_layers * B * Hkv
    ptrs = n_units * (k + 1) * 4
    unique_coeff = sum(len(ch) for ch in groups_seen.values()) * row_bytes
    summaries = n_units * cfg.n_live * r * s
    slotmap = n_units * cfg.n_chunks * 2 if cfg.n_live < cfg.n_chunks else 0
    tail = sum(2 * int(tail_len[b]) * d * (2 if i8 else s) for b in range(B)) * n_layers * Hkv
    qo = 2 * n_units * g * d * s
    w1f = n_layers * Hkv * h * r * (2 if s == 2 else 4)
    weights = n_layers * Hkv * (r * d * s + d * h * s) + w1f
    total = coeff + resid + ptrs + summaries + slotmap + tail + qo + weights
    attend = coeff + resid + ptrs + w1f
    return {"total": total, "attend": attend, "coeff": coeff, "residual": resid,
            "summary": summaries, "tail": tail, "weights": weights, "unique_coeff": unique_coeff}


# ---------------------------------------------------------------------- CPU oracle leg

def oracle_rate(cfg, cache, q, budget_s: float = 15.0, seed: int = 0):
    """Time the fp64 oracle on a bounded sample of units; returns (queries/s, sample desc,
    threads used)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    npc = S.cache_to_numpy(cache)
    oc = O.OracleCache(npc)
    qf = q.detach().cpu().double().numpy()
    rng = np.random.default_rng(seed)
    units = [(li, b, h) for li in range(q.shape[0]) for b in range(cfg.batch)
             for h in range(cfg.n_kv_heads)]
    order = rng.permutation(len(units))
    done = 0
    t0 = time.perf_counter()
    for i in order:
        li, b, h = units[i]
        O.decode_unit(oc, b, li, h, qf[li, b, h * cfg.q_per_kv:(h + 1) * cfg.q_per_kv])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    queries = done / cfg.n_kv_heads
    return queries / dt, f"{done} of {len(units)} units (seeded), {dt:.1f} s", threads


# --------------------------------------------------------------------------- lowram

def run_lowram(args, ws, rank, local):
    import kv_cache_compression_lowram_b200 as K
    cfg = replica_config(S.CONFIGS[args.config], rank)
    dev = torch.device("cuda", local)
    torch.manual_seed(0)
    cache = S.make_cache(cfg, device=dev)
    q = S.make_queries(cache)
    lc = K.LowramCache.from_synth(cache)
    path = {"auto": K.PATH_AUTO, "simt": K.PATH_SIMT, "tc": K.PATH_TC}[args.path]
    out = torch.empty_like(q)
    sel = torch.empty(cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.top_k, dtype=torch.int32,
                      device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        K.lowram_decode_attn(lc.handle, 0, cfg.n_layers, q, out, sel, path)
    torch.cuda.synchronize()
    launches_per_step = lc.last_launches
    used_path = {1: "simt", 2: "tc"}.get(lc.last_path, "?")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    queries_step = cfg.batch * cfg.n_layers
    clocks = ClockSampler(local)
    barrier(ws)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    # (1) eager calls with the library's stage events: per-kernel launch durations for the
    # roofline (the events sit between the kernels, so this pass is a little slower)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        K.lowram_cache_set_stage_events(lc.handle, evs[i])
        K.lowram_decode_attn(lc.handle, 0, cfg.n_layers, q, out, sel, path)
    end.record(stream)
    torch.cuda.synchronize()
    K.lowram_cache_set_stage_events(lc.handle, None)
    eager_ms_total = start.elapsed_time(end)
    stage_ms = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j in range(3)]
    # (2) the timed steps: the same call captured once in a CUDA graph and replayed (the
    # library launches only on the caller's stream, with no synchronisation and no
    # allocation); if capture is not possible the eager pass is the measurement
    graph_ms, graph_err = None, None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            K.lowram_decode_attn(lc.handle, 0, cfg.n_layers, q, out, sel, path)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
    except Exception as exc:
        g = None
        graph_err = str(exc).splitlines()[0][:200] if str(exc) else type(exc).__name__
    # every rank takes the same collective steps, whether or not its capture worked
    barrier(ws)
    torch.cuda.synchronize()
    if g is not None:
        gs, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gs.record(stream)
        for _ in range(args.steps):
            g.replay()
        ge.record(stream)
        torch.cuda.synchronize()
        graph_ms = gs.elapsed_time(ge)
        del g
    barrier(ws)
    clk = clocks.stop()
    eager_value, eager_total = aggregate_rate(queries_step * args.steps, eager_ms_total, ws)
    gval, gtotal = aggregate_rate(queries_step * args.steps, graph_ms if graph_ms is not None else 1e30, ws)
    graph_ok = graph_ms is not None and gtotal < 1e29
    value, ms_total = (gval, gtotal) if graph_ok else (eager_value, eager_total)
    ms_step = ms_total / args.steps
    timing = {"timed": "cuda graph replays" if graph_ok else "eager calls",
              "eager_ms_per_step": round(eager_total / args.steps, 4), "eager_value": round(eager_value, 1)}
    if not graph_ok:
        timing["graph_unavailable"] = graph_err or "capture failed on another rank"

    # end to end through the host entry point: pinned q in, pinned out back, every step
    q_h = q.cpu().pin_memory()
    out_h = torch.empty_like(q_h).pin_memory()
    for _ in range(2):
        K.lowram_decode_attn_host(lc.handle, 0, cfg.n_layers, q_h, out_h)
    barrier(ws)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e2e_steps = max(3, args.steps // 2)
    for _ in range(e2e_steps):
        K.lowram_decode_attn_host(lc.handle, 0, cfg.n_layers, q_h, out_h)
    e2e_ms = (time.perf_counter() - t0) * 1e3 / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, ws)

    host = {"res_ptr": cache.res_ptr.cpu().numpy(), "slot": cache.slot.cpu().numpy().astype(np.int64),
            "tail_len": cache.tail_len.cpu().numpy()}
    ab = algorithmic_bytes(cfg, host, sel.cpu().numpy(), 0, cfg.n_layers)
    peak, peak_kind = peaks()
    attend_ms = stage_ms[1]
    achieved = ab["attend"] / (attend_ms / 1e3) / 1e9
    call_gbs = ab["total"] / (ms_step / 1e3) / 1e9
    qbytes = q.numel() * q.element_size()
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "queries/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype if cfg.store == "native" else "int8+bf16",
        "data": "synthetic (seeded generator; shapes of the named workload, no weights or datasets)",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_layers": cfg.n_layers,
                   "n_ctx": cfg.n_ctx, "chunk": cfg.chunk, "top_k": cfg.top_k, "rank": cfg.rank,
                   "kv_heads": cfg.n_kv_heads, "q_heads": cfg.n_q_heads, "head_dim": cfg.head_dim,
                   "mlp_hidden": cfg.mlp_hidden, "tail": cfg.tail_cap, "resid_frac": cfg.resid_frac,
                   "store": cfg.store, "evict_frac": cfg.evict_frac, "path": used_path,
                   "parallelism": f"replicas x{ws}",
                   "l2": "inputs larger than L2 (%.2f GB of algorithmic bytes per step)" % (ab["total"] / 1e9)},
        "roofline": {"bound": "hbm", "kernel": "attend_" + used_path,
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": measured_traffic(cfg.name, used_path),
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": ab["attend"],
                     "launch_ms": round(attend_ms, 4)},
        # the metric's own roofline: the whole call's algorithmic bytes per step over the
        # timed ms_per_step, against the nominal 8 TB/s and against the measured copy peak
        "call_roofline": {"algorithmic_bytes": ab["total"], "achieved_gbs": round(call_gbs, 1),
                          "frac_of_8000_gbs": round(call_gbs / NOMINAL_HBM_GBS, 4),
                          "frac_of_measured": round(call_gbs / peak, 4),
                          "unique_coeff_bytes": ab["unique_coeff"],
                          "stage_ms": {"select_tail": round(stage_ms[0], 4),
                                       "attend": round(stage_ms[1], 4),
                                       "combine": round(stage_ms[2], 4)}},
        "e2e": {"value": round(queries_step * ws / (e2e_ms / 1e3), 1), "unit": "queries/s",
                "h2d_bytes_per_step": qbytes, "d2h_bytes_per_step": qbytes},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "timing": timing,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, sample, threads = oracle_rate(cfg, cache, q)
        line["cpu_baseline"] = {"value": round(rate, 3), "unit": "queries/s", "cores": threads,
                                "kind": "oracle", "sample": sample}
    lc.close()
    return line


def run_dense(args, ws, rank, local, cfg_name=DEFAULT_CONFIG):
    """Uncompressed bf16 decode attention over the same context (N + T tokens) at the largest
    batch whose dense cache fits in device memory: the baseline of the batch sweep."""
    import kv_cache_compression_lowram_b200 as K
    cfg = S.CONFIGS[cfg_name]
    dev = torch.device("cuda", local)
    S_ = cfg.n_ctx + cfg.tail_cap
    per_seq = 2 * cfg.n_layers * cfg.n_kv_heads * S_ * cfg.head_dim * 2
    free, _ = torch.cuda.mem_get_info(dev)
    B = max(1, int((free - 6e9) // per_seq))
    if getattr(args, "dense_batch", 0) > 0:
        B = min(B, args.dense_batch)
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed + 17 + rank)
    k = torch.empty(B, cfg.n_layers, cfg.n_kv_heads, S_, cfg.head_dim, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    for b in range(B):   # per sequence, to keep the fp32 temporaries small
        k[b] = torch.randn(k.shape[1:], generator=gen, device=dev).to(torch.bfloat16)
        v[b] = (0.1 * torch.randn(v.shape[1:], generator=gen, device=dev)).to(torch.bfloat16)
    q = (torch.randn(cfg.n_layers, B, cfg.n_q_heads, cfg.head_dim, generator=gen, device=dev)
         / math.sqrt(cfg.head_dim)).to(torch.bfloat16)
    out = torch.empty_like(q)
    for _ in range(args.warmup):
        K.lowram_dense_decode_attn(k, v, q, out)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    clocks = ClockSampler(local)
    barrier(ws)
    clocks.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        K.lowram_dense_decode_attn(k, v, q, out)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    value, ms_total = aggregate_rate(B * cfg.n_layers * steps, start.elapsed_time(end), ws)
    ms_step = ms_total / steps
    bytes_step = k.numel() * 2 * 2 + q.numel() * 2 * 2
    peak, peak_kind = peaks()
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "queries/s", "n_gpus": ws, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "impl": "dense_baseline",
        "config": {"workload": f"dense_bf16_{cfg.name}_b{B}", "batch": B, "n_layers": cfg.n_layers,
                   "tokens": S_, "kv_heads": cfg.n_kv_heads, "q_heads": cfg.n_q_heads,
                   "head_dim": cfg.head_dim, "dense_cache_gb": round(k.numel() * 4 / 1e9, 2)},
        "roofline": {"bound": "hbm",
                     "kernel": "dense_tc_kernel" if cfg.head_dim == 128 else "dense_kernel", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_kind": peak_kind},
        "gpu_launches": steps, "clocks": clk,
    }
    del k, v
    torch.cuda.empty_cache()
    return line


ENC_METRIC = "prefill tokens/s encoded (dense K,V -> compressed cache, all layers and KV heads)"


def encode_flops(cfg) -> float:
    """Arithmetic of one encode call: the group projections (2 G d r per token and group),
    and the predictor, evaluated twice (residual norms, then the flagged tokens' records),
    2 * 2 h (r + d) per token and layer."""
    pos = cfg.batch * cfg.n_kv_heads * cfg.n_ctx
    proj = pos * cfg.n_groups * cfg.group * cfg.head_dim * cfg.rank * 2
    pred = pos * cfg.n_layers * 2 * 2 * cfg.mlp_hidden * (cfg.rank + cfg.head_dim)
    return float(proj + pred)


def encode_oracle_rate(cfg, Kd, Vd, weights, budget_s: float = 20.0):
    """The encoder oracle on (b, group, KV head) slices until the budget is spent; returns
    (prefill tokens/s scaled to the whole workload, sample description, threads)."""
    import dataclasses as dc
    import oracle.encode as E
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    G = cfg.group
    sub = dc.asdict(cfg.replace(name="enc_slice", batch=1, n_layers=G, n_kv_heads=1))
    f64 = lambda t: t.float().double().cpu().numpy()
    basis, w1, w2 = weights
    done, t0 = 0, time.perf_counter()
    slices = [(b, grp, h) for b in range(cfg.batch) for grp in range(cfg.n_groups) for h in range(cfg.n_kv_heads)]
    rng = np.random.default_rng(0)
    for i in rng.permutation(len(slices)):
        b, grp, h = slices[i]
        ls = slice(grp * G, (grp + 1) * G)
        E.encode(sub, f64(Kd[b:b + 1, ls, h:h + 1]), f64(Vd[b:b + 1, ls, h:h + 1]), f64(basis[ls, h:h + 1]),
                 f64(w1[ls, h:h + 1]), f64(w2[ls, h:h + 1]), cfg.n_resid)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    # a slice is 1 / (groups * KV heads) of a sequence's encode
    tokens = done * cfg.n_ctx / (cfg.n_groups * cfg.n_kv_heads)
    return tokens / dt, f"{done} of {len(slices)} (b, group, KV head) slices, {dt:.1f} s", threads


def run_encode(args, ws, rank, local):
    """The prefill-side encoder on the workload's dense keys and values (resident in HBM)."""
    import kv_cache_compression_lowram_b200 as K
    cfg = replica_config(S.CONFIGS[args.config], rank).replace(evict_frac=0.0)
    dev = torch.device("cuda", local)
    Kd, Vd = S.make_dense_kv(cfg, device=dev)
    weights = [t.to(torch.bfloat16) for t in S.make_weights(cfg)]
    wd = [t.to(dev).contiguous() for t in weights]
    out = K.lowram_encode(cfg, cfg.n_resid, Kd, Vd, *wd)
    for _ in range(max(0, args.warmup - 1)):
        K.lowram_encode(cfg, cfg.n_resid, Kd, Vd, *wd, out=out)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    clocks = ClockSampler(local)
    barrier(ws)
    clocks.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        K.lowram_encode(cfg, cfg.n_resid, Kd, Vd, *wd, out=out)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    value, ms_total = aggregate_rate(cfg.batch * cfg.n_ctx * steps, start.elapsed_time(end), ws)
    ms_step = ms_total / steps
    flops = encode_flops(cfg)
    if cfg.store == "native" or cfg.chunk == 128:
        # the projection and the predictor (all but a few % of the flops) run on tcgen05
        # tensor cores in bf16 / fp16 (int8 stores: the stored rows dequantised to fp16 on
        # chip): the measured sustained bf16 GEMM rate; fp16 runs at the same nominal rate
        bound, peak, peak_kind = "tensor", tensor_peak_sustained(), "measured (bf16, sustained)"
    else:
        # int8 stores: CUDA-core fp32 kernels; 148 SMs x 128 FMA lanes x 2 flops x the
        # maximum SM clock
        bound, peak_kind = "alu", "derived (fp32 FMA lanes x clock)"
        peak = 148 * 128 * 2 * ((clk or {}).get("sm_max_mhz") or 1965.0) * 1e6 / 1e12
    achieved = flops / (ms_step / 1e3) / 1e12
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        rate, sample, threads = encode_oracle_rate(cfg, Kd, Vd, weights)
        cpu = {"value": round(rate, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": sample}
    return {
        "metric": ENC_METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.store == "native" or cfg.chunk == 128 else "f32",
        "data": "synthetic", "impl": "encoder",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_layers": cfg.n_layers, "n_ctx": cfg.n_ctx,
                   "kv_heads": cfg.n_kv_heads, "rank": cfg.rank, "chunk": cfg.chunk, "store": cfg.store,
                   "n_resid": cfg.n_resid, "dense_kv_gb": round(Kd.numel() * 4 / 1e9, 2),
                   "l2": "inputs larger than L2"},
        "roofline": {"bound": bound, "kernel": "encode (all kernels of the call)", "achieved": round(achieved, 2),
                     "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": None, "flops_per_call": flops, "peak_kind": peak_kind},
        "cpu_baseline": cpu, "e2e": None, "gpu_launches": steps * 5, "clocks": clk,
    }


REPACK_METRIC = "chunk re-packs/s (the oldest C tail tokens of every sequence, layer and KV head -> one compressed chunk)"


def repack_oracle_rate(cfg, n_res: int, budget_s: float = 20.0):
    """The re-pack oracle on one-sequence, one-layer-group slices of the workload (all KV
    heads) until the budget is spent; returns (re-packs/s scaled to the whole workload by the
    unit count, sample description, threads)."""
    import oracle.repack as RP
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    sub = cfg.replace(name=cfg.name + "_slice", batch=1, n_layers=cfg.group)
    npc = S.cache_to_numpy(S.make_cache(sub, device="cuda" if torch.cuda.is_available() else "cpu",
                                        tail_len=[cfg.chunk]))
    done, t0 = 0, time.perf_counter()
    while True:
        RP.repack(npc, n_res)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    share = (sub.batch * sub.n_layers) / (cfg.batch * cfg.n_layers)
    return done * share / dt, f"{done} re-packs of a (1 sequence, {cfg.group} layers, {cfg.n_kv_heads} KV heads) slice, {dt:.1f} s", threads


def run_repack(args, ws, rank, local):
    """Decode-loop upkeep on the workload: one step = a re-pack of the full tails into a new
    chunk and C appends of a decode token to every tail (the cache grows a chunk per step).
    The first re-pack re-lays the cache with room for more chunks (timed on its own); the
    timed steps re-pack in place."""
    import kv_cache_compression_lowram_b200 as K
    cfg = replica_config(S.CONFIGS[args.config], rank)
    C, T = cfg.chunk, cfg.tail_cap
    assert T >= C, "the workload's tail cannot hold a chunk"
    dev = torch.device("cuda", local)
    n_res = max(1, int(round(cfg.resid_frac * C)))
    cache = S.make_cache(cfg, device=dev, tail_len=[C] * cfg.batch)
    lc = K.LowramCache.from_synth(cache)
    del cache
    torch.cuda.synchronize()
    shape = (cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.head_dim)
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed + 31 + rank)
    kv_dev = [((torch.randn(shape, generator=gen, device=dev) * 0.3).to(torch.bfloat16),
               (torch.randn(shape, generator=gen, device=dev) * 0.1).to(torch.bfloat16)) for _ in range(C)]
    kv_host = [(k.cpu().pin_memory(), v.cpu().pin_memory()) for k, v in kv_dev[:8]]
    stream = torch.cuda.current_stream()
    U = cfg.batch * cfg.n_layers * cfg.n_kv_heads
    NG = cfg.n_layers // cfg.group
    sa = 1 if cfg.store == "int8" else 2

    def chunk_arrays():
        b = lc.bytes()
        return b["coeff"] + b["summary"] + b["residual"] + b["index"]

    # bytes every re-pack must move: the tail chunk read, the new chunk's stored arrays
    # written, the layer weights read by the predictor
    new_chunk = (cfg.batch * NG * cfg.n_kv_heads * (C * cfg.rank * sa + (2 * C if sa == 1 else 0) + cfg.rank * 2)
                 + U * n_res * (cfg.head_dim * sa + 2 + (2 if sa == 1 else 0)) + U * 4)
    weights = cfg.n_layers * cfg.n_kv_heads * (cfg.rank + 2 * cfg.mlp_hidden) * cfg.head_dim * 2
    inplace_bytes = 2 * U * C * cfg.head_dim * 2 + new_chunk + weights

    def appends(host: bool):
        for i in range(C):
            if host:   # end to end: the step's k, v arrive from pinned host memory
                k, v = kv_host[i % len(kv_host)]
                kd, vd = kv_dev[i]
                kd.copy_(k, non_blocking=True)
                vd.copy_(v, non_blocking=True)
                lc.append(kd, vd)
            else:
                lc.append(*kv_dev[i])

    # the first re-pack re-lays the cache (room for `spare` more chunks)
    before = chunk_arrays()
    t0 = time.perf_counter()
    lc.repack(n_res)
    relayout_ms = (time.perf_counter() - t0) * 1e3
    relayout_bytes = before + chunk_arrays() + 2 * U * C * cfg.head_dim * 2 + weights
    spare = lc.view()[0]["spare_chunks"]
    appends(False)
    for _ in range(args.warmup):
        lc.repack(n_res)
        appends(False)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10, lc.view()[0]["spare_chunks"] - 3))
    clocks = ClockSampler(local)
    barrier(ws)
    clocks.start()
    time.sleep(0.3)
    rp_ms, ap_ms = [], []
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(steps):
        ev[0].record(stream)
        lc.repack(n_res)                         # synchronous, in place
        ev[1].record(stream)
        appends(False)
        ev[2].record(stream)
        torch.cuda.synchronize()
        rp_ms.append(ev[0].elapsed_time(ev[1]))
        ap_ms.append(ev[1].elapsed_time(ev[2]))
    clk = clocks.stop()
    ms_step = max_over_ranks(sum(rp_ms) / steps + sum(ap_ms) / steps, ws)
    value = _reduce(1.0, ws, "sum") / (ms_step / 1e3)
    ms_repack = sum(rp_ms) / steps
    achieved = inplace_bytes / (ms_repack / 1e3) / 1e9
    peak, peak_kind = peaks()
    # amortised over a cycle of one re-lay and `spare` in-place re-packs
    per_step_us = 1e3 * (spare * ms_repack + relayout_ms) / ((spare + 1) * C)
    # end to end: the appended tokens come from pinned host memory, timed on the host
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(3):
        lc.repack(n_res)
        appends(True)
    torch.cuda.synchronize()
    e2e_ms = (time.perf_counter() - t0) * 1e3 / 3
    h2d = C * 2 * cfg.n_layers * cfg.batch * cfg.n_kv_heads * cfg.head_dim * 2
    d2h = cfg.batch * 4 + 4 + 8        # tail lengths, the room flag, two error words
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        rate, sample, threads = repack_oracle_rate(cfg, n_res)
        cpu = {"value": round(rate, 4), "unit": "re-packs/s", "cores": threads, "kind": "oracle", "sample": sample}
    cfg_now, _ = lc.view()
    lc.close()
    return {
        "metric": REPACK_METRIC, "value": round(value, 2), "unit": "re-packs/s", "n_gpus": ws, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "upkeep",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_layers": cfg.n_layers, "n_ctx_start": cfg.n_ctx,
                   "n_ctx_end": cfg_now["n_ctx"], "chunk": C, "n_resid_per_chunk": n_res, "store": cfg.store,
                   "step": f"1 in-place re-pack + {C} appends", "spare_chunks_after_relayout": spare,
                   "l2": "inputs larger than L2"},
        "ms_per_repack_in_place": round(ms_repack, 3), "ms_per_relayout": round(relayout_ms, 2),
        "relayout_bytes": int(relayout_bytes), "us_per_append": round(1e3 * sum(ap_ms) / steps / C, 2),
        "repack_us_per_decode_step": round(per_step_us, 2),
        "roofline": {"bound": "hbm", "kernel": "in-place re-pack (whole synchronous call)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": None, "bytes_per_repack": int(inplace_bytes), "peak_kind": peak_kind},
        "cpu_baseline": cpu,
        "e2e": {"value": round(1e3 / e2e_ms, 2), "unit": "re-packs/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": steps * (2 * C + 11), "clocks": clk,
    }


def run_reference(args, ws, rank):
    """The oracle (fp64 numpy, host cores) on the same workload, bounded samples per step."""
    if rank != 0:
        return None
    cfg = S.CONFIGS[args.config]
    cache = S.make_cache(cfg, device="cuda" if torch.cuda.is_available() else "cpu")
    q = S.make_queries(cache)
    budget = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_rate(cfg, cache, q, budget_s=budget)
    rates = []
    samples = []
    threads = 1
    for i in range(args.steps):
        rate, sample, threads = oracle_rate(cfg, cache, q, budget_s=budget, seed=i + 1)
        rates.append(rate)
        samples.append(sample)
    value = statistics.mean(rates)
    ms_step = cfg.batch * cfg.n_layers / value * 1e3
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "queries/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_layers": cfg.n_layers,
                   "n_ctx": cfg.n_ctx},
        "cpu_baseline": {"value": round(value, 3), "unit": "queries/s", "cores": threads,
                         "kind": "oracle", "sample": samples[0] + f" per step, {args.steps} steps"},
        "e2e": {"value": round(value, 3), "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


SHARD_METRIC = "context-sharded decode-attn queries/s (one sequence's chunks split over shards)"


def run_shards(args, ws, rank, local):
    """Context-sharded decode of the workload: its chunks split into P equal contiguous ranges.

    Under torchrun (P = world size) each rank holds one shard and the protocol's two gathers
    are NCCL all-gathers; on one GPU the P shards run one after another on the same device and
    the gathers are device copies (torch.stack), so the time is that of P shards' kernels in
    sequence, not a multi-GPU time.  One step = phase 1 on every shard, gather, phase 2,
    gather, merge.  Timed with CUDA events, max over ranks."""
    import kv_cache_compression_lowram_b200 as K
    from kv_cache_compression_lowram_b200.sharded import ShardDecoder, all_gather
    cfg = S.CONFIGS[args.config]
    P = args.shards if ws == 1 else ws
    if ws > 1 and args.shards not in (0, ws):
        raise SystemExit("--shards must equal the world size under torchrun")
    nC = cfg.n_chunks
    bounds = [nC * s // P for s in range(P + 1)]
    dev = torch.device("cuda", local)
    cache = S.make_cache(cfg, device=dev)            # the same seeded cache on every rank
    q = S.make_queries(cache)
    mine = range(P) if ws == 1 else [rank]
    decs = {}
    for s_ in mine:
        sh = S.shard_chunks(cache, bounds[s_], bounds[s_ + 1], keep_tail=(s_ == P - 1))
        decs[s_] = ShardDecoder(K.LowramCache.from_synth(sh), bounds[s_], P)
        del sh
    del cache
    torch.cuda.empty_cache()
    gather = all_gather() if ws > 1 else None

    def step():
        if ws > 1:
            return decs[rank].decode(q, gather=gather)[0]
        cands = [decs[s_].candidates(q) for s_ in range(P)]
        cs_all = torch.stack([c[0] for c in cands])
        ci_all = torch.stack([c[1] for c in cands])
        parts = torch.stack([decs[s_].partial(cs_all, ci_all)[0] for s_ in range(P)])
        return decs[0].merge(parts)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(local)
    barrier(ws)
    clocks.start()
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    queries = cfg.batch * cfg.n_layers * args.steps
    value, ms_total = aggregate_rate(queries / ws, start.elapsed_time(end), ws)
    for d in decs.values():
        d.cache.close()
    return {
        "metric": SHARD_METRIC, "value": round(value, 1), "unit": "queries/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_total / args.steps, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic", "impl": "lowram_sharded",
        "config": {"workload": cfg.name, "shards": P, "chunk_bounds": bounds,
                   "placement": "one shard per rank, NCCL all-gathers" if ws > 1 else
                   "all shards on one GPU in sequence, gathers as device copies"},
        "gpu_launches": (5 * P + 1) * args.steps if ws == 1 else 6 * args.steps, "clocks": clk,
    }


REUSE_METRIC = "decode-attn queries/s over compressed KV at 32K ctx, consecutive steps through a reuse store"
REUSE_DRIFTS = (0.0, 0.02, 0.1, 1.0)


def run_reuse(args, ws, rank, local):
    """Consecutive decode steps of the workload (``make_query_steps``: AR(1) query noise, rho =
    0.9, and per unit two target chunks that jump with probability ``drift`` per step) through
    a reuse store (capacity 2 U k entries, fill cap U k), at several drift rates, one JSON
    line each.  Each line also times the plain decode of the same steps; both eager calls
    timed with CUDA events (the queries change every step), inputs resident in HBM.  The
    store is warmed by the warm-up steps of the same sequence.  Per replica, no collective."""
    import kv_cache_compression_lowram_b200 as K
    cfg = replica_config(S.CONFIGS[args.config], rank)
    dev = torch.device("cuda", local)
    cache = S.make_cache(cfg, device=dev)
    lc = K.LowramCache.from_synth(cache)
    U = cfg.n_layers * cfg.batch * cfg.n_kv_heads
    cap, fill_cap = 2 * U * cfg.top_k, U * cfg.top_k
    stream = torch.cuda.current_stream()
    out = torch.empty(cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.head_dim, dtype=cfg.torch_dtype, device=dev)
    sel = torch.empty(cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.top_k, dtype=torch.int32, device=dev)
    lines = []
    for di, drift in enumerate(REUSE_DRIFTS):
        if args.reuse_drift and drift not in args.reuse_drift:
            continue
        steps = S.make_query_steps(cache, args.warmup + args.steps, 0.9, drift, seed_offset=100 + di)
        store = K.LowramReuse(lc, cap, fill_cap)
        for q in steps[:args.warmup]:
            K.lowram_decode_attn_reuse(store.handle, 0, cfg.n_layers, q, out, sel)
        torch.cuda.synchronize()
        c0 = store.counts()
        clocks = ClockSampler(local)
        barrier(ws)
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.3)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for q in steps[args.warmup:]:
            K.lowram_decode_attn_reuse(store.handle, 0, cfg.n_layers, q, out, sel)
        b.record(stream)
        torch.cuda.synchronize()
        reuse_ms = a.elapsed_time(b)
        launches = lc.last_launches
        c1 = store.counts()
        # the plain decode of the same steps
        for q in steps[:args.warmup]:
            K.lowram_decode_attn(lc.handle, 0, cfg.n_layers, q, out, sel)
        barrier(ws)
        torch.cuda.synchronize()
        a.record(stream)
        for q in steps[args.warmup:]:
            K.lowram_decode_attn(lc.handle, 0, cfg.n_layers, q, out, sel)
        b.record(stream)
        torch.cuda.synchronize()
        plain_ms = a.elapsed_time(b)
        clk = clocks.stop()
        store.close()
        del steps
        queries = cfg.batch * cfg.n_layers * args.steps
        value, ms_total = aggregate_rate(queries, reuse_ms, ws)
        pvalue, pms_total = aggregate_rate(queries, plain_ms, ws)
        hits, misses, fills = (c1[x] - c0[x] for x in ("hits", "misses", "fills"))
        # work per step by kind of chunk: a hit reads the coefficient tile and the stored
        # values and runs no predictor; a miss reads the tile and its residual records; a
        # fill reads them once more and writes the entry
        tile_b = cfg.chunk * cfg.rank * 2
        rec_b = round(cfg.resid_frac * cfg.chunk) * (cfg.head_dim * 2 + 2)
        entry_b = cfg.chunk * cfg.head_dim * 2
        work = {"silu_saved": round(hits / args.steps) * cfg.chunk * cfg.mlp_hidden,
                "hit_bytes": round(hits / args.steps) * (tile_b + entry_b),
                "miss_bytes": round(misses / args.steps) * (tile_b + rec_b),
                "fill_bytes": round(fills / args.steps) * (tile_b + rec_b + entry_b),
                "plain_bytes": round((hits + misses) / args.steps) * (tile_b + rec_b)}
        lines.append({
            "metric": REUSE_METRIC, "value": round(value, 1), "unit": "queries/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_total / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic (seeded temporal query recipe)", "impl": "lowram_reuse",
            "config": {"workload": cfg.name, "rho": 0.9, "drift": drift, "capacity": cap, "fill_cap": fill_cap,
                       "store_bytes": cap * cfg.chunk * cfg.head_dim * 2, "parallelism": f"replicas x{ws}"},
            "hit_rate": round(hits / max(1, hits + misses), 4), "fills_per_step": round(fills / args.steps, 1),
            "work_per_step": work,
            "plain": {"value": round(pvalue, 1), "ms_per_step": round(pms_total / args.steps, 4)},
            "speedup_vs_plain": round(pms_total / ms_total, 4),
            "gpu_launches": launches * args.steps, "clocks": clk,
        })
    lc.close()
    return lines


def main():
    args = parse()
    ws, rank, local = dist_init()
    if args.impl == "reference":
        line = run_reference(args, ws, rank)
    elif args.dense:
        line = run_dense(args, ws, rank, local)
    elif args.encode:
        line = run_encode(args, ws, rank, local)
    elif args.repack:
        line = run_repack(args, ws, rank, local)
    elif args.shards:
        line = run_shards(args, ws, rank, local)
    elif args.reuse:
        for ln in run_reuse(args, ws, rank, local):
            if rank == 0:
                print(json.dumps(ln), flush=True)
        line = None
    else:
        line = run_lowram(args, ws, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if args.sweep and args.impl == "lowram" and not (args.dense or args.encode or args.repack or args.shards
                                                      or args.reuse):
        import gc
        for b in (1, 4, 16, 32, 64):
            args.config = f"llama8b_32k_bf16_b{b}"
            args.no_cpu_baseline = True
            gc.collect()
            torch.cuda.empty_cache()
            line = run_lowram(args, ws, rank, local)
            if rank == 0:
                print(json.dumps(line), flush=True)
        gc.collect()
        torch.cuda.empty_cache()
        line = run_dense(args, ws, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
