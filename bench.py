#!/usr/bin/env python
"""DSA decode throughput at 128K context on B200: prints ONE JSON line.

A step is one dsa_index_topk_attn call (indexer -> Top-K -> sparse MLA) over
one batch of the long-context decode workload (8 sequences x 131072 cached
tokens, one query token each, K = 2048, 128 heads, FP8 paged index cache in a
2 Mi-token pool).  Inputs are synthetic and seeded (dsa_workloads.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank serves its own batch (weak scaling, no
collective on the data path; a MAX all-reduce of the timings only).
--impl reference times the fp64 CPU oracle on the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dsa_workloads import CONFIGS, make_workload  # noqa: E402

METRIC = "DSA decode tokens/s at 128K ctx"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes (read + write) per launch from ncu captures of the 128K decode
# workload, each valid only for the cache formats it was captured with and
# while the kernel's sources hash to what was captured: any edit turns the
# figure back into null.
NCU_CAPTURES = (
    # kernel, config keys that must match, bytes per launch, sources, digest
    ("index_scores", {"index_cache": "fp8_e4m3"}, 145.60e6, ("k_indexer.cu",), "6a6254d29a2242f3"),
    ("index_scores", {"index_cache": "mxfp8"}, 144.81e6, ("k_indexer.cu",), "6a6254d29a2242f3"),
    ("topk_filter", {}, 4.35e6, ("k_topk.cu",), "507b32e02ae94d9e"),
    ("sparse_mla", {"latent_cache": "bf16"}, 20.25e6, ("k_sparse_mla.cu",), "412a2a7f29ba3946"),
)
NCU_WORKLOAD = {"workload": "decode_b8_128k", "ctx": 131072}
CSRC = os.path.join(ROOT, "sparse_indexed_attention_b200", "csrc")


def source_digest(files) -> str:
    import hashlib
    m = hashlib.sha256()
    for f in (*files, "dsa_internal.cuh", "sm100.cuh"):
        with open(os.path.join(CSRC, f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def ncu_traffic(kernel: str, config: dict):
    """Captured DRAM traffic of `kernel` per launch for this `config` (the JSON
    line's config object), or None if not captured for it or stale."""
    for name, keys, nbytes, files, digest in NCU_CAPTURES:
        want = {**NCU_WORKLOAD, **keys}
        if name == kernel and all(config.get(k) == v for k, v in want.items()):
            return nbytes if source_digest(files) == digest else None
    return None


def index_cache(spec) -> str:
    """The index cache's format; MXFP8 overrides the per-row E4M3 flag."""
    return "mxfp8" if spec.ki_mx else ("fp8_e4m3" if spec.ki_fp8 else "bf16")


def data_desc(spec) -> str:
    return "synthetic (seeded" + (f", {spec.planted} planted keys per sequence)" if spec.planted else ")")


def index_row_bytes(spec) -> int:
    """Index-cache bytes per key: 128 codes + 4 scale bytes (one fp32, or four
    E8M0 bytes), or 128 bf16 values."""
    return 256 if index_cache(spec) == "bf16" else 132


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="decode_b8_128k", choices=list(CONFIGS))
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage-reps", type=int, default=20)
    ap.add_argument("--ctx", type=int, default=0,
                    help="override the workload's context length (profiling a smaller case of the same kernels)")
    ap.add_argument("--all-configs", action="store_true",
                    help="one JSON line per workload: fused-call time and the binding roofline of each stage")
    ap.add_argument("--no-all-configs", action="store_true",
                    help="leave out the per-workload summary that a 1-GPU headline line carries")
    ap.add_argument("--ki", choices=["workload", "mxfp8"], default="workload",
                    help="index-cache format: the workload's own (E4M3 + row scale for the headline) or MXFP8")
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="latent KV cache: bf16, or FP8 E4M3 with a power-of-two scale per 128-element tile")
    ap.add_argument("--select-in-indexer", action="store_true",
                    help="decode: select the Top-K inside the indexer kernel (DSA_SELECT_IN_INDEXER)")
    ap.add_argument("--only", choices=["index_scores", "topk", "sparse_mla", "fused"], default=None,
                    help="time one stage (or the fused call, eagerly) alone on the bench workload (profiling aid)")
    return ap.parse_args()


def dist_setup(args, backend=None):
    """World size, rank and local rank from the torchrun environment; for N > 1
    a process group (NCCL on GPUs, gloo without) with a short timeout."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def rank_spec(spec, rank: int):
    """The workload rank `rank` serves: same shape, its own seed (weak scaling)."""
    return spec.scaled(seed=spec.seed + 1000 * rank)


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.cmd = ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                        "-lms", "100"]
        except Exception:
            self.cmd = None

    def __enter__(self):
        if self.cmd:
            try:
                self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.thread = threading.Thread(target=self._read, daemon=True)
                self.thread.start()
                time.sleep(0.3)
            except Exception:
                self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def tensor_peak(kind: str):
    """Measured dense TFLOP/s: bf16 (burst), fp8 = 2 x bf16 (nominal ratio)."""
    try:
        with open(PEAKS_FILE) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        src = "measured"
    except Exception:
        bf16, src = 1590.0, "fallback"
    return (2.0 * bf16 if kind == "fp8" else bf16), src


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(wl, n_tokens: int):
    """The fp64 oracle on a bounded sample (the first n_tokens query tokens)."""
    from oracle import dsa_oracle as O
    from dsa_workloads import bits16
    seqs = O.Seqs(ctx_len=wl.ctx_len.astype(np.int64), q_seq_start=wl.q_seq_start.astype(np.int64),
                  page_table=wl.page_table, page_size=wl.spec.page_size)
    if wl.kI_scale is None:
        kI, sc = bits16(wl.kI), None
    else:
        kI, sc = wl.kI.numpy(), wl.kI_scale.numpy()
    qI, w, q = bits16(wl.qI), wl.w.numpy(), bits16(wl.q)
    kv = bits16(wl.kv) if wl.kv_scale is None else (wl.kv.numpy(), wl.kv_scale.numpy())
    toks = list(range(n_tokens))
    t0 = time.perf_counter()
    O.index_topk_attn(seqs, qI, w, kI, sc, q, kv, wl.spec.topk, wl.scale, tokens=toks)
    dt = time.perf_counter() - t0
    return dt, toks


# ---------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------


def workload_config(spec, wl, world: int) -> dict:
    """The `config` object of the JSON line, the same for both arms."""
    return {"workload": spec.name, "batch_per_gpu": spec.batch, "global_batch": wl.T * world,
            "ctx": int(wl.ctx_len[0]), "topk": spec.topk, "heads": spec.heads, "index_heads": spec.index_heads,
            "index_dim": spec.index_dim, "page_size": spec.page_size, "pool_tokens": wl.num_phys_pages * 64,
            "index_cache": index_cache(spec),
            "latent_cache": "fp8_e4m3_tile128" if spec.kv_fp8 else "bf16",
            "parallelism": f"dp{world}",
            "l2": "256 MiB buffer written before every timed GPU step"}


def bench_spec(args):
    """The workload both arms measure: the named config, with the index-cache
    format and context length the flags ask for."""
    spec = CONFIGS[args.config]
    if args.ki == "mxfp8":
        spec = spec.scaled(ki_mx=True)
    if args.kv == "fp8":
        spec = spec.scaled(kv_fp8=True)
    if args.ctx > 0:
        spec = spec.scaled(ctx=(args.ctx, args.ctx))
    return spec


def run_reference(args, world, rank):
    if rank != 0:
        return
    spec = bench_spec(args)
    wl = make_workload(spec)
    n_tok = wl.T                                   # one step = the whole batch, as in our arm
    for _ in range(args.warmup):
        cpu_baseline(wl, n_tok)
    times = []
    for _ in range(args.steps):
        dt, _ = cpu_baseline(wl, n_tok)
        times.append(dt)
    step_s = sum(times) / len(times)
    value = n_tok / step_s
    sample = (f"fp64 oracle, whole path for {n_tok} query token(s) of {spec.name} "
              f"(ctx {int(wl.ctx_len[0])}) per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": data_desc(spec),
            "config": workload_config(spec, wl, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def time_device(fn, steps, warmup, stream, flush):
    """Mean device time (ms) of fn over `steps` runs, L2 flushed before each."""
    for _ in range(warmup):
        fn()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def kernel_times(dsa, step, steps, stream, flush):
    """{kernel: [device ms per call]} over `steps` eager calls, L2 flushed before each."""
    per = {}
    dsa.dsa_launch_timing(True)
    try:
        for i in range(3 + steps):
            flush.fill_(i & 0xFF)
            step()
            got = dsa.dsa_last_launch_times()
            if i >= 3:
                for name, ms in got:
                    per.setdefault(name, []).append(ms)
    finally:
        dsa.dsa_launch_timing(False)
    torch.cuda.synchronize()
    return per


def roofline_entry(name, per, algorithmic_bytes, peak, peak_kind, config: dict):
    ms = statistics.mean(per[name])
    achieved = algorithmic_bytes / (ms / 1e3) / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": peak_kind, "algorithmic_bytes": algorithmic_bytes,
            "launch_us": ms * 1e3, "traffic": ncu_traffic(name, config)}


def run_only(args, dsa, wl, d, dev, stream, flush, world, fused=None):
    """One stage alone, `--steps` timed launches after `--warmup` (profiling aid)."""
    spec = wl.spec
    T, H, K = wl.T, spec.heads, spec.topk
    scores = torch.empty((T, (wl.max_ctx + 3) // 4 * 4), dtype=torch.float32, device=dev)
    row_len = torch.from_numpy((wl.token_pos() + 1).astype(np.int32)).to(dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev)
    dsa.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores)
    dsa.dsa_topk(scores, row_len, K, idx=idx)
    fns = {
        "index_scores": lambda: dsa.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores),
        "topk": lambda: dsa.dsa_topk(scores, row_len, K, idx=idx),
        "sparse_mla": lambda: dsa.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, idx, wl.scale, out=out, lse=lse,
                                                     kv_scale=d.kv_scale),
        "fused": fused,
    }
    times = time_device(fns[args.only], args.steps, args.warmup, stream, flush)
    if world == 1 or int(os.environ.get("RANK", "0")) == 0:
        print(json.dumps({"stage": args.only, "workload": spec.name, "us_mean": 1e3 * sum(times) / len(times),
                          "us_min": 1e3 * min(times), "launches": dsa.dsa_launches_in_last_call()}), flush=True)


def run_all_configs(args, dsa, dev, stream, flush):
    for line in all_config_lines(args, dsa, dev, stream, flush):
        print(json.dumps(line), flush=True)


def all_configs_summary(args, dsa, dev, stream, flush) -> dict:
    """The per-workload lines condensed for the headline line: time per call,
    tokens/s, launches and each stage's binding roofline fraction.  A failure
    is recorded in the summary; the headline line is printed regardless."""
    out = {}
    try:
        for ln in all_config_lines(args, dsa, dev, stream, flush):
            out[ln["config"]] = {
                "us_per_call": ln["us_per_call"], "tokens_per_s": ln["tokens_per_s"], "launches": ln["launches"],
                "stages": {k: {f: v[f] for f in ("bound", "us", "frac", "unit", "dtype") if f in v}
                           for k, v in ln["stages"].items()}}
    except Exception as exc:  # noqa: BLE001
        out["error"] = f"{type(exc).__name__}: {str(exc)[:160]}"
    return out


def all_config_lines(args, dsa, dev, stream, flush):
    """Every workload once: the fused call (graph replay, L2 flushed before each
    step) and per-kernel device times, each stage against its binding roofline."""
    from dsa_workloads import to_device
    hbm, hbm_src = hbm_peak()
    for name in CONFIGS:
        spec = CONFIGS[name].scaled(ki_mx=args.ki == "mxfp8", kv_fp8=args.kv == "fp8")
        wl = make_workload(spec)
        d = to_device(wl)
        T, H, K = wl.T, spec.heads, spec.topk
        out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((T, H), dtype=torch.float32, device=dev)
        op = dsa.DSA_OP_INDEX_TOPK_ATTN_FUSED if args.select_in_indexer else dsa.DSA_OP_INDEX_TOPK_ATTN
        ws = torch.zeros(dsa.dsa_workspace_size(op, d.seqs, K, H), dtype=torch.uint8, device=dev)

        def step():
            dsa.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, out=out, lse=lse,
                                    ws=ws, select_in_indexer=args.select_in_indexer, kv_scale=d.kv_scale)

        for _ in range(2):
            step()
        torch.cuda.synchronize()
        if dsa.dsa_check_error(ws) != dsa.DSA_OK:
            raise RuntimeError(f"device error flag set on {name}")
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        steps = 5 if T > 4096 else 20
        ms = statistics.mean(time_device(graph.replay, steps, 2, stream, flush))
        del graph
        kern = kernel_times(dsa, step, 3, stream, flush)
        us = {k: 1e3 * statistics.mean(v) for k, v in kern.items()}
        n = wl.token_pos() + 1
        pairs = int(n.sum())
        sel = int(np.minimum(n, K).sum())
        decode = spec.mode == "decode"
        stages = {}
        if "index_scores" in us:
            t_s = us["index_scores"] * 1e-6
            if decode:
                b = pairs * index_row_bytes(spec)
                stages["index_scores"] = {"bound": "hbm", "us": us["index_scores"], "achieved": b / t_s / 1e9,
                                          "peak": hbm, "unit": "GB/s", "frac": b / t_s / 1e9 / hbm}
            else:
                eight_bit = index_cache(spec) != "bf16"
                pk, src = tensor_peak("fp8" if eight_bit else "bf16")
                f = pairs * 16384
                stages["index_scores"] = {"bound": "tensor", "us": us["index_scores"], "achieved": f / t_s / 1e12,
                                          "peak": pk, "unit": "TFLOP/s", "frac": f / t_s / 1e12 / pk,
                                          "dtype": "fp8" if eight_bit else "bf16"}
        topk_us = sum(v for k, v in us.items() if k.startswith("topk"))
        b = pairs * 4 + T * K * 4
        if topk_us > 0:
            stages["topk"] = {"bound": "latency", "us": topk_us,
                              "hbm_frac_of_one_pass": b / (topk_us * 1e-6) / 1e9 / hbm}
        else:  # decode: the indexer kernel selects the Top-K itself
            stages["topk"] = {"bound": "latency", "us": 0.0, "inside": "index_scores"}
        attn_us = us.get("sparse_mla", 0.0) + us.get("sparse_mla_combine", 0.0)
        if attn_us:
            t_s = attn_us * 1e-6
            if decode:
                b = sel * (584 if spec.kv_fp8 else 1152)
                stages["sparse_mla"] = {"bound": "hbm", "us": attn_us, "achieved": b / t_s / 1e9, "peak": hbm,
                                        "unit": "GB/s", "frac": b / t_s / 1e9 / hbm}
            else:
                pk, src = tensor_peak("bf16")
                f = sel * 2 * H * (576 + 512)
                stages["sparse_mla"] = {"bound": "tensor", "us": attn_us, "achieved": f / t_s / 1e12, "peak": pk,
                                        "unit": "TFLOP/s", "frac": f / t_s / 1e12 / pk}
        line = {"config": name, "tokens": T, "us_per_call": ms * 1e3, "tokens_per_s": T / (ms / 1e3),
                "launches": dsa.dsa_launches_in_last_call(), "kernels_us": us, "stages": stages,
                "select_in_indexer": args.select_in_indexer,
                "peak_source": hbm_src, "timing": "graph replay, 256 MiB L2 flush before each step; "
                "kernels_us from events around each launch (serialised)"}
        del d, ws, out, lse
        torch.cuda.empty_cache()
        yield line


def run_ours(args, world, rank, local):
    import sparse_indexed_attention_b200 as dsa
    from dsa_workloads import to_device

    if args.all_configs:
        dev = torch.device("cuda", torch.cuda.current_device())
        run_all_configs(args, dsa, dev, torch.cuda.current_stream(dev),
                        torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev))
        return
    spec = rank_spec(bench_spec(args), rank)                         # each rank serves its own batch
    wl = make_workload(spec)
    d = to_device(wl)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    T, H, K = wl.T, spec.heads, spec.topk
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev)
    sel = args.select_in_indexer
    op = dsa.DSA_OP_INDEX_TOPK_ATTN_FUSED if sel else dsa.DSA_OP_INDEX_TOPK_ATTN
    ws = torch.zeros(dsa.dsa_workspace_size(op, d.seqs, K, H), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        dsa.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, out=out, lse=lse, ws=ws,
                                select_in_indexer=sel, kv_scale=d.kv_scale)

    if args.only:
        run_only(args, dsa, wl, d, dev, stream, flush, world, fused=step)
        return

    step()
    launches_per_step = dsa.dsa_launches_in_last_call()
    torch.cuda.synchronize()
    if dsa.dsa_check_error(ws) != dsa.DSA_OK:
        raise RuntimeError("device error flag set by the bench workload")

    graph = None
    run = step
    if not args.no_graph:
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        run = graph.replay

    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        times = time_device(run, args.steps, 0, stream, flush)
        barrier(world)
        torch.cuda.synchronize()
    ms_local = sum(times) / len(times)
    ms = reduce_max(ms_local, world)
    tokens_total = T * world
    value = tokens_total / (ms / 1e3)

    # ---- per-kernel device times inside the same call (events around every
    # launch; this pass serialises the kernels, so it is timed separately) ----
    kern = kernel_times(dsa, step, args.steps, stream, flush)

    # ---- per-stage device times (same kernels, same launch shapes) ----
    scores = torch.empty((T, (wl.max_ctx + 3) // 4 * 4), dtype=torch.float32, device=dev)
    ws_i = torch.zeros(dsa.dsa_workspace_size(dsa.DSA_OP_INDEX_SCORES, d.seqs, K, H), dtype=torch.uint8, device=dev)
    ws_t = torch.zeros(dsa.dsa_workspace_size(dsa.DSA_OP_TOPK, None, K, rows=T, ld=scores.shape[1]),
                       dtype=torch.uint8, device=dev)
    ws_a = torch.zeros(dsa.dsa_workspace_size(dsa.DSA_OP_SPARSE_MLA, d.seqs, K, H), dtype=torch.uint8, device=dev)
    row_len = torch.from_numpy((wl.token_pos() + 1).astype(np.int32)).to(dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    dsa.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores, ws=ws_i)
    dsa.dsa_topk(scores, row_len, K, idx=idx, ws=ws_t)
    reps = args.stage_reps
    t_idx = time_device(lambda: dsa.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores, ws=ws_i),
                        reps, 3, stream, flush)
    t_topk = time_device(lambda: dsa.dsa_topk(scores, row_len, K, idx=idx, ws=ws_t), reps, 3, stream, flush)
    t_attn = time_device(lambda: dsa.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, idx, wl.scale, out=out, lse=lse, ws=ws_a,
                                                        kv_scale=d.kv_scale),
                         reps, 3, stream, flush)
    n_keys = int((wl.token_pos() + 1).sum())
    n_sel = int(np.minimum(wl.token_pos() + 1, K).sum())
    idx_bytes = n_keys * index_row_bytes(spec)                   # index-cache bytes read
    attn_bytes = n_sel * (584 if spec.kv_fp8 else 1152)           # gathered latent rows (FP8: codes + 8 scale bytes)
    peak, peak_kind = hbm_peak()
    ms_idx = statistics.mean(t_idx)
    score_bytes = n_keys * 4 + T * K * 4                          # Top-K: score rows read, indices written
    roofs = {}
    for name, nbytes in (("index_scores", idx_bytes), ("topk_filter", score_bytes),
                         ("sparse_mla", attn_bytes)):
        if name in kern:
            roofs[name] = roofline_entry(name, kern, nbytes, peak, peak_kind, workload_config(spec, wl, world))
    dominant = max(roofs.values(), key=lambda r: r["launch_us"])

    # ---- end to end through the C ABI with host buffers ----
    pin = lambda x: x.pin_memory()  # noqa: E731
    h_qI, h_w, h_q = pin(wl.qI), pin(wl.w), pin(wl.q)
    h_meta = [pin(torch.from_numpy(a.astype(np.int32))) for a in (wl.q_seq_start, wl.ctx_len, wl.page_table)]
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    d_meta = [d.seqs.q_seq_start, d.seqs.ctx_len, d.seqs.page_table]

    side = torch.cuda.Stream(dev)
    q_ready = torch.cuda.Event()

    def e2e_step():
        # the indexer's inputs on the call's stream; the attention query on a
        # side stream (once the previous step's attention is done with it),
        # overlapping the indexer: the attention launch waits on q_ready
        cur = torch.cuda.current_stream(dev)
        d.qI.copy_(h_qI, non_blocking=True)
        d.w.copy_(h_w, non_blocking=True)
        for dm, hm in zip(d_meta, h_meta):
            dm.copy_(hm, non_blocking=True)
        side.wait_stream(cur)
        with torch.cuda.stream(side):
            d.q.copy_(h_q, non_blocking=True)
            q_ready.record(side)
        dsa.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, out=out, lse=lse, ws=ws,
                                q_ready=q_ready, select_in_indexer=sel, kv_scale=d.kv_scale)
        h_out.copy_(out, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)

    # The step as one CUDA graph, as a serving loop would replay it: every
    # replay still copies the inputs in from pinned host memory and the output
    # back.  Eager launches if the capture is refused.
    e2e_fn, e2e_mode, g_e2e = e2e_step, "eager", None
    if not args.no_graph:
        try:
            for _ in range(2):
                e2e_step()
            torch.cuda.synchronize()
            g_e2e = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_e2e):
                e2e_step()
            torch.cuda.synchronize()
            e2e_fn, e2e_mode = g_e2e.replay, "cuda graph replay"
        except RuntimeError as exc:
            g_e2e = None
            e2e_mode = f"eager (graph capture refused: {str(exc)[:80]})"
            torch.cuda.synchronize()
    e2e_times = time_device(e2e_fn, max(5, args.steps // 2), 2, stream, flush)
    del g_e2e
    e2e_ms = reduce_max(sum(e2e_times) / len(e2e_times), world)
    h2d = sum(x.numel() * x.element_size() for x in [h_qI, h_w, h_q, *h_meta])
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        spent, reps = 0.0, 0
        while spent < 10.0:                      # whole batches until ~10 s of host work
            dt, _ = cpu_baseline(wl, T)
            spent += dt
            reps += 1
        cpu = {"value": reps * T / spent, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"fp64 oracle, whole path for all {T} query tokens (ctx {int(wl.ctx_len[0])}), "
                         f"{reps} batch(es), {spent:.1f} s"}

    launch_mode = "cuda graph replay" if graph is not None else "eager"
    if graph is not None:
        del graph
    # every workload once more, untimed for the headline: each one's call time
    # and stage rooflines, recorded beside the headline number (1 GPU only)
    all_cfg = None
    if rank == 0 and world == 1 and not args.no_all_configs:
        all_cfg = all_configs_summary(args, dsa, dev, stream, flush)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "us_per_call": ms * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": {"mxfp8": "mxfp8", "fp8_e4m3": "fp8-e4m3", "bf16": "bf16"}[index_cache(spec)] + " index / "
                     + ("fp8-e4m3 latent, " if spec.kv_fp8 else "") + "bf16 attention / fp32 accum",
            "data": data_desc(spec),
            "config": workload_config(spec, wl, world),
            "launch": launch_mode,
            "stages_us": {"index_scores": ms_idx * 1e3, "topk": statistics.mean(t_topk) * 1e3,
                          "sparse_mla": statistics.mean(t_attn) * 1e3},
            "roofline": dominant,
            "kernel_rooflines": roofs,
            "kernels_us": {k: 1e3 * statistics.mean(v) for k, v in kern.items()},
            "e2e": {"value": tokens_total / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "launch": e2e_mode},
            "gpu_launches": launches_per_step * args.steps,
            "launches_per_step": launches_per_step,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        if all_cfg is not None:
            line["all_configs"] = all_cfg
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
