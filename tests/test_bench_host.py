"""bench.py's host-side bookkeeping on CPU: the config object both arms print,
the index-cache byte count behind the roofline, and which captured ncu
traffic figure (if any) a line may carry.  No GPU and no library call."""
import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dsa_workloads import CONFIGS  # noqa: E402


def _config(spec, ctx=131072):
    wl = SimpleNamespace(T=spec.batch, ctx_len=np.array([ctx] * spec.batch), num_phys_pages=32768)
    return bench.workload_config(spec, wl, 1)


def test_index_cache_format_and_bytes():
    dec = CONFIGS["decode_b8_128k"]
    tiny = CONFIGS["tiny_prefill_1k"]                       # bf16 index cache
    assert (bench.index_cache(dec), bench.index_row_bytes(dec)) == ("fp8_e4m3", 132)
    assert (bench.index_cache(tiny), bench.index_row_bytes(tiny)) == ("bf16", 256)
    # MXFP8 overrides the per-row flag, also on a workload whose default cache is bf16
    for s in (dec.scaled(ki_mx=True), tiny.scaled(ki_mx=True)):
        assert (bench.index_cache(s), bench.index_row_bytes(s)) == ("mxfp8", 132)
    assert _config(tiny.scaled(ki_mx=True))["index_cache"] == "mxfp8"
    assert _config(dec.scaled(kv_fp8=True))["latent_cache"] == "fp8_e4m3_tile128"


def test_data_description_follows_the_workload():
    assert bench.data_desc(CONFIGS["decode_b8_128k"]) == "synthetic (seeded, 64 planted keys per sequence)"
    assert bench.data_desc(CONFIGS["tiny_prefill_1k"]) == "synthetic (seeded)"


@pytest.fixture
def fresh_sources(monkeypatch):
    """Pretend every kernel source still hashes to what was captured."""
    digests = {files: d for _, _, _, files, d in bench.NCU_CAPTURES}
    monkeypatch.setattr(bench, "source_digest", lambda files: digests[files])


def test_captured_traffic_only_for_the_captured_formats(fresh_sources):
    dec = CONFIGS["decode_b8_128k"]
    fp8, mx, kv8 = _config(dec), _config(dec.scaled(ki_mx=True)), _config(dec.scaled(kv_fp8=True))
    assert bench.ncu_traffic("index_scores", fp8) == 145.60e6
    assert bench.ncu_traffic("index_scores", mx) == 144.81e6
    assert bench.ncu_traffic("index_scores", kv8) == 145.60e6          # the indexer does not read the latent cache
    assert bench.ncu_traffic("sparse_mla", fp8) == 20.25e6
    assert bench.ncu_traffic("sparse_mla", kv8) is None                 # FP8 attention was not captured
    assert bench.ncu_traffic("topk_filter", mx) == 4.35e6               # reads fp32 scores in every format
    assert bench.ncu_traffic("index_scores", _config(dec, ctx=65536)) is None        # another context length
    assert bench.ncu_traffic("index_scores", _config(CONFIGS["decode_b64_8k_32k"])) is None
    assert bench.ncu_traffic("topk_emit", fp8) is None                  # never captured


def test_captured_traffic_goes_stale_with_the_source(monkeypatch):
    monkeypatch.setattr(bench, "source_digest", lambda files: "0" * 16)
    assert bench.ncu_traffic("index_scores", _config(CONFIGS["decode_b8_128k"])) is None


def test_roofline_entry(fresh_sources):
    cfg = _config(CONFIGS["decode_b8_128k"])
    r = bench.roofline_entry("index_scores", {"index_scores": [0.040, 0.044]}, 138_412_032, 6552.3, "measured", cfg)
    assert r["launch_us"] == pytest.approx(42.0)
    assert r["achieved"] == pytest.approx(138_412_032 / 42.0e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6552.3)
    assert (r["bound"], r["unit"], r["traffic"]) == ("hbm", "GB/s", 145.60e6)


class _FakeGraph:
    def replay(self):
        pass


class _FakeCapture:
    def __init__(self, graph):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def _fake_library(calls, launches):
    from types import SimpleNamespace as NS
    return NS(DSA_OK=0, DSA_OP_INDEX_TOPK_ATTN=4, DSA_OP_INDEX_TOPK_ATTN_FUSED=5,
              dsa_workspace_size=lambda op, seqs, K, H: 256,
              dsa_index_topk_attn=lambda *a, **k: calls.append(k),
              dsa_check_error=lambda ws: 0,
              dsa_launches_in_last_call=lambda: len(launches),
              dsa_launch_timing=lambda on: None,
              dsa_last_launch_times=lambda: list(launches))


@pytest.fixture
def host_only_bench(monkeypatch):
    """all_config_lines on CPU: small workloads, a fake library and fake CUDA
    timing, so only the bench's own bookkeeping runs."""
    import torch
    import dsa_workloads
    from types import SimpleNamespace as NS
    small = {
        "tiny_prefill_1k": CONFIGS["tiny_prefill_1k"].scaled(ctx=(256, 256)),
        "decode_b64_8k_32k": CONFIGS["decode_b64_8k_32k"].scaled(batch=3, ctx=(300, 900)),
    }
    monkeypatch.setattr(bench, "CONFIGS", small)
    monkeypatch.setattr(dsa_workloads, "to_device", lambda wl: NS(seqs=None, qI=wl.qI, w=wl.w, kI=wl.kI,
                                                                  kI_scale=wl.kI_scale, q=wl.q, kv=wl.kv,
                                                                  kv_scale=wl.kv_scale))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "CUDAGraph", _FakeGraph)
    monkeypatch.setattr(torch.cuda, "graph", _FakeCapture)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    monkeypatch.setattr(bench, "time_device", lambda fn, steps, warmup, stream, flush: (fn(), [0.25, 0.25])[1])
    monkeypatch.setattr(bench, "hbm_peak", lambda: (6552.3, "measured"))
    monkeypatch.setattr(bench, "tensor_peak", lambda kind: (1640.5 * (2 if kind == "fp8" else 1), "measured"))
    args = NS(ki="workload", kv="bf16", select_in_indexer=False)
    return args, small


def test_all_config_lines_bookkeeping(host_only_bench):
    import torch
    args, small = host_only_bench
    calls = []
    launches = [("prep", 0.01), ("index_scores", 0.04), ("topk_row", 0.02), ("sparse_mla", 0.1)]
    lines = list(bench.all_config_lines(args, _fake_library(calls, launches), torch.device("cpu"), None,
                                        torch.empty(64, dtype=torch.uint8)))
    assert [ln["config"] for ln in lines] == list(small)
    tiny, dec = lines
    assert tiny["us_per_call"] == pytest.approx(250.0) and dec["launches"] == 4
    assert tiny["kernels_us"]["index_scores"] == pytest.approx(40.0)
    # bf16 prefill indexer: tensor bound against the bf16 peak, 16,384 flop per causal pair
    pairs = 256 * 257 // 2
    s = tiny["stages"]["index_scores"]
    assert (s["bound"], s["dtype"]) == ("tensor", "bf16")
    assert s["frac"] == pytest.approx(pairs * 16384 / 40e-6 / 1e12 / 1640.5)
    # decode indexer: HBM bound, 132 B per key of the FP8 cache
    wl = bench.make_workload(small["decode_b64_8k_32k"])
    keys = int((wl.token_pos() + 1).sum())
    s = dec["stages"]["index_scores"]
    assert s["bound"] == "hbm" and s["frac"] == pytest.approx(keys * 132 / 40e-6 / 1e9 / 6552.3)
    assert dec["stages"]["sparse_mla"]["bound"] == "hbm"
    assert all(not k.get("select_in_indexer") for k in calls)


def test_all_configs_summary_condenses_and_survives_failures(host_only_bench, monkeypatch):
    import torch
    args, small = host_only_bench
    launches = [("prep", 0.01), ("index_scores", 0.04), ("topk_row", 0.02), ("sparse_mla", 0.1)]
    flush = torch.empty(64, dtype=torch.uint8)
    summ = bench.all_configs_summary(args, _fake_library([], launches), torch.device("cpu"), None, flush)
    assert set(summ) == set(small)
    assert set(summ["tiny_prefill_1k"]) == {"us_per_call", "tokens_per_s", "launches", "stages"}
    assert summ["tiny_prefill_1k"]["stages"]["index_scores"]["bound"] == "tensor"

    def broken(*a):
        yield {"config": "first", "us_per_call": 1.0, "tokens_per_s": 1.0, "launches": 1, "stages": {}}
        raise RuntimeError("device error flag set on second")
    monkeypatch.setattr(bench, "all_config_lines", broken)
    summ = bench.all_configs_summary(args, None, None, None, None)
    assert "first" in summ and summ["error"].startswith("RuntimeError: device error flag")
