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
