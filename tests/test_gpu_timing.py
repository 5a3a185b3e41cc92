"""dsa_launch_timing / dsa_last_launch_times: one named, positive device time
per kernel of a fused call while enabled, and a call with identical results.
With the selection inside the indexer, the decode call is at most four
launches: prep, the indexer, attention and (when the index lists are split)
the merge."""
import pytest
import torch

from dsa_workloads import to_device
from tests.specs import SMALL, workload as make_workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("select_in_indexer", [False, True])
def test_launch_times_of_fused_decode(lib, select_in_indexer):
    wl = make_workload(SMALL["pool_b2_128k"])
    d = to_device(wl)
    K = wl.spec.topk

    def call():
        return lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale,
                                       select_in_indexer=select_in_indexer)

    out0, lse0 = call()
    out0, lse0 = out0.clone(), lse0.clone()
    assert lib.dsa_last_launch_times() == []            # timing off: nothing recorded
    lib.dsa_launch_timing(True)
    try:
        out1, lse1 = call()
        times = lib.dsa_last_launch_times()
        n = lib.dsa_launches_in_last_call()
    finally:
        lib.dsa_launch_timing(False)
    assert len(times) == n >= 3
    names = [nm for nm, _ in times]
    assert all(ms > 0 for _, ms in times)
    if select_in_indexer:  # the indexer selects the Top-K itself
        assert names[:3] == ["prep", "index_scores", "sparse_mla"] and n <= 4, names
        assert not any(nm.startswith("topk") for nm in names)
    else:
        assert "index_scores" in names and "sparse_mla" in names and any(nm.startswith("topk") for nm in names)
    torch.cuda.synchronize()
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)  # events change timing, not results
    call()
    assert lib.dsa_last_launch_times() == []
