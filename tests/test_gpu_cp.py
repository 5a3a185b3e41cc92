"""Zigzag context parallelism on one GPU: the two ranks of a 2-way split run
one after the other in this process (no collectives -- the pools are
concatenated rank by rank exactly as the all-gather lays them out), and the
reordered result must equal the single call on the whole sequence bit for
bit: every token's scores, selection and attention are computed by the same
kernels on the same values, only the batch around them differs."""
import numpy as np
import pytest
import torch

from dsa_workloads import CONFIGS, make_workload, to_device
from sparse_indexed_attention_b200.cp import PAGE, ZigzagPlan

pytestmark = pytest.mark.gpu


def _shard(wl, plan, r, dev="cuda"):
    pos = plan.local_positions(r)
    rows = wl.page_table[0][pos // PAGE].astype(np.int64) * PAGE + pos % PAGE
    t, rw = torch.from_numpy(pos), torch.from_numpy(rows)
    return [x.contiguous().to(dev) for x in (wl.qI[t], wl.w[t], wl.q[t], wl.kI[rw], wl.kI_scale[rw], wl.kv[rw])]


@pytest.mark.parametrize("ranks", [2, 4])
def test_zigzag_prefill_ranks_equal_one_call(lib, ranks):
    spec = CONFIGS["long_prefill_32k"].scaled(name="cp_prefill_4k", ctx=(4096, 4096))
    wl = make_workload(spec)
    d = to_device(wl)
    K = spec.topk
    full_out, full_lse = lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale,
                                                 out_dtype=torch.float32)
    plan = ZigzagPlan.make(wl.T, ranks)
    shards = [_shard(wl, plan, r) for r in range(ranks)]
    kI = torch.cat([s[3] for s in shards])           # what every rank's all-gather holds
    kI_scale = torch.cat([s[4] for s in shards])
    kv = torch.cat([s[5] for s in shards])
    outs, lses = [], []
    for r in range(ranks):
        qs, cl, pt = plan.rank_batch(r)
        seqs = lib.Seqs.from_host(qs, cl, pt, wl.T // PAGE, device="cuda")
        qI, w, q = shards[r][:3]
        o, l = lib.dsa_index_topk_attn(seqs, qI, w, kI, kI_scale, q, kv, K, wl.scale, out_dtype=torch.float32)
        outs.append(o)
        lses.append(l)
    assert lib.dsa_check_error(lib.workspace(0, "cuda", "index_topk_attn")) == lib.DSA_OK
    out = plan.restore(torch.stack(outs))
    lse = plan.restore(torch.stack(lses))
    assert torch.equal(out, full_out) and torch.equal(lse, full_lse)
