"""Zigzag context parallelism (sparse_indexed_attention_b200.cp) on CPU.

The plan is checked on its own (segment ownership, the gathered-pool page
table, balance of the causal work, order restore), then two gloo ranks run
one zigzag prefill end to end -- all-gather of the pools, each rank's
two-range batch, all-gather and reorder of the outputs -- with the fp64 oracle
standing in for the GPU call.  The per-token arithmetic is the oracle's in
both runs, so the parallel result must equal the one-rank oracle exactly."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_indexed_attention_b200.cp import PAGE, ZigzagPlan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("T,R", [(512, 2), (2048, 4), (4096, 8), (256, 1)])
def test_zigzag_plan(T, R):
    plan = ZigzagPlan.make(T, R)
    owned = np.concatenate([plan.local_positions(r) for r in range(R)])
    assert np.array_equal(np.sort(owned), np.arange(T))                  # every position exactly once
    # the gathered pool holds rank r's local rows at [2 seg r, 2 seg (r+1))
    gathered_pos = owned                                                  # row i of the gathered pool
    pt = plan.gathered_page_table()
    assert np.array_equal(np.sort(pt), np.arange(T // PAGE))              # a permutation of the pages
    for s in range(T):
        row = int(pt[s // PAGE]) * PAGE + s % PAGE
        assert gathered_pos[row] == s
    # causal work (sum of candidate counts) is the same on every rank
    work = [int((plan.local_positions(r) + 1).sum()) for r in range(R)]
    assert len(set(work)) == 1
    # rank batches: two ranges of one sequence, positions as owned
    for r in range(R):
        qs, cl, pt2 = plan.rank_batch(r)
        pos = np.concatenate([cl[b] - (qs[b + 1] - qs[b]) + np.arange(qs[b + 1] - qs[b]) for b in range(2)])
        assert np.array_equal(pos, plan.local_positions(r))
        assert np.array_equal(pt2[0], pt) and np.array_equal(pt2[1], pt)
    # restore inverts the local order
    g = torch.from_numpy(np.stack([plan.local_positions(r) for r in range(R)]))
    assert torch.equal(plan.restore(g), torch.arange(T))


def test_zigzag_plan_rejects_ragged_lengths():
    with pytest.raises(ValueError):
        ZigzagPlan.make(1000, 2)
    with pytest.raises(ValueError):
        ZigzagPlan.make(512, 0)


def _spec(kv_fp8=False, ki_mx=False):
    from dsa_workloads import CONFIGS
    return CONFIGS["long_prefill_32k"].scaled(name="cp_prefill_512", ctx=(512, 512), heads=16, topk=64,
                                              kv_fp8=kv_fp8, ki_mx=ki_mx)


def _kv_arg(kv, kv_scale):
    from dsa_workloads import bits16
    return bits16(kv) if kv_scale is None else (kv.numpy(), kv_scale.numpy())


def _oracle_attend(seqs, qI, w, kI, kI_scale, q, kv, K, scale, kv_scale=None):
    from dsa_workloads import bits16
    from oracle import dsa_oracle as O
    os_ = O.Seqs(seqs.ctx_len.numpy().astype(np.int64), seqs.q_seq_start.numpy().astype(np.int64),
                 seqs.page_table.numpy(), PAGE)
    _, _, out, lse = O.index_topk_attn(os_, bits16(qI), w.numpy(), kI.numpy(), kI_scale.numpy(), bits16(q),
                                       _kv_arg(kv, kv_scale), K, scale)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _shard(wl, plan, r):
    pos = plan.local_positions(r)
    rows = wl.page_table[0][pos // PAGE].astype(np.int64) * PAGE + pos % PAGE
    t = torch.from_numpy(pos)
    rw = torch.from_numpy(rows)
    kvs = None if wl.kv_scale is None else wl.kv_scale[rw]
    return wl.qI[t], wl.w[t], wl.q[t], wl.kI[rw], wl.kI_scale[rw], wl.kv[rw], kvs


def _rank_main(rank, world, port, q, kv_fp8, ki_mx):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from dsa_workloads import make_workload
    from sparse_indexed_attention_b200.cp import ZigzagPlan, cp_prefill
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = make_workload(_spec(kv_fp8, ki_mx))
        plan = ZigzagPlan.make(wl.T, world)
        qI, w, qq, kI, ks, kv, kvs = _shard(wl, plan, rank)
        out, lse = cp_prefill(plan, None, qI, w, qq, kI, ks, kv, wl.spec.topk, wl.scale, attend=_oracle_attend,
                              kv_scale_local=kvs)
        if rank == 0:
            q.put((out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("kv_fp8,ki_mx", [(False, False), (True, False), (False, True)],
                         ids=["bf16_latent", "fp8_latent", "mxfp8_index"])
def test_two_gloo_ranks_zigzag_prefill_equals_one_rank(kv_fp8, ki_mx):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q, kv_fp8, ki_mx)) for r in range(2)]
    for p in procs:
        p.start()
    got = None
    import queue as _queue
    import time
    deadline = time.time() + 600
    while got is None and time.time() < deadline:
        try:
            got = q.get(timeout=5)
        except _queue.Empty:
            if any(p.exitcode not in (None, 0) for p in procs):
                break
    for p in procs:
        p.join(timeout=120)
    assert got is not None, [p.exitcode for p in procs]
    out, lse = got
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    from dsa_workloads import bits16, make_workload
    from oracle import dsa_oracle as O
    wl = make_workload(_spec(kv_fp8, ki_mx))
    assert (wl.kI_scale.dim() == 2) == ki_mx      # MXFP8: E8M0 bytes [R, 4]
    seqs = O.Seqs(wl.ctx_len.astype(np.int64), wl.q_seq_start.astype(np.int64), wl.page_table, PAGE)
    _, _, ref_out, ref_lse = O.index_topk_attn(seqs, bits16(wl.qI), wl.w.numpy(), wl.kI.numpy(),
                                               wl.kI_scale.numpy(), bits16(wl.q), _kv_arg(wl.kv, wl.kv_scale),
                                               wl.spec.topk, wl.scale)
    assert np.array_equal(out, ref_out) and np.array_equal(lse, ref_lse)
