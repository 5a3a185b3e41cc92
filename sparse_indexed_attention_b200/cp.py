"""Zigzag context parallelism for one long prefill over R ranks ([P2] "Hybrid
Attention LLM Inference Acceleration...", section 6 "Optimization 3: Sequence
Parallelism and Load Balancing"; [P3] "Inference Acceleration for a New
Domestic LLM Architecture...", section 5 "Context Parallelism").

The T tokens of the sequence are cut into 2R segments of equal length; rank r
owns segments r and 2R-1-r.  A token's indexer and attention work grow with its
position, so pairing an early segment with a late one gives every rank the
same causal work.

Each rank holds the index keys (FP8 codes + scales, or bf16) and latent rows
(bf16, or FP8 codes + tile-scale bytes) of its own two segments, segment r
first.  One all-gather per pool (NCCL over NVLink, into each rank's own
memory) gives every rank the pools of the whole sequence laid out rank by
rank: rank q's rows sit at [2 seg q, 2 seg (q+1)).
Nothing is copied back into sequence order: a page table maps the sequence's
logical pages onto that layout (segments are whole pages).  Each rank then runs
the unchanged hot path (dsa_index_topk_attn) on its two segments as a batch
of two query ranges of the same sequence -- range i has context = the end of
its segment and q_len = seg, both rows of the batch's page table are the
sequence's -- and one more all-gather of the outputs restores the order.

Only the per-rank call runs kernels; this module plans, gathers and reorders.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

PAGE = 64


@dataclass(frozen=True)
class ZigzagPlan:
    T: int          # tokens of the sequence
    R: int          # ranks
    seg: int        # tokens per segment (a multiple of the page size)

    @staticmethod
    def make(T: int, R: int) -> "ZigzagPlan":
        if R < 1 or T < 1 or T % (2 * R * PAGE) != 0:
            raise ValueError(f"T={T} must be a positive multiple of 2 x ranks x {PAGE} (ranks={R})")
        return ZigzagPlan(T, R, T // (2 * R))

    def segments(self, r: int) -> tuple[int, int]:
        """The two segments rank r owns, in its local order."""
        return r, 2 * self.R - 1 - r

    def owner(self, s: int) -> tuple[int, int]:
        """(rank, first local row) of segment s."""
        if s < self.R:
            return s, 0
        return 2 * self.R - 1 - s, self.seg

    def local_positions(self, r: int) -> np.ndarray:
        """Sequence positions of rank r's local rows, in local order."""
        a, b = self.segments(r)
        return np.concatenate([np.arange(a * self.seg, (a + 1) * self.seg),
                               np.arange(b * self.seg, (b + 1) * self.seg)]).astype(np.int64)

    def gathered_page_table(self) -> np.ndarray:
        """int32 [T / 64]: logical page -> page of the rank-by-rank gathered pool."""
        pages = np.empty(self.T // PAGE, dtype=np.int32)
        for p in range(pages.shape[0]):
            s = p * PAGE // self.seg
            rank, off = self.owner(s)
            row = rank * 2 * self.seg + off + (p * PAGE - s * self.seg)
            pages[p] = row // PAGE
        return pages

    def rank_batch(self, r: int):
        """(q_seq_start [3], ctx_len [2], page_table [2, T/64]) of rank r's call."""
        a, b = self.segments(r)
        pt = self.gathered_page_table()
        return (np.array([0, self.seg, 2 * self.seg], dtype=np.int32),
                np.array([(a + 1) * self.seg, (b + 1) * self.seg], dtype=np.int32),
                np.stack([pt, pt]))

    def restore(self, gathered: torch.Tensor) -> torch.Tensor:
        """[R, 2 seg, ...] per-rank outputs (local order) -> [T, ...] in sequence order."""
        out = torch.empty((self.T, *gathered.shape[2:]), dtype=gathered.dtype, device=gathered.device)
        for s in range(2 * self.R):
            rank, off = self.owner(s)
            out[s * self.seg:(s + 1) * self.seg] = gathered[rank, off:off + self.seg]
        return out


def _all_gather(x: torch.Tensor, group) -> torch.Tensor:
    """[R, *x.shape] gathered from every rank of `group` (rank order)."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    out = torch.empty((R * x.shape[0], *x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, x.contiguous(), group=group)
    return out.view(R, *x.shape)


def _fused_call(seqs, qI, w, kI, kI_scale, q, kv, K: int, scale: float, kv_scale=None):
    import sparse_indexed_attention_b200 as dsa
    return dsa.dsa_index_topk_attn(seqs, qI, w, kI, kI_scale, q, kv, K, scale, kv_scale=kv_scale)


def cp_prefill(plan: ZigzagPlan, group, qI, w, q, kI_local, kI_scale_local, kv_local, K: int, scale: float,
               attend=None, gather_output: bool = True, kv_scale_local=None):
    """One zigzag-parallel prefill step on this rank.

    qI [2 seg, 64, 128], w [2 seg, 64], q [2 seg, H, 576]: this rank's query
    tokens in local order; kI_local [2 seg, 128] (+ kI_scale_local [2 seg],
    [2 seg, 4] for MXFP8, or None) and kv_local [2 seg, 576] (+ kv_scale_local
    [2 seg, 8] for the FP8 latent cache, or None): its rows of the pools, same
    order.  `attend(seqs, qI, w, kI, kI_scale, q, kv, K, scale[, kv_scale=])`
    -> (out, lse) runs the hot path (default: dsa_index_topk_attn; kv_scale is
    passed only for the FP8 latent cache).  Returns (out, lse) of the whole
    sequence in order when gather_output, else this rank's rows (local order).
    """
    import torch.distributed as dist
    r = dist.get_rank(group)
    if dist.get_world_size(group) != plan.R:
        raise ValueError("plan and process group disagree on the number of ranks")
    n = 2 * plan.seg
    for name, x in (("qI", qI), ("w", w), ("q", q), ("kI_local", kI_local), ("kv_local", kv_local)):
        if x.shape[0] != n:
            raise ValueError(f"{name}: {x.shape[0]} rows, expected 2 x segment = {n}")
    # whole-sequence pools, rank by rank, in this rank's own memory
    kI = _all_gather(kI_local, group).reshape(plan.R * n, *kI_local.shape[1:])
    kI_scale = None
    if kI_scale_local is not None:
        kI_scale = _all_gather(kI_scale_local, group).reshape(plan.R * n, *kI_scale_local.shape[1:])
    kv = _all_gather(kv_local, group).reshape(plan.R * n, *kv_local.shape[1:])
    kv_extra = {}
    if kv_scale_local is not None:
        kv_extra["kv_scale"] = _all_gather(kv_scale_local, group).reshape(plan.R * n, *kv_scale_local.shape[1:])
    qs, cl, pt = plan.rank_batch(r)
    from sparse_indexed_attention_b200 import Seqs
    seqs = Seqs.from_host(qs, cl, pt, plan.T // PAGE, device=q.device)
    out, lse = (attend or _fused_call)(seqs, qI, w, kI, kI_scale, q, kv, K, scale, **kv_extra)
    if not gather_output:
        return out, lse
    return plan.restore(_all_gather(out, group)), plan.restore(_all_gather(lse, group))
