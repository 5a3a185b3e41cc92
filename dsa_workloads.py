"""Seeded synthetic DSA workloads.

Only inputs are made here: batch geometry, shuffled page tables and the
tensors that the hot path reads.  Nothing in this module scores, selects or
attends; both the CUDA path and the fp64 oracle consume exactly these bytes.

Recipe (all draws from one ``torch.Generator`` seeded with ``Spec.seed``, in
the order written below):
  1. lengths: ctx_len ~ U[lo, hi] (integers, both ends included); prefill
     queries every position (q_len = ctx_len), decode queries the last position
     (q_len = 1), chunked prefill draws prefix ~ U and chunk ~ U, ctx = prefix +
     chunk, q_len = chunk;
  2. pages: each sequence needs ceil(ctx/64) pages; the physical page of every
     (sequence, logical page) is a seeded random permutation of the pool
     (pool = exactly the pages needed, or ``pool_tokens`` rows when given, the
     rest of the pool left zero); unused page-table entries are -1;
  3. per-token tensors: index query qI ~ N(0,1) as bf16 [T, 64, 128],
     head weights w ~ N(0,1)/8 fp32 [T, 64], attention query q ~ N(0,1) bf16
     [T, H, 576];
  4. pool rows, drawn in page-allocation order: index keys ~ N(0,1)
     [rows, 128] and latent KV ~ N(0,1) [rows, 576];
  5. planted keys (decode only): P positions per sequence drawn without
     replacement from 0..ctx-1.  Index key := 4*sqrt(128) * u/|u| with
     u = sum_h max(w[h], 0) qI[h] of the sequence's query; latent row :=
     3*sqrt(576) * g/|g| with g the mean over heads of the query q.  Their
     purpose is a known, clearly separated relevant set;
  6. storage: latent KV as bf16; index keys as bf16 (bf16 cache), as FP8 E4M3
     codes with one fp32 scale per row, scale = max|row| / 448 (1 for a zero
     row), codes = E4M3(row / scale) by torch's round-to-nearest cast, or as
     MXFP8: E4M3 codes with one E8M0 scale byte per 32 elements, scale
     2^(floor(log2 max|block|) - 8) (2^0 for a zero block), codes =
     E4M3(block / scale) clamped to +-448, by the same cast; latent KV as bf16
     or as the FP8 cache: per row, tiles of 128 values (the last of 64), each
     with scale 2^e, e the smallest integer with max|tile| <= 448 * 2^e (2^0
     for a zero tile), codes = E4M3(tile / 2^e), scale bytes e + 127 in [R, 8]
     (bytes 5..7 zero).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

_CHUNK = 1 << 24  # elements per random draw (bounds peak host memory)


@dataclass(frozen=True)
class Spec:
    name: str
    batch: int
    mode: str                       # "prefill" | "decode" | "chunked"
    ctx: tuple = (0, 0)             # prefill / decode context length range
    prefix: tuple = (0, 0)          # chunked: cached prefix length range
    chunk: tuple = (0, 0)           # chunked: new chunk length range
    ki_fp8: bool = True             # FP8 E4M3 index cache with per-row scale
    ki_mx: bool = False             # MXFP8 index cache (E4M3 + E8M0 per 32 elements); overrides ki_fp8
    kv_fp8: bool = False            # FP8 latent KV cache (E4M3, power-of-two scale per 128-element tile)
    heads: int = 128                # attention query heads
    topk: int = 2048
    planted: int = 0
    pool_tokens: int = 0
    seed: int = 0
    index_heads: int = 64
    index_dim: int = 128
    page_size: int = 64
    d_qk: int = 576
    d_v: int = 512

    def scaled(self, **kw) -> "Spec":
        return replace(self, **kw)


# The five workloads the library is measured on.
CONFIGS = {
    "tiny_prefill_1k": Spec("tiny_prefill_1k", 1, "prefill", ctx=(1024, 1024), ki_fp8=False,
                            heads=16, topk=256, seed=0),
    "decode_b64_8k_32k": Spec("decode_b64_8k_32k", 64, "decode", ctx=(8192, 32768), planted=32, seed=2),
    "long_prefill_32k": Spec("long_prefill_32k", 1, "prefill", ctx=(32768, 32768), seed=3),
    "decode_b8_128k": Spec("decode_b8_128k", 8, "decode", ctx=(131072, 131072), planted=64,
                           pool_tokens=2 * 1024 * 1024, seed=4),
    "chunked_prefill_16": Spec("chunked_prefill_16", 16, "chunked", prefix=(0, 65536),
                               chunk=(512, 4096), seed=5),
}
CONFIG_ORDER = list(CONFIGS)


@dataclass
class Workload:
    spec: Spec
    ctx_len: np.ndarray            # int32 [B]
    q_len: np.ndarray              # int32 [B]
    q_seq_start: np.ndarray        # int32 [B+1]
    page_table: np.ndarray         # int32 [B, max_pages]
    num_phys_pages: int
    qI: torch.Tensor               # bf16 [T, H_I, d_I]
    w: torch.Tensor                # fp32 [T, H_I]
    kI: torch.Tensor               # uint8 FP8 codes or bf16 [R, d_I]
    kI_scale: torch.Tensor | None  # fp32 [R] (FP8 cache), uint8 E8M0 [R, 4] (MXFP8) or None
    q: torch.Tensor                # bf16 [T, H, d_qk]
    kv: torch.Tensor               # bf16 [R, d_qk], or uint8 E4M3 codes [R, d_qk] (FP8 cache)
    planted: list                  # per sequence: np.ndarray of planted positions
    kv_scale: torch.Tensor | None = None  # FP8 latent cache: uint8 [R, 8] tile-scale bytes

    @property
    def T(self) -> int:
        return int(self.q_seq_start[-1])

    @property
    def max_ctx(self) -> int:
        return int(self.ctx_len.max()) if len(self.ctx_len) else 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.spec.d_qk)

    def token_pos(self) -> np.ndarray:
        """Absolute position of every query token (int64 [T])."""
        out = np.empty(self.T, dtype=np.int64)
        for b in range(len(self.ctx_len)):
            a, e = int(self.q_seq_start[b]), int(self.q_seq_start[b + 1])
            out[a:e] = int(self.ctx_len[b]) - (e - a) + np.arange(e - a)
        return out


def _randn(g: torch.Generator, shape, scale: float = 1.0) -> torch.Tensor:
    """N(0,1)*scale fp32 of the given shape, drawn in fixed-size pieces."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.float32)
    for a in range(0, n, _CHUNK):
        e = min(n, a + _CHUNK)
        out[a:e] = torch.randn(e - a, generator=g)
    if scale != 1.0:
        out.mul_(scale)
    return out.view(*shape)


def _randn_bf16(g: torch.Generator, shape) -> torch.Tensor:
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16)
    for a in range(0, n, _CHUNK):
        e = min(n, a + _CHUNK)
        out[a:e] = torch.randn(e - a, generator=g).to(torch.bfloat16)
    return out.view(*shape)


def fp8_rows(x: torch.Tensor):
    """Store fp32 rows as FP8 E4M3 codes + one fp32 scale per row (cache format)."""
    amax = x.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (x / scale[:, None]).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


def kv8_rows(x: torch.Tensor):
    """Store fp32 latent rows as the FP8 cache: E4M3 codes [R, d] and the tiles'
    scale bytes [R, 8] (tile j = elements 128j .. 128j+127)."""
    R, d = x.shape
    codes = torch.zeros((R, d), dtype=torch.uint8)
    scales = torch.zeros((R, 8), dtype=torch.uint8)
    for j in range((d + 127) // 128):
        lo, hi = 128 * j, min(d, 128 * (j + 1))
        a = x[:, lo:hi].abs().amax(dim=1).double()
        e = torch.where(a > 0, torch.ceil(torch.log2(a / 448.0)), torch.zeros_like(a))
        for _ in range(2):  # the estimate, made exact by comparisons (448 * 2^e is exact in fp64)
            e = torch.where(a > 448.0 * torch.exp2(e), e + 1, e)
            e = torch.where((a > 0) & (a <= 448.0 * torch.exp2(e - 1)), e - 1, e)
        t = (x[:, lo:hi].double() * torch.exp2(-e)[:, None]).clamp_(-448.0, 448.0).float()
        codes[:, lo:hi] = t.to(torch.float8_e4m3fn).view(torch.uint8)
        scales[:, j] = (e + 127).to(torch.uint8)
    return codes, scales


def mx_rows(x: torch.Tensor):
    """Store fp32 rows as MXFP8 (cache format): E4M3 codes [R, d] and one E8M0
    scale byte per 32 elements [R, d/32]."""
    R, d = x.shape
    blocks = x.reshape(R, d // 32, 32)
    amax = blocks.abs().amax(dim=2)
    _, ex = torch.frexp(amax)                      # amax = m * 2^ex, 0.5 <= m < 1
    e = torch.where(amax > 0, (ex - 9).clamp(-127, 127), torch.zeros_like(ex))
    codes = (blocks * torch.exp2(-e.to(torch.float32))[..., None]).clamp_(-448.0, 448.0)
    codes = codes.to(torch.float8_e4m3fn).view(torch.uint8).reshape(R, d)
    return codes, (e + 127).to(torch.uint8)


def make_workload(spec: Spec) -> Workload:
    g = torch.Generator().manual_seed(spec.seed)
    B, ps = spec.batch, spec.page_size

    def draw(rng):
        lo, hi = rng
        return torch.randint(lo, hi + 1, (B,), generator=g).numpy().astype(np.int64)

    if spec.mode == "prefill":
        ctx = draw(spec.ctx)
        q_len = ctx.copy()
    elif spec.mode == "decode":
        ctx = draw(spec.ctx)
        q_len = np.ones(B, dtype=np.int64)
    elif spec.mode == "chunked":
        prefix = draw(spec.prefix)
        chunk = draw(spec.chunk)
        ctx = prefix + chunk
        q_len = chunk
    else:
        raise ValueError(spec.mode)
    if np.any(ctx < 1) or np.any(q_len < 1) or np.any(q_len > ctx):
        raise ValueError("bad lengths")

    pages_per_seq = (ctx + ps - 1) // ps
    needed = int(pages_per_seq.sum())
    max_pages = int(pages_per_seq.max())
    num_phys = max(needed, spec.pool_tokens // ps)
    perm = torch.randperm(num_phys, generator=g)[:needed].numpy().astype(np.int64)
    page_table = np.full((B, max_pages), -1, dtype=np.int32)
    alloc_base = np.zeros(B, dtype=np.int64)   # first allocation slot of each sequence
    k = 0
    for b in range(B):
        alloc_base[b] = k
        page_table[b, : pages_per_seq[b]] = perm[k: k + pages_per_seq[b]]
        k += int(pages_per_seq[b])

    q_seq_start = np.zeros(B + 1, dtype=np.int64)
    q_seq_start[1:] = np.cumsum(q_len)
    T = int(q_seq_start[-1])
    H_I, d_I, H = spec.index_heads, spec.index_dim, spec.heads

    qI = _randn_bf16(g, (T, H_I, d_I))
    w = _randn(g, (T, H_I), 1.0 / 8.0)
    q = _randn_bf16(g, (T, H, spec.d_qk))

    n_alloc_rows = needed * ps
    ki_vals = _randn(g, (n_alloc_rows, d_I))
    kv_vals = _randn(g, (n_alloc_rows, spec.d_qk))

    planted = []
    for b in range(B):
        if spec.planted <= 0:
            planted.append(np.zeros(0, dtype=np.int64))
            continue
        P = min(spec.planted, int(ctx[b]))
        pos = torch.randperm(int(ctx[b]), generator=g)[:P].numpy().astype(np.int64)
        planted.append(np.sort(pos))
        t = int(q_seq_start[b + 1]) - 1           # the sequence's last query token
        u = (w[t].clamp(min=0)[:, None] * qI[t].float()).sum(0)
        ki_row = 4.0 * math.sqrt(d_I) * u / u.norm().clamp(min=1e-30)
        gq = q[t].float().mean(0)
        kv_row = 3.0 * math.sqrt(spec.d_qk) * gq / gq.norm().clamp(min=1e-30)
        slots = alloc_base[b] * ps + pos          # rows in allocation order
        ki_vals[torch.from_numpy(slots)] = ki_row
        kv_vals[torch.from_numpy(slots)] = kv_row

    # allocation slot -> physical row
    slot_page = np.empty(needed, dtype=np.int64)
    for b in range(B):
        slot_page[alloc_base[b]: alloc_base[b] + pages_per_seq[b]] = page_table[b, : pages_per_seq[b]]
    phys_rows = torch.from_numpy((slot_page[:, None] * ps + np.arange(ps)[None, :]).reshape(-1))

    R = num_phys * ps
    kv_scale = None
    if spec.kv_fp8:
        codes, sc = kv8_rows(kv_vals)
        kv = torch.zeros((R, spec.d_qk), dtype=torch.uint8)
        kv[phys_rows] = codes
        kv_scale = torch.zeros((R, 8), dtype=torch.uint8)
        kv_scale[:, :5] = 127
        kv_scale[phys_rows] = sc
    else:
        kv = torch.zeros((R, spec.d_qk), dtype=torch.bfloat16)
        kv[phys_rows] = kv_vals.to(torch.bfloat16)
    del kv_vals
    if spec.ki_mx:
        codes, sc = mx_rows(ki_vals)
        kI = torch.zeros((R, d_I), dtype=torch.uint8)
        kI[phys_rows] = codes
        kI_scale = torch.full((R, d_I // 32), 127, dtype=torch.uint8)
        kI_scale[phys_rows] = sc
    elif spec.ki_fp8:
        codes, sc = fp8_rows(ki_vals)
        kI = torch.zeros((R, d_I), dtype=torch.uint8)
        kI[phys_rows] = codes
        kI_scale = torch.ones(R, dtype=torch.float32)
        kI_scale[phys_rows] = sc
    else:
        kI = torch.zeros((R, d_I), dtype=torch.bfloat16)
        kI[phys_rows] = ki_vals.to(torch.bfloat16)
        kI_scale = None

    return Workload(spec=spec, ctx_len=ctx.astype(np.int32), q_len=q_len.astype(np.int32),
                    q_seq_start=q_seq_start.astype(np.int32), page_table=page_table,
                    num_phys_pages=num_phys, qI=qI, w=w, kI=kI, kI_scale=kI_scale, q=q, kv=kv,
                    planted=planted, kv_scale=kv_scale)


def bits16(x: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 CPU tensor (for the fp64 oracle)."""
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass
class DeviceWorkload:
    """A workload's tensors resident on one GPU, ready for the binding."""
    wl: Workload
    seqs: object                 # sparse_indexed_attention_b200.Seqs
    qI: torch.Tensor
    w: torch.Tensor
    kI: torch.Tensor
    kI_scale: torch.Tensor | None
    q: torch.Tensor
    kv: torch.Tensor
    kv_scale: torch.Tensor | None = None

    @property
    def K(self) -> int:
        return self.wl.spec.topk

    @property
    def scale(self) -> float:
        return self.wl.scale

    def h2d_bytes(self) -> int:
        """Bytes of the per-step inputs (queries and batch metadata)."""
        t = [self.qI, self.w, self.q, self.seqs.q_seq_start, self.seqs.ctx_len, self.seqs.page_table]
        return sum(x.numel() * x.element_size() for x in t)


def to_device(wl: Workload, device="cuda") -> DeviceWorkload:
    from sparse_indexed_attention_b200 import Seqs
    seqs = Seqs.from_host(wl.q_seq_start, wl.ctx_len, wl.page_table, wl.num_phys_pages, device=device)
    dev = lambda x: None if x is None else x.contiguous().to(device)  # noqa: E731
    return DeviceWorkload(wl, seqs, dev(wl.qI), dev(wl.w), dev(wl.kI), dev(wl.kI_scale), dev(wl.q), dev(wl.kv),
                          dev(wl.kv_scale))
