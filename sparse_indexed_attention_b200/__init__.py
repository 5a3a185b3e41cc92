"""Python binding of libdsa (include/dsa.h): index-selected sparse attention on B200.

Argument marshalling only.  Every step of the path runs in libdsa's CUDA
kernels; torch provides device memory and the current stream.  There is no
fallback: if libdsa.so is missing and cannot be built, importing this package
raises.

Functions carry the C names (``dsa_index_scores`` ...).  Outputs not passed in
are allocated with torch on the inputs' device; workspaces are allocated
zeroed and cached per (device, op), unless one is passed in (concurrent
calls on different streams pass their own).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from . import build as _build

# ---------------------------------------------------------------------------
# Library loading
# ---------------------------------------------------------------------------

if _build.is_stale():
    _build.build_library()
_lib = ctypes.CDLL(_build.LIB)
LIB_PATH = _build.LIB

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_BAD_INDEX, \
    DSA_ERR_TIMEOUT = range(7)
DSA_KI_BF16, DSA_KI_FP8_E4M3, DSA_KI_MXFP8 = 0, 1, 2
DSA_KV_BF16, DSA_KV_FP8_E4M3 = 0, 1
DSA_OUT_BF16, DSA_OUT_F32 = 0, 1
DSA_NOALLOC_SCRATCH_BYTES = 32 << 20
DSA_OP_QUANTIZE_INDEX_QUERY, DSA_OP_INDEX_SCORES, DSA_OP_TOPK, DSA_OP_SPARSE_MLA, DSA_OP_INDEX_TOPK_ATTN, \
    DSA_OP_INDEX_TOPK_ATTN_FUSED = range(6)
DSA_SELECT_IN_INDEXER = 1

# Names the C header declares (checked against include/dsa.h by the tests).
EXPORTS = ("dsa_workspace_size",
           "dsa_quantize_index_query", "dsa_quantize_index_query_mx",
           "dsa_index_scores", "dsa_topk",
           "dsa_sparse_mla_fwd", "dsa_sparse_mla_fwd_ex", "dsa_sparse_mla_fwd_noalloc",
           "dsa_index_topk_attn", "dsa_index_topk_attn_ex",
           "dsa_check_error", "dsa_check_error_noalloc", "dsa_set_wait_limit_ns",
           "dsa_launches_in_last_call", "dsa_launch_timing", "dsa_last_launch_times", "dsa_status_string")


class DsaSeqsC(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_tokens", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("num_phys_pages", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("q_seq_start", ctypes.c_void_p), ("ctx_len", ctypes.c_void_p), ("page_table", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I32, _I64, _SZ, _F = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_SEQ = ctypes.POINTER(DsaSeqsC)
_sig = {
    "dsa_workspace_size": (_SZ, [ctypes.c_int, _SEQ, ctypes.c_int, ctypes.c_int]),
    "dsa_quantize_index_query": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, _P]),
    "dsa_quantize_index_query_mx": (ctypes.c_int, [_P, ctypes.c_int, _P, _P, _P]),
    "dsa_index_scores": (ctypes.c_int, [_SEQ, _P, _P, _P, _P, ctypes.c_int, _P, _I64, _P, _SZ, _P]),
    "dsa_topk": (ctypes.c_int, [_P, _I64, ctypes.c_int, _P, ctypes.c_int, _P, _P, _SZ, _P]),
    "dsa_sparse_mla_fwd": (ctypes.c_int, [_SEQ, _P, _P, _P, ctypes.c_int, ctypes.c_int, _F, _P, ctypes.c_int, _P, _P,
                                          _SZ, _P]),
    "dsa_sparse_mla_fwd_ex": (ctypes.c_int, [_SEQ, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, ctypes.c_int, _F, _P,
                                             ctypes.c_int, _P, _P, _SZ, _P]),
    "dsa_sparse_mla_fwd_noalloc": (ctypes.c_int, [_SEQ, _P, _P, _P, ctypes.c_int, ctypes.c_int, _F, _P, ctypes.c_int,
                                                  _P, _P]),
    "dsa_index_topk_attn": (ctypes.c_int, [_SEQ, _P, _P, _P, _P, ctypes.c_int, _P, _P, ctypes.c_int, ctypes.c_int,
                                           _F, _P, ctypes.c_int, _P, _P, _P, _SZ, _P]),
    "dsa_index_topk_attn_ex": (ctypes.c_int, [_SEQ, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, _F, _P, ctypes.c_int, _P, _P, _P, _SZ,
                                              ctypes.c_uint, _P, _P]),
    "dsa_check_error": (ctypes.c_int, [_P, _P]),
    "dsa_check_error_noalloc": (ctypes.c_int, [_P]),
    "dsa_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "dsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dsa_launches_in_last_call": (ctypes.c_int, []),
    "dsa_launch_timing": (ctypes.c_int, [ctypes.c_int]),
    "dsa_last_launch_times": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_char_p),
                                             ctypes.c_int]),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype, _fn.argtypes = _res, _args


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.dsa_status_string(status).decode()}")


def _check(status: int, where: str):
    if status != DSA_OK:
        raise DsaError(status, where)


def status_string(status: int) -> str:
    return _lib.dsa_status_string(status).decode()


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name: str, dtypes, shape, device: torch.device, min_rows: int = 0):
    """Refuse, before any C call, a tensor the kernels would misread: each must
    be a contiguous tensor on `device` with one of `dtypes`, a shape matching
    `shape` (None matches any size) and at least `min_rows` rows.  The kernels
    take bare pointers, so a wrong dtype, a strided view or a short pool would
    otherwise be read out of bounds."""
    try:  # fast path: one pass over the metadata, no message building
        sz = t.shape
        ok = t.device == device and t.dtype in dtypes and len(sz) == len(shape) and sz[0] >= min_rows \
            and t.is_contiguous()
        if ok:
            for g, w in zip(sz, shape):
                if w is not None and g != w:
                    ok = False
                    break
    except (AttributeError, IndexError):
        ok = False
    if not ok:
        _refuse(t, name, dtypes, shape, device, min_rows)


def _refuse(t, name, dtypes, shape, device, min_rows):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {[str(d) for d in dtypes]}")
    if t.dim() != len(shape) or any(w is not None and w != g for g, w in zip(t.shape, shape)):
        want = "[" + ", ".join("*" if w is None else str(w) for w in shape) + "]"
        raise ValueError(f"{name}: shape {list(t.shape)}, expected {want}")
    if t.shape[0] < min_rows:
        raise ValueError(f"{name}: {t.shape[0]} rows, the page pool needs at least {min_rows}")
    raise ValueError(f"{name}: must be contiguous")


def _cuda_device(t, name: str) -> torch.device:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name}: expected a CUDA tensor")
    return t.device


_I32T, _F32T, _BF16T = (torch.int32,), (torch.float32,), (torch.bfloat16,)
_FP8T = (torch.uint8, torch.float8_e4m3fn)


def _need_seqs(seqs: "Seqs", dev: torch.device):
    _need(seqs.q_seq_start, "seqs.q_seq_start", _I32T, (seqs.batch + 1,), dev)
    _need(seqs.ctx_len, "seqs.ctx_len", _I32T, (None,), dev)
    _need(seqs.page_table, "seqs.page_table", _I32T, (seqs.batch, None), dev)


def _need_ws(ws, dev: torch.device):
    _need(ws, "ws", (torch.uint8,), (None,), dev)


def _need_index_inputs(seqs: "Seqs", qI, w, kI, kI_scale, check_seqs: bool = True) -> torch.device:
    dev = _cuda_device(qI, "qI")
    T, rows = seqs.num_q_tokens, seqs.num_phys_pages * 64
    if check_seqs:
        _need_seqs(seqs, dev)
    _need(qI, "qI", _BF16T, (T, 64, 128), dev)
    _need(w, "w", _F32T, (T, 64), dev)
    _need(kI, "kI", _FP8T if kI_scale is not None else _BF16T, (None, 128), dev, rows)
    if _is_mx(kI_scale):
        _need(kI_scale, "kI_scale", (torch.uint8,), (None, 4), dev, rows)
    elif kI_scale is not None:
        _need(kI_scale, "kI_scale", _F32T, (None,), dev, rows)
    return dev


def _is_mx(kI_scale) -> bool:
    """An MXFP8 index cache carries E8M0 group scales (uint8 [R, 4])."""
    return kI_scale is not None and kI_scale.dtype == torch.uint8


def _ki_dtype(kI_scale) -> int:
    if kI_scale is None:
        return DSA_KI_BF16
    return DSA_KI_MXFP8 if _is_mx(kI_scale) else DSA_KI_FP8_E4M3


def _need_attn_inputs(seqs: "Seqs", q, kv, out, lse, kv_scale=None) -> torch.device:
    dev = _cuda_device(q, "q")
    _need_seqs(seqs, dev)
    _need(q, "q", _BF16T, (seqs.num_q_tokens, None, 576), dev)
    T, H = q.shape[0], q.shape[1]
    rows = seqs.num_phys_pages * 64
    if kv_scale is None:
        _need(kv, "kv", _BF16T, (None, 576), dev, rows)
    else:  # FP8 latent cache: E4M3 codes and per-row tile-scale bytes
        _need(kv, "kv", _FP8T, (None, 576), dev, rows)
        _need(kv_scale, "kv_scale", (torch.uint8,), (None, 8), dev, rows)
    _need(out, "out", (torch.bfloat16, torch.float32), (T, H, 512), dev)
    if lse is not None:
        _need(lse, "lse", _F32T, (T, H), dev)
    return dev


# ---------------------------------------------------------------------------
# Batch geometry
# ---------------------------------------------------------------------------


@dataclass
class Seqs:
    """Batch geometry on the device (see dsa_seqs_t in include/dsa.h)."""
    q_seq_start: torch.Tensor   # int32 [B+1]
    ctx_len: torch.Tensor       # int32 [B]
    page_table: torch.Tensor    # int32 [B, max_pages]
    num_phys_pages: int
    max_ctx: int
    num_q_tokens: int

    @staticmethod
    def from_host(q_seq_start, ctx_len, page_table, num_phys_pages: int, device="cuda") -> "Seqs":
        qs = torch.as_tensor(q_seq_start, dtype=torch.int32)
        cl = torch.as_tensor(ctx_len, dtype=torch.int32)
        pt = torch.as_tensor(page_table, dtype=torch.int32)
        return Seqs(qs.to(device), cl.to(device), pt.contiguous().to(device), int(num_phys_pages),
                    int(cl.max()), int(qs[-1]))

    @property
    def batch(self) -> int:
        return self.ctx_len.shape[0]

    def c(self) -> DsaSeqsC:
        return DsaSeqsC(self.batch, self.num_q_tokens, 64, self.page_table.shape[1], self.num_phys_pages,
                        self.max_ctx, self.q_seq_start.data_ptr(), self.ctx_len.data_ptr(),
                        self.page_table.data_ptr())


def dsa_workspace_size(op: int, seqs: Seqs | None = None, K: int = 1, H: int = 16, *, rows: int = 0,
                       ld: int = 0) -> int:
    c = seqs.c() if seqs is not None else DsaSeqsC(1, rows, 64, 1, 1, ld, None, None, None)
    return int(_lib.dsa_workspace_size(op, ctypes.byref(c), K, H))


_ws_cache: dict = {}


def workspace(nbytes: int, device, key=None) -> torch.Tensor:
    """A zeroed device workspace of at least nbytes, cached per (device, key).

    Every call that is not given `ws` uses this cached buffer, whatever its
    stream.  Calls that may run at the same time on different streams must
    each pass a workspace of their own: the library requires that concurrent
    calls do not share one (its first word is the sticky error flag)."""
    device = torch.device(device)
    if device.type == "cuda" and device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    k = (device, key)
    ws = _ws_cache.get(k)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[k] = ws
    return ws


# ---------------------------------------------------------------------------
# Entry points
# ---------------------------------------------------------------------------


def dsa_quantize_index_query(qI: torch.Tensor, w: torch.Tensor, codes=None, w_scaled=None):
    dev = _cuda_device(qI, "qI")
    T = qI.shape[0]
    codes = codes if codes is not None else torch.empty((T, 64, 128), dtype=torch.uint8, device=qI.device)
    w_scaled = w_scaled if w_scaled is not None else torch.empty((T, 64), dtype=torch.float32, device=qI.device)
    _need(qI, "qI", _BF16T, (T, 64, 128), dev)
    _need(w, "w", _F32T, (T, 64), dev)
    _need(codes, "codes", _FP8T, (T, 64, 128), dev)
    _need(w_scaled, "w_scaled", _F32T, (T, 64), dev)
    _check(_lib.dsa_quantize_index_query(_ptr(qI), _ptr(w), T, _ptr(codes), _ptr(w_scaled), _stream(qI.device)),
           "dsa_quantize_index_query")
    return codes, w_scaled


def dsa_quantize_index_query_mx(qI: torch.Tensor, codes=None, scales=None):
    dev = _cuda_device(qI, "qI")
    T = qI.shape[0]
    codes = codes if codes is not None else torch.empty((T, 64, 128), dtype=torch.uint8, device=qI.device)
    scales = scales if scales is not None else torch.empty((T, 64, 4), dtype=torch.uint8, device=qI.device)
    _need(qI, "qI", _BF16T, (T, 64, 128), dev)
    _need(codes, "codes", _FP8T, (T, 64, 128), dev)
    _need(scales, "scales", (torch.uint8,), (T, 64, 4), dev)
    _check(_lib.dsa_quantize_index_query_mx(_ptr(qI), T, _ptr(codes), _ptr(scales), _stream(qI.device)),
           "dsa_quantize_index_query_mx")
    return codes, scales


def dsa_index_scores(seqs: Seqs, qI, w, kI, kI_scale=None, scores=None, ld=None, ws=None):
    """Scores into `scores` [T, ld] fp32 (allocated zeroed when None).  When
    `scores` is given, ld defaults to its row stride and must equal it."""
    dev = _need_index_inputs(seqs, qI, w, kI, kI_scale)
    T = seqs.num_q_tokens
    if scores is None:
        ld = ld or (seqs.max_ctx + 3) // 4 * 4
        scores = torch.zeros((T, ld), dtype=torch.float32, device=qI.device)
    else:
        _need(scores, "scores", _F32T, (T, None), dev)
        if ld is not None and ld != scores.stride(0):
            raise ValueError(f"ld={ld} differs from the row stride {scores.stride(0)} of scores")
        ld = scores.stride(0)
    ki_dtype = _ki_dtype(kI_scale)
    c = seqs.c()
    need = _lib.dsa_workspace_size(DSA_OP_INDEX_SCORES, ctypes.byref(c), 1, 16)
    ws = ws if ws is not None else workspace(need, qI.device, "index_scores")
    _need_ws(ws, dev)
    _check(_lib.dsa_index_scores(ctypes.byref(c), _ptr(qI), _ptr(w), _ptr(kI), _ptr(kI_scale), ki_dtype, _ptr(scores),
                                 ld, _ptr(ws), ws.numel(), _stream(qI.device)), "dsa_index_scores")
    return scores


def dsa_topk(scores: torch.Tensor, row_len: torch.Tensor, K: int, idx=None, ws=None):
    """Top-K of each fp32 row of `scores` [T, ld] (contiguous) over its first
    row_len[t] entries, into idx [T, K] int32."""
    dev = _cuda_device(scores, "scores")
    _need(scores, "scores", _F32T, (None, None), dev)
    T, ld = scores.shape
    idx = idx if idx is not None else torch.empty((T, K), dtype=torch.int32, device=scores.device)
    _need(row_len, "row_len", _I32T, (T,), dev)
    _need(idx, "idx", _I32T, (T, K), dev)
    c = DsaSeqsC(1, T, 64, 1, 1, ld, None, None, None)
    need = _lib.dsa_workspace_size(DSA_OP_TOPK, ctypes.byref(c), K, 16)
    ws = ws if ws is not None else workspace(need, scores.device, "topk")
    _need_ws(ws, dev)
    _check(_lib.dsa_topk(_ptr(scores), ld, T, _ptr(row_len), K, _ptr(idx), _ptr(ws), ws.numel(),
                         _stream(scores.device)), "dsa_topk")
    return idx


def _out_dtype(out: torch.Tensor) -> int:
    if out.dtype == torch.bfloat16:
        return DSA_OUT_BF16
    if out.dtype == torch.float32:
        return DSA_OUT_F32
    raise TypeError("out must be bfloat16 or float32")


def dsa_sparse_mla_fwd(seqs: Seqs, q, kv, idx, scale: float, out=None, lse=None, want_lse=True, ws=None,
                       out_dtype=torch.bfloat16, kv_scale=None):
    """Sparse MLA over the selected rows.  kv_scale (uint8 [R, 8]) marks an FP8
    latent cache: kv then holds E4M3 codes [R, 576] (dsa_sparse_mla_fwd_ex)."""
    T, H, _ = q.shape
    K = idx.shape[1]
    out = out if out is not None else torch.empty((T, H, 512), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    dev = _need_attn_inputs(seqs, q, kv, out, lse, kv_scale)
    _need(idx, "idx", _I32T, (T, K), dev)
    c = seqs.c()
    need = _lib.dsa_workspace_size(DSA_OP_SPARSE_MLA, ctypes.byref(c), K, H)
    ws = ws if ws is not None else workspace(need, q.device, "sparse_mla")
    _need_ws(ws, dev)
    kv_dtype = DSA_KV_BF16 if kv_scale is None else DSA_KV_FP8_E4M3
    _check(_lib.dsa_sparse_mla_fwd_ex(ctypes.byref(c), _ptr(q), _ptr(kv), _ptr(kv_scale), kv_dtype, _ptr(idx), K, H,
                                      scale, _ptr(out), _out_dtype(out), _ptr(lse), _ptr(ws), ws.numel(),
                                      _stream(q.device)), "dsa_sparse_mla_fwd")
    return out, lse


def dsa_sparse_mla_fwd_noalloc(seqs: Seqs, q, kv, idx, scale: float, out=None, lse=None, want_lse=True,
                               out_dtype=torch.bfloat16):
    """dsa_sparse_mla_fwd without a workspace: the library's built-in scratch
    array is used (for callers that cannot allocate device memory; see
    include/dsa.h).  Outputs not passed in are allocated here for convenience."""
    T, H, _ = q.shape
    K = idx.shape[1]
    out = out if out is not None else torch.empty((T, H, 512), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    dev = _need_attn_inputs(seqs, q, kv, out, lse)
    _need(idx, "idx", _I32T, (T, K), dev)
    c = seqs.c()
    _check(_lib.dsa_sparse_mla_fwd_noalloc(ctypes.byref(c), _ptr(q), _ptr(kv), _ptr(idx), K, H, scale, _ptr(out),
                                           _out_dtype(out), _ptr(lse), _stream(q.device)),
           "dsa_sparse_mla_fwd_noalloc")
    return out, lse


def dsa_index_topk_attn(seqs: Seqs, qI, w, kI, kI_scale, q, kv, K: int, scale: float, out=None, lse=None,
                        idx_out=None, want_lse=True, ws=None, out_dtype=torch.bfloat16, q_ready=None,
                        select_in_indexer=False, kv_scale=None):
    """The whole path.  q_ready (a torch.cuda.Event, optional): the attention
    launch waits on it, so q may still be in flight on another stream.
    select_in_indexer: decode rows that fit are selected inside the indexer
    kernel (DSA_SELECT_IN_INDEXER).  kv_scale (uint8 [R, 8]) marks an FP8
    latent cache (kv = E4M3 codes [R, 576])."""
    T, H, _ = q.shape
    out = out if out is not None else torch.empty((T, H, 512), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    dev = _need_attn_inputs(seqs, q, kv, out, lse, kv_scale)
    if _need_index_inputs(seqs, qI, w, kI, kI_scale, check_seqs=False) != dev:
        raise ValueError("qI and q are on different devices")
    if idx_out is not None:
        _need(idx_out, "idx_out", _I32T, (T, K), dev)
    ki_dtype = _ki_dtype(kI_scale)
    c = seqs.c()
    op = DSA_OP_INDEX_TOPK_ATTN_FUSED if select_in_indexer else DSA_OP_INDEX_TOPK_ATTN
    need = _lib.dsa_workspace_size(op, ctypes.byref(c), K, H)
    ws = ws if ws is not None else workspace(need, q.device, "index_topk_attn")
    _need_ws(ws, dev)
    ev = None if q_ready is None else ctypes.c_void_p(q_ready.cuda_event)
    kv_dtype = DSA_KV_BF16 if kv_scale is None else DSA_KV_FP8_E4M3
    _check(_lib.dsa_index_topk_attn_ex(ctypes.byref(c), _ptr(qI), _ptr(w), _ptr(kI), _ptr(kI_scale), ki_dtype, _ptr(q),
                                       _ptr(kv), _ptr(kv_scale), kv_dtype, K, H, scale, _ptr(out), _out_dtype(out),
                                       _ptr(lse), _ptr(idx_out), _ptr(ws), ws.numel(),
                                       DSA_SELECT_IN_INDEXER if select_in_indexer else 0, ev, _stream(q.device)),
           "dsa_index_topk_attn")
    return out, lse


def dsa_check_error(ws: torch.Tensor) -> int:
    """Synchronise the current stream and return (and clear) the device error status."""
    return int(_lib.dsa_check_error(_ptr(ws), _stream(ws.device)))


def dsa_check_error_noalloc(device=None) -> int:
    """dsa_check_error for the built-in scratch of dsa_sparse_mla_fwd_noalloc
    (synchronises the current stream of `device`)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(_lib.dsa_check_error_noalloc(_stream(dev)))


def dsa_set_wait_limit_ns(ns: int) -> None:
    """Limit of every bounded in-kernel wait of this thread's later calls (0 = the 2 s default)."""
    _check(_lib.dsa_set_wait_limit_ns(int(ns)), "dsa_set_wait_limit_ns")


def dsa_launches_in_last_call() -> int:
    """Kernels launched by this thread's most recent entry-point call."""
    return int(_lib.dsa_launches_in_last_call())


def dsa_launch_timing(enable: bool) -> None:
    """Record device events around every kernel of this thread's later calls."""
    _check(_lib.dsa_launch_timing(1 if enable else 0), "dsa_launch_timing")


def dsa_last_launch_times() -> list:
    """[(kernel name, device ms)] of this thread's last call made with timing on."""
    cap = 16
    ms = (ctypes.c_float * cap)()
    names = (ctypes.c_char_p * cap)()
    n = int(_lib.dsa_last_launch_times(ms, names, cap))
    if n < 0:
        raise DsaError(DSA_ERR_CUDA, "dsa_last_launch_times")
    return [(names[i].decode(), float(ms[i])) for i in range(min(n, cap))]


def raw():
    """The ctypes handle of libdsa (for tests that call the C ABI directly)."""
    return _lib
