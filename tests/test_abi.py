"""The C-ABI library without a GPU: it loads, exports every function that
include/dsa.h declares, and its host-side validation answers before any
launch.  No call here reaches a CUDA kernel."""
import ctypes
import os
import re
import subprocess

import sparse_indexed_attention_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^[A-Za-z_][\w \*]*?\b(dsa_\w+)\s*\(", src, flags=re.M))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared()
    assert {"dsa_index_scores", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_index_topk_attn"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dsa_\w+)", out))
    assert declared <= exported, declared - exported
    assert set(dsa.EXPORTS) == declared
    lib = dsa.raw()
    for name in declared:
        assert getattr(lib, name) is not None


def test_binding_constants_match_the_header():
    """Every enumerator and #define value of include/dsa.h has the same value
    in the binding (the binding restates them for ctypes)."""
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    consts = {n: int(v) for n, v in re.findall(r"^\s*(DSA_[A-Z0-9_]+)\s*=\s*(\d+)", src, flags=re.M)}
    for n, a, b in re.findall(r"^#define\s+(DSA_[A-Z0-9_]+)\s+\((\d+)u\s*<<\s*(\d+)\)", src, flags=re.M):
        consts[n] = int(a) << int(b)
    assert len(consts) >= 20 and "DSA_NOALLOC_SCRATCH_BYTES" in consts
    for name, value in consts.items():
        assert getattr(dsa, name) == value, name


def _ctype_of(param: str):
    """The ctypes class a C parameter (or return) declaration marshals as."""
    p = " ".join(param.replace("const", " ").split())
    if "*" in p or p.split()[0] in ("dsa_stream_t", "dsa_event_t"):
        return "pointer"
    base = p.split()[0]
    return {"int": ctypes.c_int, "int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "size_t": ctypes.c_size_t,
            "float": ctypes.c_float, "unsigned": ctypes.c_uint, "uint64_t": ctypes.c_uint64,
            "dsa_status_t": ctypes.c_int, "dsa_op_t": ctypes.c_int, "dsa_ki_dtype_t": ctypes.c_int,
            "dsa_kv_dtype_t": ctypes.c_int, "dsa_out_dtype_t": ctypes.c_int}[base]


def test_binding_signatures_match_the_header():
    """Each ctypes prototype has the header's parameter count and, parameter by
    parameter, a type of the same width (pointers as pointers)."""
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    protos = re.findall(r"^([A-Za-z_][\w \*]*?)\b(dsa_\w+)\s*\(([^;{]*?)\)\s*;", src, flags=re.M | re.S)
    assert {n for _, n, _ in protos} == set(dsa.EXPORTS)
    for ret, name, params in protos:
        res, args = dsa._sig[name]
        params = [] if params.strip() in ("", "void") else [x.strip() for x in params.split(",")]
        assert len(args) == len(params), name
        for i, (decl, got) in enumerate(zip(params, args)):
            want = _ctype_of(decl)
            if want == "pointer":
                assert got in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(got, ctypes._Pointer), (name, i, decl)
            else:
                assert ctypes.sizeof(got) == ctypes.sizeof(want), (name, i, decl, got)
        want = _ctype_of(ret.strip())
        if want == "pointer":
            assert res in (ctypes.c_void_p, ctypes.c_char_p), name
        else:
            assert ctypes.sizeof(res) == ctypes.sizeof(want), (name, "return")


def test_seqs_struct_layout_matches_the_header(tmp_path):
    """dsa_seqs_t as a C compiler lays it out (size, field offsets, enum size)
    equals the binding's ctypes structure."""
    fields = [f for f, _ in dsa.DsaSeqsC._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "dsa.h"', "int main(void) {",
            '  printf("%zu %zu\\n", sizeof(dsa_seqs_t), sizeof(dsa_ki_dtype_t));']
    prog += [f'  printf("%zu\\n", offsetof(dsa_seqs_t, {f}));' for f in fields]
    prog += ["  return 0;", "}"]
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-x", "c", "-",
                    "-o", str(exe)], input="\n".join(prog), text=True, check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    size, enum_size, *offsets = map(int, out)
    assert size == ctypes.sizeof(dsa.DsaSeqsC) and enum_size == ctypes.sizeof(ctypes.c_int)
    assert offsets == [getattr(dsa.DsaSeqsC, f).offset for f in fields]


def test_status_strings():
    for code, name in enumerate(["DSA_OK", "DSA_ERR_INVALID_ARG", "DSA_ERR_UNSUPPORTED", "DSA_ERR_WORKSPACE",
                                 "DSA_ERR_CUDA", "DSA_ERR_BAD_INDEX", "DSA_ERR_TIMEOUT"]):
        assert dsa.status_string(code) == name
    assert dsa.status_string(99) == "DSA_ERR_UNKNOWN"


def _fake_seqs(T=4, B=1, max_ctx=100, page_size=64, max_pages=2, phys=8):
    # host struct with non-null but never-dereferenced device pointers
    fake = 0x10000
    return dsa.DsaSeqsC(B, T, page_size, max_pages, phys, max_ctx, fake, fake, fake)


def test_workspace_sizes():
    lib = dsa.raw()
    s = _fake_seqs(T=8, max_ctx=131072, max_pages=2048)
    sz = {op: lib.dsa_workspace_size(op, ctypes.byref(s), 2048, 128) for op in range(5)}
    assert sz[dsa.DSA_OP_QUANTIZE_INDEX_QUERY] == 0
    assert sz[dsa.DSA_OP_INDEX_TOPK_ATTN] >= 8 * 131072 * 4 + 8 * 2048 * 4
    assert all(v % 256 == 0 for v in sz.values())
    assert lib.dsa_workspace_size(dsa.DSA_OP_SPARSE_MLA, ctypes.byref(s), 4096, 128) == 0     # K too large
    assert lib.dsa_workspace_size(dsa.DSA_OP_SPARSE_MLA, ctypes.byref(s), 2048, 100) == 0     # bad H
    assert lib.dsa_workspace_size(dsa.DSA_OP_TOPK, None, 16, 16) == 0


def test_host_validation_rejects_before_launch():
    lib = dsa.raw()
    P = ctypes.c_void_p
    good = P(0x10000)   # 256-aligned fake pointer, never dereferenced on these paths
    s = _fake_seqs()
    # dsa_topk
    assert lib.dsa_topk(None, 128, 4, good, 16, good, good, 1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk(good, 128, 4, good, 0, good, good, 1 << 20, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_topk(good, 128, 4, good, 4096, good, good, 1 << 20, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_topk(good, 128, 4, good, 16, good, None, 1 << 20, None) == dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_topk(good, 128, 4, good, 16, good, P(0x10010), 1 << 20, None) == dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_topk(P(0x10004), 128, 4, good, 16, good, good, 1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    # dsa_sparse_mla_fwd
    f = ctypes.c_float(0.04)
    B16 = dsa.DSA_OUT_BF16
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(s), good, good, good, 16, 100, f, good, B16, None, good, 1 << 20,
                                  None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(s), good, good, good, 16, 128, f, good, 7, None, good, 1 << 20,
                                  None) == dsa.DSA_ERR_UNSUPPORTED                  # unknown output dtype
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(s), good, good, good, 16, 128, ctypes.c_float(float("nan")), good,
                                  B16, None, good, 1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(s), good, good, good, 16, 128, f, good, B16, None, good, 16,
                                  None) == dsa.DSA_ERR_WORKSPACE
    bad_ps = _fake_seqs(page_size=32)
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(bad_ps), good, good, good, 16, 128, f, good, B16, None, good,
                                  1 << 20, None) == dsa.DSA_ERR_UNSUPPORTED
    for phys, want in (((1 << 25) - 1, dsa.DSA_OK), (1 << 25, dsa.DSA_ERR_UNSUPPORTED)):  # 2^31 pool rows
        big = _fake_seqs(phys=phys)
        got = lib.dsa_sparse_mla_fwd(ctypes.byref(big), good, good, good, 16, 128, f, good, B16, None, good, 16,
                                     None)
        assert got == (dsa.DSA_ERR_WORKSPACE if want == dsa.DSA_OK else want)  # past the pool check: workspace
    small_pt = _fake_seqs(max_ctx=200, max_pages=2)
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(small_pt), good, good, good, 16, 128, f, good, B16, None, good,
                                  1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    # dsa_index_scores: FP8 cache needs scales, bf16 cache must not have them
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, good, None, dsa.DSA_KI_FP8_E4M3, good, 128, good,
                                1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, good, good, dsa.DSA_KI_BF16, good, 128, good,
                                1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, good, None, dsa.DSA_KI_BF16, good, 64, good,
                                1 << 20, None) == dsa.DSA_ERR_INVALID_ARG      # ld < max_ctx
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, P(0x10040), None, dsa.DSA_KI_BF16, good, 128, good,
                                1 << 20, None) == dsa.DSA_ERR_INVALID_ARG      # pool not 128-B aligned
    assert lib.dsa_index_scores(None, good, good, good, None, dsa.DSA_KI_BF16, good, 128, good, 1 << 20,
                                None) == dsa.DSA_ERR_INVALID_ARG
    # fused entry point
    assert lib.dsa_index_topk_attn(ctypes.byref(s), good, good, good, None, dsa.DSA_KI_BF16, good, good, 0, 128, f,
                                   good, B16, None, None, good, 1 << 30, None) == dsa.DSA_ERR_UNSUPPORTED
    # quantizer
    assert lib.dsa_quantize_index_query(good, good, 0, good, good, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_check_error(None, None) == dsa.DSA_ERR_WORKSPACE


def test_host_validation_of_cache_formats_and_options():
    """The index-cache and latent-cache formats, the flags and the MXFP8
    quantizer are checked on the host, before any launch."""
    lib = dsa.raw()
    P = ctypes.c_void_p
    good = P(0x10000)
    s = _fake_seqs()
    f = ctypes.c_float(0.04)
    B16, MX, E4 = dsa.DSA_OUT_BF16, dsa.DSA_KI_MXFP8, dsa.DSA_KI_FP8_E4M3
    KB, K8 = dsa.DSA_KV_BF16, dsa.DSA_KV_FP8_E4M3
    # MXFP8 index cache: scales required; an unknown cache kind is unsupported
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, good, None, MX, good, 128, good, 1 << 20,
                                None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, good, good, 7, good, 128, good, 1 << 20,
                                None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_index_scores(ctypes.byref(s), good, good, good, P(0x10008), MX, good, 128, good, 1 << 20,
                                None) == dsa.DSA_ERR_INVALID_ARG               # scales not 16-B aligned

    def attn_ex(kv_scale, kv_dtype, flags=0, kI_scale=good, ki=E4):
        return lib.dsa_index_topk_attn_ex(ctypes.byref(s), good, good, good, kI_scale, ki, good, good, kv_scale,
                                          kv_dtype, 16, 128, f, good, B16, None, None, good, 1 << 30, flags, None,
                                          None)
    assert attn_ex(None, K8) == dsa.DSA_ERR_INVALID_ARG                        # FP8 latent cache without scales
    assert attn_ex(good, KB) == dsa.DSA_ERR_INVALID_ARG                        # bf16 pool with scales
    assert attn_ex(None, 5) == dsa.DSA_ERR_UNSUPPORTED                         # unknown latent format
    assert attn_ex(P(0x10008), K8) == dsa.DSA_ERR_INVALID_ARG                  # scales not 16-B aligned
    assert attn_ex(None, KB, flags=2) == dsa.DSA_ERR_INVALID_ARG               # unknown flag
    assert attn_ex(None, KB, kI_scale=None, ki=MX) == dsa.DSA_ERR_INVALID_ARG
    # attention alone
    assert lib.dsa_sparse_mla_fwd_ex(ctypes.byref(s), good, good, None, K8, good, 16, 128, f, good, B16, None,
                                     good, 1 << 20, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_mla_fwd_ex(ctypes.byref(s), good, good, good, 9, good, 16, 128, f, good, B16, None,
                                     good, 1 << 20, None) == dsa.DSA_ERR_UNSUPPORTED
    # MXFP8 quantizer
    assert lib.dsa_quantize_index_query_mx(good, 0, good, good, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_quantize_index_query_mx(good, 4, good, P(0x10002), None) == dsa.DSA_ERR_INVALID_ARG


def test_in_indexer_selection_workspace_has_no_score_scratch():
    """With the selection inside the indexer the decode workspace drops the
    [T, ld] fp32 scores and Top-K's scratch (row histograms and candidate
    lists take their place)."""
    lib = dsa.raw()
    s = _fake_seqs(T=8, B=8, max_ctx=131072, max_pages=2048, phys=32768)
    plain = lib.dsa_workspace_size(dsa.DSA_OP_INDEX_TOPK_ATTN, ctypes.byref(s), 2048, 128)
    fused = lib.dsa_workspace_size(dsa.DSA_OP_INDEX_TOPK_ATTN_FUSED, ctypes.byref(s), 2048, 128)
    assert 0 < fused and plain - fused >= 8 * 131072 * 4
