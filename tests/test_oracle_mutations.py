"""The oracle's pins catch plausible mistakes.

Each mutant below is the oracle with one plausible slip planted in a copy of its
source: a dropped term, a wrong sign, index or exponent, a transposed or
mis-sliced operand, a wrong tie rule.  The pin files that cover the mutated
function run against the copy in a child process, and must fail.  The
unmutated copy must pass the same files, so a failure means the pins saw the
slip and not that the harness broke.  Nothing here touches a GPU."""
import os
import shutil
import subprocess
import sys

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
ORACLE = os.path.join(ROOT, "oracle", "dsa_oracle.py")

CODEC, QUANT, INDEXER = "test_oracle_codec.py", "test_oracle_quant.py", "test_oracle_indexer.py"
TOPK, ATTN, PIPE = "test_oracle_topk.py", "test_oracle_attention.py", "test_oracle_pipeline.py"
MX, KV8 = "test_oracle_mx.py", "test_oracle_kv8.py"

# name: (text in the oracle, replacement, pin files that must fail)
MUTANTS = {
    "bf16_shift": ("<< np.uint32(16)", "<< np.uint32(15)", [CODEC]),
    "e4m3_bias": ("np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)", [CODEC]),
    "e4m3_subnormal_step": ("m * 2.0 ** -9", "m * 2.0 ** -10", [CODEC]),
    "e4m3_no_saturation": ("    code = np.where(a >= E4M3_MAX, 126, code)\n", "", [CODEC]),
    "e4m3_ties_away": ("round_up = (d_lo > d_hi) | ((d_lo == d_hi) & (i % 2 == 1))", "round_up = (d_lo >= d_hi)",
                       [CODEC]),
    "quant_exponent_off_by_one": ("        e -= 1\n    return e\n", "        e -= 1\n    return e + 1\n", [QUANT]),
    "quant_scale_dropped": ("codes = e4m3_encode(q / sq[..., None])", "codes = e4m3_encode(q)", [QUANT]),
    "index_relu_dropped": ("score = wt @ np.maximum(dots, 0.0)", "score = wt @ dots", [INDEXER]),
    "index_relu_after_head_sum": ("score = wt @ np.maximum(dots, 0.0)", "score = np.maximum(wt @ dots, 0.0)",
                                  [INDEXER]),
    "index_key_scale_wrong_row": ("score = score * np.asarray(kI_scale, dtype=np.float64)[rows]",
                                  "score = score * np.asarray(kI_scale, dtype=np.float64)[rows[::-1]]", [INDEXER]),
    "index_query_scale_dropped": ("wt = w[t] * sq[t]", "wt = w[t]", [INDEXER]),
    "index_own_position_dropped": ("rows = seqs.rows(b, np.arange(pos + 1))",
                                   "rows = seqs.rows(b, np.arange(max(pos, 1)))", [INDEXER]),
    "prefill_position_off_by_one": (
        "pos = int(self.ctx_len[b]) - q_len + (t - int(self.q_seq_start[b]))",
        "pos = int(self.ctx_len[b]) - q_len + (t - int(self.q_seq_start[b])) - (1 if q_len > 1 else 0)",
        [INDEXER]),
    "topk_ties_prefer_high_position": ("order = np.lexsort((np.arange(n), -s))",
                                       "order = np.lexsort((-np.arange(n), -s))", [TOPK]),
    "topk_not_position_sorted": ("chosen = np.sort(order[: min(K, n)])", "chosen = order[: min(K, n)]", [TOPK]),
    "topk_one_short": ("chosen = np.sort(order[: min(K, n)])", "chosen = np.sort(order[: min(K, n) - 1])", [TOPK]),
    "attn_value_slice": ("out[i] = (p @ kmat[:, :d_v]) / l", "out[i] = (p @ kmat[:, -d_v:]) / l", [ATTN]),
    "attn_lse_without_max": ("lse[i] = (m + np.log(l))[:, 0]", "lse[i] = (np.log(l))[:, 0]", [ATTN]),
    "attn_scale_dropped": ("logits = scale * (qt @ kmat.T)", "logits = qt @ kmat.T", [ATTN]),
    "attn_rope_dims_dropped": ("logits = scale * (qt @ kmat.T)", "logits = scale * (qt[:, :d_v] @ kmat[:, :d_v].T)",
                               [ATTN]),
    "dense_mask_one_short": ("logit[: pos + 1] = scale * (full[: pos + 1] @ qh)",
                             "logit[: pos] = scale * (full[: pos] @ qh)", [ATTN]),
    "path_rows_to_wrong_tokens": ("full_idx[t] = idx_rows[i]", "full_idx[i] = idx_rows[i]", [PIPE]),
    "mx_exponent_off_by_one": ("ex - 1 - E4M3_EMAX", "ex - E4M3_EMAX", [MX]),
    "mx_no_clamp": ("return int(min(127, max(-127, ex - 1 - E4M3_EMAX)))", "return int(ex - 1 - E4M3_EMAX)", [MX]),
    "mx_block_16": ("MX_BLOCK = 32        # elements sharing one scale", "MX_BLOCK = 16        # elements sharing one scale",
                    [MX]),
    "mx_e8m0_bias": ("v = np.ldexp(1.0, c - E8M0_BIAS)", "v = np.ldexp(1.0, c - E8M0_BIAS + 1)", [MX]),
    "mx_query_not_quantized": ("qvals = mxfp8_dequantize(*mxfp8_quantize(bf16_to_f64(qI_bits)))",
                               "qvals = bf16_to_f64(qI_bits)", [MX]),
    "mx_key_scale_dropped": ("kmat = mxfp8_dequantize(np.asarray(kI)[rows], np.asarray(kI_scale)[rows])",
                             "kmat = e4m3_decode_fast(np.asarray(kI)[rows])", [MX]),
    "mx_key_scale_wrong_row": ("kmat = mxfp8_dequantize(np.asarray(kI)[rows], np.asarray(kI_scale)[rows])",
                               "kmat = mxfp8_dequantize(np.asarray(kI)[rows], np.asarray(kI_scale)[rows[::-1]])", [MX]),
    "mx_blocks_strided": ("blocks = x.reshape(*x.shape[:-1], n // MX_BLOCK, MX_BLOCK)",
                          "blocks = x.reshape(*x.shape[:-1], MX_BLOCK, n // MX_BLOCK).swapaxes(-1, -2)", [MX]),
    "mx_dequantize_strided": ("v = e4m3_decode_fast(c).reshape(*c.shape[:-1], n // MX_BLOCK, MX_BLOCK)",
                              "v = e4m3_decode_fast(c).reshape(*c.shape[:-1], MX_BLOCK, n // MX_BLOCK)"
                              ".swapaxes(-1, -2)", [MX]),
    "kv8_tile_64": ("KV_TILE = 128        # elements per scale", "KV_TILE = 64         # elements per scale", [KV8]),
    "kv8_scale_dropped": ("v[..., lo:hi] *= e8m0_decode(sc[..., j])[..., None]", "v[..., lo:hi] *= 1.0", [KV8]),
    "kv8_scale_of_first_tile": ("v[..., lo:hi] *= e8m0_decode(sc[..., j])[..., None]",
                                "v[..., lo:hi] *= e8m0_decode(sc[..., 0])[..., None]", [KV8]),
    "kv8_rope_tile_unscaled": ("for j in range((c.shape[-1] + KV_TILE - 1) // KV_TILE):",
                               "for j in range(c.shape[-1] // KV_TILE):", [KV8]),
    "index_weight_of_first_token": ("wt = w[t] * sq[t]", "wt = w[0] * sq[t]", [INDEXER]),
    "page_offset_reversed": ("return pages * self.page_size + s % self.page_size",
                             "return pages * self.page_size + (self.page_size - 1 - s % self.page_size)",
                             [INDEXER, ATTN, PIPE]),
    "attn_lse_base_2": ("lse[i] = (m + np.log(l))[:, 0]", "lse[i] = (m + np.log2(l))[:, 0]", [ATTN]),
    "kv8_scale_byte_bias": ("scales[:, j] = (e + E8M0_BIAS).astype(np.uint8)",
                            "scales[:, j] = (e + E8M0_BIAS + 1).astype(np.uint8)", [KV8]),
    "kv8_attention_reads_raw_codes": ("return kv_fp8_dequantize(np.asarray(codes)[rows], np.asarray(scales)[rows])",
                                      "return e4m3_decode_fast(np.asarray(codes)[rows])", [KV8]),
}


def _tree(base, name, source):
    d = os.path.join(base, name)
    os.makedirs(os.path.join(d, "oracle"))
    with open(os.path.join(d, "oracle", "dsa_oracle.py"), "w") as f:
        f.write(source)
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(d, "oracle", "__init__.py"))
    shutil.copytree(TESTS, os.path.join(d, "tests"), ignore=shutil.ignore_patterns("__pycache__", "test_gpu_*"))
    return d


def _launch(d, files):
    env = dict(os.environ, PYTHONPATH=d, PYTHONDONTWRITEBYTECODE="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu",
           *[os.path.join("tests", f) for f in files]]
    return subprocess.Popen(cmd, cwd=d, env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(ORACLE) as f:
        src = f.read()
    for name, (old, new, _) in MUTANTS.items():
        assert src.count(old) == 1, f"{name}: the mutated text must occur exactly once in the oracle"
    all_files = sorted({f for *_, files in MUTANTS.values() for f in files})
    procs = {"unmutated": (_launch(_tree(tmp_path, "unmutated", src), all_files), True)}
    for name, (old, new, files) in MUTANTS.items():
        procs[name] = (_launch(_tree(tmp_path, name, src.replace(old, new)), files), False)
    missed, broken = [], None
    for name, (p, must_pass) in procs.items():
        out, _ = p.communicate(timeout=600)
        if must_pass and p.returncode != 0:
            broken = out[-2000:]
        elif not must_pass and p.returncode == 0:
            missed.append(name)
    assert broken is None, "the unmutated oracle failed its own pins:\n" + broken
    assert not missed, f"mutants no pin caught: {missed}"
