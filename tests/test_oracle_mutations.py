"""The oracle's pins catch plausible mistakes (CPU only).

One mistake at a time is planted in a copy of the oracle's C source (a
dropped term, a wrong sign or index, a swapped operand, a wrong rounding or
offset), the copy is rebuilt, and the oracle pin suites run against it: each
planted mistake must make at least one pin fail.  The real oracle is never
touched; every copy lives in a temporary directory.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_SUITES = ["tests/test_oracle_ops.py", "tests/test_oracle_codecs.py", "tests/test_oracle_decompress.py"]

# name: (text in the oracle source, replacement)
MUTANTS = {
    "mode 0 divides by the unrounded scale": (
        "row[64 * g + i] = (sf == 0.0f) ? 0u : enc_e4m3(xg[i] / sf);",
        "row[64 * g + i] = (sf == 0.0f) ? 0u : enc_e4m3(xg[i] / s);"),
    "E8M0 rounds down": (
        "if (ldexp(1.0, b - 127) >= (double)q) return (uint8_t)b;",
        "if (ldexp(1.0, b - 126) > (double)q) return (uint8_t)b;"),
    "RMSNorm drops epsilon": ("float rms = sqrtf(mean + eps);", "float rms = sqrtf(mean) + 0.0f * eps;"),
    "RMSNorm adds epsilon outside the root": ("float rms = sqrtf(mean + eps);", "float rms = sqrtf(mean) + eps;"),
    "RMSNorm drops gamma": ("y[i] = (x[i] / rms) * gamma[i];", "y[i] = (x[i] / rms);"),
    "RMSNorm averages over D": ("float mean = part[0] / (float)Dv;", "float mean = part[0] / (float)(Dv + 64);"),
    "interleaved RoPE sign": ("y[j] = x1 * c[j] + (-x2) * s[j];", "y[j] = x1 * c[j] + x2 * s[j];"),
    "interleaved RoPE operands swapped": (
        "y[h + j] = x2 * c[h + j] + x1 * s[h + j];", "y[h + j] = x1 * c[h + j] + x2 * s[h + j];"),
    "interleaved RoPE table index": (
        "y[h + j] = x2 * c[h + j] + x1 * s[h + j];", "y[h + j] = x2 * c[j] + x1 * s[j];"),
    "half-rotation RoPE sine not negated": ("float neg_s = -sn[j];", "float neg_s = sn[j];"),
    "half-rotation RoPE table index": (
        "out[j + h] = u[j + h] * cs[j + h] + u[j] * sn[j + h];", "out[j + h] = u[j + h] * cs[j] + u[j] * sn[j];"),
    "FP4 nibble order": (
        "row[e / 2] |= (uint8_t)(c << (4 * (e % 2)));", "row[e / 2] |= (uint8_t)(c << (4 * (1 - e % 2)));"),
    "dequant drops the activation scale": (
        "if (a->activation_scale) v = v * a->activation_scale[t];", "if (0) v = v * a->activation_scale[t];"),
    "dequant drops the bias": (
        "if (a->bias) v = v + bias_at(a->bias, a->bias_dtype, i);",
        "if (0) v = v + bias_at(a->bias, a->bias_dtype, i);"),
    "int8 drops the offset": ("if (a->offset_k) qk = qk + a->offset_k[c];", "if (0) qk = qk + a->offset_k[c];"),
    "int8 truncates": ("float r = nearbyintf(v);", "float r = truncf(v);"),
    "mode 2 rope ignores xScale": ("rope[j] = enc_e4m3(x[n + j] * x_scale);", "rope[j] = enc_e4m3(x[n + j]);"),
    "mode 1 scale byte off by one": ("scales[g] = b;\n", "scales[g] = b + 1;\n"),
    "bf16 rope bytes swapped": ("row[n + 2 * j + 0] = (uint8_t)(h & 0xFF);", "row[n + 2 * j + 0] = (uint8_t)(h >> 8);"),
    "padding not zero": ("memset(row, 0, (size_t)col);", "memset(row, 1, (size_t)col);"),
    "skipped tokens written": (
        "if (s == -1) continue;                               /* skipped token */", "if (s == -1) s = 0;"),
    "indexer format maxima swapped": (
        "const float fmax = quant_mode == KVQO_IDX_MXFP8 ? fp8_max : 6.0f;",
        "const float fmax = quant_mode == KVQO_IDX_MXFP8 ? 6.0f : fp8_max;"),
    "bf16 ties away from zero": ("return nearbyint(k) * quantum;", "return floor(k + 0.5) * quantum;"),
    "decoder drops the group scale": ("y[64 * g + i] = round_out(y_dtype, v * sf);",
                                      "y[64 * g + i] = round_out(y_dtype, v);"),
    "decoder multiplies the rope by xScale": (
        "y[n + j] = f32_to_bf16(decode_bits(&FMT_E4M3, rope[j]) / x_scale);",
        "y[n + j] = f32_to_bf16(decode_bits(&FMT_E4M3, rope[j]) * x_scale);"),
    "decoder FP4 nibble order": (
        "uint32_t c = (row[e / 2] >> (4 * (e % 2))) & 0xFu;", "uint32_t c = (row[e / 2] >> (4 * (1 - e % 2))) & 0xFu;"),
    "decoder E8M0 exponent bias": ("sf = (float)ldexp(1.0, (int)scales[g] - 127);",
                                   "sf = (float)ldexp(1.0, (int)scales[g] - 126);"),
    "rope re-encoded as bf16 instead of copied": ("uint16_t h = raw[n + j];", "uint16_t h = f32_to_bf16(x[n + j]);"),
    "f16 x read as bf16": ("xf[i] = load_half(x + t * x_row_stride, i, x_dtype);",
                           "xf[i] = load_half(x + t * x_row_stride, i, KVQO_IN_BF16);"),
    "decoder rounds f16 output as bf16": (
        "static uint16_t round_out(int y_dtype, float v) { return y_dtype == KVQO_IN_F16 ? f32_to_f16(v) : f32_to_bf16(v); }",
        "static uint16_t round_out(int y_dtype, float v) { return y_dtype == KVQO_IN_F16 ? f32_to_bf16(v) : f32_to_bf16(v); }"),
}


def _run_copy(d, src):
    """Run the pin suites against a copy of the repository's oracle whose C source is src."""
    for sub in ("oracle", "tests", "kv_cache_quantize_b200"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__", "_build"))
    with open(os.path.join(d, "oracle", "kvq_oracle.c"), "w") as f:
        f.write(src)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_SUITES],
                       cwd=d, capture_output=True, text=True, timeout=600)
    shutil.rmtree(d, ignore_errors=True)
    return r.returncode


def test_every_planted_mistake_is_caught(tmp_path):
    src = open(os.path.join(ROOT, "oracle", "kvq_oracle.c")).read()
    for name, (a, b) in MUTANTS.items():
        assert a in src, f"mutant site not found: {name}"
        assert a != b
    jobs = [("control", src)] + [(f"m{i:02d}", src.replace(a, b, 1)) for i, (a, b) in enumerate(MUTANTS.values())]
    workers = max(1, min(8, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        rcs = list(ex.map(lambda job: _run_copy(str(tmp_path / job[0]), job[1]), jobs))
    # the unmodified copy passes the suites, so the failures below are the planted mistakes'
    assert rcs[0] == 0, "the pin suites fail on an unmodified copy of the oracle"
    survived = [name for name, rc in zip(MUTANTS, rcs[1:]) if rc == 0]
    assert not survived, f"planted mistakes no pin caught: {survived}"


# The Compressor oracle (numpy): mistakes planted in a copy of its source, which
# is loaded as a module of its own; the pins of tests/test_oracle_compressor.py
# run against it in this process.
COMPRESSOR_MUTANTS = {
    "softmax over channels instead of rows": (
        "return e / e.sum(axis=1, keepdims=True)", "return e / e.sum(axis=2, keepdims=True)"),
    "softmax not normalised": ("return e / e.sum(axis=1, keepdims=True)", "return e"),
    "Ape dropped": ("+ np.asarray(ape, dtype=np.float64)[None, :, :]",
                    "+ 0.0 * np.asarray(ape, dtype=np.float64)[None, :, :]"),
    "Ape rows reversed": ("+ np.asarray(ape, dtype=np.float64)[None, :, :]",
                          "+ np.asarray(ape, dtype=np.float64)[None, ::-1, :]"),
    "scores weight the scores, not kv_state": ("sh = p * kv.reshape(T // ratio, ratio, D)",
                                               "sh = p * score.reshape(T // ratio, ratio, D)"),
    "weights swapped between kv and gate": (
        "return X @ bf16_to_f64(w_kv).T, X @ bf16_to_f64(w_gate).T",
        "return X @ bf16_to_f64(w_gate).T, X @ bf16_to_f64(w_kv).T"),
    "group sum divided by the group size": ("return np.ones(ratio) @ sh", "return np.ones(ratio) @ sh / ratio"),
    "groups offset by one row": ("s = score.reshape(T // ratio, ratio, D)",
                                 "s = np.roll(score, 1, axis=0).reshape(T // ratio, ratio, D)"),
    "bf16 decoded with the wrong shift": ("(b.astype(np.uint32) << 16)", "(b.astype(np.uint32) << 15)"),
    "stability shift taken per row (over channels)": ("s = s - s.max(axis=1, keepdims=True)",
                                                      "s = s - s.max(axis=2, keepdims=True)"),
    "C4A: b rows from the previous group": ("nxt = x[4 * i:4 * i + 4], x[4 * i + 4:4 * i + 8]",
                                            "nxt = x[4 * i:4 * i + 4], x[max(4 * i - 4, 0):4 * i]"),
    "C4A: a and b weights swapped": ("a_kv, b_kv = np.asarray(w_kv)[:D], np.asarray(w_kv)[D:]",
                                     "b_kv, a_kv = np.asarray(w_kv)[:D], np.asarray(w_kv)[D:]"),
    "C4A: Ape's a and b columns swapped": ("np.vstack([score_a + ape[:, :D], score_b + ape[:len(nxt), D:]])",
                                           "np.vstack([score_a + ape[:, D:], score_b + ape[:len(nxt), :D]])"),
    "C4A: last group padded with zero rows": (
        "own, nxt = x[4 * i:4 * i + 4], x[4 * i + 4:4 * i + 8]",
        "own, nxt = x[4 * i:4 * i + 4], np.vstack([x[4 * i + 4:4 * i + 8], "
        "np.zeros((4 - len(x[4 * i + 4:4 * i + 8]), x.shape[1]), x.dtype)])"),
    "C4A: softmax over channels": ("p = e / e.sum(axis=0, keepdims=True)", "p = e / e.sum(axis=1, keepdims=True)"),
    "C4A: gate weights of a used for b": ("a_gate, b_gate = np.asarray(w_gate)[:D], np.asarray(w_gate)[D:]",
                                          "a_gate, b_gate = np.asarray(w_gate)[:D], np.asarray(w_gate)[:D]"),
}


def test_every_planted_compressor_mistake_is_caught(tmp_path):
    import importlib.util
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import test_oracle_compressor as P
    src = open(os.path.join(ROOT, "oracle", "compressor.py")).read()

    def load(text, name):
        path = tmp_path / f"{name}.py"
        path.write_text(text)
        spec = importlib.util.spec_from_file_location(name, path)
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        return mod

    def caught(mod):
        for pin in P.PINS:
            try:
                pin(mod)
            except Exception:
                return True
        return False

    assert not caught(load(src, "control")), "the pins fail on an unmodified copy of the oracle"
    survived = []
    for i, (name, (a, b)) in enumerate(COMPRESSOR_MUTANTS.items()):
        assert a in src, f"mutant site not found: {name}"
        if not caught(load(src.replace(a, b, 1), f"mutant{i:02d}")):
            survived.append(name)
    assert not survived, f"planted mistakes no pin caught: {survived}"
