"""Mutation tests of the oracle's pins: copies of oracle/ep_oracle.c with one
plausible mistake each (a transposed index, a dropped term, a wrong rounding
rule, a flipped sign or bias) are compiled and run against the pins of
tests/test_oracle_pins.py that bear on that code; every copy must fail them,
and the unmutated source must pass the same selection.  Host only."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ep_oracle.c")
sys.path.insert(0, ROOT)
from oracle.build import CFLAGS  # noqa: E402

# name: ([(text in ep_oracle.c, replacement), ...], pins that must catch it)
MUTANTS = {
    "bf16 expert maps all use expert 0's weights": (
        [("const uint16_t *wr = w + ((int64_t)e * Nout + j) * H;",
          "const uint16_t *wr = w + ((int64_t)0 * Nout + j) * H;")],
        "expert_gemm_equals or expert_gemm_identity"),
    "MXFP4 maps take a row scale per 32 packed bytes": (
        [("orc_e2m1_at(xc + r * D, h) * orc_e8m0_value(xs[r * S + h / 32])",
          "orc_e2m1_at(xc + r * D, h) * orc_e8m0_value(xs[r * S + h / 64])")],
        "expert_gemm_mxfp4"),
    "MX weight scale read from the expert's first row": (
        [("orc_e4m3_decode(wc[wrow * H + h]) * orc_e8m0_value(ws[wrow * S + h / 32])",
          "orc_e4m3_decode(wc[wrow * H + h]) * orc_e8m0_value(ws[(int64_t)e * Nout * S + h / 32])")],
        "expert_gemm_mx"),
    "MX scale bias off by one": (
        [("ldexp(1.0, (int)b - 127)", "ldexp(1.0, (int)b - 126)")], "expert_gemm_mx"),
    "layout ties broken by descending k": (
        [("            for (int k = 0; k < K; k++) {\n                int64_t e = idx[n * K + k];\n"
          "                if (e < -1 || e >= E) st |= ORC_ST_BAD_INDEX;\n"
          "                if (e < 0 || e >= E) { token_slot[n * K + k] = -1; continue; }",
          "            for (int k = K - 1; k >= 0; k--) {\n                int64_t e = idx[n * K + k];\n"
          "                if (e < -1 || e >= E) st |= ORC_ST_BAD_INDEX;\n"
          "                if (e < 0 || e >= E) { token_slot[n * K + k] = -1; continue; }")],
        "layout"),
    "expert to rank by modulo": (
        [("is_token_in_rank[n * R + e / L] = 1;", "is_token_in_rank[n * R + e % R] = 1;")],
        "layout"),
    "packed rows not aligned": (
        [("off += (recv_count[e] + align - 1) / align * align;", "off += recv_count[e];")],
        "layout or dispatch"),
    "src_info rank and token transposed": (
        [("src_info[row] = r * M + t;", "src_info[row] = t * R + r;")], "dispatch"),
    "combine weight index without k": (
        [("acc = fmaf(w[k], orc_bf16_to_f32(yrows[k][h]), acc);",
          "acc = fmaf(w[0], orc_bf16_to_f32(yrows[k][h]), acc);")], "combine"),
    "small-float mantissa truncated": (
        [("float q = rintf(frac);", "float q = truncf(frac);")], "encoder"),
    "e8m0 exponent rounded down": (
        [("int X = (m == 0.5f) ? e - 1 : e;", "int X = e - 1;")], "mx_exponent or mx_bounds"),
    "int8 scale inverted": (
        [("s = 127.0f / amax;", "s = amax / 127.0f;")], "int8"),
    "mxfp4 nibbles swapped": (
        [("if (i % 2 == 0) data[byte] = c;", "if (i % 2 == 0) data[byte] = (uint8_t)(c << 4);"),
         ("data[byte] = (uint8_t)(data[byte] | (c << 4));", "data[byte] = (uint8_t)(data[byte] | c);")],
        "mxfp4"),
    "mxfp8 dequant bias off by one": (
        [("            v = orc_e4m3_decode(data[h]);\n            s = ldexpf(1.0f, (int)scale[h / 32] - 127);",
          "            v = orc_e4m3_decode(data[h]);\n            s = ldexpf(1.0f, (int)scale[h / 32] - 126);")],
        "dequant"),
    "backward ignores the unweighted flag": (  # both checks of the flag, else no change
        [("float w = unweighted ? 1.0f : topk_weights[n * K + k];",
          "float w = topk_weights[n * K + k];"),
         ("p[h] = unweighted ? gv : w * gv;", "p[h] = w * gv;")], "backward"),
    "weight gradient reads the token's row of y": (
        [("(double)orc_bf16_to_f32(y[row * H + h])", "(double)orc_bf16_to_f32(y[n * H + h])")],
        "wgrad"),
    "ue8m0 byte bias off by one": (
        [("            } else {\n                scale[b] = (uint8_t)(X + 127);",
          "            } else {\n                scale[b] = (uint8_t)(X + 128);")], "ue8m0"),
    "NaN wins the block maximum": (
        [("        if (v > a) a = v;", "        if (!(v <= a)) a = v;")], "nan"),
    "SwiGLU gate and up halves swapped": (
        [("const double g = (double)h[j], u = (double)h[I + j];",
          "const double g = (double)h[I + j], u = (double)h[j];")], "ffn"),
    "silu with exp of +a": (
        [("z[j] = (float)(g / (1.0 + exp(-g)) * u);", "z[j] = (float)(g / (1.0 + exp(g)) * u);")],
        "ffn"),
    "GMM2 reads the intermediate scale of the first block only": (
        [("double zv = (double)orc_e4m3_decode(zc[r * I + k]) * orc_e8m0_value(zs[r * SI + k / 32]);",
          "double zv = (double)orc_e4m3_decode(zc[r * I + k]) * orc_e8m0_value(zs[r * SI]);")],
        "ffn"),
    "GMM1 gate rows of expert 0 for every expert": (
        [("const int64_t wrow = (int64_t)e * N1 + j;", "const int64_t wrow = (int64_t)0 * N1 + j;")],
        "ffn"),
    "e4m3 NaN code decodes to 480": (
        [("if (e == 15 && m == 7) return NAN;", "if (e == 15 && m == 7) return 480.0f;")],
        "decoders"),
}


def _build(src_text, tmp):
    c = os.path.join(tmp, "ep_oracle.c")
    lib = os.path.join(tmp, "libep_oracle.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", *CFLAGS, c, "-o", lib, "-lm"])
    return lib


def _pins(lib, select):
    env = dict(os.environ, EP_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        "-q", "-x", "-p", "no:cacheprovider", "-k", select],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def _run_mutant(name):
    edits, select = MUTANTS[name]
    text = open(SRC).read()
    for old, new in edits:
        assert text.count(old) == 1, f"mutation site of '{name}' not unique: {old[:60]!r}"
        text = text.replace(old, new)
    with tempfile.TemporaryDirectory() as tmp:
        return _pins(_build(text, tmp), select)


def test_pins_catch_every_planted_mistake():
    from concurrent.futures import ThreadPoolExecutor
    names = sorted(MUTANTS)
    with ThreadPoolExecutor(max(1, min(len(names), os.cpu_count() or 1))) as pool:
        results = dict(zip(names, pool.map(_run_mutant, names)))
    missed = {n: out for n, (rc, out) in results.items() if rc != 1}
    assert not missed, "mutants not caught (or pins did not run):\n" + "\n".join(
        f"- {n} (-k '{MUTANTS[n][1]}'):\n{out}" for n, out in missed.items())


def test_unmutated_oracle_passes_every_selection():
    select = " or ".join(f"({s})" for s in sorted({s for _, s in MUTANTS.values()}))
    with tempfile.TemporaryDirectory() as tmp:
        rc, out = _pins(_build(open(SRC).read(), tmp), select)
    assert rc == 0, out
