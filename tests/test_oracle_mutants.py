"""The oracle's pins reject plausible mistakes.

Each case below plants one mistake in a scratch copy of ``oracle/oracle.c``. The mistakes cover:
- a dropped term, a wrong sign, index or bias;
- a transposed operand, a swapped gate/up half, a wrong rounding mode;
- a wrong scale rule, padding or tie rule.

The case then runs the CPU pin tests that should reject it, and the run must fail. A case whose pins
pass would be a mistake in the oracle that nothing catches. The copies live under ``_build/`` (not
tracked) and are removed afterwards. Nothing here touches the CUDA path. The unmutated copy must pass
every pin file used, so that a failure can only come from the planted mistake.

Each case costs a Python process (about 7 s, mostly the torch import). The default run therefore
plants the representative subset ``DEFAULT``, at least one case per pin file. ``ORACLE_MUTANTS=all``
plants every case.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRATCH = os.path.join(ROOT, "_build", "oracle_mutants")

IM = "test_oracle_intermediate.py"
F, P, R, K, Q, X = ("test_oracle_formats.py", "test_oracle_planner.py", "test_oracle_router.py",
                    "test_oracle_pack.py", "test_oracle_fp4.py", "test_oracle_ffn.py")

_BF16_TAIL = ("for (int h = 0; h < K; ++h) out[(int64_t)t * K + h] = orc_double_to_bf16(acc[h]);\n"
              "      if (out_f64)\n        for (int h = 0; h < K; ++h) out_f64[(int64_t)t * K + h] = acc[h];\n"
              "    }\n    free(")

# (name, pin file that must reject it, text in oracle.c (exactly once), replacement)
MUTANTS = [
    # scalar formats
    ("bf16 smallest normal binade", F, "int qe = e < -125 ? -125 : e;", "int qe = e < -126 ? -126 : e;"),
    ("bf16 seven significant bits", X, "ldexp(1.0, qe - 8);", "ldexp(1.0, qe - 7);"),
    ("bf16 ties away from zero", F, "double q = nearbyint(x / quantum) * quantum;",
     "double q = round(x / quantum) * quantum;"),
    ("e4m3 subnormal step", F, "ldexp((double)m, -9) :", "ldexp((double)m, -10) :"),
    ("e4m3 exponent bias", X, "ldexp(1.0 + m / 8.0, ex - 7)", "ldexp(1.0 + m / 8.0, ex - 8)"),
    ("e4m3 NaN codes", X, "if (ex == 0xF && m == 7) return NAN;", "if (ex == 0xF && m >= 6) return NAN;"),
    ("e4m3 smallest normal binade", F, "int qe = e < -5 ? -5 : e;", "int qe = e < -6 ? -6 : e;"),
    ("e4m3 saturation value", X, "if (q > 448.0) q = 448.0;", "if (q > 448.0) q = 416.0;"),
    ("e4m3 ties away from zero", F, "double q = nearbyint(a / quantum) * quantum;",
     "double q = round(a / quantum) * quantum;"),
    ("e4m3 subnormal encode", F, "int m = (int)nearbyint(q / ldexp(1.0, -9));",
     "int m = (int)nearbyint(q / ldexp(1.0, -8));"),
    ("e2m1 subnormal value", Q, "ex == 0 ? 0.5 * m :", "ex == 0 ? 1.0 * m :"),
    ("e2m1 exponent bias", Q, "ldexp(1.0 + 0.5 * m, ex - 1)", "ldexp(1.0 + 0.5 * m, ex - 2)"),
    ("e2m1 sign bit", Q, "int s = (code >> 3) & 1,", "int s = (code >> 2) & 1,"),
    ("e8m0 bias", X, "return ldexp(1.0, (int)code - 127);", "return ldexp(1.0, (int)code - 128);"),
    # OCP MX scale rule
    ("mx scale emax 7", X, "int shared = (e - 1) - 8;", "int shared = (e - 1) - 7;"),
    ("mx scale from ceil(log2)", X, "int shared = (e - 1) - 8;", "int shared = e - 8;"),
    ("mx all-zero block byte", F, "if (!(amax > 0.0f)) return 0;", "if (!(amax > 0.0f)) return 127;"),
    ("mx scale clamp", F, "if (shared < -127) shared = -127;", "if (shared < -126) shared = -126;"),
    ("mx amax over 31 of 32", X, "for (int i = 0; i < 32; ++i) {\n      float a = fabsf(",
     "for (int i = 0; i < 31; ++i) {\n      float a = fabsf("),
    # planner
    ("planner pads full segments", P, "int64_t padded = (count[e] + block_m - 1) / block_m * block_m;",
     "int64_t padded = (count[e] / block_m + 1) * block_m;"),
    ("planner no padding", P, "int64_t padded = (count[e] + block_m - 1) / block_m * block_m;",
     "int64_t padded = count[e];"),
    ("planner ntpp unpadded", P, "*num_tokens_post_padded = (int32_t)ntpp;",
     "*num_tokens_post_padded = (int32_t)R;"),
    ("planner segment descending", P, "sorted_token_ids[off[e] + cursor[e]] = (int32_t)i;",
     "sorted_token_ids[off[e] + count[e] - 1 - cursor[e]] = (int32_t)i;"),
    ("planner pad value 0", P, "for (int64_t p = 0; p < capacity; ++p) sorted_token_ids[p] = -1;",
     "for (int64_t p = 0; p < capacity; ++p) sorted_token_ids[p] = 0;"),
    ("planner token instead of route id", P, "sorted_token_ids[off[e] + cursor[e]] = (int32_t)i;",
     "sorted_token_ids[off[e] + cursor[e]] = (int32_t)(i / top_k);"),
    ("expert_ids tail 0", P, "for (int64_t b = 0; b < nblk_cap; ++b) expert_ids[b] = -1;",
     "for (int64_t b = 0; b < nblk_cap; ++b) expert_ids[b] = 0;"),
    ("expert_ids shifted", P, "expert_ids[p / block_m] = e;", "expert_ids[p / block_m] = e + 1 < E ? e + 1 : e;"),
    # router and shared experts
    ("router ties to the higher index", R, "if (best < 0 || z[e] > z[best]) best = e;",
     "if (best < 0 || z[e] >= z[best]) best = e;"),
    ("router ignores the bias", R, "const float b = bias ? bias[e] : 0.0f;", "const float b = 0.0f;"),
    ("router score not fp32", R, "z[e] = logits[(int64_t)t * E + e] + b;",
     "z[e] = (float)((double)logits[(int64_t)t * E + e] + (double)b + 1e-9);"),
    ("router not renormalised", R, "for (int j = 0; j < top_k; ++j) w[j] /= sum;", "(void)sum;"),
    ("router weights without bias", R, "w[j] = exp((double)z[ids[j]] - zmax);",
     "w[j] = exp((double)logits[(int64_t)t * E + ids[j]] - zmax);"),
    ("router row stride", R, "int32_t* ids = topk_ids + (int64_t)t * kk;",
     "int32_t* ids = topk_ids + (int64_t)t * top_k;"),
    ("shared expert weight", R, "w[top_k + j] = 1.0;", "w[top_k + j] = 0.5;"),
    ("shared expert ids", R, "ids[top_k + j] = E + j;", "ids[top_k + j] = E - 1 - j;"),
    # blocked scale layout
    ("blocked tile inner transpose", K, "(r % 32) * 16 + (r / 32) * 4 + c;", "(r % 32) * 16 + c * 4 + r / 32;"),
    ("blocked tile order", K, "return (((int64_t)e * MT + mt) * KT + kt) * 512",
     "return (((int64_t)e * KT + kt) * MT + mt) * 512"),
    ("blocked pad bytes", K, "memset(out, 0, (size_t)orc_pack_scales_bytes(E, MN, KS));",
     "memset(out, 0x7F, (size_t)orc_pack_scales_bytes(E, MN, KS));"),
    # FFN
    ("silu sign", X, "return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    ("silu is the sigmoid", X, "return g / (1.0 + exp(-g));", "return 1.0 / (1.0 + exp(-g));"),
    ("bf16 gate and up swapped", X, "orc_double_to_bf16(silu(H[i]) * H[I + i])",
     "orc_double_to_bf16(silu(H[I + i]) * H[i])"),
    ("bf16 intermediate not rounded", X,
     "a[i] = orc_bf16_to_double(orc_double_to_bf16(silu(H[i]) * H[I + i]));", "a[i] = silu(H[i]) * H[I + i];"),
    ("bf16 routing weight dropped", X,
     "const double wgt = (double)topk_weights[(int64_t)t * top_k + j];\n        for (int h = 0; h < K; ++h) {\n"
     "          double s = 0.0;\n          for (int i = 0; i < I; ++i) s +=",
     "const double wgt = 1.0;\n        for (int h = 0; h < K; ++h) {\n"
     "          double s = 0.0;\n          for (int i = 0; i < I; ++i) s +="),
    ("bf16 w1 transposed", X, "s += orc_bf16_to_double(W1[(int64_t)n * K + k])",
     "s += orc_bf16_to_double(W1[(int64_t)k * N + n])"),
    ("bf16 w2 transposed", X, "orc_bf16_to_double(W2[(int64_t)h * I + i])", "orc_bf16_to_double(W2[(int64_t)i * K + h])"),
    ("bf16 token list ignored", X,
     "const int t = tokens ? tokens[idx] : idx;\n      for (int h = 0; h < K; ++h) acc[h] = 0.0;",
     "const int t = idx;\n      for (int h = 0; h < K; ++h) acc[h] = 0.0;"),
    ("bf16 out rounded via fp32", X, _BF16_TAIL + "H);",
     _BF16_TAIL.replace("orc_double_to_bf16(acc[h])", "orc_double_to_bf16((float)acc[h])") + "H);"),
    ("mx gate and up swapped", X, "af[i] = (float)(silu(H[i]) * H[I + i]);", "af[i] = (float)(silu(H[I + i]) * H[i]);"),
    ("mx requant from a bf16 value", X, "af[i] = (float)(silu(H[i]) * H[I + i]);",
     "af[i] = (float)orc_bf16_to_double(orc_double_to_bf16(silu(H[i]) * H[I + i]));"),
    ("mx no requant", X, "a[i] = d->e4m3[aq[i]] * d->e8m0[as[i / 32]];", "a[i] = af[i];"),
    ("mx requant scale block", X, "a[i] = d->e4m3[aq[i]] * d->e8m0[as[i / 32]];",
     "a[i] = d->e4m3[aq[i]] * d->e8m0[as[(i / 32) ^ (IS > 1)]];"),
    ("mx x scale block", X, "x_scales[(int64_t)t * KS + k / 32]", "x_scales[(int64_t)t * KS + (k / 32 + 1) % KS]"),
    ("mx w1 scales transposed", X, "S1[(int64_t)n * KS + k / 32]", "S1[(int64_t)(k / 32) * N + n]"),
    ("mx w2 scale block", X, "S2[(int64_t)h * IS + i / 32]", "S2[(int64_t)h * IS + (i / 32 + 1) % IS]"),
    ("mx routing weight dropped", X,
     "const double wgt = (double)topk_weights[(int64_t)t * top_k + j];\n        for (int h = 0; h < K; ++h) {\n"
     "          double s = 0.0;\n          for (int i = 0; i < I; ++i)\n",
     "const double wgt = 1.0;\n        for (int h = 0; h < K; ++h) {\n"
     "          double s = 0.0;\n          for (int i = 0; i < I; ++i)\n"),
    ("mx last route dropped", X,
     "for (int j = 0; j < top_k; ++j) {\n        const int e = topk_ids[(int64_t)t * top_k + j];\n"
     "        if (e < 0 || e >= E) continue;\n        const uint8_t*",
     "for (int j = 0; j < top_k - (top_k > 1); ++j) {\n        const int e = topk_ids[(int64_t)t * top_k + j];\n"
     "        if (e < 0 || e >= E) continue;\n        const uint8_t*"),
    ("mx token list ignored", X,
     "const int t = tokens ? tokens[idx] : idx;\n      dequant_x(d, x, x_scales, t, K, xd);\n"
     "      for (int h = 0; h < K; ++h) acc[h] = 0.0;",
     "const int t = idx;\n      dequant_x(d, x, x_scales, t, K, xd);\n"
     "      for (int h = 0; h < K; ++h) acc[h] = 0.0;"),
    ("mx out rounded via fp32", X, _BF16_TAIL + "xd);",
     _BF16_TAIL.replace("orc_double_to_bf16(acc[h])", "orc_double_to_bf16((float)acc[h])") + "xd);"),
    ("fp4 nibble order", Q, "(idx & 1) ? (b >> 4) : (b & 0xF)", "(idx & 1) ? (b & 0xF) : (b >> 4)"),
    ("mx decode table off by one", X, "d->e4m3[c] = orc_e4m3_to_double((uint8_t)c);",
     "d->e4m3[c] = orc_e4m3_to_double((uint8_t)(c ^ (c == 0x38)));"),
    ("mx intermediate rows of the wrong route", IM, "float* row = act + ((int64_t)idx * top_k + j) * I;",
     "float* row = act + ((int64_t)idx * top_k + (top_k - 1 - j)) * I;"),
    ("mx intermediate of an invalid route left unwritten", IM,
     "for (int i = 0; i < I; ++i) row[i] = 0.0f;\n          continue;", "continue;"),
]


DEFAULT = ["bf16 ties away from zero", "e4m3 saturation value", "mx scale emax 7", "planner segment descending",
           "planner pads full segments", "router ties to the higher index", "shared expert weight",
           "blocked tile inner transpose", "bf16 gate and up swapped", "bf16 out rounded via fp32",
           "mx requant scale block", "fp4 nibble order", "mx intermediate rows of the wrong route"]


def _tree(name: str) -> str:
    d = os.path.join(SCRATCH, name)
    if os.path.isdir(d):
        shutil.rmtree(d)
    os.makedirs(d)
    for sub in ("oracle", "tests", "workloads"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__", "test_gpu_*", "test_oracle_mutants.py"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    return d


def _pins(tree: str, pin_file: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                           os.path.join("tests", pin_file)], cwd=tree, env=env, capture_output=True, text=True,
                          timeout=600)


def _run_mutant(i: int):
    name, pin_file, old, new = MUTANTS[i]
    tree = _tree(f"m{i:02d}")
    try:
        src_path = os.path.join(tree, "oracle", "oracle.c")
        src = open(src_path).read()
        if src.count(old) != 1:
            return name, f"pattern found {src.count(old)} times"
        open(src_path, "w").write(src.replace(old, new))
        r = _pins(tree, pin_file)
        # 0 = the pins passed (mistake not caught); 2-5 = pytest could not run the pins at all
        if r.returncode == 0:
            return name, f"not rejected by {pin_file}"
        if r.returncode in (2, 3, 4, 5):
            return name, f"pins did not run (pytest status {r.returncode}): {r.stdout[-300:]}"
        return name, None
    finally:
        shutil.rmtree(tree, ignore_errors=True)


def _baseline(pin_file: str):
    tree = _tree("unmutated_" + pin_file[:-3])
    try:
        r = _pins(tree, pin_file)
        return pin_file, None if r.returncode == 0 else r.stdout[-2000:]
    finally:
        shutil.rmtree(tree, ignore_errors=True)


def test_planted_mistakes_are_rejected():
    names = [m[0] for m in MUTANTS]
    assert len(set(names)) == len(names) and set(DEFAULT) <= set(names)
    chosen = range(len(MUTANTS)) if os.environ.get("ORACLE_MUTANTS") == "all" else \
        [names.index(n) for n in DEFAULT]
    pin_files = sorted({MUTANTS[i][1] for i in chosen})
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ThreadPoolExecutor(workers) as ex:
        base = list(ex.map(_baseline, pin_files))
        bad = [f"unmutated oracle fails {f}:\n{out}" for f, out in base if out]
        assert not bad, "\n".join(bad)
        results = list(ex.map(_run_mutant, chosen))
    shutil.rmtree(SCRATCH, ignore_errors=True)
    missed = [f"{n}: {why}" for n, why in results if why]
    assert not missed, "\n".join(missed)


@pytest.mark.parametrize("i", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_mutation_text_is_present(i):
    """Every planted change still applies to the current oracle (the oracle's text changed otherwise)."""
    name, _, old, new = MUTANTS[i]
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert src.count(old) == 1 and old != new
