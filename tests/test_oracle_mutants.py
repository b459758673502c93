"""The pins must catch plausible mistakes in the oracle.

Each case copies the oracle's C source, plants one mistake (a flipped sign, a
dropped term, a wrong exponent, a wrong index or tie rule ...), builds the
mutant on the CPU and runs the pin suite against it in a subprocess.  Every
mutant must make the pin suite fail.  The real oracle is never modified.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hqq_oracle.c")

# (name, text in the source, replacement, expected number of occurrences; a
# line the fp32 solver shares with the half-precision variant is mutated in both)
MUTANTS = [
    ("z-update-sign", "return (float)((sq - sws) / (double)g);", "return (float)((sq + sws) / (double)g);", 1),
    ("z-update-drops-We", "float ws = (w[i] - we) * s;", "float ws = (w[i] - 0.0f * we) * s;", 1),
    ("shrink-exponent", "powf(a, p - 1.0f) / beta", "powf(a, p) / beta", 1),
    ("shrink-beta-inverted", "powf(a, p - 1.0f) / beta", "powf(a, p - 1.0f) * beta", 1),
    ("residual-sign", "float r = v - qi;", "float r = qi - v + 2.0f * (qi - v) * (qi > 0.0f);", 1),
    ("residual-unscaled", "d[i] = r / s;", "d[i] = r;", 1),
    ("l1-instead-of-lp", "acc += (double)powf(fabsf(d[i]), p);", "acc += (double)fabsf(d[i]);", 1),
    ("tie-continues", "        double e = evaluate(w, g, L, s, z, p, q, d) / (double)g;\n        if (e < best) {",
     "        double e = evaluate(w, g, L, s, z, p, q, d) / (double)g;\n        if (e <= best) {", 1),
    ("keeps-last-z", "    res->zbest = zbest;", "    res->zbest = z;", 2),
    ("beta-divides", "beta = beta * kappa;", "beta = beta / kappa;", 4),
    ("z0-from-max", "*z_out = -mn * s;", "*z_out = -mx * s;", 1),
    ("scale-uses-2^b", "s = (float)L / (mx - mn);", "s = (float)(L + 1) / (mx - mn);", 2),
    ("floor-instead-of-round", "float q = nearbyintf(v);", "float q = floorf(v);", 2),
    ("tensor-stop-first-group", "double e = G ? total / (double)(G * g) : 0.0;",
     "double e = G ? gerr[0] / (double)g : 0.0;", 1),
    ("zero8-scale", "sz = 255.0f / (zmx - zmn);", "sz = 254.0f / (zmx - zmn);", 2),
    ("dequant-sign", "float v = (q - z) * sc;", "float v = (q + z) * sc;", 1),
    ("scale8-zc-sign", "const float zc = -mn * sc;", "const float zc = mn * sc;", 1),
    ("scale8-254-levels", "? 255.0f / (mx - mn) : 1.0f;", "? 254.0f / (mx - mn) : 1.0f;", 1),
    ("scale8-truncates", "float c = nearbyintf(from_f16(scale[i]) * sc + zc);",
     "float c = truncf(from_f16(scale[i]) * sc + zc);", 1),
    ("scale8-one-run", "const int64_t k1 = k0 + scale_group < G ? k0 + scale_group : G;",
     "const int64_t k1 = G;", 1),
    ("dequant-s8-first-run-meta", "const float *m = scale_meta + 2 * (j / scale_group);",
     "const float *m = scale_meta;", 1),
    ("gemv-drops-zero", "const float w = (q - z) * from_f16(scale[j]);", "const float w = q * from_f16(scale[j]);",
     1),
    ("gemv-group-index", "const int64_t j = (r * cols + c) / g;", "const int64_t j = (r * cols + c) / (2 * g);", 1),
    ("gemv-skips-last-column", "        for (int64_t c = 0; c < cols; ++c) {\n            const int64_t j = (r * cols + c) / g;",
     "        for (int64_t c = 0; c < cols - 1; ++c) {\n            const int64_t j = (r * cols + c) / g;", 1),
    ("gemm-no-16-bit-rounding",
     "const double w16 = x_dtype == ORACLE_BF16 ? (double)from_bf16(to_bf16(wr)) : (double)from_f16(to_f16(wr));",
     "const double w16 = (double)wr;", 1),
    ("gemm-rounds-to-the-other-type",
     "const double w16 = x_dtype == ORACLE_BF16 ? (double)from_bf16(to_bf16(wr)) : (double)from_f16(to_f16(wr));",
     "const double w16 = x_dtype != ORACLE_BF16 ? (double)from_bf16(to_bf16(wr)) : (double)from_f16(to_f16(wr));", 1),
    ("gemm-drops-zero", "const float wr = (q - z) * from_f16(scale[grp]);", "const float wr = q * from_f16(scale[grp]);",
     1),
    ("gemm-signed-abs-sum", "yabs[b * rows + r] += fabs(p);", "yabs[b * rows + r] += p;", 1),
    ("groups-axis0-index", "int64_t j = group_ids[k];\n            for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));",
     "int64_t j = group_ids[k];\n            for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, 1));", 1),
    ("groups-levels-reversed", "levels[k * g + i] = (uint8_t)quantize_elem(w[i], res.s, res.zbest, L);",
     "levels[k * g + (g - 1 - i)] = (uint8_t)quantize_elem(w[i], res.s, res.zbest, L);", 1),
    ("half-ws-unrounded", "        float ws = h16((double)w[i] * (double)s);\n        float v = h16((double)ws + (double)z);",
     "        float ws = (float)((double)w[i] * (double)s);\n        float v = h16((double)ws + (double)z);", 1),
    ("half-z-unrounded", "    return h16((sq - sws) / (double)g);", "    return (float)((sq - sws) / (double)g);", 1),
    ("half-s-unrounded", "    s = h16(s);\n", "", 1),
    ("half-tie-continues", "        double e = evaluate_half(w, g, L, s, z, p, q, r);\n        if (e < best) {",
     "        double e = evaluate_half(w, g, L, s, z, p, q, r);\n        if (e <= best) {", 1),
    ("half-codes-in-fp32", "    float ws = h16((double)w * (double)s);", "    float ws = w * s;", 1),
    ("pack-msb-first", "unsigned v = level << off; /* at most 8 + 7 bits */",
     "unsigned v = (off + b <= 8 ? level << (8 - b - off) : level << off);", 1),
]


def _run_mutant(tmp, name, old, new, count):
    src = open(SRC).read()
    assert src.count(old) == count, f"{name}: pattern found {src.count(old)} times"
    csrc = os.path.join(tmp, f"{name}.c")
    lib = os.path.join(tmp, f"lib{name}.so")
    open(csrc, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-std=gnu11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-w",
                    csrc, "-o", lib, "-lm"], check=True)
    env = dict(os.environ, HQQ_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-400:]


def test_every_mutant_is_caught():
    tmp = tempfile.mkdtemp(prefix="hqq_mutants_")
    try:
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda m: _run_mutant(tmp, *m), MUTANTS))
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by the pins: {survivors}"
    for n, rc, out in results:
        assert rc == 1, f"{n}: pin run ended with code {rc} (expected test failures, not an error): {out}"
