"""The pins have teeth: each plausible mistake planted in a copy of the oracle
source makes at least one pin test fail.

Every mutant below is one textual change to ``oracle/fp8_oracle.c`` of the kind
the pins are meant to catch: a wrong rounding rule, a dropped clamp, a swapped
index or operand, an off-by-one.  The copy is compiled with the oracle's own
flags, loaded through ``ORACLE_LIB_PATH``, and the pin files that cover the
changed function are run against it; the test passes only if they fail.  A
control build of the unchanged source must pass the same files, so a failure
here cannot come from the harness.  The GPU path is not involved.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fp8_oracle.c")
FORMAT, SCALING, MX, GEMM = ("tests/test_oracle_format.py", "tests/test_oracle_scaling.py",
                             "tests/test_oracle_mx.py", "tests/test_oracle_gemm.py")

# (name, exact text in the source, replacement, pin files expected to catch it)
MUTANTS = [
    ("ties away instead of to even", "else c = (lo % 2 == 0) ? lo : hi;", "else c = hi;", [FORMAT]),
    ("overflow to NaN instead of saturating", "if (a >= val[top]) return sign | top;",
     "if (a > val[top]) return sign | 0x7F;", [FORMAT]),
    ("E5M2 bias 16", "static const int EXP_BIAS[2] = {7, 15};", "static const int EXP_BIAS[2] = {7, 16};",
     [FORMAT]),
    ("bf16 rounding ties away", "if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;",
     "if (lower >= 0x8000u) upper += 1;", [FORMAT, SCALING]),
    ("amax without the absolute value", "const float a = fabsf(load_elem(x, dtype, i));",
     "const float a = load_elem(x, dtype, i);", [SCALING]),
    ("no eps clamp on the scale",
     "const float m = (amax > AMAX_EPS) ? amax : AMAX_EPS;\n    return (float)(MAX_FINITE[fmt] / (double)m);",
     "const float m = amax;\n    return (float)(MAX_FINITE[fmt] / (double)m);", [SCALING]),
    ("block amax from its first row only",
     "for (int64_t r = r0; r < r1; ++r) {\n                const float m = amax_of",
     "for (int64_t r = r0; r < r0 + 1; ++r) {\n                const float m = amax_of", [SCALING]),
    ("dequant multiplies by the scale", "const float out = v / s;", "const float out = v * s;", [SCALING]),
    ("dequant scale index transposed", "scales[(r / br) * nbc + (c / bc)]", "scales[(c / bc) * nbc + (r / br)]",
     [SCALING, MX]),
    ("history max leaves out the new amax", "    history[pos] = amax;\n    pos = (pos + 1) % window;\n    if (count < window) count += 1;\n    if (count == window) {\n        float m = 0.0f;\n        for (int i = 0; i < window; ++i)\n            if (history[i] > m) m = history[i];\n        *scale = orc_scale_from_amax(m, fmt);",
     "    if (count < window) count += 1;\n    if (count == window) {\n        float m = 0.0f;\n        for (int i = 0; i < window; ++i)\n            if (history[i] > m) m = history[i];\n        *scale = orc_scale_from_amax(m, fmt);\n    }\n    history[pos] = amax;\n    pos = (pos + 1) % window;\n    if (0) {",
     [SCALING]),
    ("margin multiplies the scale", "const float d = (float)((double)m * (double)margin);",
     "const float d = (float)((double)m / (double)margin);", [SCALING]),
    ("EMA weights swapped", "const float beta = (float)(1.0 - (double)alpha);", "const float beta = alpha;",
     [SCALING]),
    ("EMA as m + alpha * (amax - m), each step rounded",
     "history[0] = (float)((double)a_part + (double)m_part);",
     "history[0] = (float)((double)history[0] + (double)(float)((double)alpha * (double)(float)((double)amax - "
     "(double)history[0]))); (void)a_part; (void)m_part;",
     [SCALING]),
    ("EMA sum fused with the amax product (one rounding)",
     "history[0] = (float)((double)a_part + (double)m_part);",
     "history[0] = (float)fma((double)alpha, (double)amax, (double)m_part); (void)a_part;",
     [SCALING]),
    ("transposed copy not transposed", "qt[c * rows + r] = q[r * cols + c];", "qt[r * cols + c] = q[r * cols + c];",
     [SCALING]),
    ("MX exponent off by one", "int k = emax_elem - (e - 1);", "int k = emax_elem - e;", [MX]),
    ("MX byte stores k, not -k", "(uint8_t)(127 - k)", "(uint8_t)(127 + k)", [MX]),
    ("GEMM weight scale index transposed", "(double)sb[(n / b_block_rows) * nkc + kc]",
     "(double)sb[kc * ((N + b_block_rows - 1) / b_block_rows) + (n / b_block_rows)]", [GEMM]),
    ("GEMM ignores B's block height (1x128 B read as 128x128)",
     "acc += p / ((double)sa[m * nkc + kc] * (double)sb[(n / b_block_rows) * nkc + kc]);",
     "acc += p / ((double)sa[m * nkc + kc] * (double)sb[(n / 128) * nkc + kc]);", [GEMM]),
    ("GEMM drops the activation scale",
     "acc += p / ((double)sa[m * nkc + kc] * (double)sb[(n / b_block_rows) * nkc + kc]);",
     "acc += p / (double)sb[(n / b_block_rows) * nkc + kc];", [GEMM]),
]

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def _build(source: str, path: str):
    c_path = path[:-3] + ".c"
    with open(c_path, "w") as f:
        f.write(source)
    subprocess.run(["gcc", *CFLAGS, "-o", path, c_path, "-lm"], check=True, capture_output=True)


def _run_pins(lib_path: str, files) -> int:
    env = dict(os.environ, ORACLE_LIB_PATH=lib_path)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "not gpu", "-p", "no:cacheprovider", *files]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, timeout=600).returncode


def test_every_mutant_is_caught(tmp_path):
    source = open(SRC).read()
    jobs = []
    for i, (name, old, new, files) in enumerate(MUTANTS):
        assert source.count(old) >= 1, f"mutant '{name}': text not found in the oracle source"
        mutated = source.replace(old, new, 1)
        path = str(tmp_path / f"mutant{i}.so")
        _build(mutated, path)
        jobs.append((name, path, files))
    control = str(tmp_path / "control.so")
    _build(source, control)
    all_files = sorted({f for _, _, _, fs in MUTANTS for f in fs})
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as pool:
        control_rc = pool.submit(_run_pins, control, all_files)
        rcs = {name: pool.submit(_run_pins, path, files) for name, path, files in jobs}
        assert control_rc.result() == 0, "the unchanged oracle must pass its pins in this harness"
        missed = [name for name, fut in rcs.items() if fut.result() == 0]
    assert not missed, f"pins did not catch: {missed}"
