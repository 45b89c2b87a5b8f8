"""The dequantize kernels divide by the scale through a correctly rounded
reciprocal and one fma correction.  tests/c/recip_division_exhaustive.c
checks that scheme against the IEEE quotient for every mantissa of the scale
(2^23) and every FP8 significand (8): all 67,108,864 cases must match."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_reciprocal_fma_division_exact_for_every_scale_mantissa(tmp_path):
    exe = tmp_path / "recip_division_exhaustive"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                    os.path.join(HERE, "c", "recip_division_exhaustive.c"), "-lm"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout
    assert "checked 67108864 cases, 0 mismatches" in out.stdout
