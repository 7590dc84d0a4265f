"""The quantize kernels decide codes from RN(x / s) without dividing. Their fast paths
use the reciprocal correction q0 = RN(x rn), rem = fma(-q0, s, x), RN(q0 + rem rn) with
rn = RN(1/s) (Markstein's theorem). This test checks that identity against IEEE
division on the CPU, on the domain the kernels use it for: every bf16 x against
scales RN(amax / Q) derived from bf16 amax values (a sample of them; the full sweep
was run when the kernels were written), random fp32 pairs, and the scale computation
itself (fp32 dividends over each format's Qmax, with the compile-time RN(1/Qmax)).
"""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "native", "markstein_check.c")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("mk") / "markstein_check")
    # hardware FMA, no contraction: fmaf is the fused operation, x * rn stays rounded
    r = subprocess.run([cc, "-O2", "-mfma", "-ffp-contract=off", "-o", exe, SRC, "-lm"],
                       capture_output=True, text=True)
    if r.returncode != 0:
        pytest.skip("checker did not build: " + r.stderr[:200])
    return exe


def test_reciprocal_correction_is_the_ieee_quotient(checker):
    r = subprocess.run([checker, "3", "40000", "5"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches 0" in r.stdout
