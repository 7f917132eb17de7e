"""The cache writer divides by a row/group scale through Markstein's correction of
x * RN(1/scale) (IBM J. Res. Develop. 34(1), 1990) instead of a division per
element.  This CPU test checks the property the bit-exact codes rely on, with a
small C program of the same arithmetic (fmaf, no other contraction): on the
writer's domains the corrected quotient equals the correctly rounded x / scale,
except for quotients below 2^-24 (below 2^-17 every format codes them to +-0),
and always has the sign of x / scale.  Random rows, and scales checked against
every finite bf16 x of their domain (edge scales first)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_markstein_quotient_is_correctly_rounded_on_the_writer_domains(tmp_path):
    exe = str(tmp_path / "markstein_check")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe, os.path.join(HERE, "native", "markstein_check.c"),
                    "-lm"], check=True)
    for seed in (1, 2, 3):
        out = subprocess.run([exe, str(seed), "60000"], check=True, capture_output=True, text=True).stdout
        f = dict(zip(out.split()[::2], map(int, out.split()[1::2])))
        assert f["pairs"] > 3_000_000
        assert f["differ_big"] == 0, out
        assert f["sign_bad"] == 0, out


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_markstein_quotient_exhaustive_over_bf16_per_scale(tmp_path):
    """Every finite bf16 x of the domain, for the edge scales (the epsilon floor,
    the largest amax of each Q_MAX, the smallest amax the writer divides this
    way) and 600 random affine and block scales."""
    exe = str(tmp_path / "markstein_check")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe, os.path.join(HERE, "native", "markstein_check.c"),
                    "-lm"], check=True)
    out = subprocess.run([exe, "7", "600", "exhaustive"], check=True, capture_output=True, text=True).stdout
    f = dict(zip(out.split()[::2], map(int, out.split()[1::2])))
    assert f["pairs"] > 15_000_000
    assert f["differ_big"] == 0, out
    assert f["sign_bad"] == 0, out
