"""The FP8 quantiser's division, checked exhaustively on the host.

The device divides each element x of a block by the block's scale
s = amax / 448 with a corrected reciprocal product (Markstein's division:
r = 1/s, q0 = x r, q = q0 + (x - q0 s) r, two FMAs) when s >= 2^-100, and
with IEEE division otherwise.  tests/fp8_division_check.c restates those
steps in C and compares them with IEEE division for every pair of BF16
(and of FP16) values (amax, x), |x| <= amax, both signs: the binary32
quotients must be equal, or both at most 2^-10 in magnitude with the sign of
x (the same E4M3 zero).  A copy without the correction step must fail the
same check, so that the check can see a misrounded quotient.  No GPU."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "fp8_division_check.c")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not installed")
    exe = str(tmp_path_factory.mktemp("fp8div") / "fp8_division_check")
    base = ["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-ffp-contract=off",
            "-fno-fast-math", SRC, "-o", exe, "-lm"]
    r = subprocess.run(base[:1] + ["-fopenmp"] + base[1:], capture_output=True, text=True)
    if r.returncode != 0:  # no OpenMP: the same check on one core
        r = subprocess.run(base, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def _run(exe, *args):
    r = subprocess.run([exe, *args], capture_output=True, text=True, timeout=900)
    m = re.search(r"pairs (\d+) fast (\d+) zero_equiv (\d+) ieee (\d+) bad (\d+)", r.stdout)
    assert m, r.stdout + r.stderr
    return r.returncode, dict(zip(("pairs", "fast", "zero_equiv", "ieee", "bad"),
                                  map(int, m.groups()))), r.stderr


# every (amax, x) pair: sum over amax encodings a = 1..top of 2 (a + 1)
@pytest.mark.parametrize("fmt,top", [("bf16", 0x7F7F), ("fp16", 0x7BFF)])
def test_corrected_reciprocal_equals_ieee_division(checker, fmt, top):
    rc, c, err = _run(checker, fmt)
    assert rc == 0 and c["bad"] == 0, err
    assert c["pairs"] == sum(2 * (a + 1) for a in range(1, top + 1))
    assert c["fast"] + c["ieee"] == c["pairs"]
    if fmt == "fp16":
        assert c["ieee"] == 0           # every FP16 scale is >= 2^-100
    else:
        assert c["fast"] > 0.98 * c["pairs"]  # only amax below ~2^-91 takes IEEE division


def test_check_detects_a_missing_correction(checker):
    rc, c, err = _run(checker, "fp16", "nocorr")
    assert rc == 1 and c["bad"] > 1000000, (c, err)
    assert "mismatch" in err
