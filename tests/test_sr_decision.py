"""The kernels' stochastic-rounding decision, restated in C with directed
rounding (tests/sr_decision_check.c), against the rule of section 2B.4 of
"Pretraining Large Language Models with NVFP4": between the neighbouring E2M1
magnitudes, round up iff the 24-bit uniform is below the fractional
position.  The kernels compute it as one FP32 formula whose lattice step comes
from |y|'s exponent; this checks the formula over the whole range of scaled
magnitudes [0, 6.4), sampled by default and every float with
NVFP4_SR_CHECK_FULL=1 (about a minute and a half).  The GPU parity tests then
show that the kernels compute that formula (bit-exact SR codes vs the
oracle)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    exe = str(tmp_path_factory.mktemp("sr") / "sr_decision_check")
    subprocess.run(["gcc", "-O2", "-frounding-math", "-std=c99", "-o", exe,
                    os.path.join(HERE, "sr_decision_check.c"), "-lm"], check=True)
    return exe


def test_sr_decision_formula_matches_the_rule(checker):
    stride = "1" if os.environ.get("NVFP4_SR_CHECK_FULL") == "1" else "97"
    r = subprocess.run([checker, stride], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout
    assert r.stdout.strip().endswith(", 0 mismatches"), r.stdout


def test_checker_detects_a_wrong_rule(checker, tmp_path):
    # a planted mistake (round up iff u <= p instead of u < p) must be found
    src = open(os.path.join(HERE, "sr_decision_check.c")).read()
    bad = src.replace("(u < p) ? kGrid[i + 1]", "(u <= p) ? kGrid[i + 1]")
    assert bad != src
    path = tmp_path / "bad.c"
    path.write_text(bad)
    exe = str(tmp_path / "bad")
    subprocess.run(["gcc", "-O2", "-frounding-math", "-std=c99", "-o", exe, str(path), "-lm"], check=True)
    r = subprocess.run([exe, "1021"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 1 and "mismatches" in r.stdout
