"""The quantize kernels' bf16 quotient (three IEEE operations instead of a
division) gives the codes of the IEEE quotient for every bf16 input whose
tile scale lies in the kernels' fast range: an exhaustive CPU check, and a
check that the correction step is needed (without it codes differ)."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("qcheck") / "quotient_path_check")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                    "-I", os.path.join(ROOT, "oracle"), os.path.join(HERE, "quotient_path_check.c"),
                    os.path.join(ROOT, "oracle", "fp8_oracle.c"), "-o", exe, "-lm"], check=True)
    return exe


def _run(exe, *args):
    r = subprocess.run([exe, *args], capture_output=True, text=True, timeout=900)
    pairs, mism = (int(v) for v in r.stdout.split()[1::2])
    return r.returncode, pairs, mism


def test_corrected_quotient_codes_exact_for_all_bf16(checker):
    rc, pairs, mism = _run(checker)
    assert pairs > 1e9
    assert mism == 0 and rc == 0


def test_uncorrected_product_is_not_exact(checker):
    rc, pairs, mism = _run(checker, "--uncorrected")
    assert mism > 0 and rc != 0
