"""Host proof that the quantisation kernel's fast quotient gives the oracle's E4M3 codes.

The E4M3 quantisation kernel (fa_quant.cu) takes x / scale from the tile's reciprocal and
one correction step instead of an IEEE division per element.  e4m3_quotient_check.c runs
that arithmetic over every (amax, x) pair of the 16-bit input types, about 1e9 pairs, and
counts the pairs whose quotient is neither the IEEE quotient nor, with it, at or below
2^-10 (where both round to code 0).  The GPU test test_fp8_gpu.py::
test_quantize_every_value_below_sampled_amax checks the kernel itself on sampled amax."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("quotient") / "e4m3_quotient_check")
    # no contraction and no fast-math: every operation rounds as IEEE fp32 prescribes
    subprocess.run([cc, "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                    os.path.join(HERE, "e4m3_quotient_check.c"), "-o", exe, "-lm"],
                   check=True, capture_output=True)
    return exe


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_reciprocal_quotient_gives_the_division_codes(checker, dtype):
    out = subprocess.run([checker, dtype], check=True, capture_output=True, text=True).stdout
    pairs, bad = int(out.split()[1]), int(out.split()[3])
    assert pairs > 5e8 and bad == 0, out
