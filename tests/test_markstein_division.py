"""The division the gated SubLN quantizer uses for x / r (Markstein's method
from the correctly rounded reciprocal of the row constant r, one FMA
remainder and one FMA correction) equals IEEE float division for normal
dividends, and is not exact for subnormal ones, which is why the kernel
sends those to the IEEE division.  Plain C with correctly rounded fmaf on
the host; the GPU parity tests then check the kernel's x_q and s bit for bit."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    exe = str(tmp_path_factory.mktemp("mk") / "markstein_check")
    subprocess.run([gcc, "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                    os.path.join(HERE, "markstein_check.c"), "-o", exe, "-lm"], check=True)
    return exe


def _run(exe, nb, subnormal):
    out = subprocess.run([exe, str(nb), str(int(subnormal))], check=True, capture_output=True, text=True,
                         timeout=600).stdout.split()
    return int(out[0]), int(out[1])


def test_correctly_rounded_for_normal_dividends(checker):
    total, bad = _run(checker, 24, False)  # 24 divisors x 2 binades x every dividend mantissa
    assert total == 24 * 2 * (1 << 23)
    assert bad == 0


def test_not_exact_for_subnormal_dividends(checker):
    total, bad = _run(checker, 2, True)
    assert total == 2 * 2 * ((1 << 23) - 1)
    assert bad > 0  # the reason the kernel takes the IEEE division for them
