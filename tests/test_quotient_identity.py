"""The quantize kernel computes rint(fl(x/s)) without a division: q0 = x*rcp,
one residual correction (Markstein) and a round-to-integer constant.  This
host test compiles tests/quotient_identity.c and checks that identity for
every finite bf16 x and every positive finite fp16 scale s with |x/s| <= 40
(about 1.08e9 pairs); it needs no GPU."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_division_free_quotient_rounds_like_ieee_division():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "quotient_identity")
        subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-o", exe,
                        os.path.join(HERE, "quotient_identity.c"), "-lm"], check=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    pairs, bad = (int(v) for v in r.stdout.split()[1::2])
    assert bad == 0 and pairs > 1_000_000_000
