"""The quantizers' division-free quotient, checked on the CPU (no GPU).

The encode kernels never divide: each quotient x / d of the recipe is formed
from three per-divisor reciprocals and one remainder correction (Markstein's
theorem; the steps are in csrc/quant.cu's header).  tests/models/exact_div_model.c
restates those steps with C99 fmaf and compares the result with the IEEE
quotient bit for bit: over every normal bf16 dividend with quotients in
[2^-7, 2^5) against 65536 divisor significands, over random binary32
dividends, over exact ties on the E2M1 and E4M3 rounding boundaries, and over
every bf16 dividend (zeros and subnormals included) at divisors spanning the
recipe's domain.  Quotients below 2^-10 only need their sign (they code to
zero).  Not a parity test of the GPU path (the GPU tests are); this pins the
method the kernels use."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "models", "exact_div_model.c")


@pytest.fixture(scope="module")
def model_bin(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("exact_div") / "exact_div_model")
    # -ffp-contract=off: every operation rounds once, as the kernels' intrinsics do
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", out, SRC, "-lm"], check=True)
    return out


def test_quotients_are_correctly_rounded(model_bin):
    res = subprocess.run([model_bin, "128"], check=True, capture_output=True, text=True).stdout
    rows = {ln.split()[0]: (int(ln.split()[1]), int(ln.split()[2])) for ln in res.splitlines()}
    assert set(rows) == {"bf16_dividends", "binary32_dividends", "exact_ties", "edge_dividends"}
    for name, (n, bad) in rows.items():
        assert n > 0, name
        assert bad == 0, f"{name}: {bad} of {n} quotients differ from IEEE division"
    assert rows["bf16_dividends"][0] == (1 << 16) * 11 * 128 * 2
    assert rows["exact_ties"][0] > 1000
