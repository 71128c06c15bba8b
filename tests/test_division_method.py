"""Pin of the division method of the CUDA quantizer (no GPU needed).

The kernels compute x / scale from a two-term reciprocal of the scale and one
Markstein FMA correction instead of an IEEE division. tests/division_method_check.c
checks, with the host's IEEE binary32 arithmetic, that this equals the IEEE
quotient on the kernels' domain (scale >= 2^-40, |x| >= 2^-100), and that
where it may not (underflowing remainders) no quantization code can change.
The GPU parity tests then check that the kernels implement it faithfully.
"""

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_fma_division_is_exact_on_the_kernel_domain(tmp_path):
    exe = str(tmp_path / "division_method_check")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe, os.path.join(HERE, "division_method_check.c"),
                    "-lm"], check=True)
    res = subprocess.run([exe, "20000000"], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "0 violations" in res.stdout
