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


def test_constant_divisor_division_is_exact_and_matches_the_kernel_literals(tmp_path):
    """The row scale is absmax / D (or (max - min) / D) for D in {7, 15, 127, 255}.
    The kernels divide with the compile-time two-term reciprocal of D and one
    FMA correction; every significand at the subnormal, 2^-100, unit and top
    binades must give the IEEE quotient, and the literals in the CUDA header
    must be RN(1/D) and RN(RN(1 - D*y) * y)."""
    import re

    exe = str(tmp_path / "const_division_check")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe, os.path.join(HERE, "const_division_check.c"),
                    "-lm"], check=True)
    res = subprocess.run([exe, "0", "27", "127", "254"], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "0 violations" in res.stdout
    host = {int(m.group(1)): (float.fromhex(m.group(2)), float.fromhex(m.group(3)))
            for m in re.finditer(r"D=(\d+) y=(\S+) lo=(\S+)", res.stdout)}
    header = open(os.path.join(os.path.dirname(HERE), "token_dynamic_quantization_b200", "csrc", "dq_device.cuh")).read()
    kernel = {int(m.group(1)): (float.fromhex(m.group(2)), float.fromhex(m.group(3)))
              for m in re.finditer(r"struct ConstRecip<(\d+)> \{\s*static constexpr float y = ([-0-9a-fx.p]+)f, "
                                   r"lo = ([-0-9a-fx.p]+)f;", header)}
    assert set(kernel) == {7, 15, 127, 255}
    assert kernel == host
