"""The quantizer computes s = w / 15 without a division instruction, by
Markstein's correction step for a known divisor (P. Markstein, IBM J. Res. Dev.
34(1), 1990). This checks the method against IEEE division for every positive
normal binary32 w, on the CPU (fmaf is the same correctly rounded fused
multiply-add as the GPU's FFMA)."""
import os
import subprocess
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))


def test_markstein_div15_exhaustive():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "div15")
        flags = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math"]
        if "fma" in open("/proc/cpuinfo").read().split():
            flags.append("-mfma")
        subprocess.check_call(["gcc", *flags, "-o", exe, os.path.join(HERE, "div15_exhaustive.c"), "-lm"])
        out = subprocess.check_output([exe], timeout=600).decode().strip()
    assert out == "0", f"{out} mismatches"
