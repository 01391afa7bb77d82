"""The NVFP4 kernel forms y = RN32(x / d) for bf16 x with a correctly
rounded reciprocal and one FMA correction instead of a full IEEE division
per element.  tests/csrc/division_check.c proves on the CPU, by exhaustion
over every pair of significands (all bf16 x, all fp32 d), that this gives
the correctly rounded quotient; the kernel takes an exact-division path for
block scales outside the range where the argument holds."""
import os
import subprocess
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))


def _has_fma():
    try:
        with open("/proc/cpuinfo") as f:
            return " fma " in f.read()
    except OSError:
        return False


def test_reciprocal_fma_quotient_is_correctly_rounded_exhaustively():
    src = os.path.join(HERE, "csrc", "division_check.c")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "division_check")
        flags = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp"]
        if _has_fma():
            flags.append("-mfma")
        subprocess.check_call(["gcc", *flags, "-o", exe, src, "-lm"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "mismatches 0" in out.stdout
