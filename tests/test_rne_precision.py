"""The quantize+pack kernel takes the code decision rne(w/s) in IEEE fp32; the
oracle takes it in fp64.  This runs an exhaustive C check over every positive
finite bf16 w and fp16 s with w/s <= 512 that the two integers never differ
(see tests/native/rne_fp32_check.c), so both sides take the same decision."""
import os
import subprocess
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))


def test_fp32_rne_equals_fp64_rne_exhaustive():
    src = os.path.join(HERE, "native", "rne_fp32_check.c")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "rnecheck")
        subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off",
                        "-o", exe, src, "-lm"], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout
    assert "mismatches 0" in out.stdout
