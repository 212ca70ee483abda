"""The CUDA quantizer forms the group scale amax/448 with Markstein's
correction step against fp32(1/448), and divides by the scale with one IEEE
reciprocal per group and the same correction step per element (plus the sign
of x OR-ed into the code).  tests/div_exhaustive.c replays that sequence in IEEE binary32
on the host for every (amax, x) pair of bf16 values the kernels can meet
and checks each quotient gives the same e4m3 code as the IEEE division that
the quantization definition uses.  About 5 s on 8 cores."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_markstein_quotient_matches_ieee_division_exhaustively(tmp_path):
    exe = str(tmp_path / "div_exhaustive")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-pthread",
                    os.path.join(HERE, "div_exhaustive.c"), "-o", exe, "-lm"], check=True)
    r = subprocess.run([exe, str(os.cpu_count() or 4)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = r.stdout.splitlines()
    assert lines[0] == "scales 32640 bad 0"
    assert " bad 0 " in lines[1]
    assert int(lines[1].split()[1]) > 10 ** 9      # every pair was visited
