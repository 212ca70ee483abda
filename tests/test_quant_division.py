"""The CUDA quantizer divides by the group scale with one IEEE reciprocal
per group and Markstein's correction step per element (plus restoring the
sign of x).  tests/div_exhaustive.c replays that sequence in IEEE binary32
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
    assert " bad 0 " in r.stdout
    assert int(r.stdout.split()[1]) > 10 ** 9      # every pair was visited
