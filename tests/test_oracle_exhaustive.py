"""The oracle's two minifloat encoders (E2M1 and E4M3, round to nearest with
ties to the even mantissa, saturating) against an independent brute-force
rounding over every binary32 bit pattern (tests/exhaustive/codes_exhaustive.c,
compiled here with gcc and linked to the oracle library; all host cores)."""
import os
import subprocess
import tempfile

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))


def test_encoders_match_brute_force_on_every_binary32():
    lib = oracle_build.build()
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "codes_exhaustive")
        subprocess.run(["gcc", "-O2", "-std=c11", "-pthread", "-o", exe,
                        os.path.join(HERE, "exhaustive", "codes_exhaustive.c"), lib, "-lm",
                        "-Wl,-rpath," + os.path.dirname(lib)], check=True)
        r = subprocess.run([exe, str(os.cpu_count() or 1)], capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "e2m1_mismatches=0 e4m3_mismatches=0 inputs=4294967296" in r.stdout, r.stdout
