"""The oracle's e2m1, e4m3 and bf16 roundings on every binary32 bit pattern
(e4m3: every positive pattern of the binades where two codes compete, a
sample elsewhere), checked by a multi-threaded C program against
round-to-nearest-even: nearest value, ties to the even code, saturation at
6 and 448, sign from the sign bit, monotone.  Also floor_log2 on every
positive finite value and the power-of-two ceiling on every positive normal,
against their closed forms.  CPU only, under a minute on 8 cores."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_roundings_on_every_binary32_pattern(oracle, tmp_path):
    lib = oracle.build()
    exe = str(tmp_path / "rounding_exhaustive")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-pthread", "-o", exe,
                           os.path.join(HERE, "rounding_exhaustive.c"), lib,
                           "-Wl,-rpath," + os.path.dirname(lib), "-lm"])
    threads = max(1, len(os.sched_getaffinity(0)))
    r = subprocess.run([exe, str(threads)], capture_output=True, text=True, timeout=3600)
    assert r.returncode == 0, r.stdout + r.stderr
    for fmt in ("e2m1", "bf16", "e4m3", "floor_log2", "pow2_ceil"):
        assert f"{fmt} failures 0 " in r.stdout, r.stdout
