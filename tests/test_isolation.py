"""The product path and the oracle stay apart, and the product fails loudly
without its CUDA library.  CPU only: these read sources and import the
binding in a child process, nothing is launched."""
import os
import re
import subprocess
import sys

from conftest import ROOT

PKG = os.path.join(ROOT, "fp8_microscaling_quantization_b200")
CSRC = os.path.join(PKG, "csrc")


def _sources(top, exts):
    for d, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_product_sources_never_reach_the_oracle():
    """No package module imports the oracle, and no CUDA/C++ source includes,
    links or names a file under oracle/."""
    py = re.compile(r"^\s*(import\s+oracle\b|from\s+oracle\b)", re.M)
    for path in _sources(PKG, (".py",)):
        assert not py.search(open(path).read()), f"{path} imports the oracle"
    for path in _sources(CSRC, (".cu", ".cuh", ".h")):
        text = open(path).read()
        assert "bsq_oracle" not in text and "oracle/" not in text, f"{path} refers to the oracle"


def test_library_build_compiles_only_the_kernel_sources():
    from fp8_microscaling_quantization_b200 import build
    for s in build.SOURCES + build.HEADERS:
        assert os.path.exists(os.path.join(CSRC, s)), s
        assert "oracle" not in s
    assert all(os.path.dirname(f).endswith("csrc") or f.endswith("bsq.h") for f in build._inputs())


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """With the library missing the binding raises at import: there is no CPU
    or other fallback behind it."""
    env = dict(os.environ, BSQ_LIBRARY=str(tmp_path / "missing" / "libbsq.so"))
    code = "import fp8_microscaling_quantization_b200.bsq"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert r.returncode != 0
    assert "libbsq is not built" in r.stderr


def test_bench_runs_the_oracle_only_outside_the_timed_gpu_path():
    """bench.py imports the oracle only inside the functions that time it on
    the host (the CPU baseline and the reference arm)."""
    text = open(os.path.join(ROOT, "bench.py")).read()
    assert not re.search(r"^(import\s+oracle|from\s+oracle)", text, re.M), "module-level oracle import"
    funcs = re.split(r"\ndef ", text)
    users = [f.split("(", 1)[0] for f in funcs if re.search(r"\n\s+import oracle\b", f)]
    assert users and all(u in ("oracle_cases", "time_oracle_gemm", "mx_round_trip_case") for u in users), users
