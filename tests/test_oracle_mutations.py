"""The pins have teeth: plant a plausible mistake in a copy of the CPU oracle
and check that the pin written against the pages or the mathematics fails.

Each case rewrites one line of oracle/bsq_oracle.c (the text must occur
exactly once), builds the copy with gcc into a temporary directory, points
the oracle wrapper at it, and runs the real pin test, expecting an
AssertionError.  The committed oracle is never touched.  CPU only.
"""
import os
import subprocess

import pytest

import oracle as oracle_mod
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "bsq_oracle.c")

MUTATIONS = {
    # ties of the e2m1 rounding go toward zero instead of to the even code
    "e2m1_ties_toward_zero": (
        "else if (a == E2M1_MIDPOINTS[i] && ((i + 1) % 2) == 0) idx = i + 1;",
        "else if (a == E2M1_MIDPOINTS[i] && 0) idx = i + 1;",
        "test_e2m1_round_matches_bruteforce_all_bf16"),
    # the NVFP4 decode rounds s * g first instead of (e2m1 * s) * g
    "nvfp4_decode_order": (
        "            float prod = v * s;\n            float val = prod * g[r];",
        "            float val = v * (s * g[r]);",
        "test_nvfp4_decode_is_product_of_three"),
    # the MXFP4 block exponent offset is off by one
    "mxfp4_exponent_offset": (
        "int e = (amax_b == 0.0f) ? -127 : o_floor_log2(amax_b) - 2;",
        "int e = (amax_b == 0.0f) ? -127 : o_floor_log2(amax_b) - 1;",
        "test_mxfp4_exponent_rule"),
    # code 8 decodes to -0.0 (the printed table holds 0.0 there)
    "e2m1_negative_zero": (
        "0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};",
        "-0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};",
        "test_e2m1_table_and_midpoints_printed"),
    # MXFP8 uses MXFP4's exponent offset
    "mxfp8_wrong_offset": (
        "int e = (amax_b == 0.0f) ? -127 : o_floor_log2(amax_b) - 8;",
        "int e = (amax_b == 0.0f) ? -127 : o_floor_log2(amax_b) - 2;",
        "test_mxfp8_exponent_rule_and_saturation"),
    # the static two-level scale skips its min_value floor
    "static_no_floor": (
        "    if (sb <= min_value) sb = min_value;",
        "    (void)min_value;",
        "test_nvfp4_static_scale_floor_and_range"),
    # the KV cache writes each block at the previous block's offset
    "kv_block_offset": (
        "void* yb = (char*)y + (size_t)(b * rows * 128) * (size_t)elem;",
        "void* yb = (char*)y + (size_t)((b > 0 ? b - 1 : 0) * rows * 128) * (size_t)elem;",
        "test_kv_cache_layout_and_values"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pin_catches_planted_mistake(name, tmp_path, monkeypatch, golden_dir):
    before, after, pin = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site of {name} not found exactly once"
    mutated = tmp_path / "bsq_oracle_mutant.c"
    mutated.write_text(src.replace(before, after))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-o", str(lib),
                           str(mutated), "-lm"])
    # point the wrapper at the mutant (the wrapper rebuilds only when its
    # library is older than its source, which the fresh mutant is not)
    monkeypatch.setattr(oracle_mod, "_LIB_PATH", str(lib))
    monkeypatch.setattr(oracle_mod, "_SRC", str(mutated))
    monkeypatch.setattr(oracle_mod, "_lib", None)
    fn = getattr(pins, pin)
    kwargs = {"oracle": oracle_mod}
    if "golden_dir" in fn.__code__.co_varnames[:fn.__code__.co_argcount]:
        kwargs["golden_dir"] = golden_dir
    with pytest.raises(AssertionError):
        fn(**kwargs)
