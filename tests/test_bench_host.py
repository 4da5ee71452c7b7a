"""Host-side logic of bench.py that decides whether recorded ncu traffic
still describes the kernel: the hash covers the GEMM's code, not its
comments."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _reader(texts):
    return lambda f: texts[f]


def _sources():
    out = {}
    for f in bench.GEMM_SOURCES:
        with open(os.path.join(ROOT, "w4a8_integer_gemm_b200", "csrc", f)) as fh:
            out[f] = fh.read()
    return out


def test_comments_and_whitespace_leave_the_hash():
    src = _sources()
    base = bench.gemm_source_hash(_reader(src))
    assert base == bench.gemm_source_hash()
    f = bench.GEMM_SOURCES[0]
    reworded = dict(src)
    reworded[f] = "// a new line of comment\n/* and a block\n   comment */\n" + src[f].replace("\n", "\n\n", 5)
    assert bench.gemm_source_hash(_reader(reworded)) == base


def test_a_code_change_changes_the_hash():
    src = _sources()
    base = bench.gemm_source_hash(_reader(src))
    for f in bench.GEMM_SOURCES:
        changed = dict(src)
        changed[f] = src[f] + "\nstatic int qoq_probe_symbol = 1;\n"
        assert bench.gemm_source_hash(_reader(changed)) != base, f


def test_code_only_strips_both_comment_forms():
    assert bench.code_only("int a; // x\n/* y\n z */ int  b;") == "int a; int b;"


def test_single_core_oracle_leg_restores_threads():
    import oracle
    from w4a8_integer_gemm_b200 import workloads as wl

    oracle.build()
    before = oracle.num_threads()
    r = bench.oracle_single_core(wl.WORKLOADS["tiny"], 0.2)
    assert r["cores"] == 1
    assert r["value"] > 0
    assert r["sample"].startswith("tiny: 16 tokens")
    assert oracle.num_threads() == before


def test_oracle_results_do_not_depend_on_threads():
    import numpy as np
    import oracle
    from w4a8_integer_gemm_b200 import workloads as wl

    X, W = wl.make_case(wl.WORKLOADS["tiny"], 0)
    before = oracle.num_threads()
    try:
        oracle.set_num_threads(1)
        r1 = oracle.linear(X.numpy(), W.numpy(), 128)
    finally:
        oracle.set_num_threads(before)
    rn = oracle.linear(X.numpy(), W.numpy(), 128)
    assert np.array_equal(r1["acc"], rn["acc"]) and np.array_equal(r1["Y"], rn["Y"])
