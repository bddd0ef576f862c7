"""Rules the CUDA sources keep, checked statically on the CPU: every mbarrier wait is bounded
(the polling instruction appears once, inside the helper, and every poll loop carries a cycle
limit), no kernel ends itself with a trap or a device assert, and no loop is written to run
forever. (The GPU tests run the bounded waits out with a lowered cap.)"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = sorted(glob.glob(os.path.join(ROOT, "ternary_weight_matmul_b200", "csrc", "*.cu*")))


def _code(path):
    """Source without comments."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_sources_found():
    assert len(CSRC) >= 10


def test_mbarrier_polling_lives_in_one_helper():
    hits = {os.path.basename(p): _code(p).count("mbarrier.try_wait") for p in CSRC}
    assert sum(hits.values()) == 1 and hits["common.cuh"] == 1, hits


def test_every_poll_loop_is_bounded():
    loops = 0
    for path in CSRC:
        code = _code(path)
        for m in re.finditer(r"while\s*\(([^{;]*mbar_try_wait[^{;]*)\)", code):
            cond = m.group(1)
            body_start = m.end()
            body = code[body_start:body_start + 400]
            bounded = "clock64()" in cond or ("clock64()" in body and "return false" in body)
            assert bounded, (os.path.basename(path), cond)
            loops += 1
    assert loops >= 4      # the bounded wait, the drain, and the fused decode's two start-up waits


def test_no_trap_assert_or_endless_loop():
    for path in CSRC:
        code = _code(path)
        assert "__trap" not in code and "trap;" not in code, path
        assert not re.search(r"(?<!static_)\bassert\s*\(", code), path
        assert not re.search(r"for\s*\(\s*;\s*;\s*\)|while\s*\(\s*(true|1)\s*\)", code), path
