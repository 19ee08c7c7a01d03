"""Source-level rules of the CUDA library, checked without a GPU.

Every wait in the kernels must end by itself: a stuck pipeline raises a
status bit and the kernel returns, it never spins forever.  The only code
that polls an mbarrier is the pair of bounded helpers in common.cuh; every
kernel waits through them.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_07_b200", "csrc")


def _sources():
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh")):
            yield f, open(os.path.join(CSRC, f)).read()


def _function_body(text, name):
    i = text.index(name + "(")
    j = text.index("{", i)
    depth = 0
    for k in range(j, len(text)):
        depth += {"{": 1, "}": -1}.get(text[k], 0)
        if depth == 0:
            return text[j:k + 1]
    raise AssertionError(name)


def test_only_the_bounded_helpers_poll_an_mbarrier():
    calls = 0
    for f, text in _sources():
        code = re.sub(r"//[^\n]*", "", text)
        # the raw instruction appears once, inside the one-shot probe
        assert code.count("mbarrier.try_wait") == (1 if f == "common.cuh" else 0), f
        calls += len(re.findall(r"(?<!bool )\bmbar_try_wait\s*\(", code))
    common = re.sub(r"//[^\n]*", "", dict(_sources())["common.cuh"])
    inside = sum(len(re.findall(r"\bmbar_try_wait\s*\(", _function_body(common, name)))
                 for name in ("bool mbar_wait", "bool mbar_wait_teardown"))
    assert calls == inside == 2


def test_the_bounded_helpers_have_their_limits():
    text = dict(_sources())["common.cuh"]
    wait = _function_body(text, "bool mbar_wait")
    assert "limit_cycles" in wait and "abort_flag" in wait and "MOBA_DEV_TIMEOUT" in wait
    teardown = _function_body(text, "bool mbar_wait_teardown")
    assert "limit_ns" in teardown


def test_no_unconditional_loops_in_kernels():
    for f, text in _sources():
        code = re.sub(r"//[^\n]*", "", text)
        assert not re.search(r"while\s*\(\s*(true|1)\s*\)", code), f
        # the bounded wait's own loop exits through its limit
        for m in re.finditer(r"for\s*\(\s*[^;]*;\s*;", code):
            assert f == "common.cuh" and "mbar_wait" in code[max(0, m.start() - 600):m.start()], f
