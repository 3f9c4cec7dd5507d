"""Rules the CUDA sources keep so that no kernel can fault, trap or hang a
shared GPU, checked on the source text (no GPU needed):

- no trap instruction: failures are reported through a status word;
- no TMA or bulk load with cluster multicast (only the tcgen05.commit arrive
  may multicast), so every kernel is safe to run with peers' memory;
- every wait on an mbarrier gives up after a time limit: each loop whose
  condition polls a barrier also tests the elapsed time against the limit,
  and the only unconditional loop (the shared wait helper) does the same.
"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCES = sorted(glob.glob(os.path.join(ROOT, "hybrid_sparse_gemm_b200", "csrc", "*.cu")) +
                 glob.glob(os.path.join(ROOT, "hybrid_sparse_gemm_b200", "csrc", "*.cuh")))


def _code(path):
    """Source text without // and /* */ comments (string contents kept)."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", lambda m: "\n" * m.group(0).count("\n"), text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def _loops(text):
    """(condition, body start) of every while loop, parentheses balanced."""
    for m in re.finditer(r"\bwhile\s*\(", text):
        depth, i = 1, m.end()
        while depth:
            depth += {"(": 1, ")": -1}.get(text[i], 0)
            i += 1
        yield text[m.end():i - 1], i


def test_sources_found():
    names = {os.path.basename(p) for p in SOURCES}
    assert {"gemm22.cu", "gemm2.cu", "gemm.cu", "decode.cu", "common.cuh"} <= names


def test_no_trap():
    for p in SOURCES:
        code = _code(p)
        assert "__trap" not in code and not re.search(r"\btrap\s*;", code) and "brkpt" not in code, p


def test_no_multicast_loads():
    for p in SOURCES:
        for n, line in enumerate(_code(p).splitlines(), 1):
            if "multicast" in line:
                assert "tcgen05.commit" in line, f"{os.path.basename(p)}:{n}: {line.strip()}"


def test_barrier_waits_are_bounded():
    polled = 0
    for p in SOURCES:
        code = _code(p)
        for cond, body in _loops(code):
            if "mbar_try_wait" in cond or "mbar_test_wait" in cond:
                polled += 1
                assert "kWaitLimitNs" in cond and "globaltimer" in cond, f"{os.path.basename(p)}: while ({cond})"
            elif cond.strip() in ("true", "1"):
                # the shared wait helper: its body must give up after the limit
                end = code.index("\n}", body)
                assert "kWaitLimitNs" in code[body:end] and "return false" in code[body:end], p
    assert polled >= 6   # the drain and producer waits of every tensor-core kernel


def test_wait_limit_is_about_a_second():
    code = _code(os.path.join(ROOT, "hybrid_sparse_gemm_b200", "csrc", "common.cuh"))
    m = re.search(r"kWaitLimitNs\s*=\s*(\d+)ull", code)
    assert m and 1e8 <= int(m.group(1)) <= 5e9
