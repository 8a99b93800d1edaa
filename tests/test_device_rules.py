"""Static rules of the CUDA sources: kernels never trap and never spin without a
limit.  Every open-ended loop is a wait that checks the %globaltimer limit
(kWaitLimitNs) within a few lines, and every `while` loop is one of the known
bounded forms.  CPU only (reads the sources)."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCES = sorted(glob.glob(os.path.join(ROOT, "int4_routed_expert_renorm_b200", "csrc", "*.cu*"))
                 + glob.glob(os.path.join(ROOT, "synth", "csrc", "*.cu*")))
BOUNDED_WHILE = {"lo < hi"}     # binary searches over a segment table


def _code(path):
    """Source text with comments blanked out (line numbers kept)."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", lambda m: "\n" * m.group(0).count("\n"), text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_sources_found():
    assert len(SOURCES) >= 6


def test_no_trap_and_no_device_assert():
    for p in SOURCES:
        code = _code(p)
        assert "__trap" not in code, p
        assert "brkpt" not in code, p
        assert not re.search(r"(?<![A-Za-z_])assert\s*\(", code), p


def test_every_open_loop_checks_the_wait_limit():
    """An open loop compares %globaltimer with kWaitLimitNs, or with a
    `limit_ns` parameter of its function (checked below to default to
    kWaitLimitNs), within a few lines."""
    open_loop = re.compile(r"for\s*\([^;)]*;\s*;[^)]*\)|while\s*\(\s*(true|1)\s*\)|\bdo\s*\{")
    found = 0
    for p in SOURCES:
        lines = _code(p).split("\n")
        for i, ln in enumerate(lines):
            if open_loop.search(ln):
                found += 1
                window = "\n".join(lines[i:i + 12])
                assert ("kWaitLimitNs" in window or "limit_ns" in window) and "globaltimer()" in window, \
                    f"{p}:{i + 1}: {ln.strip()}"
    assert found >= 3      # the mbarrier wait, the token-block counter wait, the grid-wide counter wait


def test_wait_limit_parameters_default_to_the_limit():
    """Every `limit_ns` parameter of a wait routine defaults to kWaitLimitNs,
    so only a caller that names a limit waits less.  The one caller that does
    is the timeout test hook's kernel, whose host entry refuses any limit
    above kWaitLimitNs before launching it."""
    n = 0
    for p in SOURCES:
        code = _code(p)
        for m in re.finditer(r"(\w+)\s*\(([^()]*?)uint64_t\s+limit_ns\b([^,)]*)", code):
            if m.group(1) in ("wait_timeout_kernel", "coli_moe_test_wait_timeout"):
                assert "limit_ns > kWaitLimitNs" in code, p
                continue
            n += 1
            assert m.group(3).replace(" ", "") == "=kWaitLimitNs", f"{p}: {m.group(1)}: limit_ns{m.group(3)}"
    assert n >= 2


def test_while_loops_are_bounded_forms():
    for p in SOURCES:
        for m in re.finditer(r"\bwhile\s*\(([^)]*)\)", _code(p)):
            assert m.group(1).strip() in BOUNDED_WHILE, f"{p}: while ({m.group(1)})"
