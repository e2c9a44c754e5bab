"""Rules every kernel source of the library keeps, checked on the text of
csrc/ (no GPU): no trap instruction or device-side assert (a failure is a
status bit, never a dead context); no device allocation inside the library
(callers pass workspaces); every spin-wait bounded -- a loop polling an
mbarrier carries the cycle limit on its own line, and the only open-ended
loops are the two bounded-wait helpers (each returns on the cycle limit or
the CTA's abort flag) and the work-claiming loop (its counter only grows,
up to the item count); no TMA or bulk copy uses cluster multicast (the one
multicast is the tcgen05.commit that signals both CTAs of a GEMM pair).
"""
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "invariant_deterministic_03_b200", "csrc")
OPEN_LOOP_OK = {"mbar_wait", "mbar_wait_cluster", "claim_item"}


def _sources():
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            yield f, open(os.path.join(CSRC, f)).read()


def _code(text):
    """The text with comments removed (line structure kept)."""
    text = re.sub(r"/\*.*?\*/", lambda m: "\n" * m.group(0).count("\n"), text, flags=re.S)
    return "\n".join(line.split("//")[0] for line in text.split("\n"))


def test_no_trap_or_device_assert():
    for f, text in _sources():
        code = _code(text)
        assert "__trap" not in code, f
        assert not re.search(r"\btrap\s*;", code), f
        assert not re.search(r"\bassert\s*\(", code), f


def test_no_device_allocation_in_the_library():
    for f, text in _sources():
        code = _code(text)
        assert not re.search(r"\bcuda(Malloc|MallocAsync|MallocManaged|MallocHost)\s*\(", code), f
        assert not re.search(r"\bcuMem(Alloc|Create)\w*\s*\(", code), f


def test_every_spin_wait_is_bounded():
    fn_re = re.compile(r"(?:__device__|__global__)[^;{]*?\b(\w+)\s*\(")
    for f, text in _sources():
        current = None
        for n, line in enumerate(_code(text).split("\n"), 1):
            m = fn_re.search(line)
            if m:
                current = m.group(1)
            if re.search(r"while\s*\(\s*!\s*mbar_try_wait", line):
                assert "kWaitLimitCycles" in line, f"{f}:{n}: unbounded mbarrier poll"
            if re.search(r"while\s*\(\s*(true|1)\s*\)|for\s*\(\s*;\s*;\s*\)", line):
                assert current in OPEN_LOOP_OK, f"{f}:{n}: open-ended loop in {current}"


def test_no_multicast_copies():
    for f, text in _sources():
        for n, line in enumerate(_code(text).split("\n"), 1):
            if "multicast" in line:
                assert "tcgen05.commit" in line, f"{f}:{n}: multicast outside tcgen05.commit"
            if re.search(r"cp\.async\.bulk", line):
                assert "multicast" not in line, f"{f}:{n}: bulk copy with multicast"
