"""Static checks of the kernel sources: every device wait is bounded, no
kernel traps, and no bulk copy multicasts across a cluster.

A loop that polls memory another agent writes (an mbarrier phase, a
stream-K partner's flag) must give up after the library's cycle limit, so a
missing arrival ends in ISD_DEV_TIMEOUT instead of a hung GPU; and no
kernel may stop the context with a trap or a failing device assert.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "strided_verify_propose_b200", "csrc")
POLL = re.compile(r"\bwhile\s*\(.*(try_wait|ld_acquire|ld_volatile|atomicCAS|atomicAdd\s*\([^)]*,\s*0\))")


def _sources():
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, f)) as fh:
                yield f, fh.read().split("\n")


def test_every_polling_loop_checks_the_cycle_limit():
    polls = 0
    for name, lines in _sources():
        for i, line in enumerate(lines):
            if POLL.search(line):
                polls += 1
                body = "\n".join(lines[i:i + 4])
                assert re.search(r"clock64\(\)\s*-\s*t0\s*>\s*limit", body), f"{name}:{i + 1}: {line.strip()}"
                window = "\n".join(lines[max(0, i - 4):i])
                assert "g_wait_limit" in window, f"{name}:{i + 1}: the limit is not the library's"
    assert polls >= 2      # the mbarrier wait and the stream-K partner flag


def test_no_kernel_traps_or_asserts():
    for name, lines in _sources():
        for i, line in enumerate(lines):
            code = line.split("//")[0]
            assert "__trap" not in code and not re.search(r"\btrap;", code), f"{name}:{i + 1}"
            assert not re.search(r"\bassert\s*\(", code), f"{name}:{i + 1}"
            assert "__brkpt" not in code, f"{name}:{i + 1}"


def test_no_bulk_copy_uses_cluster_multicast():
    """Every TMA / bulk copy reads or writes this CTA's (or its pair's) own
    tile: none carries a multicast qualifier. The only multicast in the
    kernels is the tcgen05 commit's mbarrier arrive inside a 2-SM pair."""
    qualifier = "multi" + "cast"
    copies = 0
    for name, lines in _sources():
        for i, line in enumerate(lines):
            code = line.split("//")[0]
            if "cp.async.bulk" in code:
                copies += 1
                assert qualifier not in code, f"{name}:{i + 1}"
            elif qualifier + "::" in code:
                assert "tcgen05.commit" in code, f"{name}:{i + 1}"
    assert copies >= 3
