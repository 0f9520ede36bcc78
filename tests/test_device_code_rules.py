"""Static checks on the CUDA sources (CPU): no device-side assert or trap
(a failed check must be recorded in the workspace status word and the kernel
must go on), no TMA load with cluster multicast, and every mbarrier wait goes
through the bounded helper."""
import os
import re

CSRC = os.path.join(os.path.dirname(__file__), "..", "sparse_attention_aware_b200", "csrc")


def _sources():
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, f)) as fh:
                yield f, fh.read()


def _code(text):
    """The source with comments removed."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_no_device_assert_or_trap():
    for f, src in _sources():
        code = _code(src)
        assert not re.search(r"(?<![_\w])assert\s*\(", code), f
        assert "__trap" not in code and not re.search(r"\btrap\s*;", code), f
        assert "__brkpt" not in code, f


def test_no_multicast_loads():
    for f, src in _sources():
        assert "multicast::cluster" not in _code(src).replace("tcgen05.commit", ""), f


def test_mbarrier_waits_are_bounded():
    """try_wait appears only inside the bounded wait helper."""
    for f, src in _sources():
        code = _code(src)
        n = len(re.findall(r"mbarrier\.try_wait", code))
        if f == "tc_ptx.cuh":
            assert n == 1
        else:
            assert n == 0, f
        assert "mbarrier.wait" not in code.replace("try_wait", ""), f
