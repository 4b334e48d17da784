"""Static checks on the CUDA/C++ sources (no GPU): rules every kernel of the library keeps.

- No trap or breakpoint instruction: failures are reported through status words, not faults.
- No TMA or bulk copy with cluster multicast.  The CTA-pair GEMM multicasts only
  tcgen05.commit arrivals inside its own cluster; its loads use the cta_group::2 form, in which
  each CTA loads only into its own shared memory.
- Every mbarrier poll goes through the bounded helpers of ptx.cuh.  Those give up after a time
  limit or when the CTA's abort flag is set.
"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rotation_int4_w4a4_b200", "csrc")


def sources():
    files = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                   glob.glob(os.path.join(CSRC, "*.cpp")) + glob.glob(os.path.join(CSRC, "*.h")))
    assert files
    out = {}
    for f in files:
        text = open(f).read()
        # drop comments, keep string literals (inline PTX lives in them)
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        out[os.path.basename(f)] = text
    return out


def string_literals(code):
    return re.findall(r'"((?:[^"\\]|\\.)*)"', code)


def test_no_trap_or_breakpoint():
    for name, code in sources().items():
        assert not re.search(r"__trap\s*\(|__brkpt\s*\(", code), name
        for lit in string_literals(code):
            assert not re.search(r"\btrap\b|\bbrkpt\b|\bexit\s*;", lit), (name, lit)


def test_no_bulk_copy_with_cluster_multicast():
    seen_bulk = 0
    for name, code in sources().items():
        for lit in string_literals(code):
            if "cp.async.bulk" in lit:
                seen_bulk += 1
                assert "multicast" not in lit, (name, lit)
            if "multicast" in lit:
                assert lit.startswith("tcgen05.commit"), (name, lit)
    assert seen_bulk >= 2          # the checks above did see the TMA loads


def test_mbarrier_polls_only_in_bounded_helpers():
    src = sources()
    for name, code in src.items():
        if name == "ptx.cuh":
            continue
        for lit in string_literals(code):
            assert "mbarrier.try_wait" not in lit and "mbarrier.test_wait" not in lit, (name, lit)
        assert not re.search(r"\bmbar_try_wait\w*\s*\(", code), name
    ptx = src["ptx.cuh"]
    # split ptx.cuh into function bodies and find every caller of the raw polls
    bodies = re.findall(r"__device__ __forceinline__ [\w:<>]+ (\w+)\(([^)]*)\)\s*\{(.*?)\n\}", ptx, flags=re.S)
    callers = {fn for fn, _, body in bodies if re.search(r"\bmbar_try_wait\w*\s*\(", body)}
    assert callers == {"mbar_wait_bounded", "mbar_wait_bounded_cl"}, callers
    for fn, args, body in bodies:
        if fn in callers:
            assert "globaltimer_ns() - t0 > limit_ns" in body, fn
            assert "if (*abort) return false;" in body, fn
