"""Source checks of the programmatic dependent launches (CPU only).

A kernel launched as a programmatic dependent may start while the kernel before it
on the stream is still running.  It is correct only if every thread waits on the
grid dependency before its first access to global memory.  These tests read the
CUDA sources and check two things for every such kernel:
  * nothing but declarations (constants, static asserts, type aliases, the
    reference to the kernel parameters) comes before `grid_dependency_wait()`;
  * the decode sources launch nothing with `<<<...>>>`, which would drop the
    launch attribute.
"""

import os
import re

CSRC = os.path.join(os.path.dirname(__file__), "..", "paged_kv_cache_413_b200", "csrc")

# kernel -> source file; each is launched with programmatic stream serialization
DEPENDENTS = {
    "decode_kernel": "pa_decode.cu",
    "decode_mma_kernel": "pa_decode.cu",
    "lse_reduce_kernel": "pa_decode.cu",
    "decode_shared_prefix_kernel": "pa_decode_shared.cu",
    "decode_shared_tc_kernel": "pa_decode_shared.cu",
}

ALLOWED_BEFORE_WAIT = re.compile(
    r"^\s*(//.*|constexpr\b.*|static_assert\b.*|using\b.*|const Params& p = \w+\.p;|"
    r"\"[^\"]*\"\);|)$")


def _read(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def _body_lines(src, kernel):
    """Lines of the kernel's body, from the line after its opening brace."""
    m = re.search(r"__global__ void[^{;]*?\b" + kernel + r"\s*\(", src)
    assert m, f"{kernel} not found"
    return src[src.index("{", m.end()) + 1:].split("\n")


def test_every_dependent_kernel_waits_before_any_global_access():
    for kernel, fname in DEPENDENTS.items():
        lines = _body_lines(_read(fname), kernel)
        for i, line in enumerate(lines):
            if "grid_dependency_wait();" in line:
                break
            assert ALLOWED_BEFORE_WAIT.match(line), (
                f"{kernel}: statement before grid_dependency_wait(): {line.strip()!r}")
        else:
            raise AssertionError(f"{kernel}: no grid_dependency_wait()")
        assert i < 20, f"{kernel}: grid_dependency_wait() is not at the top"


def test_decode_sources_launch_only_with_attributes():
    for fname in sorted(set(DEPENDENTS.values())):
        src = _read(fname)
        assert "<<<" not in src, f"{fname} has a <<<...>>> launch"
        assert "cudaLaunchAttributeProgrammaticStreamSerialization" in src or \
            "launch_dependent(" in src, fname


def test_helpers_issue_the_ptx_they_name():
    src = _read("pa_common.cuh")
    wait = re.search(r"void grid_dependency_wait\(\)\s*\{([^}]*)\}", src)
    trig = re.search(r"void grid_dependents_may_launch\(\)\s*\{([^}]*)\}", src)
    assert wait and "griddepcontrol.wait;" in wait.group(1)
    assert trig and "griddepcontrol.launch_dependents;" in trig.group(1)
    launch = re.search(r"cudaError_t launch_dependent\((.*?)\n\}", src, re.S)
    assert launch and "cudaLaunchAttributeProgrammaticStreamSerialization" in launch.group(1)
    assert "programmaticStreamSerializationAllowed = 1" in launch.group(1)
