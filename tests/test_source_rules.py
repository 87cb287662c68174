"""Static rules of the CUDA sources, checked on the CPU.

- Every kernel is launched with programmatic stream serialisation, so each
  must wait on its predecessor (grid_dep_sync) before anything else: a kernel
  that read or wrote global memory first could race the kernel before it.
  One kernel may skip that wait on purpose: the decode step's routed pass
  routes while the append kernel before it still runs (that append triggers
  it early), reading only what the append does not write; it starts with
  grid_dep_sync_unless(...) and waits before anything else.
- Every launch goes through launch_kernel (the one place that sets the launch
  attributes); no triple-chevron launches.
"""
import glob
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "long_context_misa_b200", "csrc")
SOURCES = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                 glob.glob(os.path.join(CSRC, "*.h")))


def _strip_comments(src: str) -> str:
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def _kernels(src: str):
    """(name, first statement of the body) of every __global__ definition."""
    for m in re.finditer(r"__global__", src):
        brace = src.index("{", m.end())
        head = src[m.end():brace]
        if ";" in head:  # a declaration, not a definition
            continue
        # the kernel's name: the identifier right before its parameter list
        names = [n for n in re.findall(r"([A-Za-z_]\w*)\s*\(", head) if n != "__launch_bounds__"]
        first = src[brace + 1:].lstrip().split(";", 1)[0].strip()
        yield (names[0] if names else "?"), first


def test_sources_found():
    assert any(p.endswith("topk.cu") for p in SOURCES)


EARLY_KERNELS = {"score_stream_kernel"}


@pytest.mark.parametrize("path", [p for p in SOURCES if p.endswith(".cu")], ids=os.path.basename)
def test_every_kernel_waits_on_its_predecessor_first(path):
    src = _strip_comments(open(path).read())
    kernels = list(_kernels(src))
    for name, first in kernels:
        ok = first in ("grid_dep_sync()", "misa::grid_dep_sync()") or (
            name in EARLY_KERNELS and first.startswith("grid_dep_sync_unless("))
        assert ok, f"{os.path.basename(path)}: kernel {name} starts with `{first}`"


def test_only_the_append_triggers_early():
    """griddepcontrol.launch_dependents is issued by the append kernel alone
    (its successor in the decode step is the early kernel above)."""
    users = []
    for p in SOURCES:
        src = _strip_comments(open(p).read())
        if "grid_dep_launch()" in src and not p.endswith("common.cuh"):
            users.append(os.path.basename(p))
    assert users == ["pool.cu"], users


def test_kernel_count():
    n = sum(len(list(_kernels(_strip_comments(open(p).read())))) for p in SOURCES if p.endswith(".cu"))
    assert n >= 19


@pytest.mark.parametrize("path", SOURCES, ids=os.path.basename)
def test_no_triple_chevron_launches(path):
    src = _strip_comments(open(path).read())
    assert "<<<" not in src, f"{os.path.basename(path)} launches a kernel outside launch_kernel"
