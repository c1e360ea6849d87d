"""Static checks of the tensor-core kernel sources (CPU, no GPU).

Every mbarrier a kernel declares in its shared-memory barrier area must be
initialised exactly once by that kernel: a wait or an arrive on an
uninitialised barrier is undefined behaviour on the device, and a second
initialisation of a live barrier loses its phase.
"""

import pathlib
import re

import pytest

CSRC = pathlib.Path(__file__).resolve().parents[1] / "dynamic_block_sparse_variance_b200" / "csrc"
SOURCES = ["attn_tc_fwd.cuh", "attn_tc_bwd.cuh"]


def _kernels(text):
    starts = [m.start() for m in re.finditer(r"__global__ void", text)]
    for a, b in zip(starts, starts[1:] + [len(text)]):
        body = text[a:b]
        name = re.search(r"(\w+)\s*\(", body[body.index("void") + 4:]).group(1)
        yield name, body


def _barrier_inits(body):
    declared = set(re.findall(r"const uint32_t (b_\w+) = sBar", body))
    declared |= set(re.findall(r"auto (b_\w+) = \[&\]\(int \w+\) \{ return sBar", body))
    inits = re.findall(r"mbar_init\((b_\w+)", body)
    return declared, inits


@pytest.mark.parametrize("src", SOURCES)
def test_every_declared_barrier_is_initialised_once(src):
    text = (CSRC / src).read_text()
    seen = 0
    for name, body in _kernels(text):
        declared, inits = _barrier_inits(body)
        if not declared:
            continue
        seen += 1
        for b in declared:
            assert inits.count(b) == 1, f"{src}:{name}: barrier {b} initialised {inits.count(b)} times"
        for b in set(inits):
            assert b in declared, f"{src}:{name}: initialises undeclared barrier {b}"
    assert seen >= 1


def test_no_cluster_multicast():
    """The library issues no copy with cluster multicast (the kernels may run
    beside peer-memory code on multi-GPU nodes)."""
    for path in CSRC.glob("*.cu*"):
        assert ".multicast::cluster" not in path.read_text(), path.name


def test_every_launch_is_traced():
    """Every kernel launch of the library sits inside a PRISM_TRACED statement, so
    the launch hook (per-kernel CUDA events, the bench's launch count) sees all of
    them and a rejected launch fails the call at once."""
    for path in sorted(CSRC.glob("*.cu*")):
        text = path.read_text()
        for m in re.finditer(r"<<<", text):
            stmt_start = max(text.rfind(";", 0, m.start()), text.rfind("{", 0, m.start()),
                             text.rfind("}", 0, m.start()))
            assert "PRISM_TRACED(" in text[stmt_start:m.start()], f"{path.name}: untraced launch at {m.start()}"
