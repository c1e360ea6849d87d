"""The allocation-free indicator entry point against the workspace one.

prism_zone_indicator_noalloc keeps its scratch in a fixed array inside the
library, for callers that cannot allocate device memory when they call (a
plugin handed only its input and output buffers, an allocator-free runtime).
It is called here through the C ABI twice in a row on the same inputs; each
result must match prism_zone_indicator's within the indicator tolerance.  This
file runs last so that a failure here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth

pytestmark = pytest.mark.gpu


def _run_workspace_version(p, v, audio, Z):
    ind, _ = P.prism_workspace_size(p, P.PRISM_WS_INDICATOR)
    ws = torch.empty(ind, dtype=torch.uint8, device="cuda")
    g = torch.empty(Z, 3, device="cuda")
    rho = torch.empty(Z, device="cuda")
    dbg = torch.empty(Z, 8, device="cuda")
    P.prism_zone_indicator(p, v, audio, g, rho, dbg, ws)
    torch.cuda.synchronize()
    return g.cpu().numpy(), rho.cpu().numpy(), dbg.cpu().numpy()


def _check_noalloc(name):
    wl = synth.get_workload(name)
    gen = "cpu" if name == "mix16" else "cuda"
    inp = synth.make_inputs(wl, gen, with_dout=False)
    v = inp["v"].cuda()
    audio = inp["audio"].cuda()
    p = P.make_params(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p)
    g_ref, rho_ref, dbg_ref = _run_workspace_version(p, v, audio, wl.zones)
    lib = P.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):   # two calls in a row share the fixed scratch
        g = torch.full((wl.zones, 3), float("nan"), device="cuda")
        rho = torch.full((wl.zones,), float("nan"), device="cuda")
        dbg = torch.full((wl.zones, 8), float("nan"), device="cuda")
        rc = lib.prism_zone_indicator_noalloc(ctypes.byref(p), ctypes.c_void_p(v.data_ptr()), P.PRISM_BF16,
                                              ctypes.c_void_p(audio.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                                              ctypes.c_void_p(rho.data_ptr()), ctypes.c_void_p(dbg.data_ptr()), stream)
        assert rc == P.PRISM_OK, lib.prism_last_error()
        P.prism_device_status()
        np.testing.assert_allclose(g.cpu().numpy(), g_ref, rtol=2e-4, atol=1e-6)
        np.testing.assert_allclose(rho.cpu().numpy(), rho_ref, rtol=2e-4, atol=1e-6)
        np.testing.assert_allclose(dbg.cpu().numpy(), dbg_ref, rtol=2e-4, atol=1e-8)


@pytest.mark.parametrize("name", ["mix16", "720p"])
def test_noalloc_indicator_matches_workspace_indicator(name):
    _check_noalloc(name)


def test_noalloc_indicator_smaller_grid_after_a_larger_one():
    """The array keeps what the last call left in it: a small grid run after a
    large one must read none of the large grid's partial sums."""
    _check_noalloc("720p")
    _check_noalloc("mix16")


def test_noalloc_indicator_rejects_grids_beyond_its_scratch():
    lib = P.lib()
    p = P.make_params(8, 8 * 72, 8 * 64, 1, 64, 1, 0.5)   # 4608 zones > the 4096-zone limit
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.prism_zone_indicator_noalloc(ctypes.byref(p), fake, P.PRISM_BF16, None, fake, fake, None, None)
    assert rc == P.PRISM_EINVAL
    assert b"scratch" in lib.prism_last_error()
