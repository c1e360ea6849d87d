"""GPU parity on the degenerate cases of the method, each against the oracle.

A grid of one macro-zone; a value field with no variance and audio norms that
are all zero (the indicator's every ratio is 0 and g = eps on all axes); k = 1
with a vanishing p (one key block per query block, the most probable); p = 1
(every key block: dense attention); and the README's ratio at its extreme.
"""

import dataclasses

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from oracle import prism_oracle as po
from tests.helpers import check_whole_path, f64

pytestmark = pytest.mark.gpu


def _wl(T, H, W, heads, d, k, p, index):
    return synth.Workload("edge", T, H, W, heads, d, "bf16", k, p, 2, 0.2, False, 1.0, index)


def test_single_zone_grid():
    wl = _wl(8, 8, 8, 1, 128, 1, 0.5, 30)
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    att, ora, _ = check_whole_path(wl, inp)
    assert att.host_layout()["nblk"] in (2, 4, 8)


def test_constant_values_and_silent_audio():
    """V constant: every axis variance is 0, so r = 0; audio all zero: abar = vhat = 0;
    g = eps exactly, rho = 0, every zone takes B = 256 and the isotropic shape (4,8,8)."""
    wl = _wl(16, 16, 24, 2, 128, 2, 0.9, 31)
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    inp["v"] = torch.full_like(inp["v"], 0.75)
    zero_audio = torch.zeros_like(inp["audio"])
    # dP_rc = dO_r . v is the same for every key c and equals D_r, so dS = 0:
    # dQ and dK are exactly zero
    att, ora, out = check_whole_path(wl, inp, audio=zero_audio, zero_grads=("dQ", "dK"))
    eps32 = np.float32(1e-4)
    assert (att.g.cpu().numpy() == eps32).all() and (att.rho.cpu().numpy() == 0).all()
    assert (ora["shape_id"] == 13).all() and po.SHAPES[13] == (4, 8, 8)
    # every output row is a convex combination of identical rows of V
    np.testing.assert_allclose(f64(out), 0.75, atol=2e-3)


def test_one_block_per_query_block():
    """k = 1 and p vanishing: S_i is the single most probable key block."""
    wl = _wl(16, 16, 16, 2, 128, 1, 1e-6, 32)
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    att, ora, _ = check_whole_path(wl, inp)
    rp, _ = att.host_csr()
    assert (np.diff(rp, axis=1) == 1).all()


def test_top_p_one_is_dense_attention():
    """p = 1 keeps every key block (only the whole row has mass 1), so the
    output is dense softmax attention over the grid."""
    wl = _wl(8, 16, 16, 2, 128, 1, 1.0, 33)
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    att, ora, _ = check_whole_path(wl, inp)
    rp, _ = att.host_csr()
    nb = att.host_layout()["nblk"]
    assert (np.diff(rp, axis=1) == nb).all()


def test_sparsity_one_keeps_at_least_one_block():
    """The README ratio at its extreme (skip every block): k = max(1, 0) = 1."""
    wl = _wl(8, 16, 24, 2, 64, 1, 1e-6, 34)
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    att, _, _ = check_whole_path(wl, inp, att_kw=dict(sparsity=1.0), ora_kw=dict(sparsity=1.0))
    rp, _ = att.host_csr()
    assert (np.diff(rp, axis=1) == 1).all()
