"""GPU parity of the README's variants and of the audio-norm producer.

The variants come from the Prism repository's configuration table: the fixed
4x4x4 block mode (dynamic block shapes switched off) and the ratio form of k
(bsa_sparsity).  Each runs the whole path on the GPU and is compared with the
oracle run in the same mode: block layout bit for bit, selections exactly (or
a valid alternative at a near-tie), attention outputs and gradients within
rel-RMS 1e-2 and max-abs 3e-2 beyond half a bf16 ulp.  The audio norms
a = ||h||_2 are compared with the oracle within the float summation bound.
"""

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from oracle import prism_oracle as po
from tests.helpers import check_whole_path, f64

pytestmark = pytest.mark.gpu

# Squares summed in float: along any path of the kernel's summation (a lane's
# four accumulator chains of 16-byte vectors, their pairwise sum, a 5-level
# butterfly) there are fewer than 45 roundings for every channel count used
# here (C in {4, 8, 64, 1024, 3072}: at most 3 full rounds of 9), so the sum of
# positive terms is within 45 * 2^-24 (2.7e-6) relative; the square root
# halves that and adds half an ulp.
NORM_RTOL = 4e-6


def _norm_input(N, C, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(N, C, generator=g) * torch.exp(2 * torch.randn(N, 1, generator=g))
    if N > 2:
        h[1] = 0.0                       # a zero row: exactly 0
        h[2] = 300.0                     # a constant row: 300 sqrt(C)
    return h.to(dtype)


@pytest.mark.parametrize("dtype,N,C", [(torch.bfloat16, 2053, 3072), (torch.float32, 1001, 64),
                                       (torch.bfloat16, 7, 8), (torch.float32, 33, 4),
                                       (torch.bfloat16, 4099, 1024)])
def test_audio_norms_against_oracle(dtype, N, C):
    h = _norm_input(N, C, dtype, seed=N + C)
    a = torch.full((N,), -1.0, device="cuda")
    P.prism_audio_norms(h.cuda(), a)
    P.prism_device_status()
    ref = po.audio_norms(f64(h))
    got = a.cpu().double().numpy()
    np.testing.assert_allclose(got, ref, rtol=NORM_RTOL, atol=0)
    if N > 2:
        assert got[1] == 0.0


def test_audio_norms_empty_launches_nothing():
    a = torch.full((4,), -1.0, device="cuda")
    P.prism_audio_norms(torch.empty(0, 3072, dtype=torch.bfloat16, device="cuda"), a)
    P.prism_device_status()
    assert (a == -1.0).all()


def test_audio_norms_full_size_sampled():
    """The 2K-like grid's token count with 24 x 128 channels (6 GB in bf16),
    checked on sampled rows and on the last one."""
    N, C = 64 * 96 * 160, 24 * 128
    g = torch.Generator(device="cuda").manual_seed(5)
    h = torch.randn(N, C, device="cuda", dtype=torch.bfloat16, generator=g)
    a = torch.empty(N, device="cuda")
    P.prism_audio_norms(h, a)
    P.prism_device_status()
    rows = np.unique(np.concatenate([np.random.default_rng(0).integers(0, N, 512), [0, N - 1]]))
    idx = torch.from_numpy(rows).cuda()
    ref = po.audio_norms(f64(h[idx]))
    np.testing.assert_allclose(a[idx].cpu().double().numpy(), ref, rtol=NORM_RTOL, atol=0)


MODES = {
    "fixed444": dict(fixed_shape=P.PRISM_FIXED_444),
    "ratio": dict(sparsity=0.75),
    "fixed444+ratio": dict(fixed_shape=P.PRISM_FIXED_444, sparsity=0.85),
}


@pytest.mark.parametrize("name,mode", [("aniso8", "fixed444"), ("aniso8", "ratio"), ("aniso8", "fixed444+ratio"),
                                       ("mix16", "ratio"), ("mix16", "fixed444+ratio")])
def test_variant_end_to_end(name, mode):
    kw = MODES[mode]
    wl = synth.get_workload(name)
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    fixed = kw["fixed_shape"] - 1 if "fixed_shape" in kw else None
    att, _, _ = check_whole_path(wl, inp, att_kw=kw, ora_kw=dict(fixed_shape=fixed, sparsity=kw.get("sparsity")))
    if fixed is not None:
        assert (att.host_layout()["shape_id"] == 3).all()


@pytest.mark.parametrize("name", ["aniso8", "mix16"])
def test_inference_reuses_layout_and_selection(name):
    """forward_reuse on the inputs of a later step attends over the selection the
    first step chose: the oracle's attention on the new inputs with the first
    step's layout and CSR is the reference."""
    from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
    from tests.helpers import assert_close_attn
    wl = synth.get_workload(name)
    first = synth.make_inputs(wl, "cpu", with_dout=False)
    g = torch.Generator().manual_seed(77)
    later = {n: (first[n].float() + 0.3 * torch.randn(first[n].shape, generator=g)).to(first[n].dtype)
             for n in ("q", "k", "v")}
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, training=False)
    cu = lambda t: None if t is None else t.cuda()
    att.forward(cu(first["q"]), cu(first["k"]), cu(first["v"]), cu(first["audio"]))
    lay0, csr0 = att.host_layout(), att.host_csr()
    out = att.forward_reuse(cu(later["q"]), cu(later["k"]), cu(later["v"]))
    P.prism_device_status()
    lay1, csr1 = att.host_layout(), att.host_csr()
    np.testing.assert_array_equal(lay0["blocks"], lay1["blocks"])
    for a, b in zip(csr0[1], csr1[1]):
        np.testing.assert_array_equal(a, b)
    perm = po.permutation(wl.T, wl.H, wl.W, lay0["shape_id"])
    pm = {n: po.permute(f64(later[n].to(torch.bfloat16)), perm) for n in ("q", "k", "v")}
    O, _ = po.bsa_forward(pm["q"], pm["k"], pm["v"], lay0["blocks"].astype(np.int64), csr0[0], csr0[1],
                          1.0 / np.sqrt(wl.head_dim))
    assert_close_attn(f64(out), po.unpermute(O, perm), "O with the reused selection")
