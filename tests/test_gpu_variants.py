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
from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
from oracle import prism_oracle as po
from tests.helpers import assert_close_attn, f64, selection_row_ok

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
    audio = None if inp["audio"] is None else inp["audio"].numpy().astype(np.float64)
    fixed = kw["fixed_shape"] - 1 if "fixed_shape" in kw else None
    ora = po.pipeline(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), wl.T, wl.H, wl.W, audio, wl.top_k, wl.top_p,
                      fixed_shape=fixed, sparsity=kw.get("sparsity"))
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, **kw)
    cu = lambda t: None if t is None else t.cuda()
    out = att.forward(cu(inp["q"]), cu(inp["k"]), cu(inp["v"]), cu(inp["audio"]))
    P.prism_device_status()
    lay = att.host_layout()
    np.testing.assert_array_equal(lay["shape_id"], ora["shape_id"])
    np.testing.assert_array_equal(lay["blocks"], ora["blocks"])
    if fixed is not None:
        assert (lay["shape_id"] == 3).all()
    nb = len(ora["blocks"])
    k_eff = po.top_k_from_sparsity(kw["sparsity"], nb) if "sparsity" in kw else wl.top_k
    rp_g, cols_g = att.host_csr()
    # the oracle's probabilities, from its own pooled vectors, for the near-tie check
    scale = ora["scale"]
    exact = total = 0
    for h in range(wl.heads):
        s = po.block_scores(ora["qbar"][h], ora["kbar"][h], scale)
        for i in range(nb):
            g = cols_g[h][rp_g[h, i]:rp_g[h, i + 1]]
            o = ora["cols"][h][ora["row_ptr"][h, i]:ora["row_ptr"][h, i + 1]]
            ex, ok = selection_row_ok(po.block_probabilities(s[i]), g, o, k_eff, wl.top_p)
            assert ok, (h, i, g, o)
            assert len(g) >= min(k_eff, nb)
            exact += ex
            total += 1
    assert exact >= 0.99 * total, f"{exact}/{total} rows bit-exact"
    bf = lambda t: f64(t.to(torch.bfloat16))
    pm = {n: po.permute(bf(inp[n]), ora["perm"]) for n in ("q", "k", "v", "dout")}
    O, _ = po.bsa_forward(pm["q"], pm["k"], pm["v"], ora["blocks"], rp_g, cols_g, scale)
    assert_close_attn(f64(out), po.unpermute(O, ora["perm"]), f"O ({mode})")
    dq, dk, dv = att.backward(cu(inp["dout"]))
    P.prism_device_status()
    gq, gk, gv = po.bsa_backward(pm["q"], pm["k"], pm["v"], pm["dout"], ora["blocks"], rp_g, cols_g, scale)
    for got, ref, w in ((dq, gq, "dQ"), (dk, gk, "dK"), (dv, gv, "dV")):
        assert_close_attn(f64(got), po.unpermute(ref, ora["perm"]), f"{w} ({mode})")
