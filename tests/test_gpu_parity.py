"""GPU parity: each C-ABI step against the fp64 oracle on the same seeded inputs.

Discrete steps (block assignment, permutation, selection) are compared bit for
bit when both sides are fed the same fp32 values; attention outputs and
gradients against fp64 within rel-RMS 1e-2 and max-abs 3e-2.
"""

import math

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
from oracle import prism_oracle as po
from tests.helpers import (assert_close_attn, assert_dq_consistent, blocks_to_device, csr_to_device,
                           f64, selection_row_ok)

pytestmark = pytest.mark.gpu
CASES = ["tiny", "aniso8", "mix16", "smoke128"]
_CACHE = {}


def problem(name):
    """Seeded inputs (CPU) and the oracle's whole forward path on them."""
    if name not in _CACHE:
        wl = synth.get_workload(name)
        inp = synth.make_inputs(wl, "cpu", with_dout=True)
        a = None if inp["audio"] is None else inp["audio"].numpy().astype(np.float64)
        ora = po.pipeline(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), wl.T, wl.H, wl.W, a, wl.top_k, wl.top_p)
        _CACHE[name] = (wl, inp, ora)
    return _CACHE[name]


def make_att(wl, **kw):
    return PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, **kw)


def cuda(t):
    return None if t is None else t.cuda()


@pytest.mark.parametrize("name", CASES)
def test_indicator(name):
    wl, inp, ora = problem(name)
    att = make_att(wl)
    att.indicator(cuda(inp["v"]), cuda(inp["audio"]))
    ind = ora["ind"]
    np.testing.assert_allclose(f64(att.g), ind["g"], rtol=2e-4, atol=1e-6)
    np.testing.assert_allclose(f64(att.rho), ind["rho"], rtol=2e-4, atol=1e-6)
    dbg = f64(att.debug)
    np.testing.assert_allclose(dbg[:, :3], ind["sigma2_v"], rtol=2e-4, atol=1e-8)
    np.testing.assert_allclose(dbg[:, 3], ind["info"], rtol=2e-4, atol=1e-8)
    np.testing.assert_allclose(dbg[:, 4], ind["abar"], rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(dbg[:, 5:], ind["vhat_a"], rtol=1e-4, atol=1e-6)


def _assign_both(g32, rho32, T, H, W):
    Z = len(rho32)
    p = P.make_params(T, H, W, 1, 64, 1, 0.5)
    shape_id = torch.empty(Z, dtype=torch.uint8, device="cuda")
    zbb = torch.empty(Z + 1, dtype=torch.int32, device="cuda")
    blocks = torch.empty(8 * Z, 4, dtype=torch.int32, device="cuda")
    nblk = torch.empty(1, dtype=torch.int32, device="cuda")
    P.prism_assign_blocks(p, torch.from_numpy(g32).cuda(), torch.from_numpy(rho32).cuda(), shape_id, zbb, blocks,
                          nblk)
    sid_o, zbb_o, blocks_o = po.assign_blocks(g32.astype(np.float64), rho32.astype(np.float64), T, H, W)
    nb = int(nblk.item())
    assert nb == len(blocks_o)
    np.testing.assert_array_equal(shape_id.cpu().numpy(), sid_o)
    np.testing.assert_array_equal(zbb.cpu().numpy(), zbb_o)
    np.testing.assert_array_equal(blocks[:nb].cpu().numpy(), blocks_o)


@pytest.mark.parametrize("name", CASES)
def test_assign_blocks_bitexact(name):
    wl, inp, ora = problem(name)
    _assign_both(ora["ind"]["g"].astype(np.float32), ora["ind"]["rho"].astype(np.float32), wl.T, wl.H, wl.W)


def test_assign_blocks_ties_and_thresholds():
    """Isotropic indicators (exact 3-way distance ties), rho on the thresholds,
    and enough zones to span several scan chunks of the kernel."""
    rng = np.random.default_rng(30)
    T, H, W = 8, 8 * 40, 8 * 40            # 1600 zones
    Z = 1600
    g = rng.uniform(1e-4, 2.0, size=(Z, 3)).astype(np.float32)
    g[::5] = np.float32(0.37)
    g[1::7, 2] = g[1::7, 1]
    rho = rng.uniform(0, 1, size=Z).astype(np.float32)
    rho[::3] = np.float32(0.5)
    rho[1::11] = np.float32(0.25)
    rho[2::13] = np.nextafter(np.float32(0.25), np.float32(0))
    _assign_both(g, rho, T, H, W)


@pytest.mark.parametrize("name", CASES)
def test_permute_and_pool(name):
    wl, inp, ora = problem(name)
    att = make_att(wl)
    att.shape_id.copy_(torch.from_numpy(ora["shape_id"].astype(np.uint8)))
    att.zone_blk_base.copy_(torch.from_numpy(ora["zone_blk_base"].astype(np.int32)))
    q = cuda(inp["q"])
    P.prism_permute(att.p, att.shape_id, att.zone_blk_base, q, att.qp, att.qbar)
    # permuted values: the oracle's permutation of the input rounded to bf16 (exact for bf16 input)
    expect = torch.from_numpy(po.permute(inp["q"].float().numpy(), ora["perm"])).to(torch.bfloat16)
    assert torch.equal(att.qp.cpu(), expect)
    nb = len(ora["blocks"])
    np.testing.assert_allclose(f64(att.qbar[:, :nb]), ora["qbar"], rtol=1e-5, atol=1e-6)
    # inverse, in both output types
    back = torch.empty(wl.N, wl.heads, wl.head_dim, dtype=torch.bfloat16, device="cuda")
    P.prism_unpermute(att.p, att.shape_id, att.qp, back)
    assert torch.equal(back.cpu(), inp["q"].to(torch.bfloat16))
    back32 = torch.empty(wl.N, wl.heads, wl.head_dim, dtype=torch.float32, device="cuda")
    P.prism_unpermute(att.p, att.shape_id, att.qp, back32)
    assert torch.equal(back32.cpu(), inp["q"].to(torch.bfloat16).float())


@pytest.mark.parametrize("name", CASES)
def test_block_select_bitexact(name):
    """GPU and oracle select from the same fp32 pooled vectors."""
    wl, inp, ora = problem(name)
    att = make_att(wl)
    nb = len(ora["blocks"])
    q32 = ora["qbar"].astype(np.float32)
    k32 = ora["kbar"].astype(np.float32)
    att.qbar.zero_()
    att.kbar.zero_()
    att.qbar[:, :nb] = torch.from_numpy(q32).cuda()
    att.kbar[:, :nb] = torch.from_numpy(k32).cuda()
    att.nblk.fill_(nb)
    att.select()
    P.prism_device_status()
    rp_g, cols_g = att.host_csr()
    rp_o, cols_o, probs = po.block_select(q32.astype(np.float64), k32.astype(np.float64), wl.top_k, wl.top_p,
                                          1 / math.sqrt(wl.head_dim))
    exact = total = 0
    for h in range(wl.heads):
        for i in range(nb):
            g = cols_g[h][rp_g[h, i]:rp_g[h, i + 1]]
            o = cols_o[h][rp_o[h, i]:rp_o[h, i + 1]]
            ex, ok = selection_row_ok(probs[h][i], g, o, wl.top_k, wl.top_p)
            assert ok, (h, i, g, o)
            exact += ex
            total += 1
    assert exact >= 0.99 * total, f"{exact}/{total} rows bit-exact"


def _oracle_layout_on_gpu(att, ora, inp, wl):
    """Feed the oracle's layout, permuted bf16 tensors and CSR to the GPU buffers."""
    nb = len(ora["blocks"])
    att.shape_id.copy_(torch.from_numpy(ora["shape_id"].astype(np.uint8)))
    att.zone_blk_base.copy_(torch.from_numpy(ora["zone_blk_base"].astype(np.int32)))
    att.blocks.copy_(blocks_to_device(ora["blocks"], att.cap, "cuda"))
    att.nblk.fill_(nb)
    for name, dst in (("q", att.qp), ("k", att.kp), ("v", att.vp)):
        dst.copy_(torch.from_numpy(po.permute(inp[name].float().numpy(), ora["perm"])).to(torch.bfloat16))
    rp, col, nnz = csr_to_device(ora["row_ptr"], ora["cols"], att.cap, "cuda")
    att.row_ptr.copy_(rp)
    att.col[:col.numel()] = col
    att.nnz.copy_(nnz)
    bf = lambda t: f64(t.to(torch.bfloat16))
    return {n: po.permute(bf(inp[n]), ora["perm"]) for n in ("q", "k", "v", "dout")}


@pytest.mark.parametrize("name", CASES)
def test_bsa_forward(name):
    wl, inp, ora = problem(name)
    att = make_att(wl)
    pm = _oracle_layout_on_gpu(att, ora, inp, wl)
    att.attend()
    O, L = po.bsa_forward(pm["q"], pm["k"], pm["v"], ora["blocks"], ora["row_ptr"], ora["cols"], ora["scale"])
    assert_close_attn(f64(att.op), O, "O")
    np.testing.assert_allclose(f64(att.lse), L, rtol=0, atol=2e-2)


@pytest.mark.parametrize("name", CASES)
def test_bsa_backward(name):
    """The backward (one tensor-core kernel for head_dim 128, dQ by fp32
    reductions; warp-MMA kernels for head_dim 64) against the oracle."""
    wl, inp, ora = problem(name)
    att = make_att(wl)
    pm = _oracle_layout_on_gpu(att, ora, inp, wl)
    att.attend()
    b = att._bwd_buffers()
    b["dop"].copy_(torch.from_numpy(pm["dout"]).to(torch.bfloat16))
    att.attend_backward()
    P.prism_device_status()
    dq, dk, dv = po.bsa_backward(pm["q"], pm["k"], pm["v"], pm["dout"], ora["blocks"], ora["row_ptr"],
                                 ora["cols"], ora["scale"])
    assert_close_attn(f64(b["dqp"]), dq, "dQ")
    assert_close_attn(f64(b["dkp"]), dk, "dK")
    assert_close_attn(f64(b["dvp"]), dv, "dV")


@pytest.mark.parametrize("name", CASES)
def test_end_to_end(name):
    """The whole GPU path from natural inputs against the whole oracle path."""
    wl, inp, ora = problem(name)
    att = make_att(wl)
    out = att.forward(cuda(inp["q"]), cuda(inp["k"]), cuda(inp["v"]), cuda(inp["audio"]))
    P.prism_device_status()
    lay = att.host_layout()
    np.testing.assert_array_equal(lay["shape_id"], ora["shape_id"])
    np.testing.assert_array_equal(lay["blocks"], ora["blocks"])
    rp_g, cols_g = att.host_csr()
    same = all(np.array_equal(rp_g[h], ora["row_ptr"][h]) and np.array_equal(cols_g[h], ora["cols"][h])
               for h in range(wl.heads))
    if same:
        assert_close_attn(f64(out), ora["O"], "O end to end")
    else:
        # selections differ at near-ties only: rerun the oracle attention on the GPU's selection
        pm = {n: po.permute(f64(inp[n].to(torch.bfloat16)), ora["perm"]) for n in ("q", "k", "v")}
        O, _ = po.bsa_forward(pm["q"], pm["k"], pm["v"], ora["blocks"], rp_g, cols_g, ora["scale"])
        assert_close_attn(f64(out), po.unpermute(O, ora["perm"]), "O end to end (GPU selection)")
    dq, dk, dv = att.backward(cuda(inp["dout"]))
    P.prism_device_status()
    pm = {n: po.permute(f64(inp[n].to(torch.bfloat16)), ora["perm"]) for n in ("q", "k", "v", "dout")}
    gq, gk, gv = po.bsa_backward(pm["q"], pm["k"], pm["v"], pm["dout"], ora["blocks"], rp_g, cols_g, ora["scale"])
    for got, ref, w in ((dq, gq, "dQ"), (dk, gk, "dK"), (dv, gv, "dV")):
        assert_close_attn(f64(got), po.unpermute(ref, ora["perm"]), w + " end to end")


def test_top_k_all_is_dense_attention():
    """k >= nblk selects every block: the output is dense softmax attention
    (checked against torch SDPA in fp32 on the same bf16 inputs)."""
    wl = synth.get_workload("aniso8")
    inp = synth.make_inputs(wl, "cpu", with_dout=False)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, 10**6, 0.5)
    out = att.forward(cuda(inp["q"]), cuda(inp["k"]), cuda(inp["v"]), None)
    P.prism_device_status()
    q, k, v = (inp[n].to(torch.bfloat16).float().cuda().transpose(0, 1) for n in ("q", "k", "v"))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).transpose(0, 1)
    assert_close_attn(f64(out), f64(ref), "dense")


def test_capacity_overflow_is_reported_and_safe():
    wl = synth.get_workload("tiny")
    inp = synth.make_inputs(wl, "cpu", with_dout=False)
    att = make_att(wl, col_capacity=4)
    att.forward(cuda(inp["q"]), cuda(inp["k"]), cuda(inp["v"]), cuda(inp["audio"]))
    with pytest.raises(P.PrismError) as e:
        P.prism_device_status()
    assert e.value.code == P.PRISM_ECAPACITY
    assert int(att.nnz.item()) > 4
    assert int(att.row_ptr.max().item()) == 0     # every row left empty
    P.prism_device_status()                       # cleared


def test_tc_forward_matches_warp_mma_forward():
    """The tcgen05 forward (default for head_dim 128) and the warp-level MMA
    forward agree on the same layout and selection (both are also checked
    against the oracle above)."""
    wl, inp, ora = problem("mix16")
    outs = []
    for backend in (0, 1):
        P.prism_set_option(P.PRISM_OPT_ATTN_BACKEND, backend)
        try:
            att = make_att(wl)
            _oracle_layout_on_gpu(att, ora, inp, wl)
            att.attend()
            P.prism_device_status()
            outs.append((att.op.float().cpu(), att.lse.cpu(), att.op_res.float().cpu()))
        finally:
            P.prism_set_option(P.PRISM_OPT_ATTN_BACKEND, 0)
    (o0, l0, r0), (o1, l1, r1) = outs
    assert_close_attn(o0.double().numpy(), o1.double().numpy(), "O tc vs mma")
    assert float((l0 - l1).abs().max()) <= 1e-3
    assert_close_attn((o0 + r0).double().numpy(), (o1 + r1).double().numpy(), "O+residual tc vs mma")


def test_forward_v_scale_is_exact():
    """The tensor-core forward takes V as fp16 scaled by a power of two per
    head, chosen from the head's max |v|.  V times 2^k gives the same fp16
    operand, so O and its residual scale by exactly 2^k and LSE is unchanged,
    with max |v| anywhere from about 2^-57 to 2^63; a head whose V is all
    zero gives O = 0 and a zero residual."""
    wl, inp, ora = problem("mix16")
    att = make_att(wl)
    _oracle_layout_on_gpu(att, ora, inp, wl)
    v0 = att.vp.clone()
    att.attend()
    P.prism_device_status()
    o_ref, r_ref, l_ref = att.op.float().clone(), att.op_res.float().clone(), att.lse.clone()
    assert float(o_ref.abs().max()) > 0.1
    for k in (-60, -20, 7, 60):
        att.vp.copy_((v0.float() * 2.0 ** k).to(torch.bfloat16))
        att.attend()
        P.prism_device_status()
        assert torch.equal(att.op.float(), o_ref * 2.0 ** k), k
        assert torch.equal(att.op_res.float(), r_ref * 2.0 ** k), k
        assert torch.equal(att.lse, l_ref), k
    att.vp.copy_(v0)
    att.vp[1].zero_()
    att.attend()
    P.prism_device_status()
    assert torch.equal(att.op[1].float(), torch.zeros_like(o_ref[1]))
    assert torch.equal(att.op_res[1].float(), torch.zeros_like(r_ref[1]))
    assert torch.equal(att.op[0].float(), o_ref[0]) and torch.equal(att.op[2].float(), o_ref[2])


def test_backward_runs_reproduce_dk_dv_and_agree_on_dq():
    """Three runs of the tensor-core backward on the same layout, selection
    and forward: dK and dV bit for bit (each accumulates in tensor memory in
    a fixed order), dQ within the spread of its fp32 reduction order."""
    wl, inp, ora = problem("mix16")
    att = make_att(wl)
    pm = _oracle_layout_on_gpu(att, ora, inp, wl)
    att.attend()
    b = att._bwd_buffers()
    b["dop"].copy_(torch.from_numpy(pm["dout"]).to(torch.bfloat16))
    runs = []
    for _ in range(3):
        att.attend_backward()
        P.prism_device_status()
        runs.append({n: b[n].clone() for n in ("dqp", "dkp", "dvp")})
    for run in runs[1:]:
        assert torch.equal(run["dkp"], runs[0]["dkp"])
        assert torch.equal(run["dvp"], runs[0]["dvp"])
        assert_dq_consistent(run["dqp"], runs[0]["dqp"])
