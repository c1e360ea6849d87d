"""The head-sharded layer on one GPU.

(1) Every rank's stages driven in one process, the exchanges done by slicing:
the decomposition (slab records -> whole-grid g and rho, slab and whole-grid
layouts, slab permutation, head groups) must give bit for bit the unsharded
layer's O, dK, dV, since every kernel works per zone or per head, and its dQ
to within the spread of the fp32 reduction order that sums dQ.
(2) The layer through TorchDistExchange with a one-rank NCCL group.
(3) The emulated two-rank layer against the fp64 oracle on the same seeded
inputs: the whole grid's g and rho on every rank, the block layout exactly,
every selection row exact or a valid near-tie alternative, and O, dQ, dK, dV
within rel-RMS 1e-2 and max-abs 3e-2 (beyond half a bf16 ulp).
"""

import os
import socket

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
from dynamic_block_sparse_variance_b200.sharded import ShardedPrismAttention, TorchDistExchange
from oracle import prism_oracle as po
from tests.helpers import assert_close_attn, assert_dq_consistent, f64, selection_row_ok

pytestmark = pytest.mark.gpu


def _workload():
    # 4 zone layers in T, 4 heads: shardable over 2 and 4 ranks, every block volume present
    return synth.Workload("shard", 32, 16, 24, 4, 128, "bf16", 3, 0.9, 3, 0.15, True, 1.0, 40)


def _unsharded(wl, inp):
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p)
    o = att.forward(inp["q"], inp["k"], inp["v"], inp["audio"])
    dq, dk, dv = att.backward(inp["dout"])
    P.prism_device_status()
    return [o, dq, dk, dv]


def _emulated(wl, inp, R, ranks=None):
    sh = [ShardedPrismAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, rank=r, world=R)
          for r in range(R)]
    Nl, hpr = sh[0].Nl, sh[0].hpr
    sl = lambda x, r: None if x is None else x[r * Nl:(r + 1) * Nl]
    for r, s in enumerate(sh):
        s.stage_records(sl(inp["v"], r), sl(inp["audio"], r))
    rec = torch.cat([s.rec_loc for s in sh])
    for r, s in enumerate(sh):
        s.rec_all.copy_(rec)
        s.stage_layout()
        s.stage_permute(sl(inp["q"], r), sl(inp["k"], r), sl(inp["v"], r))

    def seq_to_heads(get_loc, get_h, rows):
        for g in range(R):
            for s in range(R):
                r0, n = rows(sh[s], s)
                for hh in range(hpr):
                    get_h(sh[g])[hh, r0:r0 + n] = get_loc(sh[s])[g * hpr + hh, :n]

    def heads_to_seq(get_h, get_loc, rows):
        for g in range(R):
            for s in range(R):
                r0, n = rows(sh[s], s)
                for hh in range(hpr):
                    get_loc(sh[s])[g * hpr + hh, :n] = get_h(sh[g])[hh, r0:r0 + n]

    tok = lambda s, r: (r * Nl, Nl)
    blk = lambda s, r: s.slab_blocks[r]
    seq_to_heads(lambda s: s.qp, lambda s: s.inner.qp, tok)
    seq_to_heads(lambda s: s.kp, lambda s: s.inner.kp, tok)
    seq_to_heads(lambda s: s.vp, lambda s: s.inner.vp, tok)
    seq_to_heads(lambda s: s.qbar, lambda s: s.inner.qbar, blk)
    seq_to_heads(lambda s: s.kbar, lambda s: s.inner.kbar, blk)
    for s in sh:
        s.stage_attend()
    heads_to_seq(lambda s: s.inner.op, lambda s: s.qp, tok)
    outs = {n: [] for n in ("o", "dq", "dk", "dv")}
    for r, s in enumerate(sh):
        o = torch.empty(Nl, wl.heads, wl.head_dim, dtype=torch.bfloat16, device="cuda")
        s.stage_unpermute(s.qp, o)
        outs["o"].append(o)
        s.stage_permute_dout(sl(inp["dout"], r), s.kp)
    seq_to_heads(lambda s: s.kp, lambda s: s.inner._bwd_buffers()["dop"], tok)
    for s in sh:
        s.inner.attend_backward()
    for n in ("dq", "dk", "dv"):
        heads_to_seq(lambda s: s.inner._bwd_buffers()[n + "p"], lambda s: s.vp, tok)
        for s in sh:
            x = torch.empty(Nl, wl.heads, wl.head_dim, dtype=torch.bfloat16, device="cuda")
            s.stage_unpermute(s.vp, x)
            outs[n].append(x)
    P.prism_device_status()
    if ranks is not None:
        ranks.extend(sh)
    return [torch.cat(outs[n]) for n in ("o", "dq", "dk", "dv")]


@pytest.mark.parametrize("R", [2, 4])
def test_emulated_ranks_equal_the_unsharded_layer(R):
    wl = _workload()
    inp = synth.make_inputs(wl, "cuda", with_dout=True)
    ref = _unsharded(wl, inp)
    got = _emulated(wl, inp, R)
    for name, a, b in zip(("O", "dQ", "dK", "dV"), got, ref):
        if name == "dQ":
            assert_dq_consistent(a, b)
        else:
            assert torch.equal(a, b), name


def test_one_rank_nccl_group_equals_the_unsharded_layer():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = _workload()
        inp = synth.make_inputs(wl, "cuda", with_dout=True)
        ref = _unsharded(wl, inp)
        layer = ShardedPrismAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p, rank=0,
                                      world=1, exchange=TorchDistExchange(0, 1))
        o = layer.forward(inp["q"], inp["k"], inp["v"], inp["audio"])
        dq, dk, dv = layer.backward(inp["dout"])
        P.prism_device_status()
        for name, a, b in zip(("O", "dQ", "dK", "dV"), (o, dq, dk, dv), ref):
            if name == "dQ":
                assert_dq_consistent(a, b)
            else:
                assert torch.equal(a, b), name
    finally:
        dist.destroy_process_group()


def test_emulated_ranks_against_the_oracle():
    wl = _workload()
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    cu = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    sh = []
    o, dq, dk, dv = _emulated(wl, cu, 2, ranks=sh)
    a64 = inp["audio"].numpy().astype(np.float64)
    ora = po.pipeline(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), wl.T, wl.H, wl.W, a64, wl.top_k, wl.top_p)
    for s in sh:   # every rank finalised the whole grid from the gathered slab records
        np.testing.assert_allclose(f64(s.inner.g), ora["ind"]["g"], rtol=2e-4, atol=1e-6)
        np.testing.assert_allclose(f64(s.inner.rho), ora["ind"]["rho"], rtol=2e-4, atol=1e-6)
        lay = s.inner.host_layout()
        np.testing.assert_array_equal(lay["shape_id"], ora["shape_id"])
        np.testing.assert_array_equal(lay["blocks"], ora["blocks"])
    # the head groups' selections, as one per-head CSR
    nb = len(ora["blocks"])
    rp_g, cols_g = [], []
    for s in sh:
        rp, cols = s.inner.host_csr()
        rp_g += list(rp)
        cols_g += cols
    rp_g = np.stack(rp_g)
    exact = 0
    for h in range(wl.heads):
        S = po.block_scores(ora["qbar"][h], ora["kbar"][h], ora["scale"])
        for i in range(nb):
            g = cols_g[h][rp_g[h, i]:rp_g[h, i + 1]]
            r = ora["cols"][h][ora["row_ptr"][h, i]:ora["row_ptr"][h, i + 1]]
            ex, ok = selection_row_ok(po.block_probabilities(S[i]), g, r, wl.top_k, wl.top_p)
            assert ok, (h, i, g, r)
            exact += ex
    assert exact >= 0.99 * wl.heads * nb
    # attention on the selection the ranks made
    pm = {n: po.permute(f64(inp[n].to(torch.bfloat16)), ora["perm"]) for n in ("q", "k", "v", "dout")}
    O, _ = po.bsa_forward(pm["q"], pm["k"], pm["v"], ora["blocks"], rp_g, cols_g, ora["scale"])
    assert_close_attn(f64(o), po.unpermute(O, ora["perm"]), "sharded O")
    gq, gk, gv = po.bsa_backward(pm["q"], pm["k"], pm["v"], pm["dout"], ora["blocks"], rp_g, cols_g, ora["scale"])
    for got, ref, w in ((dq, gq, "dQ"), (dk, gk, "dK"), (dv, gv, "dV")):
        assert_close_attn(f64(got), po.unpermute(ref, ora["perm"]), "sharded " + w)
