"""Parity at the full benchmark grids (Small, 720p, 1080p, 2K), on sampled outputs.

The GPU runs the whole path in the launch configuration bench.py times (one
PrismSparseAttention layer over all heads).  The fp64 oracle then works from
the same inputs on its own: the indicator and block layout of the whole grid,
the selection of sampled query blocks (and of every query block of one head,
for the exact selectors of sampled key blocks), and the outputs those samples
determine: O and LSE and dQ of sampled query blocks, dK and dV of sampled key
blocks.  Query blocks are drawn from a few heads, stratified by block volume
(at 1080p and 2K: 256 (head, block) pairs); key blocks are the two with the
fewest selectors and the one at the median selector count (below 2K also the
90th percentile and the maximum), each checked against every query block that
selects it.
Discrete results are compared exactly (selections up to near-ties); attention
outputs within rel-RMS 1e-2, max-abs 3e-2 beyond half a bf16 ulp and raw
max-abs 3e-2 where |ref| < 2.
"""

import math
import os
import time

import numpy as np
import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
from oracle import prism_oracle as po
from tests.helpers import assert_close_attn, selection_row_ok

pytestmark = pytest.mark.gpu

# heads drawn for the query-side samples, and query blocks per head (a third per volume)
QUERY_HEADS = {"small": 2, "720p": 2, "1080p": 4, "2k": 4}
QUERY_PER_HEAD = {"small": 12, "720p": 12, "1080p": 64, "2k": 64}


def _phase(name, what, t0):
    """Seconds since t0, appended to PRISM_PARITY_LOG (when set) as a timing line."""
    log = os.environ.get("PRISM_PARITY_LOG")
    if log:
        with open(log, "a") as fh:
            fh.write(f"timing\t{name}\t{what}\t{time.perf_counter() - t0:.1f}s\n")
    return time.perf_counter()


def _head(x_cpu, h, perm):
    """Head h of a natural-layout CPU tensor, permuted, as [1, N, d] float64."""
    return x_cpu[:, h, :].double().numpy()[perm][None]


def _stratified(rng, sizes, count):
    """About count // 3 query blocks of each volume present (more of the others
    when a volume has too few blocks), without repeats."""
    vols = [B for B in (64, 128, 256) if (sizes == B).any()]
    picks = []
    for n, B in enumerate(vols):
        cand = np.setdiff1d(np.flatnonzero(sizes == B), picks)
        want = (count - len(picks)) // (len(vols) - n)
        picks += [int(c) for c in rng.choice(cand, size=min(len(cand), want), replace=False)]
    return picks


@pytest.mark.parametrize("name", ["small", "720p", "1080p", "2k"])
def test_fullsize_sampled_parity(name):
    t0 = time.perf_counter()
    wl = synth.get_workload(name)
    inp = synth.make_inputs(wl, "cuda", with_dout=wl.backward)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p)
    att.forward(inp["q"], inp["k"], inp["v"], inp["audio"])
    if wl.backward:
        att.backward(inp["dout"])
    P.prism_device_status()
    lay = att.host_layout()
    g_gpu, rho_gpu = att.g.cpu().numpy(), att.rho.cpu().numpy()
    rp_gpu, cols_gpu = att.host_csr()
    cpu = {n: (None if inp[n] is None else inp[n].cpu()) for n in inp}
    del inp
    t0 = _phase(name, "gpu path and host copies", t0)

    # ---- oracle: indicator and layout of the whole grid
    v32 = cpu["v"].float().numpy()
    audio = cpu["audio"].double().numpy()
    ind = po.zone_indicator(v32, wl.T, wl.H, wl.W, audio)
    del v32
    np.testing.assert_allclose(g_gpu, ind["g"], rtol=2e-4, atol=1e-6)
    np.testing.assert_allclose(rho_gpu, ind["rho"], rtol=2e-4, atol=1e-6)
    shape_id, base, blocks = po.assign_blocks(ind["g"], ind["rho"], wl.T, wl.H, wl.W)
    np.testing.assert_array_equal(lay["shape_id"], shape_id)
    np.testing.assert_array_equal(lay["blocks"], blocks)
    perm = po.permutation(wl.T, wl.H, wl.W, shape_id)
    nb = len(blocks)
    scale = 1.0 / math.sqrt(wl.head_dim)
    rng = np.random.default_rng(7)
    bwd = att._bwd if wl.backward else None
    t0 = _phase(name, "oracle indicator and layout", t0)

    # ---- sampled query blocks: a few heads, stratified by block volume
    heads = sorted(int(h) for h in rng.choice(wl.heads, size=QUERY_HEADS[name], replace=False))
    sampled = exact = 0
    for h in heads:
        picks = _stratified(rng, blocks[:, 1], QUERY_PER_HEAD[name])
        q32, k32 = (cpu[n][:, h:h + 1, :].float().numpy() for n in ("q", "k"))
        kbar = po.pool_blocks_natural(k32, perm, blocks)[0]
        qbar = po.pool_blocks_natural(q32, perm, blocks[picks])[0]
        S = po.block_scores(qbar, kbar, scale)
        rows = []      # (block, oracle selection) of the rows selected exactly alike
        for r, i in enumerate(picks):
            prob = po.block_probabilities(S[r])
            sel_o = po.select_row(prob, wl.top_k, wl.top_p)
            sel_g = cols_gpu[h][rp_gpu[h, i]:rp_gpu[h, i + 1]]
            ex, ok = selection_row_ok(prob, sel_g, sel_o, wl.top_k, wl.top_p)
            assert ok, (name, h, i)
            sampled += 1
            exact += ex
            if ex:     # a valid near-tie alternative changes the outputs legitimately
                rows.append((i, sel_o))
        row_ptr = np.zeros((1, nb + 1), dtype=np.int64)
        cnt = np.zeros(nb, dtype=np.int64)
        for i, sel in rows:
            cnt[i] = len(sel)
        row_ptr[0, 1:] = np.cumsum(cnt)
        flat = np.concatenate([sel for _, sel in sorted(rows, key=lambda t: t[0])])
        qh, kh, vh = (_head(cpu[n], h, perm) for n in ("q", "k", "v"))
        done = [i for i, _ in rows]
        O, L = po.bsa_forward(qh, kh, vh, blocks, row_ptr, [flat], scale, query_blocks=done)
        gq = po.bsa_query_block_dq(qh, kh, vh, _head(cpu["dout"], h, perm), blocks, row_ptr, [flat], scale,
                                   done) if wl.backward else None
        for i in done:
            s0, sz = blocks[i][0], blocks[i][1]
            assert_close_attn(att.op[h, s0:s0 + sz].double().cpu().numpy(), O[0, s0:s0 + sz], f"{name} O h{h} b{i}")
            np.testing.assert_allclose(att.lse[h, s0:s0 + sz].double().cpu().numpy(), L[0, s0:s0 + sz], atol=2e-2)
            if wl.backward:
                assert_close_attn(bwd["dqp"][h, s0:s0 + sz].double().cpu().numpy(), gq[i], f"{name} dQ h{h} b{i}")
        del qh, kh, vh, O, L
    assert exact >= 0.98 * sampled, f"{exact}/{sampled} sampled selections bit-exact"
    t0 = _phase(name, f"{sampled} sampled query blocks", t0)

    # ---- dK, dV of sampled key blocks: the oracle selects every row of one head
    if wl.backward:
        h = heads[0]
        q32, k32 = (cpu[n][:, h:h + 1, :].float().numpy() for n in ("q", "k"))
        S = po.block_scores(po.pool_blocks_natural(q32, perm, blocks)[0],
                            po.pool_blocks_natural(k32, perm, blocks)[0], scale)
        rp_o = np.zeros((1, nb + 1), dtype=np.int64)
        cols_o = []
        sel_of_o, sel_of_g = {}, {}
        mismatch = 0
        for i in range(nb):
            prob = po.block_probabilities(S[i])
            sel_o = po.select_row(prob, wl.top_k, wl.top_p)
            sel_g = cols_gpu[h][rp_gpu[h, i]:rp_gpu[h, i + 1]]
            ex, ok = selection_row_ok(prob, sel_g, sel_o, wl.top_k, wl.top_p)
            assert ok, (name, "head", h, "row", i)
            mismatch += not ex
            cols_o.append(sel_o)
            rp_o[0, i + 1] = rp_o[0, i] + len(sel_o)
            for j in sel_o:
                sel_of_o.setdefault(int(j), []).append(i)
            for j in sel_g:
                sel_of_g.setdefault(int(j), []).append(i)
        del S
        assert mismatch <= max(1, nb // 100), f"{mismatch} of {nb} rows differ at near-ties"
        t0 = _phase(name, "oracle selection of one head", t0)
        # key blocks whose selectors agree on both sides, by selector count: the two
        # with the fewest and the median; below 2K also the 90th percentile and the
        # top (at 2K those hold 500 to 1000 selectors, each a whole fp64 row here)
        same = sorted((len(v), j) for j, v in sel_of_o.items() if sel_of_g.get(j) == v)
        assert len(same) >= 5
        idx = {0, 1, len(same) // 2}
        if name != "2k":
            idx |= {int(0.9 * (len(same) - 1)), len(same) - 1}
        keys = [same[t][1] for t in sorted(idx)]
        qh, kh, vh, doh = (_head(cpu[n], h, perm) for n in ("q", "k", "v", "dout"))
        kv = po.bsa_key_block_dkdv(qh, kh, vh, doh, blocks, rp_o, [np.concatenate(cols_o)], scale, keys)
        for j in keys:
            s0, sz = blocks[j][0], blocks[j][1]
            dk, dv = kv[j]
            tag = f"{name} h{h} b{j} ({len(sel_of_o[j])} selectors)"
            assert_close_attn(bwd["dkp"][h, s0:s0 + sz].double().cpu().numpy(), dk, "dK " + tag)
            assert_close_attn(bwd["dvp"][h, s0:s0 + sz].double().cpu().numpy(), dv, "dV " + tag)
        _phase(name, f"dK, dV of {len(keys)} key blocks ({sum(len(sel_of_o[j]) for j in keys)} selectors)", t0)
