"""The bench's accounting on CPU: executed attention FLOPs from a selection,
the algorithmic bytes of the memory-bound kernels, and the rule that a
profiled traffic figure is reported only for the kernel sources it was taken on."""

import types

import numpy as np
import torch

import bench
from dynamic_block_sparse_variance_b200 import synth


def _fake_layer(seed=0, heads=3, cap=16, nb=11):
    """A PrismSparseAttention-shaped object on CPU: block table, per-head CSR."""
    rng = np.random.default_rng(seed)
    sizes = rng.choice([64, 128, 256], size=nb)
    blocks = torch.zeros(cap, 4, dtype=torch.int32)
    blocks[:nb, 1] = torch.from_numpy(sizes.astype(np.int32))
    row_ptr = torch.zeros(heads * cap + 1, dtype=torch.int32)
    cols, off, sel = [], 0, {}
    for h in range(heads):
        for i in range(cap):
            row_ptr[h * cap + i] = off
            if i < nb:
                c = np.sort(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False))
                sel[(h, i)] = c
                cols.append(c)
                off += len(c)
        # rows past nblk are empty
    row_ptr[heads * cap] = off
    att = types.SimpleNamespace(nblk=torch.tensor([nb], dtype=torch.int32), blocks=blocks, heads=heads, cap=cap,
                                row_ptr=row_ptr, col=torch.from_numpy(np.concatenate(cols).astype(np.int32)),
                                nnz=torch.tensor([off], dtype=torch.int64))
    return att, sizes, sel


def test_executed_pairs_is_the_sum_over_selected_block_pairs():
    att, sizes, sel = _fake_layer()
    total, nnz, nb, _, big = bench.executed_pairs(att)
    brute = sum(int(sizes[i]) * int(sizes[j]) for (h, i), c in sel.items() for j in c)
    brute256 = sum(int(sizes[i]) * int(sizes[j]) for (h, i), c in sel.items() for j in c if sizes[i] == 256)
    assert total == brute and big == brute256
    assert nnz == sum(len(c) for c in sel.values()) and nb == len(sizes)


def test_hbm_bytes_count_each_tensor_once():
    wl = synth.get_workload("2k")
    t = wl.N * wl.heads * wl.head_dim * 2
    b = bench.hbm_kernel_bytes(wl, 4900, 2.0)
    assert b["zone_stats_kernel"] == t                     # V read once
    assert b["permute_kernel"] == b["unpermute_kernel"] == 8 * t   # four tensors, read + write
    assert b["row_cut_kernel"] == wl.heads * 4900 ** 2 * 4
    assert b["block_scores_kernel"] == 2 * b["row_cut_kernel"]     # scores written twice per step


def _sources_hash():
    import hashlib
    import os
    h = hashlib.sha256()
    for f in bench.ATTN_SOURCES:
        with open(os.path.join(bench.ROOT, "dynamic_block_sparse_variance_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def test_profiled_traffic_only_for_the_profiled_sources(monkeypatch):
    rec = dict(bytes=4.0e9, flops=2.0e13, grid="test grid", sha256=_sources_hash())
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "bsa_bwd_tc_kernel", rec)
    got, src = bench.profiled_traffic("bsa_bwd_tc_kernel", 2 * rec["flops"])
    assert got == 2 * rec["bytes"] and "scaled" in src
    assert bench.profiled_traffic("bsa_dq_mma_kernel", 1.0) == (None, None)
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "bsa_bwd_tc_kernel", dict(rec, sha256="0" * 64))
    assert bench.profiled_traffic("bsa_bwd_tc_kernel", 1.0)[0] is None
