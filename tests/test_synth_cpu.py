"""The seeded input generator (shared by both sides of every parity test):
deterministic, distinct per tensor and per workload, with the stated shapes,
dtypes and ranges, and free of the method's arithmetic."""

import ast
import pathlib

import torch

from dynamic_block_sparse_variance_b200 import synth


def test_same_seed_same_inputs_and_tensors_differ():
    wl = synth.get_workload("aniso8")
    a = synth.make_inputs(wl, "cpu", with_dout=True)
    b = synth.make_inputs(wl, "cpu", with_dout=True)
    for n in ("q", "k", "v", "dout", "audio"):
        assert torch.equal(a[n], b[n]), n
    assert not torch.equal(a["q"], a["k"]) and not torch.equal(a["k"], a["v"])
    other = synth.make_inputs(synth.get_workload("mix16"), "cpu", with_dout=True)
    assert other["q"].shape != a["q"].shape or not torch.equal(other["q"], a["q"])


def test_shapes_dtypes_and_audio_range():
    for name in ("tiny", "aniso8", "mix16"):
        wl = synth.get_workload(name)
        x = synth.make_inputs(wl, "cpu", with_dout=True)
        want = torch.float32 if wl.dtype == "f32" else torch.bfloat16
        for n in ("q", "k", "v", "dout"):
            assert x[n].shape == (wl.N, wl.heads, wl.head_dim) and x[n].dtype == want, (name, n)
            assert torch.isfinite(x[n].float()).all()
        a = x["audio"]
        assert a is not None and a.shape == (wl.N,) and a.dtype == torch.float32
        assert float(a.min()) >= 0.0 and abs(float(a.max()) - 1.0) < 1e-6     # bumps scaled to max 1


def test_zone_classes_on_the_mixed_grids():
    """The mixed workloads deal zones into static / temporal / spatial thirds."""
    wl = synth.get_workload("mix16")
    A = synth.zone_amplitudes(wl)
    static = (A == 0.1).all(dim=1)
    temporal = (A[:, 0] >= 1.0) & (A[:, 1] == 0.1) & (A[:, 2] == 0.1)
    spatial = (A[:, 0] == 0.1) & (A[:, 1] >= 1.0) & (A[:, 2] >= 1.0)
    assert bool((static | temporal | spatial).all())
    assert int(static.sum()) > 0 and int(temporal.sum()) > 0 and int(spatial.sum()) > 0


def test_generator_holds_none_of_the_method():
    """The generator module names none of the oracle's or the library's steps."""
    src = pathlib.Path(synth.__file__).read_text()
    tree = ast.parse(src)
    imported = {a.name for n in ast.walk(tree) if isinstance(n, (ast.Import, ast.ImportFrom))
                for a in n.names} | {n.module for n in ast.walk(tree) if isinstance(n, ast.ImportFrom) and n.module}
    assert not any("oracle" in m or "prism" in m for m in imported if m), imported
    for word in ("softmax", "log2", "quantis", "top_p_cut", "permut"):
        assert word not in src.lower(), word
