"""HostStepper (inputs and outputs in pinned host memory, copies overlapped
with the kernels of neighbouring steps) against the same steps run one by one
on device tensors.  O, dK and dV must agree bit for bit, step by step; dQ
too on the warp-MMA path (head_dim 64), and on the tensor-core path (summed
by fp32 reductions in arrival order) to within the spread of that order."""

import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from dynamic_block_sparse_variance_b200.attention import HostStepper, PrismSparseAttention
from tests.helpers import assert_dq_consistent

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,own_buffers", [("mix16", False), ("aniso8", True)])
def test_host_stepper_matches_step_by_step(name, own_buffers):
    _check_host_stepper(name, own_buffers, exact_dq=synth.get_workload(name).head_dim != 128)


def _check_host_stepper(name, own_buffers, exact_dq):
    wl = synth.get_workload(name)
    base = synth.make_inputs(wl, "cpu", with_dout=True)
    g = torch.Generator().manual_seed(5)
    steps = []
    for i in range(3):   # three steps with different inputs
        st = {}
        for n in ("q", "k", "v", "dout"):
            x = base[n].float() + (0.5 * i) * torch.randn(base[n].shape, generator=g)
            st[n] = x.to(base[n].dtype).pin_memory()
        st["audio"] = None if base["audio"] is None else base["audio"].pin_memory()
        steps.append(st)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p)
    ref = []
    for st in steps:
        cu = {n: None if st[n] is None else st[n].cuda() for n in st}
        o = att.forward(cu["q"], cu["k"], cu["v"], cu["audio"])
        dq, dk, dv = att.backward(cu["dout"])
        ref.append({n: t.cpu() for n, t in zip(("o", "dq", "dk", "dv"), (o, dq, dk, dv))})
    P.prism_device_status()
    outs = [{n: torch.empty((wl.N, wl.heads, wl.head_dim), dtype=torch.bfloat16).pin_memory()
             for n in ("o", "dq", "dk", "dv")} for _ in steps]
    dev = None
    if own_buffers:
        dev = {n: (None if steps[0][n] is None else torch.empty_like(steps[0][n], device="cuda"))
               for n in ("q", "k", "v", "audio", "dout")}
        dev.update({n: torch.empty((wl.N, wl.heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
                    for n in ("o", "dq", "dk", "dv")})
    HostStepper(att, device_buffers=dev).run(steps, outs)
    torch.cuda.synchronize()
    P.prism_device_status()
    for i in range(len(steps)):
        for n in ("o", "dq", "dk", "dv"):
            if n == "dq" and not exact_dq:
                assert_dq_consistent(outs[i][n], ref[i][n], f"step {i} dQ")
            else:
                assert torch.equal(outs[i][n], ref[i][n]), (i, n)
