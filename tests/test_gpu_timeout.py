"""Failure detection without a GPU fault: a forward wait that nothing
satisfies gives up after a short poll limit, the kernel latches
PRISM_ETIMEOUT, frees its tensor memory and returns; the context stays usable."""

import pytest
import torch

from dynamic_block_sparse_variance_b200 import prism as P
from dynamic_block_sparse_variance_b200 import synth
from dynamic_block_sparse_variance_b200.attention import PrismSparseAttention
from tests.helpers import assert_dq_consistent

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_recovers():
    wl = synth.get_workload("mix16")
    inp = synth.make_inputs(wl, "cpu", with_dout=False)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p)
    q, k, v, a = (inp[n].cuda() for n in ("q", "k", "v", "audio"))
    ref = att.forward(q, k, v, a).clone()
    P.prism_device_status()
    P.prism_set_option(P.PRISM_OPT_WAIT_LIMIT, 20000)
    P.prism_set_option(P.PRISM_OPT_DEBUG_STALL, 1)
    try:
        att.attend()
        with pytest.raises(P.PrismError) as e:
            P.prism_device_status()
        assert e.value.code == P.PRISM_ETIMEOUT
    finally:
        P.prism_set_option(P.PRISM_OPT_DEBUG_STALL, 0)
        P.prism_set_option(P.PRISM_OPT_WAIT_LIMIT, 0)
    out = att.forward(q, k, v, a)
    P.prism_device_status()
    assert torch.equal(out, ref)


def test_backward_bounded_wait_times_out_and_recovers():
    """The one-kernel backward: the elementwise warps never signal the first
    P^T tile, so the MMA issuer's wait runs out; every role of the CTA leaves
    its loop, the kernel latches PRISM_ETIMEOUT and frees its tensor memory,
    and the next backward is correct (dK, dV bit for bit)."""
    wl = synth.get_workload("mix16")
    inp = synth.make_inputs(wl, "cpu", with_dout=True)
    att = PrismSparseAttention(wl.T, wl.H, wl.W, wl.heads, wl.head_dim, wl.top_k, wl.top_p)
    q, k, v, a, do = (inp[n].cuda() for n in ("q", "k", "v", "audio", "dout"))
    att.forward(q, k, v, a)
    dq0, dk0, dv0 = (t.clone() for t in att.backward(do))
    P.prism_device_status()
    P.prism_set_option(P.PRISM_OPT_WAIT_LIMIT, 20000)
    P.prism_set_option(P.PRISM_OPT_DEBUG_STALL, 1)
    try:
        att.attend_backward()
        with pytest.raises(P.PrismError) as e:
            P.prism_device_status()
        assert e.value.code == P.PRISM_ETIMEOUT
    finally:
        P.prism_set_option(P.PRISM_OPT_DEBUG_STALL, 0)
        P.prism_set_option(P.PRISM_OPT_WAIT_LIMIT, 0)
    dq, dk, dv = att.backward(do)
    P.prism_device_status()
    assert torch.equal(dk, dk0) and torch.equal(dv, dv0)
    assert_dq_consistent(dq, dq0)
