"""Failure path on the GPU: bounded waits run out, report KLA_ERR_TIMEOUT, and
leave the context usable.  Nothing here faults, traps or hangs the GPU: the
waits target a device word that nothing sets and give up after a short limit."""
import numpy as np
import pytest
import torch

import oracle
import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture
def kla():
    import kalman_linear_attention_b200 as kla
    kla.set_wait_limit_ns(2_000_000)  # 2 ms
    kla.debug_force_forward_kernel(1)  # the kernel whose chunks wait on each other across CTAs
    yield kla
    kla.debug_force_forward_kernel(0)
    kla.debug_stall_chunk(-1)
    kla.set_wait_limit_ns(1_000_000_000)


def test_unset_flag_wait_reports_timeout(kla):
    assert kla.get_error() == 0
    kla.debug_unset_flag_wait()
    assert kla.get_error() == 5  # KLA_ERR_TIMEOUT
    assert kla.get_error() == 0  # cleared


def test_stalled_chunk_poisons_only_what_depends_on_it(kla):
    L = kla.chunk_tokens()
    w = wl.WORKLOADS["tiny"]  # T = 256 = 4 chunks of 64
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
    stall = 2
    kla.debug_stall_chunk(stall)
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    assert kla.get_error() == 5
    kla.debug_stall_chunk(-1)
    lam = out[0].double().cpu().numpy()
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    cut = stall * L
    ok = {k: o.double().cpu().numpy()[:, :cut] for k, o in zip(parity.OUTPUTS, out)}
    parity.assert_parity(ok, {k: ref[k][:, :cut] for k in parity.OUTPUTS}, 1e-5, time_axis=1)
    # the stalled chunk itself is NaN
    assert np.isnan(lam[:, cut:cut + L]).all()
    # a later chunk either composed the stalled chunk's published aggregate
    # (decoupled look-back: exact) or read its poisoned inclusive state (NaN)
    for c0 in range(cut + L, w.T, L):
        blk = {k: o.double().cpu().numpy()[:, c0:c0 + L] for k, o in zip(parity.OUTPUTS, out)}
        if np.isnan(blk["lam"]).all():
            continue
        assert np.isfinite(blk["lam"]).all()
        parity.assert_parity(blk, {k: ref[k][:, c0:c0 + L] for k in parity.OUTPUTS}, 1e-5, time_axis=1)
    # the context is still usable and a normal call is correct again
    out2 = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, out2)}
    parity.assert_parity(got, ref, 1e-5, time_axis=1)


def test_stalled_chunk_in_streaming_kernel(kla):
    """The streaming kernel hands the state from chunk to chunk inside the CTA:
    a carry wait that runs out poisons that chunk and every later token of its
    channels, leaves earlier tokens exact, and the context stays usable."""
    kla.debug_force_forward_kernel(2)
    L = kla.chunk_tokens()
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=512, H=2, N=64)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
    kla.debug_stall_chunk(3)
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    assert kla.get_error() == 5
    kla.debug_stall_chunk(-1)
    cut = 3 * L
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    ok = {k: o.double().cpu().numpy()[:, :cut] for k, o in zip(parity.OUTPUTS, out)}
    parity.assert_parity(ok, {k: ref[k][:, :cut] for k in parity.OUTPUTS}, 1e-5, time_axis=1)
    assert np.isnan(out[0].double().cpu().numpy()[:, cut:]).all()
    out2 = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, out2)}
    parity.assert_parity(got, ref, 1e-5, time_axis=1)


def test_stalled_chunk_in_backward_kernel(kla):
    """The streaming backward kernel hands the gradient carry from the later
    chunk to the earlier one: a carry wait that runs out poisons that chunk's
    gradients and those of every earlier token of its channels, leaves later
    tokens exact, reports KLA_ERR_TIMEOUT, and the context stays usable."""
    import test_backward_gpu as tb
    kla.debug_force_backward_kernel(2)
    try:
        w = wl.WORKLOADS["tiny"].with_shape(B=2, T=512, H=2, N=64)
        x = wl.generate(w)
        go = wl.generate_output_grads(w)
        d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
        g = [torch.from_numpy(go[k]).to(DEV) for k in wl.GRAD_NAMES]
        lam, eta, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
        assert kla.get_error() == 0
        kla.debug_stall_chunk(3)  # the backward chunk holding token 3 * chunk_tokens()
        out = kla.scan_backward(d["a"], d["p"], d["lam0"], d["eta0"], lam, eta, *g)
        assert kla.get_error() == 5
        kla.debug_stall_chunk(-1)
        stalled = 3 * kla.chunk_tokens()
        ref = oracle.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"],
                              *(go[k] for k in wl.GRAD_NAMES))
        got = [o.double().cpu().numpy() for o in out]
        # the chunk holding the stalled token ends at most 16 tokens later
        exact_from = stalled + 16
        later = {k: got[i][:, exact_from:] for i, k in enumerate(tb.GRADS)}
        tb.assert_grad_parity(later, {k: ref[k][:, exact_from:] for k in tb.GRADS}, 1e-5, "after the stall")
        for i in range(4):
            assert np.isnan(got[i][:, :stalled + 1]).all()
        assert np.isnan(got[4]).all() and np.isnan(got[5]).all()
        out2 = kla.scan_backward(d["a"], d["p"], d["lam0"], d["eta0"], lam, eta, *g)
        assert kla.get_error() == 0
        got2 = {k: o.double().cpu().numpy() for k, o in zip(tb.GRADS + ("lam0", "eta0"), out2)}
        tb.assert_grad_parity(got2, ref, 1e-5, "after recovery")
    finally:
        kla.debug_force_backward_kernel(0)
