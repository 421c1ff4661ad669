"""kla_scan_forward_static, the forward scan for callers that cannot allocate
device memory (code inside a CUDA stream capture, code under a fixed memory
budget, host runtimes without an allocator): it uses the library's own static
device scratch instead of a caller-allocated workspace.

The calls below run one after another on the same scratch, with different
shapes and both forward kernels, so that every call starts from what the
previous one left there: the streaming kernel with its tiles split into runs
(ticket, run flags and run-boundary states), the chunked kernel forced on a
shape the streaming kernel would take (ticket, per-chunk flags, aggregates and
carried states: the whole layout), the chunked kernel chosen by geometry, the
streaming kernel without a split (whole tiles by ticket, then round-robin),
and the split again after the chunked kernel's layout.  Every call is checked against the oracle and, bit for bit,
against kla_scan_forward with its own workspace.  Collected last on purpose."""
import pytest
import torch

import oracle
import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# (workload, forced forward kernel: 0 = chosen by shape, 1 = chunked)
CASES = [
    # 320 tiles of 32 channels, 22 chunks: the streaming kernel in 3 runs per tile
    (wl.WORKLOADS["tiny"].with_shape(B=10, H=8, N=128, T=700, seed=21), 0),
    # the same kind of shape on the chunked kernel: every part of its layout
    (wl.WORKLOADS["lm_layer"].with_shape(B=2, T=1500, H=4, seed=22), 1),
    # H*N = 24 < 32: the chunked kernel by geometry
    (wl.WORKLOADS["tiny"].with_shape(B=3, H=3, N=8, T=333, seed=23), 0),
    # the streaming kernel with whole tiles taken by ticket (256 tiles of 22 chunks)
    (wl.WORKLOADS["stiff"].with_shape(B=16, T=700, seed=24), 0),
    # the streaming kernel with whole tiles round-robin (7 chunks per tile): no workspace
    (wl.WORKLOADS["stiff"].with_shape(B=16, T=200, seed=27), 0),
    # the chunked kernel on the first shape, then the run split again on
    # what the chunked kernel left behind
    (wl.WORKLOADS["tiny"].with_shape(B=10, H=8, N=128, T=700, seed=25), 1),
    (wl.WORKLOADS["tiny"].with_shape(B=10, H=8, N=128, T=700, seed=26), 0),
]


def _run(kla, w, force):
    x = wl.generate(w)
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    pri = wl.prior(w)
    d["lam0"] = torch.from_numpy(pri["lam0"]).to(DEV)
    d["eta0"] = torch.from_numpy(pri["eta0"]).to(DEV)
    args = (d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    kla.debug_force_forward_kernel(force)
    try:
        plan = kla.forward_plan(d["a"], d["p"], d["phi"], d["b"])
        outs = [torch.full((w.B, w.T, w.H, w.N), float("nan"), device=DEV) for _ in range(4)]
        kla.scan_forward_static(*args, out=outs)
        ref = kla.scan_forward(*args)
        torch.cuda.synchronize()
    finally:
        kla.debug_force_forward_kernel(0)
    assert kla.get_error() == 0
    return x, pri, plan, outs, ref


def test_static_scratch_reused_across_calls_and_kernels():
    import kalman_linear_attention_b200 as kla
    seen = set()
    for w, force in CASES:
        x, pri, plan, outs, ref = _run(kla, w, force)
        kernel = plan[0]
        # the streaming kernel launches twice (clear + scan) when it takes its units by ticket
        seen.add(("stream" if kernel == 2 else "chunked", plan[1]))
        got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, outs)}
        exp = oracle.forward(x["a"], x["p"], x["phi"], x["b"], pri["lam0"], pri["eta0"], threads=8)
        parity.assert_parity(got, exp, parity.RTOL[w.dtype], time_axis=1,
                             what=f"{w.summary}, kernel {kernel}")
        for o, r in zip(outs, ref):
            assert torch.equal(o, r)  # same kernel and carry order as the workspace entry point
    # the calls above went through both layouts of the scratch
    assert ("stream", 2) in seen and ("stream", 1) in seen and ("chunked", 2) in seen, seen


def test_static_scratch_rejects_problems_that_do_not_fit():
    import kalman_linear_attention_b200 as kla
    from kalman_linear_attention_b200 import api
    w = wl.WORKLOADS["long"]
    assert kla.workspace_size(w.B, w.T, w.H, w.N) > api.STATIC_SCRATCH_BYTES
    st = api.lib().kla_scan_forward_static(None, None, None, None, 0, None, None, None, None,
                                           None, None, w.B, w.T, w.H, w.N, None)
    assert st == api.KLA_ERR_TOO_LARGE
    # the largest standard workload that fits: the LM-layer shape
    w = wl.WORKLOADS["lm_layer"]
    assert kla.workspace_size(w.B, w.T, w.H, w.N, torch.bfloat16) <= api.STATIC_SCRATCH_BYTES
