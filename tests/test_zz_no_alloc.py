"""kla_scan_forward_static, the forward scan for callers that cannot allocate
device memory (code inside a CUDA stream capture, code under a fixed memory
budget, host runtimes without an allocator): it uses the library's own static
device scratch instead of a caller-allocated workspace.  Checked against
kla_scan_forward, the entry point with a workspace, on several calls in a row
that reuse the shared scratch.  Collected last on purpose."""
import numpy as np
import pytest
import torch

import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(w):
    x = wl.generate(w)
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    d["lam0"] = torch.from_numpy(x["lam0"]).to(DEV)
    d["eta0"] = torch.from_numpy(x["eta0"]).to(DEV)
    return d


def test_static_scratch_matches_workspace_entry_point():
    import kalman_linear_attention_b200 as kla
    # two different problems, then the first again: every call inherits the
    # previous call's scratch contents
    cases = [wl.WORKLOADS["stiff"].with_shape(B=16, T=700),
             wl.WORKLOADS["lm_layer"].with_shape(B=2, T=1500, H=4),
             wl.WORKLOADS["stiff"].with_shape(B=16, T=700)]
    for w in cases:
        d = _inputs(w)
        args = (d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
        ref = kla.scan_forward(*args)
        outs = [torch.full((w.B, w.T, w.H, w.N), float("nan"), device=DEV) for _ in range(4)]
        kla.scan_forward_static(*args, out=outs)
        torch.cuda.synchronize()
        assert kla.get_error() == 0
        got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, outs)}
        exp = {k: r.double().cpu().numpy() for k, r in zip(parity.OUTPUTS, ref)}
        parity.assert_parity(got, exp, parity.RTOL[w.dtype], time_axis=1, what=w.name)
        for o, r in zip(outs, ref):
            assert torch.equal(o, r)  # same kernel and carry order: bit-identical


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
