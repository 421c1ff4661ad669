"""kla_scan_forward_host: host buffers in and out, copies pipelined with the
scan in blocks of t_block tokens, against the oracle and the device path."""
import numpy as np
import pytest
import torch

import oracle
import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _kla():
    import kalman_linear_attention_b200 as kla
    return kla


@pytest.mark.parametrize("case", [
    dict(family="tiny", B=1, T=1000, H=2, N=64, t_block=192, pinned=True),    # ragged last block
    dict(family="stiff", B=3, T=700, H=1, N=96, t_block=128, pinned=True),    # B > 1: 2-D copies
    dict(family="lm_layer", B=2, T=640, H=2, N=64, t_block=0, pinned=True),   # bf16, auto block
    dict(family="tiny", B=2, T=300, H=1, N=40, t_block=64, pinned=False),     # pageable, ragged width
    dict(family="tiny", B=1, T=50, H=1, N=64, t_block=0, pinned=True),        # one block
], ids=lambda c: f"{c['family']}-B{c['B']}-T{c['T']}-tb{c['t_block']}-{'pin' if c['pinned'] else 'page'}")
def test_host_path_parity(case):
    kla = _kla()
    from kalman_linear_attention_b200 import api
    w = wl.WORKLOADS[case["family"]].with_shape(B=case["B"], T=case["T"], H=case["H"], N=case["N"])
    x = wl.generate(w)
    dt = parity.torch_dtype(w)
    host = {k: torch.from_numpy(x[k]).to(dt) for k in wl.INPUT_NAMES}
    host["lam0"] = torch.from_numpy(x["lam0"])
    host["eta0"] = torch.from_numpy(x["eta0"])
    if case["pinned"]:
        host = {k: v.pin_memory() for k, v in host.items()}
    args = [host[k] for k in ("a", "p", "phi", "b", "lam0", "eta0")]
    out = api._scan_forward_host(*args, want_mu=True, want_var=True, out=None, workspace=None, stream=None,
                                 t_block=case["t_block"])
    assert kla.get_error() == 0
    got = {k: o.double().numpy() for k, o in zip(parity.OUTPUTS, out)}
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    parity.assert_parity(got, ref, parity.RTOL[w.dtype], time_axis=1, what=str(case))
    dev = kla.scan_forward(*[t.to(DEV) for t in args])
    devn = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, dev)}
    parity.assert_parity(got, devn, 2e-6, time_axis=1, what="host vs device path")


def test_host_path_optional_outputs_and_public_api():
    kla = _kla()
    w = wl.WORKLOADS["tiny"].with_shape(B=1, T=900, H=1, N=64)
    x = wl.generate(w)
    host = [torch.from_numpy(x[k]).pin_memory() for k in ("a", "p", "phi", "b", "lam0", "eta0")]
    full = kla.scan_forward(*host)                                   # CPU tensors: the host path
    part = kla.scan_forward(*host, want_mu=False, want_var=False)
    assert part[2] is None and part[3] is None and not full[0].is_cuda
    assert torch.equal(full[0], part[0]) and torch.equal(full[1], part[1])
