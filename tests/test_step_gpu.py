"""kla_scan_step (recurrent decode, CUDA through the C ABI) against the oracle."""
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


@pytest.mark.parametrize("shape", [(2, 3, 64), (1, 1, 1), (3, 5, 7), (4, 2, 6)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("family", ["tiny", "lm_layer", "stiff"])
def test_step_parity(shape, family):
    """Vectorised (C % 4 == 0) and scalar paths, fp32 and bf16, 40 tokens."""
    kla = _kla()
    B, H, N = shape
    w = wl.WORKLOADS[family].with_shape(B=B, T=40, H=H, N=N)
    x = wl.generate(w)
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    lam = torch.from_numpy(x["lam0"]).to(DEV).clone()
    eta = torch.from_numpy(x["eta0"]).to(DEV).clone()
    mus, vars_ = [], []
    for t in range(w.T):
        mu = torch.empty_like(lam)
        var = torch.empty_like(lam)
        kla.scan_step(*(d[k][:, t].contiguous() for k in wl.INPUT_NAMES), lam, eta,
                      mu_out=mu, var_out=var)
        mus.append(mu)
        vars_.append(var)
    torch.cuda.synchronize()
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    got = {"mu": torch.stack(mus, 1).double().cpu().numpy(),
           "var": torch.stack(vars_, 1).double().cpu().numpy()}
    parity.assert_parity(got, ref, parity.RTOL[w.dtype], time_axis=1, what=f"step {family} {shape}")
    last = {"lam": lam.double().cpu().numpy()[:, None], "eta": eta.double().cpu().numpy()[:, None]}
    ref_last = {"lam": ref["lam"][:, -1:], "eta": ref["eta"][:, -1:]}
    assert np.max(np.abs(last["lam"] - ref_last["lam"]) / ref_last["lam"]) <= parity.RTOL[w.dtype]
    rms = np.sqrt(np.mean(ref["eta"] ** 2, axis=1, keepdims=True))
    assert np.max(np.abs(last["eta"] - ref_last["eta"]) / (np.abs(ref_last["eta"]) + rms)) \
        <= parity.RTOL[w.dtype]


def test_step_optional_outputs():
    kla = _kla()
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=3, H=2, N=8)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
    l1, e1 = d["lam0"].clone(), d["eta0"].clone()
    l2, e2 = d["lam0"].clone(), d["eta0"].clone()
    mu, var = torch.empty_like(l1), torch.empty_like(l1)
    for t in range(3):
        inp = [d[k][:, t].contiguous() for k in wl.INPUT_NAMES]
        kla.scan_step(*inp, l1, e1, mu_out=mu, var_out=var)
        kla.scan_step(*inp, l2, e2)
    assert torch.equal(l1, l2) and torch.equal(e1, e2)


@pytest.mark.slow
def test_decode_workload_full_size():
    """1024 one-token steps over B=256, H=32, N=128 channels from resident fp32
    state: the final state equals (i) the oracle over T = 1024 on a channel
    sample and (ii) the last row of kla_scan_forward over the same tokens on
    every channel; mu and var of every step match the oracle's rows."""
    kla = _kla()
    w = wl.WORKLOADS["decode"]
    sample = wl.channel_sample(w, 48)
    d, sampled = parity.to_device(w, DEV, sample)
    B, T, H, N = w.B, w.T, w.H, w.N
    HN = H * N
    fl, fe, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"],
                                    want_mu=False, want_var=False)
    last_fwd = (fl[:, -1].clone(), fe[:, -1].clone())
    del fl, fe
    steps = {k: d.pop(k).transpose(0, 1).contiguous() for k in wl.INPUT_NAMES}  # [T, B, H, N]
    lam, eta = d["lam0"].clone(), d["eta0"].clone()
    sb, shn = np.divmod(sample, HN)
    ib = torch.as_tensor(sb, device=DEV)
    ic = torch.as_tensor(shn, device=DEV)
    mu = torch.empty_like(lam)
    var = torch.empty_like(lam)
    mus = torch.empty((T, len(sample)), device=DEV)
    vars_ = torch.empty((T, len(sample)), device=DEV)
    for t in range(T):
        kla.scan_step(steps["a"][t], steps["p"][t], steps["phi"][t], steps["b"][t], lam, eta,
                      mu_out=mu, var_out=var)
        mus[t] = mu.view(B, HN)[ib, ic]
        vars_[t] = var.view(B, HN)[ib, ic]
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    ref = parity.oracle_on_sample(sampled, np.ones(len(sample)), np.zeros(len(sample)))
    got = {"mu": mus.double().cpu().numpy(), "var": vars_.double().cpu().numpy()}
    parity.assert_parity(got, ref, 1e-5, time_axis=0, what="decode per-step outputs")
    lam_s = lam.view(B, HN)[ib, ic].double().cpu().numpy()
    eta_s = eta.view(B, HN)[ib, ic].double().cpu().numpy()
    assert np.max(np.abs(lam_s - ref["lam"][-1]) / ref["lam"][-1]) <= 1e-5
    rms = np.sqrt(np.mean(ref["eta"] ** 2, axis=0))
    assert np.max(np.abs(eta_s - ref["eta"][-1]) / (np.abs(ref["eta"][-1]) + rms)) <= 1e-5
    # every channel: decode state == last row of the forward scan
    rl = ((lam - last_fwd[0]).abs() / last_fwd[0]).max().item()
    assert rl <= 1e-5, rl
    re_ = ((eta - last_fwd[1]).abs() / (last_fwd[1].abs() + 1.0)).max().item()
    assert re_ <= 1e-5, re_
