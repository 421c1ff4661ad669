"""Parity of kla_attention_weights (the Kalman attention weights: products of
the filter's gates over windows of tokens) with the oracle, element by
element, through the C ABI.

The kernel forms its gates from the forward scan's own lambda (computed here
by kla_scan_forward on the GPU); the oracle forms them from its fp64 filter.
Tolerance: |F - F_ref| <= rtol |F_ref| + 2^-126 (rtol 1e-5 for fp32 inputs,
2e-2 for bf16): an entry is a product of up to W - 1 gates, each with the
error of one hardware reciprocal and a multiply, plus what the forward
scan's lambda carries in; entries below the fp32 normal range flush to 0.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TINY = 2.0 ** -126

# (B, T, H, N, t0, span, W)
SHAPES = [
    (2, 100, 1, 64, 0, 100, 16),     # whole sequence, several windows
    (1, 40, 2, 16, 5, 30, 7),        # offset span, ragged last window
    (2, 70, 3, 7, 3, 64, 64),        # H*N = 21: one channel per lane, ragged channel tile
    (1, 256, 1, 64, 0, 256, 64),     # the tiny workload's shape, largest window
    (3, 33, 1, 8, 0, 33, 1),         # W = 1: only the diagonal
    (1, 130, 2, 64, 1, 128, 33),     # odd window, ragged
    (2, 90, 2, 66, 10, 75, 20),      # H*N = 132 (a multiple of 4, not of 128)
]


def _problem(B, T, H, N, dtype, seed):
    fam = "lm_layer" if dtype == "bf16" else "tiny"
    w = wl.WORKLOADS[fam].with_shape(B=B, T=T, H=H, N=N, seed=seed)
    x = wl.generate(w)
    x["a"] = x["a"] * np.where(np.random.default_rng(seed).random(x["a"].shape) < 0.2, -1.0, 1.0
                               ).astype(np.float32)
    x.update(wl.random_prior(w))
    return w, x


def _gpu_weights(kla, w, x, t0, span, W):
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    lam0 = torch.from_numpy(x["lam0"]).to(DEV)
    eta0 = torch.from_numpy(x["eta0"]).to(DEV)
    lam, eta, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], lam0, eta0)
    F = kla.attention_weights(d["a"], d["p"], lam, t0=t0, span=span, W=W)
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    return F, lam, eta, d


def _check(got, ref, rtol, what):
    err = np.abs(got - ref)
    bad = err > rtol * np.abs(ref) + TINY
    assert not bad.any(), (f"{what}: {int(bad.sum())} entries off, max rel "
                           f"{float(np.max(err / (np.abs(ref) + TINY))):.3e}")
    return float(np.max(err / (np.abs(ref) + 1e-30)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_attention_weights_match_oracle(shape, dtype):
    import kalman_linear_attention_b200 as kla
    B, T, H, N, t0, span, W = shape
    w, x = _problem(B, T, H, N, dtype, seed=sum(shape))
    F, _, _, _ = _gpu_weights(kla, w, x, t0, span, W)
    ref = oracle.attention_weights(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], t0, span, W)
    assert tuple(F.shape) == ref.shape
    _check(F.double().cpu().numpy(), ref, parity.RTOL[dtype], f"{shape} {dtype}")


def test_attention_weights_empty_and_errors():
    import kalman_linear_attention_b200 as kla
    w, x = _problem(1, 20, 1, 32, "f32", seed=3)
    F, lam, _, d = _gpu_weights(kla, w, x, 0, 0, 8)
    assert F.shape[1] == 0
    with pytest.raises(kla.KlaError):
        kla.attention_weights(d["a"], d["p"], lam, t0=15, span=10, W=8)   # past the end
    with pytest.raises(kla.KlaError):
        kla.attention_weights(d["a"], d["p"], lam, W=65)


@pytest.mark.slow
def test_attention_weights_lm_layer_full_size():
    """The LM-layer workload (B=8, T=2048, H=16, N=128, bf16), every window of
    64 tokens, as the benchmark runs it: sampled whole channels against the
    oracle, and on every channel of a few windows the unrolled mean,
    eta_t = F(t, s) eta_s + sum_r F(t, r) b_r, against the scan's eta."""
    import kalman_linear_attention_b200 as kla
    w = wl.WORKLOADS["lm_layer"]
    W = 64
    sample = wl.channel_sample(w, 48)
    d, sampled = parity.to_device(w, DEV, sample)
    lam, eta, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    F = kla.attention_weights(d["a"], d["p"], lam, W=W)
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    nwin = w.T // W
    HN = w.H * w.N
    # sampled channels against the oracle
    K = len(sample)
    xs = {k: sampled[k].reshape(1, w.T, 1, K) for k in wl.INPUT_NAMES}
    ref = oracle.attention_weights(xs["a"], xs["p"], xs["phi"], xs["b"], np.ones((1, 1, K)), np.zeros((1, 1, K)),
                                   0, w.T, W, threads=8)
    sb, shn = np.divmod(sample, HN)
    Fv = F.view(w.B, nwin, W, W, HN)
    got = Fv[torch.as_tensor(sb, device=DEV), :, :, :, torch.as_tensor(shn, device=DEV)]  # [K, nwin, W, W]
    got = got.permute(1, 2, 3, 0).double().cpu().numpy()
    _check(got, ref[0, :, :, :, 0, :], parity.RTOL["bf16"], "lm_layer sampled")
    # the unrolled information mean on every channel, windows 0, 17 and 31
    bv = d["b"].float().double().view(w.B, w.T, HN)
    ev = eta.double().view(w.B, w.T, HN)
    for win in (0, 17, 31):
        s0 = win * W
        Fw = Fv[:, win].double()                                           # [B, W, W, HN]
        x_in = torch.cat([ev[:, s0:s0 + 1], bv[:, s0 + 1:s0 + W]], dim=1)  # eta_s, then b_{s+1..}
        terms = Fw * x_in[:, None, :, :]
        rhs = terms.sum(dim=2)                                              # [B, W, HN]
        lhs = ev[:, s0:s0 + W]
        rms = ev.pow(2).mean(dim=1, keepdim=True).sqrt()
        scale = terms.abs().sum(dim=2) + lhs.abs() + rms
        worst = float(((lhs - rhs).abs() / scale).max())
        assert worst <= 1e-5, f"window {win}: unrolled mean off by {worst:.3e}"
