"""Parity of kla_scan_forward_lti (the convolutional form of deterministic
time-invariant channels: p = 0, a constant decay per channel) with the
oracle, element by element, through the C ABI.

Small shapes are checked against the oracle's convolution sums
(``oracle.lti_forward``) and the large ones against its covariance-form filter
run with p = 0 (the two are pinned equal).

Tolerances: lambda and var relative, 1e-5 (fp32) / 2e-2 (bf16): lambda is a
sum of non-negative terms.  eta_t is the sum of the terms a^-(t+1) eta_0 and
a^-(t-s) b_s, of either sign; with |a| < 1 they grow with the distance, so
eta can be far smaller than its terms, and any evaluation in fp32 (this
kernel's, or the general scan's) is accurate relative to the sum of the
terms' absolute values, not to eta.  So eta and mu are checked as
|x - ref| <= rtol (|ref| + E) with E that absolute sum (for mu, E / lambda),
which the oracle gives by filtering |a|, |b| and |eta_0|.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# (B, T, H, N, dtype): streaming kernel unless noted
SHAPES = [
    (2, 100, 1, 64, "f32"),        # ragged last chunk
    (1, 700, 2, 64, "f32"),        # 22 chunks: the warp-to-warp carry
    (3, 33, 1, 7, "f32"),          # H*N = 7: one thread per channel
    (2, 31, 2, 32, "f32"),         # T below one chunk: one thread per channel
    (1, 1, 1, 32, "f32"),          # one token
    (2, 300, 4, 64, "bf16"),       # bf16 evidence
    (4, 96, 3, 40, "f32"),         # ragged channel tile (H*N = 120)
]


def _problem(B, T, H, N, dtype, seed, lo=0.98, hi=1.02):
    w = wl.LTI_WORKLOADS["lti"].with_shape(B=B, T=T, H=H, N=N, seed=seed,
                                           dtype="bf16" if dtype == "bf16" else "f32")
    x = wl.generate_lti(w, (lo, hi))
    rng = np.random.default_rng(seed)
    x["a"] = (x["a"] * np.where(rng.random(x["a"].shape) < 0.3, -1.0, 1.0)).astype(np.float32)
    x.update(wl.random_prior(w))
    return w, x


def _check(got, ref, ref_abs, rtol, what):
    """lambda, var relative; eta, mu relative to the absolute-term sums."""
    errs = {}
    for k in ("lam", "var"):
        errs[k] = float(np.max(np.abs(got[k] - ref[k]) / ref[k]))
    scale = {"eta": ref_abs["eta"], "mu": ref_abs["eta"] / ref["lam"]}
    for k in ("eta", "mu"):
        errs[k] = float(np.max(np.abs(got[k] - ref[k]) / (np.abs(ref[k]) + scale[k])))
    bad = {k: v for k, v in errs.items() if not v <= rtol}
    assert not bad, f"{what}: errors above rtol={rtol:g}: {bad} (all: {errs})"
    return errs


def _abs_terms(x, lti=True):
    """The oracle on |a|, |b|, |eta_0|: every term of eta taken by absolute value."""
    if lti:
        return oracle.lti_forward(np.abs(x["a"]), x["phi"], np.abs(x["b"]), x["lam0"], np.abs(x["eta0"]))
    a = np.broadcast_to(np.abs(x["a"])[:, None], x["phi"].shape)
    return oracle.forward(a, np.zeros(x["phi"].shape), x["phi"], np.abs(x["b"]), x["lam0"], np.abs(x["eta0"]),
                          threads=8)


def _filter_p0(x):
    return oracle.forward(np.broadcast_to(x["a"][:, None], x["phi"].shape), np.zeros(x["phi"].shape), x["phi"],
                          x["b"], x["lam0"], x["eta0"], threads=8)


def _gpu(kla, w, x):
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in ("phi", "b")}
    for k in ("a", "lam0", "eta0"):
        d[k] = torch.from_numpy(x[k]).to(DEV)
    outs = kla.scan_forward_lti(d["a"], d["phi"], d["b"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    return d, outs


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_lti_matches_convolution_oracle(shape):
    import kalman_linear_attention_b200 as kla
    B, T, H, N, dtype = shape
    w, x = _problem(B, T, H, N, dtype, seed=B * 1000 + T)
    _, outs = _gpu(kla, w, x)
    ref = oracle.lti_forward(x["a"], x["phi"], x["b"], x["lam0"], x["eta0"])
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, outs)}
    _check(got, ref, _abs_terms(x), parity.RTOL[dtype], str(shape))


def test_lti_kernels_and_run_split():
    """The streaming kernel with its tiles split into runs (320 tiles of 32
    channels) and the one-thread-per-channel kernel on the same problem (a
    misaligned view forces it) agree with the oracle's filter with p = 0."""
    import kalman_linear_attention_b200 as kla
    w, x = _problem(10, 700, 8, 128, "f32", seed=77)
    d, outs = _gpu(kla, w, x)
    assert kla.lti_plan(d["phi"], d["b"]) == (2, 2)
    ref = _filter_p0(x)
    ref_abs = _abs_terms(x, lti=False)
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, outs)}
    _check(got, ref, ref_abs, 1e-5, "run split")
    # plain loads: inputs shifted by one element (4 bytes) off the 16-byte grid
    B, T, H, N = x["phi"].shape
    buf = {k: torch.empty(B * T * H * N + 1, device=DEV) for k in ("phi", "b")}
    for k in buf:
        buf[k][1:].copy_(d[k].reshape(-1))
    phi1, b1 = (buf[k][1:].view(B, T, H, N) for k in ("phi", "b"))
    assert kla.lti_plan(phi1, b1)[0] == 1
    outs1 = kla.scan_forward_lti(d["a"], phi1, b1, d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    got1 = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, outs1)}
    _check(got1, ref, ref_abs, 1e-5, "one thread per channel")


def test_lti_ticketed_whole_tiles():
    """160 tiles of 32 channels, one run each, taken whole by ticket: the plan
    reports the clear launch and every element matches the oracle's filter."""
    import kalman_linear_attention_b200 as kla
    w, x = _problem(160, 300, 1, 32, "f32", seed=91)
    d, outs = _gpu(kla, w, x)
    assert kla.lti_plan(d["phi"], d["b"]) == (2, 2)
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, outs)}
    _check(got, _filter_p0(x), _abs_terms(x, lti=False), 1e-5, "ticketed whole tiles")


def test_lti_agrees_with_general_scan_and_skips_outputs():
    """Same inputs through kla_scan_forward (a broadcast over time, p = 0):
    both agree with the oracle (64 tokens: the general scan repeats the same
    rounding of a^2 and of its reciprocal at every token of a constant decay,
    so its error grows by about 2 ulp per token); mu / var skipped leave
    lambda, eta bit-identical."""
    import kalman_linear_attention_b200 as kla
    w, x = _problem(2, 64, 2, 64, "f32", seed=5)
    d, outs = _gpu(kla, w, x)
    ag = d["a"][:, None].expand(d["phi"].shape).contiguous()
    gen = kla.scan_forward(ag, torch.zeros_like(ag), d["phi"], d["b"], d["lam0"], d["eta0"])
    ref = oracle.lti_forward(x["a"], x["phi"], x["b"], x["lam0"], x["eta0"])
    ref_abs = _abs_terms(x)
    for res, what in ((outs, "convolutional form"), (gen, "general scan")):
        got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, res)}
        _check(got, ref, ref_abs, 1e-5, what)
    lam2, eta2, mu2, var2 = kla.scan_forward_lti(d["a"], d["phi"], d["b"], d["lam0"], d["eta0"],
                                                 want_mu=False, want_var=False)
    torch.cuda.synchronize()
    assert mu2 is None and var2 is None
    assert torch.equal(lam2, outs[0]) and torch.equal(eta2, outs[1])


@pytest.mark.slow
def test_lti_full_size():
    """The time-invariant workload (B=1, H=32, N=128, T=65536, a within 5e-4
    of 1, both sides), launched as the benchmark launches it: 48 sampled whole
    channels against the oracle's filter with p = 0, properties on every
    element."""
    import kalman_linear_attention_b200 as kla
    w = wl.LTI_WORKLOADS["lti"]
    x = wl.generate_lti(w)
    _, outs = _gpu(kla, w, x)
    HN = w.H * w.N
    sample = wl.channel_sample(w, 48)
    sb, shn = np.divmod(sample, HN)
    K = len(sample)
    a_s = x["a"].reshape(w.B, HN)[sb, shn]
    phi_s = x["phi"].reshape(w.B, w.T, HN)[sb, :, shn].T.reshape(1, w.T, 1, K)
    b_s = x["b"].reshape(w.B, w.T, HN)[sb, :, shn].T.reshape(1, w.T, 1, K)
    xs = {"a": a_s.reshape(1, 1, K), "phi": phi_s, "b": b_s, "lam0": np.ones((1, 1, K)),
          "eta0": np.zeros((1, 1, K))}
    ref = {k: v.reshape(w.T, K) for k, v in _filter_p0(xs).items()}
    ref_abs = {k: v.reshape(w.T, K) for k, v in _abs_terms(xs, lti=False).items()}
    got = {k: parity.gather_channels(o, sample, HN) for k, o in zip(parity.OUTPUTS, outs)}
    errs = _check(got, ref, ref_abs, 1e-5, "lti full size")
    print("lti full-size max errors:", errs)
    lam, _, _, var = outs
    assert bool(torch.isfinite(lam).all()) and bool((lam > 0).all())
    assert float((var * lam - 1).abs().max()) < 1e-5
