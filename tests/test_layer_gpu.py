"""kla_layer_forward (the KLA layer's filter with evidence formation and
readout fused; CUDA, through the C ABI) against the fp64 oracle's layer
function.

Tolerances as for the scan: y crosses zero, so |y - ref| <= rtol (|ref| +
rms_t(ref)); s and the final precision are positive (pure relative test); the
final information mean uses the rms over channels.  rtol = 1e-5 for fp32
inputs, 2e-2 for bf16 inputs.
"""
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


def layer_errors(got, ref, time_axis=1):
    errs = {}
    for k in ("y", "s", "lam_T", "eta_T"):
        if got.get(k) is None:
            continue
        g = np.asarray(got[k], dtype=np.float64)
        r = np.asarray(ref[k], dtype=np.float64)
        assert g.shape == r.shape, (k, g.shape, r.shape)
        if g.size == 0:
            errs[k] = 0.0
            continue
        if not np.all(np.isfinite(g)):
            errs[k] = float("inf")
            continue
        if k in ("s", "lam_T"):
            errs[k] = float(np.max(np.abs(g - r) / np.abs(r)))
        else:
            axis = time_axis if k == "y" else None
            rms = np.sqrt(np.mean(r * r, axis=axis, keepdims=axis is not None))
            errs[k] = float(np.max(np.abs(g - r) / (np.abs(r) + rms + 1e-300)))
    return errs


def to_dev(x, dtype):
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dtype) for k in wl.LAYER_TOKEN_NAMES}
    for k in ("a", "p", "lam0", "eta0"):
        d[k] = torch.from_numpy(x[k]).to(DEV)
    return d


def run_layer(w, prior="random", **kw):
    kla = _kla()
    x = wl.generate_layer(w)
    if prior == "random":
        x.update(wl.random_layer_prior(w))
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = to_dev(x, dt)
    out = kla.layer_forward(d["k"], d["q"], d["v"], d["w"], d["a"], d["p"], d["lam0"], d["eta0"], **kw)
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: (None if o is None else o.double().cpu().numpy()) for k, o in zip(("y", "s", "lam_T", "eta_T"), out)}
    ref = oracle.layer_forward(x["k"], x["q"], x["v"], x["w"], x["a"], x["p"], x["lam0"], x["eta0"], threads=8)
    return got, ref, x, d


# (B, T, H, D, Ns): whole chunks, ragged last chunk, one token, several
# chunks and tiles, a long single-tile sequence.
SHAPES = [
    (2, 96, 2, 4, 16),
    (1, 64, 1, 8, 8),
    (3, 33, 3, 6, 16),
    (1, 1, 1, 2, 16),
    (2, 300, 2, 8, 8),
    (1, 2000, 1, 2, 16),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_layer_parity_small_shapes(shape, dtype):
    B, T, H, D, Ns = shape
    w = wl.LAYER_WORKLOADS["layer"].with_shape(B=B, T=T, H=H, D=D, Ns=Ns)
    w = w.__class__(**{**w.__dict__, "dtype": dtype})
    got, ref, _, _ = run_layer(w)
    errs = layer_errors(got, ref)
    rtol = parity.RTOL[dtype]
    assert max(errs.values()) <= rtol, (shape, dtype, errs)


def test_layer_optional_outputs_and_run_split():
    """s and the final state may be skipped (y bit-identical); 640 tiles of
    32 channels split each tile's sequence into runs."""
    kla = _kla()
    w = wl.LAYER_WORKLOADS["layer"].with_shape(B=10, T=512, H=4, D=32, Ns=16)
    full, ref, x, d = run_layer(w)
    errs = layer_errors(full, ref)
    assert max(errs.values()) <= parity.RTOL["bf16"], errs
    part = kla.layer_forward(d["k"], d["q"], d["v"], d["w"], d["a"], d["p"], d["lam0"], d["eta0"],
                             want_s=False, want_state=False)
    torch.cuda.synchronize()
    assert part[1] is None and part[2] is None and part[3] is None
    np.testing.assert_array_equal(part[0].double().cpu().numpy(), full["y"])


def test_layer_matches_unfused_path():
    """The fused kernel agrees (to rounding) with the unfused path: phi and b
    formed on the device, kla_scan_forward over the H x D x Ns channels, and
    the readout (torch only stages the unfused path's intermediates)."""
    kla = _kla()
    w = wl.LAYER_WORKLOADS["layer"].with_shape(B=2, T=700, H=2, D=8, Ns=16)
    w = w.__class__(**{**w.__dict__, "dtype": "f32"})
    got, ref, x, d = run_layer(w)
    B, T, H, D, Ns = w.B, w.T, w.H, w.D, w.Ns
    kk = d["k"][:, :, :, None, :]
    ww = d["w"][:, :, :, :, None]
    phi = (kk * kk * ww).reshape(B, T, H, D * Ns).contiguous()
    info = (kk * ww * d["v"][:, :, :, :, None]).reshape(B, T, H, D * Ns).contiguous()
    aa = d["a"].expand(B, T, H, D, Ns).reshape(B, T, H, D * Ns).contiguous()
    pp = d["p"].expand(B, T, H, D, Ns).reshape(B, T, H, D * Ns).contiguous()
    lam, eta, mu, var = kla.scan_forward(aa, pp, phi, info, d["lam0"].reshape(B, H, D * Ns).contiguous(),
                                         d["eta0"].reshape(B, H, D * Ns).contiguous())
    qq = d["q"][:, :, :, None, :]
    y = (qq * mu.reshape(B, T, H, D, Ns)).sum(-1)
    s = (qq * qq * var.reshape(B, T, H, D, Ns)).sum(-1)
    torch.cuda.synchronize()
    unf = {"y": y.double().cpu().numpy(), "s": s.double().cpu().numpy(),
           "lam_T": lam[:, -1].reshape(B, H, D, Ns).double().cpu().numpy(),
           "eta_T": eta[:, -1].reshape(B, H, D, Ns).double().cpu().numpy()}
    errs = layer_errors(got, unf)
    assert max(errs.values()) <= 2e-6, errs
    assert max(layer_errors(got, ref).values()) <= 1e-5


def test_layer_zero_tokens_and_errors():
    kla = _kla()
    B, H, D, Ns = 2, 2, 4, 16
    e = torch.empty((B, 0, H, Ns), device=DEV)
    ev = torch.empty((B, 0, H, D), device=DEV)
    a = torch.full((H, D, Ns), 0.9, device=DEV)
    p = torch.full((H, D, Ns), 0.01, device=DEV)
    lam0 = torch.rand((B, H, D, Ns), device=DEV) + 0.5
    eta0 = torch.randn((B, H, D, Ns), device=DEV)
    y, s, lt, et = kla.layer_forward(e, e, ev, ev, a, p, lam0, eta0)
    torch.cuda.synchronize()
    assert torch.equal(lt, lam0) and torch.equal(et, eta0) and y.numel() == 0
    k = torch.randn((1, 8, 1, 4), device=DEV)
    v = torch.randn((1, 8, 1, 8), device=DEV)
    with pytest.raises(kla.KlaError):        # Ns = 4 is not supported
        kla.layer_forward(k, k, v, v, torch.ones((1, 8, 4), device=DEV), torch.ones((1, 8, 4), device=DEV),
                          torch.ones((1, 1, 8, 4), device=DEV), torch.zeros((1, 1, 8, 4), device=DEV))
    k = torch.randn((1, 8, 1, 16), device=DEV)
    v = torch.randn((1, 8, 1, 3), device=DEV)
    with pytest.raises(kla.KlaError):        # D = 3 is not a multiple of 32 / 16
        kla.layer_forward(k, k, v, v, torch.ones((1, 3, 16), device=DEV), torch.ones((1, 3, 16), device=DEV),
                          torch.ones((1, 1, 3, 16), device=DEV), torch.zeros((1, 1, 3, 16), device=DEV))
    assert kla.get_error() == 0


def test_layer_full_size_sampled():
    """The layer workload at full size, launched as the bench launches it;
    the oracle on a seeded sample of (b, h, d) value coordinates, every token."""
    kla = _kla()
    w = wl.LAYER_WORKLOADS["layer"]
    x = wl.generate_layer(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = to_dev(x, dt)
    y, s, lt, et = kla.layer_forward(d["k"], d["q"], d["v"], d["w"], d["a"], d["p"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    yh, sh = y.double().cpu().numpy(), s.double().cpu().numpy()
    assert np.all(np.isfinite(yh)) and np.all(sh > 0)
    rng = np.random.default_rng(99)
    worst = {}
    for _ in range(24):
        b, h, dd = int(rng.integers(w.B)), int(rng.integers(w.H)), int(rng.integers(w.D))
        sl = lambda arr: arr[b:b + 1, :, h:h + 1]
        r = oracle.layer_forward(sl(x["k"]), sl(x["q"]), sl(x["v"])[..., dd:dd + 1], sl(x["w"])[..., dd:dd + 1],
                                 x["a"][h:h + 1, dd:dd + 1], x["p"][h:h + 1, dd:dd + 1],
                                 x["lam0"][b:b + 1, h:h + 1, dd:dd + 1], x["eta0"][b:b + 1, h:h + 1, dd:dd + 1])
        got = {"y": yh[b:b + 1, :, h:h + 1, dd:dd + 1], "s": sh[b:b + 1, :, h:h + 1, dd:dd + 1],
               "lam_T": lt[b:b + 1, h:h + 1, dd:dd + 1].double().cpu().numpy(),
               "eta_T": et[b:b + 1, h:h + 1, dd:dd + 1].double().cpu().numpy()}
        for k, v in layer_errors(got, r).items():
            worst[k] = max(worst.get(k, 0.0), v)
    print("layer full-size sampled max errors", worst)
    assert max(worst.values()) <= parity.RTOL[w.dtype], worst


@pytest.mark.parametrize("dtype,Ns", [("f32", 16), ("bf16", 8)])
def test_layer_prefill_then_decode(dtype, Ns):
    """kla_layer_forward over the first tokens, then kla_layer_step token by
    token from its final state: every decoded readout and the final state
    against the oracle over the whole sequence, and the decoded readouts
    against the fused kernel's own rows over the same tokens."""
    import dataclasses
    kla = _kla()
    w = dataclasses.replace(wl.LAYER_WORKLOADS["layer"].with_shape(B=2, T=80, H=2, D=4, Ns=Ns), dtype=dtype)
    x = wl.generate_layer(w)
    x.update(wl.random_layer_prior(w))
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = to_dev(x, dt)
    ref = oracle.layer_forward(x["k"], x["q"], x["v"], x["w"], x["a"], x["p"], x["lam0"], x["eta0"])
    full = kla.layer_forward(d["k"], d["q"], d["v"], d["w"], d["a"], d["p"], d["lam0"], d["eta0"])
    T1 = 50
    pre = kla.layer_forward(d["k"][:, :T1].contiguous(), d["q"][:, :T1].contiguous(), d["v"][:, :T1].contiguous(),
                            d["w"][:, :T1].contiguous(), d["a"], d["p"], d["lam0"], d["eta0"])
    lam, eta = pre[2].clone(), pre[3].clone()
    ys, ss = [], []
    for t in range(T1, w.T):
        y, s = kla.layer_step(d["k"][:, t].contiguous(), d["q"][:, t].contiguous(), d["v"][:, t].contiguous(),
                              d["w"][:, t].contiguous(), d["a"], d["p"], lam, eta)
        ys.append(y.clone())
        ss.append(s.clone())
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {"y": torch.stack(ys, 1).double().cpu().numpy(), "s": torch.stack(ss, 1).double().cpu().numpy(),
           "lam_T": lam.double().cpu().numpy(), "eta_T": eta.double().cpu().numpy()}
    tail = {"y": ref["y"][:, T1:], "s": ref["s"][:, T1:], "lam_T": ref["lam_T"], "eta_T": ref["eta_T"]}
    errs = layer_errors(got, tail)
    assert max(errs.values()) <= 1e-5, errs
    own = {"y": full[0][:, T1:].double().cpu().numpy(), "s": full[1][:, T1:].double().cpu().numpy(),
           "lam_T": full[2].double().cpu().numpy(), "eta_T": full[3].double().cpu().numpy()}
    assert max(layer_errors(got, own).values()) <= 2e-6


def test_layer_negative_decay_and_no_process_noise():
    """Channels with negative decay (the gate follows the sign of a) and
    channels without process noise (p = 0, the affine Moebius case; there the
    precision grows like a^(-2t), so those channels take |a| = 0.995 to stay in
    fp32 range over 200 tokens), set by a fixed pattern over the channel
    index."""
    import dataclasses
    kla = _kla()
    w = dataclasses.replace(wl.LAYER_WORKLOADS["layer"].with_shape(B=2, T=200, H=2, D=4, Ns=16), dtype="f32")
    x = wl.generate_layer(w)
    x.update(wl.random_layer_prior(w))
    idx = np.arange(x["a"].size).reshape(x["a"].shape)
    x["a"] = np.where(idx % 3 == 0, -x["a"], x["a"]).astype(np.float32)
    no_noise = idx % 4 == 1
    x["p"] = np.where(no_noise, 0.0, x["p"]).astype(np.float32)
    x["a"] = np.where(no_noise, 0.995 * np.sign(x["a"]), x["a"]).astype(np.float32)
    d = to_dev(x, torch.float32)
    out = kla.layer_forward(d["k"], d["q"], d["v"], d["w"], d["a"], d["p"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(("y", "s", "lam_T", "eta_T"), out)}
    ref = oracle.layer_forward(x["k"], x["q"], x["v"], x["w"], x["a"], x["p"], x["lam0"], x["eta0"])
    errs = layer_errors(got, ref)
    assert max(errs.values()) <= 1e-5, errs
