"""kla_scan_backward (CUDA, through the C ABI) against the fp64 oracle's
reverse-mode gradients.

The device backward consumes the device forward's fp32 lambda / eta; the
oracle recomputes its own fp64 forward.  Every gradient crosses zero, so each
uses the rms-scaled test |x - ref| <= rtol (|ref| + rms(ref)), rms over the
time axis (over channels for the prior's gradients).  rtol = 1e-5 for fp32
inputs, 2e-2 for bf16 inputs (whose input gradients are stored in bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from kalman_linear_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GRADS = ("a", "p", "phi", "b")


def _kla():
    import kalman_linear_attention_b200 as kla
    return kla


@pytest.fixture(params=[1, 2], ids=["per-channel", "stream"])
def kernel(request):
    """Force one of the two backward kernels (1: one thread per channel; 2: the
    channel-owning streaming kernel, where its geometry holds)."""
    kla = _kla()
    kla.debug_force_backward_kernel(request.param)
    yield request.param
    kla.debug_force_backward_kernel(0)


def scaled_errors(got, ref, time_axis=1):
    errs = {}
    for k, r in ref.items():
        g = got[k]
        if g is None:
            continue
        g = np.asarray(g, dtype=np.float64)
        r = np.asarray(r, dtype=np.float64)
        assert g.shape == r.shape, (k, g.shape, r.shape)
        if g.size == 0:
            errs[k] = 0.0
            continue
        if not np.all(np.isfinite(g)):
            errs[k] = float("inf")
            continue
        axis = None if k in ("lam0", "eta0") else time_axis
        rms = np.sqrt(np.mean(r * r, axis=axis, keepdims=axis is not None))
        errs[k] = float(np.max(np.abs(g - r) / (np.abs(r) + rms + 1e-300)))
    return errs


def assert_grad_parity(got, ref, rtol, what=""):
    errs = scaled_errors(got, ref)
    bad = {k: v for k, v in errs.items() if not v <= rtol}
    assert not bad, f"{what}: gradient errors above rtol={rtol:g}: {bad} (all: {errs})"
    return errs


def run_backward(w, present=(0, 1, 2, 3), want=(True,) * 6, prior="random"):
    """Device forward + backward of workload w with the seeded output
    gradients listed in `present`; returns (device grads as host fp64 or None,
    oracle grads)."""
    kla = _kla()
    x = wl.generate(w)
    if prior == "random":
        x.update(wl.random_prior(w))
    go = wl.generate_output_grads(w)
    gsel = [go[k] if i in present else None for i, k in enumerate(wl.GRAD_NAMES)]
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    lam0 = torch.from_numpy(x["lam0"]).to(DEV)
    eta0 = torch.from_numpy(x["eta0"]).to(DEV)
    lam, eta, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], lam0, eta0,
                                      want_mu=False, want_var=False)
    gdev = [None if g is None else torch.from_numpy(g).to(DEV) for g in gsel]
    out = kla.scan_backward(d["a"], d["p"], lam0, eta0, lam, eta, *gdev, want=want)
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: (None if o is None else o.double().cpu().numpy())
           for k, o in zip(GRADS + ("lam0", "eta0"), out)}
    ref = oracle.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], *gsel, threads=8)
    return got, ref


# (B, T, H, N): whole chunks, ragged last chunk, ragged channel tile, shapes
# only the per-channel kernel takes, one token, a long multi-chunk sequence.
SHAPES = [
    (1, 256, 1, 64),     # the tiny workload's shape
    (2, 200, 3, 40),     # HN = 120: ragged channel tile, ragged last chunk
    (3, 130, 1, 7),      # HN = 7: per-channel kernel only
    (1, 1, 1, 32),       # one token
    (1, 1, 1, 1),        # one token, one channel
    (2, 15, 2, 32),      # T shorter than one backward chunk
    (2, 16, 2, 32),      # exactly one chunk
    (1, 4099, 2, 64),    # many chunks, ragged tail
    (5, 96, 4, 16),      # B > 1
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("family", ["tiny", "stiff", "lm_layer"])
def test_backward_parity_small_shapes(shape, family, kernel):
    B, T, H, N = shape
    w = wl.WORKLOADS[family].with_shape(B=B, T=T, H=H, N=N)
    got, ref = run_backward(w)
    assert_grad_parity(got, ref, parity.RTOL[w.dtype], what=f"{family} {shape}")


@pytest.mark.parametrize("present", [(2,), (0, 3), (1,), (0, 1, 2, 3)], ids=str)
def test_backward_absent_output_gradients(present, kernel):
    """NULL output gradients are zeros (the typical loss reads mu only)."""
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=300, H=2, N=64)
    got, ref = run_backward(w, present=present)
    assert_grad_parity(got, ref, parity.RTOL["f32"], what=f"present {present}")


def test_backward_skipped_outputs_bitwise(kernel):
    """Input gradients not wanted are not written; the rest are bit-identical."""
    w = wl.WORKLOADS["stiff"].with_shape(B=3, T=200, H=2, N=64)
    full, _ = run_backward(w)
    part, _ = run_backward(w, want=(False, True, False, True, False, True))
    assert part["a"] is None and part["phi"] is None and part["lam0"] is None
    for k in ("p", "b", "eta0"):
        np.testing.assert_array_equal(full[k], part[k])


def test_backward_kernels_agree():
    """The per-channel and streaming kernels compute the same gradients (to
    rounding) on a shape both take; each is deterministic run to run."""
    kla = _kla()
    w = wl.WORKLOADS["lm_layer"].with_shape(B=2, T=1000, H=2, N=64)
    res = {}
    try:
        for k in (1, 2, 2):
            kla.debug_force_backward_kernel(k)
            got, ref = run_backward(w)
            if k in res:
                for n in got:
                    np.testing.assert_array_equal(got[n], res[k][n])
            res[k] = got
    finally:
        kla.debug_force_backward_kernel(0)
    errs = scaled_errors(res[1], res[2])
    assert max(errs.values()) <= parity.RTOL["bf16"], errs


def test_backward_run_split():
    """Enough tiles that each tile's sequence is cut into runs handed over
    through the workspace (the plan reports the extra clear launch)."""
    kla = _kla()
    w = wl.WORKLOADS["stiff"].with_shape(B=80, T=512, H=2, N=64)  # 320 tiles of 32 channels
    a = torch.empty((w.B, w.T, w.H, w.N), device=DEV)
    assert kla.backward_plan(a, a) == (2, 2)
    got, ref = run_backward(w)
    assert_grad_parity(got, ref, parity.RTOL["f32"], what="run split")


def test_backward_ticketed_whole_tiles():
    """More tiles than SMs, one run each, long enough to be taken whole by
    ticket: the plan reports the clear launch and the gradients match the
    oracle."""
    kla = _kla()
    w = wl.WORKLOADS["stiff"].with_shape(B=160, T=300, H=1, N=32)  # 160 tiles, 19 chunks
    a = torch.empty((w.B, w.T, w.H, w.N), device=DEV)
    assert kla.backward_plan(a, a) == (2, 2)
    got, ref = run_backward(w)
    assert_grad_parity(got, ref, parity.RTOL["f32"], what="ticketed whole tiles")


def test_backward_empty_and_zero_length():
    kla = _kla()
    z = torch.empty((2, 0, 1, 32), device=DEV)
    lam0 = torch.rand((2, 1, 32), device=DEV) + 0.5
    eta0 = torch.randn((2, 1, 32), device=DEV)
    out = kla.scan_backward(z, z, lam0, eta0, z, z, z, None, None, None)
    torch.cuda.synchronize()
    assert out[0].shape == (2, 0, 1, 32)
    assert torch.count_nonzero(out[4]) == 0 and torch.count_nonzero(out[5]) == 0
    e = torch.empty((0, 5, 1, 32), device=DEV)
    kla.scan_backward(e, e, torch.empty((0, 1, 32), device=DEV), torch.empty((0, 1, 32), device=DEV),
                      e, e, e)
    assert kla.get_error() == 0


def test_autograd_matches_oracle():
    """torch.autograd through KalmanFilterScan (forward and backward kernels)
    against the oracle's gradients of the same loss."""
    kla = _kla()
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=333, H=2, N=32)
    x = wl.generate(w)
    x.update(wl.random_prior(w))
    go = wl.generate_output_grads(w)
    leaves = {k: torch.from_numpy(x[k]).to(DEV).requires_grad_(True)
              for k in wl.INPUT_NAMES + ("lam0", "eta0")}
    lam, eta, mu, var = kla.kalman_filter(*(leaves[k] for k in wl.INPUT_NAMES + ("lam0", "eta0")))
    loss = sum((torch.from_numpy(go[g]).to(DEV) * o).sum()
               for g, o in zip(wl.GRAD_NAMES, (lam, eta, mu, var)))
    loss.backward()
    ref = oracle.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"],
                          *(go[g] for g in wl.GRAD_NAMES))
    got = {k: leaves[k].grad.double().cpu().numpy() for k in GRADS + ("lam0", "eta0")}
    assert_grad_parity(got, ref, parity.RTOL["f32"], what="autograd")
    # a loss on mu alone leaves the other outputs' gradients absent
    for t in leaves.values():
        t.grad = None
    _, _, mu, _ = kla.kalman_filter(*(leaves[k] for k in wl.INPUT_NAMES + ("lam0", "eta0")))
    (torch.from_numpy(go["g_mu"]).to(DEV) * mu).sum().backward()
    ref = oracle.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], g_mu=go["g_mu"])
    got = {k: leaves[k].grad.double().cpu().numpy() for k in GRADS + ("lam0", "eta0")}
    assert_grad_parity(got, ref, parity.RTOL["f32"], what="autograd, loss on mu")


def _sampled_full_size(name, count):
    """Full-size workload on the device (forward + backward, the bench's
    launch configuration); the oracle on `count` sampled channels."""
    kla = _kla()
    w = wl.WORKLOADS[name]
    sample = wl.channel_sample(w, count)
    d, sampled = parity.to_device(w, DEV, sample)
    B, T, H, N = w.B, w.T, w.H, w.N
    HN = H * N
    lam, eta, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"],
                                      want_mu=False, want_var=False)
    gdev = {k: torch.empty((B, T, H, N), device=DEV) for k in wl.GRAD_NAMES}
    flat = {k: v.view(B * T, HN) for k, v in gdev.items()}
    gs = {k: np.empty((T, len(sample)), dtype=np.float32) for k in wl.GRAD_NAMES}
    sb, shn = np.divmod(sample, HN)
    for r0, r1, blk in wl.iter_output_grad_rows(w):
        rows = np.arange(r0, r1)
        for k in wl.GRAD_NAMES:
            xb = blk[k].reshape(r1 - r0, HN)
            flat[k][r0:r1].copy_(torch.from_numpy(xb))
            for j in range(len(sample)):
                m = (rows // T) == sb[j]
                if m.any():
                    gs[k][rows[m] % T, j] = xb[m, shn[j]]
    out = kla.scan_backward(d["a"], d["p"], d["lam0"], d["eta0"], lam, eta,
                            *(gdev[k] for k in wl.GRAD_NAMES))
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: parity.gather_channels(o, sample, HN) for k, o in zip(GRADS, out[:4])}
    got["lam0"] = out[4].view(-1)[torch.as_tensor(sample, device=DEV)].double().cpu().numpy()
    got["eta0"] = out[5].view(-1)[torch.as_tensor(sample, device=DEV)].double().cpu().numpy()
    K = len(sample)
    lam0 = d["lam0"].view(-1)[torch.as_tensor(sample, device=DEV)].double().cpu().numpy()
    eta0 = d["eta0"].view(-1)[torch.as_tensor(sample, device=DEV)].double().cpu().numpy()
    r = oracle.backward(*(sampled[k].reshape(1, T, 1, K) for k in wl.INPUT_NAMES),
                        lam0.reshape(1, 1, K), eta0.reshape(1, 1, K),
                        *(gs[k].reshape(1, T, 1, K) for k in wl.GRAD_NAMES), threads=8)
    ref = {k: r[k].reshape(T, K) for k in GRADS}
    ref["lam0"] = r["lam0"].reshape(K)
    ref["eta0"] = r["eta0"].reshape(K)
    errs = scaled_errors(got, ref, time_axis=0)
    return w, errs


@pytest.mark.parametrize("name,count", [("long", 48), ("lm_layer", 128), ("stiff", 512)])
def test_backward_full_size_sampled(name, count):
    w, errs = _sampled_full_size(name, count)
    print(name, "backward max scaled errors", errs)
    assert max(errs.values()) <= parity.RTOL[w.dtype], errs


@pytest.mark.parametrize("kind", wl.SPECIAL_CASES)
def test_backward_special_cases(kind, kernel):
    """Gradients in the degenerate cases of the method: no process noise
    (a near +-1), no observation (phi = b = 0), the precision sum (a = 1,
    p = 0), negative decay and mixed zeros, against the oracle, with all four
    output gradients present."""
    kla = _kla()
    x = wl.special_inputs(kind, T=300)
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=300, H=2, N=48)
    go = wl.generate_output_grads(w)
    d = {k: torch.from_numpy(v).to(DEV) for k, v in x.items()}
    lam, eta, _, _ = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"],
                                      want_mu=False, want_var=False)
    g = [torch.from_numpy(go[k]).to(DEV) for k in wl.GRAD_NAMES]
    out = kla.scan_backward(d["a"], d["p"], d["lam0"], d["eta0"], lam, eta, *g)
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(GRADS + ("lam0", "eta0"), out)}
    ref = oracle.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"],
                          *(go[k] for k in wl.GRAD_NAMES), threads=8)
    assert_grad_parity(got, ref, parity.RTOL["f32"], what=kind)
