"""kla_scan_forward (CUDA, through the C ABI) against the fp64 oracle."""
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


@pytest.fixture(params=[1, 2], ids=["chunked", "stream"])
def kernel(request):
    """Force one of the two forward kernels (1: chunks exchange carries through
    the workspace; 2: channel-owning streaming kernel, where its geometry holds)."""
    kla = _kla()
    kla.debug_force_forward_kernel(request.param)
    yield request.param
    kla.debug_force_forward_kernel(0)


def _run_full(w, **kw):
    """Device run + oracle over every channel (small shapes)."""
    kla = _kla()
    x = wl.generate(w)
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], torch.from_numpy(x["lam0"]).to(DEV),
                           torch.from_numpy(x["eta0"]).to(DEV), **kw)
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: (None if o is None else o.double().cpu().numpy()) for k, o in zip(parity.OUTPUTS, out)}
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], threads=8)
    return got, ref, x


# (B, T, H, N): tile-aligned, ragged chunk tail, ragged channel tile, tiny and
# odd shapes that take the plain-load path, long enough for deep look-back.
SHAPES = [
    (1, 256, 1, 64),     # the tiny workload's shape
    (2, 200, 3, 40),     # HN = 120: ragged channel tile, ragged last chunk (TMA path)
    (3, 130, 1, 7),      # HN = 7: plain-load path, ragged everything
    (1, 1, 1, 1),        # one token, one channel
    (2, 63, 2, 32),      # T shorter than a chunk
    (1, 4099, 2, 64),    # 65 chunks: multi-hop look-back
    (5, 96, 4, 16),      # B > 1 with a second chunk
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("family", ["tiny", "stiff", "lm_layer"])
def test_parity_small_shapes(shape, family, kernel):
    B, T, H, N = shape
    w = wl.WORKLOADS[family].with_shape(B=B, T=T, H=H, N=N)
    got, ref, _ = _run_full(w)
    parity.assert_parity(got, ref, parity.RTOL[w.dtype], time_axis=1, what=f"{family} {shape}")


def test_tiny_workload_exact_sizes(kernel):
    w = wl.WORKLOADS["tiny"]
    got, ref, _ = _run_full(w)
    errs = parity.assert_parity(got, ref, parity.RTOL["f32"], time_axis=1, what="tiny")
    print("tiny max errors", errs)


def test_optional_outputs_skipped(kernel):
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=300, H=2, N=64)
    full, ref, _ = _run_full(w)
    part, _, _ = _run_full(w, want_mu=False, want_var=False)
    assert part["mu"] is None and part["var"] is None
    np.testing.assert_array_equal(full["lam"], part["lam"])
    np.testing.assert_array_equal(full["eta"], part["eta"])


def test_tma_and_plain_paths_agree():
    """The same inputs through the chunked kernel's TMA path (16-byte aligned)
    and its plain-load path (inputs offset by one element) give bit-identical
    outputs."""
    kla = _kla()
    kla.debug_force_forward_kernel(1)
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=700, H=2, N=64)
    x = wl.generate(w)
    outs = []
    for offset in (0, 1):
        d = {}
        for k in wl.INPUT_NAMES:
            buf = torch.empty(x[k].size + offset, dtype=torch.float32, device=DEV)
            d[k] = buf[offset:].view(x[k].shape)
            d[k].copy_(torch.from_numpy(x[k]))
        o = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], torch.from_numpy(x["lam0"]).to(DEV),
                             torch.from_numpy(x["eta0"]).to(DEV))
        outs.append([t.cpu() for t in o])
    kla.debug_force_forward_kernel(0)
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_kernels_agree_to_rounding():
    """The two forward kernels chunk the scan differently; their outputs agree
    within the fp32 tolerance (and each matches the oracle elsewhere)."""
    kla = _kla()
    w = wl.WORKLOADS["stiff"].with_shape(B=8, T=3000, H=2, N=64)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
    res = []
    for which in (1, 2):
        kla.debug_force_forward_kernel(which)
        assert kla.forward_plan(d["a"], d["p"], d["phi"], d["b"])[0] == which
        o = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
        res.append({k: t.double().cpu().numpy() for k, t in zip(parity.OUTPUTS, o)})
    kla.debug_force_forward_kernel(0)
    parity.assert_parity(res[1], res[0], 2e-6, time_axis=1, what="stream vs chunked")


def test_workspace_contents_do_not_matter(kernel):
    kla = _kla()
    w = wl.WORKLOADS["stiff"].with_shape(B=3, T=500, H=2, N=64)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
    ws = kla.new_workspace(w.B, w.T, w.H, w.N, torch.float32, DEV)
    results = []
    for fill in (0x00, 0xFF, 0x5A):
        ws.fill_(fill)
        o = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"], workspace=ws)
        results.append([t.clone() for t in o])
    for r in results[1:]:
        for a, b in zip(results[0], r):
            assert torch.equal(a, b)


def test_empty_problems():
    kla = _kla()
    for shape in ((0, 5, 1, 4), (1, 0, 1, 4), (1, 5, 0, 4)):
        B, T, H, N = shape
        z = torch.zeros(shape, device=DEV)
        pri = torch.ones((B, H, N), device=DEV)
        out = kla.scan_forward(z, z, z, z, pri, pri * 0)
        assert out[0].shape == shape
    torch.cuda.synchronize()
    assert kla.get_error() == 0


def test_prefill_then_decode_continues_the_filter(kernel):
    """The last row of a forward scan is the decode state: forward over T1,
    then T2 decode steps, equals the oracle over T1 + T2 tokens."""
    kla = _kla()
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=150, H=2, N=64)
    x = wl.generate(w)
    T1 = 100
    d = {k: torch.from_numpy(np.ascontiguousarray(x[k])).to(DEV) for k in x}
    lam, eta, _, _ = kla.scan_forward(*(d[k][:, :T1].contiguous() for k in wl.INPUT_NAMES),
                                      d["lam0"], d["eta0"])
    ls, es = lam[:, -1].contiguous(), eta[:, -1].contiguous()
    mu = torch.empty_like(ls)
    var = torch.empty_like(ls)
    for t in range(T1, w.T):
        kla.scan_step(*(d[k][:, t].contiguous() for k in wl.INPUT_NAMES), ls, es, mu_out=mu, var_out=var)
    torch.cuda.synchronize()
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    got = {"lam": ls.double().cpu().numpy(), "eta": es.double().cpu().numpy(),
           "mu": mu.double().cpu().numpy(), "var": var.double().cpu().numpy()}
    last = {k: ref[k][:, -1] for k in parity.OUTPUTS}
    # time axis is gone; scale eta / mu by the channel's rms over the whole sequence
    rms = {k: np.sqrt(np.mean(ref[k] ** 2, axis=1)) for k in ("eta", "mu")}
    for k in ("lam", "var"):
        assert np.max(np.abs(got[k] - last[k]) / last[k]) <= 1e-5, k
    for k in ("eta", "mu"):
        assert np.max(np.abs(got[k] - last[k]) / (np.abs(last[k]) + rms[k])) <= 1e-5, k


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny", "lm_layer", "long", "stiff"])
def test_workload_full_size_sampled(name):
    """Full-size workloads, launched exactly as the benchmark launches them
    (default kernel choice), then with each forward kernel forced; the oracle
    checks a seeded sample of whole channels (every token)."""
    kla = _kla()
    w = wl.WORKLOADS[name]
    sample = wl.channel_sample(w, 48)
    d, sampled = parity.to_device(w, DEV, sample)
    ref = parity.oracle_on_sample(sampled, np.ones(len(sample)), np.zeros(len(sample)))
    HN = w.H * w.N
    try:
        for which in (0, 1, 2):
            kla.debug_force_forward_kernel(which)
            out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
            torch.cuda.synchronize()
            assert kla.get_error() == 0
            got = {k: parity.gather_channels(o, sample, HN) for k, o in zip(parity.OUTPUTS, out)}
            errs = parity.assert_parity(got, ref, parity.RTOL[w.dtype], time_axis=0,
                                        what=f"{name} kernel={which}")
            print(name, "kernel", which, "max errors", errs)
            # properties over every output element
            lam = out[0]
            assert bool(torch.isfinite(lam).all()) and bool((lam > 0).all())
            assert bool(torch.isfinite(out[1]).all())
            vl = out[3] * lam
            assert float((vl - 1).abs().max()) < 1e-6
            del out, lam, vl
            torch.cuda.empty_cache()
    finally:
        kla.debug_force_forward_kernel(0)


def test_bitwise_reproducible(kernel):
    """The carry is composed in a fixed order, so repeated calls agree bit for bit."""
    kla = _kla()
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=6000, H=4, N=64)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV) for k in x}
    first = [t.clone() for t in kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])]
    for _ in range(5):
        again = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
        for a, b in zip(first, again):
            assert torch.equal(a, b)


def test_plan_matches_workloads():
    """On a B200 the standard workloads take the streaming kernel except the
    tiny one (2 tiles of 32 channels cannot occupy the GPU); 64 tiles take it
    for short sequences (at most 16 chunks) and not for longer ones."""
    kla = _kla()
    for name, expect in (("tiny", 1), ("lm_layer", 2), ("long", 2), ("stiff", 2)):
        w = wl.WORKLOADS[name]
        dt = parity.torch_dtype(w)
        z = torch.empty((w.B, w.T, w.H, w.N), dtype=dt, device=DEV)
        assert kla.forward_plan(z, z, z, z)[0] == expect, name
        del z
    for T, expect in ((512, (2, 1)), (1024, (1, 2))):
        z = torch.empty((32, T, 1, 64), device=DEV)
        assert kla.forward_plan(z, z, z, z) == expect, T
        del z


SPECIAL = wl.SPECIAL_CASES
_special_inputs = wl.special_inputs


@pytest.mark.parametrize("kind", SPECIAL)
def test_special_cases_forward(kind, kernel):
    kla = _kla()
    x = _special_inputs(kind)
    d = {k: torch.from_numpy(v).to(DEV) for k, v in x.items()}
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, out)}
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    parity.assert_parity(got, ref, 1e-5, time_axis=1, what=kind)


@pytest.mark.parametrize("kind", SPECIAL)
def test_special_cases_decode(kind):
    kla = _kla()
    x = _special_inputs(kind, T=60)
    d = {k: torch.from_numpy(v).to(DEV) for k, v in x.items()}
    lam, eta = d["lam0"].clone(), d["eta0"].clone()
    mu, var = torch.empty_like(lam), torch.empty_like(lam)
    mus = []
    for t in range(x["a"].shape[1]):
        kla.scan_step(*(d[k][:, t].contiguous() for k in wl.INPUT_NAMES), lam, eta, mu_out=mu, var_out=var)
        mus.append(mu.clone())
    torch.cuda.synchronize()
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    got = {"mu": torch.stack(mus, 1).double().cpu().numpy()}
    parity.assert_parity(got, {"mu": ref["mu"]}, 1e-5, time_axis=1, what=kind)
    assert np.max(np.abs(lam.double().cpu().numpy() - ref["lam"][:, -1]) / ref["lam"][:, -1]) <= 1e-5


@pytest.mark.parametrize("family,shape", [
    ("stiff", dict(B=160, T=300, H=1, N=32)),        # 160 tiles of 32 channels, 10 chunks, ragged
    ("lm_layer", dict(B=5, T=200, H=16, N=128)),     # bf16: 160 tiles of 64 channels, 13 chunks
])
def test_ticketed_whole_tiles_parity(family, shape):
    """More tiles than SMs, one run each, long enough to be taken by ticket
    (a CTA on a faster SM takes more of them): the plan reports the clear
    launch, every element matches the oracle, and a second call is
    bit-identical whatever order the tickets were taken in."""
    kla = _kla()
    w = wl.WORKLOADS[family].with_shape(**shape)
    x = wl.generate(w)
    dt = parity.torch_dtype(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(dt) for k in wl.INPUT_NAMES}
    for k in ("lam0", "eta0"):
        d[k] = torch.from_numpy(x[k]).to(DEV)
    assert kla.forward_plan(d["a"], d["p"], d["phi"], d["b"]) == (2, 2)
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, out)}
    xin = {k: torch.from_numpy(x[k]).to(dt).double().numpy() for k in wl.INPUT_NAMES}
    ref = oracle.forward(xin["a"], xin["p"], xin["phi"], xin["b"], x["lam0"], x["eta0"], threads=8)
    parity.assert_parity(got, ref, parity.RTOL[w.dtype], time_axis=1, what=f"{family} ticketed tiles")
    again = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    for a_, b_ in zip(out, again):
        assert torch.equal(a_, b_)


def test_run_split_parity_two_channels():
    """bf16, 320 tiles of 64 channels: the two-channel kernel cuts each tile
    into 4 runs of decreasing length (the last tickets the shortest); every
    element against the oracle on the bf16-rounded inputs."""
    kla = _kla()
    w = wl.WORKLOADS["lm_layer"].with_shape(B=10, T=1024, H=16, N=128)
    x = wl.generate(w)
    d = {k: torch.from_numpy(x[k]).to(DEV).to(torch.bfloat16) for k in wl.INPUT_NAMES}
    for k in ("lam0", "eta0"):
        d[k] = torch.from_numpy(x[k]).to(DEV)
    assert kla.forward_plan(d["a"], d["p"], d["phi"], d["b"]) == (2, 2)
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, out)}
    xin = {k: d[k].double().cpu().numpy() for k in wl.INPUT_NAMES}
    ref = oracle.forward(xin["a"], xin["p"], xin["phi"], xin["b"], x["lam0"], x["eta0"], threads=8)
    parity.assert_parity(got, ref, parity.RTOL["f32"], time_axis=1, what="two-channel run split")


def test_run_split_parity():
    """320 tiles of 32 channels do not divide evenly over the SMs, so the
    streaming kernel cuts each tile's sequence into runs taken by ticket; a
    run enters with the state the previous run published.  Every element
    against the oracle, and the plan reports the extra clear launch."""
    kla = _kla()
    w = wl.WORKLOADS["tiny"].with_shape(B=10, T=1024, H=1, N=1024)
    x = wl.generate(w)
    d = {k: torch.from_numpy(v).to(DEV) for k, v in x.items()}
    kernel, launches = kla.forward_plan(d["a"], d["p"], d["phi"], d["b"])
    assert kernel == 2
    out = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    torch.cuda.synchronize()
    assert kla.get_error() == 0
    got = {k: o.double().cpu().numpy() for k, o in zip(parity.OUTPUTS, out)}
    ref = oracle.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], threads=8)
    parity.assert_parity(got, ref, 1e-5, time_axis=1, what="run split")
    print("plan", kernel, launches)
    again = kla.scan_forward(d["a"], d["p"], d["phi"], d["b"], d["lam0"], d["eta0"])
    for a_, b_ in zip(out, again):
        assert torch.equal(a_, b_)  # deterministic despite dynamic tickets
