"""Pins that tie the fp64 oracle to facts other than its own code.

Each ``pin_*`` function takes an ``oracle.Oracle`` handle and raises
``AssertionError`` when the oracle disagrees with the fact it checks.  The facts
come from the pages' definitions and from mathematics, never from the oracle:

* exact rational arithmetic (Python ``fractions``) of the Moebius precision map
  M_t = [[1 + p phi, a^2 phi], [p, a^2]] and of the precision-ratio gate
  f_t = a_t / (a_t^2 + p_t lambda_{t-1}) -- the matrix form of the KLA review
  ("What carries the argument", and its reference [13] on linear-fractional
  maps) -- against the oracle's covariance-form filter;
* the Riccati fixed point of constant parameters, via ``numpy.roots``;
* special cases with textbook closed forms: the plain precision sum and the
  precision-weighted average of observations (a = 1, p = 0), the affine case
  without process noise (p = 0, "c = 0 gives az + b" in reference [13]), the
  no-observation case (phi = 0: the update leaves the prior unchanged, primer
  section 5.1) with its geometric-series variance;
* identities of the map: f_t^2 = d lambda_t / d lambda_{t-1}, and the gate
  product over a span equals prod(a) / (C lambda_s + D) from the matrix product;
* invariants: lambda_t > 0, lambda_t - phi_t > 0, var * lambda = 1, mu * lambda = eta.

The same functions run against deliberately broken copies of the oracle in
``test_oracle_mutants.py``; each broken copy must fail at least one pin.
"""
from __future__ import annotations

import math
from fractions import Fraction as Fr

import numpy as np

from kalman_linear_attention_b200 import workloads as wl


# ---------------------------------------------------------------- helpers
def _rel_close(got, ref, rtol, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bound = rtol * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: max rel err {np.max(err / np.maximum(np.abs(ref), 1e-300)):.3e}"
                           f" > {rtol:g}")


def _scaled_close(got, ref, rtol, what, axis=1):
    """|got - ref| <= rtol (|ref| + rms(ref along the time axis))."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = np.sqrt(np.mean(ref * ref, axis=axis, keepdims=True)) if ref.ndim > 1 else \
        np.sqrt(np.mean(ref * ref))
    bound = rtol * (np.abs(ref) + rms)
    err = np.abs(got - ref)
    assert not (err > bound).any(), f"{what}: max scaled err {np.max(err / (np.abs(ref) + rms)):.3e}"


def _as4(x):
    """[T] -> [1, T, 1, 1]"""
    return np.asarray(x, dtype=np.float64).reshape(1, -1, 1, 1)


# ---------------------------------------------------- exact rational reference
def _random_fraction(rng, lo, hi, den_max):
    return Fr(int(rng.integers(lo, hi + 1)), int(rng.integers(1, den_max + 1)))


def exact_moebius_filter(a, p, phi, b, lam0, eta0):
    """Exact rationals: lambda_t from the explicit Moebius matrix product
    M_t ... M_1 applied to lambda_0, eta_t from the gated affine recursion."""
    T = len(a)
    # running product P = M_t ... M_1 as a 2x2 of Fractions
    A, B_, C, D = Fr(1), Fr(0), Fr(0), Fr(1)
    lam_prev, eta = lam0, eta0
    lam_out, eta_out = [], []
    for t in range(T):
        m11, m12 = 1 + p[t] * phi[t], a[t] * a[t] * phi[t]
        m21, m22 = p[t], a[t] * a[t]
        A, B_, C, D = (m11 * A + m12 * C, m11 * B_ + m12 * D,
                       m21 * A + m22 * C, m21 * B_ + m22 * D)
        lam_t = (A * lam0 + B_) / (C * lam0 + D)
        f_t = a[t] / (a[t] * a[t] + p[t] * lam_prev)
        eta = f_t * eta + b[t]
        lam_out.append(lam_t)
        eta_out.append(eta)
        lam_prev = lam_t
    return lam_out, eta_out


def exact_homogeneous_filter(a, p, phi, b, lam0, eta0):
    """Exact rationals: one product of 3x3 block-lower-triangular matrices
    G_t = [[1+p phi, a^2 phi, 0], [p, a^2, 0], [b p, b a^2, a]] applied to
    (lambda_0, 1, eta_0); lambda_t = n_t / d_t and eta_t = h_t / d_t."""
    n, d, h = lam0, Fr(1), eta0
    lam_out, eta_out = [], []
    for t in range(len(a)):
        a2 = a[t] * a[t]
        n, d, h = ((1 + p[t] * phi[t]) * n + a2 * phi[t] * d,
                   p[t] * n + a2 * d,
                   b[t] * p[t] * n + b[t] * a2 * d + a[t] * h)
        lam_out.append(n / d)
        eta_out.append(h / d)
    return lam_out, eta_out


def random_rational_problem(seed, B=2, T=10, H=1, N=3, allow_negative_a=True):
    rng = np.random.default_rng(seed)
    shape = (B, T, H, N)
    fr = {}
    fr["a"] = np.empty(shape, dtype=object)
    fr["p"] = np.empty(shape, dtype=object)
    fr["phi"] = np.empty(shape, dtype=object)
    fr["b"] = np.empty(shape, dtype=object)
    for idx in np.ndindex(shape):
        a = _random_fraction(rng, 1, 9, 8)
        if allow_negative_a and rng.random() < 0.25:
            a = -a
        fr["a"][idx] = a
        fr["p"][idx] = _random_fraction(rng, 0, 6, 8)
        fr["phi"][idx] = _random_fraction(rng, 0, 6, 8)
        fr["b"][idx] = _random_fraction(rng, -6, 6, 8)
    fr["lam0"] = np.empty((B, H, N), dtype=object)
    fr["eta0"] = np.empty((B, H, N), dtype=object)
    for idx in np.ndindex((B, H, N)):
        fr["lam0"][idx] = _random_fraction(rng, 1, 6, 4)
        fr["eta0"][idx] = _random_fraction(rng, -4, 4, 4)
    return fr


def exact_solution(fr, method=exact_moebius_filter):
    B, T, H, N = fr["a"].shape
    lam = np.empty((B, T, H, N), dtype=object)
    eta = np.empty((B, T, H, N), dtype=object)
    for bi in range(B):
        for h in range(H):
            for n in range(N):
                sl = (bi, slice(None), h, n)
                l, e = method(list(fr["a"][sl]), list(fr["p"][sl]), list(fr["phi"][sl]),
                              list(fr["b"][sl]), fr["lam0"][bi, h, n], fr["eta0"][bi, h, n])
                lam[sl] = l
                eta[sl] = e
    return lam, eta


def _to_f64(obj_arr):
    return np.vectorize(float, otypes=[np.float64])(obj_arr)


# ------------------------------------------------------------------- pins
def pin_exact_rational(orc, seeds=(1, 2, 3)):
    """fp64 oracle == exact Moebius/affine solution to ~1e-13 (B=2 catches
    batch-stride mistakes, N=3 and per-channel priors catch channel mix-ups,
    negative a catches a^2 vs a in the gate)."""
    for seed in seeds:
        fr = random_rational_problem(seed)
        lam_x, eta_x = exact_solution(fr)
        f64 = {k: _to_f64(v) for k, v in fr.items()}
        out = orc.forward(f64["a"], f64["p"], f64["phi"], f64["b"], f64["lam0"], f64["eta0"])
        lam_r = _to_f64(lam_x)
        eta_r = _to_f64(eta_x)
        mu_r = _to_f64(eta_x / lam_x)
        var_r = _to_f64(1 / lam_x)
        _rel_close(out["lam"], lam_r, 1e-13, f"lambda (seed {seed})")
        _rel_close(out["var"], var_r, 1e-13, f"var (seed {seed})")
        _scaled_close(out["eta"], eta_r, 1e-13, f"eta (seed {seed})")
        _scaled_close(out["mu"], mu_r, 1e-13, f"mu (seed {seed})")


def pin_exact_rational_step(orc, seed=7):
    """The one-token decode step, iterated, equals the exact solution too."""
    fr = random_rational_problem(seed, B=1, T=8, H=2, N=2)
    lam_x, eta_x = exact_solution(fr)
    f64 = {k: _to_f64(v) for k, v in fr.items()}
    lam, eta = f64["lam0"][0].copy(), f64["eta0"][0].copy()
    for t in range(f64["a"].shape[1]):
        o = orc.step(f64["a"][0, t], f64["p"][0, t], f64["phi"][0, t], f64["b"][0, t], lam, eta)
        lam, eta = o["lam"], o["eta"]
        _rel_close(lam, _to_f64(lam_x[0, t]), 1e-13, f"step lambda t={t}")
        _scaled_close(eta.ravel(), _to_f64(eta_x[0, t]).ravel(), 1e-13, f"step eta t={t}")
        _rel_close(o["var"], _to_f64(1 / lam_x[0, t]), 1e-13, f"step var t={t}")
        _scaled_close(o["mu"].ravel(), _to_f64(eta_x[0, t] / lam_x[0, t]).ravel(), 1e-13,
                      f"step mu t={t}")


def riccati_fixed_point(a, p, phi):
    """Positive root of p lam^2 + (a^2 - 1 - p phi) lam - a^2 phi = 0 (numpy.roots)."""
    roots = np.roots([p, a * a - 1.0 - p * phi, -a * a * phi])
    pos = [r.real for r in roots if abs(r.imag) < 1e-12 and r.real > 0]
    assert len(pos) == 1
    return pos[0]


def pin_riccati(orc):
    """Constant (a, p, phi, b) converge to the Riccati fixed point lambda* and
    to eta* = b / (1 - f*), f* = a / (a^2 + p lambda*)."""
    # worked value: a = 0.75, p = 0.03, phi = 0.3
    lam_star = riccati_fixed_point(0.75, 0.03, 0.3)
    assert abs(lam_star - 15.2521341800603) < 1e-9
    f_star = 0.75 / (0.75 ** 2 + 0.03 * lam_star)
    assert abs(f_star - 0.73524796613) < 1e-9
    rng = np.random.default_rng(11)
    cases = [(0.75, 0.03, 0.3, 0.4), (1.0, 0.01, 0.5, -1.0), (0.5, 1.0, 10.0, 2.0),
             (-0.9, 0.2, 0.05, 1.5)]
    for _ in range(6):
        cases.append((rng.uniform(0.5, 1.0), float(np.exp(rng.uniform(np.log(1e-3), 0))),
                      float(np.exp(rng.uniform(np.log(1e-2), np.log(10)))), rng.standard_normal()))
    T = 6000
    for a, p, phi, b in cases:
        lam_s = riccati_fixed_point(a, p, phi)
        f_s = a / (a * a + p * lam_s)
        eta_s = b / (1.0 - f_s)
        out = orc.forward(_as4(np.full(T, a)), _as4(np.full(T, p)), _as4(np.full(T, phi)),
                          _as4(np.full(T, b)), [[[2.0]]], [[[0.5]]])
        _rel_close(out["lam"][0, -1, 0, 0], lam_s, 1e-11, f"lambda* a={a} p={p} phi={phi}")
        assert abs(out["eta"][0, -1, 0, 0] - eta_s) <= 1e-10 * (abs(eta_s) + 1), \
            f"eta* a={a} p={p} phi={phi}: {out['eta'][0, -1, 0, 0]} vs {eta_s}"
        _rel_close(out["mu"][0, -1, 0, 0], eta_s / lam_s, 1e-10, "mu*")


def pin_precision_sum(orc):
    """a = 1, p = 0: lambda_t = lambda_0 + sum phi, eta_t = eta_0 + sum b, and
    mu_t is the precision-weighted average of the observations y_s = b_s/phi_s
    and the prior mean (numpy.average)."""
    rng = np.random.default_rng(5)
    T = 300
    phi = np.exp(rng.uniform(np.log(1e-2), np.log(10), T))
    y = rng.standard_normal(T) * 3 + 1
    b = phi * y
    lam0, eta0 = 2.5, -1.25
    out = orc.forward(_as4(np.ones(T)), _as4(np.zeros(T)), _as4(phi), _as4(b),
                      [[[lam0]]], [[[eta0]]])
    lam_ref = np.array([lam0 + math.fsum(phi[:t + 1]) for t in range(T)])
    eta_ref = np.array([eta0 + math.fsum(b[:t + 1]) for t in range(T)])
    _rel_close(out["lam"][0, :, 0, 0], lam_ref, 1e-13, "precision sum")
    _scaled_close(out["eta"][0, :, 0, 0], eta_ref, 1e-13, "information sum")
    mu0 = eta0 / lam0
    for t in (0, 1, 17, T - 1):
        ref = np.average(np.concatenate([[mu0], y[:t + 1]]),
                         weights=np.concatenate([[lam0], phi[:t + 1]]))
        got = out["mu"][0, t, 0, 0]
        assert abs(got - ref) <= 1e-12 * (abs(ref) + 1), f"weighted mean t={t}: {got} vs {ref}"


def pin_no_process_noise(orc):
    """p = 0 (affine Moebius case): brute-force sums of products
    lambda_t = lambda_0 prod a^-2 + sum_s phi_s prod_{j>s} a_j^-2 and
    eta_t = eta_0 prod a^-1 + sum_s b_s prod_{j>s} a_j^-1."""
    rng = np.random.default_rng(9)
    T = 40
    a = rng.uniform(0.8, 1.2, T) * np.where(rng.random(T) < 0.3, -1.0, 1.0)
    phi = rng.uniform(0.0, 2.0, T)
    b = rng.standard_normal(T)
    lam0, eta0 = 0.7, 0.3
    out = orc.forward(_as4(a), _as4(np.zeros(T)), _as4(phi), _as4(b), [[[lam0]]], [[[eta0]]])
    for t in range(T):
        lam_ref = lam0 * np.prod(a[:t + 1] ** -2.0)
        eta_ref = eta0 * np.prod(1.0 / a[:t + 1])
        for s in range(t + 1):
            lam_ref += phi[s] * np.prod(a[s + 1:t + 1] ** -2.0)
            eta_ref += b[s] * np.prod(1.0 / a[s + 1:t + 1])
        _rel_close(out["lam"][0, t, 0, 0], lam_ref, 1e-12, f"p=0 lambda t={t}")
        assert abs(out["eta"][0, t, 0, 0] - eta_ref) <= 1e-12 * (abs(eta_ref) + 1), f"p=0 eta t={t}"


def pin_no_observation(orc):
    """phi = 0, b = 0 (missing observations): the update leaves the prior
    unchanged, so with constant a, p the variance is the geometric series
    P_t = a^(2t) P_0 + p (1 - a^(2t)) / (1 - a^2) and mu_t = a^t mu_0."""
    T = 200
    for a, p in ((0.9, 0.05), (1.1, 0.02), (-0.95, 0.3)):
        lam0, eta0 = 4.0, 2.0
        out = orc.forward(_as4(np.full(T, a)), _as4(np.full(T, p)), _as4(np.zeros(T)),
                          _as4(np.zeros(T)), [[[lam0]]], [[[eta0]]])
        t = np.arange(1, T + 1)
        P_ref = a ** (2 * t) / lam0 + p * (1 - a ** (2 * t)) / (1 - a * a)
        _rel_close(out["var"][0, :, 0, 0], P_ref, 1e-12, f"no-obs variance a={a}")
        mu_ref = a ** t * (eta0 / lam0)
        _rel_close(out["mu"][0, :, 0, 0], mu_ref, 1e-12, f"no-obs mean a={a}")


def pin_gate_derivative(orc):
    """f_t^2 = d lambda_t / d lambda_{t-1}: the gate measured on the mean path
    (b = 0, eta_0 = 1 gives eta_1 = f_1) against a central finite difference of
    the precision path."""
    rng = np.random.default_rng(21)
    for _ in range(20):
        a = rng.uniform(0.5, 1.0) * (1 if rng.random() < 0.7 else -1)
        p = float(np.exp(rng.uniform(np.log(1e-3), 0)))
        phi = float(np.exp(rng.uniform(np.log(1e-2), np.log(10))))
        lam0 = float(np.exp(rng.uniform(-1, 3)))
        one = lambda l0, e0, bb: orc.forward(_as4([a]), _as4([p]), _as4([phi]), _as4([bb]),
                                              [[[l0]]], [[[e0]]])
        f1 = one(lam0, 1.0, 0.0)["eta"][0, 0, 0, 0]
        h = 1e-5 * lam0
        d = (one(lam0 + h, 0.0, 0.0)["lam"][0, 0, 0, 0] -
             one(lam0 - h, 0.0, 0.0)["lam"][0, 0, 0, 0]) / (2 * h)
        assert abs(f1 * f1 - d) <= 1e-6 * abs(d), f"f^2={f1 * f1} vs dlam={d}"
        assert np.sign(f1) == np.sign(a), "gate sign must follow a"


def pin_gate_product(orc):
    """Over a span s..t the product of gates equals prod(a) / (C lambda_s + D),
    [[A, B], [C, D]] = M_t ... M_{s+1} (numpy matrix products of the pages'
    M_t).  The gate product is read off the mean path with b = 0, eta_s = 1."""
    rng = np.random.default_rng(33)
    w = wl.WORKLOADS["tiny"]
    for span in (1, 5, 24):
        a = rng.uniform(0.5, 1.0, span)
        p = np.exp(rng.uniform(np.log(1e-3), 0, span))
        phi = np.exp(rng.uniform(np.log(1e-2), np.log(10), span))
        lam_s = 1.7
        out = orc.forward(_as4(a), _as4(p), _as4(phi), _as4(np.zeros(span)), [[[lam_s]]], [[[1.0]]])
        prod = np.eye(2)
        for t in range(span):
            M = np.array([[1 + p[t] * phi[t], a[t] ** 2 * phi[t]], [p[t], a[t] ** 2]])
            prod = M @ prod
            ref = np.prod(a[:t + 1]) / (prod[1, 0] * lam_s + prod[1, 1])
            got = out["eta"][0, t, 0, 0]
            assert abs(got - ref) <= 1e-12 * abs(ref), f"gate product span {t + 1}: {got} vs {ref}"
            lam_ref = (prod[0, 0] * lam_s + prod[0, 1]) / (prod[1, 0] * lam_s + prod[1, 1])
            _rel_close(out["lam"][0, t, 0, 0], lam_ref, 1e-12, "Moebius product")
    del w


def pin_invariants(orc):
    """On every workload's distribution family: lambda_t > 0, the prior
    precision lambda_t - phi_t > 0 ("update never makes things worse"),
    var * lambda = 1 and mu * lambda = eta."""
    for name in ("tiny", "lm_layer", "stiff"):
        w = wl.WORKLOADS[name].with_shape(B=2, T=64, H=2, N=8)
        x = wl.generate(w)
        out = orc.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
        assert np.all(out["lam"] > 0), name
        assert np.all(out["lam"] - x["phi"] > 0), name
        _rel_close(out["var"] * out["lam"], np.ones_like(out["lam"]), 1e-14, f"{name} var*lam")
        _scaled_close(out["mu"] * out["lam"], out["eta"], 1e-14, f"{name} mu*lam")


# ------------------------------------------------------ gradients (backward)
class Dual:
    """Exact forward-mode derivative: value + eps * derivative, eps^2 = 0, with
    Fraction components (so a derivative of the exact filter is exact too)."""

    __slots__ = ("v", "d")

    def __init__(self, v, d=0):
        self.v, self.d = Fr(v), Fr(d)

    @staticmethod
    def _of(x):
        return x if isinstance(x, Dual) else Dual(x)

    def __add__(self, o):
        o = Dual._of(o)
        return Dual(self.v + o.v, self.d + o.d)

    __radd__ = __add__

    def __sub__(self, o):
        o = Dual._of(o)
        return Dual(self.v - o.v, self.d - o.d)

    def __rsub__(self, o):
        return Dual._of(o) - self

    def __mul__(self, o):
        o = Dual._of(o)
        return Dual(self.v * o.v, self.d * o.v + self.v * o.d)

    __rmul__ = __mul__

    def __truediv__(self, o):
        o = Dual._of(o)
        return Dual(self.v / o.v, (self.d * o.v - self.v * o.d) / (o.v * o.v))

    def __rtruediv__(self, o):
        return Dual._of(o) / self


_GRAD_INPUTS = ("a", "p", "phi", "b")


def _exact_loss_gradient(fr, w, bi, h, n):
    """Exact gradient of L = sum_t w_lam lam_t + w_eta eta_t + w_mu mu_t +
    w_var var_t for one channel, one forward-mode pass per input element
    (the exact Moebius/affine filter with a Dual seeded on that element)."""
    T = fr["a"].shape[1]
    sl = (bi, slice(None), h, n)
    base = {k: list(fr[k][sl]) for k in _GRAD_INPUTS}
    base["lam0"], base["eta0"] = fr["lam0"][bi, h, n], fr["eta0"][bi, h, n]
    wl_, we, wm, wv = (list(x[sl]) for x in w)

    def loss_derivative(key, t):
        args = {k: ([Dual(x) for x in v] if isinstance(v, list) else Dual(v)) for k, v in base.items()}
        if t is None:
            args[key] = Dual(base[key], 1)
        else:
            args[key][t] = Dual(base[key][t], 1)
        lam, eta = exact_moebius_filter(args["a"], args["p"], args["phi"], args["b"],
                                        args["lam0"], args["eta0"])
        tot = Fr(0)
        for s in range(T):
            tot += (wl_[s] * lam[s] + we[s] * eta[s] + wm[s] * (eta[s] / lam[s])
                    + wv[s] * (1 / lam[s])).d
        return tot

    g = {k: [loss_derivative(k, t) for t in range(T)] for k in _GRAD_INPUTS}
    g["lam0"] = loss_derivative("lam0", None)
    g["eta0"] = loss_derivative("eta0", None)
    return g


def pin_backward_exact_dual(orc, seeds=(4, 5)):
    """Reverse-mode gradients of the oracle == exact forward-mode derivatives
    (Dual numbers over Fractions) of the exact Moebius/affine filter, for every
    input element, with random rational output gradients (B=2, per-channel
    priors and negative a as in the forward pin)."""
    for seed in seeds:
        fr = random_rational_problem(seed, B=2, T=5, H=1, N=2)
        rng = np.random.default_rng(seed + 100)
        shape = fr["a"].shape
        w = []
        for _ in range(4):
            arr = np.empty(shape, dtype=object)
            for idx in np.ndindex(shape):
                arr[idx] = _random_fraction(rng, -5, 5, 4)
            w.append(arr)
        B, T, H, N = shape
        exact = {k: np.empty(shape, dtype=object) for k in _GRAD_INPUTS}
        exact["lam0"] = np.empty((B, H, N), dtype=object)
        exact["eta0"] = np.empty((B, H, N), dtype=object)
        for bi in range(B):
            for h in range(H):
                for n in range(N):
                    g = _exact_loss_gradient(fr, w, bi, h, n)
                    for k in _GRAD_INPUTS:
                        exact[k][bi, :, h, n] = g[k]
                    exact["lam0"][bi, h, n] = g["lam0"]
                    exact["eta0"][bi, h, n] = g["eta0"]
        f64 = {k: _to_f64(v) for k, v in fr.items()}
        got = orc.backward(f64["a"], f64["p"], f64["phi"], f64["b"], f64["lam0"], f64["eta0"],
                           *[_to_f64(x) for x in w])
        for k in exact:
            ref = _to_f64(exact[k])
            _scaled_close(got[k], ref, 1e-12, f"exact gradient d/d{k} (seed {seed})",
                          axis=1 if ref.ndim == 4 else None)


def _torch_info_form_loss(a, p, phi, b, lam0, eta0, w):
    """The information form of the filter written with torch fp64 ops (the
    Moebius precision map and the precision-ratio gate), for autograd."""
    import torch
    lam, eta = lam0, eta0
    tot = torch.zeros((), dtype=torch.float64)
    for t in range(a.shape[1]):
        at, pt, ft, bt = a[:, t], p[:, t], phi[:, t], b[:, t]
        gate = at / (at * at + pt * lam)
        lam_new = ((1 + pt * ft) * lam + at * at * ft) / (pt * lam + at * at)
        eta = gate * eta + bt
        lam = lam_new
        tot = tot + (w[0][:, t] * lam + w[1][:, t] * eta + w[2][:, t] * (eta / lam)
                     + w[3][:, t] / lam).sum()
    return tot


def pin_backward_autograd(orc):
    """Oracle gradients == torch autograd through the information form
    (Moebius map + gate, fp64) on a random problem with every output gradient
    present, and again with only some present (the others zero)."""
    import torch
    rng = np.random.default_rng(77)
    B, T, H, N = 2, 40, 2, 3
    x = {"a": rng.uniform(0.5, 1.0, (B, T, H, N)) * np.where(rng.random((B, T, H, N)) < 0.2, -1, 1),
         "p": np.exp(rng.uniform(np.log(1e-3), 0, (B, T, H, N))),
         "phi": np.exp(rng.uniform(np.log(1e-2), np.log(10), (B, T, H, N))),
         "b": rng.standard_normal((B, T, H, N)),
         "lam0": np.exp(rng.uniform(-1, 1, (B, H, N))),
         "eta0": rng.standard_normal((B, H, N))}
    w_all = [rng.standard_normal((B, T, H, N)) for _ in range(4)]
    for present in ((0, 1, 2, 3), (2,), (0, 3), (1,)):
        w = [w_all[i] if i in present else None for i in range(4)]
        got = orc.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], *w)
        tx = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in x.items()}
        tw = [torch.tensor(v if v is not None else np.zeros((B, T, H, N)), dtype=torch.float64)
              for v in w]
        loss = _torch_info_form_loss(tx["a"], tx["p"], tx["phi"], tx["b"], tx["lam0"], tx["eta0"], tw)
        loss.backward()
        for k in x:
            ref = tx[k].grad.numpy()
            _scaled_close(got[k], ref, 1e-11, f"autograd d/d{k} (outputs {present})",
                          axis=1 if ref.ndim == 4 else None)


def pin_backward_finite_difference(orc):
    """Oracle gradients == central finite differences of the oracle's own
    (pinned) forward pass, on sampled elements of every input, for a loss on
    all four outputs with workload-like inputs."""
    rng = np.random.default_rng(91)
    w = wl.WORKLOADS["lm_layer"].with_shape(B=2, T=48, H=1, N=3)
    x = dict(wl.generate(w))
    x = {k: np.asarray(v, dtype=np.float64) for k, v in x.items()}
    x["lam0"] = np.exp(rng.uniform(-1, 1, x["lam0"].shape))
    x["eta0"] = rng.standard_normal(x["eta0"].shape)
    gw = [rng.standard_normal(x["a"].shape) for _ in range(4)]
    got = orc.backward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], *gw)

    def loss(arrs):
        o = orc.forward(arrs["a"], arrs["p"], arrs["phi"], arrs["b"], arrs["lam0"], arrs["eta0"])
        return math.fsum(float((g * o[k]).sum()) for g, k in zip(gw, ("lam", "eta", "mu", "var")))

    for k in ("a", "p", "phi", "b", "lam0", "eta0"):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in x[k].shape)
            h = 1e-6 * max(abs(x[k][idx]), 1e-3)
            up = {kk: v.copy() for kk, v in x.items()}
            dn = {kk: v.copy() for kk, v in x.items()}
            up[k][idx] += h
            dn[k][idx] -= h
            fd = (loss(up) - loss(dn)) / (2 * h)
            g = got[k][idx]
            assert abs(g - fd) <= 2e-5 * (abs(fd) + 1e-3), f"d/d{k}{idx}: {g} vs finite difference {fd}"


def pin_backward_closed_forms(orc):
    """Textbook sums: with a = 1, p = 0 the precision and information are
    running sums, so d/dphi_s = sum_{t>=s} g_lam_t and d/db_s = sum_{t>=s} g_eta_t
    (and the prior collects the full sums); with p = 0 and a loss on the last
    token only, d lam_T/d phi_s = prod_{j>s} a_j^-2 and d eta_T/d b_s =
    prod_{j>s} a_j^-1 (the affine case of the Moebius map)."""
    rng = np.random.default_rng(13)
    T = 64
    phi = np.exp(rng.uniform(np.log(1e-2), np.log(10), T))
    b = rng.standard_normal(T)
    gl, ge = rng.standard_normal(T), rng.standard_normal(T)
    got = orc.backward(_as4(np.ones(T)), _as4(np.zeros(T)), _as4(phi), _as4(b), [[[1.5]]], [[[0.2]]],
                       g_lam=_as4(gl), g_eta=_as4(ge))
    suf_l = np.array([math.fsum(gl[s:]) for s in range(T)])
    suf_e = np.array([math.fsum(ge[s:]) for s in range(T)])
    _scaled_close(got["phi"][0, :, 0, 0], suf_l, 1e-13, "a=1,p=0: d/dphi = suffix sum of g_lam", axis=None)
    _scaled_close(got["b"][0, :, 0, 0], suf_e, 1e-13, "a=1,p=0: d/db = suffix sum of g_eta", axis=None)
    assert abs(got["lam0"][0, 0, 0] - suf_l[0]) <= 1e-12 * (abs(suf_l[0]) + 1)
    assert abs(got["eta0"][0, 0, 0] - suf_e[0]) <= 1e-12 * (abs(suf_e[0]) + 1)
    a = rng.uniform(0.8, 1.2, T) * np.where(rng.random(T) < 0.3, -1.0, 1.0)
    last = np.zeros(T)
    last[-1] = 1.0
    got = orc.backward(_as4(a), _as4(np.zeros(T)), _as4(phi), _as4(b), [[[0.7]]], [[[0.3]]],
                       g_lam=_as4(last))
    ref = np.array([np.prod(a[s + 1:] ** -2.0) for s in range(T)])
    _rel_close(got["phi"][0, :, 0, 0], ref, 1e-12, "p=0: d lam_T / d phi_s")
    _rel_close(got["lam0"][0, 0, 0], np.prod(a ** -2.0), 1e-12, "p=0: d lam_T / d lam_0")
    got = orc.backward(_as4(a), _as4(np.zeros(T)), _as4(phi), _as4(b), [[[0.7]]], [[[0.3]]],
                       g_eta=_as4(last))
    ref = np.array([np.prod(1.0 / a[s + 1:]) for s in range(T)])
    _rel_close(got["b"][0, :, 0, 0], ref, 1e-12, "p=0: d eta_T / d b_s")
    _rel_close(got["eta0"][0, 0, 0], np.prod(1.0 / a), 1e-12, "p=0: d eta_T / d eta_0")
    assert np.max(np.abs(got["phi"])) <= 1e-12 * np.max(np.abs(got["b"])), \
        "p=0: eta does not depend on the precision path"


# ------------------------------------------------------------ layer (fused)
def random_rational_layer(seed, B=2, T=4, H=2, D=2, Ns=3):
    rng = np.random.default_rng(seed)
    def arr(shape, lo, hi, den, neg=False):
        x = np.empty(shape, dtype=object)
        for idx in np.ndindex(shape):
            x[idx] = _random_fraction(rng, lo, hi, den) * (-1 if neg and rng.random() < 0.3 else 1)
        return x
    return {"k": arr((B, T, H, Ns), -5, 5, 4), "q": arr((B, T, H, Ns), -5, 5, 4),
            "v": arr((B, T, H, D), -6, 6, 4), "w": arr((B, T, H, D), 1, 6, 4),
            "a": arr((H, D, Ns), 1, 9, 8, neg=True), "p": arr((H, D, Ns), 0, 6, 8),
            "lam0": arr((B, H, D, Ns), 1, 6, 4), "eta0": arr((B, H, D, Ns), -4, 4, 4)}


def pin_layer_exact(orc, seeds=(31, 32)):
    """The layer oracle == exact rationals done channel by channel with plain
    loops: phi = k_n^2 w_d, b = k_n w_d v_d, the exact Moebius/affine filter,
    y_d = sum_n q_n mu, s_d = sum_n q_n^2 var, final state = last posterior
    (Ns = 3 and D = 2 so that a transposed or mis-broadcast axis shows)."""
    for seed in seeds:
        fr = random_rational_layer(seed)
        B, T, H, Ns = fr["k"].shape
        D = fr["v"].shape[3]
        y = np.empty((B, T, H, D), dtype=object)
        s_ = np.empty((B, T, H, D), dtype=object)
        lam_T = np.empty((B, H, D, Ns), dtype=object)
        eta_T = np.empty((B, H, D, Ns), dtype=object)
        for bi in range(B):
            for h in range(H):
                for d in range(D):
                    ysum = [Fr(0)] * T
                    ssum = [Fr(0)] * T
                    for n in range(Ns):
                        ks = [fr["k"][bi, t, h, n] for t in range(T)]
                        ws = [fr["w"][bi, t, h, d] for t in range(T)]
                        vs = [fr["v"][bi, t, h, d] for t in range(T)]
                        phi = [kk * kk * ww for kk, ww in zip(ks, ws)]
                        info = [kk * ww * vv for kk, ww, vv in zip(ks, ws, vs)]
                        lam, eta = exact_moebius_filter([fr["a"][h, d, n]] * T, [fr["p"][h, d, n]] * T, phi, info,
                                                        fr["lam0"][bi, h, d, n], fr["eta0"][bi, h, d, n])
                        for t in range(T):
                            qq = fr["q"][bi, t, h, n]
                            ysum[t] += qq * eta[t] / lam[t]
                            ssum[t] += qq * qq / lam[t]
                        lam_T[bi, h, d, n] = lam[-1]
                        eta_T[bi, h, d, n] = eta[-1]
                    for t in range(T):
                        y[bi, t, h, d] = ysum[t]
                        s_[bi, t, h, d] = ssum[t]
        f64 = {kk: _to_f64(vv) for kk, vv in fr.items()}
        got = orc.layer_forward(f64["k"], f64["q"], f64["v"], f64["w"], f64["a"], f64["p"],
                                f64["lam0"], f64["eta0"])
        _scaled_close(got["y"], _to_f64(y), 1e-12, f"layer y (seed {seed})")
        _rel_close(got["s"], _to_f64(s_), 1e-12, f"layer s (seed {seed})")
        _rel_close(got["lam_T"], _to_f64(lam_T), 1e-12, f"layer final lambda (seed {seed})")
        _scaled_close(got["eta_T"].reshape(-1), _to_f64(eta_T).reshape(-1), 1e-12, f"layer final eta (seed {seed})",
                      axis=None)


def pin_layer_one_hot_readout(orc):
    """A one-hot readout q = e_m returns the filter outputs of state channel m
    (against the oracle's plain filter fed with phi = k_m^2 w, b = k_m w v), and
    scaling q by c scales y by c and s by c^2."""
    rng = np.random.default_rng(41)
    B, T, H, D, Ns = 2, 30, 2, 3, 4
    k = rng.standard_normal((B, T, H, Ns))
    v = rng.standard_normal((B, T, H, D))
    w = np.exp(rng.uniform(-1, 1, (B, T, H, D)))
    a = rng.uniform(0.5, 1.0, (H, D, Ns))
    p = np.exp(rng.uniform(np.log(1e-3), 0, (H, D, Ns)))
    lam0 = np.exp(rng.uniform(-1, 1, (B, H, D, Ns)))
    eta0 = rng.standard_normal((B, H, D, Ns))
    for m in (0, Ns - 1):
        q = np.zeros((B, T, H, Ns))
        q[..., m] = 1.0
        got = orc.layer_forward(k, q, v, w, a, p, lam0, eta0)
        for h in range(H):
            for d in range(D):
                km = k[:, :, h, m]
                ref = orc.forward(np.broadcast_to(a[h, d, m], (B, T)).reshape(B, T, 1, 1),
                                  np.broadcast_to(p[h, d, m], (B, T)).reshape(B, T, 1, 1),
                                  (km * km * w[:, :, h, d]).reshape(B, T, 1, 1),
                                  (km * w[:, :, h, d] * v[:, :, h, d]).reshape(B, T, 1, 1),
                                  lam0[:, h, d, m].reshape(B, 1, 1), eta0[:, h, d, m].reshape(B, 1, 1))
                _scaled_close(got["y"][:, :, h, d], ref["mu"][:, :, 0, 0], 1e-13, f"one-hot y m={m}")
                _rel_close(got["s"][:, :, h, d], ref["var"][:, :, 0, 0], 1e-13, f"one-hot s m={m}")
    q = rng.standard_normal((B, T, H, Ns))
    g1 = orc.layer_forward(k, q, v, w, a, p, lam0, eta0)
    g3 = orc.layer_forward(k, -3.0 * q, v, w, a, p, lam0, eta0)
    _scaled_close(g3["y"], -3.0 * g1["y"], 1e-14, "readout linear in q")
    _rel_close(g3["s"], 9.0 * g1["s"], 1e-14, "variance readout quadratic in q")


def _exact_layer_loss(fr, w4):
    """Exact loss sum g_y y + g_s s + g_lamT lam_T + g_etaT eta_T of the layer,
    channel by channel with plain loops, on Fraction or Dual entries."""
    g_y, g_s, g_lT, g_eT = w4
    B, T, H, Ns = fr["k"].shape
    D = fr["v"].shape[3]
    tot = Fr(0)
    for bi in range(B):
        for h in range(H):
            for d in range(D):
                for n in range(Ns):
                    phi = [fr["k"][bi, t, h, n] * fr["k"][bi, t, h, n] * fr["w"][bi, t, h, d] for t in range(T)]
                    info = [fr["k"][bi, t, h, n] * fr["w"][bi, t, h, d] * fr["v"][bi, t, h, d] for t in range(T)]
                    lam, eta = exact_moebius_filter([fr["a"][h, d, n]] * T, [fr["p"][h, d, n]] * T, phi, info,
                                                    fr["lam0"][bi, h, d, n], fr["eta0"][bi, h, d, n])
                    for t in range(T):
                        qq = fr["q"][bi, t, h, n]
                        tot = tot + g_y[bi, t, h, d] * (qq * (eta[t] / lam[t])) + g_s[bi, t, h, d] * (qq * qq / lam[t])
                    tot = tot + g_lT[bi, h, d, n] * lam[-1] + g_eT[bi, h, d, n] * eta[-1]
    return tot


def pin_layer_backward_exact_dual(orc, seed=51):
    """Layer gradients == exact forward-mode derivatives (Dual numbers over
    Fractions) of the exact layer, for every element of every input
    (B = 2, T = 3, H = 1, D = 2, Ns = 2), with gradients on all four outputs."""
    fr = random_rational_layer(seed, B=2, T=3, H=1, D=2, Ns=2)
    rng = np.random.default_rng(seed + 7)
    def rarr(shape):
        x = np.empty(shape, dtype=object)
        for idx in np.ndindex(shape):
            x[idx] = _random_fraction(rng, -5, 5, 4)
        return x
    B, T, H, Ns = fr["k"].shape
    D = fr["v"].shape[3]
    w4 = (rarr((B, T, H, D)), rarr((B, T, H, D)), rarr((B, H, D, Ns)), rarr((B, H, D, Ns)))
    exact = {}
    for key, arr in fr.items():
        g = np.empty(arr.shape, dtype=object)
        for idx in np.ndindex(arr.shape):
            dual = {kk: np.vectorize(Dual, otypes=[object])(vv) for kk, vv in fr.items()}
            dual[key][idx] = Dual(arr[idx], 1)
            g[idx] = _exact_layer_loss(dual, w4).d
        exact[key] = g
    f64 = {kk: _to_f64(vv) for kk, vv in fr.items()}
    got = orc.layer_backward(f64["k"], f64["q"], f64["v"], f64["w"], f64["a"], f64["p"], f64["lam0"], f64["eta0"],
                             *[_to_f64(x) for x in w4])
    for key in exact:
        ref = _to_f64(exact[key])
        _scaled_close(got[key].reshape(-1), ref.reshape(-1), 1e-12, f"exact layer gradient d/d{key}", axis=None)


def pin_layer_backward_finite_difference(orc):
    """Layer gradients == central finite differences of the pinned layer
    forward, sampled elements of every input, workload-like values."""
    import dataclasses
    rng = np.random.default_rng(61)
    w = dataclasses.replace(wl.LAYER_WORKLOADS["layer"].with_shape(B=2, T=20, H=2, D=2, Ns=8), dtype="f32")
    x = {kk: np.asarray(vv, dtype=np.float64) for kk, vv in wl.generate_layer(w).items()}
    x.update({kk: np.asarray(vv, dtype=np.float64) for kk, vv in wl.random_layer_prior(w).items()})
    gw = (rng.standard_normal((w.B, w.T, w.H, w.D)), rng.standard_normal((w.B, w.T, w.H, w.D)),
          rng.standard_normal((w.B, w.H, w.D, w.Ns)), rng.standard_normal((w.B, w.H, w.D, w.Ns)))
    names = ("k", "q", "v", "w", "a", "p", "lam0", "eta0")
    got = orc.layer_backward(*(x[n] for n in names), *gw)

    def loss(arrs):
        o = orc.layer_forward(*(arrs[n] for n in names))
        return math.fsum(float((g * o[kk]).sum()) for g, kk in zip(gw, ("y", "s", "lam_T", "eta_T")))

    for key in names:
        for _ in range(4):
            idx = tuple(int(rng.integers(0, s_)) for s_ in x[key].shape)
            h = 1e-6 * max(abs(x[key][idx]), 1e-2)
            up = dict(x)
            dn = dict(x)
            up[key] = x[key].copy()
            dn[key] = x[key].copy()
            up[key][idx] += h
            dn[key][idx] -= h
            fd = (loss(up) - loss(dn)) / (2 * h)
            g = got[key][idx]
            assert abs(g - fd) <= 2e-5 * (abs(fd) + 1e-2), f"layer d/d{key}{idx}: {g} vs finite difference {fd}"


LAYER_PINS = [pin_layer_exact, pin_layer_one_hot_readout, pin_layer_backward_exact_dual,
              pin_layer_backward_finite_difference]


# ------------------------------------------------- attention weights (gates)
def _attention_problem(seed, B=2, T=40, H=1, N=3):
    w = wl.WORKLOADS["tiny"].with_shape(B=B, T=T, H=H, N=N, seed=seed)
    x = wl.generate(w)
    x["a"] = x["a"] * np.where(np.random.default_rng(seed).random(x["a"].shape) < 0.25, -1.0, 1.0)
    pri = wl.random_prior(w)
    x.update(pri)
    return {k: np.asarray(v, dtype=np.float64) for k, v in x.items()}


def _windows(t0, span, W):
    """(window index, first token, valid tokens) of the span cut into W-token windows."""
    return [(w, t0 + w * W, min(W, t0 + span - (t0 + w * W))) for w in range(-(-span // W))]


def pin_attention_moebius_product(orc):
    """F(t, s) = prod_{k=s+1..t} a_k / (C lambda_s + D) with [[A, B], [C, D]] =
    M_t ... M_{s+1}, numpy matrix products of the pages' M_k and lambda_s
    from the pinned filter (the denominators of the Moebius product
    telescope into the gates' denominators)."""
    x = _attention_problem(41)
    t0, span, W = 3, 30, 12
    F = orc.attention_weights(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], t0, span, W)
    lam = orc.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])["lam"]
    B, T, H, N = x["a"].shape
    assert F.shape == (B, 3, W, W, H, N), F.shape
    for bi in range(B):
        for n in range(N):
            a, p, phi = (x[k][bi, :, 0, n] for k in ("a", "p", "phi"))
            for w, start, nv in _windows(t0, span, W):
                for j in range(W):
                    s = start + j
                    P = np.eye(2)
                    for i in range(W):
                        got = F[bi, w, i, j, 0, n]
                        if i >= nv or j >= nv or i < j:
                            assert got == 0.0, (bi, w, i, j, got)
                            continue
                        if i > j:
                            t = start + i
                            M = np.array([[1 + p[t] * phi[t], a[t] ** 2 * phi[t]], [p[t], a[t] ** 2]])
                            P = M @ P
                        ref = np.prod(a[s + 1:start + i + 1]) / (P[1, 0] * lam[bi, s, 0, n] + P[1, 1])
                        assert abs(got - ref) <= 1e-12 * abs(ref), (bi, w, i, j, got, ref)


def pin_attention_mean_ratio(orc):
    """With b = 0 after token s, eta_t = F(t, s) eta_s: F read off the pinned
    filter's information mean as eta_t / eta_s (zeroing b leaves lambda, so
    every gate, unchanged)."""
    x = _attention_problem(42, B=1, T=24, N=2)
    t0, span, W = 2, 20, 7
    F = orc.attention_weights(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], t0, span, W)
    for w, start, nv in _windows(t0, span, W):
        for j in range(nv):
            s = start + j
            bz = x["b"].copy()
            bz[:, s + 1:] = 0.0
            eta = orc.forward(x["a"], x["p"], x["phi"], bz, x["lam0"], x["eta0"])["eta"]
            for i in range(j, nv):
                ref = eta[:, start + i] / eta[:, s]
                got = F[:, w, i, j]
                assert np.all(np.abs(got - ref) <= 1e-12 * np.abs(ref)), (w, i, j, got, ref)


def pin_attention_exact(orc):
    """Exact rationals: lambda from the exact Moebius product, the gates and
    their products in Fractions, against the fp64 weights."""
    fr = random_rational_problem(43, B=2, T=9, H=1, N=2)
    lam_x, _ = exact_solution(fr)
    f64 = {k: _to_f64(v) for k, v in fr.items()}
    t0, span, W = 1, 8, 3
    F = orc.attention_weights(f64["a"], f64["p"], f64["phi"], f64["b"], f64["lam0"], f64["eta0"], t0, span, W)
    B, T, H, N = fr["a"].shape
    for bi in range(B):
        for n in range(N):
            lam_before = [fr["lam0"][bi, 0, n]] + list(lam_x[bi, :, 0, n])
            gate = [fr["a"][bi, k, 0, n] / (fr["a"][bi, k, 0, n] ** 2 + fr["p"][bi, k, 0, n] * lam_before[k])
                    for k in range(T)]
            for w, start, nv in _windows(t0, span, W):
                for i in range(nv):
                    for j in range(i + 1):
                        ref = Fr(1)
                        for k in range(start + j + 1, start + i + 1):
                            ref *= gate[k]
                        got = F[bi, w, i, j, 0, n]
                        assert abs(got - float(ref)) <= 1e-13 * abs(float(ref)), (bi, w, i, j, got, ref)


ATTENTION_PINS = [pin_attention_moebius_product, pin_attention_mean_ratio, pin_attention_exact]


# ------------------------------- convolutional form (deterministic, time-invariant)
def _lti_problem(seed, B=2, T=60, H=1, N=3):
    rng = np.random.default_rng(seed)
    a = rng.uniform(0.9, 1.1, (B, H, N)) * np.where(rng.random((B, H, N)) < 0.3, -1.0, 1.0)
    phi = np.exp(rng.uniform(np.log(1e-2), np.log(10.0), (B, T, H, N)))
    b = rng.standard_normal((B, T, H, N))
    lam0 = np.exp(rng.uniform(np.log(0.1), np.log(10.0), (B, H, N)))
    eta0 = rng.standard_normal((B, H, N))
    return a, phi, b, lam0, eta0


def pin_lti_equals_filter(orc):
    """The convolution sums equal the covariance-form filter run with p = 0
    and the same decay at every token (Theorem 3 is a rearrangement of the
    filter in this case)."""
    a, phi, b, lam0, eta0 = _lti_problem(61)
    B, T, H, N = phi.shape
    got = orc.lti_forward(a, phi, b, lam0, eta0)
    ref = orc.forward(np.broadcast_to(a[:, None], phi.shape), np.zeros(phi.shape), phi, b, lam0, eta0)
    _rel_close(got["lam"], ref["lam"], 1e-12, "lti lambda")
    _rel_close(got["var"], ref["var"], 1e-12, "lti var")
    _scaled_close(got["eta"], ref["eta"], 1e-12, "lti eta")
    _scaled_close(got["mu"], ref["mu"], 1e-12, "lti mu")


def pin_lti_exact(orc):
    """Exact rationals: the affine recursions lambda_t = a^-2 lambda_{t-1} +
    phi_t, eta_t = eta_{t-1} / a + b_t stepped in Fractions."""
    rng = np.random.default_rng(62)
    B, T, H, N = 2, 10, 1, 2
    fa = np.empty((B, H, N), dtype=object)
    fphi = np.empty((B, T, H, N), dtype=object)
    fb = np.empty((B, T, H, N), dtype=object)
    for idx in np.ndindex(fa.shape):
        fa[idx] = _random_fraction(rng, 4, 9, 7) * (-1 if rng.random() < 0.3 else 1)
    for idx in np.ndindex(fphi.shape):
        fphi[idx] = _random_fraction(rng, 0, 6, 8)
        fb[idx] = _random_fraction(rng, -6, 6, 8)
    lam0, eta0 = Fr(3, 2), Fr(-1, 3)
    got = orc.lti_forward(_to_f64(fa), _to_f64(fphi), _to_f64(fb), float(lam0), float(eta0))
    for idx in np.ndindex((B, H, N)):
        bi, h, n = idx
        lam, eta = lam0, eta0
        for t in range(T):
            lam = lam / (fa[idx] ** 2) + fphi[bi, t, h, n]
            eta = eta / fa[idx] + fb[bi, t, h, n]
            assert abs(got["lam"][bi, t, h, n] - float(lam)) <= 1e-13 * abs(float(lam)), (idx, t)
            assert abs(got["eta"][bi, t, h, n] - float(eta)) <= 1e-13 * (abs(float(eta)) + 1), (idx, t)


def pin_lti_closed_forms(orc):
    """a = 1: lambda_t = lambda_0 + sum phi (math.fsum), eta_t = eta_0 + sum b;
    no evidence (phi = b = 0): lambda_t = a^(-2(t+1)) lambda_0, eta_t =
    a^(-(t+1)) eta_0 (the prior decays geometrically)."""
    rng = np.random.default_rng(63)
    T = 50
    phi = rng.uniform(0, 3, (1, T, 1, 1))
    b = rng.standard_normal((1, T, 1, 1))
    got = orc.lti_forward(np.ones((1, 1, 1)), phi, b, 0.5, 0.25)
    for t in range(T):
        _rel_close(got["lam"][0, t, 0, 0], 0.5 + math.fsum(phi[0, :t + 1, 0, 0]), 1e-13, f"a=1 lambda t={t}")
        ref = 0.25 + math.fsum(b[0, :t + 1, 0, 0])
        assert abs(got["eta"][0, t, 0, 0] - ref) <= 1e-12 * (abs(ref) + 1), f"a=1 eta t={t}"
    for a in (0.95, -1.05):
        z = np.zeros((1, T, 1, 1))
        got = orc.lti_forward(np.full((1, 1, 1), a), z, z, 2.0, -0.5)
        t = np.arange(1, T + 1)
        _rel_close(got["lam"][0, :, 0, 0], 2.0 * a ** (-2.0 * t), 1e-13, f"no-evidence lambda a={a}")
        _rel_close(got["eta"][0, :, 0, 0], -0.5 * a ** (-1.0 * t), 1e-13, f"no-evidence eta a={a}")


LTI_PINS = [pin_lti_equals_filter, pin_lti_exact, pin_lti_closed_forms]

BACKWARD_PINS = [pin_backward_exact_dual, pin_backward_autograd, pin_backward_finite_difference,
                 pin_backward_closed_forms]

ALL_PINS = [pin_exact_rational, pin_exact_rational_step, pin_riccati, pin_precision_sum,
            pin_no_process_noise, pin_no_observation, pin_gate_derivative, pin_gate_product,
            pin_invariants] + BACKWARD_PINS + LAYER_PINS + ATTENTION_PINS + LTI_PINS
