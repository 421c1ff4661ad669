"""The fp64 oracle against its pins (closed forms, exact rationals, invariants)."""
import numpy as np
import pytest

import oracle
import oracle_pins as pins
from kalman_linear_attention_b200 import workloads as wl


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_exact_forms_agree():
    """The Moebius/affine form and the 3x3 homogeneous form are the same exact
    rational recursion (the identity the CUDA path's chunk aggregates rely on)."""
    for seed in (1, 2):
        fr = pins.random_rational_problem(seed, B=1, T=9, H=1, N=2)
        l1, e1 = pins.exact_solution(fr, pins.exact_moebius_filter)
        l2, e2 = pins.exact_solution(fr, pins.exact_homogeneous_filter)
        assert (l1 == l2).all() and (e1 == e2).all()


def test_step_iterates_to_forward(orc):
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=50, H=2, N=4)
    x = wl.generate(w)
    out = orc.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    lam, eta = x["lam0"].astype(np.float64), x["eta0"].astype(np.float64)
    for t in range(w.T):
        o = orc.step(x["a"][:, t], x["p"][:, t], x["phi"][:, t], x["b"][:, t], lam, eta)
        lam, eta = o["lam"], o["eta"]
        for k in ("lam", "eta", "mu", "var"):
            assert np.array_equal(o[k], out[k][:, t]), (k, t)


def test_threads_do_not_change_results(orc):
    w = wl.WORKLOADS["stiff"].with_shape(B=4, T=40)
    x = wl.generate(w)
    one = orc.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], threads=1)
    many = orc.forward(x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"], threads=4)
    for k in one:
        assert np.array_equal(one[k], many[k])


def test_empty_and_bad_shapes(orc):
    z = np.zeros((1, 0, 1, 4))
    out = orc.forward(z, z, z, z, np.ones((1, 1, 4)), np.zeros((1, 1, 4)))
    assert out["lam"].shape == (1, 0, 1, 4)
    with pytest.raises(ValueError):
        orc.forward(np.zeros((1, 2, 1, 4)), z, z, z, 1.0, 0.0)


def test_moebius_factorization():
    """M_t = [[1, phi], [0, 1]] [[1, 0], [p, a^2]] (update after predict) and
    the information row of the 3x3 token matrix is b times the predicted
    denominator row plus a times the old information row -- the forms the
    CUDA kernels append tokens with -- in exact rational arithmetic."""
    from fractions import Fraction as F
    rng = np.random.default_rng(3)
    for _ in range(200):
        a, b = (F(int(rng.integers(-9, 10)), int(rng.integers(1, 8))) for _ in range(2))
        p, phi = (F(int(rng.integers(0, 10)), int(rng.integers(1, 8))) for _ in range(2))
        M = [[1 + p * phi, a * a * phi], [p, a * a]]
        U = [[1, phi], [0, 1]]
        P = [[1, 0], [p, a * a]]
        UP = [[sum(U[i][k] * P[k][j] for k in range(2)) for j in range(2)] for i in range(2)]
        assert UP == M
        m = [[F(int(rng.integers(-5, 6)), int(rng.integers(1, 5))) for _ in range(2)] for _ in range(2)]
        g = [F(int(rng.integers(-5, 6)), int(rng.integers(1, 5))) for _ in range(2)]
        d = [p * m[0][j] + a * a * m[1][j] for j in range(2)]
        direct = [b * p * m[0][j] + b * a * a * m[1][j] + a * g[j] for j in range(2)]
        assert direct == [b * d[j] + a * g[j] for j in range(2)]


def test_backward_threads_and_absent_gradients(orc):
    """Threads split channels only (bitwise equal), and an absent output
    gradient is the same as a zero one."""
    w = wl.WORKLOADS["stiff"].with_shape(B=3, T=30)
    x = wl.generate(w)
    rng = np.random.default_rng(2)
    g = [rng.standard_normal(x["a"].shape) for _ in range(4)]
    args = (x["a"], x["p"], x["phi"], x["b"], x["lam0"], x["eta0"])
    one = orc.backward(*args, *g, threads=1)
    many = orc.backward(*args, *g, threads=4)
    for k in one:
        assert np.array_equal(one[k], many[k]), k
    absent = orc.backward(*args, g[0], None, g[2], None)
    zeros = orc.backward(*args, g[0], np.zeros_like(g[1]), g[2], np.zeros_like(g[3]))
    for k in absent:
        assert np.array_equal(absent[k], zeros[k]), k


def test_backward_empty_and_bad_shapes(orc):
    """T = 0: no outputs, so the prior's gradients are zero."""
    z = np.zeros((2, 0, 1, 4))
    out = orc.backward(z, z, z, z, np.ones((2, 1, 4)), np.zeros((2, 1, 4)), z, z, z, z)
    assert out["a"].shape == (2, 0, 1, 4)
    assert np.array_equal(out["lam0"], np.zeros((2, 1, 4)))
    assert np.array_equal(out["eta0"], np.zeros((2, 1, 4)))
    with pytest.raises(ValueError):
        orc.backward(np.zeros((1, 2, 1, 4)), z, z, z, 1.0, 0.0)
    with pytest.raises(ValueError):
        orc.backward(*(np.zeros((1, 2, 1, 4)),) * 4, 1.0, 0.0, g_mu=np.zeros((1, 3, 1, 4)))
