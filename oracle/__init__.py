"""fp64 CPU oracle for the Kalman Linear Attention filter.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``kalman_linear_attention_b200``) never imports it, and this
package never imports the product path: the two share no code.

The filter's arithmetic lives in ``kla_oracle.c`` (plain sequential
covariance-form Kalman filter and its reverse-mode gradients, fp64, one channel
at a time).  This module compiles it with gcc, loads it with ctypes and
converts arrays to contiguous fp64 (an exact upcast for fp32 and bf16 inputs).
The arithmetic written here is the KLA layer around the filter
(``layer_forward``: the evidence formed from the layer's operators by numpy
broadcasting, and the readout by sums over the state channels), the attention
weights (``attention_weights``: products of the filter's gates over windows of
tokens) and the convolutional form of the deterministic time-invariant case
(``lti_forward``: geometric-kernel convolution sums), all in fp64.

Pins: every function here is pinned by ``tests/test_oracle.py`` against exact
rational arithmetic, closed forms (Riccati fixed point, precision sums, the
no-process-noise affine case, the no-observation covariance recursion) and
invariants.  The gradients (``backward``, reverse mode through the covariance
form) are pinned against exact forward-mode derivatives (dual numbers over
Fractions) of the exact Moebius/affine filter, torch autograd through the
information form, central finite differences of the pinned forward pass, and
closed-form sums of the a = 1 / p = 0 cases.  The layer function is pinned
against exact rationals computed channel by channel with plain loops and
against one-hot readouts of the pinned filter; its gradients
(``layer_backward``, not yet matched by a kernel) against exact forward-mode
derivatives of the exact layer and finite differences of the pinned layer
function.  The attention weights are pinned against the matrix-product
identity prod(a) / (C lambda_s + D) of the Moebius product M_t ... M_{s+1},
against ratios of the information mean when b = 0 after s (read off the
pinned filter), and exact rationals; the convolutional form against the
covariance-form filter with p = 0, exact rationals and closed forms (a = 1:
precision sums; no evidence: geometric decay of the prior).  None is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "kla_oracle.c")
LIBRARY = os.path.join(_HERE, "libkla_oracle.so")

CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11"]


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Compile ``source`` into a shared library at ``output`` with gcc."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    tmp = output + ".tmp"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, source, "-lm"], check=True)
    os.replace(tmp, output)
    return output


_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x: np.ndarray):
    return x.ctypes.data_as(_D)


@dataclass
class Oracle:
    """ctypes handle on one compiled copy of the oracle."""

    lib: ctypes.CDLL

    @classmethod
    def load(cls, path: str | None = None) -> "Oracle":
        lib = ctypes.CDLL(path or build())
        lib.kla_oracle_forward.restype = ctypes.c_int
        lib.kla_oracle_forward.argtypes = [_D] * 10 + [_I64] * 4 + [ctypes.c_int]
        lib.kla_oracle_step.restype = ctypes.c_int
        lib.kla_oracle_step.argtypes = [_D] * 8 + [_I64]
        lib.kla_oracle_backward.restype = ctypes.c_int
        lib.kla_oracle_backward.argtypes = [_D] * 16 + [_I64] * 4 + [ctypes.c_int]
        lib.kla_oracle_max_threads.restype = ctypes.c_int
        lib.kla_oracle_max_threads.argtypes = []
        return cls(lib)

    def max_threads(self) -> int:
        return int(self.lib.kla_oracle_max_threads())

    def forward(self, a, p, phi, b, lam0, eta0, threads: int = 1):
        """Filter every channel of [B, T, H, N] inputs from the [B, H, N] prior.

        Returns a dict with fp64 arrays ``lam``, ``eta``, ``mu``, ``var`` of
        shape [B, T, H, N].
        """
        a, p, phi, b = (_f64(x) for x in (a, p, phi, b))
        if a.ndim != 4 or not (a.shape == p.shape == phi.shape == b.shape):
            raise ValueError("a, p, phi, b must share one [B, T, H, N] shape")
        B, T, H, N = a.shape
        lam0 = _f64(np.broadcast_to(np.asarray(lam0, dtype=np.float64), (B, H, N)))
        eta0 = _f64(np.broadcast_to(np.asarray(eta0, dtype=np.float64), (B, H, N)))
        out = {k: np.empty((B, T, H, N), dtype=np.float64) for k in ("lam", "eta", "mu", "var")}
        rc = self.lib.kla_oracle_forward(
            _ptr(a), _ptr(p), _ptr(phi), _ptr(b), _ptr(lam0), _ptr(eta0),
            _ptr(out["lam"]), _ptr(out["eta"]), _ptr(out["mu"]), _ptr(out["var"]),
            B, T, H, N, int(threads))
        if rc != 0:
            raise ValueError(f"kla_oracle_forward failed ({rc})")
        return out

    def step(self, a, p, phi, b, lam_state, eta_state):
        """One decode token for every channel; returns the new state and outputs.

        Inputs are arrays of one common shape; the state arrays are not
        modified (copies are advanced and returned).
        """
        a, p, phi, b = (_f64(x) for x in (a, p, phi, b))
        shape = a.shape
        lam = _f64(lam_state).copy()
        eta = _f64(eta_state).copy()
        if not (p.shape == phi.shape == b.shape == lam.shape == eta.shape == shape):
            raise ValueError("step inputs and state must share one shape")
        mu = np.empty(shape, dtype=np.float64)
        var = np.empty(shape, dtype=np.float64)
        rc = self.lib.kla_oracle_step(_ptr(a), _ptr(p), _ptr(phi), _ptr(b),
                                      _ptr(lam), _ptr(eta), _ptr(mu), _ptr(var), a.size)
        if rc != 0:
            raise ValueError(f"kla_oracle_step failed ({rc})")
        return {"lam": lam, "eta": eta, "mu": mu, "var": var}

    def backward(self, a, p, phi, b, lam0, eta0, g_lam=None, g_eta=None, g_mu=None, g_var=None,
                 threads: int = 1):
        """Gradients of a loss through the whole-sequence filter.

        ``g_lam``, ``g_eta``, ``g_mu``, ``g_var`` are the loss gradients with
        respect to the four [B, T, H, N] outputs (None: zero).  Returns a dict
        with fp64 ``a``, ``p``, ``phi``, ``b`` ([B, T, H, N]) and ``lam0``,
        ``eta0`` ([B, H, N]): the gradients with respect to each input.
        """
        a, p, phi, b = (_f64(x) for x in (a, p, phi, b))
        if a.ndim != 4 or not (a.shape == p.shape == phi.shape == b.shape):
            raise ValueError("a, p, phi, b must share one [B, T, H, N] shape")
        B, T, H, N = a.shape
        lam0 = _f64(np.broadcast_to(np.asarray(lam0, dtype=np.float64), (B, H, N)))
        eta0 = _f64(np.broadcast_to(np.asarray(eta0, dtype=np.float64), (B, H, N)))
        grads = []
        for g in (g_lam, g_eta, g_mu, g_var):
            if g is None:
                grads.append(None)
                continue
            g = _f64(g)
            if g.shape != a.shape:
                raise ValueError("output gradients must be [B, T, H, N]")
            grads.append(g)
        out = {k: np.empty((B, T, H, N), dtype=np.float64) for k in ("a", "p", "phi", "b")}
        out["lam0"] = np.empty((B, H, N), dtype=np.float64)
        out["eta0"] = np.empty((B, H, N), dtype=np.float64)
        gp = [None if g is None else _ptr(g) for g in grads]
        rc = self.lib.kla_oracle_backward(
            _ptr(a), _ptr(p), _ptr(phi), _ptr(b), _ptr(lam0), _ptr(eta0), *gp,
            _ptr(out["a"]), _ptr(out["p"]), _ptr(out["phi"]), _ptr(out["b"]),
            _ptr(out["lam0"]), _ptr(out["eta0"]), B, T, H, N, int(threads))
        if rc != 0:
            raise ValueError(f"kla_oracle_backward failed ({rc})")
        return out

    def layer_forward(self, k, q, v, w, a, p, lam0, eta0, threads: int = 1):
        """The KLA layer around the filter: evidence formed from the layer's
        operators, the filter, and the readout.

        Shapes: k, q [B, T, H, Ns] (observation and readout operators); v, w
        [B, T, H, D] (values and their precision Lambda^v); a, p [H, D, Ns]
        (time-invariant decay and process noise per state channel); lam0, eta0
        [B, H, D, Ns] (prior).  State channel (h, d, n) is an independent
        scalar filter observing value coordinate d through k_n:

          phi = k_n^2 w_d,   b = k_n w_d v_d          (evidence precision and
                                                       information, KLA review
                                                       "Circularity Check")
          y_d = sum_n q_n mu_{d,n},   s_d = sum_n q_n^2 var_{d,n}
                                                      (readout of the posterior
                                                       mean and of its variance
                                                       under the diagonal posterior)

        Returns fp64 ``y``, ``s`` [B, T, H, D] and the state after the last
        token ``lam_T``, ``eta_T`` [B, H, D, Ns] (the prior when T = 0).
        """
        k, q, v, w = (_f64(x) for x in (k, q, v, w))
        a, p = _f64(a), _f64(p)
        if k.ndim != 4 or q.shape != k.shape or v.ndim != 4 or w.shape != v.shape:
            raise ValueError("k, q must be [B, T, H, Ns] and v, w [B, T, H, D]")
        B, T, H, Ns = k.shape
        D = v.shape[3]
        if v.shape[:3] != (B, T, H) or a.shape != (H, D, Ns) or p.shape != (H, D, Ns):
            raise ValueError("v, w must be [B, T, H, D] and a, p [H, D, Ns]")
        lam0 = _f64(np.broadcast_to(np.asarray(lam0, dtype=np.float64), (B, H, D, Ns)))
        eta0 = _f64(np.broadcast_to(np.asarray(eta0, dtype=np.float64), (B, H, D, Ns)))
        kk = k[:, :, :, None, :]                       # [B, T, H, 1, Ns]
        ww = w[:, :, :, :, None]                       # [B, T, H, D, 1]
        vv = v[:, :, :, :, None]
        phi = kk * kk * ww                             # [B, T, H, D, Ns]
        info = kk * ww * vv
        shape5 = (B, T, H, D, Ns)
        aa = np.broadcast_to(a, shape5)
        pp = np.broadcast_to(p, shape5)
        flat = lambda x: np.ascontiguousarray(x).reshape(B, T, H, D * Ns)
        out = self.forward(flat(aa), flat(pp), flat(phi), flat(info),
                           lam0.reshape(B, H, D * Ns), eta0.reshape(B, H, D * Ns), threads=threads)
        mu = out["mu"].reshape(shape5)
        var = out["var"].reshape(shape5)
        qq = q[:, :, :, None, :]
        y = np.sum(qq * mu, axis=4)
        s_ = np.sum(qq * qq * var, axis=4)
        if T > 0:
            lam_T = out["lam"][:, T - 1].reshape(B, H, D, Ns)
            eta_T = out["eta"][:, T - 1].reshape(B, H, D, Ns)
        else:
            lam_T, eta_T = lam0.copy(), eta0.copy()
        return {"y": y, "s": s_, "lam_T": lam_T, "eta_T": eta_T}

    def attention_weights(self, a, p, phi, b, lam0, eta0, t0: int, span: int, W: int, threads: int = 1):
        """The Kalman attention weights of the information mean, window by window.

        Between two tokens s <= t of one channel, the information mean of the
        later one responds to the earlier one through the gates between them
        (the affine recursion eta_k = f_k eta_{k-1} + b_k, KLA review "Core
        claim"; the "Kalman Attention Matrix" of its minor comment on
        App. E.3/E.4):

          eta_t = F(t, s) eta_s + sum_{r = s+1..t} F(t, r) b_r,
          F(t, s) = prod_{k = s+1..t} f_k,   f_k = a_k / (a_k^2 + p_k lambda_{k-1}),

        with lambda_{k-1} the posterior precision before token k (this
        oracle's own filter; the prior before the first token).  Rows are
        0-based tokens.  The span [t0, t0 + span) is cut into windows of W
        tokens; returns F, fp64 [B, nwin, W, W, H, N] with nwin =
        ceil(span / W): entry [b, w, i, j, h, n] = F(t0 + w W + i, t0 + w W + j)
        for j <= i inside the span (1 on the diagonal), 0 above the diagonal
        and past the span.
        """
        a, p = _f64(a), _f64(p)
        if a.ndim != 4 or p.shape != a.shape:
            raise ValueError("a, p must share one [B, T, H, N] shape")
        B, T, H, N = a.shape
        if W < 1 or t0 < 0 or span < 0 or t0 + span > T:
            raise ValueError("need W >= 1 and 0 <= t0 <= t0 + span <= T")
        lam0 = _f64(np.broadcast_to(np.asarray(lam0, dtype=np.float64), (B, H, N)))
        out = self.forward(a, p, phi, b, lam0, eta0, threads=threads)
        lam_before = np.concatenate([lam0[:, None], out["lam"][:, :T - 1]], axis=1)
        gate = a / (a * a + p * lam_before)           # f_k for every token k
        nwin = -(-span // W)
        F = np.zeros((B, nwin, W, W, H, N))
        for w in range(nwin):
            start = t0 + w * W
            n_valid = min(W, t0 + span - start)
            for j in range(n_valid):
                F[:, w, j, j] = 1.0
                F[:, w, j + 1:n_valid, j] = np.cumprod(gate[:, start + j + 1:start + n_valid], axis=1)
        return F

    def lti_forward(self, a, phi, b, lam0, eta0):
        """The convolutional form of the filter for a deterministic
        time-invariant system (KLA review, Theorem 3: deterministic LTI
        systems, evaluated as a convolution).

        With no process noise (p = 0) and a decay a constant in time, the
        precision map is affine, lambda_t = a^-2 lambda_{t-1} + phi_t, and
        the gate is 1 / a, so both recursions unroll into causal
        convolutions with geometric kernels (rows 0-based):

          lambda_t = a^(-2(t+1)) lambda_0 + sum_{s=0..t} a^(-2(t-s)) phi_s,
          eta_t    = a^(-(t+1))  eta_0    + sum_{s=0..t} a^(-(t-s))  b_s,

        mu_t = eta_t / lambda_t, var_t = 1 / lambda_t.  Here the sums are
        evaluated as written (kernel powers by ``numpy.power``, O(T^2) per
        channel): it is the definition, for small cases.

        a: [B, H, N] (per channel); phi, b: [B, T, H, N]; lam0, eta0:
        [B, H, N].  Returns fp64 ``lam``, ``eta``, ``mu``, ``var``
        [B, T, H, N].
        """
        phi, b = _f64(phi), _f64(b)
        if phi.ndim != 4 or b.shape != phi.shape:
            raise ValueError("phi, b must share one [B, T, H, N] shape")
        B, T, H, N = phi.shape
        a = _f64(np.broadcast_to(np.asarray(a, dtype=np.float64), (B, H, N)))
        lam0 = _f64(np.broadcast_to(np.asarray(lam0, dtype=np.float64), (B, H, N)))
        eta0 = _f64(np.broadcast_to(np.asarray(eta0, dtype=np.float64), (B, H, N)))
        m = np.arange(T + 1, dtype=np.float64)
        kappa = np.power(a[..., None], -2.0 * m)      # [B, H, N, T+1]: a^(-2m)
        nu = np.power(a[..., None], -m)                # a^(-m)
        lam = np.empty((B, T, H, N))
        eta = np.empty((B, T, H, N))
        for t in range(T):
            # kernel index t - s for s = 0..t
            lam[:, t] = kappa[..., t + 1] * lam0 + np.einsum("bhns,bshn->bhn", kappa[..., t::-1], phi[:, :t + 1])
            eta[:, t] = nu[..., t + 1] * eta0 + np.einsum("bhns,bshn->bhn", nu[..., t::-1], b[:, :t + 1])
        return {"lam": lam, "eta": eta, "mu": eta / lam, "var": 1.0 / lam}

    def layer_backward(self, k, q, v, w, a, p, lam0, eta0, g_y=None, g_s=None, g_lam_T=None, g_eta_T=None,
                       threads: int = 1):
        """Gradients of a loss through ``layer_forward``.

        ``g_y``, ``g_s`` [B, T, H, D] and ``g_lam_T``, ``g_eta_T``
        [B, H, D, Ns] are the loss gradients with respect to the layer's
        outputs (None: zero).  Returns fp64 gradients with respect to every
        input: ``k``, ``q``, ``v``, ``w``, ``a``, ``p``, ``lam0``, ``eta0``.

        The chain rule over the layer's three parts: the readout (d y / d mu =
        q_n, d s / d var = q_n^2, d y / d q_n = mu, d s / d q_n = 2 q_n var), the
        filter (the reverse-mode ``backward`` of the C oracle, with the final
        state's gradients added at the last token), and the evidence (phi =
        k^2 w, b = k w v; a and p are shared by every token and batch row, so
        their gradients are sums).
        """
        k, q, v, w = (_f64(x) for x in (k, q, v, w))
        a, p = _f64(a), _f64(p)
        B, T, H, Ns = k.shape
        D = v.shape[3]
        shape5 = (B, T, H, D, Ns)
        lam0 = _f64(np.broadcast_to(np.asarray(lam0, dtype=np.float64), (B, H, D, Ns)))
        eta0 = _f64(np.broadcast_to(np.asarray(eta0, dtype=np.float64), (B, H, D, Ns)))
        zero4 = np.zeros((B, T, H, D))
        g_y = zero4 if g_y is None else _f64(g_y)
        g_s = zero4 if g_s is None else _f64(g_s)
        kk = k[:, :, :, None, :]
        ww = w[:, :, :, :, None]
        vv = v[:, :, :, :, None]
        qq = q[..., None, :]
        phi = ww * (kk * kk)                  # the forward's evidence, recomputed
        info = (kk * vv) * ww
        flat = lambda x: np.ascontiguousarray(np.broadcast_to(x, shape5)).reshape(B, T, H, D * Ns)
        fwd = self.forward(flat(a), flat(p), flat(phi), flat(info), lam0.reshape(B, H, D * Ns),
                           eta0.reshape(B, H, D * Ns), threads=threads)
        mu = fwd["mu"].reshape(shape5)
        var = fwd["var"].reshape(shape5)
        # readout
        g_mu = g_y[..., None] * qq
        g_var = g_s[..., None] * qq * qq
        g_q = np.sum(g_y[..., None] * mu + 2.0 * g_s[..., None] * qq * var, axis=3)
        # final state -> gradients of the last row of lambda, eta
        g_lam = np.zeros(shape5)
        g_eta = np.zeros(shape5)
        if T > 0:
            if g_lam_T is not None:
                g_lam[:, T - 1] = _f64(g_lam_T)
            if g_eta_T is not None:
                g_eta[:, T - 1] = _f64(g_eta_T)
        gr = self.backward(flat(a), flat(p), flat(phi), flat(info), lam0.reshape(B, H, D * Ns),
                           eta0.reshape(B, H, D * Ns), flat(g_lam), flat(g_eta), flat(g_mu), flat(g_var),
                           threads=threads)
        g_phi = gr["phi"].reshape(shape5)
        g_b = gr["b"].reshape(shape5)
        out = {
            # evidence: phi = k^2 w, b = k w v
            "k": np.sum(g_phi * 2.0 * kk * ww + g_b * ww * vv, axis=3),
            "w": np.sum(g_phi * kk * kk + g_b * kk * vv, axis=4),
            "v": np.sum(g_b * kk * ww, axis=4),
            "q": g_q,
            # time-invariant parameters: summed over batch rows and tokens
            "a": np.sum(gr["a"].reshape(shape5), axis=(0, 1)),
            "p": np.sum(gr["p"].reshape(shape5), axis=(0, 1)),
            "lam0": gr["lam0"].reshape(B, H, D, Ns),
            "eta0": gr["eta0"].reshape(B, H, D, Ns),
        }
        if T == 0:
            # no tokens: the final state is the prior
            if g_lam_T is not None:
                out["lam0"] = out["lam0"] + _f64(g_lam_T)
            if g_eta_T is not None:
                out["eta0"] = out["eta0"] + _f64(g_eta_T)
        return out


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``kla_oracle.c`` in this directory."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle.load()
    return _DEFAULT


def forward(a, p, phi, b, lam0, eta0, threads: int = 1):
    return default().forward(a, p, phi, b, lam0, eta0, threads=threads)


def step(a, p, phi, b, lam_state, eta_state):
    return default().step(a, p, phi, b, lam_state, eta_state)


def backward(a, p, phi, b, lam0, eta0, g_lam=None, g_eta=None, g_mu=None, g_var=None,
             threads: int = 1):
    return default().backward(a, p, phi, b, lam0, eta0, g_lam, g_eta, g_mu, g_var, threads=threads)


def layer_forward(k, q, v, w, a, p, lam0, eta0, threads: int = 1):
    return default().layer_forward(k, q, v, w, a, p, lam0, eta0, threads=threads)


def layer_backward(k, q, v, w, a, p, lam0, eta0, g_y=None, g_s=None, g_lam_T=None, g_eta_T=None,
                   threads: int = 1):
    return default().layer_backward(k, q, v, w, a, p, lam0, eta0, g_y, g_s, g_lam_T, g_eta_T, threads=threads)


def attention_weights(a, p, phi, b, lam0, eta0, t0: int, span: int, W: int, threads: int = 1):
    return default().attention_weights(a, p, phi, b, lam0, eta0, t0, span, W, threads=threads)


def lti_forward(a, phi, b, lam0, eta0):
    return default().lti_forward(a, phi, b, lam0, eta0)
