"""Seeded synthetic inputs for the KLA filter (shapes, distributions, seeds).

This module holds no arithmetic of the filter itself: it only draws the four
per-token inputs (a, p, phi, b) and the prior (lambda_0, eta_0) of the five
standard workloads.  Both the CUDA path (tests, bench) and the fp64 oracle read
their inputs from here, so that they see bit-identical values.

Recipe (fixed, documented in the design notes):

* Each input array k in (a, p, phi, b) has its own stream
  ``np.random.Generator(np.random.PCG64(SeedSequence(seed).spawn(4)[k]))``.
* Each stream is drawn in fp64, in C order over [B, T, H, N] (N fastest),
  in blocks of whole (b, t) rows; block boundaries do not change the values.
* fp64 draws are rounded to fp32 (numpy cast).  bf16 workloads further round
  the fp32 values to bf16 (round to nearest even on the bit pattern) and keep
  them in fp32 arrays, so the values are exactly bf16-representable.
* lambda_0 = 1 and eta_0 = 0 for every channel, as fp32 [B, H, N].

Distributions ("logU(lo, hi)" = exp(U(ln lo, ln hi)); softplus(x) = ln(1+e^x);
sigmoid(x) = 1/(1+e^-x); all evaluated in fp64):

* ``base``:  a ~ U(0.5, 1), p ~ logU(1e-3, 1), phi ~ logU(1e-2, 10), b ~ N(0, 1)
* ``lm``:    a = sigmoid(N(2, 1)), p = softplus(N(-3, 1)), phi = softplus(N(0, 1)),
             b ~ N(0, 1)
* ``stiff``: a ~ U(0.99, 1), p ~ logU(1e-6, 1e-3), phi ~ logU(1e-3, 1e3),
             b ~ N(0, 1)
"""
from __future__ import annotations

import dataclasses
import re
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Dict, Iterator, Tuple

import numpy as np

INPUT_NAMES = ("a", "p", "phi", "b")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    T: int
    dtype: str          # "f32" or "bf16": the dtype of a, p, phi, b on the device
    dist: str           # "base", "lm" or "stiff"
    seed: int
    decode: bool = False  # True: T sequential one-token decode steps
    summary: str = ""

    @property
    def channels(self) -> int:
        return self.B * self.H * self.N

    @property
    def token_channels(self) -> int:
        return self.B * self.T * self.H * self.N

    def with_shape(self, **kw) -> "Workload":
        """The same distributions and seed at another shape; the summary
        names the new sizes."""
        summary = self.summary
        for k, v in kw.items():
            if k in ("B", "H", "N"):
                summary = re.sub(rf"\b{k}=\d+", f"{k}={v}", summary)
            elif k == "T":
                summary = re.sub(r"\bT=\d+", f"T={v}", summary)
                summary = re.sub(r"\b\d+ one-token steps", f"{v} one-token steps", summary)
        return dataclasses.replace(self, summary=summary, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 1, 64, 256, "f32", "base", 0,
                     summary="tiny forward scan, fp32, B=1 H=1 N=64 T=256"),
    "lm_layer": Workload("lm_layer", 8, 16, 128, 2048, "bf16", "lm", 1,
                         summary="LM-layer-shaped forward scan, bf16 in / fp32 state, "
                                 "B=8 H=16 N=128 T=2048"),
    "long": Workload("long", 1, 32, 128, 65536, "f32", "base", 2,
                     summary="long-sequence forward scan, fp32, B=1 H=32 N=128 T=65536"),
    "stiff": Workload("stiff", 256, 8, 64, 128, "f32", "stiff", 3,
                      summary="stiff state-tracking-shaped scan, fp32, B=256 H=8 N=64 T=128"),
    "decode": Workload("decode", 256, 32, 128, 1024, "f32", "base", 4, decode=True,
                       summary="recurrent decode, fp32 resident state, B=256 H=32 N=128, "
                               "1024 one-token steps"),
}

# Elements drawn per block; any value gives the same arrays.
_BLOCK_ELEMS = 1 << 24


def _log_uniform(rng: np.random.Generator, lo: float, hi: float, n: int) -> np.ndarray:
    return np.exp(rng.uniform(np.log(lo), np.log(hi), n))


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _draw(dist: str, name: str, rng: np.random.Generator, n: int) -> np.ndarray:
    """n fp64 values of input `name` under distribution family `dist`."""
    if dist == "base":
        if name == "a":
            return rng.uniform(0.5, 1.0, n)
        if name == "p":
            return _log_uniform(rng, 1e-3, 1.0, n)
        if name == "phi":
            return _log_uniform(rng, 1e-2, 10.0, n)
        return rng.standard_normal(n)
    if dist == "lm":
        if name == "a":
            return _sigmoid(rng.normal(2.0, 1.0, n))
        if name == "p":
            return _softplus(rng.normal(-3.0, 1.0, n))
        if name == "phi":
            return _softplus(rng.normal(0.0, 1.0, n))
        return rng.standard_normal(n)
    if dist == "stiff":
        if name == "a":
            return rng.uniform(0.99, 1.0, n)
        if name == "p":
            return _log_uniform(rng, 1e-6, 1e-3, n)
        if name == "phi":
            return _log_uniform(rng, 1e-3, 1e3, n)
        return rng.standard_normal(n)
    raise ValueError(f"unknown distribution family {dist!r}")


def round_to_bf16(x32: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); result stays fp32."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _streams(seed: int):
    children = np.random.SeedSequence(seed).spawn(len(INPUT_NAMES))
    return [np.random.Generator(np.random.PCG64(c)) for c in children]


def iter_rows(w: Workload, rows_per_block: int | None = None
              ) -> Iterator[Tuple[int, int, Dict[str, np.ndarray]]]:
    """Yield (row0, row1, arrays) blocks of the flattened (B*T) row axis.

    Each array in ``arrays`` is fp32 of shape [row1 - row0, H, N]; row r is
    token t = r % T of batch b = r // T.
    """
    HN = w.H * w.N
    rows = w.B * w.T
    if rows_per_block is None:
        rows_per_block = max(1, _BLOCK_ELEMS // max(HN, 1))
    rngs = _streams(w.seed)

    def one(name, rng, n):
        x = _draw(w.dist, name, rng, n).astype(np.float32)
        return round_to_bf16(x) if w.dtype == "bf16" else x

    # the four streams are independent: draw them in parallel (numpy releases the GIL)
    with ThreadPoolExecutor(max_workers=len(INPUT_NAMES)) as pool:
        r0 = 0
        while r0 < rows:
            r1 = min(rows, r0 + rows_per_block)
            n = (r1 - r0) * HN
            futs = [pool.submit(one, name, rng, n) for name, rng in zip(INPUT_NAMES, rngs)]
            out = {name: f.result().reshape(r1 - r0, w.H, w.N) for name, f in zip(INPUT_NAMES, futs)}
            yield r0, r1, out
            r0 = r1


def generate(w: Workload) -> Dict[str, np.ndarray]:
    """All inputs of a workload as fp32 arrays: a, p, phi, b [B, T, H, N];
    lam0, eta0 [B, H, N]."""
    HN = w.H * w.N
    full = {k: np.empty((w.B * w.T, w.H, w.N), dtype=np.float32) for k in INPUT_NAMES}
    if w.B * w.T * HN:
        for r0, r1, blk in iter_rows(w):
            for k in INPUT_NAMES:
                full[k][r0:r1] = blk[k]
    out = {k: v.reshape(w.B, w.T, w.H, w.N) for k, v in full.items()}
    out.update(prior(w))
    return out


def prior(w: Workload) -> Dict[str, np.ndarray]:
    return {"lam0": np.ones((w.B, w.H, w.N), dtype=np.float32),
            "eta0": np.zeros((w.B, w.H, w.N), dtype=np.float32)}


def random_prior(w: Workload, seed: int = 777) -> Dict[str, np.ndarray]:
    """A non-trivial prior: lam0 ~ logU(0.1, 10), eta0 ~ N(0, 1), fp32 [B, H, N]."""
    rng = np.random.default_rng([w.seed, seed])
    n = w.B * w.H * w.N
    return {"lam0": _log_uniform(rng, 0.1, 10.0, n).astype(np.float32).reshape(w.B, w.H, w.N),
            "eta0": rng.standard_normal(n).astype(np.float32).reshape(w.B, w.H, w.N)}


# Loss gradients with respect to the four outputs (lambda, eta, mu, var), the
# inputs of the backward scan: standard normal fp32, i.e. the gradients of a
# random linear loss.  Their streams are spawned from (seed, 1), independent
# of the forward inputs' streams.
GRAD_NAMES = ("g_lam", "g_eta", "g_mu", "g_var")


def iter_output_grad_rows(w: Workload, rows_per_block: int | None = None
                          ) -> Iterator[Tuple[int, int, Dict[str, np.ndarray]]]:
    """Like iter_rows, for the four output gradients."""
    HN = w.H * w.N
    rows = w.B * w.T
    if rows_per_block is None:
        rows_per_block = max(1, _BLOCK_ELEMS // max(HN, 1))
    children = np.random.SeedSequence([w.seed, 1]).spawn(len(GRAD_NAMES))
    rngs = [np.random.Generator(np.random.PCG64(c)) for c in children]
    with ThreadPoolExecutor(max_workers=len(GRAD_NAMES)) as pool:
        r0 = 0
        while r0 < rows:
            r1 = min(rows, r0 + rows_per_block)
            n = (r1 - r0) * HN
            futs = [pool.submit(lambda g, m: g.standard_normal(m, dtype=np.float32), rng, n) for rng in rngs]
            yield r0, r1, {k: f.result().reshape(r1 - r0, w.H, w.N) for k, f in zip(GRAD_NAMES, futs)}
            r0 = r1


def generate_output_grads(w: Workload) -> Dict[str, np.ndarray]:
    """All four output gradients of a workload, fp32 [B, T, H, N]."""
    full = {k: np.empty((w.B * w.T, w.H, w.N), dtype=np.float32) for k in GRAD_NAMES}
    if w.B * w.T * w.H * w.N:
        for r0, r1, blk in iter_output_grad_rows(w):
            for k in GRAD_NAMES:
                full[k][r0:r1] = blk[k]
    return {k: v.reshape(w.B, w.T, w.H, w.N) for k, v in full.items()}


def channel_sample(w: Workload, count: int, seed: int = 12345) -> np.ndarray:
    """A sorted, seeded sample of flat channel indices (b*H*N + h*N + n)."""
    C = w.channels
    count = min(count, C)
    rng = np.random.default_rng(seed)
    idx = rng.choice(C, size=count, replace=False)
    # always include the first and last channel (tile edges)
    idx = np.unique(np.concatenate([idx, [0, C - 1]]))
    return idx


# --------------------------------------------------------------------------
# The fused KLA layer: per-token operators and values of H heads, per-channel
# time-invariant decay and process noise over H x D x Ns state channels.
@dataclass(frozen=True)
class LayerWorkload:
    name: str
    B: int
    T: int
    H: int
    D: int          # value dimension per head
    Ns: int         # state expansion: state channels per value coordinate
    dtype: str      # "f32" or "bf16": dtype of k, q, v, w on the device
    seed: int
    summary: str = ""

    @property
    def channels(self) -> int:
        return self.B * self.H * self.D * self.Ns

    @property
    def token_channels(self) -> int:
        return self.T * self.channels

    def with_shape(self, **kw) -> "LayerWorkload":
        summary = self.summary
        for k, v in kw.items():
            if k in ("B", "T", "H", "D", "Ns"):
                summary = re.sub(rf"\b{k}=\d+", f"{k}={v}", summary)
        return dataclasses.replace(self, summary=summary, **kw)


LAYER_WORKLOADS: Dict[str, LayerWorkload] = {
    "layer": LayerWorkload("layer", 8, 2048, 4, 32, 16, "bf16", 5,
                           summary="fused KLA layer forward, bf16 operators and values / fp32 state, "
                                   "B=8 T=2048 H=4 D=32 Ns=16"),
}

LAYER_TOKEN_NAMES = ("k", "q", "v", "w")


def generate_layer(w: LayerWorkload) -> Dict[str, np.ndarray]:
    """Inputs of a layer workload as fp32 arrays: k, q [B, T, H, Ns] ~ N(0,
    1/Ns); v [B, T, H, D] ~ N(0, 1); w (value precision) [B, T, H, D] =
    softplus(N(0, 1)); a [H, D, Ns] = sigmoid(N(2, 1)) and p [H, D, Ns] =
    softplus(N(-3, 1)) (the LM-layer families of a and p, time-invariant per
    channel); prior lam0 = 1, eta0 = 0 [B, H, D, Ns].  k, q, v, w are rounded
    to bf16 for bf16 workloads."""
    children = np.random.SeedSequence([w.seed, 2]).spawn(6)
    rngs = [np.random.Generator(np.random.PCG64(c)) for c in children]
    B, T, H, D, Ns = w.B, w.T, w.H, w.D, w.Ns
    rnd = (lambda x: round_to_bf16(x.astype(np.float32))) if w.dtype == "bf16" else \
        (lambda x: x.astype(np.float32))
    out = {
        "k": rnd(rngs[0].standard_normal((B, T, H, Ns)) / np.sqrt(Ns)),
        "q": rnd(rngs[1].standard_normal((B, T, H, Ns)) / np.sqrt(Ns)),
        "v": rnd(rngs[2].standard_normal((B, T, H, D))),
        "w": rnd(_softplus(rngs[3].standard_normal((B, T, H, D)))),
        "a": _sigmoid(rngs[4].normal(2.0, 1.0, (H, D, Ns))).astype(np.float32),
        "p": _softplus(rngs[5].normal(-3.0, 1.0, (H, D, Ns))).astype(np.float32),
        "lam0": np.ones((B, H, D, Ns), dtype=np.float32),
        "eta0": np.zeros((B, H, D, Ns), dtype=np.float32),
    }
    return out


def random_layer_prior(w: LayerWorkload, seed: int = 778) -> Dict[str, np.ndarray]:
    """A non-trivial layer prior: lam0 ~ logU(0.1, 10), eta0 ~ N(0, 1), fp32 [B, H, D, Ns]."""
    rng = np.random.default_rng([w.seed, seed])
    shape = (w.B, w.H, w.D, w.Ns)
    return {"lam0": _log_uniform(rng, 0.1, 10.0, int(np.prod(shape))).astype(np.float32).reshape(shape),
            "eta0": rng.standard_normal(shape).astype(np.float32)}


# --------------------------------------------------------------------------
# Deterministic time-invariant channels (the convolutional form): p = 0 and a
# decay per channel, constant in time.  phi and b are the "base" family's
# streams of the same seed (drawn exactly as for a ``base`` workload); a is
# drawn per channel from its own stream, U(a_lo, a_hi) fp32 [B, H, N].
LTI_WORKLOADS: Dict[str, Workload] = {
    "lti": Workload("lti", 1, 32, 128, 65536, "f32", "base", 6,
                    summary="deterministic time-invariant forward scan (convolutional form), fp32, "
                            "B=1 H=32 N=128 T=65536, p=0, a~U(0.9995,1.0005) per channel"),
}
LTI_DECAY_RANGE = (0.9995, 1.0005)


def iter_lti_rows(w: Workload, rows_per_block: int | None = None
                  ) -> Iterator[Tuple[int, int, Dict[str, np.ndarray]]]:
    """Like iter_rows, for phi and b only (fp32 [rows, H, N] blocks)."""
    HN = w.H * w.N
    rows = w.B * w.T
    if rows_per_block is None:
        rows_per_block = max(1, _BLOCK_ELEMS // max(HN, 1))
    rngs = _streams(w.seed)[2:]

    def one(name, rng, n):
        x = _draw(w.dist, name, rng, n).astype(np.float32)
        return round_to_bf16(x) if w.dtype == "bf16" else x

    with ThreadPoolExecutor(max_workers=2) as pool:
        r0 = 0
        while r0 < rows:
            r1 = min(rows, r0 + rows_per_block)
            n = (r1 - r0) * HN
            futs = [pool.submit(one, name, rng, n) for name, rng in zip(("phi", "b"), rngs)]
            yield r0, r1, {name: f.result().reshape(r1 - r0, w.H, w.N) for name, f in zip(("phi", "b"), futs)}
            r0 = r1


def lti_decay(w: Workload, lo: float = LTI_DECAY_RANGE[0], hi: float = LTI_DECAY_RANGE[1]) -> np.ndarray:
    """The per-channel decay of a time-invariant workload: U(lo, hi), fp32 [B, H, N]."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, 3])))
    return rng.uniform(lo, hi, (w.B, w.H, w.N)).astype(np.float32)


def generate_lti(w: Workload, decay: Tuple[float, float] = LTI_DECAY_RANGE) -> Dict[str, np.ndarray]:
    """All inputs of a time-invariant workload: a [B, H, N], phi, b
    [B, T, H, N] (fp32 arrays; bf16-rounded values for bf16 workloads),
    lam0 = 1, eta0 = 0 [B, H, N]."""
    HN = w.H * w.N
    full = {k: np.empty((w.B * w.T, w.H, w.N), dtype=np.float32) for k in ("phi", "b")}
    if w.B * w.T * HN:
        for r0, r1, blk in iter_lti_rows(w):
            for k in ("phi", "b"):
                full[k][r0:r1] = blk[k]
    out = {k: v.reshape(w.B, w.T, w.H, w.N) for k, v in full.items()}
    out["a"] = lti_decay(w, *decay)
    out.update(prior(w))
    return out


SPECIAL_CASES = ["no_process_noise", "no_observation", "precision_sum", "negative_decay", "mixed_zeros"]


def special_inputs(kind: str, B: int = 2, T: int = 400, H: int = 2, N: int = 48, seed: int = 77
                   ) -> Dict[str, np.ndarray]:
    """Degenerate and special cases of the method, seeded, fp32: p = 0 with
    a near +-1 (the affine Moebius case), phi = b = 0 (no observation), a = 1
    and p = 0 (precision sum), a of either sign, and a mix of zero noise and
    missing observations; a non-trivial prior."""
    rng = np.random.default_rng(seed)
    sh = (B, T, H, N)
    a = rng.uniform(0.5, 1.0, sh)
    p = np.exp(rng.uniform(np.log(1e-3), 0.0, sh))
    phi = np.exp(rng.uniform(np.log(1e-2), np.log(10.0), sh))
    b = rng.standard_normal(sh)
    if kind == "no_process_noise":      # p = 0: the affine Moebius case
        p[:] = 0.0
        a = rng.uniform(0.98, 1.02, sh) * np.where(rng.random(sh) < 0.3, -1.0, 1.0)
    elif kind == "no_observation":      # phi = 0, b = 0: every update leaves the prior
        phi[:] = 0.0
        b[:] = 0.0
    elif kind == "precision_sum":       # a = 1, p = 0: lambda is a running sum of phi
        a[:] = 1.0
        p[:] = 0.0
    elif kind == "negative_decay":      # the gate follows the sign of a
        a *= np.where(rng.random(sh) < 0.5, -1.0, 1.0)
    elif kind == "mixed_zeros":         # some tokens without noise, some without evidence
        p[rng.random(sh) < 0.3] = 0.0
        z = rng.random(sh) < 0.3
        phi[z] = 0.0
        b[z] = 0.0
    x = {k: v.astype(np.float32) for k, v in (("a", a), ("p", p), ("phi", phi), ("b", b))}
    x["lam0"] = rng.uniform(0.5, 2.0, (B, H, N)).astype(np.float32)
    x["eta0"] = rng.standard_normal((B, H, N)).astype(np.float32)
    return x
