"""Helpers for the CUDA-vs-oracle parity tests.

Tolerances (per output tensor, per element):

* lambda and var are strictly positive: |x - ref| <= rtol * |ref|.
* eta and mu cross zero (b ~ N(0, 1)), so a pure relative test is ill-posed
  near their zeros; they use |x - ref| <= rtol * (|ref| + rms_t(ref)), where
  rms_t is the root-mean-square of that channel's reference values over time.

rtol = 1e-5 for fp32 inputs and 2e-2 for bf16 inputs (fp32 state and
arithmetic on the exact bf16 values).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

import oracle
from kalman_linear_attention_b200 import workloads as wl

RTOL = {"f32": 1e-5, "bf16": 2e-2}
OUTPUTS = ("lam", "eta", "mu", "var")


def max_errors(got: Dict[str, np.ndarray], ref: Dict[str, np.ndarray], time_axis: int
               ) -> Dict[str, float]:
    """Max relative error (lam, var) and max rms-scaled error (eta, mu)."""
    errs = {}
    for k in OUTPUTS:
        if k not in got or got[k] is None:
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
        if k in ("lam", "var"):
            errs[k] = float(np.max(np.abs(g - r) / np.abs(r)))
        else:
            rms = np.sqrt(np.mean(r * r, axis=time_axis, keepdims=True))
            errs[k] = float(np.max(np.abs(g - r) / (np.abs(r) + rms + 1e-300)))
    return errs


def assert_parity(got, ref, rtol: float, time_axis: int, what: str = "") -> Dict[str, float]:
    errs = max_errors(got, ref, time_axis)
    bad = {k: v for k, v in errs.items() if not v <= rtol}
    assert not bad, f"{what}: errors above rtol={rtol:g}: {bad} (all: {errs})"
    return errs


def torch_dtype(w: wl.Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_device(w: wl.Workload, device, sample: Optional[np.ndarray] = None):
    """Stream a workload's inputs into device tensors [B, T, H, N].

    Returns (inputs, sampled): ``inputs`` maps a, p, phi, b, lam0, eta0 to
    device tensors; ``sampled`` maps a, p, phi, b to host fp32 arrays [T, K]
    holding the K channels listed in ``sample`` (flat channel indices), or is
    None.
    """
    B, T, H, N = w.B, w.T, w.H, w.N
    HN = H * N
    dt = torch_dtype(w)
    dev = {k: torch.empty((B, T, H, N), dtype=dt, device=device) for k in wl.INPUT_NAMES}
    flat = {k: v.view(B * T, HN) for k, v in dev.items()}
    sampled = None
    if sample is not None:
        sb, shn = np.divmod(np.asarray(sample), HN)
        sampled = {k: np.empty((T, len(sample)), dtype=np.float32) for k in wl.INPUT_NAMES}
    for r0, r1, blk in wl.iter_rows(w):
        rows = np.arange(r0, r1)
        for k in wl.INPUT_NAMES:
            x = blk[k].reshape(r1 - r0, HN)
            flat[k][r0:r1].copy_(torch.from_numpy(x).to(dt))
            if sampled is not None:
                for j in range(len(sample)):
                    m = (rows // T) == sb[j]
                    if m.any():
                        sampled[k][rows[m] % T, j] = x[m, shn[j]]
    pri = wl.prior(w)
    dev["lam0"] = torch.from_numpy(pri["lam0"]).to(device)
    dev["eta0"] = torch.from_numpy(pri["eta0"]).to(device)
    return dev, sampled


def gather_channels(t: torch.Tensor, sample: np.ndarray, HN: int) -> np.ndarray:
    """[B, T, H, N] device tensor -> host fp64 [T, K] of the sampled channels."""
    B, T = t.shape[0], t.shape[1]
    sb, shn = np.divmod(np.asarray(sample), HN)
    v = t.view(B, T, HN)
    idx_b = torch.as_tensor(sb, device=t.device)
    idx_c = torch.as_tensor(shn, device=t.device)
    return v[idx_b, :, idx_c].transpose(0, 1).double().cpu().numpy()


def oracle_on_sample(sampled: Dict[str, np.ndarray], lam0: np.ndarray, eta0: np.ndarray,
                     threads: int = 8) -> Dict[str, np.ndarray]:
    """Run the oracle on sampled channels ([T, K] arrays); returns [T, K] fp64."""
    T, K = sampled["a"].shape
    x = {k: sampled[k].reshape(1, T, 1, K) for k in wl.INPUT_NAMES}
    out = oracle.forward(x["a"], x["p"], x["phi"], x["b"],
                         np.asarray(lam0, dtype=np.float64).reshape(1, 1, K),
                         np.asarray(eta0, dtype=np.float64).reshape(1, 1, K), threads=threads)
    return {k: v.reshape(T, K) for k, v in out.items()}
