"""Thin Python binding of the C ABI in ``include/kla.h`` (ctypes).

Argument marshalling only: every step of the filter runs in the CUDA kernels
of ``libkla.so``.  PyTorch is used for device memory and streams.  There is no
CPU fallback: without the built library, or without a CUDA device, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libkla.so")

KLA_F32 = 0
KLA_BF16 = 1
STATUS = {0: "KLA_OK", 1: "KLA_ERR_INVALID_ARG", 2: "KLA_ERR_UNSUPPORTED_DTYPE",
          3: "KLA_ERR_WORKSPACE_TOO_SMALL", 4: "KLA_ERR_CUDA", 5: "KLA_ERR_TIMEOUT",
          6: "KLA_ERR_MISALIGNED", 7: "KLA_ERR_TOO_LARGE"}
KLA_OK, KLA_ERR_INVALID_ARG, KLA_ERR_UNSUPPORTED_DTYPE = 0, 1, 2
KLA_ERR_WORKSPACE_TOO_SMALL, KLA_ERR_CUDA, KLA_ERR_TIMEOUT, KLA_ERR_MISALIGNED = 3, 4, 5, 6
KLA_ERR_TOO_LARGE = 7
STATIC_SCRATCH_BYTES = 32 << 20  # KLA_STATIC_SCRATCH_BYTES

# Every exported symbol of include/kla.h, with (restype, argtypes).
_VP, _I64, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
SIGNATURES = {
    "kla_abi_version": (ctypes.c_int, []),
    "kla_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "kla_scan_forward_workspace_size": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int,
                                                       ctypes.POINTER(_SZ)]),
    "kla_scan_forward": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP,
                                        _VP, _I64, _I64, _I64, _I64, _VP, _SZ, _VP]),
    "kla_scan_step": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP,
                                     _I64, _I64, _I64, _VP]),
    "kla_get_error": (ctypes.c_int, [_VP]),
    "kla_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "kla_debug_unset_flag_wait": (ctypes.c_int, [_VP]),
    "kla_forward_chunk_tokens": (ctypes.c_int, []),
    "kla_debug_stall_chunk": (ctypes.c_int, [_I64]),
    "kla_debug_force_forward_kernel": (ctypes.c_int, [ctypes.c_int]),
    "kla_scan_forward_plan": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP, _VP,
                                             ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "kla_scan_forward_static": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP,
                                               _VP, _VP, _I64, _I64, _I64, _I64, _VP]),
    "kla_scan_forward_host_workspace_size": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int, _I64,
                                                            ctypes.POINTER(_SZ)]),
    "kla_scan_forward_host": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP, _VP,
                                             _I64, _I64, _I64, _I64, _I64, _VP, _SZ, _VP]),
    "kla_scan_backward_workspace_size": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int,
                                                        ctypes.POINTER(_SZ)]),
    "kla_scan_backward": (ctypes.c_int, [_VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                         _VP, _VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _I64, _VP, _SZ, _VP]),
    "kla_scan_backward_plan": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP,
                                              ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "kla_debug_force_backward_kernel": (ctypes.c_int, [ctypes.c_int]),
    "kla_layer_forward_workspace_size": (ctypes.c_int, [_I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                                                        ctypes.POINTER(_SZ)]),
    "kla_layer_forward": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                         _VP, _I64, _I64, _I64, _I64, _I64, _VP, _SZ, _VP]),
    "kla_layer_step": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP, _VP,
                                      _I64, _I64, _I64, _I64, _VP]),
    "kla_attention_weights": (ctypes.c_int, [_VP, _VP, ctypes.c_int, _VP, _VP, _I64, _I64, _I64, _I64,
                                             _I64, _I64, _I64, _VP]),
    "kla_scan_forward_lti_workspace_size": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int,
                                                           ctypes.POINTER(_SZ)]),
    "kla_scan_forward_lti": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP, _VP,
                                            _I64, _I64, _I64, _I64, _VP, _SZ, _VP]),
    "kla_scan_forward_lti_plan": (ctypes.c_int, [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP,
                                                 ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
}
ATTENTION_MAX_WINDOW = 64  # KLA_ATTENTION_MAX_WINDOW

_lib: Optional[ctypes.CDLL] = None


class KlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def load_library(path: str = LIBRARY) -> ctypes.CDLL:
    """Load ``libkla.so`` and declare the C signatures (raises if it is missing)."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is not built; build it with "
            "`python -m kalman_linear_attention_b200._build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _check(status: int, what: str) -> None:
    if status != KLA_OK:
        raise KlaError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KLA_F32
    if t.dtype == torch.bfloat16:
        return KLA_BF16
    raise TypeError(f"inputs must be float32 or bfloat16, got {t.dtype}")


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _require_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensor must be on a CUDA device")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensor must be contiguous")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def workspace_size(B: int, T: int, H: int, N: int, dtype: torch.dtype = torch.float32) -> int:
    code = KLA_BF16 if dtype == torch.bfloat16 else KLA_F32
    out = ctypes.c_size_t(0)
    _check(lib().kla_scan_forward_workspace_size(B, T, H, N, code, ctypes.byref(out)),
           "kla_scan_forward_workspace_size")
    return int(out.value)


def forward_plan(a: torch.Tensor, p: torch.Tensor, phi: torch.Tensor, b: torch.Tensor) -> Tuple[int, int]:
    """(kernel, launches) that scan_forward would use for these inputs:
    kernel 1 = chunked (workspace carries), 2 = channel-owning streaming."""
    B, T, H, N = a.shape
    k, n = ctypes.c_int(0), ctypes.c_int(0)
    with torch.cuda.device(a.device):
        _check(lib().kla_scan_forward_plan(B, T, H, N, _dtype_code(a), _ptr(a), _ptr(p), _ptr(phi),
                                           _ptr(b), ctypes.byref(k), ctypes.byref(n)),
               "kla_scan_forward_plan")
    return int(k.value), int(n.value)


def chunk_tokens() -> int:
    return int(lib().kla_forward_chunk_tokens())


def new_workspace(B: int, T: int, H: int, N: int, dtype: torch.dtype, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(workspace_size(B, T, H, N, dtype), 1), dtype=torch.uint8, device=device)


def scan_forward(a: torch.Tensor, p: torch.Tensor, phi: torch.Tensor, b: torch.Tensor,
                 lam0: torch.Tensor, eta0: torch.Tensor, *,
                 want_mu: bool = True, want_var: bool = True,
                 out: Optional[Sequence[Optional[torch.Tensor]]] = None,
                 workspace: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None,
                 ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor], Optional[torch.Tensor]]:
    """Filter [B, T, H, N] inputs from the [B, H, N] prior.

    Returns (lambda, eta, mu, var) as fp32 [B, T, H, N] tensors (mu / var are
    None when not wanted).  CUDA inputs give CUDA outputs, enqueued on
    ``stream`` (default: the current stream) without synchronising.  CPU
    inputs (ideally pinned) are copied to the current CUDA device, filtered
    there, and copied back; the call then returns CPU tensors after a
    synchronise.  ``out`` may supply the four output tensors (None entries
    for skipped outputs) on the side the results are returned on.
    """
    if not (a.shape == p.shape == phi.shape == b.shape) or a.dim() != 4:
        raise ValueError("a, p, phi, b must share one [B, T, H, N] shape")
    if not (a.dtype == p.dtype == phi.dtype == b.dtype):
        raise TypeError("a, p, phi, b must share one dtype")
    B, T, H, N = a.shape
    if lam0.shape != (B, H, N) or eta0.shape != (B, H, N):
        raise ValueError("lam0 and eta0 must be [B, H, N]")
    if lam0.dtype != torch.float32 or eta0.dtype != torch.float32:
        raise TypeError("lam0 and eta0 must be float32")
    host = not a.is_cuda
    if host:
        return _scan_forward_host(a, p, phi, b, lam0, eta0, want_mu=want_mu, want_var=want_var, out=out,
                                  workspace=workspace, stream=stream)

    _require_cuda(a, p, phi, b, lam0, eta0)
    code = _dtype_code(a)
    dev = a.device
    if out is None:
        outs = [torch.empty((B, T, H, N), dtype=torch.float32, device=dev),
                torch.empty((B, T, H, N), dtype=torch.float32, device=dev),
                torch.empty((B, T, H, N), dtype=torch.float32, device=dev) if want_mu else None,
                torch.empty((B, T, H, N), dtype=torch.float32, device=dev) if want_var else None]
    else:
        outs = list(out)
        _require_cuda(*[o for o in outs if o is not None])
    if workspace is None:
        workspace = new_workspace(B, T, H, N, a.dtype, dev)
    with torch.cuda.device(dev):
        st = kla_scan_forward_raw(a, p, phi, b, code, lam0, eta0, outs, B, T, H, N, workspace,
                                  _stream_handle(stream))
    _check(st, "kla_scan_forward")
    return tuple(outs)


def host_workspace_size(B: int, T: int, H: int, N: int, dtype: torch.dtype = torch.float32,
                        t_block: int = 0) -> int:
    code = KLA_BF16 if dtype == torch.bfloat16 else KLA_F32
    out = ctypes.c_size_t(0)
    _check(lib().kla_scan_forward_host_workspace_size(B, T, H, N, code, t_block, ctypes.byref(out)),
           "kla_scan_forward_host_workspace_size")
    return int(out.value)


def _scan_forward_host(a, p, phi, b, lam0, eta0, *, want_mu, want_var, out, workspace, stream,
                       t_block: int = 0):
    """kla_scan_forward_host: host tensors in and out, copies pipelined with
    the scan on the current CUDA device; returns after the outputs are in
    host memory."""
    for t in (a, p, phi, b, lam0, eta0):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host path: every tensor must be a contiguous CPU tensor")
    B, T, H, N = a.shape
    pinned = a.is_pinned()
    if out is None:
        outs = [torch.empty((B, T, H, N), dtype=torch.float32, pin_memory=pinned),
                torch.empty((B, T, H, N), dtype=torch.float32, pin_memory=pinned),
                torch.empty((B, T, H, N), dtype=torch.float32, pin_memory=pinned) if want_mu else None,
                torch.empty((B, T, H, N), dtype=torch.float32, pin_memory=pinned) if want_var else None]
    else:
        outs = list(out)
    dev = torch.device("cuda", torch.cuda.current_device())
    if workspace is None:
        workspace = torch.empty(max(host_workspace_size(B, T, H, N, a.dtype, t_block), 1), dtype=torch.uint8,
                                device=dev)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        st = lib().kla_scan_forward_host(
            _ptr(a), _ptr(p), _ptr(phi), _ptr(b), _dtype_code(a), _ptr(lam0), _ptr(eta0),
            _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), _ptr(outs[3]), B, T, H, N, t_block,
            _ptr(workspace), workspace.numel(), s.cuda_stream)
    _check(st, "kla_scan_forward_host")
    s.synchronize()
    return tuple(outs)


def kla_scan_forward_raw(a, p, phi, b, code, lam0, eta0, outs, B, T, H, N, workspace, stream) -> int:
    """Direct C-ABI call; returns the status code."""
    return lib().kla_scan_forward(
        _ptr(a), _ptr(p), _ptr(phi), _ptr(b), code, _ptr(lam0), _ptr(eta0),
        _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), _ptr(outs[3]), B, T, H, N,
        _ptr(workspace), workspace.numel() if workspace is not None else 0, stream)


def scan_step(a: torch.Tensor, p: torch.Tensor, phi: torch.Tensor, b: torch.Tensor,
              lam_state: torch.Tensor, eta_state: torch.Tensor, *,
              mu_out: Optional[torch.Tensor] = None, var_out: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> None:
    """One decode token for every channel of [B, H, N] inputs; updates
    ``lam_state`` / ``eta_state`` in place and writes ``mu_out`` / ``var_out``
    when given.  Enqueued on ``stream`` (default: the current stream)."""
    if not (a.shape == p.shape == phi.shape == b.shape == lam_state.shape == eta_state.shape):
        raise ValueError("step inputs and state must share one [B, H, N] shape")
    if a.dim() != 3:
        raise ValueError("step tensors are [B, H, N]")
    if lam_state.dtype != torch.float32 or eta_state.dtype != torch.float32:
        raise TypeError("state must be float32")
    _require_cuda(a, p, phi, b, lam_state, eta_state, mu_out, var_out)
    B, H, N = a.shape
    with torch.cuda.device(a.device):
        st = lib().kla_scan_step(_ptr(a), _ptr(p), _ptr(phi), _ptr(b), _dtype_code(a),
                                 _ptr(lam_state), _ptr(eta_state), _ptr(mu_out), _ptr(var_out),
                                 B, H, N, _stream_handle(stream))
    _check(st, "kla_scan_step")


def get_error(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise and return the device-side status (KLA_OK, KLA_ERR_TIMEOUT, ...)."""
    return int(lib().kla_get_error(_stream_handle(stream)))


def set_wait_limit_ns(ns: int) -> None:
    _check(lib().kla_set_wait_limit_ns(int(ns)), "kla_set_wait_limit_ns")


def debug_unset_flag_wait(stream: Optional[torch.cuda.Stream] = None) -> None:
    _check(lib().kla_debug_unset_flag_wait(_stream_handle(stream)), "kla_debug_unset_flag_wait")


def debug_force_forward_kernel(which: int) -> None:
    """0: choose by shape; 1: chunked kernel (workspace carries); 2: streaming kernel."""
    _check(lib().kla_debug_force_forward_kernel(int(which)), "kla_debug_force_forward_kernel")


def debug_stall_chunk(chunk: int) -> None:
    _check(lib().kla_debug_stall_chunk(int(chunk)), "kla_debug_stall_chunk")


def scan_forward_static(a: torch.Tensor, p: torch.Tensor, phi: torch.Tensor, b: torch.Tensor,
                        lam0: torch.Tensor, eta0: torch.Tensor,
                        out: Sequence[Optional[torch.Tensor]],
                        stream: Optional[torch.cuda.Stream] = None) -> None:
    """kla_scan_forward_static: the forward scan for callers that cannot
    allocate device memory.  The caller passes every tensor, outputs
    included (``out`` = lambda, eta, mu, var; mu / var may be None); the
    library uses its own fixed static device scratch (KLA_STATIC_SCRATCH_BYTES),
    so nothing is allocated.  Calls that overlap on the GPU share that scratch
    and must be serialised.  Raises KlaError(KLA_ERR_TOO_LARGE) when the
    problem does not fit."""
    if not (a.shape == p.shape == phi.shape == b.shape) or a.dim() != 4:
        raise ValueError("a, p, phi, b must share one [B, T, H, N] shape")
    B, T, H, N = a.shape
    outs = list(out)
    _require_cuda(a, p, phi, b, lam0, eta0, *outs)
    with torch.cuda.device(a.device):
        st = lib().kla_scan_forward_static(
            _ptr(a), _ptr(p), _ptr(phi), _ptr(b), _dtype_code(a), _ptr(lam0), _ptr(eta0),
            _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), _ptr(outs[3]), B, T, H, N,
            _stream_handle(stream))
    _check(st, "kla_scan_forward_static")


# ---------------------------------------------------------------- gradients
def backward_workspace_size(B: int, T: int, H: int, N: int, dtype: torch.dtype = torch.float32) -> int:
    code = KLA_BF16 if dtype == torch.bfloat16 else KLA_F32
    out = ctypes.c_size_t(0)
    _check(lib().kla_scan_backward_workspace_size(B, T, H, N, code, ctypes.byref(out)),
           "kla_scan_backward_workspace_size")
    return int(out.value)


def backward_plan(a: torch.Tensor, p: torch.Tensor) -> Tuple[int, int]:
    """(kernel, launches) that scan_backward would use: kernel 1 = one thread
    per channel, 2 = channel-owning streaming kernel."""
    B, T, H, N = a.shape
    k, n = ctypes.c_int(0), ctypes.c_int(0)
    with torch.cuda.device(a.device):
        _check(lib().kla_scan_backward_plan(B, T, H, N, _dtype_code(a), _ptr(a), _ptr(p), ctypes.byref(k),
                                            ctypes.byref(n)), "kla_scan_backward_plan")
    return int(k.value), int(n.value)


def debug_force_backward_kernel(which: int) -> None:
    """0: choose by shape; 1: one thread per channel; 2: streaming kernel."""
    _check(lib().kla_debug_force_backward_kernel(int(which)), "kla_debug_force_backward_kernel")


def scan_backward(a: torch.Tensor, p: torch.Tensor, lam0: torch.Tensor, eta0: torch.Tensor,
                  lam: torch.Tensor, eta: torch.Tensor,
                  g_lam: Optional[torch.Tensor] = None, g_eta: Optional[torch.Tensor] = None,
                  g_mu: Optional[torch.Tensor] = None, g_var: Optional[torch.Tensor] = None, *,
                  want: Sequence[bool] = (True,) * 6,
                  out: Optional[Sequence[Optional[torch.Tensor]]] = None,
                  workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> Tuple[Optional[torch.Tensor], ...]:
    """Gradients through scan_forward (kla_scan_backward).

    ``a``, ``p`` are the forward inputs, ``lam0``, ``eta0`` its prior and
    ``lam``, ``eta`` its outputs; ``g_*`` are the loss gradients with respect
    to the four outputs (None = zero).  Returns the gradients with respect to
    (a, p, phi, b, lam0, eta0): the first four in the inputs' dtype, the prior
    ones fp32, None where ``want`` is False.  Enqueued on ``stream`` without
    synchronising.
    """
    if a.dim() != 4 or a.shape != p.shape or a.dtype != p.dtype:
        raise ValueError("a and p must share one [B, T, H, N] shape and dtype")
    B, T, H, N = a.shape
    if lam.shape != a.shape or eta.shape != a.shape:
        raise ValueError("lam and eta must be the forward outputs, [B, T, H, N]")
    if lam0.shape != (B, H, N) or eta0.shape != (B, H, N):
        raise ValueError("lam0 and eta0 must be [B, H, N]")
    grads_in = [g_lam, g_eta, g_mu, g_var]
    for t in [lam, eta, lam0, eta0] + [g for g in grads_in if g is not None]:
        if t.dtype != torch.float32:
            raise TypeError("states, prior and output gradients must be float32")
    for g in grads_in:
        if g is not None and g.shape != a.shape:
            raise ValueError("output gradients must be [B, T, H, N]")
    _require_cuda(a, p, lam0, eta0, lam, eta, *grads_in)
    code = _dtype_code(a)
    dev = a.device
    if out is None:
        outs = [torch.empty((B, T, H, N), dtype=a.dtype, device=dev) if w else None for w in want[:4]]
        outs += [torch.empty((B, H, N), dtype=torch.float32, device=dev) if w else None for w in want[4:6]]
    else:
        outs = list(out)
        _require_cuda(*outs)
    if workspace is None:
        n = backward_workspace_size(B, T, H, N, a.dtype)
        workspace = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    with torch.cuda.device(dev):
        st = lib().kla_scan_backward(
            _ptr(a), _ptr(p), code, _ptr(lam0), _ptr(eta0), _ptr(lam), _ptr(eta),
            *[_ptr(g) for g in grads_in], *[_ptr(o) for o in outs], B, T, H, N,
            _ptr(workspace), workspace.numel() if workspace is not None else 0, _stream_handle(stream))
    _check(st, "kla_scan_backward")
    return tuple(outs)


class KalmanFilterScan(torch.autograd.Function):
    """Differentiable filter scan: forward = kla_scan_forward, backward =
    kla_scan_backward.  Inputs (a, p, phi, b, lam0, eta0) as in scan_forward
    (CUDA tensors); returns (lambda, eta, mu, var)."""

    @staticmethod
    def forward(ctx, a, p, phi, b, lam0, eta0):
        ctx.set_materialize_grads(False)
        lam, eta, mu, var = scan_forward(a, p, phi, b, lam0, eta0)
        ctx.save_for_backward(a, p, lam0, eta0, lam, eta)
        return lam, eta, mu, var

    @staticmethod
    def backward(ctx, g_lam, g_eta, g_mu, g_var):
        a, p, lam0, eta0, lam, eta = ctx.saved_tensors
        grads = [None if g is None else g.contiguous() for g in (g_lam, g_eta, g_mu, g_var)]
        if all(g is None for g in grads):
            return (None,) * 6
        return scan_backward(a, p, lam0, eta0, lam, eta, *grads, want=ctx.needs_input_grad)


def kalman_filter(a: torch.Tensor, p: torch.Tensor, phi: torch.Tensor, b: torch.Tensor,
                  lam0: torch.Tensor, eta0: torch.Tensor):
    """(lambda, eta, mu, var) of the filter, differentiable with respect to
    every input through the CUDA backward scan."""
    return KalmanFilterScan.apply(a, p, phi, b, lam0, eta0)


# ------------------------------------------------------------ fused layer
def layer_workspace_size(B: int, T: int, H: int, D: int, Ns: int, dtype: torch.dtype = torch.float32) -> int:
    code = KLA_BF16 if dtype == torch.bfloat16 else KLA_F32
    out = ctypes.c_size_t(0)
    _check(lib().kla_layer_forward_workspace_size(B, T, H, D, Ns, code, ctypes.byref(out)),
           "kla_layer_forward_workspace_size")
    return int(out.value)


def layer_forward(k: torch.Tensor, q: torch.Tensor, v: torch.Tensor, w: torch.Tensor,
                  a: torch.Tensor, p: torch.Tensor, lam0: torch.Tensor, eta0: torch.Tensor, *,
                  want_s: bool = True, want_state: bool = True,
                  out: Optional[Sequence[Optional[torch.Tensor]]] = None,
                  workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None):
    """The KLA layer's filter with evidence formation and readout fused
    (kla_layer_forward): k, q [B, T, H, Ns]; v, w [B, T, H, D] (one dtype,
    fp32 or bf16); a, p [H, D, Ns] fp32; lam0, eta0 [B, H, D, Ns] fp32.
    Returns (y, s, lam_T, eta_T): y, s fp32 [B, T, H, D], the final state fp32
    [B, H, D, Ns]; s / the state are None when not wanted."""
    if k.dim() != 4 or q.shape != k.shape or v.dim() != 4 or w.shape != v.shape:
        raise ValueError("k, q must be [B, T, H, Ns] and v, w [B, T, H, D]")
    if not (k.dtype == q.dtype == v.dtype == w.dtype):
        raise TypeError("k, q, v, w must share one dtype")
    B, T, H, Ns = k.shape
    D = v.shape[3]
    if tuple(v.shape[:3]) != (B, T, H) or a.shape != (H, D, Ns) or p.shape != (H, D, Ns):
        raise ValueError("v, w must be [B, T, H, D] and a, p [H, D, Ns]")
    if lam0.shape != (B, H, D, Ns) or eta0.shape != (B, H, D, Ns):
        raise ValueError("lam0 and eta0 must be [B, H, D, Ns]")
    for t in (a, p, lam0, eta0):
        if t.dtype != torch.float32:
            raise TypeError("a, p, lam0, eta0 must be float32")
    _require_cuda(k, q, v, w, a, p, lam0, eta0)
    dev = k.device
    if out is None:
        outs = [torch.empty((B, T, H, D), dtype=torch.float32, device=dev),
                torch.empty((B, T, H, D), dtype=torch.float32, device=dev) if want_s else None,
                torch.empty((B, H, D, Ns), dtype=torch.float32, device=dev) if want_state else None,
                torch.empty((B, H, D, Ns), dtype=torch.float32, device=dev) if want_state else None]
    else:
        outs = list(out)
        _require_cuda(*outs)
    if workspace is None:
        n = layer_workspace_size(B, T, H, D, Ns, k.dtype)
        workspace = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    with torch.cuda.device(dev):
        st = lib().kla_layer_forward(
            _ptr(k), _ptr(q), _ptr(v), _ptr(w), _dtype_code(k), _ptr(a), _ptr(p), _ptr(lam0), _ptr(eta0),
            *[_ptr(o) for o in outs], B, T, H, D, Ns,
            _ptr(workspace), workspace.numel() if workspace is not None else 0, _stream_handle(stream))
    _check(st, "kla_layer_forward")
    return tuple(outs)


def layer_step(k: torch.Tensor, q: torch.Tensor, v: torch.Tensor, w: torch.Tensor,
               a: torch.Tensor, p: torch.Tensor, lam_state: torch.Tensor, eta_state: torch.Tensor, *,
               y: Optional[torch.Tensor] = None, s: Optional[torch.Tensor] = None, want_s: bool = True,
               stream: Optional[torch.cuda.Stream] = None):
    """One decode token of the fused layer (kla_layer_step): k, q [B, H, Ns];
    v, w [B, H, D]; a, p [H, D, Ns]; the state [B, H, D, Ns] is updated in
    place.  Returns (y, s), fp32 [B, H, D] (s None when not wanted)."""
    if k.dim() != 3 or q.shape != k.shape or v.dim() != 3 or w.shape != v.shape:
        raise ValueError("k, q must be [B, H, Ns] and v, w [B, H, D]")
    if not (k.dtype == q.dtype == v.dtype == w.dtype):
        raise TypeError("k, q, v, w must share one dtype")
    B, H, Ns = k.shape
    D = v.shape[2]
    if tuple(v.shape[:2]) != (B, H) or lam_state.shape != (B, H, D, Ns) or eta_state.shape != (B, H, D, Ns):
        raise ValueError("v, w must be [B, H, D] and the state [B, H, D, Ns]")
    _require_cuda(k, q, v, w, a, p, lam_state, eta_state, y, s)
    if y is None:
        y = torch.empty((B, H, D), dtype=torch.float32, device=k.device)
    if s is None and want_s:
        s = torch.empty((B, H, D), dtype=torch.float32, device=k.device)
    with torch.cuda.device(k.device):
        st = lib().kla_layer_step(_ptr(k), _ptr(q), _ptr(v), _ptr(w), _dtype_code(k), _ptr(a), _ptr(p),
                                  _ptr(lam_state), _ptr(eta_state), _ptr(y), _ptr(s), B, H, D, Ns,
                                  _stream_handle(stream))
    _check(st, "kla_layer_step")
    return y, s


def attention_weights(a: torch.Tensor, p: torch.Tensor, lam: torch.Tensor, *, t0: int = 0,
                      span: Optional[int] = None, W: int = ATTENTION_MAX_WINDOW,
                      out: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The Kalman attention weights F(t, s) = prod_{k=s+1..t} f_k of the
    windows of W tokens of [t0, t0 + span), from the forward inputs a, p and
    the forward scan's lambda ([B, T, H, N]).  Returns fp32
    [B, ceil(span / W), W, W, H, N] (kla_attention_weights)."""
    if a.dim() != 4 or p.shape != a.shape or lam.shape != a.shape:
        raise ValueError("a, p, lam must share one [B, T, H, N] shape")
    if p.dtype != a.dtype or lam.dtype != torch.float32:
        raise TypeError("a and p share one dtype; lam is float32")
    B, T, H, N = a.shape
    span = T - t0 if span is None else span
    nwin = -(-span // W) if W > 0 else 0
    _require_cuda(a, p, lam)
    if out is None:
        out = torch.empty((B, nwin, W, W, H, N), dtype=torch.float32, device=a.device)
    else:
        _require_cuda(out)
        if out.shape != (B, nwin, W, W, H, N) or out.dtype != torch.float32:
            raise ValueError("out must be float32 [B, nwin, W, W, H, N]")
    with torch.cuda.device(a.device):
        _check(lib().kla_attention_weights(_ptr(a), _ptr(p), _dtype_code(a), _ptr(lam), _ptr(out), B, T, H, N,
                                           t0, span, W, _stream_handle(stream)), "kla_attention_weights")
    return out


def lti_workspace_size(B: int, T: int, H: int, N: int, dtype: torch.dtype = torch.float32) -> int:
    code = KLA_BF16 if dtype == torch.bfloat16 else KLA_F32
    out = ctypes.c_size_t(0)
    _check(lib().kla_scan_forward_lti_workspace_size(B, T, H, N, code, ctypes.byref(out)),
           "kla_scan_forward_lti_workspace_size")
    return int(out.value)


def lti_plan(phi: torch.Tensor, b: torch.Tensor) -> Tuple[int, int]:
    """(kernel, launches) of scan_forward_lti: 1 = one thread per channel,
    2 = channel-owning streaming."""
    B, T, H, N = phi.shape
    k, n = ctypes.c_int(0), ctypes.c_int(0)
    with torch.cuda.device(phi.device):
        _check(lib().kla_scan_forward_lti_plan(B, T, H, N, _dtype_code(phi), _ptr(phi), _ptr(b), ctypes.byref(k),
                                               ctypes.byref(n)), "kla_scan_forward_lti_plan")
    return int(k.value), int(n.value)


def scan_forward_lti(a: torch.Tensor, phi: torch.Tensor, b: torch.Tensor, lam0: torch.Tensor,
                     eta0: torch.Tensor, *, want_mu: bool = True, want_var: bool = True,
                     out: Optional[Sequence[Optional[torch.Tensor]]] = None,
                     workspace: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None,
                     ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor], Optional[torch.Tensor]]:
    """The deterministic time-invariant filter (p = 0, decay a [B, H, N]
    constant in time) in its convolutional form (kla_scan_forward_lti):
    phi, b [B, T, H, N]; returns (lambda, eta, mu, var) as scan_forward does."""
    if phi.dim() != 4 or b.shape != phi.shape or b.dtype != phi.dtype:
        raise ValueError("phi, b must share one [B, T, H, N] shape and dtype")
    B, T, H, N = phi.shape
    for t, name in ((a, "a"), (lam0, "lam0"), (eta0, "eta0")):
        if t.shape != (B, H, N) or t.dtype != torch.float32:
            raise ValueError(f"{name} must be float32 [B, H, N]")
    _require_cuda(a, phi, b, lam0, eta0)
    dev = phi.device
    if out is None:
        outs = [torch.empty((B, T, H, N), dtype=torch.float32, device=dev),
                torch.empty((B, T, H, N), dtype=torch.float32, device=dev),
                torch.empty((B, T, H, N), dtype=torch.float32, device=dev) if want_mu else None,
                torch.empty((B, T, H, N), dtype=torch.float32, device=dev) if want_var else None]
    else:
        outs = list(out)
        _require_cuda(*[o for o in outs if o is not None])
    if workspace is None:
        workspace = torch.empty(max(lti_workspace_size(B, T, H, N, phi.dtype), 1), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = lib().kla_scan_forward_lti(_ptr(a), _ptr(phi), _ptr(b), _dtype_code(phi), _ptr(lam0), _ptr(eta0),
                                        _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), _ptr(outs[3]), B, T, H, N,
                                        _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(st, "kla_scan_forward_lti")
    return tuple(outs)
