"""The C-ABI library loads and exports every symbol of include/kla.h; host-side
argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kla_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from kalman_linear_attention_b200 import _build, api
    _build.build()
    return api.load_library()


def test_every_declared_symbol_is_exported(lib):
    from kalman_linear_attention_b200 import api
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(api.SIGNATURES), "binding and header disagree"


def test_abi_version(lib):
    src = open(os.path.join(ROOT, "include", "kla.h")).read()
    v = int(re.search(r"#define KLA_ABI_VERSION (\d+)", src).group(1))
    assert lib.kla_abi_version() == v


def test_strerror(lib):
    for code in range(8):
        assert lib.kla_strerror(code)
    assert b"unknown" in lib.kla_strerror(99)


def test_workspace_size(lib):
    out = ctypes.c_size_t(0)
    assert lib.kla_scan_forward_workspace_size(1, 65536, 32, 128, 0, ctypes.byref(out)) == 0
    L = lib.kla_forward_chunk_tokens()
    chunks = 65536 // L
    tiles = chunks * (4096 // 64)
    # carries: 7 + 2 floats per channel per chunk, plus flags and a header
    assert out.value >= tiles * 64 * 9 * 4
    assert out.value < 0.05 * (65536 * 4096 * 32)
    assert lib.kla_scan_forward_workspace_size(-1, 1, 1, 1, 0, ctypes.byref(out)) == 1
    assert lib.kla_scan_forward_workspace_size(1, 1, 1, 1, 7, ctypes.byref(out)) == 2
    assert lib.kla_scan_forward_workspace_size(1, 1, 1, 1, 0, None) == 1
    assert lib.kla_scan_forward_workspace_size(0, 100, 1, 1, 0, ctypes.byref(out)) == 0
    assert out.value == 0


def test_host_argument_errors(lib):
    """Rejected before any CUDA call: negative sizes, bad dtype, null pointers,
    overlapping outputs, small or misaligned workspace; empty problems are OK."""
    fwd = lib.kla_scan_forward
    P = 1 << 20  # fake, never dereferenced: every case returns before a launch
    args = lambda **kw: [kw.get("a", P), kw.get("p", 2 * P), kw.get("phi", 3 * P), kw.get("b", 4 * P),
                         kw.get("dt", 0), kw.get("lam0", 5 * P), kw.get("eta0", 6 * P),
                         kw.get("lam", 7 * P), kw.get("eta", 8 * P), kw.get("mu", None),
                         kw.get("var", None), kw.get("B", 1), kw.get("T", 4), kw.get("H", 1),
                         kw.get("N", 4), kw.get("ws", 16 * P), kw.get("wsb", 1 << 20), None]
    assert fwd(*args(B=-1)) == 1
    assert fwd(*args(dt=3)) == 2
    assert fwd(*args(a=None)) == 1
    assert fwd(*args(lam=None)) == 1
    assert fwd(*args(eta=7 * P)) == 1          # eta_out overlaps lambda_out
    assert fwd(*args(mu=P)) == 1               # mu_out overlaps input a
    assert fwd(*args(wsb=16)) == 3             # workspace too small
    assert fwd(*args(ws=None)) == 3
    assert fwd(*args(ws=16 * P + 8)) == 6      # misaligned workspace
    assert fwd(*args(T=0)) == 0                # empty: nothing enqueued
    assert fwd(*args(B=0, a=None)) == 0
    step = lib.kla_scan_step
    sargs = lambda **kw: [kw.get("a", P), kw.get("p", 2 * P), kw.get("phi", 3 * P), kw.get("b", 4 * P),
                          kw.get("dt", 0), kw.get("lam", 5 * P), kw.get("eta", 6 * P),
                          kw.get("mu", None), kw.get("var", None), kw.get("B", 1), kw.get("H", 1),
                          kw.get("N", 4), None]
    assert step(*sargs(N=-2)) == 1
    assert step(*sargs(dt=9)) == 2
    assert step(*sargs(lam=None)) == 1
    assert step(*sargs(eta=5 * P)) == 1
    assert step(*sargs(B=0)) == 0
    assert lib.kla_set_wait_limit_ns(0) == 1
    assert lib.kla_debug_stall_chunk(-5) == 1


def test_forward_plan_host_decision(lib):
    """The plan query answers on the host: empty problems launch nothing, and
    inputs the streaming kernel cannot take (unaligned, narrow, short) go to
    the chunked kernel (2 launches: workspace clear + scan)."""
    k, n = ctypes.c_int(-1), ctypes.c_int(-1)
    A = 1 << 20
    assert lib.kla_scan_forward_plan(1, 0, 32, 128, 0, A, A, A, A, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) == (0, 0)
    assert lib.kla_scan_forward_plan(1, 65536, 32, 128, 0, A + 4, A, A, A, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) == (1, 2)                      # unaligned input
    assert lib.kla_scan_forward_plan(1, 65536, 1, 7, 0, A, A, A, A, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) == (1, 2)                      # H*N = 7
    assert lib.kla_scan_forward_plan(1, 65536, 32, 128, 0, A, A, A, A, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) in ((1, 2), (2, 1))           # 2 needs a driver for TMA maps
    assert lib.kla_scan_forward_plan(-1, 1, 1, 1, 0, A, A, A, A, ctypes.byref(k), ctypes.byref(n)) == 1
    assert lib.kla_scan_forward_plan(1, 1, 1, 1, 5, A, A, A, A, ctypes.byref(k), ctypes.byref(n)) == 2


def test_host_workspace_size(lib):
    out = ctypes.c_size_t(0)
    assert lib.kla_scan_forward_host_workspace_size(1, 65536, 32, 128, 0, 0, ctypes.byref(out)) == 0
    # about 64 blocks: 2 slots x one block x (16 + 16 bytes per token-channel) + one scan workspace
    block = 1024 * 4096
    assert 2 * block * 32 <= out.value <= 2 * block * 32 * 1.1
    assert lib.kla_scan_forward_host_workspace_size(1, 0, 1, 1, 0, 0, ctypes.byref(out)) == 0 and out.value == 0
    assert lib.kla_scan_forward_host_workspace_size(1, 10, 1, 1, 0, -1, ctypes.byref(out)) == 1
    assert lib.kla_scan_forward_host_workspace_size(1, 10, 1, 1, 4, 0, ctypes.byref(out)) == 2


def test_backward_host_argument_errors(lib):
    """kla_scan_backward: the same host-side checks, before any CUDA call."""
    bwd = lib.kla_scan_backward
    P = 1 << 20  # fake, never dereferenced
    names = ["a", "p", "dt", "lam0", "eta0", "lam", "eta", "gl", "ge", "gm", "gv",
             "ga", "gp", "gphi", "gb", "glam0", "geta0", "B", "T", "H", "N", "ws", "wsb", "stream"]
    base = dict(a=P, p=2 * P, dt=0, lam0=3 * P, eta0=4 * P, lam=5 * P, eta=6 * P, gl=7 * P, ge=None,
                gm=8 * P, gv=None, ga=9 * P, gp=10 * P, gphi=11 * P, gb=12 * P, glam0=13 * P,
                geta0=14 * P, B=1, T=4, H=1, N=4, ws=16 * P, wsb=1 << 20, stream=None)
    args = lambda **kw: [kw.get(n, base[n]) for n in names]
    assert bwd(*args(H=-1)) == 1
    assert bwd(*args(dt=2)) == 2
    assert bwd(*args(a=None)) == 1
    assert bwd(*args(lam=None)) == 1
    assert bwd(*args(lam0=None)) == 1
    assert bwd(*args(gp=9 * P)) == 1              # grad_p overlaps grad_a
    assert bwd(*args(gb=5 * P)) == 1              # grad_b overlaps lambda_out
    assert bwd(*args(glam0=7 * P)) == 1           # prior gradient overlaps g_lambda
    assert bwd(*args(ga=16 * P)) == 1             # overlaps the workspace
    assert bwd(*args(wsb=16)) == 3
    assert bwd(*args(ws=None, wsb=0)) == 3
    assert bwd(*args(ws=16 * P + 8)) == 6
    assert bwd(*args(B=0, a=None, lam0=None)) == 0  # no channels: nothing enqueued
    out = ctypes.c_size_t(7)
    assert lib.kla_scan_backward_workspace_size(1, 0, 32, 128, 0, ctypes.byref(out)) == 0 and out.value == 0
    assert lib.kla_scan_backward_workspace_size(1, 65536, 32, 128, 1, ctypes.byref(out)) == 0
    # run-boundary carries: at most 3 boundaries x 64 floats per 32-channel tile, plus flags
    assert 128 * 3 * 64 * 4 <= out.value <= 128 * 3 * 64 * 4 + 128 * 3 * 4 + 4096
    assert lib.kla_scan_backward_workspace_size(1, 1, 1, 1, 3, ctypes.byref(out)) == 2
    k, n = ctypes.c_int(-1), ctypes.c_int(-1)
    assert lib.kla_scan_backward_plan(0, 5, 1, 1, 0, P, P, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) == (0, 0)
    assert lib.kla_scan_backward_plan(1, 64, 1, 7, 0, P, P, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) == (1, 1)                      # H*N = 7: one thread per channel
    assert lib.kla_scan_backward_plan(1, 64, 32, 128, 0, P + 4, P, ctypes.byref(k), ctypes.byref(n)) == 0
    assert k.value == 1                                       # unaligned input
    assert lib.kla_debug_force_backward_kernel(3) == 1


def test_layer_host_argument_errors(lib):
    """kla_layer_forward: shape, pointer, alignment and overlap checks answer on
    the host."""
    f = lib.kla_layer_forward
    P = 1 << 20  # fake, never dereferenced
    names = ["k", "q", "v", "w", "dt", "a", "p", "lam0", "eta0", "y", "s", "lamT", "etaT",
             "B", "T", "H", "D", "Ns", "ws", "wsb", "stream"]
    base = dict(k=P, q=2 * P, v=3 * P, w=4 * P, dt=0, a=5 * P, p=6 * P, lam0=7 * P, eta0=8 * P, y=9 * P,
                s=10 * P, lamT=11 * P, etaT=12 * P, B=1, T=64, H=2, D=4, Ns=16, ws=16 * P, wsb=1 << 20, stream=None)
    args = lambda **kw: [kw.get(n, base[n]) for n in names]
    assert f(*args(Ns=4)) == 1                  # unsupported state expansion
    assert f(*args(Ns=32)) == 1
    assert f(*args(D=3)) == 1                   # D not a multiple of 32 / Ns
    assert f(*args(dt=5)) == 2
    assert f(*args(k=None)) == 1
    assert f(*args(a=None)) == 1
    assert f(*args(lamT=None)) == 1             # final state: both or neither
    assert f(*args(k=P + 4)) == 1               # k not 16-byte aligned
    assert f(*args(y=P)) == 1                   # y overlaps k
    assert f(*args(s=9 * P)) == 1               # s overlaps y
    assert f(*args(wsb=16)) == 3
    assert f(*args(ws=16 * P + 8)) == 6
    assert f(*args(B=0)) == 0                   # no channels: nothing enqueued
    out = ctypes.c_size_t(7)
    assert lib.kla_layer_forward_workspace_size(8, 2048, 4, 32, 16, 1, ctypes.byref(out)) == 0
    assert out.value > 0
    assert lib.kla_layer_forward_workspace_size(8, 0, 4, 32, 16, 1, ctypes.byref(out)) == 0 and out.value == 0
    assert lib.kla_layer_forward_workspace_size(8, 16, 4, 30, 8, 1, ctypes.byref(out)) == 1


def test_layer_step_host_argument_errors(lib):
    f = lib.kla_layer_step
    P = 1 << 20
    names = ["k", "q", "v", "w", "dt", "a", "p", "lam", "eta", "y", "s", "B", "H", "D", "Ns", "stream"]
    base = dict(k=P, q=2 * P, v=3 * P, w=4 * P, dt=0, a=5 * P, p=6 * P, lam=7 * P, eta=8 * P, y=9 * P, s=None,
                B=2, H=2, D=4, Ns=16, stream=None)
    args = lambda **kw: [kw.get(n, base[n]) for n in names]
    assert f(*args(Ns=4)) == 1
    assert f(*args(D=5)) == 1
    assert f(*args(dt=3)) == 2
    assert f(*args(lam=None)) == 1
    assert f(*args(y=P)) == 1          # y overlaps k
    assert f(*args(eta=7 * P)) == 1    # state halves overlap
    assert f(*args(B=0)) == 0


def test_header_is_plain_c(lib, tmp_path):
    """include/kla.h compiles as strict C99 (a C caller can use the ABI) and
    its prototypes match the library's exports in a C program that takes the
    address of every function."""
    import subprocess
    names = declared_functions()
    src = tmp_path / "use.c"
    src.write_text('#include "kla.h"\ntypedef void (*any_fn)(void);\nint main(void) {\n    int n = 0;\n'
                   + "".join(f"    n += (any_fn){n} != (any_fn)0;\n" for n in names)
                   + f"    return n == {len(names)} && kla_abi_version() == KLA_ABI_VERSION ? 0 : 1;\n}}\n")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    # link a C program against the library and run it (no CUDA call is made)
    pkg = os.path.dirname(lib._name)
    exe = tmp_path / "use"
    r = subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", pkg, "-l:libkla.so", f"-Wl,-rpath,{pkg}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0


def test_size_overflow_is_rejected(lib):
    """Sizes whose products overflow int64 are argument errors, answered on
    the host for every entry point that takes a shape."""
    P = 1 << 20
    big = 1 << 40
    assert lib.kla_scan_forward(P, 2 * P, 3 * P, 4 * P, 0, 5 * P, 6 * P, 7 * P, 8 * P, None, None,
                                big, big, 1, 1, 16 * P, 1 << 20, None) == 1
    out = ctypes.c_size_t(0)
    assert lib.kla_scan_forward_workspace_size(big, big, 1, 1, 0, ctypes.byref(out)) == 1
    assert lib.kla_scan_backward_workspace_size(1, big, big, 1, 0, ctypes.byref(out)) == 1
    assert lib.kla_scan_backward(P, 2 * P, 0, 3 * P, 4 * P, 5 * P, 6 * P, None, None, None, None,
                                 7 * P, 8 * P, 9 * P, 10 * P, 11 * P, 12 * P, big, big, 1, 1,
                                 16 * P, 1 << 20, None) == 1
    assert lib.kla_scan_step(P, 2 * P, 3 * P, 4 * P, 0, 5 * P, 6 * P, None, None, big, big, 1, None) == 1
    assert lib.kla_layer_forward(P, 2 * P, 3 * P, 4 * P, 0, 5 * P, 6 * P, 7 * P, 8 * P, 9 * P, None, None, None,
                                 big, big, 1, 2, 16, 16 * P, 1 << 20, None) == 1
    assert lib.kla_layer_step(P, 2 * P, 3 * P, 4 * P, 0, 5 * P, 6 * P, 7 * P, 8 * P, 9 * P, None,
                              big, big, 2, 16, None) == 1


def test_attention_and_lti_host_argument_errors(lib):
    """The attention weights and the convolutional form reject bad arguments
    on the host, before any CUDA call; empty problems are valid."""
    P = 1 << 20  # fake pointers, never dereferenced
    att = lib.kla_attention_weights
    aargs = lambda **kw: [kw.get("a", P), kw.get("p", 2 * P), kw.get("dt", 0), kw.get("lam", 3 * P),
                          kw.get("F", 8 * P), kw.get("B", 1), kw.get("T", 100), kw.get("H", 1), kw.get("N", 4),
                          kw.get("t0", 0), kw.get("span", 100), kw.get("W", 16), None]
    assert att(*aargs(W=0)) == 1
    assert att(*aargs(W=65)) == 1                  # above KLA_ATTENTION_MAX_WINDOW
    assert att(*aargs(t0=-1)) == 1
    assert att(*aargs(t0=50, span=51)) == 1        # past the end of the sequence
    assert att(*aargs(dt=4)) == 2
    assert att(*aargs(lam=None)) == 1
    assert att(*aargs(F=2 * P)) == 1               # F overlaps p
    assert att(*aargs(span=0)) == 0                # empty
    assert att(*aargs(B=0, a=None)) == 0
    lti = lib.kla_scan_forward_lti
    largs = lambda **kw: [kw.get("a", P), kw.get("phi", 2 * P), kw.get("b", 3 * P), kw.get("dt", 0),
                          kw.get("lam0", 4 * P), kw.get("eta0", 5 * P), kw.get("lam", 6 * P),
                          kw.get("eta", 7 * P), kw.get("mu", None), kw.get("var", None), kw.get("B", 1),
                          kw.get("T", 4), kw.get("H", 1), kw.get("N", 4), kw.get("ws", 16 * P),
                          kw.get("wsb", 1 << 20), None]
    assert lti(*largs(B=-1)) == 1
    assert lti(*largs(dt=2)) == 2
    assert lti(*largs(a=None)) == 1
    assert lti(*largs(eta=6 * P)) == 1             # eta_out overlaps lambda_out
    assert lti(*largs(ws=2 * P)) == 1              # workspace overlaps phi
    assert lti(*largs(ws=16 * P + 8)) == 6
    assert lti(*largs(T=0)) == 0
    out = ctypes.c_size_t(0)
    assert lib.kla_scan_forward_lti_workspace_size(1, 65536, 32, 128, 0, ctypes.byref(out)) == 0
    assert 0 < out.value < (1 << 20)               # run-boundary states only
    assert lib.kla_scan_forward_lti_workspace_size(0, 1, 1, 1, 0, ctypes.byref(out)) == 0 and out.value == 0
    k, n = ctypes.c_int(-1), ctypes.c_int(-1)
    assert lib.kla_scan_forward_lti_plan(1, 65536, 1, 7, 0, P, P, ctypes.byref(k), ctypes.byref(n)) == 0
    assert (k.value, n.value) == (1, 1)            # H*N = 7: one thread per channel
