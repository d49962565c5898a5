"""Host-side tests of the C ABI (no GPU needed).

The library must load and export every entry point ``include/kda.h`` declares, and
every argument error must be reported before anything is launched — so these
calls are safe without a GPU: they pass invalid arguments (null, misaligned or
unsupported), which the library rejects on the host.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_155_b200 import build

    build.build()
    from gated_delta_rule_155_b200 import kda

    return kda.library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("kda_forward_chunked", "kda_decode_step", "kda_layer_forward", "kda_status_string",
              "kda_layer_workspace_size", "kda_check_device_error", "kda_abi_version"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), f"libkda.so does not export {s}"
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (kda_[a-z0-9_]+)\b", out))
    assert set(declared_symbols()) <= exported


def test_status_strings(lib):
    for code in range(7):
        s = lib.kda_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.kda_status_string(99) == b"unknown status"
    assert lib.kda_abi_version() == 103


P = ctypes.c_void_p
A16 = P(0x100000)  # aligned fake address: never dereferenced (every call below fails validation)
MIS = P(0x100008)


def _chunked(lib, q=A16, k=A16, v=A16, g=A16, beta=A16, s0=None, out=A16, sT=None,
             B=1, T=8, H=1, dk=64, dv=64, chunk=64, io=0):
    return lib.kda_forward_chunked(q, k, v, g, beta, s0, out, sT, B, T, H, dk, dv, chunk, io, None)


def test_forward_chunked_rejects_bad_arguments(lib):
    assert _chunked(lib, q=None) == 1
    assert _chunked(lib, out=None) == 1
    assert _chunked(lib, B=0) == 1
    assert _chunked(lib, H=-1) == 1
    assert _chunked(lib, T=-1) == 1
    assert _chunked(lib, io=7) == 1
    assert _chunked(lib, chunk=32) == 2
    assert _chunked(lib, dk=96) == 2
    assert _chunked(lib, dv=256) == 2
    assert _chunked(lib, g=MIS) == 3
    assert _chunked(lib, s0=MIS) == 3
    assert _chunked(lib, sT=MIS) == 3
    assert _chunked(lib, B=1 << 20, T=1 << 20) == 2
    # beta of the tensor-core shape must be aligned like every other tensor
    assert _chunked(lib, beta=P(0x100002), dk=128, dv=128, io=1) == 3


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="needs a machine without an sm_100 GPU")
def test_tensor_core_shape_has_no_slower_substitute(lib):
    """bf16 at dk = dv = 128 runs on the tcgen05 kernel only: where that kernel cannot run (here:
    no B200), the call is refused before any launch instead of running another kernel."""
    assert _chunked(lib, dk=128, dv=128, io=1) == 2
    assert lib.kda_forward_chunked_varlen(A16, A16, A16, A16, A16, None, A16, None, A16, 2, 100, 2, 128, 128,
                                          64, 1, None) == 2
    # the layer core's bf16 d = 128 kernel likewise
    assert lib.kda_layer_forward(A16, A16, A16, A16, A16, A16, A16, A16, None, ctypes.c_float(-5.0), A16, A16,
                                 None, ctypes.c_float(1e-6), None, A16, None, None, 0, 1, 40, 2, 128, 128, 1,
                                 None) == 2


def test_forward_chunked_varlen_rejects_bad_arguments(lib):
    def call(cu=A16, q=A16, N=3, Tt=100, chunk=64, dk=128, s0=None, io=1):
        return lib.kda_forward_chunked_varlen(q, A16, A16, A16, A16, s0, A16, None, cu, N, Tt, 2, dk, 128,
                                              chunk, io, None)
    assert call(cu=None) == 1           # offsets are required
    assert call(q=None) == 1
    assert call(N=0) == 1
    assert call(Tt=-1) == 1
    assert call(io=5) == 1
    assert call(chunk=16) == 2
    assert call(dk=32) == 2
    assert call(cu=MIS) == 3
    assert call(s0=MIS) == 3


def test_backward_rejects_bad_arguments(lib):
    n = ctypes.c_size_t(0)
    assert lib.kda_backward_workspace_size(2, 33, 3, 128, 128, 1, ctypes.byref(n)) == 0
    # three 16-token chunks per head, each: the state, U and X, and three 16 x 16 matrices
    assert n.value == 2 * 3 * 3 * (128 * 128 + 2 * 16 * 128 + 3 * 16 * 16) * 4
    assert lib.kda_backward_workspace_size(2, 33, 3, 128, 64, 1, ctypes.byref(n)) == 2

    def call(q=A16, ws=A16, ws_bytes=1 << 40, dk=128, dv=128, T=33, dgp=A16):
        return lib.kda_backward_chunked(q, A16, A16, A16, A16, None, A16, None, A16, A16, A16, dgp, A16, None,
                                        ws, ws_bytes, 2, T, 3, dk, dv, 1, None)
    assert call(q=None) == 1
    assert call(dgp=None) == 1
    assert call(T=-1) == 1
    assert call(dk=128, dv=64) == 2
    assert call(q=MIS) == 3
    assert call(ws=None) == 6
    assert call(ws_bytes=1024) == 6
    assert call(ws=P(0x100010)) == 3


def test_decode_rejects_bad_arguments(lib):
    args = [A16] * 7
    ok = lambda **kw: lib.kda_decode_step(*[kw.get(n, a) for n, a in zip("qkvgbso", args)],
                                          kw.get("B", 2), kw.get("H", 3), kw.get("dk", 128),
                                          kw.get("dv", 128), kw.get("io", 1), None)
    assert ok(s=None) == 1
    assert ok(o=None) == 1
    assert ok(B=0) == 1
    assert ok(dk=32) == 2
    assert ok(v=MIS) == 3


def test_layer_decode_rejects_bad_arguments(lib):
    names = ["qr", "kr", "vr", "cq", "ck", "cv", "xq", "xk", "xv", "g", "al", "dt", "b", "z", "w"]

    def step(eps=1e-6, lb=-5.0, **kw):
        ptrs = [kw.get(n, None if n in ("dt", "w") else A16) for n in names]
        ptrs.insert(12, ctypes.c_float(lb))
        return lib.kda_layer_decode_step(*ptrs, ctypes.c_float(eps), kw.get("S", A16), kw.get("o", A16),
                                         kw.get("B", 2), kw.get("H", 3), kw.get("dk", 128), kw.get("dv", 128),
                                         kw.get("io", 1), None)
    assert step(S=None) == 1
    assert step(xk=None) == 1
    assert step(eps=-1.0) == 1
    assert step(lb=0.5) == 1            # a bound above 0 would let the state grow
    assert step(lb=float("nan")) == 1
    assert step(H=0) == 1
    assert step(dk=64, dv=64) == 2      # d = 128 only
    assert step(xv=MIS) == 3
    assert step(dt=MIS) == 3


def test_layer_workspace_and_argument_checks(lib):
    n = ctypes.c_size_t(0)
    # fp32 I/O runs prologue -> fp32 chunk kernel -> epilogue through a workspace
    assert lib.kda_layer_workspace_size(2, 16, 3, 128, 128, 0, ctypes.byref(n)) == 0
    N = 2 * 16 * 3
    assert n.value >= 4 * N * (3 * 128 + 128 + 1 + 128)
    # bf16 at d = 128 is one tensor-core kernel and needs none
    assert lib.kda_layer_workspace_size(2, 16, 3, 128, 128, 1, ctypes.byref(n)) == 0 and n.value == 0
    assert lib.kda_layer_workspace_size(2, 0, 3, 128, 128, 0, ctypes.byref(n)) == 0 and n.value == 0
    assert lib.kda_layer_workspace_size(2, 16, 3, 128, 128, 1, None) == 1
    assert lib.kda_layer_workspace_size(2, 16, 3, 100, 128, 1, ctypes.byref(n)) == 2

    def layer(ws=A16, ws_bytes=1 << 40, q=A16, eps=1e-6, lb=float("-inf"), io=0, **kw):
        return lib.kda_layer_forward(q, A16, A16, A16, A16, A16, A16, A16, None, ctypes.c_float(lb),
                                     A16, A16, None,
                                     ctypes.c_float(eps), None, A16, None, ws, ws_bytes,
                                     kw.get("B", 1), kw.get("T", 16), kw.get("H", 2), 128, 128, io, None)
    assert layer(q=None) == 1
    assert layer(eps=-1.0) == 1
    assert layer(lb=1.0) == 1
    assert layer(lb=float("nan")) == 1
    assert layer(q=MIS) == 3
    assert layer(ws=None) == 6
    assert layer(ws_bytes=16) == 6
    assert layer(ws=P(0x100010)) == 3  # workspace must be 256-byte aligned


def test_layer_varlen_rejects_bad_arguments(lib):
    def call(cu=A16, q=A16, N=3, Tt=100, eps=1e-6):
        return lib.kda_layer_forward_varlen(q, A16, A16, A16, A16, A16, A16, A16, None, ctypes.c_float(-5.0),
                                            A16, A16, None, ctypes.c_float(eps), None, A16, None, cu, A16, 1 << 40,
                                            N, Tt, 2, 128, 128, 1, None)
    assert call(cu=None) == 1
    assert call(q=None) == 1
    assert call(N=0) == 1
    assert call(eps=-1.0) == 1
    assert call(cu=MIS) == 3


def header_prototypes():
    """{name: number of parameters} of every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"\b(kda_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        protos[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_declares_every_prototype_with_its_arity(lib):
    """Each C entry point's ctypes declaration has as many arguments as its prototype in
    include/kda.h, so a signature change cannot leave the binding behind."""
    protos = header_prototypes()
    assert len(protos) >= 13
    for name, n in protos.items():
        fn = getattr(lib, name)
        if n == 0:
            assert not fn.argtypes, f"{name} takes no arguments"
            continue
        assert fn.argtypes is not None, f"{name} has no argtypes in the binding"
        assert len(fn.argtypes) == n, f"{name}: header has {n} parameters, binding {len(fn.argtypes)}"


def test_binding_rejects_tensors_off_the_current_device(monkeypatch):
    """Kernels launch on the current device, so a tensor on another GPU is an error, caught
    before any pointer reaches the library."""
    import types

    import torch

    from gated_delta_rule_155_b200 import kda

    fake = types.SimpleNamespace(is_cuda=True, device=types.SimpleNamespace(index=1), shape=(2, 3),
                                 dtype=torch.float32, is_contiguous=lambda: True)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current device is cuda:0"):
        kda._need(fake, (2, 3), torch.float32, "q")
    fake.device.index = 0
    kda._need(fake, (2, 3), torch.float32, "q")        # same device: accepted


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding raises at import when libkda.so is missing — there is no fallback."""
    import importlib.util
    import shutil
    src = os.path.join(ROOT, "gated_delta_rule_155_b200", "kda.py")
    dst = tmp_path / "kda.py"
    shutil.copy(src, dst)
    spec = importlib.util.spec_from_file_location("kda_nolib", dst)
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="no CPU fallback"):
        spec.loader.exec_module(mod)
