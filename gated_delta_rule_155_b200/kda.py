"""ctypes binding of libkda.so — argument marshalling only.

Every function here has the name of the C entry point it calls (``include/kda.h``)
and takes torch tensors that live on the GPU; each one checks shapes, dtypes and
contiguity, passes raw device pointers and the current CUDA stream, and raises
:class:`KdaError` on a non-OK status.  All computation happens in the library's
CUDA kernels.  There is no fallback: if ``libkda.so`` is missing or fails to load,
importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")

KDA_OK = 0
KDA_F32, KDA_BF16 = 0, 1
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_MISALIGNED", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_TIMEOUT",
                6: "KDA_ERR_WORKSPACE"}


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.kda_status_string(status).decode() if _lib is not None else "?"
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg})")


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libkda.so not found at {_LIB_PATH}; build it with "
            "`python -m gated_delta_rule_155_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [i]
    lib.kda_abi_version.restype = i
    lib.kda_forward_chunked.restype = i
    lib.kda_forward_chunked.argtypes = [vp] * 8 + [i] * 6 + [i, vp]
    lib.kda_decode_step.restype = i
    lib.kda_decode_step.argtypes = [vp] * 7 + [i] * 4 + [i, vp]
    lib.kda_layer_forward_varlen.restype = i
    lib.kda_layer_forward_varlen.argtypes = [vp] * 9 + [f] + [vp] * 3 + [f] + [vp] * 5 + [sz] + [i] * 5 + [i, vp]
    lib.kda_backward_workspace_size.restype = i
    lib.kda_backward_workspace_size.argtypes = [i] * 6 + [ctypes.POINTER(sz)]
    lib.kda_backward_chunked.restype = i
    lib.kda_backward_chunked.argtypes = [vp] * 15 + [sz] + [i] * 5 + [i, vp]
    lib.kda_forward_chunked_varlen.restype = i
    lib.kda_forward_chunked_varlen.argtypes = [vp] * 9 + [i] * 6 + [i, vp]
    lib.kda_layer_workspace_size.restype = i
    lib.kda_layer_workspace_size.argtypes = [i] * 6 + [ctypes.POINTER(sz)]
    lib.kda_layer_forward.restype = i
    lib.kda_layer_forward.argtypes = [vp] * 9 + [f] + [vp] * 3 + [f] + [vp] * 4 + [sz] + [i] * 5 + [i, vp]
    lib.kda_layer_forward_noalloc.restype = i
    lib.kda_layer_forward_noalloc.argtypes = [vp] * 9 + [f] + [vp] * 3 + [f] + [vp] * 3 + [i] * 5 + [i, vp]
    lib.kda_check_device_error.restype = i
    lib.kda_layer_decode_step.argtypes = [vp] * 12 + [f] + [vp] * 3 + [f] + [vp] * 2 + [i] * 4 + [i, vp]
    lib.kda_layer_decode_step.restype = i
    lib.kda_check_device_error.argtypes = [vp]
    lib.kda_set_wait_test_hooks.restype = i
    lib.kda_set_wait_test_hooks.argtypes = [ctypes.c_ulonglong, i]
    return lib


_lib = _load()

EXPORTED_SYMBOLS = ("kda_status_string", "kda_abi_version", "kda_forward_chunked",
                    "kda_decode_step", "kda_layer_workspace_size", "kda_layer_forward",
                    "kda_layer_forward_noalloc", "kda_layer_decode_step", "kda_forward_chunked_varlen",
                    "kda_backward_workspace_size", "kda_backward_chunked", "kda_layer_forward_varlen",
                    "kda_check_device_error", "kda_set_wait_test_hooks")

NOALLOC_SCRATCH_BYTES = 64 << 20  # KDA_NOALLOC_SCRATCH_BYTES


def library():
    """The loaded ctypes library handle."""
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _io_code(dtype):
    if dtype == torch.float32:
        return KDA_F32
    if dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"unsupported io dtype {dtype}")


def _check(status, where):
    if status != KDA_OK:
        raise KdaError(status, where)


def _need(t, shape, dtype, name, *, allow_none=False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    # the library launches on the current device, so every tensor must live there
    cur = torch.cuda.current_device()
    if t.device.index is not None and t.device.index != cur:
        raise ValueError(f"{name} is on cuda:{t.device.index} but the current device is cuda:{cur}; "
                         f"call under torch.cuda.device({t.device.index})")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def kda_forward_chunked(q, k, v, g, beta, initial_state=None, out=None, final_state=None,
                        *, chunk=64, stream=None):
    """Chunked prefill.  q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H] (io dtype);
    initial_state / final_state: [B, H, dk, dv] fp32 or None.  Returns (out, final_state)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    io = q.dtype
    for t, s, n in ((q, (B, T, H, dk), "q"), (k, (B, T, H, dk), "k"), (g, (B, T, H, dk), "g"),
                    (v, (B, T, H, dv), "v"), (beta, (B, T, H), "beta")):
        _need(t, s, io, n)
    _need(initial_state, (B, H, dk, dv), torch.float32, "initial_state", allow_none=True)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=io, device=q.device)
    _need(out, (B, T, H, dv), io, "out")
    _need(final_state, (B, H, dk, dv), torch.float32, "final_state", allow_none=True)
    _check(_lib.kda_forward_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    _ptr(initial_state), _ptr(out), _ptr(final_state),
                                    B, T, H, dk, dv, chunk, _io_code(io), _stream(stream)),
           "kda_forward_chunked")
    return out, final_state


def kda_forward_chunked_varlen(q, k, v, g, beta, cu_seqlens, initial_state=None, out=None,
                               final_state=None, *, chunk=64, stream=None):
    """Chunked prefill of N packed sequences.  q, k, g: [T_total, H, dk]; v: [T_total, H, dv];
    beta: [T_total, H] (io dtype); cu_seqlens: int32 CUDA tensor [N + 1] of sequence offsets
    (0 .. T_total, non-decreasing); initial_state / final_state: [N, H, dk, dv] fp32 or None.
    Returns (out [T_total, H, dv], final_state)."""
    Tt, H, dk = q.shape
    dv = v.shape[-1]
    io = q.dtype
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D tensor of N + 1 >= 2 offsets")
    N = cu_seqlens.numel() - 1
    _need(cu_seqlens, (N + 1,), torch.int32, "cu_seqlens")
    for t, s, n in ((q, (Tt, H, dk), "q"), (k, (Tt, H, dk), "k"), (g, (Tt, H, dk), "g"),
                    (v, (Tt, H, dv), "v"), (beta, (Tt, H), "beta")):
        _need(t, s, io, n)
    _need(initial_state, (N, H, dk, dv), torch.float32, "initial_state", allow_none=True)
    if out is None:
        out = torch.empty((Tt, H, dv), dtype=io, device=q.device)
    _need(out, (Tt, H, dv), io, "out")
    _need(final_state, (N, H, dk, dv), torch.float32, "final_state", allow_none=True)
    _check(_lib.kda_forward_chunked_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                           _ptr(initial_state), _ptr(out), _ptr(final_state),
                                           _ptr(cu_seqlens), N, Tt, H, dk, dv, chunk, _io_code(io),
                                           _stream(stream)),
           "kda_forward_chunked_varlen")
    return out, final_state


def kda_backward_workspace_size(B, T, H, dk, dv, dtype):
    n = ctypes.c_size_t(0)
    _check(_lib.kda_backward_workspace_size(B, T, H, dk, dv, _io_code(dtype), ctypes.byref(n)),
           "kda_backward_workspace_size")
    return int(n.value)


def kda_backward_chunked(q, k, v, g, beta, d_out, initial_state=None, d_final_state=None, *,
                         grads=None, d_initial_state=None, workspace=None, stream=None):
    """Gradients of kda_forward_chunked.  Returns dict dq, dk, dv, dg, dbeta (io dtype) and
    d_initial_state (fp32 [B, H, dk, dv]).  ``grads`` may hold preallocated outputs;
    ``workspace`` (uint8 CUDA tensor) is allocated with torch when not given."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    io = q.dtype
    for t, s, n in ((q, (B, T, H, dk), "q"), (k, (B, T, H, dk), "k"), (g, (B, T, H, dk), "g"),
                    (v, (B, T, H, dv), "v"), (beta, (B, T, H), "beta"), (d_out, (B, T, H, dv), "d_out")):
        _need(t, s, io, n)
    _need(initial_state, (B, H, dk, dv), torch.float32, "initial_state", allow_none=True)
    _need(d_final_state, (B, H, dk, dv), torch.float32, "d_final_state", allow_none=True)
    gr = dict(grads or {})
    shapes = {"dq": (B, T, H, dk), "dk": (B, T, H, dk), "dg": (B, T, H, dk), "dv": (B, T, H, dv),
              "dbeta": (B, T, H)}
    for n, s in shapes.items():
        if gr.get(n) is None:
            gr[n] = torch.empty(s, dtype=io, device=q.device)
        _need(gr[n], s, io, n)
    if d_initial_state is None:
        d_initial_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(d_initial_state, (B, H, dk, dv), torch.float32, "d_initial_state")
    need = kda_backward_workspace_size(B, T, H, dk, dv, io)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kda_backward_chunked(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(d_out), _ptr(d_final_state),
        _ptr(gr["dq"]), _ptr(gr["dk"]), _ptr(gr["dv"]), _ptr(gr["dg"]), _ptr(gr["dbeta"]), _ptr(d_initial_state),
        _ptr(workspace), ws_bytes, B, T, H, dk, dv, _io_code(io), _stream(stream)), "kda_backward_chunked")
    gr["d_initial_state"] = d_initial_state
    return gr


def kda_decode_step(q, k, v, g, beta, state, out=None, *, stream=None):
    """One decode step; ``state`` [B, H, dk, dv] fp32 is updated in place.  Returns out [B, H, dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    io = q.dtype
    for t, s, n in ((q, (B, H, dk), "q"), (k, (B, H, dk), "k"), (g, (B, H, dk), "g"),
                    (v, (B, H, dv), "v"), (beta, (B, H), "beta")):
        _need(t, s, io, n)
    _need(state, (B, H, dk, dv), torch.float32, "state")
    if out is None:
        out = torch.empty((B, H, dv), dtype=io, device=q.device)
    _need(out, (B, H, dv), io, "out")
    _check(_lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                _ptr(out), B, H, dk, dv, _io_code(io), _stream(stream)),
           "kda_decode_step")
    return out


def _lb(bound):
    """The gate's lower bound as the C ABI takes it: -inf for none."""
    return float("-inf") if bound is None else float(bound)


def kda_layer_workspace_size(B, T, H, dk, dv, dtype):
    n = ctypes.c_size_t(0)
    _check(_lib.kda_layer_workspace_size(B, T, H, dk, dv, _io_code(dtype), ctypes.byref(n)),
           "kda_layer_workspace_size")
    return int(n.value)


def kda_layer_forward(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, b_raw,
                      o_gate_raw, o_norm_w=None, *, norm_eps=1e-6, initial_state=None, out=None,
                      final_state=None, workspace=None, gate_lower_bound=None, stream=None):
    """KDA layer core (prologue -> chunked gated delta rule -> epilogue).  Returns (out, final_state).
    ``workspace`` (a uint8 CUDA tensor) is allocated with torch when not given.
    ``gate_lower_bound`` (<= 0, e.g. -5.0) bounds every log-decay g from below; None: unbounded."""
    B, T, H, dk = g_raw.shape
    dv = o_gate_raw.shape[-1]
    io = g_raw.dtype
    f32 = torch.float32
    for t, s, d, n in ((q_raw, (B, T, H * dk), io, "q_raw"), (k_raw, (B, T, H * dk), io, "k_raw"),
                       (v_raw, (B, T, H * dv), io, "v_raw"), (b_raw, (B, T, H), io, "b_raw"),
                       (o_gate_raw, (B, T, H, dv), io, "o_gate_raw"),
                       (conv_q, (H * dk, 4), f32, "conv_q"), (conv_k, (H * dk, 4), f32, "conv_k"),
                       (conv_v, (H * dv, 4), f32, "conv_v"), (A_log, (H,), f32, "A_log")):
        _need(t, s, d, n)
    _need(dt_bias, (H * dk,), f32, "dt_bias", allow_none=True)
    _need(o_norm_w, (dv,), f32, "o_norm_w", allow_none=True)
    _need(initial_state, (B, H, dk, dv), f32, "initial_state", allow_none=True)
    _need(final_state, (B, H, dk, dv), f32, "final_state", allow_none=True)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=io, device=g_raw.device)
    _need(out, (B, T, H, dv), io, "out")
    need = kda_layer_workspace_size(B, T, H, dk, dv, io)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=g_raw.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kda_layer_forward(
        _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_q), _ptr(conv_k), _ptr(conv_v),
        _ptr(g_raw), _ptr(A_log), _ptr(dt_bias), _lb(gate_lower_bound), _ptr(b_raw), _ptr(o_gate_raw),
        _ptr(o_norm_w), float(norm_eps), _ptr(initial_state), _ptr(out), _ptr(final_state), _ptr(workspace),
        ws_bytes, B, T, H, dk, dv, _io_code(io), _stream(stream)), "kda_layer_forward")
    return out, final_state


def kda_layer_forward_varlen(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, b_raw,
                             o_gate_raw, cu_seqlens, o_norm_w=None, *, norm_eps=1e-6, initial_state=None,
                             out=None, final_state=None, workspace=None, gate_lower_bound=None, stream=None):
    """The layer core over N packed sequences.  q_raw, k_raw: [T_total, H*dk]; v_raw: [T_total, H*dv];
    g_raw: [T_total, H, dk]; b_raw: [T_total, H]; o_gate_raw: [T_total, H, dv]; cu_seqlens: int32 CUDA
    [N + 1]; states [N, H, dk, dv].  Returns (out [T_total, H, dv], final_state)."""
    Tt, H, dk = g_raw.shape
    dv = o_gate_raw.shape[-1]
    io = g_raw.dtype
    f32 = torch.float32
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D tensor of N + 1 >= 2 offsets")
    N = cu_seqlens.numel() - 1
    _need(cu_seqlens, (N + 1,), torch.int32, "cu_seqlens")
    for t, s, d, n in ((q_raw, (Tt, H * dk), io, "q_raw"), (k_raw, (Tt, H * dk), io, "k_raw"),
                       (v_raw, (Tt, H * dv), io, "v_raw"), (b_raw, (Tt, H), io, "b_raw"),
                       (o_gate_raw, (Tt, H, dv), io, "o_gate_raw"),
                       (conv_q, (H * dk, 4), f32, "conv_q"), (conv_k, (H * dk, 4), f32, "conv_k"),
                       (conv_v, (H * dv, 4), f32, "conv_v"), (A_log, (H,), f32, "A_log")):
        _need(t, s, d, n)
    _need(dt_bias, (H * dk,), f32, "dt_bias", allow_none=True)
    _need(o_norm_w, (dv,), f32, "o_norm_w", allow_none=True)
    _need(initial_state, (N, H, dk, dv), f32, "initial_state", allow_none=True)
    _need(final_state, (N, H, dk, dv), f32, "final_state", allow_none=True)
    if out is None:
        out = torch.empty((Tt, H, dv), dtype=io, device=g_raw.device)
    _need(out, (Tt, H, dv), io, "out")
    need = kda_layer_workspace_size(1, Tt, H, dk, dv, io)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=g_raw.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.kda_layer_forward_varlen(
        _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_q), _ptr(conv_k), _ptr(conv_v),
        _ptr(g_raw), _ptr(A_log), _ptr(dt_bias), _lb(gate_lower_bound), _ptr(b_raw), _ptr(o_gate_raw),
        _ptr(o_norm_w), float(norm_eps), _ptr(initial_state), _ptr(out), _ptr(final_state), _ptr(cu_seqlens),
        _ptr(workspace), ws_bytes, N, Tt, H, dk, dv, _io_code(io), _stream(stream)), "kda_layer_forward_varlen")
    return out, final_state


def kda_layer_decode_step(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, cache_q, cache_k, cache_v, g_raw,
                          A_log, dt_bias, b_raw, o_gate_raw, state, o_norm_w=None, *, norm_eps=1e-6,
                          out=None, gate_lower_bound=None, stream=None):
    """One decode step of the layer core.  ``cache_*`` [B, 3, H*d] (io dtype, oldest tap first)
    and ``state`` [B, H, dk, dv] fp32 are updated in place.  Returns out [B, H, dv]."""
    B, H, dk = g_raw.shape
    dv = o_gate_raw.shape[-1]
    io = g_raw.dtype
    f32 = torch.float32
    for t, s_, d, n in ((q_raw, (B, H * dk), io, "q_raw"), (k_raw, (B, H * dk), io, "k_raw"),
                        (v_raw, (B, H * dv), io, "v_raw"), (b_raw, (B, H), io, "b_raw"),
                        (o_gate_raw, (B, H, dv), io, "o_gate_raw"),
                        (cache_q, (B, 3, H * dk), io, "cache_q"), (cache_k, (B, 3, H * dk), io, "cache_k"),
                        (cache_v, (B, 3, H * dv), io, "cache_v"),
                        (conv_q, (H * dk, 4), f32, "conv_q"), (conv_k, (H * dk, 4), f32, "conv_k"),
                        (conv_v, (H * dv, 4), f32, "conv_v"), (A_log, (H,), f32, "A_log"),
                        (state, (B, H, dk, dv), f32, "state")):
        _need(t, s_, d, n)
    _need(dt_bias, (H * dk,), f32, "dt_bias", allow_none=True)
    _need(o_norm_w, (dv,), f32, "o_norm_w", allow_none=True)
    if out is None:
        out = torch.empty((B, H, dv), dtype=io, device=g_raw.device)
    _need(out, (B, H, dv), io, "out")
    _check(_lib.kda_layer_decode_step(
        _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_q), _ptr(conv_k), _ptr(conv_v),
        _ptr(cache_q), _ptr(cache_k), _ptr(cache_v), _ptr(g_raw), _ptr(A_log), _ptr(dt_bias),
        _lb(gate_lower_bound), _ptr(b_raw), _ptr(o_gate_raw), _ptr(o_norm_w), float(norm_eps), _ptr(state), _ptr(out),
        B, H, dk, dv, _io_code(io), _stream(stream)), "kda_layer_decode_step")
    return out


def kda_layer_forward_noalloc(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias,
                              b_raw, o_gate_raw, o_norm_w=None, *, norm_eps=1e-6, initial_state=None,
                              out=None, final_state=None, gate_lower_bound=None, stream=None):
    """kda_layer_forward with its scratch in the library's own fixed device buffer (no
    workspace argument, no allocation inside the call except ``out`` when it is not given —
    pass ``out`` to allocate nothing at all).  Sizes needing more than NOALLOC_SCRATCH_BYTES
    of scratch raise KdaError (KDA_ERR_WORKSPACE).  Returns (out, final_state)."""
    B, T, H, dk = g_raw.shape
    dv = o_gate_raw.shape[-1]
    io = g_raw.dtype
    f32 = torch.float32
    for t, s, d, n in ((q_raw, (B, T, H * dk), io, "q_raw"), (k_raw, (B, T, H * dk), io, "k_raw"),
                       (v_raw, (B, T, H * dv), io, "v_raw"), (b_raw, (B, T, H), io, "b_raw"),
                       (o_gate_raw, (B, T, H, dv), io, "o_gate_raw"),
                       (conv_q, (H * dk, 4), f32, "conv_q"), (conv_k, (H * dk, 4), f32, "conv_k"),
                       (conv_v, (H * dv, 4), f32, "conv_v"), (A_log, (H,), f32, "A_log")):
        _need(t, s, d, n)
    _need(dt_bias, (H * dk,), f32, "dt_bias", allow_none=True)
    _need(o_norm_w, (dv,), f32, "o_norm_w", allow_none=True)
    _need(initial_state, (B, H, dk, dv), f32, "initial_state", allow_none=True)
    _need(final_state, (B, H, dk, dv), f32, "final_state", allow_none=True)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=io, device=g_raw.device)
    _need(out, (B, T, H, dv), io, "out")
    _check(_lib.kda_layer_forward_noalloc(
        _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_q), _ptr(conv_k), _ptr(conv_v),
        _ptr(g_raw), _ptr(A_log), _ptr(dt_bias), _lb(gate_lower_bound), _ptr(b_raw), _ptr(o_gate_raw),
        _ptr(o_norm_w), float(norm_eps), _ptr(initial_state), _ptr(out), _ptr(final_state),
        B, T, H, dk, dv, _io_code(io), _stream(stream)), "kda_layer_forward_noalloc")
    return out, final_state


def kda_check_device_error(stream=None):
    """Synchronise the stream and raise if a kernel flagged a bounded-wait timeout or CUDA error."""
    _check(_lib.kda_check_device_error(_stream(stream)), "kda_check_device_error")


def kda_set_wait_test_hooks(wait_limit_ns=0, skip_load_chunk=-1):
    """Limit of the tensor-core kernels' bounded waits (0: the default 2 s) and an injected
    failure (the tile load of chunk `skip_load_chunk` is never issued; -1: off).  Process-wide."""
    _check(_lib.kda_set_wait_test_hooks(int(wait_limit_ns), int(skip_load_chunk)), "kda_set_wait_test_hooks")


# short names
forward_chunked = kda_forward_chunked
forward_chunked_varlen = kda_forward_chunked_varlen
backward_chunked = kda_backward_chunked
decode_step = kda_decode_step
layer_forward = kda_layer_forward
layer_workspace_size = kda_layer_workspace_size
check_device_error = kda_check_device_error
