"""fp64 CPU oracle for the KDA gated delta rule — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg
of ``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything under ``oracle/``,
and this package imports nothing from the product.

The arithmetic lives in ``kda_oracle.c`` (plain C, double precision, token by
token, OpenMP over independent heads); this module only builds it with gcc and
marshals numpy arrays.  ``chunked.py`` holds the chunkwise rewrite that exists
solely to pin the recurrence (its self-check), never to compute expected values
for the GPU.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def declare(lib):
    """Set the argument types of every oracle entry point on a loaded copy of the C library
    (the built one, or a test's deliberately mutated build of the same source)."""
    i = ctypes.c_int
    d = ctypes.c_double
    sz = ctypes.c_size_t
    lib.kda_oracle_recurrent.argtypes = [_dp] * 8 + [i] * 7
    lib.kda_oracle_recurrent_backward.argtypes = [_dp] * 14 + [i] * 6
    lib.kda_oracle_decode.argtypes = [_dp] * 7 + [i] * 5
    lib.kda_oracle_short_conv_silu.argtypes = [_dp] * 3 + [i] * 5
    lib.kda_oracle_l2norm.argtypes = [_dp, _dp, sz, i, d]
    lib.kda_oracle_gate.argtypes = [_dp] * 3 + [d, _dp] + [i] * 4
    lib.kda_oracle_sigmoid.argtypes = [_dp, _dp, sz]
    lib.kda_oracle_out_norm_gate.argtypes = [_dp, _dp, _dp, d, i, _dp, sz, i]
    lib.kda_oracle_layer.argtypes = [_dp] * 9 + [d] + [_dp] * 3 + [d, d, i, _dp, _dp, _dp] + [i] * 6
    lib.kda_oracle_max_threads.restype = i
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = declare(ctypes.CDLL(build()))
    return _lib


def _f64(a):
    """Contiguous float64 copy/view of ``a`` (None passes through)."""
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def recurrent(q, k, v, g, beta, s0=None, *, delta=True, nthreads=0):
    """Token-by-token gated delta rule.

    q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; s0: [B, H, dk, dv] or None.
    Returns (o [B, T, H, dv], S_T [B, H, dk, dv]) in float64.
    ``delta=False`` removes the correction term (test-only variant: plain gated
    linear attention with write strength beta).
    """
    q, k, v, g, beta, s0 = map(_f64, (q, k, v, g, beta, s0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and g.shape == q.shape and v.shape == (B, T, H, dv)
    assert beta.shape == (B, T, H)
    assert s0 is None or s0.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    _load().kda_oracle_recurrent(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0), _ptr(o), _ptr(sT),
        B, T, H, dk, dv, 1 if delta else 0, nthreads,
    )
    return o, sT


def recurrent_backward(q, k, v, g, beta, s0, d_o, d_sT=None, *, nthreads=0):
    """Gradients of the recurrence by reverse mode, token by token, in fp64.

    Arguments as ``recurrent`` plus d_o = dL/do [B, T, H, dv] and d_sT = dL/dS_T
    [B, H, dk, dv] (None: zero).  Returns dict dq, dk, dv, dg, dbeta, ds0.
    """
    q, k, v, g, beta, s0, d_o, d_sT = map(_f64, (q, k, v, g, beta, s0, d_o, d_sT))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert d_o.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    assert d_sT is None or d_sT.shape == (B, H, dk, dv)
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v), "dg": np.zeros_like(g),
           "dbeta": np.zeros_like(beta), "ds0": np.zeros((B, H, dk, dv))}
    _load().kda_oracle_recurrent_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0), _ptr(d_o), _ptr(d_sT),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
        _ptr(out["ds0"]), B, T, H, dk, dv, nthreads,
    )
    return out


def recurrent_varlen(q, k, v, g, beta, cu_seqlens, s0=None, *, nthreads=0):
    """N packed sequences of different lengths, each through the token-by-token recurrence
    from its own initial state (no state crosses a sequence boundary).

    q, k, g: [T_total, H, dk]; v: [T_total, H, dv]; beta: [T_total, H]; cu_seqlens: N + 1
    offsets (sequence n is tokens cu[n] .. cu[n+1]-1); s0: [N, H, dk, dv] or None.
    Returns (o [T_total, H, dv], S_T [N, H, dk, dv]); o is zero at tokens no sequence covers.
    """
    q, k, v, g, beta, s0 = map(_f64, (q, k, v, g, beta, s0))
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    N = len(cu) - 1
    Tt, H, dk = q.shape
    dv = v.shape[-1]
    assert N >= 1 and cu[0] >= 0 and cu[-1] <= Tt and all(a <= b for a, b in zip(cu, cu[1:]))
    assert s0 is None or s0.shape == (N, H, dk, dv)
    o = np.zeros((Tt, H, dv))
    sT = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        s_n = None if s0 is None else s0[n:n + 1]
        if b == a:
            sT[n] = 0.0 if s_n is None else s_n[0]
            continue
        on, sn = recurrent(q[None, a:b], k[None, a:b], v[None, a:b], g[None, a:b], beta[None, a:b],
                           s_n, nthreads=nthreads)
        o[a:b] = on[0]
        sT[n] = sn[0]
    return o, sT


def layer_varlen(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, b_raw,
                 o_gate_raw, cu_seqlens, o_norm_w=None, *, s0=None, **kw):
    """The layer core over N packed sequences, each run by ``layer`` on its own tokens (so the
    conv history and the state start fresh at every sequence).  Token-major inputs
    ([T_total, H*dk], [T_total, H, dk], ...); s0 [N, H, dk, dv] or None.
    Returns (out [T_total, H, dv], S_T [N, H, dk, dv])."""
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    N = len(cu) - 1
    Tt, H, dk = np.shape(g_raw)
    dv = np.shape(o_gate_raw)[-1]
    out = np.zeros((Tt, H, dv))
    sT = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        s_n = None if s0 is None else _f64(s0)[n:n + 1]
        if b == a:
            sT[n] = 0.0 if s_n is None else s_n[0]
            continue
        o, st = layer(*(_f64(x)[None, a:b] for x in (q_raw, k_raw, v_raw)), conv_q, conv_k, conv_v,
                      _f64(g_raw)[None, a:b], A_log, dt_bias, _f64(b_raw)[None, a:b], _f64(o_gate_raw)[None, a:b],
                      o_norm_w, s0=s_n, **kw)
        out[a:b] = o[0]
        sT[n] = st[0]
    return out, sT


def decode(q, k, v, g, beta, state, *, nthreads=0):
    """One decode step.  q, k, g: [B, H, dk]; v: [B, H, dv]; beta: [B, H];
    state: [B, H, dk, dv].  Returns (o [B, H, dv], new_state) — the input is not modified."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    st = np.array(state, dtype=np.float64, order="C", copy=True)
    B, H, dk = q.shape
    dv = v.shape[-1]
    assert st.shape == (B, H, dk, dv)
    o = np.zeros((B, H, dv))
    _load().kda_oracle_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(st), _ptr(o), B, H, dk, dv, nthreads
    )
    return o, st


def short_conv(x, w, *, silu=True, nthreads=0):
    """Depthwise causal conv (kernel 4, zero history) [+ SiLU].  x: [B, T, C]; w: [C, 4]."""
    x, w = _f64(x), _f64(w)
    B, T, C = x.shape
    assert w.shape == (C, 4)
    y = np.zeros_like(x)
    _load().kda_oracle_short_conv_silu(_ptr(x), _ptr(w), _ptr(y), B, T, C, 1 if silu else 0, nthreads)
    return y


def l2norm(x, eps=1e-6):
    """x / sqrt(sum(x^2) + eps) over the last dim."""
    x = _f64(x)
    y = np.zeros_like(x)
    d = x.shape[-1]
    _load().kda_oracle_l2norm(_ptr(x), _ptr(y), x.size // d, d, float(eps))
    return y


def gate(x, A_log, dt_bias=None, *, lower_bound=None):
    """g = max(-exp(A_log[h]) * softplus(x + dt_bias[h, c]), lower_bound).

    x: [B, T, H, dk]; A_log: [H]; lower_bound None means no bound (the Kimi-K3
    linear-attention config's gate_lower_bound, read as a bound on the log-decay).
    """
    x, A_log, dt_bias = _f64(x), _f64(A_log), _f64(dt_bias)
    B, T, H, dk = x.shape
    assert A_log.shape == (H,)
    assert dt_bias is None or dt_bias.size == H * dk
    g = np.zeros_like(x)
    lb = float("-inf") if lower_bound is None else float(lower_bound)
    _load().kda_oracle_gate(_ptr(x), _ptr(A_log), _ptr(dt_bias), lb, _ptr(g), B, T, H, dk)
    return g


def sigmoid(x):
    x = _f64(x)
    y = np.zeros_like(x)
    _load().kda_oracle_sigmoid(_ptr(x), _ptr(y), x.size)
    return y


def out_norm_gate(o, z, gain=None, eps=1e-6, io_bf16=False):
    """Per-row RMSNorm (cast to the io dtype, times gain) times sigmoid(z).  o, z: [..., dv]."""
    o, z, gain = _f64(o), _f64(z), _f64(gain)
    dv = o.shape[-1]
    assert z.shape == o.shape and (gain is None or gain.shape == (dv,))
    out = np.zeros_like(o)
    _load().kda_oracle_out_norm_gate(
        _ptr(o), _ptr(z), _ptr(gain), float(eps), 1 if io_bf16 else 0, _ptr(out), o.size // dv, dv
    )
    return out


def layer(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, b_raw,
          o_gate_raw, o_norm_w=None, *, norm_eps=1e-6, l2_eps=1e-6, io_bf16=True,
          s0=None, gate_lower_bound=None, nthreads=0):
    """The KDA layer core: conv+SiLU, q/k L2-norm, gate, beta, recurrence, RMSNorm x sigmoid gate.

    q_raw, k_raw: [B, T, H*dk]; v_raw: [B, T, H*dv]; g_raw: [B, T, H, dk]; b_raw: [B, T, H];
    o_gate_raw: [B, T, H, dv]; gate_lower_bound None = unbounded gate.
    Returns (out [B, T, H, dv], S_T [B, H, dk, dv]).
    """
    arrs = [q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, b_raw,
            o_gate_raw, o_norm_w, s0]
    (q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, b_raw, o_gate_raw,
     o_norm_w, s0) = map(_f64, arrs)
    B, T, H, dk = g_raw.shape
    dv = o_gate_raw.shape[-1]
    assert q_raw.shape == (B, T, H * dk) and k_raw.shape == (B, T, H * dk)
    assert v_raw.shape == (B, T, H * dv) and b_raw.shape == (B, T, H)
    assert conv_q.shape == (H * dk, 4) and conv_k.shape == (H * dk, 4)
    assert conv_v.shape == (H * dv, 4)
    out = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    _load().kda_oracle_layer(
        _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_q), _ptr(conv_k), _ptr(conv_v),
        _ptr(g_raw), _ptr(A_log), _ptr(dt_bias),
        float("-inf") if gate_lower_bound is None else float(gate_lower_bound),
        _ptr(b_raw), _ptr(o_gate_raw), _ptr(o_norm_w),
        float(norm_eps), float(l2_eps), 1 if io_bf16 else 0, _ptr(s0), _ptr(out), _ptr(sT),
        B, T, H, dk, dv, nthreads,
    )
    return out, sT
