"""Seeded synthetic inputs for the KDA hot path — shared by the tests and the benchmark.

This module only draws random numbers and shapes them into the distributions the
workloads state; it contains none of the path's arithmetic (no recurrence, no
prologue, no epilogue).  Both the CUDA path and the CPU oracle consume exactly
the tensors produced here, already rounded to the I/O dtype (round-to-nearest-even
via ``torch.Tensor.to``), so parity measures kernel error only.

Distributions (per workload):
  * A_log[h] ~ U(0, ln 8) per head (exp(A_log) in [1, 8]).
  * q, k ~ N(0, 1), then unit-normalised over dk for each (token, head).
  * v ~ N(0, 1).
  * log-decay g = -exp(A_log[h]) * softplus(x), x ~ N(0, 1): the workloads state the
    recurrence's decay input by this law, so it is drawn here as an input
    distribution.  (The layer path computes its own gate from raw inputs
    inside the kernel and inside the oracle, independently.)
  * beta = sigmoid(x), x ~ N(0, 1) — likewise the stated law of the beta input.
  * initial state ~ N(0, std^2) in fp32 where a workload has one, else zeros.
  * layer: raw q/k/v ~ N(0, 1) on [B, T, H*d]; conv weights ~ N(0, 0.5^2) (0.5 read as
    the standard deviation); raw gate/beta inputs ~ N(0, 1); output-gate input ~ N(0, 1).

Random draws are made block by block from counter-keyed streams
``SeedSequence([seed, tensor_id, block])`` so that the values do not depend on
how many threads generate them.  Tensor ids follow the fixed draw order
A_log, q, k, v, g, b, S0, conv weights, o_gate.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

_BLOCK = 1 << 22
_TID = {"A_log": 0, "q": 1, "k": 2, "v": 3, "g": 4, "b": 5, "s0": 6,
        "conv_q": 7, "conv_k": 8, "conv_v": 9, "o_gate": 10}
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(16, max(1, (torch.get_num_threads() or 4))))
    return _POOL


def _draw(seed: int, name: str, n: int, kind: str, step: int = 0) -> np.ndarray:
    """n float32 draws of `kind` ('normal' or 'uniform01') from the stream of (seed, tensor, step)."""
    out = np.empty(n, dtype=np.float32)
    tid = _TID[name] + 100 * step
    nblk = (n + _BLOCK - 1) // _BLOCK

    def fill(blk):
        lo, hi = blk * _BLOCK, min(n, (blk + 1) * _BLOCK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, blk])))
        if kind == "normal":
            out[lo:hi] = rng.standard_normal(hi - lo, dtype=np.float32)
        else:
            out[lo:hi] = rng.random(hi - lo, dtype=np.float32)

    if nblk <= 1:
        for b in range(nblk):
            fill(b)
    else:
        list(_pool().map(fill, range(nblk)))
    return out


def _normal(seed, name, shape, std=1.0, step=0):
    a = _draw(seed, name, int(np.prod(shape)), "normal", step).reshape(shape)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _unit_rows(a: np.ndarray) -> np.ndarray:
    """Scale each last-dim row of `a` to unit Euclidean norm (input shaping, in place)."""
    n = np.sqrt(np.einsum("...c,...c->...", a, a, dtype=np.float32))
    a /= np.maximum(n, np.float32(1e-30))[..., None]
    return a


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(np.float32(0.0), x)


def _to_io(a: np.ndarray, io: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(torch.bfloat16) if io == "bf16" else t.to(torch.float32)


def a_log(seed: int, H: int) -> np.ndarray:
    """Per-head A_log ~ U(0, ln 8), fp32."""
    return (_draw(seed, "A_log", H, "uniform01") * np.float32(math.log(8.0))).astype(np.float32)


def prefill_inputs(B, T, H, dk, dv, *, io="bf16", seed=0, s0_std=0.0, step=0):
    """Inputs of the chunked prefill: dict with q, k, v, g, beta (io dtype, torch CPU),
    s0 (fp32 [B, H, dk, dv] or None) and A_log (fp32 [H], for the record)."""
    A = a_log(seed, H)
    q = _to_io(_unit_rows(_normal(seed, "q", (B, T, H, dk), step=step)), io)
    k = _to_io(_unit_rows(_normal(seed, "k", (B, T, H, dk), step=step)), io)
    v = _to_io(_normal(seed, "v", (B, T, H, dv), step=step), io)
    x = _normal(seed, "g", (B, T, H, dk), step=step)
    g = _softplus(x)
    g *= -np.exp(A)[None, None, :, None]
    g = _to_io(g, io)
    del x
    xb = _normal(seed, "b", (B, T, H), step=step)
    beta = _to_io((1.0 / (1.0 + np.exp(-xb))).astype(np.float32), io)
    s0 = None
    if s0_std > 0.0:
        s0 = torch.from_numpy(_normal(seed, "s0", (B, H, dk, dv), std=s0_std))
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta, "s0": s0, "A_log": A}


def decode_inputs(B, H, dk, dv, *, steps=1, io="bf16", seed=3, s0_std=0.02):
    """Decode workload: fp32 state [B, H, dk, dv] ~ N(0, s0_std^2) and `steps` fresh
    single-token input sets (q, k, g: [B, H, dk]; v: [B, H, dv]; beta: [B, H])."""
    A = a_log(seed, H)
    state = torch.from_numpy(_normal(seed, "s0", (B, H, dk, dv), std=s0_std))
    per_step = []
    for s in range(steps):
        d = prefill_inputs(B, 1, H, dk, dv, io=io, seed=seed, step=s + 1)
        per_step.append({n: d[n].reshape(B, H, -1) if n != "beta" else d[n].reshape(B, H)
                         for n in ("q", "k", "v", "g", "beta")})
    # every step shares the workload's per-head A_log law; record the first draw
    return {"state": state, "steps": per_step, "A_log": A}


def layer_inputs(B, T, H, dk, dv, *, io="bf16", seed=4, conv_std=0.5, s0_std=0.0,
                 dt_bias_std=0.0, gain_std=0.0):
    """Raw inputs of the KDA layer core.

    q_raw, k_raw: [B, T, H*dk]; v_raw: [B, T, H*dv]; g_raw: [B, T, H, dk]; b_raw: [B, T, H];
    o_gate_raw: [B, T, H, dv] (io dtype); conv_q/k/v: [H*d, 4] fp32; A_log: [H] fp32;
    dt_bias: [H*dk] fp32 or None; o_norm_w: [dv] fp32 or None (unit gain); s0 or None.
    """
    A = a_log(seed, H)
    q_raw = _to_io(_normal(seed, "q", (B, T, H * dk)), io)
    k_raw = _to_io(_normal(seed, "k", (B, T, H * dk)), io)
    v_raw = _to_io(_normal(seed, "v", (B, T, H * dv)), io)
    g_raw = _to_io(_normal(seed, "g", (B, T, H, dk)), io)
    b_raw = _to_io(_normal(seed, "b", (B, T, H)), io)
    s0 = None
    if s0_std > 0.0:
        s0 = torch.from_numpy(_normal(seed, "s0", (B, H, dk, dv), std=s0_std))
    conv_q = torch.from_numpy(_normal(seed, "conv_q", (H * dk, 4), std=conv_std))
    conv_k = torch.from_numpy(_normal(seed, "conv_k", (H * dk, 4), std=conv_std))
    conv_v = torch.from_numpy(_normal(seed, "conv_v", (H * dv, 4), std=conv_std))
    o_gate = _to_io(_normal(seed, "o_gate", (B, T, H, dv)), io)
    dt_bias = None
    if dt_bias_std > 0.0:
        dt_bias = torch.from_numpy(_normal(seed, "o_gate", (H * dk,), std=dt_bias_std, step=7))
    gain = None
    if gain_std > 0.0:
        gain = torch.from_numpy(1.0 + _normal(seed, "o_gate", (dv,), std=gain_std, step=8))
    return {"q_raw": q_raw, "k_raw": k_raw, "v_raw": v_raw, "conv_q": conv_q, "conv_k": conv_k,
            "conv_v": conv_v, "g_raw": g_raw, "A_log": torch.from_numpy(A), "dt_bias": dt_bias,
            "b_raw": b_raw, "o_gate_raw": o_gate, "o_norm_w": gain, "s0": s0}


def packed_lengths(total: int, max_len: int, seed: int) -> list:
    """Sequence lengths for a packed batch of `total` tokens: uniform draws in [1, max_len]
    until the sum reaches `total`, the last one trimmed to fit."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x5E9]))
    lens = []
    while sum(lens) < total:
        lens.append(int(min(rng.integers(1, max_len + 1), total - sum(lens))))
    return lens


def varlen_inputs(lengths, H, dk, dv, *, io="bf16", seed=5, s0_std=0.0):
    """Packed variable-length prefill: the prefill laws over sum(lengths) tokens, laid out
    [T_total, H, d] (beta [T_total, H]); cu_seqlens int32 [N + 1]; s0 [N, H, dk, dv] or None."""
    Tt, N = int(sum(lengths)), len(lengths)
    d = prefill_inputs(1, Tt, H, dk, dv, io=io, seed=seed)
    out = {n: d[n][0] for n in ("q", "k", "v", "g", "beta")}
    out["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    out["s0"] = torch.from_numpy(_normal(seed, "s0", (N, H, dk, dv), std=s0_std)) if s0_std > 0 else None
    out["A_log"] = d["A_log"]
    return out


# The workloads, by what they are.
WORKLOADS = {
    "recurrence_f32_B1_T256_H2_d64": dict(kind="prefill", io="f32", B=1, T=256, H=2, dk=64, dv=64,
                                           s0_std=0.0, seed=0),
    "prefill_bf16_B1_T4096_H32_d128": dict(kind="prefill", io="bf16", B=1, T=4096, H=32, dk=128,
                                            dv=128, s0_std=0.02, seed=1),
    "prefill_bf16_B4_T8192_H96_d128": dict(kind="prefill", io="bf16", B=4, T=8192, H=96, dk=128,
                                            dv=128, s0_std=0.0, seed=2),
    "decode_bf16_B256_H96_d128_x20": dict(kind="decode", io="bf16", B=256, H=96, dk=128, dv=128,
                                          steps=20, s0_std=0.02, seed=3),
    "layer_bf16_B2_T16384_H96_d128": dict(kind="layer", io="bf16", B=2, T=16384, H=96, dk=128,
                                          dv=128, conv_std=0.5, seed=4),
    # the headline prefill's 32768 tokens per step, packed as sequences of 1..4096 tokens
    "varlen_bf16_T32768_H96_d128": dict(kind="varlen", io="bf16", total=32768, max_len=4096, H=96,
                                        dk=128, dv=128, s0_std=0.0, seed=5),
}
