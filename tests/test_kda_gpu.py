"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances (written here, applied to the output o and, separately, to the final state):
  * fp32 I/O:  max|gpu - ref| / max|ref|  <= 1e-4
  * bf16 I/O (fp32 state), the 2e-2 bound relative to the RMS of the reference:
      final state (stored in fp32):   max|gpu - ref| <= 2e-2 rms(ref)
      outputs (stored in bf16):       |gpu - ref| <= 2e-2 rms(ref) + 2^-8 |ref|  elementwise
    The 2^-8 |ref| term is the bf16 output format's own rounding (round-to-nearest
    of the exact result is within half an ulp, at most 2^-8 relative): with outputs
    whose max/RMS ratio is ~17, rounding the exact fp64 result to bf16 alone gives
    max|err| = 0.039 rms, so no bf16-output kernel could meet 2e-2 rms without it.
Inputs come from the seeded generators in ``gated_delta_rule_155_b200.inputs``; the
oracle reads the same values the GPU reads (already rounded to the I/O dtype).
Large workloads are checked on sampled heads — heads are independent, so the
oracle computes those heads exactly — at the full sizes and launch shape the
benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_155_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_155_b200 import build

    build.build()
    from gated_delta_rule_155_b200 import kda as k

    return k


def f64(t):
    return t.detach().double().cpu().numpy()


BF16_FORMAT_REL = 2.0 ** -8


def err(gpu, ref, io, stored_bf16=None):
    """Error as a fraction of the allowed bound (passes when <= 1).  `stored_bf16` is the
    number of bf16 roundings the GPU value went through (True = 1: outputs under bf16 I/O;
    2: the layer output, whose RMSNorm casts to the activation dtype before the gain and
    gate and the result is stored in bf16 again; 0 / False: the fp32 final state).  Each
    rounding of a value that differs from the oracle's by any amount may land one bf16 step
    (2^-8 relative) apart."""
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    if gpu.size == 0:
        return 0.0
    d = np.abs(gpu - ref)
    if io == torch.float32:
        return np.max(d) / max(np.max(np.abs(ref)), 1e-30) / TOL_F32
    if stored_bf16 is None:
        stored_bf16 = True
    bound = TOL_BF16 * max(np.sqrt(np.mean(ref * ref)), 1e-30)
    if stored_bf16:
        bound = bound + int(stored_bf16) * BF16_FORMAT_REL * np.abs(ref)
    return float(np.max(d / bound))


def serr(gpu, ref, io):
    """Error of a final state (fp32 storage) as a fraction of its bound: max|gpu - ref| <=
    2e-2 rms(ref) under bf16 I/O, with no rounding term (the state is never stored in bf16)."""
    return err(gpu, ref, io, stored_bf16=0)


def tol(io):
    return 1.0


def run_prefill(kda, d, with_final=True):
    dev = "cuda"
    q, k, v, g, beta = (d[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    s0 = None if d["s0"] is None else d["s0"].to(dev)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    sT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if with_final else None
    out, sT = kda.kda_forward_chunked(q, k, v, g, beta, s0, None, sT)
    kda.kda_check_device_error()
    return out, sT


def oracle_prefill(d, heads=None):
    """Oracle on all heads, or on a list of (b, h) heads gathered into one [1, T, n, .] batch."""
    q, k, v, g, beta = (f64(d[n]) for n in ("q", "k", "v", "g", "beta"))
    s0 = None if d["s0"] is None else f64(d["s0"])
    if heads is None:
        return oracle.recurrent(q, k, v, g, beta, s0)
    bs = [b for b, _ in heads]
    hs = [h for _, h in heads]
    sel = lambda a: np.ascontiguousarray(a[bs, :, hs].transpose(1, 0, *range(2, a.ndim - 1))[None])
    s0s = None if s0 is None else np.ascontiguousarray(s0[bs, hs][None])
    return oracle.recurrent(sel(q), sel(k), sel(v), sel(g),
                            np.ascontiguousarray(beta[bs, :, hs].T[None]), s0s)


def check_heads(out, sT, ref_o, ref_s, heads, io, roundings=1):
    o_gpu = np.stack([f64(out[b, :, h]) for b, h in heads], axis=1)[None]
    s_gpu = np.stack([f64(sT[b, h]) for b, h in heads], axis=0)[None]
    eo, es = err(o_gpu, ref_o, io, stored_bf16=roundings), serr(s_gpu, ref_s, io)
    assert eo <= 1.0, f"output error {eo:.3e} of bound"
    assert es <= 1.0, f"state error {es:.3e} of bound"
    return eo, es


# ------------------------------------------------------------------------ the workloads


def test_recurrence_f32_workload(kda):
    """fp32, B=1, T=256, H=2, dk=dv=64: every output and the final state."""
    w = inputs.WORKLOADS["recurrence_f32_B1_T256_H2_d64"]
    d = inputs.prefill_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"])
    out, sT = run_prefill(kda, d)
    ro, rs = oracle_prefill(d)
    assert err(f64(out), ro, torch.float32) <= 1.0
    assert serr(f64(sT), rs, torch.float32) <= 1.0


def test_prefill_bf16_B1_T4096_H32(kda):
    """bf16, nonzero fp32 initial state: every head."""
    w = inputs.WORKLOADS["prefill_bf16_B1_T4096_H32_d128"]
    d = inputs.prefill_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"],
                              s0_std=w["s0_std"])
    out, sT = run_prefill(kda, d)
    ro, rs = oracle_prefill(d)
    assert err(f64(out), ro, torch.bfloat16) <= 1.0
    assert serr(f64(sT), rs, torch.bfloat16) <= 1.0


def test_prefill_bf16_B4_T8192_H96_sampled_heads(kda):
    """Full-size H=96 prefill in the benchmark's launch shape; six heads checked exactly."""
    w = inputs.WORKLOADS["prefill_bf16_B4_T8192_H96_d128"]
    d = inputs.prefill_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"])
    out, sT = run_prefill(kda, d)
    heads = [(0, 0), (1, 17), (2, 48), (3, 95), (0, 71), (3, 5)]
    ro, rs = oracle_prefill(d, heads)
    check_heads(out, sT, ro, rs, heads, torch.bfloat16)
    assert torch.isfinite(out.float()).all() and torch.isfinite(sT).all()


# ------------------------------------------------------------------------ shapes and tails


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 130])
def test_prefill_shapes_and_ragged_tails(kda, io, dk, dv, T):
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(2, T, 3, dk, dv, io=ioname, seed=1000 + T + dk + dv // 2,
                              s0_std=0.05)
    out, sT = run_prefill(kda, d)
    ro, rs = oracle_prefill(d)
    assert err(f64(out), ro, io) <= tol(io)
    assert serr(f64(sT), rs, io) <= 1.0


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_prefill_zero_length_copies_state(kda, io):
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(2, 0, 3, 128, 128, io=ioname, seed=5, s0_std=0.1)
    out, sT = run_prefill(kda, d)
    assert out.numel() == 0
    torch.testing.assert_close(sT.cpu(), d["s0"], rtol=0, atol=0)
    d["s0"] = None
    _, sT = run_prefill(kda, d)
    assert torch.count_nonzero(sT) == 0


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_prefill_without_initial_or_final_state(kda, io):
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(1, 100, 2, 128, 128, io=ioname, seed=6)
    out, sT = run_prefill(kda, d, with_final=False)
    assert sT is None
    ro, _ = oracle_prefill(d)
    assert err(f64(out), ro, io) <= tol(io)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_state_passing_in_place_across_calls(kda, io):
    """Two calls over [0, 100) and [100, 230) with the state updated in place equal one call."""
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(2, 230, 3, 128, 128, io=ioname, seed=7, s0_std=0.05)
    dev = "cuda"
    S = d["s0"].clone().to(dev)
    outs = []
    for a, b in ((0, 100), (100, 230)):
        part = [d[n][:, a:b].contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")]
        o, _ = kda.kda_forward_chunked(*part, S, None, S)
        outs.append(o)
    kda.kda_check_device_error()
    ro, rs = oracle_prefill(d)
    assert err(f64(torch.cat(outs, 1)), ro, io) <= tol(io)
    assert serr(f64(S), rs, io) <= 1.0


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gval", [-40.0, -9.0, -1e-4])
def test_extreme_gates(kda, io, gval):
    """Very strong (-40 per step: every block's decay below e^-168, the exact diagonal
    path on every channel), strong (-9: the fp32 kernel's exact path, not the tensor-core
    kernel's) and very weak (-1e-4 per step) decay on every channel."""
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(1, 200, 2, 128, 128, io=ioname, seed=8, s0_std=0.05)
    d["g"] = torch.full_like(d["g"], gval)
    out, sT = run_prefill(kda, d)
    ro, rs = oracle_prefill(d)
    assert err(f64(out), ro, io) <= 1.0
    assert serr(f64(sT), rs, io) <= 1.0


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("bval", [0.0, 1.0])
def test_beta_extremes(kda, io, bval):
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(1, 150, 2, 128, 128, io=ioname, seed=9, s0_std=0.05)
    d["beta"] = torch.full_like(d["beta"], bval)
    out, sT = run_prefill(kda, d)
    ro, rs = oracle_prefill(d)
    assert err(f64(out), ro, io) <= 1.0
    assert serr(f64(sT), rs, io) <= 1.0


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_prefill_is_deterministic(kda, io):
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(2, 300, 4, 128, 128, io=ioname, seed=10, s0_std=0.02)
    o1, s1 = run_prefill(kda, d)
    o2, s2 = run_prefill(kda, d)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


# ------------------------------------------------------------------------ failure path


@pytest.mark.parametrize("skip_chunk,packed", [(0, False), (1, False), (2, True)])
def test_a_wait_that_runs_out_reports_timeout_and_the_next_call_is_green(kda, skip_chunk, packed):
    """A tile load that is never issued (injected through kda_set_wait_test_hooks): the
    tensor-core kernel's bounded wait for it runs out after 1 ms, the CTAs drain what they
    issued and return, kda_check_device_error reports KDA_ERR_TIMEOUT once, and a normal
    call right after it on the same context matches the oracle."""
    d = inputs.prefill_inputs(2, 200, 3, 128, 128, io="bf16", seed=40 + skip_chunk, s0_std=0.05)
    dv = d if not packed else inputs.varlen_inputs([200, 170, 130], 3, 128, 128, io="bf16", seed=41,
                                                   s0_std=0.05)
    run = (lambda: run_varlen(kda, dv)) if packed else (lambda: run_prefill(kda, d))
    kda.kda_set_wait_test_hooks(1_000_000, skip_chunk)
    try:
        with pytest.raises(kda.KdaError) as e:
            run()
        assert e.value.status == 5            # KDA_ERR_TIMEOUT
    finally:
        kda.kda_set_wait_test_hooks(0, -1)
    kda.kda_check_device_error()              # the word was cleared by the report
    out, sT = run()
    ro, rs = oracle_varlen(dv) if packed else oracle_prefill(d)
    assert err(f64(out), ro, torch.bfloat16) <= 1.0
    assert serr(f64(sT), rs, torch.bfloat16) <= 1.0


# ------------------------------------------------------------------------ decode


def _decode_steps(kda, dd, io_t, steps):
    dev = "cuda"
    S = dd["state"].clone().to(dev)
    outs = []
    for s in range(steps):
        st = dd["steps"][s]
        outs.append(kda.kda_decode_step(*(st[n].to(dev) for n in ("q", "k", "v", "g", "beta")), S))
    kda.kda_check_device_error()
    return outs, S


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_decode_small(kda, io, dk, dv):
    ioname = "f32" if io == torch.float32 else "bf16"
    dd = inputs.decode_inputs(3, 5, dk, dv, steps=4, io=ioname, seed=20 + dk + dv)
    outs, S = _decode_steps(kda, dd, io, 4)
    st = f64(dd["state"])
    for s in range(4):
        x = dd["steps"][s]
        ro, st = oracle.decode(*(f64(x[n]) for n in ("q", "k", "v", "g", "beta")), st)
        assert err(f64(outs[s]), ro, io) <= tol(io)
    assert serr(f64(S), st, io) <= 1.0


def test_decode_workload_B256_H96_20_steps_sampled_heads(kda):
    """The full decode workload (state [256, 96, 128, 128] fp32, 20 chained steps in place);
    the outputs of every step and the final state are checked on 48 sampled heads."""
    w = inputs.WORKLOADS["decode_bf16_B256_H96_d128_x20"]
    dd = inputs.decode_inputs(w["B"], w["H"], w["dk"], w["dv"], steps=w["steps"], io=w["io"],
                              seed=w["seed"], s0_std=w["s0_std"])
    rng = np.random.default_rng(0)
    bs = rng.integers(0, w["B"], 48)
    hs = rng.integers(0, w["H"], 48)
    st = f64(dd["state"][bs, hs])[None]                     # [1, 48, dk, dv]
    outs, S = _decode_steps(kda, dd, torch.bfloat16, w["steps"])
    for s in range(w["steps"]):
        x = dd["steps"][s]
        args = [f64(x[n][bs, hs])[None] for n in ("q", "k", "v", "g", "beta")]
        ro, st = oracle.decode(*args, st)
        assert err(f64(outs[s][bs, hs])[None], ro, torch.bfloat16) <= 1.0
    assert serr(f64(S[bs, hs])[None], st, torch.bfloat16) <= 1.0


def test_decode_chain_equals_prefill(kda):
    """20 decode steps equal one prefill over the same 20 tokens (T = 1 prefill == decode)."""
    d = inputs.prefill_inputs(2, 20, 3, 128, 128, io="f32", seed=30, s0_std=0.05)
    dev = "cuda"
    o_p, s_p = run_prefill(kda, d)
    S = d["s0"].clone().to(dev)
    for t in range(20):
        o = kda.kda_decode_step(*(d[n][:, t].contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")), S)
        torch.testing.assert_close(o, o_p[:, t], rtol=1e-4, atol=1e-5)
    torch.testing.assert_close(S, s_p, rtol=1e-4, atol=1e-5)


# ------------------------------------------------------------------------ packed variable length


def run_varlen(kda, d, with_final=True):
    dev = "cuda"
    q, k, v, g, beta = (d[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    cu = d["cu_seqlens"].to(dev)
    s0 = None if d["s0"] is None else d["s0"].to(dev)
    N, H, dk, dv = cu.numel() - 1, q.shape[1], q.shape[2], v.shape[2]
    sT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev) if with_final else None
    out, sT = kda.kda_forward_chunked_varlen(q, k, v, g, beta, cu, s0, None, sT)
    kda.kda_check_device_error()
    return out, sT


def oracle_varlen(d):
    return oracle.recurrent_varlen(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]),
                                   d["cu_seqlens"].numpy(), None if d["s0"] is None else f64(d["s0"]))


# lengths: empty first and middle sequences, 1 token, one short of / exactly / one past a
# chunk, several chunks with a ragged tail, and a ragged last sequence
VARLEN_LENS = [0, 1, 63, 64, 65, 0, 130, 7, 200]


@pytest.mark.parametrize("io,d_", [(torch.bfloat16, 128), (torch.float32, 128),
                                   (torch.bfloat16, 64), (torch.float32, 64)])
def test_varlen_ragged_lengths(kda, io, d_):
    """Every token's output and every sequence's final state against the oracle run per
    sequence (tcgen05 kernel for bf16 d = 128, exact fp32 kernels otherwise)."""
    d = inputs.varlen_inputs(VARLEN_LENS, 3, d_, d_, io="f32" if io == torch.float32 else "bf16",
                             seed=80 + d_, s0_std=0.05)
    out, sT = run_varlen(kda, d)
    ro, rs = oracle_varlen(d)
    assert err(f64(out), ro, io) <= tol(io)
    assert serr(f64(sT), rs, io) <= 1.0
    # zero-length sequences pass the initial state through exactly
    for n in (0, 5):
        assert torch.equal(sT[n].cpu(), d["s0"][n])


@pytest.mark.parametrize("io,d_", [(torch.bfloat16, 128), (torch.float32, 128), (torch.bfloat16, 64)])
def test_varlen_equal_lengths_equal_the_fixed_length_call(kda, io, d_):
    """Three packed sequences of 150 tokens give the batched B = 3, T = 150 call's results bit
    for bit (same kernel; the packed tail chunk's foreign rows are masked)."""
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.varlen_inputs([150, 150, 150], 2, d_, d_, io=ioname, seed=90, s0_std=0.05)
    ov, sv = run_varlen(kda, d)
    fixed = {n: d[n].reshape((3, 150) + tuple(d[n].shape[1:])) for n in ("q", "k", "v", "g", "beta")}
    fixed["s0"] = d["s0"]
    of, sf = run_prefill(kda, fixed)
    assert torch.equal(ov.reshape(of.shape), of)
    assert torch.equal(sv, sf)


def test_varlen_many_short_sequences(kda):
    """200 packed sequences of 0..20 tokens (every chunk is a sequence's last, so every output
    goes through the tail-chunk stores) on the tcgen05 path."""
    lens = [int(x) for x in np.random.default_rng(91).integers(0, 21, 200)]
    d = inputs.varlen_inputs(lens, 2, 128, 128, io="bf16", seed=92, s0_std=0.05)
    out, sT = run_varlen(kda, d)
    ro, rs = oracle_varlen(d)
    assert err(f64(out), ro, torch.bfloat16) <= 1.0
    assert serr(f64(sT), rs, torch.bfloat16) <= 1.0


def test_prefill_and_backward_replay_in_a_cuda_graph(kda):
    """The tcgen05 prefill and the backward captured in one CUDA graph (as a serving or
    training loop would launch them) and replayed give the eager results bit for bit."""
    dev = "cuda"
    d = inputs.prefill_inputs(1, 150, 2, 128, 128, io="bf16", seed=93, s0_std=0.05)
    x = [d[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
    s0 = d["s0"].to(dev)
    dO = grad_inputs(d, 94)[0].to(dev)
    B, T, H, D = x[0].shape
    ws = torch.empty(kda.kda_backward_workspace_size(B, T, H, D, D, torch.bfloat16), dtype=torch.uint8, device=dev)
    out_e, sT_e = kda.kda_forward_chunked(*x, s0, None, torch.empty_like(s0))
    gr_e = kda.kda_backward_chunked(*x, dO, s0, None, workspace=ws)
    torch.cuda.synchronize()
    out_g = torch.empty_like(out_e)
    sT_g = torch.empty_like(sT_e)
    grads = {n: torch.empty_like(gr_e[n]) for n in ("dq", "dk", "dv", "dg", "dbeta")}
    ds0 = torch.empty_like(gr_e["d_initial_state"])
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            kda.kda_forward_chunked(*x, s0, out_g, sT_g)
            kda.kda_backward_chunked(*x, dO, s0, None, grads=grads, d_initial_state=ds0, workspace=ws)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    kda.kda_check_device_error()
    assert torch.equal(out_g, out_e) and torch.equal(sT_g, sT_e)
    for n in grads:
        assert torch.equal(grads[n], gr_e[n]), n
    assert torch.equal(ds0, gr_e["d_initial_state"])


def test_varlen_workload_T32768_H96_sampled(kda):
    """The packed workload (32768 tokens of 15 sequences, 1..4096 tokens each, H = 96) in the
    benchmark's launch shape; sampled (sequence, head) pairs against the oracle."""
    w = inputs.WORKLOADS["varlen_bf16_T32768_H96_d128"]
    lens = inputs.packed_lengths(w["total"], w["max_len"], w["seed"])
    d = inputs.varlen_inputs(lens, w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"])
    out, sT = run_varlen(kda, d)
    cu = d["cu_seqlens"].numpy()
    longest = int(np.argmax(lens))
    for n, h in [(0, 0), (longest, 95), (len(lens) - 1, 17), (len(lens) // 2, 50)]:
        a, b = int(cu[n]), int(cu[n + 1])
        ro, rs = oracle.recurrent(*(f64(d[x][a:b, h:h + 1])[None] for x in ("q", "k", "v", "g", "beta")))
        assert err(f64(out[a:b, h:h + 1])[None], ro, torch.bfloat16) <= 1.0
        assert serr(f64(sT[n, h])[None, None], rs, torch.bfloat16) <= 1.0


# ------------------------------------------------------------------------ backward


def grad_inputs(d, seed, dsT_std=0.0):
    """Upstream gradients: dO ~ N(0, 1) in the io dtype; dS_T ~ N(0, dsT_std^2) fp32 or None."""
    gen = torch.Generator().manual_seed(seed)
    dO = torch.randn(d["v"].shape, generator=gen).to(d["v"].dtype)
    dsT = None
    if dsT_std > 0:
        B, T, H, dk = d["q"].shape
        dsT = torch.randn((B, H, dk, d["v"].shape[-1]), generator=gen) * dsT_std
    return dO, dsT


def run_backward(kda, d, dO, dsT):
    dev = "cuda"
    to = lambda x: None if x is None else x.to(dev)
    gr = kda.kda_backward_chunked(to(d["q"]), to(d["k"]), to(d["v"]), to(d["g"]), to(d["beta"]), to(dO),
                                  to(d["s0"]), to(dsT))
    kda.kda_check_device_error()
    return gr


def check_grads(gr, ref, io, index=None):
    sel = (lambda x: x) if index is None else index
    for name, key in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dg", "dg"), ("dbeta", "dbeta")):
        e = err(sel(f64(gr[name])), sel(ref[key]), io, stored_bf16=io == torch.bfloat16)
        assert e <= 1.0, f"{name}: {e:.3e} of bound"


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_", [64, 128])
@pytest.mark.parametrize("T", [1, 17, 64, 100])
def test_backward_small(kda, io, d_, T):
    """All gradients (q, k, v, g, beta, S_0) against the reverse-mode oracle, with a nonzero
    initial state and a nonzero upstream gradient of the final state; ragged chunk tails."""
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.prefill_inputs(2, T, 2, d_, d_, io=ioname, seed=100 + T + d_, s0_std=0.1)
    dO, dsT = grad_inputs(d, 200 + T, dsT_std=0.3)
    gr = run_backward(kda, d, dO, dsT)
    ref = oracle.recurrent_backward(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]),
                                    f64(d["s0"]), f64(dO), f64(dsT))
    check_grads(gr, ref, io)
    assert serr(f64(gr["d_initial_state"]), ref["ds0"], io) <= 1.0


def test_backward_extreme_gates(kda):
    """Log-decays down to -40 per token (every exp of the pairwise form underflows or stays
    below 1) and near zero: no overflow, gradients still match in fp32."""
    d = inputs.prefill_inputs(1, 80, 2, 128, 128, io="f32", seed=120, s0_std=0.1)
    g = d["g"].clone()
    g[:, 10:30] = -40.0
    g[:, 50:] = -1e-4
    d["g"] = g
    dO, dsT = grad_inputs(d, 121, dsT_std=0.2)
    gr = run_backward(kda, d, dO, dsT)
    ref = oracle.recurrent_backward(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]),
                                    f64(d["s0"]), f64(dO), f64(dsT))
    check_grads(gr, ref, torch.float32)
    assert serr(f64(gr["d_initial_state"]), ref["ds0"], torch.float32) <= 1.0


def test_backward_without_states_and_zero_length(kda):
    """No initial state and no upstream state gradient (zeros); and T = 0, where the gradient
    of the initial state is the upstream one."""
    d = inputs.prefill_inputs(2, 33, 2, 64, 64, io="f32", seed=125)
    assert d["s0"] is None
    dO, _ = grad_inputs(d, 126)
    gr = run_backward(kda, d, dO, None)
    ref = oracle.recurrent_backward(*(f64(d[n]) for n in ("q", "k", "v", "g", "beta")), None, f64(dO), None)
    check_grads(gr, ref, torch.float32)
    assert serr(f64(gr["d_initial_state"]), ref["ds0"], torch.float32) <= 1.0
    d0 = inputs.prefill_inputs(2, 0, 2, 128, 128, io="bf16", seed=127)
    dsT = torch.randn((2, 2, 128, 128), generator=torch.Generator().manual_seed(128))
    gr0 = run_backward(kda, d0, torch.empty((2, 0, 2, 128), dtype=torch.bfloat16), dsT)
    assert torch.equal(gr0["d_initial_state"].cpu(), dsT)


def test_backward_is_deterministic(kda):
    d = inputs.prefill_inputs(1, 100, 3, 128, 128, io="bf16", seed=129, s0_std=0.05)
    dO, dsT = grad_inputs(d, 130, dsT_std=0.2)
    g1 = run_backward(kda, d, dO, dsT)
    g2 = run_backward(kda, d, dO, dsT)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "d_initial_state"):
        assert torch.equal(g1[n], g2[n]), n


def test_backward_workload_B1_T4096_H32_sampled_heads(kda):
    """The bf16 T = 4096, H = 32 prefill workload (S_0 ~ N(0, 0.02^2)) with dO ~ N(0, 1):
    sampled heads against the oracle over the whole sequence."""
    w = inputs.WORKLOADS["prefill_bf16_B1_T4096_H32_d128"]
    d = inputs.prefill_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"],
                              s0_std=w["s0_std"])
    dO, _ = grad_inputs(d, 130)
    gr = run_backward(kda, d, dO, None)
    for h in (0, 17, 31):
        sl = lambda x: x[:, :, h:h + 1]
        ref = oracle.recurrent_backward(*(f64(sl(d[n])) for n in ("q", "k", "v", "g", "beta")),
                                        f64(d["s0"][:, h:h + 1]), f64(sl(dO)), None, nthreads=1)
        check_grads(gr, ref, torch.bfloat16, index=lambda x, h=h: x[:, :, h:h + 1] if x.shape[2] == 32 else x)
        assert serr(f64(gr["d_initial_state"][:, h:h + 1]), ref["ds0"], torch.bfloat16) <= 1.0


def test_backward_workload_B4_T8192_H96_sampled_heads(kda):
    """The backward as the benchmark launches it: the B = 4, T = 8192, H = 96 bf16 prefill
    workload with dO ~ N(0, 1) (torch generator, seed 7), no state gradients; four heads
    checked over the whole 8192-token sequence against the reverse-mode oracle."""
    w = inputs.WORKLOADS["prefill_bf16_B4_T8192_H96_d128"]
    d = inputs.prefill_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"])
    gen = torch.Generator().manual_seed(7)
    dO = torch.randn(d["v"].shape, generator=gen).to(torch.bfloat16)
    gr = run_backward(kda, d, dO, None)
    for b, h in ((0, 0), (1, 40), (2, 77), (3, 95)):
        sl = lambda x, b=b, h=h: x[b:b + 1, :, h:h + 1]
        ref = oracle.recurrent_backward(*(f64(sl(d[n])) for n in ("q", "k", "v", "g", "beta")), None,
                                        f64(sl(dO)), None, nthreads=1)
        for name in ("dq", "dk", "dv", "dg", "dbeta"):
            e = err(f64(sl(gr[name])), ref[name], torch.bfloat16, stored_bf16=True)
            assert e <= 1.0, f"({b}, {h}) {name}: {e:.3e} of bound"
        assert serr(f64(gr["d_initial_state"][b:b + 1, h:h + 1]), ref["ds0"], torch.bfloat16) <= 1.0
    assert all(bool(torch.isfinite(gr[n]).all()) for n in ("dq", "dk", "dv", "dg", "dbeta"))


# ------------------------------------------------------------------------ layer


def run_layer(kda, d, with_final=True, lb=None):
    dev = "cuda"
    to = lambda x: None if x is None else x.to(dev)
    B, T, H, dk = d["g_raw"].shape
    dv = d["o_gate_raw"].shape[-1]
    sT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if with_final else None
    out, sT = kda.kda_layer_forward(
        to(d["q_raw"]), to(d["k_raw"]), to(d["v_raw"]), to(d["conv_q"]), to(d["conv_k"]),
        to(d["conv_v"]), to(d["g_raw"]), to(d["A_log"]), to(d["dt_bias"]), to(d["b_raw"]),
        to(d["o_gate_raw"]), to(d["o_norm_w"]), initial_state=to(d["s0"]), final_state=sT,
        gate_lower_bound=lb)
    kda.kda_check_device_error()
    return out, sT


def oracle_layer(d, io, heads=None, lb=None):
    a = {n: (None if d[n] is None else f64(d[n])) for n in d}
    io_bf16 = io == torch.bfloat16
    if heads is None:
        return oracle.layer(a["q_raw"], a["k_raw"], a["v_raw"], a["conv_q"], a["conv_k"], a["conv_v"],
                            a["g_raw"], a["A_log"], a["dt_bias"], a["b_raw"], a["o_gate_raw"],
                            a["o_norm_w"], io_bf16=io_bf16, s0=a["s0"], gate_lower_bound=lb)
    B, T, H, dk = a["g_raw"].shape
    dv = a["o_gate_raw"].shape[-1]
    outs, states = [], []
    for b, h in heads:
        ck = slice(h * dk, (h + 1) * dk)
        cv = slice(h * dv, (h + 1) * dv)
        o, s = oracle.layer(a["q_raw"][b:b + 1, :, ck], a["k_raw"][b:b + 1, :, ck],
                            a["v_raw"][b:b + 1, :, cv], a["conv_q"][ck], a["conv_k"][ck],
                            a["conv_v"][cv], a["g_raw"][b:b + 1, :, h:h + 1], a["A_log"][h:h + 1],
                            None if a["dt_bias"] is None else a["dt_bias"][ck], a["b_raw"][b:b + 1, :, h:h + 1],
                            a["o_gate_raw"][b:b + 1, :, h:h + 1], a["o_norm_w"], io_bf16=io_bf16,
                            s0=None if a["s0"] is None else a["s0"][b:b + 1, h:h + 1], gate_lower_bound=lb)
        outs.append(o[0, :, 0])
        states.append(s[0, 0])
    return np.stack(outs, 1)[None], np.stack(states, 0)[None]


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_", [64, 128])
@pytest.mark.parametrize("T", [1, 5, 64, 150])
def test_layer_small(kda, io, d_, T):
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.layer_inputs(2, T, 3, d_, d_, io=ioname, seed=40 + T + d_, s0_std=0.05,
                            dt_bias_std=0.5, gain_std=0.2)
    out, sT = run_layer(kda, d)
    ro, rs = oracle_layer(d, io)
    assert err(f64(out), ro, io, stored_bf16=2) <= tol(io)
    assert serr(f64(sT), rs, io) <= 1.0


@pytest.mark.parametrize("io,d_", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_layer_zero_length_copies_state(kda, io, d_):
    """T = 0: no output rows; the final state is the initial state, or zeros without one."""
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.layer_inputs(2, 0, 3, d_, d_, io=ioname, seed=47, s0_std=0.1)
    out, sT = run_layer(kda, d)
    assert out.numel() == 0
    assert torch.equal(sT.cpu(), d["s0"])
    d["s0"] = None
    _, sT = run_layer(kda, d)
    assert torch.count_nonzero(sT) == 0


def clamped_fraction(d, lb):
    g = oracle.gate(f64(d["g_raw"]), f64(d["A_log"]), None if d["dt_bias"] is None else f64(d["dt_bias"]))
    return float(np.mean(g < lb))


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_", [64, 128])
def test_layer_gate_lower_bound(kda, io, d_):
    """gate_lower_bound = -5 (the Kimi-K3 linear-attention config's value) on a draw where a
    good part of the log-decays fall below it: the layer equals the oracle with the bound."""
    ioname = "f32" if io == torch.float32 else "bf16"
    d = inputs.layer_inputs(2, 150, 3, d_, d_, io=ioname, seed=70 + d_, s0_std=0.05,
                            dt_bias_std=0.5, gain_std=0.2)
    assert clamped_fraction(d, -5.0) > 0.05
    out, sT = run_layer(kda, d, lb=-5.0)
    ro, rs = oracle_layer(d, io, lb=-5.0)
    assert err(f64(out), ro, io, stored_bf16=2) <= tol(io)
    assert serr(f64(sT), rs, io) <= 1.0
    ru, _ = oracle_layer(d, io)
    assert np.max(np.abs(ru - ro)) > 10 * np.max(np.abs(f64(out) - ro))   # the bound matters


@pytest.mark.parametrize("graw", [3.0, 1.0])
def test_layer_extreme_gates(kda, graw):
    """The layer kernel's exact diagonal path: with exp(A_log) = 8 and g_raw = 3 every token
    decays each channel by about e^-24, so every 16-token block is far below the e^-168 the
    midpoint factorisation takes (the kernel recomputes q, k and g of those channels from the
    raw tiles); g_raw = 1.0 puts about half the blocks on each side of it.  Against the oracle."""
    d = inputs.layer_inputs(2, 150, 3, 128, 128, io="bf16", seed=77, s0_std=0.05, dt_bias_std=0.2)
    d["A_log"] = torch.full_like(d["A_log"], float(np.log(8.0)))
    d["g_raw"] = (torch.full_like(d["g_raw"], graw).float() +
                  0.3 * torch.randn(d["g_raw"].shape, generator=torch.Generator().manual_seed(78))).to(torch.bfloat16)
    out, sT = run_layer(kda, d)
    ro, rs = oracle_layer(d, torch.bfloat16)
    assert err(f64(out), ro, torch.bfloat16, stored_bf16=2) <= 1.0
    assert serr(f64(sT), rs, torch.bfloat16) <= 1.0


def test_layer_a_wait_that_runs_out_reports_timeout(kda):
    """The fused layer kernel shares the bounded waits and the drain of the prefill kernel: a
    tile load that is never issued (chunk 2 of 5) makes its wait run out, the call reports
    KDA_ERR_TIMEOUT once, and the next call matches the oracle."""
    d = inputs.layer_inputs(2, 150, 3, 128, 128, io="bf16", seed=79, s0_std=0.05)
    kda.kda_set_wait_test_hooks(1_000_000, 2)
    try:
        with pytest.raises(kda.KdaError) as e:
            run_layer(kda, d)
        assert e.value.status == 5
    finally:
        kda.kda_set_wait_test_hooks(0, -1)
    kda.kda_check_device_error()
    out, sT = run_layer(kda, d)
    ro, rs = oracle_layer(d, torch.bfloat16)
    assert err(f64(out), ro, torch.bfloat16, stored_bf16=2) <= 1.0
    assert serr(f64(sT), rs, torch.bfloat16) <= 1.0


def test_layer_workload_B2_T16384_H96_sampled_heads(kda):
    """The full layer workload (bf16, unit gain, zero state) in the benchmark's launch shape."""
    w = inputs.WORKLOADS["layer_bf16_B2_T16384_H96_d128"]
    d = inputs.layer_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], io=w["io"], seed=w["seed"],
                            conv_std=w["conv_std"])
    out, sT = run_layer(kda, d)
    heads = [(0, 0), (1, 95), (0, 50), (1, 13)]
    ro, rs = oracle_layer(d, torch.bfloat16, heads)
    check_heads(out, sT, ro, rs, heads, torch.bfloat16, roundings=2)


def packed_layer_inputs(lens, H, d, io, seed, s0_std=0.05):
    """Token-major layer inputs over sum(lens) tokens, their offsets and a per-sequence S_0."""
    L = inputs.layer_inputs(1, int(sum(lens)), H, d, d, io=io, seed=seed, dt_bias_std=0.4, gain_std=0.2)
    P = {n: (v[0] if n in ("q_raw", "k_raw", "v_raw", "g_raw", "b_raw", "o_gate_raw") else v) for n, v in L.items()}
    P["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    P["s0"] = torch.randn((len(lens), H, d, d), generator=torch.Generator().manual_seed(seed)) * s0_std
    return P


def run_layer_varlen(kda, P, lb=None):
    dev = "cuda"
    to = lambda x: None if x is None else x.contiguous().to(dev)
    N, H, d = P["s0"].shape[0], P["g_raw"].shape[1], P["g_raw"].shape[2]
    sT = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    out, sT = kda.kda_layer_forward_varlen(
        to(P["q_raw"]), to(P["k_raw"]), to(P["v_raw"]), to(P["conv_q"]), to(P["conv_k"]), to(P["conv_v"]),
        to(P["g_raw"]), to(P["A_log"]), to(P["dt_bias"]), to(P["b_raw"]), to(P["o_gate_raw"]),
        to(P["cu_seqlens"]), to(P["o_norm_w"]), initial_state=to(P["s0"]), final_state=sT, gate_lower_bound=lb)
    kda.kda_check_device_error()
    return out, sT


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_", [64, 128])
def test_layer_varlen_ragged(kda, io, d_):
    """Packed sequences shorter than the conv (1, 2 tokens), shorter than a prologue run,
    around a chunk and several chunks long, with empty ones between: every output and every
    final state against the oracle run per sequence."""
    lens = [0, 1, 2, 5, 63, 64, 0, 65, 7, 130]
    P = packed_layer_inputs(lens, 3, d_, "f32" if io == torch.float32 else "bf16", seed=140 + d_)
    out, sT = run_layer_varlen(kda, P, lb=-6.0)
    a = {n: (None if v is None else f64(v)) for n, v in P.items()}
    ro, rs = oracle.layer_varlen(a["q_raw"], a["k_raw"], a["v_raw"], a["conv_q"], a["conv_k"], a["conv_v"],
                                 a["g_raw"], a["A_log"], a["dt_bias"], a["b_raw"], a["o_gate_raw"],
                                 P["cu_seqlens"].numpy(), a["o_norm_w"], s0=a["s0"],
                                 io_bf16=io == torch.bfloat16, gate_lower_bound=-6.0)
    assert err(f64(out), ro, io, stored_bf16=2) <= tol(io)
    assert serr(f64(sT), rs, io) <= 1.0


def test_layer_varlen_many_short_sequences(kda):
    """200 packed sequences of 0..20 tokens (the final states are a few nearly rank-one
    updates of a small initial state, the case that bounds the state's rounding), bf16 at
    d = 128 on the fused tensor-core kernel: every output and every final state."""
    lens = [int(x) for x in np.random.default_rng(93).integers(0, 21, 200)]
    P = packed_layer_inputs(lens, 2, 128, "bf16", seed=94, s0_std=0.02)
    out, sT = run_layer_varlen(kda, P)
    a = {n: (None if v is None else f64(v)) for n, v in P.items()}
    ro, rs = oracle.layer_varlen(a["q_raw"], a["k_raw"], a["v_raw"], a["conv_q"], a["conv_k"], a["conv_v"],
                                 a["g_raw"], a["A_log"], a["dt_bias"], a["b_raw"], a["o_gate_raw"],
                                 P["cu_seqlens"].numpy(), a["o_norm_w"], s0=a["s0"], io_bf16=True)
    assert err(f64(out), ro, torch.bfloat16, stored_bf16=2) <= tol(torch.bfloat16)
    assert serr(f64(sT), rs, torch.bfloat16) <= 1.0


def test_layer_varlen_equal_lengths_equal_the_batched_layer(kda):
    """Three packed sequences of 70 tokens give kda_layer_forward's B = 3 results bit for bit."""
    P = packed_layer_inputs([70, 70, 70], 2, 128, "bf16", seed=150)
    ov, sv = run_layer_varlen(kda, P)
    d = {n: (v.reshape((3, 70) + tuple(v.shape[1:])) if n in ("q_raw", "k_raw", "v_raw", "g_raw", "b_raw",
                                                               "o_gate_raw") else v) for n, v in P.items()}
    ob, sb = run_layer(kda, d)
    assert torch.equal(ov.reshape(ob.shape), ob)
    assert torch.equal(sv, sb)


def test_layer_zero_gate_input_halves_output(kda):
    """o_gate_raw = 0: the output is exactly half the gain-scaled normalised output of the
    same call with a saturated gate (sigmoid(0) = 1/2)."""
    d = inputs.layer_inputs(1, 70, 2, 128, 128, io="f32", seed=50)
    d["o_gate_raw"] = torch.zeros_like(d["o_gate_raw"])
    half, _ = run_layer(kda, d)
    d["o_gate_raw"] = torch.full_like(d["o_gate_raw"], 100.0)
    full, _ = run_layer(kda, d)
    torch.testing.assert_close(2 * half, full, rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------------ layer decode (conv cache)


@pytest.mark.parametrize("lb", [None, -2.0])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_layer_decode_steps_equal_layer_over_the_same_tokens(kda, io, lb):
    """n layer-decode steps from an empty conv cache give the layer's outputs over those n
    tokens and its final state; the cache ends holding the last three raw tokens, bit for bit."""
    ioname = "f32" if io == torch.float32 else "bf16"
    B, T, H, d = 3, 9, 4, 128
    L = inputs.layer_inputs(B, T, H, d, d, io=ioname, seed=60, s0_std=0.05, dt_bias_std=0.4, gain_std=0.2)
    dev = "cuda"
    to = lambda x: None if x is None else x.contiguous().to(dev)
    state = L["s0"].clone().to(dev)
    caches = [torch.zeros((B, 3, H * d), dtype=io, device=dev) for _ in range(3)]
    outs = []
    for t in range(T):
        o = kda.kda_layer_decode_step(
            to(L["q_raw"][:, t]), to(L["k_raw"][:, t]), to(L["v_raw"][:, t]), to(L["conv_q"]), to(L["conv_k"]),
            to(L["conv_v"]), *caches, to(L["g_raw"][:, t]), to(L["A_log"]), to(L["dt_bias"]), to(L["b_raw"][:, t]),
            to(L["o_gate_raw"][:, t]), state, to(L["o_norm_w"]), gate_lower_bound=lb)
        outs.append(o)
    kda.kda_check_device_error()
    out = torch.stack(outs, 1)
    if lb is not None:
        assert clamped_fraction(L, lb) > 0.05
    ro, rs = oracle_layer(L, io, lb=lb)
    assert err(f64(out), ro, io, stored_bf16=2) <= 1.0
    assert serr(f64(state), rs, io) <= 1.0
    for c, n in zip(caches, ("q_raw", "k_raw", "v_raw")):
        assert torch.equal(c.cpu(), L[n][:, T - 3:T].contiguous())


def test_layer_decode_continues_a_layer_prefill(kda):
    """Prefill the layer over 70 tokens, then decode 5 more with the cache seeded from the last
    three raw tokens and the prefill's final state: the outputs equal the layer over 75 tokens."""
    B, T0, T1, H, d = 2, 70, 5, 3, 128
    L = inputs.layer_inputs(B, T0 + T1, H, d, d, io="bf16", seed=61, dt_bias_std=0.3)
    dev = "cuda"
    to = lambda x: None if x is None else x.contiguous().to(dev)
    head = {n: (v if v is None or n in ("conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "o_norm_w", "s0")
                else v[:, :T0].contiguous()) for n, v in L.items()}
    _, state = run_layer(kda, head)
    caches = [to(L[n][:, T0 - 3:T0]) for n in ("q_raw", "k_raw", "v_raw")]
    outs = []
    for t in range(T0, T0 + T1):
        outs.append(kda.kda_layer_decode_step(
            to(L["q_raw"][:, t]), to(L["k_raw"][:, t]), to(L["v_raw"][:, t]), to(L["conv_q"]), to(L["conv_k"]),
            to(L["conv_v"]), *caches, to(L["g_raw"][:, t]), to(L["A_log"]), to(L["dt_bias"]), to(L["b_raw"][:, t]),
            to(L["o_gate_raw"][:, t]), state, to(L["o_norm_w"])))
    kda.kda_check_device_error()
    ro, rs = oracle_layer(L, torch.bfloat16)
    assert err(f64(torch.stack(outs, 1)), ro[:, T0:], torch.bfloat16, stored_bf16=2) <= 1.0
    assert serr(f64(state), rs, torch.bfloat16) <= 1.0
