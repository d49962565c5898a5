"""Pins for the fp64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: an equivalent
blocked algebra (the chunked rewrite), dense brute force, closed forms, textbook
linear attention computed by an independent triple loop, library routines
(torch conv1d / silu, numpy logaddexp, scipy expit) and invariants that the
mathematics fixes.  A plausible slip in the oracle (a dropped term, a sign, an
index, the order of decay and correction, reading before instead of after the
update, a transposed operand) fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle.chunked import chunked


def _rand_inputs(rng, B, T, H, dk, dv, *, gscale=1.0, unit_k=True, s0_std=0.1):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    A = rng.uniform(0, math.log(8.0), H)
    g = -np.exp(A)[None, None, :, None] * np.logaddexp(0, rng.standard_normal((B, T, H, dk))) * gscale
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    s0 = rng.standard_normal((B, H, dk, dv)) * s0_std if s0_std > 0 else None
    return q, k, v, g, beta, s0


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --------------------------------------------------------------- recurrence


@pytest.mark.parametrize("chunk", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("T", [1, 7, 16, 37])
def test_chunked_rewrite_equals_recurrence(chunk, T):
    """Self-check 1: the chunkwise (UT/WY) rewrite equals the token recurrence."""
    rng = np.random.default_rng(100 + 7 * chunk + T)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 2, T, 2, 8, 5, gscale=0.3)
    o_r, s_r = oracle.recurrent(q, k, v, g, beta, s0)
    o_c, s_c = chunked(q, k, v, g, beta, s0, chunk=chunk)
    assert _rel(o_c, o_r) < 1e-12
    assert _rel(s_c, s_r) < 1e-12


def test_zero_decay_zero_beta_is_readout_of_initial_state():
    """Self-check 2(i): g = 0, beta = 0 => o_t = S0^T q_t and S_T = S0, exactly."""
    rng = np.random.default_rng(1)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 9, 2, 6, 4)
    o, sT = oracle.recurrent(q, k, v, np.zeros_like(g), np.zeros_like(beta), s0)
    np.testing.assert_array_equal(sT, s0)
    ref = np.einsum("bthc,bhcv->bthv", q, s0)
    assert _rel(o, ref) < 1e-14


def _causal_linear_attention(q, k, v):
    """Textbook causal linear attention, o_t = sum_{j<=t} (q_t . k_j) v_j, by triple loop."""
    B, T, H, dk = q.shape
    o = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for j in range(t + 1):
                    o[b, t, h] += np.dot(q[b, t, h], k[b, j, h]) * v[b, j, h]
    return o


def test_small_beta_limit_is_causal_linear_attention():
    """Self-check 2(ii): g = 0, beta = eps -> (o(eps) - o(0)) / eps = linear attention + O(eps t)."""
    rng = np.random.default_rng(2)
    q, k, v, g, beta, _ = _rand_inputs(rng, 1, 12, 2, 5, 3)
    eps = 1e-7
    o, _ = oracle.recurrent(q, k, v, np.zeros_like(g), np.full_like(beta, eps), None)
    ref = _causal_linear_attention(q, k, v)
    assert _rel(o / eps, ref) < 1e-5


def test_without_correction_is_exact_linear_attention():
    """Self-check 2(iii): with the correction term removed (test-only variant), g = 0,
    beta = 1: o_t = S0^T q_t + sum_{j<=t} (q_t.k_j) v_j.  Pins write k v^T, read after update."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 2, 10, 2, 4, 6, unit_k=False)
    o, sT = oracle.recurrent(q, k, v, np.zeros_like(g), np.ones_like(beta), s0, delta=False)
    ref = _causal_linear_attention(q, k, v) + np.einsum("bthc,bhcv->bthv", q, s0)
    assert _rel(o, ref) < 1e-13
    assert _rel(sT, s0 + np.einsum("bthc,bthv->bhcv", k, v)) < 1e-13


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_unrolled_product_of_transition_matrices(T):
    """Self-check 3: S_t = M_t S_{t-1} + beta_t k_t v_t^T with dense
    M_t = (I - beta_t k_t k_t^T) Diag(exp g_t), built and multiplied explicitly."""
    rng = np.random.default_rng(10 + T)
    dk, dv = 5, 4
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, T, 1, dk, dv, unit_k=False, gscale=0.5)
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    S = s0[0, 0].copy()
    o_ref = np.zeros((T, dv))
    for t in range(T):
        kt, bt = k[0, t, 0], beta[0, t, 0]
        M = (np.eye(dk) - bt * np.outer(kt, kt)) @ np.diag(np.exp(g[0, t, 0]))
        S = M @ S + bt * np.outer(kt, v[0, t, 0])
        o_ref[t] = S.T @ q[0, t, 0]
    assert _rel(sT[0, 0], S) < 1e-13
    assert _rel(o[0, :, 0], o_ref) < 1e-13


def test_wrong_operator_order_is_detected():
    """The unrolled product distinguishes decay-then-correct from correct-then-decay."""
    rng = np.random.default_rng(5)
    dk, dv = 4, 3
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 3, 1, dk, dv, unit_k=False, gscale=2.0)
    _, sT = oracle.recurrent(q, k, v, g, beta, s0)
    S = s0[0, 0].copy()
    for t in range(3):
        kt, bt = k[0, t, 0], beta[0, t, 0]
        M = np.diag(np.exp(g[0, t, 0])) @ (np.eye(dk) - bt * np.outer(kt, kt))
        S = M @ S + bt * np.outer(kt, v[0, t, 0])
    assert _rel(sT[0, 0], S) > 1e-3


def test_delta_rule_retrieval():
    """||k|| = 1, beta = 1: after the write, S_t^T k_t = v_t exactly (any decay).
    General beta: S_t^T k_t = (1 - beta ||k||^2) (D S_{t-1})^T k_t + beta ||k||^2 v_t."""
    rng = np.random.default_rng(6)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 6, 2, 8, 5)
    _, sT = oracle.recurrent(q, k, v, g, np.ones_like(beta), s0)
    kt, vt = k[0, -1], v[0, -1]
    assert _rel(np.einsum("hcv,hc->hv", sT[0], kt), vt) < 1e-12
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 6, 2, 8, 5, unit_k=False)
    _, s_prev = oracle.recurrent(q[:, :5], k[:, :5], v[:, :5], g[:, :5], beta[:, :5], s0)
    _, s_t = oracle.recurrent(q, k, v, g, beta, s0)
    kt, vt, bt, gt = k[0, 5], v[0, 5], beta[0, 5], g[0, 5]
    DS = np.exp(gt)[:, :, None] * s_prev[0]
    kk = np.sum(kt * kt, axis=-1)
    ref = (1 - bt * kk)[:, None] * np.einsum("hcv,hc->hv", DS, kt) + (bt * kk)[:, None] * vt
    assert _rel(np.einsum("hcv,hc->hv", s_t[0], kt), ref) < 1e-12


def test_pure_decay_closed_form():
    """beta = 0: S_T = Diag(exp sum_t g_t) S0 and o_t = (exp(G_t) * q_t)^T S0."""
    rng = np.random.default_rng(7)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 2, 11, 2, 6, 4, gscale=0.2)
    o, sT = oracle.recurrent(q, k, v, g, np.zeros_like(beta), s0)
    G = np.cumsum(g, axis=1)
    assert _rel(sT, np.exp(G[:, -1])[..., None] * s0) < 1e-13
    assert _rel(o, np.einsum("bthc,bhcv->bthv", np.exp(G) * q, s0)) < 1e-13


def test_small_beta_limit_is_gated_linear_attention():
    """S0 = 0, beta = eps: o_t / eps -> sum_{j<=t} sum_c q_t[c] k_j[c] exp(G_t[c] - G_j[c]) v_j."""
    rng = np.random.default_rng(8)
    q, k, v, g, beta, _ = _rand_inputs(rng, 1, 10, 1, 4, 3, gscale=0.3)
    eps = 1e-7
    o, _ = oracle.recurrent(q, k, v, g, np.full_like(beta, eps), None)
    G = np.cumsum(g[0, :, 0], axis=0)
    ref = np.zeros((10, 3))
    for t in range(10):
        for j in range(t + 1):
            w = np.sum(q[0, t, 0] * k[0, j, 0] * np.exp(G[t] - G[j]))
            ref[t] += w * v[0, j, 0]
    assert _rel(o[0, :, 0] / eps, ref) < 1e-5


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(9)
    q, k, v1, g, beta, s1 = _rand_inputs(rng, 1, 13, 2, 6, 5)
    v2 = rng.standard_normal(v1.shape)
    s2 = rng.standard_normal(s1.shape)
    a, b = 0.7, -1.3
    o1, t1 = oracle.recurrent(q, k, v1, g, beta, s1)
    o2, t2 = oracle.recurrent(q, k, v2, g, beta, s2)
    o3, t3 = oracle.recurrent(q, k, a * v1 + b * v2, g, beta, a * s1 + b * s2)
    assert _rel(o3, a * o1 + b * o2) < 1e-12
    assert _rel(t3, a * t1 + b * t2) < 1e-12


def test_value_columns_are_separable():
    rng = np.random.default_rng(10)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 15, 2, 6, 7)
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    oa, sa = oracle.recurrent(q, k, v[..., :3], g, beta, s0[..., :3])
    ob, sb = oracle.recurrent(q, k, v[..., 3:], g, beta, s0[..., 3:])
    assert _rel(np.concatenate([oa, ob], -1), o) < 1e-14
    assert _rel(np.concatenate([sa, sb], -1), sT) < 1e-14


def test_state_passing_and_decode_consistency():
    rng = np.random.default_rng(11)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 2, 20, 3, 6, 4)
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    oa, sa = oracle.recurrent(q[:, :7], k[:, :7], v[:, :7], g[:, :7], beta[:, :7], s0)
    ob, sb = oracle.recurrent(q[:, 7:], k[:, 7:], v[:, 7:], g[:, 7:], beta[:, 7:], sa)
    assert _rel(np.concatenate([oa, ob], 1), o) < 1e-13
    assert _rel(sb, sT) < 1e-13
    # decode x 20 == prefill over the same 20 tokens; prefill with T = 1 == decode
    st = s0.copy()
    for t in range(20):
        od, st = oracle.decode(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], st)
        assert _rel(od, o[:, t]) < 1e-13
    assert _rel(st, sT) < 1e-13


def test_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 0, 2, 4, 4)
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    assert o.shape == (1, 0, 2, 4)
    np.testing.assert_array_equal(sT, s0)


def test_varlen_equal_lengths_equal_the_batched_call():
    """Packed sequences of one common length give the batched result bit for bit."""
    rng = np.random.default_rng(14)
    B, T, H = 3, 11, 2
    q, k, v, g, beta, s0 = _rand_inputs(rng, B, T, H, 6, 5)
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    pk = lambda x: x.reshape((B * T,) + x.shape[2:])
    ov, sv = oracle.recurrent_varlen(pk(q), pk(k), pk(v), pk(g), pk(beta), np.arange(B + 1) * T, s0)
    np.testing.assert_array_equal(ov, pk(o))
    np.testing.assert_array_equal(sv, sT)


def test_varlen_ragged_equals_chunked_form_per_sequence():
    """Ragged lengths (0 and 1 among them): every sequence equals the chunkwise rewrite run
    on it alone, and a zero-length sequence passes its initial state through."""
    rng = np.random.default_rng(15)
    lens = [5, 0, 1, 17, 9, 0, 33]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Tt, H, dk, dv = int(cu[-1]), 2, 6, 4
    q, k, v, g, beta, _ = _rand_inputs(rng, 1, Tt, H, dk, dv, s0_std=0)
    s0 = rng.standard_normal((len(lens), H, dk, dv)) * 0.1
    o, sT = oracle.recurrent_varlen(q[0], k[0], v[0], g[0], beta[0], cu, s0)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if a == b:
            np.testing.assert_array_equal(sT[n], s0[n])
            continue
        oc, sc = chunked(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b], s0[n:n + 1], chunk=4)
        assert _rel(o[a:b], oc[0]) < 1e-12 and _rel(sT[n], sc[0]) < 1e-12


def test_varlen_sequences_are_isolated():
    """Changing one sequence's tokens changes no other sequence's outputs or final state."""
    rng = np.random.default_rng(16)
    cu = np.array([0, 6, 13, 20])
    q, k, v, g, beta, _ = _rand_inputs(rng, 1, 20, 2, 5, 5, s0_std=0)
    o1, s1 = oracle.recurrent_varlen(q[0], k[0], v[0], g[0], beta[0], cu)
    v2 = v.copy()
    v2[0, 6:13] += 1.0
    o2, s2 = oracle.recurrent_varlen(q[0], k[0], v2[0], g[0], beta[0], cu)
    np.testing.assert_array_equal(o1[:6], o2[:6])
    np.testing.assert_array_equal(o1[13:], o2[13:])
    np.testing.assert_array_equal(s1[[0, 2]], s2[[0, 2]])
    assert np.max(np.abs(o1[6:13] - o2[6:13])) > 1e-3


# --------------------------------------------------------------- gradients


def _loss(q, k, v, g, beta, s0, Wo, Ws):
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    return float(np.sum(Wo * o) + np.sum(Ws * sT))


def test_backward_equals_central_differences():
    """Every gradient of L = <Wo, o> + <Ws, S_T> against central differences of the forward
    oracle (step 1e-6; the difference error is O(1e-12) here)."""
    rng = np.random.default_rng(31)
    B, T, H, dk, dv = 1, 6, 2, 4, 3
    q, k, v, g, beta, s0 = _rand_inputs(rng, B, T, H, dk, dv, s0_std=0.5)
    Wo = rng.standard_normal((B, T, H, dv))
    Ws = rng.standard_normal((B, H, dk, dv))
    gr = oracle.recurrent_backward(q, k, v, g, beta, s0, Wo, Ws)
    args = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "s0": s0}
    eps = 1e-6
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("s0", "ds0")):
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + eps
            lp = _loss(**args, Wo=Wo, Ws=Ws)
            x[idx] = old - eps
            lm = _loss(**args, Wo=Wo, Ws=Ws)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        assert _rel(gr[key], fd) < 1e-7, name


def test_backward_equals_torch_autograd():
    """The same gradients from torch autograd through a plain fp64 token loop of the
    recurrence (an independent route: library reverse mode, no hand-written chain rule)."""
    rng = np.random.default_rng(32)
    B, T, H, dk, dv = 2, 9, 2, 5, 4
    q, k, v, g, beta, s0 = _rand_inputs(rng, B, T, H, dk, dv, s0_std=0.3)
    Wo = rng.standard_normal((B, T, H, dv))
    Ws = rng.standard_normal((B, H, dk, dv))
    ts = {n: torch.tensor(x, requires_grad=True) for n, x in
          (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("s0", s0))}
    S = ts["s0"]
    outs = []
    for t in range(T):
        Sp = torch.exp(ts["g"][:, t])[..., None] * S
        r = torch.einsum("bhcj,bhc->bhj", Sp, ts["k"][:, t])
        u = ts["beta"][:, t][..., None] * (ts["v"][:, t] - r)
        S = Sp + ts["k"][:, t][..., None] * u[:, :, None, :]
        outs.append(torch.einsum("bhcj,bhc->bhj", S, ts["q"][:, t]))
    o = torch.stack(outs, 1)
    (torch.sum(torch.tensor(Wo) * o) + torch.sum(torch.tensor(Ws) * S)).backward()
    gr = oracle.recurrent_backward(q, k, v, g, beta, s0, Wo, Ws)
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("s0", "ds0")):
        assert _rel(gr[key], ts[name].grad.numpy()) < 1e-12, name


def test_backward_without_decay_or_write_is_a_readout():
    """g = 0, beta = 0: o_t = S_0^T q_t, so dq_t = S_0 do_t, dS_0 = dS_T + sum_t q_t do_t^T,
    and nothing flows to v or k (u = 0 and the correction is scaled by beta = 0)."""
    rng = np.random.default_rng(33)
    B, T, H, dk, dv = 1, 5, 1, 4, 3
    q, k, v, _, _, s0 = _rand_inputs(rng, B, T, H, dk, dv, s0_std=1.0)
    g = np.zeros((B, T, H, dk))
    beta = np.zeros((B, T, H))
    Wo = rng.standard_normal((B, T, H, dv))
    Ws = rng.standard_normal((B, H, dk, dv))
    gr = oracle.recurrent_backward(q, k, v, g, beta, s0, Wo, Ws)
    assert _rel(gr["dq"], np.einsum("bhcj,bthj->bthc", s0, Wo)) < 1e-14
    assert _rel(gr["ds0"], Ws + np.einsum("bthc,bthj->bhcj", q, Wo)) < 1e-14
    assert np.all(gr["dv"] == 0.0) and np.all(gr["dk"] == 0.0)


def test_state_norm_bound():
    """||k|| = 1, beta in [0, 1], g <= 0  =>  ||S_t||_2 <= ||S_{t-1}||_2 + beta_t ||v_t||."""
    rng = np.random.default_rng(13)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 25, 1, 6, 5, s0_std=1.0)
    prev = s0
    for t in range(25):
        _, s = oracle.recurrent(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], g[:, t:t + 1],
                                beta[:, t:t + 1], prev)
        lhs = np.linalg.norm(s[0, 0], 2)
        rhs = np.linalg.norm(prev[0, 0], 2) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert lhs <= rhs * (1 + 1e-12)
        prev = s


def test_extreme_gates_have_no_overflow():
    """Very strong decay (g ~ -40 per step) and very weak decay (g ~ -1e-4): finite, and
    strong decay leaves only the last token: o_T ~ (q.k)(beta v) with S0 forgotten."""
    rng = np.random.default_rng(14)
    q, k, v, g, beta, s0 = _rand_inputs(rng, 1, 70, 2, 8, 4)
    o, sT = oracle.recurrent(q, k, v, np.full_like(g, -40.0), beta, s0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(sT))
    last = np.sum(q[0, -1] * k[0, -1], -1)[:, None] * beta[0, -1][:, None] * v[0, -1]
    assert _rel(o[0, -1], last) < 1e-12
    o2, s2 = oracle.recurrent(q, k, v, np.full_like(g, -1e-4), beta, s0)
    o3, s3 = chunked(q, k, v, np.full_like(g, -1e-4), beta, s0, chunk=16)
    assert _rel(o2, o3) < 1e-11 and _rel(s2, s3) < 1e-11


# --------------------------------------------------------------- prologue / epilogue


def test_short_conv_matches_torch_depthwise_conv1d():
    """Depthwise causal conv == torch Conv1d(groups=C, padding=3) truncated to T, then SiLU."""
    rng = np.random.default_rng(20)
    B, T, C = 2, 11, 6
    x = rng.standard_normal((B, T, C))
    w = rng.standard_normal((C, 4))
    xt = torch.from_numpy(x).permute(0, 2, 1)
    ref = torch.nn.functional.conv1d(xt, torch.from_numpy(w)[:, None, :], padding=3, groups=C)
    ref = ref[:, :, :T].permute(0, 2, 1).numpy()
    assert _rel(oracle.short_conv(x, w, silu=False), ref) < 1e-14
    ref_silu = torch.nn.functional.silu(torch.from_numpy(ref)).numpy()
    assert _rel(oracle.short_conv(x, w, silu=True), ref_silu) < 1e-14


def test_short_conv_one_hot_taps_shift():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((1, 9, 3))
    for tap, shift in ((3, 0), (2, 1), (0, 3)):
        w = np.zeros((3, 4))
        w[:, tap] = 1.0
        y = oracle.short_conv(x, w, silu=False)
        ref = np.zeros_like(x)
        ref[:, shift:] = x[:, :9 - shift]
        np.testing.assert_array_equal(y, ref)


def test_l2norm_closed_form():
    rng = np.random.default_rng(22)
    x = rng.standard_normal((4, 7, 16))
    eps = 1e-6
    y = oracle.l2norm(x, eps)
    s = np.sum(x * x, -1)
    assert _rel(np.sum(y * y, -1), s / (s + eps)) < 1e-14
    assert _rel(y * np.sqrt(s + eps)[..., None], x) < 1e-14


def test_gate_special_values_and_library_softplus():
    rng = np.random.default_rng(23)
    B, T, H, dk = 1, 3, 4, 5
    A = rng.uniform(0, math.log(8), H)
    bias = rng.standard_normal(H * dk)
    g0 = oracle.gate(-bias.reshape(1, 1, H, dk).repeat(3, 1), A, bias)
    assert _rel(g0, np.broadcast_to(-np.exp(A)[None, None, :, None] * math.log(2), g0.shape)) < 1e-15
    x = rng.standard_normal((B, T, H, dk)) * 30
    g = oracle.gate(x, A, None)
    ref = -np.exp(A)[None, None, :, None] * np.logaddexp(0, x)
    assert _rel(g, ref) < 1e-14
    assert np.all(g < 0)


def test_gate_lower_bound():
    """The bound replaces exactly the log-decays below it and leaves the rest bit for bit;
    a bound of 0 removes every decay; -inf is no bound."""
    rng = np.random.default_rng(27)
    B, T, H, dk = 2, 5, 3, 16
    A = rng.uniform(0, math.log(8), H)
    bias = rng.standard_normal(H * dk) * 0.5
    x = rng.standard_normal((B, T, H, dk)) * 2
    g = oracle.gate(x, A, bias)
    gb = oracle.gate(x, A, bias, lower_bound=-5.0)
    below = g < -5.0
    assert 0.05 < below.mean() < 0.95   # the draw exercises both sides
    np.testing.assert_array_equal(gb[~below], g[~below])
    assert np.all(gb[below] == -5.0) and np.all(gb >= -5.0)
    np.testing.assert_array_equal(oracle.gate(x, A, bias, lower_bound=float("-inf")), g)
    assert np.all(oracle.gate(x, A, bias, lower_bound=0.0) == 0.0)


def test_sigmoid_matches_scipy():
    x = np.linspace(-40, 40, 101)
    assert _rel(oracle.sigmoid(x), scipy.special.expit(x)) < 1e-15


def test_out_norm_gate_closed_forms():
    rng = np.random.default_rng(24)
    o = rng.standard_normal((6, 32)) * 3
    eps = 1e-6
    # zero gate input: exactly half of the normalised output
    y = oracle.out_norm_gate(o, np.zeros_like(o), None, eps, io_bf16=False)
    m = np.mean(o * o, -1)
    assert _rel(2 * y, o / np.sqrt(m + eps)[:, None]) < 1e-14
    assert _rel(np.mean((2 * y) ** 2, -1), m / (m + eps)) < 1e-13
    # per-channel gain multiplies after the normalisation
    gain = rng.uniform(0.5, 2, 32)
    yg = oracle.out_norm_gate(o, np.zeros_like(o), gain, eps, io_bf16=False)
    assert _rel(yg, y * gain) < 1e-14
    # bf16 cast: saturate the gate (sigmoid -> 1) and check the result is a bf16 value
    yb = oracle.out_norm_gate(o, np.full_like(o, 800.0), None, eps, io_bf16=True)
    rt = torch.from_numpy(yb).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(yb, rt)
    assert np.max(np.abs(yb - 2 * y) / np.abs(2 * y)) <= 2.0 ** -8


@pytest.mark.parametrize("lb", [None, -1.5])
def test_layer_wiring_with_identity_conv(lb):
    """One-hot (identity) conv taps: the layer equals the prologue built from torch library
    ops, the recurrence, then RMSNorm x sigmoid gate built from numpy (with the gate's
    lower bound, when given, applied by numpy's maximum)."""
    rng = np.random.default_rng(25)
    B, T, H, d = 2, 9, 2, 8
    q_raw = rng.standard_normal((B, T, H * d))
    k_raw = rng.standard_normal((B, T, H * d))
    v_raw = rng.standard_normal((B, T, H * d))
    g_raw = rng.standard_normal((B, T, H, d))
    b_raw = rng.standard_normal((B, T, H))
    z = rng.standard_normal((B, T, H, d))
    A = rng.uniform(0, math.log(8), H)
    bias = rng.standard_normal(H * d) * 0.3
    gain = rng.uniform(0.5, 1.5, d)
    s0 = rng.standard_normal((B, H, d, d)) * 0.1
    w = np.zeros((H * d, 4))
    w[:, 3] = 1.0
    out, sT = oracle.layer(q_raw, k_raw, v_raw, w, w, w, g_raw, A, bias, b_raw, z, gain,
                           io_bf16=False, s0=s0, gate_lower_bound=lb)
    F = torch.nn.functional
    silu = lambda a: F.silu(torch.from_numpy(a)).numpy()
    qn = silu(q_raw).reshape(B, T, H, d)
    kn = silu(k_raw).reshape(B, T, H, d)
    qn = qn / np.sqrt(np.sum(qn * qn, -1, keepdims=True) + 1e-6)
    kn = kn / np.sqrt(np.sum(kn * kn, -1, keepdims=True) + 1e-6)
    vn = silu(v_raw).reshape(B, T, H, d)
    gg = -np.exp(A)[None, None, :, None] * F.softplus(
        torch.from_numpy(g_raw + bias.reshape(H, d))).numpy()
    if lb is not None:
        assert np.mean(gg < lb) > 0.1
        gg = np.maximum(gg, lb)
    bb = scipy.special.expit(b_raw)
    o, s_ref = oracle.recurrent(qn, kn, vn, gg, bb, s0)
    rms = np.sqrt(np.mean(o * o, -1, keepdims=True) + 1e-6)
    ref = gain * (o / rms) * scipy.special.expit(z)
    assert _rel(out, ref) < 1e-12
    assert _rel(sT, s_ref) < 1e-12


def test_layer_gate_bound_zero_equals_vanishing_decay_rate():
    """A gate bound of 0 and exp(A_log) -> 0 are two routes to g = 0 (the ungated delta
    rule); a bound below every log-decay changes nothing."""
    rng = np.random.default_rng(28)
    B, T, H, d = 1, 10, 2, 8
    raw = [rng.standard_normal((B, T, H * d)) for _ in range(3)]
    ws = [rng.standard_normal((H * d, 4)) * 0.5 for _ in range(3)]
    g_raw = rng.standard_normal((B, T, H, d))
    b_raw = rng.standard_normal((B, T, H))
    z = rng.standard_normal((B, T, H, d))
    A = rng.uniform(0, math.log(8), H)
    s0 = rng.standard_normal((B, H, d, d)) * 0.2
    o1, s1 = oracle.layer(*raw, *ws, g_raw, A, None, b_raw, z, None, io_bf16=False, s0=s0,
                          gate_lower_bound=0.0)
    o2, s2 = oracle.layer(*raw, *ws, g_raw, np.full(H, -800.0), None, b_raw, z, None,
                          io_bf16=False, s0=s0)
    assert _rel(o1, o2) < 1e-14 and _rel(s1, s2) < 1e-14
    gmin = oracle.gate(g_raw, A, None).min()
    o3, s3 = oracle.layer(*raw, *ws, g_raw, A, None, b_raw, z, None, io_bf16=False, s0=s0,
                          gate_lower_bound=gmin - 1.0)
    o4, s4 = oracle.layer(*raw, *ws, g_raw, A, None, b_raw, z, None, io_bf16=False, s0=s0)
    np.testing.assert_array_equal(o3, o4)
    np.testing.assert_array_equal(s3, s4)
    o5, _ = oracle.layer(*raw, *ws, g_raw, A, None, b_raw, z, None, io_bf16=False, s0=s0,
                         gate_lower_bound=-1.0)
    assert np.max(np.abs(o5 - o4)) > 1e-3


def _layer_raw(rng, T, H, d):
    return dict(q_raw=rng.standard_normal((T, H * d)), k_raw=rng.standard_normal((T, H * d)),
                v_raw=rng.standard_normal((T, H * d)), g_raw=rng.standard_normal((T, H, d)),
                b_raw=rng.standard_normal((T, H)), o_gate_raw=rng.standard_normal((T, H, d)))


def test_layer_varlen_equal_lengths_equal_the_batched_layer():
    rng = np.random.default_rng(34)
    B, T, H, d = 3, 7, 2, 4
    r = _layer_raw(rng, B * T, H, d)
    ws = [rng.standard_normal((H * d, 4)) * 0.5 for _ in range(3)]
    A = rng.uniform(0, 1, H)
    s0 = rng.standard_normal((B, H, d, d)) * 0.1
    ub = lambda x: x.reshape((B, T) + x.shape[1:])
    ob, sb = oracle.layer(ub(r["q_raw"]), ub(r["k_raw"]), ub(r["v_raw"]), *ws, ub(r["g_raw"]), A, None,
                          ub(r["b_raw"]), ub(r["o_gate_raw"]), None, io_bf16=False, s0=s0)
    ov, sv = oracle.layer_varlen(r["q_raw"], r["k_raw"], r["v_raw"], *ws, r["g_raw"], A, None, r["b_raw"],
                                 r["o_gate_raw"], np.arange(B + 1) * T, None, s0=s0, io_bf16=False)
    np.testing.assert_array_equal(ov, ob.reshape(ov.shape))
    np.testing.assert_array_equal(sv, sb)


def test_layer_varlen_conv_does_not_cross_sequences():
    """Changing the last raw tokens of one sequence leaves the next sequence's outputs
    unchanged (its conv history starts from zeros) and changes its own."""
    rng = np.random.default_rng(35)
    H, d = 2, 4
    cu = np.array([0, 5, 11, 11, 14])
    r = _layer_raw(rng, 14, H, d)
    ws = [rng.standard_normal((H * d, 4)) * 0.5 for _ in range(3)]
    A = rng.uniform(0, 1, H)
    o1, _ = oracle.layer_varlen(*(r[n] for n in ("q_raw", "k_raw", "v_raw")), *ws, r["g_raw"], A, None,
                                r["b_raw"], r["o_gate_raw"], cu, io_bf16=False)
    r2 = {n: x.copy() for n, x in r.items()}
    for n in ("q_raw", "k_raw", "v_raw"):
        r2[n][3:5] += 1.0
    o2, _ = oracle.layer_varlen(*(r2[n] for n in ("q_raw", "k_raw", "v_raw")), *ws, r2["g_raw"], A, None,
                                r2["b_raw"], r2["o_gate_raw"], cu, io_bf16=False)
    np.testing.assert_array_equal(o1[5:], o2[5:])
    assert np.max(np.abs(o1[3:5] - o2[3:5])) > 1e-3


def test_layer_conv_is_causal_per_channel():
    """Changing raw inputs at token t changes no layer output before t."""
    rng = np.random.default_rng(26)
    B, T, H, d = 1, 12, 2, 4
    args = [rng.standard_normal((B, T, H * d)) for _ in range(3)]
    ws = [rng.standard_normal((H * d, 4)) * 0.5 for _ in range(3)]
    g_raw = rng.standard_normal((B, T, H, d))
    b_raw = rng.standard_normal((B, T, H))
    z = rng.standard_normal((B, T, H, d))
    A = rng.uniform(0, 1, H)
    out1, _ = oracle.layer(*args, *ws, g_raw, A, None, b_raw, z, None, io_bf16=False)
    args2 = [a.copy() for a in args]
    for a in args2:
        a[:, 6:] += 1.0
    out2, _ = oracle.layer(*args2, *ws, g_raw, A, None, b_raw, z, None, io_bf16=False)
    np.testing.assert_array_equal(out1[:, :6], out2[:, :6])
    assert np.max(np.abs(out1[:, 6:] - out2[:, 6:])) > 1e-3


def test_golden_regression_fixture():
    """The oracle still reproduces the committed fixture written by tests/golden/make_golden.py."""
    import os
    import sys
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    sys.path.insert(0, here)
    from make_golden import tiny_inputs
    vals = np.loadtxt(os.path.join(here, "oracle_tiny.txt"))
    q, k, v, g, beta, s0 = tiny_inputs()
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    np.testing.assert_allclose(o[0, :, 0], vals[:6], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(sT[0, 0], vals[6:], rtol=1e-13, atol=1e-15)
