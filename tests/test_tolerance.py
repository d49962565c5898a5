"""The rounding floors behind the bf16 tolerance readings (CPU, fp64 arithmetic only).

Final state.  A tensor-core state update multiplies U by K~ = k exp(G_C - G), which enters
the MMA in bf16.  The first test builds the final states of a packed batch of 200 sequences
of 0..20 tokens exactly (checked against the oracle), then with K~ rounded once to bf16, and
then with K~ split into a bf16 hi part plus a bf16 residual.  One rounding already exceeds
2e-2 of the batch's state RMS (the states are a few nearly rank-one updates whose largest
elements reach ~10x the RMS); the hi + lo pair stays far inside that RMS-only bound.  So the
final state keeps the plain bound, and the kernel feeds K~ as a hi + lo pair.

Outputs.  Storing exact outputs in bf16 alone exceeds 2e-2 of their RMS, which is why the
output bound carries the format's own rounding term.
"""
import numpy as np
import torch

import oracle
from gated_delta_rule_155_b200 import inputs


def _bf16(x):
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


def _hi_lo(x):
    hi = _bf16(x)
    return hi + _bf16(x - hi)


def test_the_state_update_operand_needs_a_hi_lo_pair_for_the_rms_bound():
    lens = [int(x) for x in np.random.default_rng(91).integers(0, 21, 200)]
    d = inputs.varlen_inputs(lens, 2, 128, 128, io="bf16", seed=92, s0_std=0.05)
    q, k, v, g, b = (d[n].double().numpy() for n in ("q", "k", "v", "g", "beta"))
    s0 = d["s0"].double().numpy()
    cu = d["cu_seqlens"].numpy()
    _, ref = oracle.recurrent_varlen(q, k, v, g, b, cu, s0)
    exact = np.zeros_like(ref)
    rounded = np.zeros_like(ref)
    split = np.zeros_like(ref)
    for n in range(len(lens)):
        lo, hi = int(cu[n]), int(cu[n + 1])
        for h in range(2):
            # the token recurrence gives u_t and the in-sequence cumulative log-decays
            S = s0[n, h].copy()
            us, Gs, G = [], [], np.zeros(128)
            for t in range(lo, hi):
                S = np.exp(g[t, h])[:, None] * S
                u = b[t, h] * (v[t, h] - S.T @ k[t, h])
                S = S + np.outer(k[t, h], u)
                G = G + g[t, h]
                us.append(u)
                Gs.append(G.copy())
            # S_T = Diag(exp G_C) S_0 + sum_t K~_t u_t^T, with K~ exact or rounded once
            Se = np.exp(G)[:, None] * s0[n, h]
            Sr, Ss = Se.copy(), Se.copy()
            for u, Gt, t in zip(us, Gs, range(lo, hi)):
                kt = k[t, h] * np.exp(G - Gt)
                Se += np.outer(kt, u)
                Sr += np.outer(_bf16(kt), u)
                Ss += np.outer(_hi_lo(kt), u)
            exact[n, h], rounded[n, h], split[n, h] = Se, Sr, Ss
    assert np.max(np.abs(exact - ref)) <= 1e-12 * np.max(np.abs(ref))
    rms = np.sqrt(np.mean(ref * ref))
    assert np.abs(rounded - ref).max() / (2e-2 * rms) > 1.2     # one rounding: the RMS bound fails
    assert np.abs(split - ref).max() / (2e-2 * rms) < 0.01      # hi + lo: far inside it


def test_storing_exact_outputs_in_bf16_needs_the_output_rounding_term():
    """The exact fp64 outputs of 8 heads of the T = 4096 bf16 workload, merely rounded to
    bf16 (what any bf16-output kernel must store), sit 1.9x above 2e-2 of the output RMS —
    the outputs reach 17x their RMS — and within the bound once each element may be one bf16
    rounding away, the term the output bound carries."""
    d = inputs.prefill_inputs(1, 4096, 8, 128, 128, io="bf16", seed=1, s0_std=0.02)
    o, _ = oracle.recurrent(*(d[n].double().numpy() for n in ("q", "k", "v", "g", "beta")),
                            d["s0"].double().numpy())
    err = np.abs(_bf16(o) - o)
    rms = np.sqrt(np.mean(o * o))
    assert err.max() / (2e-2 * rms) > 1.5
    assert np.max(err / (2e-2 * rms + 2.0 ** -8 * np.abs(o))) < 0.8
