"""Run one KDA entry point a few times on a chosen size — a driver for profilers.

    python -m gated_delta_rule_155_b200.profile_case prefill --B 2 --T 4096 --H 96 --launches 3
    python -m gated_delta_rule_155_b200.profile_case decode  --B 64 --H 96 --launches 3
    python -m gated_delta_rule_155_b200.profile_case layer   --B 1 --T 4096 --H 96 --launches 2
    python -m gated_delta_rule_155_b200.profile_case varlen  --T 8192 --H 96 --launches 3
    python -m gated_delta_rule_155_b200.profile_case backward --B 1 --T 1024 --H 148 --launches 2
    python -m gated_delta_rule_155_b200.profile_case layer_decode --B 64 --H 96 --launches 3

Inputs come from the seeded generators; nothing is checked or timed here (use the
tests for parity and bench.py for timing).  Sizes should keep the inputs larger than
L2 (126 MB) so DRAM counters mean something, but small enough for a profiler's
per-kernel replay.
"""
from __future__ import annotations

import argparse

import torch


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("kind", choices=["prefill", "decode", "layer", "varlen", "backward", "layer_decode"])
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--H", type=int, default=96)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args(argv)

    from gated_delta_rule_155_b200 import build, inputs
    build.build()
    from gated_delta_rule_155_b200 import kda

    dev = torch.device("cuda", 0)
    if a.kind == "prefill":
        d = inputs.prefill_inputs(a.B, a.T, a.H, a.d, a.d, io="bf16", seed=2)
        args = [d[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
        out = torch.empty_like(args[2])
        sT = torch.empty((a.B, a.H, a.d, a.d), device=dev)
        for _ in range(a.launches):
            kda.kda_forward_chunked(*args, None, out, sT)
    elif a.kind == "decode":
        dd = inputs.decode_inputs(a.B, a.H, a.d, a.d, steps=1, seed=3)
        st = dd["state"].to(dev)
        x = {n: dd["steps"][0][n].to(dev) for n in ("q", "k", "v", "g", "beta")}
        for _ in range(a.launches):
            kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], st)
    elif a.kind == "varlen":
        # packed sequences of 1..4096 tokens, a.T tokens in all (the packed workload's law)
        lens = inputs.packed_lengths(a.T, 4096, 5)
        dl = inputs.varlen_inputs(lens, a.H, a.d, a.d, io="bf16", seed=5)
        x = [dl[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
        cu = dl["cu_seqlens"].to(dev)
        sT = torch.empty((len(lens), a.H, a.d, a.d), device=dev)
        for _ in range(a.launches):
            kda.kda_forward_chunked_varlen(*x, cu, None, None, sT)
    elif a.kind == "layer_decode":
        # one new token per sequence through the whole layer, conv caches and state in place
        L = inputs.layer_inputs(a.B, 1, a.H, a.d, a.d, io="bf16", seed=3, conv_std=0.5, s0_std=0.02)
        to = lambda t: None if t is None else t.contiguous().to(dev)
        st = to(L["s0"])
        caches = [torch.zeros((a.B, 3, a.H * a.d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
        x = {n: to(L[n][:, 0]) for n in ("q_raw", "k_raw", "v_raw", "g_raw", "b_raw", "o_gate_raw")}
        for _ in range(a.launches):
            kda.kda_layer_decode_step(x["q_raw"], x["k_raw"], x["v_raw"], to(L["conv_q"]), to(L["conv_k"]),
                                      to(L["conv_v"]), *caches, x["g_raw"], to(L["A_log"]), to(L["dt_bias"]),
                                      x["b_raw"], x["o_gate_raw"], st, to(L["o_norm_w"]))
    elif a.kind == "backward":
        d = inputs.prefill_inputs(a.B, a.T, a.H, a.d, a.d, io="bf16", seed=2)
        x = [d[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
        dO = torch.randn(x[2].shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).to(dev)
        for _ in range(a.launches):
            kda.kda_backward_chunked(*x, dO)
    else:
        L = inputs.layer_inputs(a.B, a.T, a.H, a.d, a.d, io="bf16", seed=4)
        to = lambda t: None if t is None else t.to(dev)
        args = [to(L[n]) for n in ("q_raw", "k_raw", "v_raw", "conv_q", "conv_k", "conv_v", "g_raw",
                                   "A_log", "dt_bias", "b_raw", "o_gate_raw", "o_norm_w")]
        sT = torch.empty((a.B, a.H, a.d, a.d), device=dev)
        for _ in range(a.launches):
            kda.kda_layer_forward(*args, final_state=sT)
    kda.kda_check_device_error()
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main()
