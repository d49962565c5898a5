"""kda_layer_forward_noalloc — the layer forward for callers that cannot allocate.

Some callers must not allocate device memory on their call path (a serving loop whose
memory is planned once at start-up, a plugin or callback interface that hands over no
allocator, latency-critical code that cannot pay for cudaMalloc's possible device-wide
synchronisation).  For them the library offers a variant of the layer forward whose
intermediate buffers live in a fixed device array owned by the library.  These tests
call it through the C ABI and check it against kda_layer_forward (which uses a caller
workspace) on two calls in a row with different inputs and sizes — the shared scratch
keeps the previous call's contents, and the second, smaller call places its buffers at
other offsets over that stale data, so it must not depend on it.  Both entry points run
the same kernels on the same inputs, so the results must be identical bit for bit.  The
tests also check that sizes beyond the built-in scratch are refused before anything runs.

This file is named to be collected last.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_155_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_155_b200 import build

    build.build()
    from gated_delta_rule_155_b200 import kda as k

    return k


def _args(d, dev):
    to = lambda x: None if x is None else x.to(dev)
    return [to(d[n]) for n in ("q_raw", "k_raw", "v_raw", "conv_q", "conv_k", "conv_v", "g_raw",
                               "A_log", "dt_bias", "b_raw", "o_gate_raw", "o_norm_w")], to(d["s0"])


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_noalloc_matches_layer_forward_on_two_calls(kda, io):
    dev = "cuda"
    ioname = "bf16" if io == torch.bfloat16 else "f32"
    d_ = 128
    # a larger call, then a smaller one whose scratch regions start at other offsets
    for call, (B, T, H, seed) in enumerate(((2, 150, 4, 71), (1, 97, 3, 72))):
        d = inputs.layer_inputs(B, T, H, d_, d_, io=ioname, seed=seed, s0_std=0.05, dt_bias_std=0.4,
                                gain_std=0.2)
        args, s0 = _args(d, dev)
        ref_s = torch.empty((B, H, d_, d_), device=dev)
        ref, _ = kda.kda_layer_forward(*args, initial_state=s0, final_state=ref_s)
        out = torch.empty_like(ref)
        st = torch.empty_like(ref_s)
        kda.kda_layer_forward_noalloc(*args, initial_state=s0, out=out, final_state=st)
        kda.kda_check_device_error()
        assert torch.equal(out, ref), f"output differs on call {call}"
        assert torch.equal(st, ref_s), f"final state differs on call {call}"


def test_noalloc_rejects_sizes_beyond_its_scratch(kda):
    lib = kda.library()
    # fp32 I/O runs through the workspace; this size needs far more than the built-in scratch
    need = kda.kda_layer_workspace_size(4, 8192, 96, 128, 128, torch.float32)
    assert need > kda.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x100000)   # never dereferenced: the call is refused before any launch
    st = lib.kda_layer_forward_noalloc(*([fake] * 8), None, ctypes.c_float(float("-inf")), fake, fake, None,
                                       ctypes.c_float(1e-6),
                                       None, fake, None, 4, 8192, 96, 128, 128, 0, None)
    assert st == 6  # KDA_ERR_WORKSPACE
