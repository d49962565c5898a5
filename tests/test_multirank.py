"""Multi-rank host logic on CPU (gloo, world size 2) — no GPU.

The KDA path shards without any data-path collective: heads are independent, so
ranks split the head list (or run replicas of a batch) and only a barrier and a
max-reduction of timings cross ranks.  These tests run two gloo ranks that each
compute their shard of a small problem with the fp64 oracle and check that the
shards reassemble into the single-process result, and that the timing reduction
and aggregate-throughput arithmetic the benchmark uses behave.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_155_b200.dist_util import aggregate_rate, max_over_ranks, shard_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_range_tiles_exactly():
    for n in (0, 1, 5, 96, 384, 1001):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                lo, hi = shard_range(n, r, world)
                assert hi - lo in (n // world, n // world + 1)
                seen.extend(range(lo, hi))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_aggregate_rate():
    assert aggregate_rate(32768, 1000.0, 1) == pytest.approx(32768.0)
    assert aggregate_rate(32768, 500.0, 4) == pytest.approx(4 * 65536.0)


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from gated_delta_rule_155_b200 import inputs

    d = inputs.prefill_inputs(2, 40, 3, 16, 8, io="f32", seed=5, s0_std=0.1)
    f = lambda t: t.double().numpy()
    q, k, v, g, beta, s0 = (f(d[n]) for n in ("q", "k", "v", "g", "beta", "s0"))
    heads = [(b, h) for b in range(2) for h in range(3)]
    lo, hi = shard_range(len(heads), rank, world)
    mine = heads[lo:hi]
    outs, states = [], []
    for b, h in mine:
        o, s = oracle.recurrent(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1],
                                g[b:b + 1, :, h:h + 1], beta[b:b + 1, :, h:h + 1], s0[b:b + 1, h:h + 1])
        outs.append(o[0, :, 0])
        states.append(s[0, 0])
    np.savez(os.path.join(outdir, f"rank{rank}.npz"), heads=np.array(mine), o=np.array(outs),
             s=np.array(states))
    # timing reduction: the reported time is the slowest rank's
    t = max_over_ranks(10.0 + rank, dist)
    dist.barrier()
    np.save(os.path.join(outdir, f"t{rank}.npy"), np.array([t]))
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_heads_and_reduce_time():
    world = 2
    with tempfile.TemporaryDirectory() as tmp:
        mp.start_processes(_worker, args=(world, _free_port(), tmp), nprocs=world, start_method="spawn",
                           join=True)
        import oracle
        from gated_delta_rule_155_b200 import inputs

        d = inputs.prefill_inputs(2, 40, 3, 16, 8, io="f32", seed=5, s0_std=0.1)
        f = lambda t: t.double().numpy()
        o_all, s_all = oracle.recurrent(*(f(d[n]) for n in ("q", "k", "v", "g", "beta", "s0")))
        covered = set()
        for r in range(world):
            z = np.load(os.path.join(tmp, f"rank{r}.npz"))
            for (b, h), o, s in zip(z["heads"], z["o"], z["s"]):
                np.testing.assert_array_equal(o, o_all[b, :, h])
                np.testing.assert_array_equal(s, s_all[b, h])
                covered.add((int(b), int(h)))
            assert np.load(os.path.join(tmp, f"t{r}.npy"))[0] == 11.0
        assert covered == {(b, h) for b in range(2) for h in range(3)}
