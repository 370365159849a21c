"""Multi-rank host logic on CPU with the gloo backend (world size 2).

The layer shards over tokens with no exchange: every rank holds all the
experts and runs its own tokens (replicas).  These tests check, on the CPU,
that (1) splitting a batch across ranks gives exactly the rows of the
unsplit batch (the oracle run per shard and gathered equals the oracle on
the whole batch), and (2) the benchmark's timing reduction takes the max
over ranks and its throughput counts every rank's tokens."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        import synth
        # (2) timing reduction and job throughput
        m = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        tps = bench.job_tokens_per_s(world, 4096, 10, m)
        # (1) token-sharded replicas: rank r takes rows [r*T/world, (r+1)*T/world) of one batch
        s = synth.MoEShape("mr", 64, 64, 128, 8, 2, "f32")
        per = s.T // world
        w = synth.host_inputs(s, seed=5, with_x=False)
        x_shard = synth.normal_values(5, synth.tensor_id(synth.TENSOR_X), per * s.d, 1.0, "f32",
                                      start=rank * per * s.d).reshape(per, s.d)
        y, idx, _ = oracle.moe_forward(x_shard, w["Wg"], w["W1"], w["W3"], w["W2"], s.k)
        ys = [torch.zeros(per, s.d, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(ys, torch.from_numpy(y))          # test-side gather, not part of the layer
        ids = [torch.zeros(per, s.k, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(ids, torch.from_numpy(idx))
        if rank == 0:
            np.save(os.path.join(out_dir, "y.npy"), torch.cat(ys).numpy())
            np.save(os.path.join(out_dir, "idx.npy"), torch.cat(ids).numpy())
            np.save(os.path.join(out_dir, "timing.npy"), np.array([m, tps]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_token_sharded_replicas_and_timing(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle
    import synth
    s = synth.MoEShape("mr", 64, 64, 128, 8, 2, "f32")
    t = synth.host_inputs(s, seed=5)
    y_full, idx_full, _ = oracle.moe_forward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k)
    np.testing.assert_array_equal(np.load(tmp_path / "idx.npy"), idx_full)
    np.testing.assert_allclose(np.load(tmp_path / "y.npy"), y_full, rtol=1e-13, atol=1e-15)
    m, tps = np.load(tmp_path / "timing.npy")
    assert m == 15.0                                  # max over ranks (10 and 15 ms)
    assert tps == pytest.approx(2 * 4096 * 10 / 15e-3)
