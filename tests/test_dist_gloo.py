"""Multi-rank calibration host logic on CPU (gloo, world size 2): sharded
statistics combined by all-reduce(MAX) equal the single-process oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from w8a8_post_quantization_calib_b200.dist import allreduce_absmax_, shard_range


def test_shard_range_covers_everything_once():
    for n in (0, 1, 7, 64, 65):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = shard_range(n, r, world)
                seen.extend(range(a, b))
            assert seen == list(range(n))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.qkv_7b(M=8, K=256, N=64, calib_batches=6, calib_rows=32)
        a, b = shard_range(len(wl.calib), rank, world)
        local = np.zeros(wl.K, np.float32)
        for x in wl.calib[a:b]:
            oracle.calib_absmax(x, synth.F16, local)       # this rank's statistic (CPU stand-in)
        t = torch.from_numpy(local.copy())
        allreduce_absmax_(t)
        np.save(os.path.join(out_dir, f"act_max_{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_calibration_equals_single_process(tmp_path):
    import oracle
    import synth
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    wl = synth.qkv_7b(M=8, K=256, N=64, calib_batches=6, calib_rows=32)
    full = np.zeros(wl.K, np.float32)
    for x in wl.calib:
        oracle.calib_absmax(x, synth.F16, full)
    for r in range(world):
        got = np.load(tmp_path / f"act_max_{r}.npy")
        assert np.array_equal(got, full)
    # every rank derives the same smoothing factors as one process would
    wm = oracle.calib_absmax(wl.w, synth.F16)
    assert np.array_equal(oracle.smooth_scales(got, wm, 0.5), oracle.smooth_scales(full, wm, 0.5))
