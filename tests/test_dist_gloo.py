"""Multi-rank calibration host logic on CPU (gloo, world size 2): sharded
statistics combined by all-reduce(MAX) equal the single-process oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from w8a8_post_quantization_calib_b200.dist import allgather_columns, allreduce_absmax_, column_shard, shard_range


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


def test_column_shard_whole_groups():
    for n in (16, 48, 4096, 12288, 12304):
        for world in (1, 2, 3, 8):
            spans = [column_shard(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a % 16 == 0 and b % 16 == 0 and a <= b for a, b in spans)
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
    with pytest.raises(ValueError):
        column_shard(40, 0, 2)


def _tp_worker(rank, world, port, out_dir):
    """Column-parallel linear on CPU (the oracle stands in for the kernels):
    each rank holds its weight rows, completes max|W_j| with all-reduce(MAX),
    quantises its rows, runs its columns and gathers them."""
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.qkv_7b(M=12, K=128, N=80, calib_batches=4, calib_rows=16)
        act_max = np.zeros(wl.K, np.float32)
        for x in wl.calib:
            oracle.calib_absmax(x, synth.F16, act_max)
        a, b = column_shard(wl.N, rank, world)
        w_rows = wl.w[a:b]
        w_max = torch.from_numpy(oracle.calib_absmax(w_rows, synth.F16).copy())
        allreduce_absmax_(w_max)                             # the column statistic spans every rank's rows
        s = oracle.smooth_scales(act_max, w_max.numpy(), 0.5)
        a_st = oracle.static_scale(act_max, s)
        wq, ws = oracle.quant_weight(w_rows, s, synth.F16)
        xq, _ = oracle.smooth_quant_act(wl.x, s, oracle.STATIC, a_st, synth.F16)
        y = oracle.dequant(oracle.gemm_s32(xq, wq), np.array([a_st], np.float32), oracle.STATIC, ws, synth.F16)
        full = allgather_columns(torch.from_numpy(y.view(np.int16).copy()).view(torch.float16), wl.N)
        np.save(os.path.join(out_dir, f"y_{rank}.npy"), full.view(torch.int16).numpy().view(np.uint16))
    finally:
        dist.destroy_process_group()


def test_two_rank_column_parallel_linear_equals_single_process(tmp_path):
    import oracle
    import synth
    world = 2
    mp.start_processes(_tp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    wl = synth.qkv_7b(M=12, K=128, N=80, calib_batches=4, calib_rows=16)
    st = oracle.calibrate_and_quantize(wl.calib, wl.w, 0.5, synth.F16, synth.F16)
    xq, _ = oracle.smooth_quant_act(wl.x, st.s, oracle.STATIC, st.a_static, synth.F16)
    ref = oracle.dequant(oracle.gemm_s32(xq, st.wq), np.array([st.a_static], np.float32), oracle.STATIC,
                         st.w_scale, synth.F16)
    for r in range(world):
        got = np.load(tmp_path / f"y_{r}.npy")
        assert got.shape == ref.shape and np.array_equal(got, ref)

