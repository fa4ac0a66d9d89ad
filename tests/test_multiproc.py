"""Two-rank runs on CPU (gloo): the one exchange of sharded calibration and
the benchmark's max-over-ranks timing."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _calib_rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import oracle
        from w8a8_post_quantization_sq_b200 import sharded
        import bench

        g = torch.Generator().manual_seed(5)
        X = torch.randn((5 * 37, 96), generator=g)
        X[:, 11] *= 80
        X[3, 50] = -400.0    # the column's extreme sits in batch 0 (rank 0's shard) ...
        X[40, 51] = 800.0    # ... and this one in batch 1 (rank 1's)
        batches = [X[i * 37:(i + 1) * 37] for i in range(5)]  # 5 batches: the ranks' shards differ in size
        seen = []

        def update(b, m):  # the oracle's running maxima stand in for the CUDA call on CPU ranks
            seen.append(next(i for i, c in enumerate(batches) if c is b))
            m.copy_(torch.from_numpy(oracle.col_absmax(b.numpy(), m.numpy())))

        local = sharded.calibrate_sharded(batches, torch.zeros(96), update)
        full = oracle.col_absmax(X.numpy())
        ok_calib = bool(np.array_equal(local.numpy(), full)) and seen == list(range(rank, 5, world))
        # the benchmark's timing: the max over the ranks of each rank's own time
        t = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
        out[rank] = (ok_calib, t)
    finally:
        dist.destroy_process_group()


def test_sharded_calibration_and_max_over_ranks():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_calib_rank, args=(world, port, out), nprocs=world, join=True)
    assert all(out[r][0] for r in range(world)), "sharded maxima differ from the maxima of all tokens"
    assert [out[r][1] for r in range(world)] == [2.5, 2.5]


def test_reference_arm_under_torchrun():
    """`bench.py --impl reference` launched by torchrun with two ranks:
    rank 0 prints one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def _calib_rank_cuda(rank, world, port, out):
    """The same exchange with each rank's maxima from the library's CUDA
    column absmax over its shard (both ranks on the one visible GPU: the
    kernels are independent launches that wait on nothing)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import oracle
        import w8a8_post_quantization_sq_b200 as sq
        from w8a8_post_quantization_sq_b200 import inputs, sharded

        d = inputs.c5_175b(device="cpu", M=64, n_calib=4, w_frac=1 / 4096)
        batches = d["calib"]  # bf16 [64, 12288] each, 8 channels x100
        xmax = torch.zeros(12288, device="cuda")
        sharded.calibrate_sharded(batches, xmax, lambda b, m: sq.sq_calib_absmax(b.cuda(), m))
        local = xmax.cpu()
        full = np.zeros(12288, np.float32)
        for b in batches:
            full = oracle.col_absmax(b, full)
        out[rank] = bool(np.array_equal(local.numpy(), full))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_sharded_calibration_with_cuda_maxima():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_calib_rank_cuda, args=(world, port, out), nprocs=world, join=True)
    assert all(out[r] for r in range(world)), "sharded CUDA maxima differ from the oracle's maxima of all tokens"


def test_shard_assignment():
    """Batch i goes to rank i mod world; the shards partition the batches."""
    from w8a8_post_quantization_sq_b200 import sharded

    for n, world in [(16, 1), (16, 2), (5, 2), (7, 3), (2, 4)]:
        shards = [list(sharded.shard(n, r, world)) for r in range(world)]
        assert sorted(i for s in shards for i in s) == list(range(n))
        assert all(i % world == r for r, s in enumerate(shards) for i in s)
    with pytest.raises(ValueError):
        sharded.shard(4, 2, 2)
