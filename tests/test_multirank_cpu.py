"""The N > 1 path of bench.py on CPU: two gloo ranks, each scanning its own batch
(replicas sharded by batch, no collective on the data path).  The per-rank scan
here is the CPU oracle on a tiny shape; the checks are the host logic around
it: distinct per-rank inputs, the max-over-ranks time and the whole-job value."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from linear_attention_sequence_shortconv_b200 import synth
    from oracle import prism_seq

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.Workload("tiny_bf16", B=2, T=40, H=2, d_k=16, d_v=16, L=3, chunk=16)
        wr = bench.rank_workload(w, rank)
        inp = synth.make_inputs(wr)
        x = synth.to_float64_numpy(inp)
        o, _ = prism_seq(**x)
        local_ms = 10.0 * (rank + 1)          # a stand-in per-rank time: rank 1 is the slowest
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.aggregate_throughput(w.B * w.T, world, ms)
        np.save(os.path.join(out_dir, f"o_{rank}.npy"), o)
        np.save(os.path.join(out_dir, f"res_{rank}.npy"), np.array([ms, value]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    o0, o1 = np.load(tmp_path / "o_0.npy"), np.load(tmp_path / "o_1.npy")
    assert o0.shape == o1.shape and not np.allclose(o0, o1)   # each rank scanned its own batch
    r0, r1 = np.load(tmp_path / "res_0.npy"), np.load(tmp_path / "res_1.npy")
    assert r0[0] == r1[0] == pytest.approx(20.0)               # max over ranks
    assert r0[1] == pytest.approx(2 * 2 * 40 / 0.020)          # all ranks' tokens / slowest time


def test_aggregate_and_workload_helpers():
    import bench
    from linear_attention_sequence_shortconv_b200 import synth

    w = synth.WORKLOADS["lm_130m"]
    assert bench.rank_workload(w, 3).seed == w.seed + 3
    assert bench.rank_workload(w, 3).B == w.B
    assert bench.aggregate_throughput(32768, 8, 0.5) == pytest.approx(8 * 32768 / 5e-4)
    work = bench.algorithmic_work(w)
    assert work["bytes"] == 513540096 and work["flops"] == 93415538688 and work["tokens"] == 32768
