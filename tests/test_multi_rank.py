"""Replica logic of the multi-GPU benchmark, on CPU with two gloo ranks.

The batch-1 path does not shard: N GPUs run N independent replicas (same weights, their own
inputs) with no collective on the data path; the only collectives are the timing barrier and the
max-over-ranks reduction of the loop time.  These tests run that host logic with real
torch.distributed collectives on CPU.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import oracle
    from synth import config, generate_inputs, generate_weights
    d = config("tiny", n_layers=1, hidden=64, n_q_heads=2, n_kv_heads=1, head_dim=64, inter=64, steps=2)
    w = generate_weights(d, 0)                                   # shared weights
    x = generate_inputs(d, seed=bench.replica_seed(rank))         # this replica's inputs
    act = oracle.denoise_batch(w, x, d)                           # each rank works alone
    local_ms = 1.0 + rank                                         # a per-rank "loop time"
    dist.barrier()
    ms = bench.max_over_ranks(local_ms, world)
    value = bench.job_throughput_gbs(bench.algorithmic_bytes(d), world, ms)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), act=act, ms=ms, value=value,
             noise=x["noise"], bytes=bench.algorithmic_bytes(d))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replicas_are_independent_and_time_is_max_over_ranks(tmp_path, world):
    port = _free_port()
    mp.spawn(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    # every rank agrees on the slowest rank's time and on the whole-job throughput
    for r in res:
        assert float(r["ms"]) == float(world)
        want = world * int(r["bytes"]) / (world * 1e-3) / 1e9
        assert abs(float(r["value"]) - want) < 1e-9
    # replicas draw different inputs and produce their own results
    assert not np.array_equal(res[0]["noise"], res[1]["noise"])
    assert not np.allclose(res[0]["act"], res[1]["act"])


def test_single_rank_needs_no_collective():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput_gbs(10 ** 9, 1, 1.0) == pytest.approx(1000.0)
    assert bench.job_throughput_gbs(10 ** 9, 4, 2.0) == pytest.approx(2000.0)
