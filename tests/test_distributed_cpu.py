"""Host logic of the multi-GPU bench path, run as 2 gloo ranks on the CPU, and
the bench's FLOP count against the oracle's count of allowed pairs."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        mx = bench.max_over_ranks(10.0 + rank, world, dev)
        sm = bench.sum_over_ranks(1.5 * (rank + 1), world, dev)
        bench.barrier(world)
        out[rank] = (mx, sm)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        assert out[r] == (11.0, 4.5)  # max over ranks of the time, sum of the work


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.sum_over_ranks(3.0, 1, None) == 3.0


@pytest.mark.parametrize("name", ["tiny", "t2i", "edit3", "maxref", "hires", "orig"])
def test_bench_flops_match_oracle_pair_count(name):
    cfg = W.WORKLOADS[name]
    L, P, T = W.sizes(name)
    orig = cfg.get("original", False)
    _, kv_end = (O.positions_original if orig else O.positions)(cfg["segments"])
    full, cached = bench.step_flops(name)
    bh = cfg["B"] * cfg["H"]
    assert full == 4 * 128 * O.allowed_pairs(kv_end) * bh
    assert cached == (0 if orig else 4 * 128 * T * (P + T) * bh)


def _worker_one_leaves(rank, world, port, out):
    """Rank 1 leaves between steps (no collective in flight); rank 0's next
    collective must end with an error within the short timeout, not hang."""
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    dev = torch.device("cpu")
    bench.max_over_ranks(1.0, world, dev)  # one good step together
    if rank == 1:
        out[rank] = "left"
        os._exit(0)
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(2.0, world, dev)
        out[rank] = "no error"
    except Exception:
        out[rank] = "error after %.1f s" % (time.monotonic() - t0)
    os._exit(0)


def test_rank_that_leaves_is_detected_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker_one_leaves, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    assert out[1] == "left"
    assert out[0].startswith("error after"), out[0]
    assert float(out[0].split()[2]) < 30.0
