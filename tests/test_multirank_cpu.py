"""The bench's N > 1 path on CPU: two gloo ranks (127.0.0.1) run the same
reductions the NCCL ranks run on GPUs -- the slowest rank's time, the
sum of all ranks' tokens -- and draw their independent layers (weak scaling:
same shapes, different seeds)."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, ROOT)
        from block_sparse_long_exp_b200 import workloads as W
        B = _bench()
        # rank r ran (r + 1) * 1000 tokens in (r + 1) * 10 ms
        value, ms_max = B.job_rate((rank + 1) * 1000, (rank + 1) * 10.0, torch, dist)
        w = B.rank_workload(W.WORKLOADS["tiny_n4096"], rank, W)
        inp = W.make_inputs(w, "cpu", T_override=256)
        torch.save({"value": value, "ms_max": ms_max, "seed": w.seed, "q": inp["q"][:4].float(),
                    "shape": tuple(inp["q"].shape)}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [torch.load(tmp_path / f"r{i}.pt") for i in range(world)]
    for x in r:
        assert x["ms_max"] == pytest.approx(20.0)
        assert x["value"] == pytest.approx((1000 + 2000) / 0.020)   # whole-job tokens/s
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["shape"] == r[1]["shape"]                          # same layer shape per rank
    assert not torch.equal(r[0]["q"], r[1]["q"])                   # independent inputs
