"""Query-range sharding of one sequence's prefill (block_sparse_long_exp_b200/
shard.py).  The planner's ranges cover every query once and balance the
algorithmic work.  On two gloo ranks, each rank's chunked-prefill oracle result
(queries [a, b) over keys [0, b)), gathered on rank 0, equals the unsharded
oracle result row for row.  For the backward of the split, on two and on three
ranks, sum_key_grads sums each rank's key-side gradients (dk, dv, the KL
target's dk_idx); with the query-side ones (dq, dq_idx) gathered, they equal
the unsharded backward oracles.  Split by GQA group on two and four ranks,
every rank's selection equals its groups' columns of the unsharded one, and
the outputs gathered over the heads equal the unsharded output."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_exp_b200 import roofline as R
from block_sparse_long_exp_b200 import shard as SH


def test_ranges_cover_and_balance():
    H, G, d, d_idx, B_k, k = 64, 4, 128, 64, 128, 16
    S = 131072
    work = SH.query_work(S, H, G, d, d_idx, B_k, k)
    # the per-query work sums to the layer's algorithmic FLOPs
    w = R.prefill_work([S], [S], H, G, d, d_idx, B_k, k)
    assert work.sum() == pytest.approx(w["flops"], rel=1e-12)
    for world in (1, 2, 3, 8):
        ranges = SH.split_query_ranges(work, world, align=128)
        assert ranges[0][0] == 0 and ranges[-1][1] == S
        assert all(a <= b for a, b in ranges) and all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
        assert all(a % 128 == 0 for a, _ in ranges)
        assert SH.imbalance(work, ranges) < 1.01
        if world > 1:   # equal row counts would be far worse: the index work grows with position
            even = [(r * S // world, (r + 1) * S // world) for r in range(world)]
            assert SH.imbalance(work, even) > SH.imbalance(work, ranges) + 0.1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_long_exp_b200 import workloads as W
        from oracle import msa_oracle as O
        w = W.Workload("shard", "prefill", H=8, G=2, d=16, d_idx=8, B_k=4, k=3, seed=5, hot_frac=0.1)
        inp = W.make_inputs(w, "cpu", lengths=[61])
        work = SH.query_work(61, w.H, w.G, w.d, w.d_idx, w.B_k, w.k)
        a, b = SH.split_query_ranges(work, world)[rank]
        c = SH.chunk_of(inp, a, b)
        f = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
        sel = O.index_topk(f(c["q_idx"]), f(c["k_idx"]), c["cu_q_host"], c["cu_k_host"], w.k, w.B_k)
        o, lse = O.msa_forward_rows(f(c["q"]), f(c["k"]), f(c["v"]), sel, c["cu_q_host"], c["cu_k_host"],
                                    list(range(b - a)), w.B_k, w.sm_scale)
        parts = [None] * world
        dist.all_gather_object(parts, (a, b, sel, o, lse))
        if rank == 0:
            full_sel = O.index_topk(f(inp["q_idx"]), f(inp["k_idx"]), [0, 61], [0, 61], w.k, w.B_k)
            full_o, full_l = O.msa_forward_rows(f(inp["q"]), f(inp["k"]), f(inp["v"]), full_sel, [0, 61], [0, 61],
                                                list(range(61)), w.B_k, w.sm_scale)
            ok = sorted(p[:2] for p in parts) == sorted(SH.split_query_ranges(work, world))
            for a_, b_, s_, o_, l_ in parts:
                ok = ok and np.array_equal(s_, full_sel[a_:b_])
                ok = ok and np.allclose(o_, full_o[a_:b_], rtol=0, atol=1e-12)
                ok = ok and np.allclose(l_, full_l[a_:b_], rtol=0, atol=1e-12)
            result.put(bool(ok))
    finally:
        dist.destroy_process_group()


def test_sharded_oracle_equals_unsharded_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, result)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    assert result.get(timeout=10) is True


def _rank_bwd(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_long_exp_b200 import workloads as W
        from oracle import index_kl as K
        from oracle import main_backward as B
        from oracle import msa_oracle as O
        w = W.Workload("shard_bwd", "prefill", H=8, G=2, d=16, d_idx=8, B_k=4, k=3, seed=7, hot_frac=0.1)
        S, tau = 61, 0.5
        inp = W.make_inputs(w, "cpu", lengths=[S])
        dout = torch.randn(inp["q"].shape, generator=torch.Generator().manual_seed(8), dtype=torch.float64)
        work = SH.query_work(S, w.H, w.G, w.d, w.d_idx, w.B_k, w.k)
        a, b = SH.split_query_ranges(work, world)[rank]
        c = SH.chunk_of(inp, a, b)
        f = lambda t: t.double().numpy()  # noqa: E731
        cq, ck = c["cu_q_host"], c["cu_k_host"]
        sel = O.index_topk(f(c["q_idx"]), f(c["k_idx"]), cq, ck, w.k, w.B_k)
        dq, dk, dv = B.main_branch_backward(f(c["q"]), f(c["k"]), f(c["v"]), sel, dout[a:b].numpy(), cq, ck,
                                            w.B_k, w.sm_scale)
        loss, dqi, dki = K.index_kl_loss_and_grad(f(c["q"]), f(c["k"]), f(c["q_idx"]), f(c["k_idx"]), sel, cq, ck,
                                                  w.B_k, w.sm_scale, tau)
        assert dk.shape[0] == b and dki.shape[0] == b
        loss_t = torch.tensor([loss], dtype=torch.float64)
        dist.all_reduce(loss_t)
        sk, sv, ski = SH.sum_key_grads([torch.from_numpy(dk), torch.from_numpy(dv), torch.from_numpy(dki)], S)
        parts = [None] * world
        dist.all_gather_object(parts, (a, b, dq, dqi))
        if rank == 0:
            fi = {k_: f(inp[k_]) for k_ in ("q", "k", "v", "q_idx", "k_idx")}
            full_sel = O.index_topk(fi["q_idx"], fi["k_idx"], [0, S], [0, S], w.k, w.B_k)
            w_dq, w_dk, w_dv = B.main_branch_backward(fi["q"], fi["k"], fi["v"], full_sel, dout.numpy(), [0, S],
                                                      [0, S], w.B_k, w.sm_scale)
            w_loss, w_dqi, w_dki = K.index_kl_loss_and_grad(fi["q"], fi["k"], fi["q_idx"], fi["k_idx"], full_sel,
                                                            [0, S], [0, S], w.B_k, w.sm_scale, tau)
            close = lambda x, y: np.allclose(x, y, rtol=0, atol=1e-12 * max(1.0, np.abs(y).max()))  # noqa: E731
            ok = all(close(x.numpy(), y) for x, y in ((sk, w_dk), (sv, w_dv), (ski, w_dki)))
            ok = ok and abs(float(loss_t[0]) - w_loss) <= 1e-12 * max(1.0, abs(w_loss))
            for a_, b_, dq_, dqi_ in parts:
                ok = ok and close(dq_, w_dq[a_:b_]) and close(dqi_, w_dqi[a_:b_])
            # the exchange is needed: the later rank's queries reach rank 0's key rows too
            ok = ok and not np.allclose(dk, w_dk[:b]) and not np.allclose(dki, w_dki[:b])
            result.put(bool(ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_backward_sums_key_grads_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_bwd, args=(r, world, port, result)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    assert result.get(timeout=10) is True


def _rank_groups(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_long_exp_b200 import workloads as W
        from oracle import msa_oracle as O
        w = W.Workload("shard_groups", "prefill", H=8, G=4, d=16, d_idx=8, B_k=4, k=3, seed=9, hot_frac=0.1)
        inp = W.make_inputs(w, "cpu", lengths=[45, 30])
        cq, ck = inp["cu_q_host"], inp["cu_k_host"]
        f = lambda t: t.double().numpy()  # noqa: E731
        g0, g1 = SH.split_groups(w.G, world)[rank]
        part = SH.group_slice(inp, w.H, w.G, g0, g1)
        assert part["q"].shape[1] == w.H * (g1 - g0) // w.G and part["k_idx"] is inp["k_idx"]
        sel = O.index_topk(f(part["q_idx"]), f(part["k_idx"]), cq, ck, w.k, w.B_k)
        o, lse = O.msa_forward_rows(f(part["q"]), f(part["k"]), f(part["v"]), sel, cq, ck, list(range(cq[-1])),
                                    w.B_k, w.sm_scale)
        full_o = SH.gather_heads(torch.from_numpy(o))
        full_l = SH.gather_heads(torch.from_numpy(lse)[:, :, None])[:, :, 0]
        sels = [None] * world
        dist.all_gather_object(sels, (g0, g1, sel))
        if rank == 0:
            want_sel = O.index_topk(f(inp["q_idx"]), f(inp["k_idx"]), cq, ck, w.k, w.B_k)
            want_o, want_l = O.msa_forward_rows(f(inp["q"]), f(inp["k"]), f(inp["v"]), want_sel, cq, ck,
                                                list(range(cq[-1])), w.B_k, w.sm_scale)
            ok = all(np.array_equal(s_, want_sel[:, a_:b_]) for a_, b_, s_ in sels)
            ok = ok and np.allclose(full_o.numpy(), want_o, rtol=0, atol=1e-12)
            ok = ok and np.allclose(full_l.numpy(), want_l, rtol=0, atol=1e-12)
            result.put(bool(ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_group_sharded_oracle_equals_unsharded_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_groups, args=(r, world, port, result)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    assert result.get(timeout=10) is True


def test_split_groups():
    assert SH.split_groups(4, 1) == [(0, 4)]
    assert SH.split_groups(4, 2) == [(0, 2), (2, 4)]
    assert SH.split_groups(4, 4) == [(0, 1), (1, 2), (2, 3), (3, 4)]
    for bad in (3, 8, 0):
        with pytest.raises(ValueError):
            SH.split_groups(4, bad)


def test_sum_key_grads_without_a_group_pads():
    g = torch.arange(6, dtype=torch.float32).reshape(3, 2)
    (out,) = SH.sum_key_grads([g], 5)
    assert out.shape == (5, 2) and torch.equal(out[:3], g) and not out[3:].any()
    with pytest.raises(ValueError):
        SH.sum_key_grads([torch.zeros(6, 2)], 5)


def test_decode_shards_cover_and_balance():
    from block_sparse_long_exp_b200 import workloads as W
    w = W.WORKLOADS["decode_b32_l128k_1m_hot2"]
    L = W.seq_lengths(w, torch.Generator().manual_seed(w.seed))
    for world in (1, 2, 4, 8):
        parts = SH.decode_shards(L, world)
        assert sorted(i for p in parts for i in p) == list(range(len(L)))
        loads = [sum(L[i] for i in p) for p in parts]
        # longest-first greedy: no rank exceeds the mean by more than the longest cache
        assert max(loads) <= sum(loads) / world + max(L)
        assert max(loads) / (sum(loads) / world) < 1.2
