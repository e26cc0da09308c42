"""Decode of long sequences split across ranks by key range (block_sparse_long_exp_b200/shard.py:
split_key_blocks, key_slice, gather_candidates, gather_rank_outputs, rank_partials), on two
and four gloo ranks with the fp64 oracle in the library's place.  Each rank scores only the
blocks of its own key range and keeps their first k-1 (the oracle's block_candidates); the
candidates are all-gathered and merged (merge_block_candidates); the merged selection must
equal the unsharded oracle selection bit for bit on every rank.  Each rank attends its own
selected blocks; the outputs, all-gathered and merged by log-sum-exp, must equal the
unsharded oracle output (fp64: 1e-12; through rank_partials' f16 layout for the library's
combine: 2e-3).  Without the candidate all-gather the selection differs."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_exp_b200 import shard as SH


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_split_key_blocks_cover():
    for L, world, B_k in ((1000, 3, 128), (1025, 2, 64), (4096, 4, 32), (129, 2, 128)):
        r = SH.split_key_blocks(L, world, B_k)
        nb = -(-L // B_k)
        assert r[0][0] == 0 and r[-1][1] == nb and all(a < b for a, b in r)
        assert all(r[i][1] == r[i + 1][0] for i in range(world - 1))
        assert r[-1][0] <= (L - 1) // B_k < r[-1][1]           # the last rank holds the query's block
    with pytest.raises(ValueError):
        SH.split_key_blocks(100, 2, 128)


def _rank_keysplit(rank, world, port, with_gather, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_long_exp_b200 import workloads as W
        from oracle import msa_oracle as O
        w = W.Workload("keysplit", "decode", H=8, G=2, d=16, d_idx=8, B_k=4, k=4, seed=11, hot_frac=0.1)
        lengths = [61, 45, 33]
        inp = W.make_inputs(w, "cpu", lengths=lengths)
        f = lambda t: t.double().numpy()  # noqa: E731
        B, G, Hg, kc = len(lengths), w.G, w.H // w.G, w.k - 1
        part = SH.key_slice(inp, lengths, rank, world, w.B_k)
        ck = part["cu_k_host"]
        ids = torch.full((B, G, kc), -1, dtype=torch.int32)
        scs = torch.full((B, G, kc), float("-inf"), dtype=torch.float64)
        qi, ki = f(inp["q_idx"]), f(part["k_idx"])
        for b in range(B):
            s_all = ki[ck[b]:ck[b + 1]] @ qi[b].T                    # [keys of the range, G]
            for g in range(G):
                S = O.block_max_pool(s_all[:, g], w.B_k)
                if not part["all_blocks"]:
                    S = S[:-1]                                       # the query's own block competes for nothing
                ci, cs = O.block_candidates(S, w.k)
                ids[b, g, :len(ci)] = torch.tensor(ci, dtype=torch.int32)
                scs[b, g, :len(cs)] = torch.tensor(cs, dtype=torch.float64)
        if with_gather:
            cand_i, cand_s = SH.gather_candidates(ids, scs, part["blk_lo"])
        else:                                                        # planted: no exchange
            cand_i = torch.where(ids >= 0, ids + part["blk_lo"].view(-1, 1, 1), ids)
            cand_s = scs
        sel = np.full((B, G, w.k), -1, dtype=np.int32)
        for b in range(B):
            for g in range(G):
                keep = cand_i[b, g] >= 0
                m = O.merge_block_candidates(cand_i[b, g][keep].tolist(), cand_s[b, g][keep].tolist(),
                                             int(part["local_block"][b]), w.k)
                sel[b, g, :len(m)] = m
        want_sel = O.index_topk(f(inp["q_idx"]), f(inp["k_idx"]), inp["cu_q_host"], inp["cu_k_host"], w.k, w.B_k)
        sel_ok = np.array_equal(sel, want_sel)
        # this rank's selected blocks, relative to its range, and its attention over them
        lo, hi = part["blk_lo"].numpy(), part["blk_hi"].numpy()
        sel_loc = np.full_like(sel, -1)
        o = np.zeros((B, w.H, w.d))
        lse = np.full((B, w.H), -np.inf)
        q, kk, vv = f(inp["q"]), f(part["k"]), f(part["v"])
        for b in range(B):
            n_keys = ck[b + 1] - ck[b]
            for g in range(G):
                mine = [int(x) - int(lo[b]) for x in sel[b, g] if lo[b] <= x < hi[b]]
                sel_loc[b, g, :len(mine)] = mine
                J = np.concatenate([np.arange(j * w.B_k, min((j + 1) * w.B_k, n_keys)) for j in mine]) \
                    if mine else np.zeros(0, dtype=np.int64)
                if len(J):
                    ob, lb_ = O.attend(q[b, g * Hg:(g + 1) * Hg], kk[ck[b] + J, g], vv[ck[b] + J, g], w.sm_scale)
                    o[b, g * Hg:(g + 1) * Hg] = ob
                    lse[b, g * Hg:(g + 1) * Hg] = lb_
        outs, lses, sels = SH.gather_rank_outputs(torch.from_numpy(o), torch.from_numpy(lse),
                                                  torch.from_numpy(sel_loc))
        if rank == 0:
            want_o, want_l = O.msa_forward_rows(f(inp["q"]), f(inp["k"]), f(inp["v"]), want_sel, inp["cu_q_host"],
                                                inp["cu_k_host"], list(range(B)), w.B_k, w.sm_scale)
            got_o, got_l = np.zeros_like(want_o), np.zeros_like(want_l)
            for b in range(B):
                for h in range(w.H):
                    rs = [r for r in range(world) if (sels[r][b, h // Hg] >= 0).any()]
                    got_o[b, h], got_l[b, h] = O.lse_combine(np.stack([outs[r][b, h].numpy() for r in rs]),
                                                             np.array([lses[r][b, h].item() for r in rs]))
            ok = sel_ok and np.allclose(got_o, want_o, rtol=0, atol=1e-12) and np.allclose(got_l, want_l, atol=1e-12)
            # the same merge read through the f16 layout the library's combine takes
            acc, plse, slot = SH.rank_partials([t.float() for t in outs], [t.float() for t in lses], sels, w.H, G)
            lay_o = np.zeros_like(want_o)
            for b in range(B):
                for g in range(G):
                    rs = [r for r in range(world) if slot[b, g, r] >= 0]
                    for i in range(Hg):
                        a_ = np.stack([acc[b, g, r, :, i, :].reshape(-1).double().numpy() for r in rs])
                        l_ = np.array([plse[b, g, r, i].item() for r in rs])
                        lay_o[b, g * Hg + i] = O.lse_combine(a_, l_)[0]
            ok = ok and float(np.max(np.abs(lay_o - want_o))) < 2e-3
            result.put((bool(ok), bool(sel_ok)))
        else:
            dist.barrier()
        if rank == 0:
            dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, with_gather):
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_keysplit, args=(r, world, port, with_gather, result)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    return result.get(timeout=10)


@pytest.mark.parametrize("world", [2, 4])
def test_key_split_oracle_equals_unsharded_on_gloo_ranks(world):
    ok, sel_ok = _run(world, True)
    assert ok and sel_ok


def test_key_split_without_the_candidate_exchange_fails():
    _, sel_ok = _run(2, False)
    assert not sel_ok
