"""Expert parallelism on the host: two (or four) gloo ranks, each with its own tokens and
its share of the experts, exchange routed rows with mixture_experts_ffn_05_b200.ep and
must reproduce, bit for bit, the MoE branch that one rank holding every expert computes
for the same tokens.
The expert arithmetic is the oracle's (fp64, one row at a time, so that a row's result
does not depend on which rows share its matmul), on both sides of the comparison."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from mixture_experts_ffn_05_b200 import ep

SHAPE = synth.Shape(T=7, H=32, E=8, k=2, I=16, D=16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    p = synth.make_layer(77, SHAPE)
    wgu = oracle.bf16(p["w_gate_up"])  # [E][2I][H]
    wd = oracle.bf16(p["w_down"])      # [E][H][I]
    return p, wgu, wd


def _row_mlp(row, wgu, wd):
    return oracle.gated_mlp(row[None, :], wgu, wd)[0]


def _tokens(rank, bias):
    """The rank's tokens, their routing (oracle router) and sorted order (oracle permute)."""
    p, _, _ = _layer()
    x = oracle.bf16(synth.x_rows(1000 + rank, SHAPE.H, SHAPE.T))
    r = oracle.router(x, oracle.bf16(p["router_scale"]), oracle.bf16(p["w_router"]), bias,
                      oracle.bf16(p["per_expert_scale"]), SHAPE.k, SHAPE.eps)
    xn = r["xhat"] * oracle.bf16(p["g_pre_moe"])
    offsets, sorted_src, inv_pos = oracle.permute(r["topk_idx"], SHAPE.E)
    return xn, r["topk_idx"], r["topk_w"], offsets, sorted_src, inv_pos


def _reference(xn, idx, w, wgu, wd):
    """The branch with every expert local: slot order, one row at a time."""
    T, k = idx.shape
    out = np.zeros_like(xn)
    for t in range(T):
        for j in range(k):
            out[t] += w[t, j] * _row_mlp(xn[t], wgu[idx[t, j]], wd[idx[t, j]])
    return out


def _rank(rank, world, port, bias, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        part = ep.ExpertPartition(SHAPE.E, world)
        _, wgu, wd = _layer()
        xn, idx, w, offsets, sorted_src, inv_pos = _tokens(rank, bias)
        rows_sorted = torch.from_numpy(xn[sorted_src // SHAPE.k])

        def compute(rows, local_offsets):
            # this rank's experts only, one row at a time
            out = torch.empty_like(rows)
            for el in range(part.local):
                e = part.first(rank) + el
                for q in range(int(local_offsets[el]), int(local_offsets[el + 1])):
                    out[q] = torch.from_numpy(_row_mlp(rows[q].numpy(), wgu[e], wd[e]))
            return out

        y_sorted = ep.ep_moe_forward(rows_sorted, torch.from_numpy(offsets), part, compute).numpy()
        T, k = idx.shape
        moe = np.zeros_like(xn)
        for t in range(T):
            for j in range(k):  # slot order, as the block's combine
                moe[t] += w[t, j] * y_sorted[inv_pos[t * k + j]]
        ref = _reference(xn, idx, w, wgu, wd)
        remote = int(np.sum(part.owner(idx) != rank))
        results[rank] = (bool(np.array_equal(moe, ref)), remote, float(np.abs(moe - ref).max()))
    finally:
        dist.destroy_process_group()


def _run(bias, world=2):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank, args=(world, port, bias, results), nprocs=world, join=True,
                       start_method="spawn")
    return dict(results)


def test_two_ranks_reproduce_the_single_rank_branch():
    res = _run(None)
    for rank in (0, 1):
        same, remote, err = res[rank]
        assert same, (rank, err)
    assert res[0][1] > 0 and res[1][1] > 0  # rows really crossed ranks both ways


def test_four_ranks_reproduce_the_single_rank_branch():
    """Four ranks of two experts each: every rank's rows scatter over three peers."""
    res = _run(None, world=4)
    for rank in range(4):
        same, remote, err = res[rank]
        assert same, (rank, err)
    assert sum(res[r][1] for r in range(4)) > 0


def test_four_ranks_all_pairs_to_one_owner():
    """Every pair routed to the experts of rank 3 (a logit offset on experts 6 and 7): rank
    3 receives all 4 x T x k rows, the others none, and every rank still reproduces its
    branch (the receive buffers are sized from the exchanged counts)."""
    bias = np.array([0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 50.0, 49.0])
    res = _run(bias, world=4)
    for rank in range(4):
        assert res[rank][0], (rank, res[rank][2])
    assert res[3][1] == 0  # rank 3 sends nothing away
    for rank in range(3):
        assert res[rank][1] == SHAPE.T * SHAPE.k  # every pair of the others crosses


def test_one_sided_exchange():
    """A logit offset sends every pair to experts 0..3 (rank 0's): rank 1 receives nothing
    (zero-size splits) and still gets every result back."""
    bias = np.array([50.0, 49.0, 48.0, 47.0, 0.0, 0.0, 0.0, 0.0])
    res = _run(bias)
    for rank in (0, 1):
        assert res[rank][0], (rank, res[rank][2])
    assert res[0][1] == 0 and res[1][1] == SHAPE.T * SHAPE.k


def test_receive_layout_by_hand():
    """Rows from source 0: experts (0: 2 rows, 1: 1 row); from source 1: (0: 1, 1: 2).
    Arrival order 0a 0b | 0c(e1) | 1a(e0) | 1b 1c (e1) = indices 0..5; expert-major stable
    order: e0 from s0 (0, 1), e0 from s1 (3), e1 from s0 (2), e1 from s1 (4, 5)."""
    counts = torch.tensor([[2, 1], [1, 2]])
    off, order = ep.receive_layout(counts)
    assert off.tolist() == [0, 3, 6]
    assert order.tolist() == [0, 1, 3, 2, 4, 5]
    part = ep.ExpertPartition(4, 2)
    offsets = torch.tensor([0, 2, 3, 3, 7])
    assert ep.send_counts(offsets, part).tolist() == [3, 4]
    assert ep.local_counts(offsets, part).tolist() == [[2, 1], [0, 4]]
