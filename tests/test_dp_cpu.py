"""Layer-sharded data parallelism (quantized_rank_gradient_b200.dp) on CPU: two
gloo ranks (127.0.0.1), with the oracle's optimizer step standing in for
qg_step_batch on the owned matrices.

Every rank holds the gradients of its own slice of the batch for all matrices;
after the reduce-scatter each owner steps its matrices on the mean gradient, and
after the all-gather every rank must hold, bit for bit, the weights of one
process that averaged the gradients and stepped every matrix itself.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

SHAPES = [(48, 64), (64, 40), (96, 32), (64, 64), (40, 48), (32, 96)]
R = 32


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _initial_state(i, m, n):
    import oracle as O
    import synth
    cfg = O.Config(m=m, n=n, r=R, seed=17 + i, layer_id=i)
    st = O.LayerState.create(cfg, synth.weight_codes(m, n, seed=i), synth.weight_scales(m, n, seed=i))
    G0, _ = synth.lowrank_gradient(m, n, rank=16, seed=500 + i).draw(0)
    O.set_projection(st, O.exact_topr(G0, R)[0])
    return st


def _local_gradient(rank, i, m, n):
    import synth
    G, _ = synth.lowrank_gradient(m, n, rank=16, seed=1000 * (rank + 1) + i).draw(1)
    return np.asarray(G, np.float32)


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist

    import oracle as O
    from quantized_rank_gradient_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = dp.plan_shards(SHAPES, [R] * len(SHAPES), world)
        flat_g = torch.zeros(world * plan.grad_shard, dtype=torch.float32)
        flat_w = torch.zeros(world * plan.weight_shard, dtype=torch.uint8)
        states = [_initial_state(i, m, n) for i, (m, n) in enumerate(SHAPES)]
        for i, (m, n) in enumerate(SHAPES):
            dp.grad_view(flat_g, plan, i, (m, n))[:, :n] = torch.from_numpy(_local_gradient(rank, i, m, n))
            dp.weight_view(flat_w, plan, i, (m, n))[:, :n] = torch.from_numpy(states[i].Wq.view(np.uint8))
        dp.reduce_scatter_gradients(flat_g, plan, rank)
        for i in plan.owned(rank):
            m, n = SHAPES[i]
            G = dp.grad_view(flat_g, plan, i, (m, n))[:, :n].numpy().astype(np.float32)
            O.step(states[i], G)
            dp.weight_view(flat_w, plan, i, (m, n))[:, :n] = torch.from_numpy(states[i].Wq.view(np.uint8))
        dp.all_gather_weights(flat_w, plan, rank)
        W = [dp.weight_view(flat_w, plan, i, s)[:, : s[1]].numpy().view(np.int8).copy() for i, s in enumerate(SHAPES)]
        out.put((rank, plan.owner, plan.work, W))
    finally:
        dist.destroy_process_group()


def test_plan_balances_work_and_aligns_every_matrix():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from quantized_rank_gradient_b200 import dp
    shapes = [(4096, 4096)] * 4 + [(4096, 11008)] * 2 + [(11008, 4096)]
    shapes = shapes * 32
    for world in (1, 2, 3, 8):
        plan = dp.plan_shards(shapes, [1024] * len(shapes), world)
        assert sorted(set(plan.owner)) == list(range(world))
        assert max(plan.work) <= 1.05 * min(plan.work)
        spans_g, spans_w = [], []
        for i, (m, n) in enumerate(shapes):
            assert plan.grad_offset[i] % dp.GRAD_ALIGN == 0 and plan.weight_offset[i] % dp.WEIGHT_ALIGN == 0
            k = plan.owner[i]
            assert k * plan.grad_shard <= plan.grad_offset[i] < (k + 1) * plan.grad_shard
            assert plan.grad_offset[i] + m * plan.ldg[i] <= (k + 1) * plan.grad_shard
            assert plan.weight_offset[i] + m * plan.ldw[i] <= (k + 1) * plan.weight_shard
            spans_g.append((plan.grad_offset[i], plan.grad_offset[i] + m * plan.ldg[i]))
            spans_w.append((plan.weight_offset[i], plan.weight_offset[i] + m * plan.ldw[i]))
        for spans in (spans_g, spans_w):
            spans.sort()
            assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))  # no overlap


def test_two_gloo_ranks_match_one_process_bit_for_bit():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, owner, work, W = out.get(timeout=180)
        res[rank] = (owner, work, W)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] and set(res[0][0]) == {0, 1}
    # one process: the mean gradient (two float32 terms, then a halving: exact
    # and order-free) and every matrix stepped here
    for i, (m, n) in enumerate(SHAPES):
        st = _initial_state(i, m, n)
        G = ((_local_gradient(0, i, m, n) + _local_gradient(1, i, m, n)) / np.float32(2)).astype(np.float32)
        O.step(st, G)
        for rank in (0, 1):
            np.testing.assert_array_equal(res[rank][2][i], st.Wq, err_msg=f"matrix {i} on rank {rank}")
