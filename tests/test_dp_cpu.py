"""Layer-sharded data parallelism (quantized_rank_gradient_b200.dp) on CPU: two
and three gloo ranks (127.0.0.1), with the oracle's optimizer step standing in
for qg_step_batch on the owned matrices.

Every rank holds the bf16 gradients of its own slice of the batch for all
matrices.  The reduce-scatter must deliver to each owner
G = bf16(fl32(fl32(sum_k G_k) / world)): a float32 sum over the ranks, one
float32 division and one rounding to bf16.  The local gradients differ in
magnitude by up to 2^20 between ranks, so that some float32 sums are inexact and
their order matters: with two ranks the float32 sum is the same in either order
and the result is checked bit for bit; with three, every element must equal the
rule taken in one of the three association orders, and lie within the rule's
error bound of the exact mean.  Each owner then steps its matrices on the
gradient it received, and after the all-gather every rank must hold, bit for
bit, the weights (codes and group scales) of one process that stepped every
matrix itself on those gradients.  The mixed case also varies projection sides
and weight policies: a matrix whose groups are re-scaled (w_rescale = 1)
changes its scales on the owner, and the all-gather must carry them.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

SHAPES = [(48, 64), (64, 40), (96, 32), (64, 64), (40, 48), (32, 96)]
# (m, n, proj_side, w_rescale)
MIXED = [(64, 256, 0, 1), (96, 256, 1, 1), (48, 64, 0, 0), (256, 64, 1, 0), (32, 512, 0, 1), (40, 48, 1, 0)]
R = 32


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spec(s):
    return s if len(s) == 4 else (s[0], s[1], 0, 0)


def _initial_state(i, spec):
    import oracle as O
    import synth
    m, n, side, wr = _spec(spec)
    cfg = O.Config(m=m, n=n, r=R, seed=17 + i, layer_id=i, proj_side=side, w_rescale=wr)
    st = O.LayerState.create(cfg, synth.weight_codes(m, n, seed=i), synth.weight_scales(m, n, seed=i))
    G0, _ = synth.lowrank_gradient(m, n, rank=16, seed=500 + i).draw(0)
    O.set_projection(st, O.exact_topr(G0 if side == 0 else G0.T, R)[0])
    return st


def _local_gradient(rank, i, m, n):
    """Rank `rank`'s bf16 gradient of matrix i (float32 values, uint16 bits).
    The ranks' magnitudes differ (a factor 2^(10 rank) on alternate rows), so
    the float32 sums over ranks are not all exact."""
    import synth
    G, _ = synth.lowrank_gradient(m, n, rank=16, seed=1000 * (rank + 1) + i).draw(1)
    scale = np.ones((m, 1))
    scale[1::2] = 2.0 ** (10 * rank)
    return synth.to_bf16(np.asarray(G, np.float64) * scale)


def _worker(rank, world, port, out, specs):
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
        shapes = [_spec(s)[:2] for s in specs]
        plan = dp.plan_shards(shapes, [R] * len(shapes), world)
        flat_g = torch.zeros(world * plan.grad_shard, dtype=torch.bfloat16)
        flat_w = torch.zeros(world * plan.weight_shard, dtype=torch.uint8)
        states = [_initial_state(i, s) for i, s in enumerate(specs)]
        for i, (m, n) in enumerate(shapes):
            bits = _local_gradient(rank, i, m, n)[1]
            dp.grad_view(flat_g, plan, i, (m, n))[:, :n] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
            dp.weight_view(flat_w, plan, i, (m, n))[:, :n] = torch.from_numpy(states[i].Wq.view(np.uint8))
            dp.scale_view(flat_w, plan, i, (m, n))[:] = torch.from_numpy(states[i].sW)
        dp.reduce_scatter_gradients(flat_g, plan, rank)
        received = {}
        for i in plan.owned(rank):
            m, n = shapes[i]
            G = dp.grad_view(flat_g, plan, i, (m, n))[:, :n].float().numpy()
            received[i] = G.copy()
            O.step(states[i], G)
            dp.weight_view(flat_w, plan, i, (m, n))[:, :n] = torch.from_numpy(states[i].Wq.view(np.uint8))
            dp.scale_view(flat_w, plan, i, (m, n))[:] = torch.from_numpy(states[i].sW)
        dp.all_gather_weights(flat_w, plan, rank)
        W = [dp.weight_view(flat_w, plan, i, s)[:, : s[1]].numpy().view(np.int8).copy() for i, s in enumerate(shapes)]
        S = [dp.scale_view(flat_w, plan, i, s).numpy().copy() for i, s in enumerate(shapes)]
        out.put((rank, plan.owner, plan.work, W, S, received))
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
            assert plan.scale_offset[i] % dp.WEIGHT_ALIGN == 0
            k = plan.owner[i]
            ns = -(-(m * n) // 256)
            assert k * plan.grad_shard <= plan.grad_offset[i] < (k + 1) * plan.grad_shard
            assert plan.grad_offset[i] + m * plan.ldg[i] <= (k + 1) * plan.grad_shard
            assert k * plan.weight_shard <= plan.weight_offset[i]
            assert plan.scale_offset[i] + 4 * ns <= (k + 1) * plan.weight_shard
            spans_g.append((plan.grad_offset[i], plan.grad_offset[i] + m * plan.ldg[i]))
            spans_w.append((plan.weight_offset[i], plan.weight_offset[i] + m * plan.ldw[i]))
            spans_w.append((plan.scale_offset[i], plan.scale_offset[i] + 4 * ns))
        for spans in (spans_g, spans_w):
            spans.sort()
            assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))  # no overlap


@pytest.mark.parametrize("world,specs", [(2, SHAPES), (2, MIXED), (3, MIXED)],
                         ids=["2-default", "2-mixed-sides-and-rescale", "3-mixed"])
def test_gloo_ranks_match_one_process_bit_for_bit(world, specs):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out, specs)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, owner, work, W, S, got = out.get(timeout=180)
        res[rank] = (owner, work, W, S, got)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(res[k][0] == res[0][0] for k in range(world)) and set(res[0][0]) == set(range(world))
    owner = res[0][0]
    f32 = np.float32
    grown, inexact = 0, 0
    for i, spec in enumerate(specs):
        m, n = _spec(spec)[:2]
        g = [_local_gradient(k, i, m, n)[0].astype(np.float32) for k in range(world)]
        G = res[owner[i]][4][i]
        # the rule in every association order of the float32 sum
        if world == 2:
            orders = [(g[0] + g[1]).astype(f32)]
        else:
            orders = [((g[a] + g[b]).astype(f32) + g[c]).astype(f32) for a, b, c in ((0, 1, 2), (0, 2, 1), (1, 2, 0))]
        cands = [O.bf16_round((s / f32(world)).astype(f32)) for s in orders]
        assert np.all(np.any([G == c for c in cands], axis=0)), f"matrix {i}: a mean outside the rule"
        exact = sum(x.astype(np.float64) for x in g)
        inexact += int((orders[0].astype(np.float64) != exact).sum())
        bound = (world - 1) * 2.0 ** -24 * sum(np.abs(x.astype(np.float64)) for x in g) / world
        err = np.abs(G.astype(np.float64) - exact / world)
        assert np.all(err <= 2.0 ** -8 * np.abs(exact / world) * (1 + 2.0 ** -23) + bound * (1 + 2.0 ** -8) + 1e-45)
        # one process stepping every matrix on the gradient its owner received
        st = _initial_state(i, spec)
        s0 = st.sW.copy()
        O.step(st, G)
        grown += int((st.sW != s0).sum())
        for rank in range(world):
            np.testing.assert_array_equal(res[rank][2][i], st.Wq, err_msg=f"matrix {i} on rank {rank}")
            np.testing.assert_array_equal(res[rank][3][i], st.sW, err_msg=f"scales {i} on rank {rank}")
    assert inexact > 0  # some float32 sums rounded: the rule, not an exact grid, is what is checked
    if specs is MIXED:
        assert grown > 0  # some owner changed its scales, and every rank received them
