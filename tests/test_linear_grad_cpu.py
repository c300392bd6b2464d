"""The linear-layer gradient source of the second refresh workload, checked on
CPU with the oracle: G = D^T X (the weight-gradient model of Theorem 3.1 on the
AIMech Q-GaLore page, paper section 3.1) has a top-r subspace that keeps moving
while the output-gradient mixing turns and stays put once it has settled, which
is what the layer-adaptive schedule (same page, Eq. (5)) is meant to detect."""
import numpy as np
import torch

import oracle as O
import synth


def _top_r(gen, t, r):
    X, D = gen.draw(t)
    Xf = X[:, : gen.n].float().numpy()
    Df = D[:, : gen.m].float().numpy()
    G = O.linear_backward_weight(Df, Xf)
    return O.exact_topr(G, r)[0]


def test_subspace_moves_while_mixing_turns_and_settles_after():
    # k = r: the top-r left subspace of G is the output-gradient subspace, and
    # 10 steps of turning are 1 rad in every plane, so CosSim falls to about
    # cos(1) = 0.54 while it turns and stays near 1 once it has settled
    m, n, B, k, r = 64, 96, 2048, 8, 8
    gen = synth.DeviceLinearLayerBatch(m, n, B, k, 0.9, 1e-3, 0.1, 40, seed=3, device=torch.device("cpu"))
    early = [O.cossim(_top_r(gen, t, r), _top_r(gen, t + 10, r)) for t in (0, 10, 20)]
    late = [O.cossim(_top_r(gen, t, r), _top_r(gen, t + 10, r)) for t in (50, 60, 70)]
    assert min(late) > 0.98, late
    assert max(early) < 0.65, early
    assert all(abs(c - np.cos(1.0)) < 0.08 for c in early), early


def test_draws_are_seeded_and_shaped():
    a = synth.DeviceLinearLayerBatch(24, 40, 64, 8, 0.9, 1e-3, 0.1, 5, seed=9, device=torch.device("cpu"))
    b = synth.DeviceLinearLayerBatch(24, 40, 64, 8, 0.9, 1e-3, 0.1, 5, seed=9, device=torch.device("cpu"))
    Xa, Da = (t.clone() for t in a.draw(3))
    Xb, Db = b.draw(3)
    assert Xa.shape == (64, a.ldx) and Da.shape == (64, a.ldd)
    assert torch.equal(Xa, Xb) and torch.equal(Da, Db)
    assert not torch.equal(a.draw(4)[0], Xa)
