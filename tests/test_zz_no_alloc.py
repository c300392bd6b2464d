"""qg_step_noalloc, the step entry point that takes no workspace.

It exists for callers that cannot allocate device memory for a workspace (a
host program whose device memory belongs to another allocator with a fixed
budget, or a thread that must not take cudaMalloc's implicit synchronisation).
Its scratch lives in a static device array inside the library.  These tests
drive it through the C ABI on two calls in a row and check that it leaves the
weights and moments exactly as the regular qg_step (with a caller workspace)
does on the same inputs; they also check that an oversized matrix is refused.

This file is collected last so that a run stopping at the first failure has
run every other test before it.
"""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_rank_gradient_b200 as qg
import synth
from gpu_layer import GpuLayer, stream, upload_gradient

pytestmark = pytest.mark.gpu


def _twin_layers(m, n, r, seed, side=0):
    oc = O.Config(m=m, n=n, r=r, seed=seed, layer_id=7, proj_side=side)
    Wq = synth.weight_codes(m, n, seed)
    sW = synth.weight_scales(m, n, seed=seed)
    P = synth.orthonormal(n if side else m, r, seed)
    codes, sP = O.quant_int4_groups(P.astype(np.float32))
    Pq = O.pack_int4(codes)
    a, b = GpuLayer(oc, Wq, sW), GpuLayer(oc, Wq, sW)
    a.set_projection(Pq, sP)
    b.set_projection(Pq, sP)
    return a, b


# Left-side layouts (P m x r, N r x n) and right-side ones (P n x r, N m x r),
# among them the largest LLaMA-7B matrices at r = 1024 on both sides: the
# 11008 x 4096 down projection is the one a right-side caller projects.
@pytest.mark.parametrize("m,n,r,side", [(512, 1376, 128, 0), (640, 1365, 96, 0), (4096, 11008, 1024, 0),
                                        (700, 300, 64, 1), (11008, 4096, 1024, 1)])
def test_noalloc_step_matches_workspace_step_twice(cuda_ok, m, n, r, side):
    a, b = _twin_layers(m, n, r, seed=m + n, side=side)
    gen = synth.lowrank_gradient(m, n, rank=min(64, m, n), seed=m + n)
    for t in range(2):
        _, Gb = gen.draw(t)
        dG, ldg = upload_gradient(Gb)
        a.step(dG, ldg)
        qg.check(qg.qg_step_noalloc(b.h, dG.data_ptr(), ldg, stream()), "qg_step_noalloc")
        torch.cuda.synchronize()
        np.testing.assert_array_equal(b.weights(), a.weights())
        for x, y in zip(b.moments(), a.moments()):
            np.testing.assert_array_equal(x, y)
    assert b.sched().t == 2
    assert b.status() == qg.QG_OK
    a.close()
    b.close()


def test_noalloc_refuses_matrices_beyond_its_scratch(cuda_ok):
    m, n, r = 8192, 8448, 1024  # P~ (16 MiB) + N (16.5 MiB) exceed the 32 MiB array
    oc = O.Config(m=m, n=n, r=r)
    gl = GpuLayer(oc, np.zeros((m, n), np.int8), np.ones(m * n // 256, np.float32))
    gl.set_projection(np.zeros(m * r // 2, np.uint8), np.zeros(m * r // 64, np.float32))
    dG = torch.zeros((m, n), dtype=torch.int16, device="cuda")
    assert qg.qg_step_noalloc(gl.h, dG.data_ptr(), n, stream()) == qg.QG_ESHAPE
    assert gl.sched().t == 0
    gl.close()
