"""Failure detection on the GPU without a fault: a bounded device wait that runs
out, and resuming a layer from a copy of its state.

* Every device wait in the library is bounded.  qg_selfcheck_wait_timeout makes
  one run out (an mbarrier that nothing arrives at): the wait must give up after
  its limit, set the timeout bit and return, and the context must stay usable.
* A layer's state is the caller's device buffer plus the host schedule
  (qg_layer_sched_get / _set): a copy of both, taken between steps and restored
  into a fresh handle, continues bit-identically (the Philox counters depend on
  the step, the layer and the element only).
"""
from ctypes import byref

import numpy as np
import pytest
import torch

import oracle as O
import quantized_rank_gradient_b200 as qg
import synth
from gpu_layer import GpuLayer, stream, upload_gradient

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda(cuda_ok):
    torch.cuda.synchronize()
    yield
    torch.cuda.synchronize()


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, dtype=torch.int64, device="cuda")
    limit = 20_000_000  # 20 ms
    qg.check(qg.qg_selfcheck_wait_timeout(limit, status.data_ptr(), out.data_ptr(), stream()))
    torch.cuda.synchronize()
    gave_up, ns = (int(v) for v in out.cpu())
    assert gave_up == 1
    assert limit <= ns < limit + 50_000_000
    assert int(status.item()) & 1
    # the context still runs kernels: a Philox call matches the oracle
    c = torch.arange(4 * 256, dtype=torch.int32, device="cuda").view(4, 256)
    res = torch.zeros(4 * 256, dtype=torch.int32, device="cuda")
    qg.check(qg.qg_philox4x32_10(*(c[i].data_ptr() for i in range(4)), 256, 7, 9, res.data_ptr(), stream()))
    got = res.cpu().numpy().view(np.uint32).reshape(256, 4)
    cc = c.cpu().numpy().astype(np.uint32)
    ref = np.stack(O.philox4x32_10(cc[0], cc[1], cc[2], cc[3], 7, 9), axis=1)
    np.testing.assert_array_equal(got, ref)
    assert qg.qg_selfcheck_wait_timeout(0, status.data_ptr(), out.data_ptr(), stream()) == qg.QG_EINVAL


def test_resume_from_a_state_copy_is_bit_identical():
    m, n, r = 512, 1376, 128
    oc = O.Config(m=m, n=n, r=r, seed=21, layer_id=4)
    Wq, sW = synth.weight_codes(m, n, 21), synth.weight_scales(m, n, seed=21)
    gen = synth.lowrank_gradient(m, n, rank=128, seed=21)
    P, _ = O.exact_topr(gen.draw(0)[0], r)
    codes, sP = O.quant_int4_groups(P.astype(np.float32))
    Pq = O.pack_int4(codes)
    grads = [upload_gradient(gen.draw(t)[1]) for t in range(4)]

    ref = GpuLayer(oc, Wq, sW)
    ref.set_projection(Pq, sP)
    for t in range(4):
        ref.step(*grads[t])

    a = GpuLayer(oc, Wq, sW)
    a.set_projection(Pq, sP)
    for t in range(2):
        a.step(*grads[t])
    torch.cuda.synchronize()
    state_copy, w_copy = a.state.clone(), a.W.clone()
    sched = qg.qg_sched()
    qg.check(qg.qg_layer_sched_get(a.h, byref(sched)))
    a.close()

    b = GpuLayer(oc, Wq, sW)          # fresh handle, then the saved bytes and schedule
    b.state.copy_(state_copy)
    b.W.copy_(w_copy)
    qg.check(qg.qg_layer_sched_set(b.h, byref(sched)))
    for t in range(2, 4):
        b.step(*grads[t])
    np.testing.assert_array_equal(b.weights(), ref.weights())
    for x, y in zip(b.moments(), ref.moments()):
        np.testing.assert_array_equal(x, y)
    assert b.sched().t == 4 and b.status() == qg.QG_OK
