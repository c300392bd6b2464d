"""GPU parity of the subspace refresh and of CosSim against the CPU oracle.

Bars:
  * CosSim (qg_cossim, identical float32 inputs): |gpu - oracle| <= 1e-4.
  * Refreshed subspace: principal-angle cosines >= 0.999 between the GPU's
    float32 projection and the oracle's, on every direction for inputs with a
    singular-value gap after r, and on the signal-dominated leading directions
    for noise-dominated inputs (the rest are reported, not gated: near-equal
    noise singular values have no stable basis).
  * The layer-adaptive schedule (refresh times, interval doubling) follows the
    oracle's decisions.
"""
from ctypes import byref, c_void_p

import numpy as np
import pytest
import scipy.linalg
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


def gpu_cossim(Pa, Pb):
    m, r = Pa.shape
    a = torch.from_numpy(np.ascontiguousarray(Pa, np.float32)).cuda()
    b = torch.from_numpy(np.ascontiguousarray(Pb, np.float32)).cuda()
    out = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(qg.qg_cossim_workspace_bytes(m, r), dtype=torch.uint8, device="cuda")
    qg.check(qg.qg_cossim(a.data_ptr(), b.data_ptr(), m, r, r, out.data_ptr(), ws.data_ptr(), ws.numel(), stream()))
    return float(out.item())


@pytest.mark.parametrize("m,r", [(256, 32), (512, 128), (2048, 1024)])
def test_cossim_closed_forms(m, r):
    # r = 32: the float32 Newton-Schulz steps only; r = 128 and 1024: the
    # tensor-core steps (bf16 hi + lo operands) followed by float32 ones
    rng = np.random.default_rng(r)
    P = np.linalg.qr(rng.standard_normal((m, r)))[0]
    Orot = np.linalg.qr(rng.standard_normal((r, r)))[0]
    assert abs(gpu_cossim(P, P) - 1) < 1e-4
    assert abs(gpu_cossim(P, P @ Orot) - 1) < 1e-4
    F = np.linalg.qr(rng.standard_normal((m, 2 * r)))[0]
    assert abs(gpu_cossim(F[:, :r], F[:, r:])) < 1e-4
    theta = np.linspace(0, 1.5, r)
    A = np.zeros((m, r))
    B = np.zeros((m, r))
    A[np.arange(r), np.arange(r)] = 1
    B[np.arange(r), np.arange(r)] = np.cos(theta)
    B[r + np.arange(r), np.arange(r)] = np.sin(theta)
    assert abs(gpu_cossim(A, B) - np.cos(theta).mean()) < 1e-4


def test_cossim_matches_oracle():
    rng = np.random.default_rng(0)
    for (mm, rr) in [(300, 64), (1376, 128), (4096, 1024), (11008, 1024)]:
        X = np.linalg.qr(rng.standard_normal((mm, rr)))[0]
        Y = np.linalg.qr(X + 0.7 * rng.standard_normal((mm, rr)) / np.sqrt(mm))[0]
        assert abs(gpu_cossim(X, Y) - O.cossim(X.astype(np.float32), Y.astype(np.float32))) < 1e-4


def principal_cosines(A, B):
    return np.sort(np.cos(scipy.linalg.subspace_angles(np.asarray(A, np.float64), np.asarray(B, np.float64))))[::-1]


def _refresh_pair(m, n, r, G_vals, G_bits, seed=3, layer_id=2, side=0):
    oc = O.Config(m=m, n=n, r=r, seed=seed, layer_id=layer_id, proj_side=side)
    ost = O.LayerState.create(oc, np.zeros((m, n), np.int8), np.ones(-(-m * n // 256), np.float32))
    oinfo = O.refresh(ost, G_vals, force=True)
    gl = GpuLayer(oc, np.zeros((m, n), np.int8), np.ones(-(-m * n // 256), np.float32))
    dG, ldg = upload_gradient(G_bits)
    info, Pg = gl.refresh(dG, ldg, force=1)
    return ost, oinfo, gl, info, Pg


@pytest.mark.parametrize("m,n,r,side", [(256, 256, 32, 0), (300, 250, 32, 0), (1376, 512, 128, 0),
                                        (512, 1376, 96, 0), (300, 250, 32, 1), (1376, 512, 128, 1)])
def test_refresh_gap_input_matches_oracle_subspace(m, n, r, side):
    G, Gb = synth.gap_gradient(m, n, r, seed=m + n)
    ost, oinfo, gl, info, Pg = _refresh_pair(m, n, r, G, Gb, side=side)
    assert info.refreshed == 1 and info.has_cossim == 0 and info.n_refresh == 1
    Po = oinfo["P"]
    cos = principal_cosines(Pg, Po)
    assert cos.min() >= 0.999, cos.min()
    # orthonormal, sorted, sign-canonical columns agree one by one; the sign
    # rule (largest-magnitude entry positive) may only differ where the
    # oracle's two largest magnitudes in the column are within 1e-3 of each
    # other (a numerical tie between float32 and float64)
    np.testing.assert_allclose(Pg.T @ Pg, np.eye(r), atol=2e-3)
    col = np.sum(Pg.astype(np.float64) * Po, axis=0)
    top2 = -np.sort(-np.abs(Po), axis=0)[:2]
    tie = (top2[0] - top2[1]) / top2[0] < 1e-3
    assert np.all((col > 0.99) | ((col < -0.99) & tie)), col.min()
    assert np.all(np.abs(col) > 0.99)
    # the GPU's own columns obey the rule
    idx = np.argmax(np.abs(Pg), axis=0)
    assert np.all(Pg[idx, np.arange(r)] > 0)
    # the INT4 projection installed in the layer is the quantization of that P
    Pq, sP = gl.projection()
    ref_codes, ref_s = O.quant_int4_groups(Po.astype(np.float32))
    got_codes = O.unpack_int4(Pq, Po.shape[0] * r)
    assert (got_codes == ref_codes).mean() > 0.98
    np.testing.assert_allclose(sP, ref_s, rtol=2e-2)
    assert gl.status() == qg.QG_OK


def leading_block(sigma, edge, min_gap=0.05, margin=1.5):
    """Largest j whose leading j singular values sit above margin * noise edge
    and are separated from sigma_j by a relative gap >= min_gap."""
    best = 0
    for j in range(1, len(sigma)):
        if sigma[j - 1] < margin * edge:
            break
        if (sigma[j - 1] - sigma[j]) / sigma[j - 1] >= min_gap:
            best = j
    return best


@pytest.mark.parametrize("m,n,r,s0", [(256, 256, 32, 1e-2), (512, 512, 128, 1e-2), (1376, 512, 128, 3e-2)])
def test_refresh_noise_dominated_leading_directions(m, n, r, s0):
    gen = synth.lowrank_gradient(m, n, rank=min(256, m, n), s0=s0, decay=0.8, sigma=1e-4, seed=m)
    G, Gb = gen.draw(0)
    ost, oinfo, gl, info, Pg = _refresh_pair(m, n, r, G, Gb)
    edge = 1e-4 * (np.sqrt(m) + np.sqrt(n))
    k_sig = leading_block(np.linalg.svd(G.astype(np.float64), compute_uv=False), edge)
    assert k_sig >= 1
    Po = oinfo["P"]
    cos = principal_cosines(Pg[:, :k_sig], Po[:, :k_sig])
    assert cos.min() >= 0.999, (k_sig, cos.min())
    np.testing.assert_allclose(Pg.T @ Pg, np.eye(r), atol=2e-3)


def test_quantize_projection_bit_exact():
    for (m, r) in [(256, 32), (300, 64), (4096, 1024)]:
        P = synth.orthonormal(m, r, seed=r).astype(np.float32)
        codes, s = O.quant_int4_groups(P)
        dP = torch.from_numpy(P).cuda()
        Pq = torch.zeros((m * r + 1) // 2, dtype=torch.uint8, device="cuda")
        sP = torch.zeros(-(-m * r // 64), dtype=torch.float32, device="cuda")
        qg.check(qg.qg_quantize_projection(dP.data_ptr(), r, m, r, Pq.data_ptr(), sP.data_ptr(), stream()))
        np.testing.assert_array_equal(Pq.cpu().numpy(), O.pack_int4(codes))
        np.testing.assert_array_equal(sP.cpu().numpy(), s)


def test_schedule_follows_oracle_over_refreshes():
    m, n, r = 256, 320, 32
    oc = O.Config(m=m, n=n, r=r, delta0=2, gamma=0.4, seed=9, layer_id=1)
    Wq, sW = synth.weight_codes(m, n, 9), synth.weight_scales(m, n, seed=9)
    ost = O.LayerState.create(oc, Wq, sW)
    gl = GpuLayer(oc, Wq, sW)
    gen = synth.lowrank_gradient(m, n, rank=32, s0=1.0, decay=0.9, sigma=1e-3, seed=9)
    trace = []
    for t in range(9):
        G, Gb = gen.draw(t)
        dG, ldg = upload_gradient(Gb)
        oi = O.refresh(ost, G, force=(t == 0))
        info, _ = gl.refresh(dG, ldg, force=1 if t == 0 else 0)
        assert bool(info.refreshed) == (oi is not None)
        if oi is not None:
            assert info.delta == ost.delta and info.t_next == ost.t_next and info.n_refresh == ost.n_refresh
            if oi["cossim"] is not None:
                assert abs(info.cossim - oi["cossim"]) < 2e-2
                trace.append(info.cossim)
        gl.step(dG, ldg)
        O.step(ost, G)
    assert len(trace) >= 2 and min(trace) > 0.4   # stable subspace -> intervals doubled
    assert gl.sched().delta > 2


# ---------------------------------------------------------------- moments at a refresh

@pytest.mark.parametrize("policy,side", [(1, 0), (2, 0), (2, 1)])
def test_refresh_moment_policy_matches_oracle(policy, side):
    # a starting projection and three steps give non-zero moments; a forced
    # refresh then replaces P.  The oracle applies the same moment map to the
    # GPU's own moments and projections (teacher-forced), so only the map is
    # compared: reset bit-exact, rotation within the step's moment bar
    m, n, r = (300, 700, 64) if side == 0 else (700, 300, 64)
    oc = O.Config(m=m, n=n, r=r, seed=7, layer_id=3, mom_refresh=policy, proj_side=side)
    Wq, sW = synth.weight_codes(m, n, 7), synth.weight_scales(m, n, seed=7)
    gen = synth.lowrank_gradient(m, n, rank=32, seed=7)
    gl = GpuLayer(oc, Wq, sW)
    G0, _ = gen.draw(0)
    codes, sP = O.quant_int4_groups(O.exact_topr(G0 if side == 0 else G0.T, r)[0].astype(np.float32))
    Pq = O.pack_int4(codes)
    gl.set_projection(Pq, sP)
    for t in range(3):
        _, Gb = gen.draw(t)
        dG, ldg = upload_gradient(Gb)
        gl.step(dG, ldg)
    torch.cuda.synchronize()
    Mq, sM, Vq, sV = gl.moments()
    assert np.abs(Mq).sum() > 0 and np.abs(Vq).sum() > 0
    _, Gb = gen.draw(5)
    dG, ldg = upload_gradient(Gb)
    info, _P = gl.refresh(dG, ldg, force=1)
    assert info.refreshed == 1 and info.has_cossim == 1
    Pq_new, sP_new = gl.projection()
    st = O.LayerState.create(oc, Wq, sW)
    st.Mq, st.sM, st.Vq, st.sV = Mq.copy(), sM.copy(), Vq.copy(), sV.copy()
    p = m if side == 0 else n
    O.refresh_moments(st, O.dequant_int4_f32(Pq_new, sP_new, p, r), O.dequant_int4_f32(Pq, sP, p, r))
    gMq, gsM, gVq, gsV = gl.moments()
    if policy == 1:
        assert not gMq.any() and not gVq.any() and not gsM.any() and not gsV.any()
        return
    for (gq, gs, oq, os_, second) in ((gMq, gsM, st.Mq, st.sM, False), (gVq, gsV, st.Vq, st.sV, True)):
        g = O.dequant_second_moment(gq, gs) if second else O.dequant_rowblock(gq, gs)
        o = O.dequant_second_moment(oq, os_) if second else O.dequant_rowblock(oq, os_)
        assert np.linalg.norm(g - o) <= 1e-2 * np.linalg.norm(o), (second, np.linalg.norm(g - o) / np.linalg.norm(o))
        np.testing.assert_allclose(gs, os_, rtol=1e-4, atol=0)
        assert np.abs(gq.astype(np.int32) - oq.astype(np.int32)).max() <= 1
    assert gl.status() == qg.QG_OK


# ---------------------------------------------------------------- LLaMA-7B shapes, r = 1024 (k = 1040)

def test_refresh_gap_input_r1024_matches_oracle_subspace():
    # k = 1040: the Jacobi runs a 65-block tournament, the Cholesky takes many
    # 32-wide panels and the Gram matrices are split over K.  The top 1024
    # singular values lie in [0.2, 1] (relative neighbour gaps of 0.4 % and
    # less), so single columns are not stable under float32 rounding but every
    # leading subspace is: the top 128, 256, 512 and all 1024 directions must
    # agree with the oracle's (principal cosines >= 0.999).
    m = n = 4096
    r = 1024
    G, Gb = synth.gap_gradient(m, n, r, seed=77)
    ost, oinfo, gl, info, Pg = _refresh_pair(m, n, r, G, Gb, seed=5, layer_id=9)
    assert info.refreshed == 1 and info.n_refresh == 1
    Po = oinfo["P"]
    for j in (128, 256, 512, 1024):
        cos = principal_cosines(Pg[:, :j], Po[:, :j])
        assert cos.min() >= 0.999, (j, cos.min())
    G64 = np.asarray(G, np.float64)
    cos = principal_cosines(Pg, O.exact_topr(G64, r)[0])
    assert cos.min() >= 0.999, cos.min()
    np.testing.assert_allclose(Pg.T @ Pg, np.eye(r), atol=2e-3)
    assert gl.status() == qg.QG_OK


def test_refresh_noise_dominated_4096x11008_leading_directions():
    # The gate-projection shape at r = 1024 with a signal whose leading
    # singular values stand clear of the noise edge 1e-4 (sqrt(m) + sqrt(n)):
    # the well-separated leading block must agree with the oracle's.
    m, n, r = 4096, 11008, 1024
    gen = synth.lowrank_gradient(m, n, rank=256, s0=0.1, decay=0.8, sigma=1e-4, seed=4096)
    G, Gb = gen.draw(0)
    ost, oinfo, gl, info, Pg = _refresh_pair(m, n, r, G, Gb, seed=6, layer_id=4)
    edge = 1e-4 * (np.sqrt(m) + np.sqrt(n))
    k_sig = leading_block(np.linalg.svd(G.astype(np.float64), compute_uv=False), edge)
    assert k_sig >= 4
    cos = principal_cosines(Pg[:, :k_sig], oinfo["P"][:, :k_sig])
    assert cos.min() >= 0.999, (k_sig, cos.min())
    np.testing.assert_allclose(Pg.T @ Pg, np.eye(r), atol=2e-3)
    assert gl.status() == qg.QG_OK


# ---------------------------------------------------------------- the schedule on drifting gradients

def _schedule_parity(m, n, r, delta0, steps, draw):
    """Runs qg_refresh (force only at t = 0) + qg_step and the oracle's refresh +
    step on the same gradients, the oracle taking the GPU's INT4 projection
    after every refresh (teacher forcing).  Returns the refreshes as
    (t, gpu CosSim, oracle CosSim, delta after)."""
    oc = O.Config(m=m, n=n, r=r, delta0=delta0, gamma=0.4, seed=21, layer_id=5)
    Wq, sW = synth.weight_codes(m, n, 21), synth.weight_scales(m, n, seed=21)
    ost = O.LayerState.create(oc, Wq, sW)
    gl = GpuLayer(oc, Wq, sW)
    log = []
    for t in range(steps):
        dG, ldg, G = draw(t)
        oi = O.refresh(ost, G, force=(t == 0))
        info, _ = gl.refresh(dG, ldg, force=1 if t == 0 else 0)
        assert bool(info.refreshed) == (oi is not None), t
        if oi is not None:
            assert (info.delta, info.t_next, info.n_refresh) == (ost.delta, ost.t_next, ost.n_refresh), t
            assert bool(info.has_cossim) == (oi["cossim"] is not None)
            if oi["cossim"] is not None:
                assert abs(info.cossim - oi["cossim"]) <= 1e-3, (t, info.cossim, oi["cossim"])
            log.append((t, info.cossim if info.has_cossim else None, oi["cossim"], info.delta))
            ost.Pq, ost.sP = (x.copy() for x in gl.projection())      # teacher forcing
        gl.step(dG, ldg)
        O.step(ost, G)
    assert gl.sched().t == steps and gl.status() == qg.QG_OK
    return log


def test_schedule_parity_on_a_drifting_gradient():
    # The refresh-stress drift law at a reduced shape: a rank-128 signal whose
    # left singular vectors turn in fixed planes by 0.075 rad per step until
    # step 100 and then stay.  With an interval of 20 steps the subspace turns
    # 1.5 rad between refreshes (CosSim = |cos 1.5| = 0.07, no doubling); once
    # it has settled CosSim is 1 and the interval doubles at every check.
    m, n, r = 512, 1376, 128
    gen = synth.DeviceDriftingGradient(m, n, rank=r, s0=1.0, decay=0.99, sigma=1e-4, rate=0.075, freeze=100,
                                       seed=8, device=torch.device("cuda"))

    def draw(t):
        g = gen.draw(t)
        return g, gen.ld, g[:, :n].float().cpu().numpy()

    log = _schedule_parity(m, n, r, 20, 200, draw)
    assert [t for t, *_ in log] == [0, 20, 40, 60, 80, 100, 120, 160]
    assert [d for *_, d in log] == [20, 20, 20, 20, 20, 20, 40, 80]
    turning = [c for t, c, _, _ in log if 0 < t <= 100]
    assert max(turning) < 0.2 and min(c for t, c, _, _ in log if t > 100) > 0.9


def test_schedule_parity_on_linear_layer_gradients():
    # The weight-gradient model of the second refresh workload, G = D^T X over
    # 1024 tokens (D and X drawn on the device, G formed here in float64 and
    # rounded to bf16): the output-gradient subspace turns 1.5 rad between
    # refreshes until step 100 and then settles.
    m, n, r = 512, 1376, 64
    gen = synth.DeviceLinearLayerBatch(m, n, 1024, r, 0.99, 1e-3, 0.075, 100, seed=12, device=torch.device("cuda"))

    def draw(t):
        X, D = gen.draw(t)
        Xf = X[:, :n].double().cpu().numpy()
        Df = D[:, :m].double().cpu().numpy()
        G, Gb = synth.to_bf16(Df.T @ Xf)
        dG, ldg = upload_gradient(Gb)
        return dG, ldg, G

    log = _schedule_parity(m, n, r, 20, 200, draw)
    assert [t for t, *_ in log] == [0, 20, 40, 60, 80, 100, 120, 160]
    assert [d for *_, d in log] == [20, 20, 20, 20, 20, 20, 40, 80]
