"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a library routine, a closed form,
a brute-force computation or a hand-worked golden fixture, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand)
fails at least one of them.  No GPU needed.
"""
import ctypes
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- Philox

def _curand_host_philox(seed, count):
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "lib64", "libcurand.so")
    if not os.path.exists(path):
        pytest.skip("libcurand not found")
    lib = ctypes.CDLL(path)
    gen = ctypes.c_void_p()
    CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        out = np.zeros(count, dtype=np.uint32)
        assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(count)) == 0
    finally:
        lib.curandDestroyGenerator(gen)
    return out


@pytest.mark.parametrize("seed", [0, 1, 0x123456789ABCDEF0, 2**64 - 1])
def test_philox4x32_matches_curand_host_generator(seed):
    # cuRAND's host Philox4x32-10 emits block s as Philox(counter=(0,0,s,0), key=seed).
    blocks = 96
    ref = _curand_host_philox(seed, 4 * blocks)
    s = np.arange(blocks)
    w = O.philox4x32_10(0, 0, s, 0, seed & 0xFFFFFFFF, seed >> 32)
    got = np.stack(w, axis=1).ravel()
    np.testing.assert_array_equal(got, ref)


def test_philox_round_structure_matches_numpy_philox4x64():
    # numpy's Philox is the 4x64-10 member of the same family; its first block
    # uses counter + 1.  Same round function, other word width and constants.
    rng = np.random.default_rng(5)
    for _ in range(20):
        key = [int(x) for x in rng.integers(0, 2**63, size=2, dtype=np.int64)]
        ctr = [int(x) for x in rng.integers(0, 2**62, size=4, dtype=np.int64)]
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(ctr, dtype=np.uint64))
        raw = [int(x) for x in bg.random_raw(4)]
        ref = O.philox_generic([ctr[0] + 1] + ctr[1:], key, **O.PHILOX4x64)
        assert raw == ref


def test_philox_vectorised_equals_generic():
    rng = np.random.default_rng(9)
    c = rng.integers(0, 2**32, size=(4, 500), dtype=np.uint64)
    for key in [(0, 0), (0xFFFFFFFF, 0xFFFFFFFF), (123456789, 987654321)]:
        w = O.philox4x32_10(c[0], c[1], c[2], c[3], *key)
        for i in range(0, 500, 37):
            ref = O.philox_generic([int(c[j, i]) for j in range(4)], key, **O.PHILOX4x32)
            assert [int(w[j][i]) for j in range(4)] == ref


def test_philox_top_byte_uniform_chi2():
    e = np.arange(250_000, dtype=np.uint64)
    w = np.concatenate(O.philox4x32_10(e, 0, 7, 3, 42, 0))
    hist = np.bincount((w >> np.uint32(24)).astype(np.int64), minlength=256)
    exp = w.size / 256
    chi2 = float(((hist - exp) ** 2 / exp).sum())
    # 255 degrees of freedom: mean 255, sd ~22.6; 6 sd bound
    assert chi2 < 255 + 6 * math.sqrt(2 * 255)


# ---------------------------------------------------------------- bf16

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200_000) * np.exp2(rng.integers(-60, 60, 200_000))).astype(np.float32)
    ties = (np.arange(1, 2001, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    edge = np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 1e-40, -1e-45, np.inf, -np.inf], np.float32)
    x = np.concatenate([x, ties.view(np.float32), edge])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.bf16_bits(x), ref)


# ---------------------------------------------------------------- quantizers

def test_bf16_from_bits_matches_torch():
    # every bf16 bit pattern, decoded by torch as the reference
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = O.bf16_from_bits(bits)
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_dequant_P_bf16_is_torch_bf16_of_the_int4_product():
    rng = np.random.default_rng(12)
    m, r = 96, 64
    P = rng.standard_normal((m, r))
    packed, scales = O.quant_int4_groups(P)
    codes = O.unpack_int4(packed, m * r).reshape(m, r).astype(np.float32)
    prod = codes * np.repeat(scales.astype(np.float32), 64).reshape(m, r)   # one float32 product each
    ref = torch.from_numpy(prod).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(O.dequant_P_bf16(packed, scales, m, r), ref)


def test_proj_dims_and_adam_constants_closed_forms():
    assert O.proj_dims(O.Config(m=300, n=700, r=64)) == (300, 64, 700)
    assert O.proj_dims(O.Config(m=300, n=700, r=64, proj_side=1)) == (700, 300, 64)
    with pytest.raises(ValueError):
        O.proj_dims(O.Config(m=300, n=700, r=64, proj_side=2))
    cfg = O.Config(m=64, n=64, r=32, lr=1e-3, beta1=0.9, beta2=0.999)
    om1, om2, c1, c2 = O.adam_constants(cfg, 1)
    # t = 1: c1 = -lr / (1 - b1) and c2 = 1 / sqrt(1 - b2), with b1, b2 and lr the float32 values
    b1, b2, lr = float(np.float32(0.9)), float(np.float32(0.999)), float(np.float32(1e-3))
    assert om1 == np.float32(1 - b1) and om2 == np.float32(1 - b2)
    assert c1 == np.float32(-lr / (1 - b1)) and c2 == np.float32(1 / math.sqrt(1 - b2))
    # bias corrections vanish as t grows
    _, _, c1_inf, c2_inf = O.adam_constants(cfg, 100000)
    assert c1_inf == np.float32(-lr) and c2_inf == np.float32(1.0)


def test_refresh_due_rule():
    st, _ = _small_layer()
    st.t, st.t_next = 5, 7
    assert not O.refresh_due(st) and O.refresh_due(st, force=True)
    st.t = 7
    assert O.refresh_due(st)


def test_int4_golden_groups():
    g = json.load(open(os.path.join(GOLDEN, "int4_groups.json")))
    for case in g["cases"]:
        v = np.zeros(g["group"], np.float32)
        v[: len(case["values"])] = case["values"]
        codes, s = O.quant_int4_groups(v, g["group"])
        assert s.shape == (1,) and float(s[0]) == case["scale"]
        assert codes[: len(case["codes"])].tolist() == case["codes"]
    pk = g["packing"]
    assert O.pack_int4(np.array(pk["codes"], np.int8)).tolist() == pk["bytes"]
    assert O.unpack_int4(np.array(pk["bytes"], np.uint8), len(pk["codes"])).tolist() == pk["codes"]


def test_int4_roundtrip_bound_and_idempotence():
    rng = np.random.default_rng(2)
    m, r = 96, 32   # groups of 64 span two rows of 32
    P = O.qgalore.np.linalg.qr(rng.standard_normal((m, r)))[0].astype(np.float32)
    codes, s = O.quant_int4_groups(P)
    assert codes.min() >= -7 and codes.max() <= 7
    deq = O.dequant_int4_f32(O.pack_int4(codes), s, m, r)
    err = np.abs(deq - P).ravel()
    bound = s[np.arange(m * r) // 64] / 2 * (1 + 1e-6)
    assert np.all(err <= bound)
    codes2, s2 = O.quant_int4_groups(deq)
    np.testing.assert_array_equal(codes2, codes)
    np.testing.assert_array_equal(s2, s)
    # every group reaches +-7 at its absmax element
    g = np.abs(codes.reshape(-1, 64)).max(axis=1)
    assert np.all(g == 7)


def test_int8_rowblock_golden():
    g = json.load(open(os.path.join(GOLDEN, "int8_rowblock.json")))
    row = np.zeros((1, 256), np.float32)
    row[0, :5] = g["signed"]["row"]
    c, s = O.quant_rowblock_int8(row, g["block"])
    assert float(s[0, 0]) == g["signed"]["scale"] and c[0, :5].tolist() == g["signed"]["codes"]
    row = np.zeros((1, 256), np.float32)
    row[0, :4] = g["unsigned"]["row"]
    c, s = O.quant_rowblock_int8(row, g["block"], unsigned=True)
    assert float(s[0, 0]) == g["unsigned"]["scale"] and c[0, :4].tolist() == g["unsigned"]["codes"]
    rg = g["ragged"]
    row = np.zeros((1, rg["n"]), np.float32)
    row[0, 0] = rg["head_absmax"]
    row[0, 256:258] = rg["tail_values"]
    c, s = O.quant_rowblock_int8(row, g["block"])
    assert s.shape == (1, 2)
    assert float(s[0, 0]) == rg["head_scale"] and float(s[0, 1]) == rg["tail_scale"]
    assert c[0, 256:258].tolist() == rg["tail_codes"]


def test_zero_and_subnormal_groups_quantize_to_zero():
    x = np.zeros((2, 256), np.float32)
    x[1, 3] = np.float32(1e-39)   # subnormal absmax
    c, s = O.quant_rowblock_int8(x, 256)
    assert np.all(c == 0) and np.all(s == 0)
    q4, s4 = O.quant_int4_groups(np.full(64, 1e-40, np.float32))
    assert np.all(q4 == 0) and s4[0] == 0
    c, s = O.quant_rowblock_int8(np.full((1, 4), 2.0 ** -121, np.float32), 256)
    assert np.all(c == 0) and s[0, 0] == 0
    c, s = O.quant_rowblock_int8(np.array([[2.0 ** -120, 0.0, -2.0 ** -121]], np.float32), 256)
    assert c[0].tolist() == [127, 0, -64] and s[0, 0] > 0


def test_int8_rowblock_roundtrip():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((7, 600)) * 1e-3).astype(np.float32)
    c, s = O.quant_rowblock_int8(x, 256)
    d = O.dequant_rowblock(c, s, 256)
    cols = np.arange(600) // 256
    assert np.all(np.abs(d - x) <= s[:, cols] / 2 * (1 + 1e-6))
    c2, s2 = O.quant_rowblock_int8(d, 256)
    np.testing.assert_array_equal(c2, c)
    v = np.abs(x)
    cu, su = O.quant_rowblock_int8(v, 256, unsigned=True)
    assert cu.min() >= 0 and cu.max() == 127


# ---------------------------------------------------------------- Adam

def test_adam_matches_torch_optim_adam():
    cfg = O.Config(m=8, n=50, r=4, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8)
    rng = np.random.default_rng(4)
    shape = (4, 50)
    p = torch.zeros(shape, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.Adam([p], lr=float(np.float32(cfg.lr)),
                           betas=(float(np.float32(cfg.beta1)), float(np.float32(cfg.beta2))),
                           eps=float(np.float32(cfg.eps)))
    m0 = np.zeros(shape, np.float32)
    v0 = np.zeros(shape, np.float32)
    # magnitudes from 1e-9 (epsilon matters) to 1
    scale = np.exp2(rng.integers(-30, 0, size=shape)).astype(np.float32)
    for t in range(1, 8):
        R = (rng.standard_normal(shape).astype(np.float32) * scale).astype(np.float32)
        before = p.detach().clone()
        p.grad = torch.from_numpy(R.astype(np.float64))
        opt.step()
        ref = (p.detach() - before).numpy()
        N, m0, v0 = O.adam_moments(R, m0, v0, cfg, t)
        np.testing.assert_allclose(N, ref, rtol=1e-4, atol=1e-9)


def test_adam_first_step_closed_form():
    cfg = O.Config(m=8, n=300, r=4)
    rng = np.random.default_rng(6)
    R = (rng.standard_normal((4, 300)) * 1e-2).astype(np.float32)
    z8 = np.zeros((4, 300), np.int8)
    z = np.zeros((4, 2), np.float32)
    N, Mq, sM, Vq, sV = O.lowrank_adam_int8(R, z8, z, z8, z, cfg, 1)
    # t = 1, zero moments: m_hat = R, v_hat = R^2, N = -lr R / (|R| + eps)
    ref = -np.float64(np.float32(cfg.lr)) * R / (np.abs(R.astype(np.float64)) + np.float32(cfg.eps))
    np.testing.assert_allclose(N, ref, rtol=2 ** -8)
    assert np.all(np.sign(N) == -np.sign(R))
    # second moment codes are non-negative, first-moment codes carry R's sign
    assert Vq.min() >= 0
    assert np.all((Mq == 0) | (np.sign(Mq) == np.sign(R)))


def test_int8_moments_keep_adam_step_bound():
    # Adam's normalised step obeys |m_hat / sqrt(v_hat)| <= (1 - b1) / sqrt(1 - b2)
    # (Kingma and Ba, section 2.1); the INT8 moment grids must not break it.
    import synth
    cfg = O.Config(m=512, n=512, r=128, seed=4)
    st = O.LayerState.create(cfg, synth.weight_codes(512, 512, 4), synth.weight_scales(512, 512, seed=4))
    gen = synth.lowrank_gradient(512, 512, rank=256, seed=4)
    O.set_projection(st, O.exact_topr(gen.draw(0)[0], 128)[0])
    bound = np.float32(cfg.lr) * (1 - np.float32(cfg.beta1)) / math.sqrt(1 - np.float32(cfg.beta2))
    for t in range(6):
        inter = O.step(st, gen.draw(t)[0])
        assert np.abs(inter["N"]).max() <= bound * 1.01


def test_second_moment_grid_is_sqrt_of_v():
    rng = np.random.default_rng(21)
    R = (rng.standard_normal((3, 300)) * np.exp2(rng.integers(-12, 0, (3, 300)))).astype(np.float32)
    cfg = O.Config(m=8, n=300, r=3)
    z8 = np.zeros((3, 300), np.int8)
    z = np.zeros((3, 2), np.float32)
    _, _, _, Vq, sV = O.lowrank_adam_int8(R, z8, z, z8, z, cfg, 1)
    v = (np.float32(1 - np.float32(cfg.beta2)) * (R * R)).astype(np.float32)
    root = np.sqrt(v)
    cols = np.arange(300) // 256
    assert np.all(np.abs(O.dequant_rowblock(Vq, sV) - root) <= sV[:, cols] / 2 * (1 + 1e-6))
    np.testing.assert_allclose(O.dequant_second_moment(Vq, sV), O.dequant_rowblock(Vq, sV) ** 2, rtol=1e-6)


# ---------------------------------------------------------------- projections

def test_project_and_backproject_brute_force():
    rng = np.random.default_rng(7)
    m, n, r = 6, 9, 3
    P = O.bf16_round(rng.standard_normal((m, r)).astype(np.float32))
    G = O.bf16_round(rng.standard_normal((m, n)).astype(np.float32))
    N = O.bf16_round(rng.standard_normal((r, n)).astype(np.float32))
    R = O.project(P, G)
    U = O.backproject(P, N)
    assert R.shape == (r, n) and U.shape == (m, n)
    for a in range(r):
        for j in range(n):
            s = math.fsum(float(P[i, a]) * float(G[i, j]) for i in range(m))
            assert R[a, j] == np.float32(s)
    for i in range(m):
        for j in range(n):
            s = math.fsum(float(P[i, a]) * float(N[a, j]) for a in range(r))
            assert U[i, j] == np.float32(s)


# ---------------------------------------------------------------- stochastic rounding

def _sr(Wq, sW, U, alpha=1.0, seed=0, t=1, layer=0):
    m, n = Wq.shape
    cfg = O.Config(m=m, n=n, r=1, alpha=alpha, seed=seed, layer_id=layer)
    return O.stochastic_round_update(Wq, sW, U, cfg, t)


@pytest.mark.parametrize("x", [0.1, 0.5, 0.9, 0.01, 1e-3, -0.3, 2.75])
def test_sr_unbiased_over_a_million_draws(x):
    m, n = 1000, 1000
    W = np.zeros((m, n), np.int8)
    sW = np.ones(-(-m * n // 256), np.float32)
    U = np.full((m, n), x, np.float32)
    out = _sr(W, sW, U, seed=11, t=3)
    f = math.floor(np.float32(x))
    phi = float(np.float32(x)) - f
    mean = out.astype(np.float64).mean()
    sd = math.sqrt(max(phi * (1 - phi), 1e-12) / (m * n))
    # the draws' mean is within 5 sd of x, plus the 2^-17 code of the nearest-point
    # rounding of the update onto the 2^-16 draw grid
    assert abs(mean - float(np.float32(x))) <= 5 * sd + 2 ** -17
    assert set(np.unique(out).tolist()) <= {f, f + 1}


def test_sr_integers_fixed_clamp_and_zero_scale():
    rng = np.random.default_rng(8)
    W = rng.integers(-120, 121, size=(64, 64)).astype(np.int8)
    sW = np.full(16, 0.5, np.float32)
    np.testing.assert_array_equal(_sr(W, sW, np.zeros((64, 64), np.float32)), W)
    # x = U * alpha / s = 3 exactly
    np.testing.assert_array_equal(_sr(W, sW, np.full((64, 64), 1.5, np.float32)), W + 3)
    top = np.full((8, 32), 127, np.int8)
    assert np.all(_sr(top, np.ones(1, np.float32), np.full((8, 32), 5.0, np.float32)) == 127)
    assert np.all(_sr(-top, np.ones(1, np.float32), np.full((8, 32), -5.0, np.float32)) == -127)
    sW0 = np.ones(16, np.float32)
    sW0[3] = 0
    out = _sr(W, sW0, np.full((64, 64), 7.0, np.float32))
    flat_w, flat_o = W.ravel(), out.ravel()
    np.testing.assert_array_equal(flat_o[3 * 256:4 * 256], flat_w[3 * 256:4 * 256])


def test_sr_group_index_is_flattened_logical():
    # n = 100 (not a multiple of 256): groups straddle rows; scale g applies to e // 256
    m, n = 10, 100
    sW = np.arange(1, 5, dtype=np.float32)   # ceil(1000/256) = 4 groups
    U = np.ones((m, n), np.float32)
    W = np.zeros((m, n), np.int8)
    out = _sr(W, sW, U * 12.0, alpha=1.0)
    e = np.arange(m * n).reshape(m, n)
    expect = 12.0 / sW[e // 256]
    assert np.all(np.abs(out - expect) < 1.0)


@pytest.mark.parametrize("X", [0.0, 1.0, 0.25, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 32767.5, 65535.25, 65536.0,
                               98304.75, -1.0, -65536.0, -70000.1, 3.0e6, -3.0e6 + 0.5])
def test_sr_exhaustive_over_the_draw_space(X):
    # alpha = 1, s_g = 2^16: c' = 1, so the update in units of 2^-16 code is X itself.
    # Over all 2^16 draws the rounded result takes only the two neighbouring codes,
    # and the draws sum to rint(X) exactly (nearest integer, ties to even): the mean
    # is X / 2^16 rounded to the nearest point of the draw grid.  A ceiling or a
    # floor in place of the nearest point, a missing draw or an off-by-one in the
    # shift changes the sum (the ties 0.5, 1.5, 2.5, -0.5, -1.5, -2.5 and 32767.5
    # each separate rint from ceil, floor and round-half-away).
    W = np.zeros((256, 256), np.int8)
    sW = np.full(256, 65536.0, np.float32)
    U = np.full((256, 256), X, np.float32)
    cfg = O.Config(m=256, n=256, r=1, alpha=1.0)
    out = O.stochastic_round_update(W, sW, U, cfg, 1, u16=np.arange(65536, dtype=np.uint32).reshape(256, 256))
    Xf = float(np.float32(X))
    lo = math.floor(Xf / 65536.0)
    assert set(np.unique(out).tolist()) <= {lo, lo + 1}
    assert int(out.astype(np.int64).sum()) == round(Xf)      # Python's round: ties to even


def _draw_space_sums(X):
    """For each value of X (the update in units of 2^-16 code), the sum of the
    oracle's code changes over all 2^16 draws: one row of 2^16 elements per value."""
    X = np.asarray(X, np.float32)
    out = np.empty(X.size, np.int64)
    rows = 32
    d = np.tile(np.arange(65536, dtype=np.uint32), (rows, 1))
    for b in range(0, X.size, rows):
        x = X[b:b + rows]
        m = x.size
        W = np.zeros((m, 65536), np.int8)
        sW = np.full(m * 256, 65536.0, np.float32)
        U = np.repeat(x[:, None], 65536, axis=1)
        cfg = O.Config(m=m, n=65536, r=1, alpha=1.0)
        q = O.stochastic_round_update(W, sW, U, cfg, 1, u16=d[:m])
        out[b:b + m] = q.astype(np.int64).sum(axis=1)
    return out


def _dense_update_grid():
    # fractions i / 256 on both sides of integers of both parities and signs
    f = np.arange(256, dtype=np.float64) / 256.0
    return np.concatenate([k + f for k in (-3.0, -2.0, 2.0, 3.0, 1000.0, 1001.0)]).astype(np.float32)


def test_sr_expected_update_is_odd_in_the_update():
    # E[xi(-x)] = -E[xi(x)] exactly over the whole draw space, for non-integer
    # updates too: an update and its negation move the weight by opposite amounts
    # on average.  A ceiling (or floor) on the draw grid fails at every
    # non-integer X: ceil(X) + ceil(-X) = 1 there.
    X = _dense_update_grid()
    X = X[X != np.rint(X)]
    np.testing.assert_array_equal(_draw_space_sums(X) + _draw_space_sums(-X), 0)


def test_sr_no_drift_over_a_dense_grid_of_updates():
    # The exact expected change (sum over all draws) minus the update, averaged
    # over a dense grid of fractional parts, is zero: the residue of the
    # nearest-point rounding has no sign.  Each value is also within half a draw
    # step of its update.  A ceiling leaves a mean residue of +1/2 step.
    X = _dense_update_grid()
    res = _draw_space_sums(X).astype(np.float64) - X.astype(np.float64)
    assert np.max(np.abs(res)) <= 0.5
    assert abs(res.mean()) <= 1e-12


def test_sr_nan_keeps_code_inf_and_huge_saturate():
    W = np.array([[5, -5, 100, -100, 0, 7, -7, 3]], np.int8)
    sW = np.ones(1, np.float32)
    U = np.array([[np.nan, np.nan, np.inf, -np.inf, 1e30, -1e30, 2.0 ** 31, 0.0]], np.float32)
    out = O.stochastic_round_update(W, sW, U, O.Config(m=1, n=8, r=1, alpha=1.0), 1,
                                    u16=np.full((1, 8), 12345, np.uint32))
    np.testing.assert_array_equal(out, [[5, -5, 127, -127, 127, -127, 127, 3]])
    # an overflowing alpha / s (c' = inf): a zero update stays a NaN -> kept; nonzero saturates
    tiny = np.full(1, 1e-38, np.float32)
    out = O.stochastic_round_update(np.array([[4, 4]], np.int8), tiny, np.array([[0.0, 1e-3]], np.float32),
                                    O.Config(m=1, n=2, r=1, alpha=1.0), 1, u16=np.zeros((1, 2), np.uint32))
    np.testing.assert_array_equal(out, [[4, 127]])


def test_sr_uniform_draw_mapping():
    # element (i, j): half (j mod 2) of word ((j / 2) mod 4) of Philox(j / 8, i, t, layer)
    u = O.sr_uniform16(3, 21, seed=(5 << 32) | 77, t=2, layer_id=9)
    for (i, j) in [(0, 0), (0, 1), (0, 7), (1, 8), (2, 13), (2, 20)]:
        w = O.philox_generic([j // 8, i, 2, 9], [77, 5], **O.PHILOX4x32)[(j // 2) % 4]
        assert int(u[i, j]) == (w >> (16 * (j % 2))) & 0xFFFF
    assert u.max() < 2 ** 16
    # rows draw independent streams: the same column of two rows differs
    assert (u[0] != u[1]).mean() > 0.9


def test_sr_small_updates_keep_their_mean():
    # an update far below one code (x = 1e-3) is kept on average, not rounded away
    m, n = 1000, 1000
    out = _sr(np.zeros((m, n), np.int8), np.ones(-(-m * n // 256), np.float32),
              np.full((m, n), 1e-3, np.float32), seed=5)
    assert abs(out.mean() - 1e-3) < 5 * np.sqrt(1e-3 / (m * n)) + 2 ** -17


# ---------------------------------------------------------------- re-scaling instead of saturating

def test_rescale_equals_saturating_inside_the_grid():
    # nothing reaches +-127: codes are those of the saturating form, scales unchanged
    rng = np.random.default_rng(21)
    W = rng.integers(-100, 101, size=(16, 512)).astype(np.int8)
    sW = rng.uniform(0.005, 0.02, 32).astype(np.float32)
    U = (rng.standard_normal((16, 512)) * 0.05).astype(np.float32)
    U[3, 7] = np.nan
    cfg = O.Config(m=16, n=512, r=1, alpha=0.5, seed=3)
    q, s2 = O.stochastic_round_rescale(W, sW, U, cfg, 4)
    np.testing.assert_array_equal(q, O.stochastic_round_update(W, sW, U, cfg, 4))
    np.testing.assert_array_equal(s2, sW)
    assert q[3, 7] == W[3, 7]


@pytest.mark.parametrize("q0,X", [(127, 1.0), (120, 8 * 65536 + 0.5), (100, 2.0 ** 29), (-127, -1.0),
                                  (-90, -100 * 65536 - 12345.25), (0, 2.0 ** 31)])
def test_rescale_exhaustive_over_the_draw_space(q0, X):
    # alpha = 1, s_g = 2^16: c' = 1, so every element of the 256 x 256 array has the
    # same value T = q0 2^16 + rint(X) (X clipped to 2^30) in units of 2^-16 code,
    # outside the grid, and meets each 16-bit draw once.  Every group is re-scaled
    # to the same s', so the codes' sum over the draws is their exact mean: the
    # value q0 s + X 2^-16 s must come back as sum / 2^16 * s' up to float32
    # rounding (4 roundings) and the 2^-16 draw grid.  Every code lands on the top
    # of the new grid (126 or 127 in magnitude) and s' = s |T| / (127 2^16).
    W = np.full((256, 256), q0, np.int8)
    sW = np.full(256, 65536.0, np.float32)
    U = np.full((256, 256), X, np.float32)
    cfg = O.Config(m=256, n=256, r=1, alpha=1.0)
    q, s2 = O.stochastic_round_rescale(W, sW, U, cfg, 1, u16=np.arange(65536, dtype=np.uint32).reshape(256, 256))
    T = q0 * 65536 + round(max(-2.0 ** 30, min(2.0 ** 30, float(np.float32(X)))))
    assert abs(T) > 127 * 65536
    assert np.all(s2 == s2[0]) and s2[0] > sW[0]
    assert abs(float(s2[0]) - 65536.0 * abs(T) / (127 * 65536)) <= 3e-7 * float(s2[0])
    assert set(np.abs(np.unique(q)).tolist()) <= {126, 127}
    mean_value = int(q.astype(np.int64).sum()) / 65536.0 * float(s2[0])
    target = T / 65536.0 * 65536.0
    assert abs(mean_value - target) <= 5e-7 * abs(target) + 2.0 ** -16 * float(s2[0])


def test_rescale_keeps_each_element_unbiased():
    # one outlier per group pushes its group off the grid; every other element of
    # the group must keep its value q s + alpha U on average over the draws
    m, n, draws = 4, 256, 1500
    rng = np.random.default_rng(5)
    W = rng.integers(-60, 61, size=(m, n)).astype(np.int8)
    sW = np.full(m, 0.01, np.float32)
    U = (rng.standard_normal((m, n)) * 0.2).astype(np.float32)
    U[:, 17] = 3.0                     # q + 300 codes: far off the grid
    cfg = O.Config(m=m, n=n, r=1, alpha=1.0, seed=9)
    acc = np.zeros((m, n))
    acc2 = np.zeros((m, n))
    for t in range(draws):
        q, s2 = O.stochastic_round_rescale(W, sW, U, cfg, t)
        v = q.astype(np.float64) * s2[:, None]
        acc += v
        acc2 += v * v
    assert np.all(s2 > sW)
    mean = acc / draws
    sd = np.sqrt(np.maximum(acc2 / draws - mean ** 2, 0) / draws)
    expect = W.astype(np.float64) * np.float64(sW[:, None]) + np.float64(U)
    use = sd > 1e-4
    z = ((mean - expect) / np.where(use, sd, 1))[use]
    assert z.size > 0.9 * m * n
    assert abs(z.mean()) < 5 / math.sqrt(z.size)
    assert (z ** 2).mean() < 1.3
    # a saturating update loses the outlier's value; the re-scaled one keeps it
    assert np.all(np.abs(mean[:, 17] - expect[:, 17]) < 0.02 * np.abs(expect[:, 17]))


def test_rescale_zero_scale_nan_and_mixed_groups():
    # group 0: zero scale (frozen); group 1: leaves the grid; group 2: stays inside
    W = np.zeros((3, 256), np.int8)
    W[1, 0], W[2, 0] = 126, 5
    sW = np.array([0.0, 1.0, 1.0], np.float32)
    U = np.zeros((3, 256), np.float32)
    U[0] = 50.0
    U[1, 0], U[1, 1] = 3.0, np.nan
    U[2, 1] = 0.5
    cfg = O.Config(m=3, n=256, r=1, alpha=1.0)
    q, s2 = O.stochastic_round_rescale(W, sW, U, cfg, 2, u16=np.full((3, 256), 40000, np.uint32))
    np.testing.assert_array_equal(q[0], W[0])
    assert s2[0] == 0 and s2[2] == 1
    # group 1: T_max = 129 2^16, rho = 127/129, s' = 129/127; the outlier lands on 127
    assert s2[1] == np.float32(np.float32(1.0) / np.float32(np.float32(127 * 65536) / np.float32(129 * 65536)))
    assert q[1, 0] == 127 and np.all(q[1, 1:] == 0)   # zeros (and the NaN's zero) stay zero
    np.testing.assert_array_equal(q[2], O.stochastic_round_update(W[2:], sW[2:], U[2:], O.Config(m=1, n=256, r=1, alpha=1.0), 2,
                                                                  u16=np.full((1, 256), 40000, np.uint32))[0])


def test_rescale_step_with_small_alpha_equals_saturating_step():
    import synth
    m, n, r = 64, 256, 16
    base = dict(m=m, n=n, r=r, alpha=0.25, seed=4)
    out = []
    for wr in (0, 1):
        st = O.LayerState.create(O.Config(**base, w_rescale=wr), np.clip(synth.weight_codes(m, n, 4), -100, 100),
                                 synth.weight_scales(m, n, seed=4))
        O.set_projection(st, synth.orthonormal(m, r, 4))
        gen = synth.lowrank_gradient(m, n, rank=8, seed=4)
        for t in range(3):
            O.step(st, gen.draw(t)[0])
        out.append((st.Wq.copy(), st.sW.copy()))
    sat = np.abs(out[0][0]) == 127
    assert not sat.any()
    np.testing.assert_array_equal(out[0][0], out[1][0])
    np.testing.assert_array_equal(out[0][1], out[1][1])


# ---------------------------------------------------------------- composed step

def _small_layer(m=64, n=96, r=32, seed=0, alpha=0.25):
    import synth
    cfg = O.Config(m=m, n=n, r=r, alpha=alpha, seed=seed)
    st = O.LayerState.create(cfg, synth.weight_codes(m, n, seed), synth.weight_scales(m, n, seed=seed))
    O.set_projection(st, synth.orthonormal(m, r, seed))
    gen = synth.lowrank_gradient(m, n, rank=16, seed=seed)
    return st, gen


def test_step_alpha_zero_keeps_weights():
    st, gen = _small_layer(alpha=0.0)
    W0 = st.Wq.copy()
    for t in range(3):
        G, _ = gen.draw(t)
        O.step(st, G)
    np.testing.assert_array_equal(st.Wq, W0)
    assert np.abs(st.Mq).max() > 0 and st.Vq.max() > 0


def test_step_mean_update_is_alpha_P_N_over_scale():
    base, gen = _small_layer()
    G, _ = gen.draw(0)
    diffs = []
    for seed in range(200):
        st = O.LayerState.create(O.Config(**{**base.cfg.__dict__, "seed": seed}), base.Wq, base.sW)
        st.Pq, st.sP = base.Pq, base.sP
        inter = O.step(st, G)
        diffs.append(st.Wq.astype(np.float64) - base.Wq)
    mean = np.mean(diffs, axis=0)
    m, n = base.Wq.shape
    e = np.arange(m * n).reshape(m, n)
    expect = np.float64(base.cfg.alpha) * inter["U"] / base.sW[e // 256]
    y = base.Wq.astype(np.float64) + expect
    phi = y - np.floor(y)
    sd = np.sqrt(phi * (1 - phi) / len(diffs))
    use = (np.abs(y) < 126) & (sd > 0.01)
    z = ((mean - expect) / np.where(use, sd, 1))[use]
    # standardized errors: no bias, unit variance (a wrong factor or index fails)
    assert abs(z.mean()) < 5 / math.sqrt(z.size)
    assert 0.8 < (z ** 2).mean() < 1.2


# ---------------------------------------------------------------- CosSim

def test_cossim_closed_forms():
    rng = np.random.default_rng(10)
    m, r = 40, 6
    P = np.linalg.qr(rng.standard_normal((m, r)))[0]
    Orot = np.linalg.qr(rng.standard_normal((r, r)))[0]
    assert abs(O.cossim(P, P) - 1) < 1e-12
    assert abs(O.cossim(P, P @ Orot) - 1) < 1e-12
    Pfull = np.linalg.qr(rng.standard_normal((m, 2 * r)))[0]
    assert abs(O.cossim(Pfull[:, :r], Pfull[:, r:])) < 1e-12
    theta = np.linspace(0.0, 1.4, r)
    A = np.zeros((m, r))
    B = np.zeros((m, r))
    A[np.arange(r), np.arange(r)] = 1
    B[np.arange(r), np.arange(r)] = np.cos(theta)
    B[r + np.arange(r), np.arange(r)] = np.sin(theta)
    assert abs(O.cossim(A, B) - np.cos(theta).mean()) < 1e-12


def test_cossim_matches_scipy_subspace_angles():
    rng = np.random.default_rng(12)
    for m, r in [(30, 5), (64, 16)]:
        A = np.linalg.qr(rng.standard_normal((m, r)))[0]
        B = np.linalg.qr(A + 0.3 * rng.standard_normal((m, r)))[0]
        ang = scipy.linalg.subspace_angles(A, B)
        assert abs(O.cossim(A, B) - np.cos(ang).mean()) < 1e-10


# ---------------------------------------------------------------- refresh (randomized SVD)

def test_randomized_topr_full_width_equals_exact_svd():
    rng = np.random.default_rng(13)
    m, n, r = 40, 24, 5
    G = rng.standard_normal((m, n)) * np.exp(-np.arange(n) / 3)[None, :]
    k = min(m, n)
    Om = O.rademacher_omega(n, k, 1, 0, 0)
    P, s = O.randomized_topr(G, r, k, 2, Om)
    Pe, se = O.exact_topr(G, r)
    np.testing.assert_allclose(s, se, rtol=1e-10)
    np.testing.assert_allclose(P, Pe, atol=1e-9)


def test_randomized_topr_gap_input_matches_exact_subspace():
    import synth
    G, _ = synth.gap_gradient(200, 150, 12, seed=3)
    cfg = O.Config(m=200, n=150, r=12)
    Om = O.rademacher_omega(150, O.refresh_width(cfg), 5, 0, 0)
    P, s = O.randomized_topr(G, 12, O.refresh_width(cfg), 2, Om)
    Pe, se = O.exact_topr(G, 12)
    cos = np.cos(scipy.linalg.subspace_angles(P, Pe))
    assert cos.min() > 0.99999
    np.testing.assert_allclose(s, se, rtol=1e-6)
    np.testing.assert_allclose(P.T @ P, np.eye(12), atol=1e-12)


def test_randomized_range_exact_on_rank_k_input():
    rng = np.random.default_rng(14)
    m, n, k = 60, 50, 8
    G = rng.standard_normal((m, k)) @ rng.standard_normal((k, n))
    Om = O.rademacher_omega(n, k, 2, 0, 0)
    P, _ = O.randomized_topr(G, k, k, 0, Om)
    # P spans range(G) exactly
    resid = G - P @ (P.T @ G)
    assert np.abs(resid).max() < 1e-9 * np.abs(G).max()


def test_canonical_signs_rule():
    P = np.array([[0.1, -0.9], [-0.8, 0.2], [0.3, 0.9]])
    C = O.canonical_signs(P)
    np.testing.assert_array_equal(C[:, 0], -P[:, 0])   # largest |.| is -0.8 -> flip
    np.testing.assert_array_equal(C[:, 1], -P[:, 1])   # tie 0.9: first row (-0.9) decides


def test_omega_rademacher_mapping():
    n, k = 37, 11
    Om = O.rademacher_omega(n, k, seed=0xABCDEF0123, refresh_idx=4, layer_id=6)
    assert set(np.unique(Om).tolist()) <= {-1.0, 1.0}
    for e in [0, 31, 32, 127, 128, 300, n * k - 1]:
        w = O.philox_generic([e // 128, 4, 6, 0],
                             [(0xABCDEF0123 & 0xFFFFFFFF) ^ O.OMEGA_KEY_SALT, 0xABCDEF0123 >> 32],
                             **O.PHILOX4x32)[(e // 32) % 4]
        bit = (w >> (e % 32)) & 1
        assert Om.ravel()[e] == (-1.0 if bit else 1.0)
    big = O.rademacher_omega(1000, 400, 1, 0, 0)
    assert abs(big.mean()) < 5 / math.sqrt(big.size)
    assert not np.array_equal(big, O.rademacher_omega(1000, 400, 1, 1, 0))


# ---------------------------------------------------------------- schedule

def test_schedule_doubling_rule_scripted():
    seq = [None, 0.5, 0.3, 0.41, 0.4, 0.9]
    t, delta, log = 0, 200, []
    for cs in seq:
        delta, t_next = O.schedule_after_refresh(t, delta, cs, 0.4)
        log.append((t, delta, t_next))
        t = t_next
    assert log == [(0, 200, 200), (200, 400, 600), (600, 400, 1000),
                   (1000, 800, 1800), (1800, 800, 2600), (2600, 1600, 4200)]


def test_schedule_gamma_limits():
    # gamma > 1: CosSim <= 1 never exceeds it -> GaLore's fixed interval
    t, delta = 0, 50
    for cs in [None, 1.0, 0.99, 1.0]:
        delta, t = O.schedule_after_refresh(t, delta, cs, 1.5)
    assert delta == 50 and t == 200
    t, delta = 0, 50
    for cs in [None, 0.0, 0.1]:
        delta, t = O.schedule_after_refresh(t, delta, cs, -1.5)
    assert delta == 200 and t == 50 + 100 + 200


def test_refresh_layer_state_flow():
    import synth
    m, n, r = 64, 80, 8
    cfg = O.Config(m=m, n=n, r=r, delta0=3, gamma=0.4, seed=1)
    st = O.LayerState.create(cfg, synth.weight_codes(m, n), synth.weight_scales(m, n))
    gen = synth.lowrank_gradient(m, n, rank=8, s0=1.0, decay=0.7, sigma=1e-4, seed=1)
    counts = []
    for t in range(10):
        G, _ = gen.draw(t)
        info = O.refresh(st, G, force=(t == 0))
        counts.append(info is not None)
        O.step(st, G)
    # refreshes at t = 0, 3 (cs ~ 1 -> delta 6), 9
    assert counts == [True, False, False, True, False, False, False, False, False, True]
    assert st.cossim_trace[0][1] is None and st.cossim_trace[1][1] > 0.9
    assert st.n_refresh == 3


# ---------------------------------------------------------------- linear layers (INT8 weights)

def test_dequant_weight_matches_torch_bf16_of_the_fp32_product():
    # each element is one float32 product rounded by torch's float32 -> bf16 RNE;
    # the group of (i, j) is floor((i n + j) / 256), with n = 300 so that groups
    # straddle rows
    rng = np.random.default_rng(11)
    m, n = 5, 300
    Wq = rng.integers(-127, 128, size=(m, n)).astype(np.int8)
    ng = -(-(m * n) // 256)
    sW = (rng.uniform(0.5, 1.5, size=ng) * 3.7e-3).astype(np.float32)
    got = O.dequant_weight_bf16(Wq, sW)
    for i in range(m):
        for j in range(n):
            p = np.float32(np.float32(Wq[i, j]) * sW[(i * n + j) // 256])
            ref = torch.tensor([float(p)], dtype=torch.float32).to(torch.bfloat16).to(torch.float32).item()
            assert got[i, j] == np.float32(ref), (i, j)


def test_dequant_weight_exact_cases():
    # unit scales give the codes; power-of-two scales give q * s with no rounding
    Wq = np.arange(-127, 128, dtype=np.int64).reshape(5, 51).astype(np.int8)
    assert np.array_equal(O.dequant_weight_bf16(Wq, np.ones(1, np.float32)), Wq.astype(np.float32))
    s = np.float32(2.0 ** -9)
    assert np.array_equal(O.dequant_weight_bf16(Wq, np.array([s], np.float32)), Wq.astype(np.float32) * s)
    # a zero scale gives zeros
    assert not O.dequant_weight_bf16(Wq, np.zeros(1, np.float32)).any()


def test_linear_products_brute_force_and_integer_exact():
    rng = np.random.default_rng(12)
    T, m, n = 4, 3, 5
    X = rng.standard_normal((T, n)).astype(np.float32)
    dY = rng.standard_normal((T, m)).astype(np.float32)
    Wt = rng.standard_normal((m, n)).astype(np.float32)
    Y, dX, G = O.linear_forward(X, Wt), O.linear_backward_data(dY, Wt), O.linear_backward_weight(dY, X)
    assert Y.shape == (T, m) and dX.shape == (T, n) and G.shape == (m, n)
    for t in range(T):
        for i in range(m):
            assert Y[t, i] == math.fsum(float(X[t, j]) * float(Wt[i, j]) for j in range(n))
        for j in range(n):
            assert dX[t, j] == math.fsum(float(dY[t, i]) * float(Wt[i, j]) for i in range(m))
    for i in range(m):
        for j in range(n):
            assert G[i, j] == math.fsum(float(dY[t, i]) * float(X[t, j]) for t in range(T))
    # integer inputs: the products equal integer matrix products exactly
    Xi = rng.integers(-50, 50, size=(7, 11))
    Wi = rng.integers(-127, 128, size=(6, 11))
    Di = rng.integers(-50, 50, size=(7, 6))
    assert np.array_equal(O.linear_forward(Xi, Wi), (Xi @ Wi.T).astype(np.float64))
    assert np.array_equal(O.linear_backward_data(Di, Wi), (Di @ Wi).astype(np.float64))
    assert np.array_equal(O.linear_backward_weight(Di, Xi), (Di.T @ Xi).astype(np.float64))


# ---------------------------------------------------------------- moments at a refresh

def _state_with_moments(m=64, n=300, r=32, policy=2, seed=5):
    cfg = O.Config(m=m, n=n, r=r, seed=seed, mom_refresh=policy)
    rng = np.random.default_rng(seed)
    st = O.LayerState.create(cfg, np.zeros((m, n), np.int8), np.ones(-(-m * n // 256), np.float32))
    mom = rng.standard_normal((r, n)).astype(np.float32) * 1e-3
    st.Mq, st.sM = O.quant_rowblock_int8(mom, 256)
    st.Vq, st.sV = O.quant_rowblock_int8(np.abs(mom) * 2, 256, unsigned=True)
    return st


def test_refresh_moments_reset_and_keep():
    st = _state_with_moments(policy=1)
    P = synth.orthonormal(64, 32, seed=1)
    O.refresh_moments(st, P, P)
    assert not st.Mq.any() and not st.Vq.any() and not st.sM.any() and not st.sV.any()
    st = _state_with_moments(policy=0)
    before = (st.Mq.copy(), st.sM.copy(), st.Vq.copy(), st.sV.copy())
    O.refresh_moments(st, P, synth.orthonormal(64, 32, seed=2))
    for a, b in zip(before, (st.Mq, st.sM, st.Vq, st.sV)):
        assert np.array_equal(a, b)


def test_refresh_moments_rotation_identity_and_permutation():
    # the same basis (C = I) reproduces the codes: quantizing a dequantized array
    # gives its codes back
    st = _state_with_moments()
    Mq, sM, Vq, sV = st.Mq.copy(), st.sM.copy(), st.Vq.copy(), st.sV.copy()
    P = synth.orthonormal(64, 32, seed=1)
    O.refresh_moments(st, P, P)
    assert np.array_equal(st.Mq, Mq) and np.array_equal(st.Vq, Vq)
    # a new basis that permutes the old columns permutes the moment rows: the new
    # column a is old column perm[a], so new row a of m is old row perm[a]; the
    # second moment's codes follow exactly (C o C is the same permutation)
    st = _state_with_moments()
    m_old = O.dequant_rowblock(st.Mq, st.sM)
    Vq_old = st.Vq.copy()
    perm = np.random.default_rng(3).permutation(32)
    O.refresh_moments(st, P[:, perm], P)
    np.testing.assert_allclose(O.dequant_rowblock(st.Mq, st.sM), m_old[perm], rtol=0, atol=1e-9)
    assert np.array_equal(st.Vq, Vq_old[perm])
    # sign flips of new columns: m rows flip sign, v is unchanged (C o C = I)
    st = _state_with_moments()
    m_old, Vq_old = O.dequant_rowblock(st.Mq, st.sM), st.Vq.copy()
    flip = np.where(np.arange(32) % 3 == 0, -1.0, 1.0)
    O.refresh_moments(st, P * flip[None, :], P)
    np.testing.assert_allclose(O.dequant_rowblock(st.Mq, st.sM), m_old * flip[:, None], rtol=0, atol=1e-9)
    assert np.array_equal(st.Vq, Vq_old)


# ---------------------------------------------------------------- right-side projection (P n x r)

def test_right_side_products_brute_force():
    rng = np.random.default_rng(17)
    m, n, r = 7, 5, 3
    P = O.bf16_round(rng.standard_normal((n, r)).astype(np.float32))
    G = O.bf16_round(rng.standard_normal((m, n)).astype(np.float32))
    N = O.bf16_round(rng.standard_normal((m, r)).astype(np.float32))
    R, U = O.project_right(G, P), O.backproject_right(N, P)
    assert R.shape == (m, r) and U.shape == (m, n)
    for i in range(m):
        for a in range(r):
            assert R[i, a] == np.float32(math.fsum(float(G[i, j]) * float(P[j, a]) for j in range(n)))
        for j in range(n):
            assert U[i, j] == np.float32(math.fsum(float(N[i, a]) * float(P[j, a]) for a in range(r)))


def test_right_side_refresh_finds_the_right_singular_vectors():
    # a gap input with m > n: the right-side refresh returns P (n x r) spanning
    # the top-r right singular vectors that LAPACK's SVD gives
    m, n, r = 160, 96, 32
    G, _ = synth.gap_gradient(m, n, r, seed=31)
    cfg = O.Config(m=m, n=n, r=r, seed=3, proj_side=1)
    st = O.LayerState.create(cfg, np.zeros((m, n), np.int8), np.ones(-(-m * n // 256), np.float32))
    assert st.Mq.shape == (m, r) and st.sM.shape == (m, 1)
    out = O.refresh(st, G, force=True)
    P = out["P"]
    assert P.shape == (n, r)
    Vt = np.linalg.svd(np.asarray(G, np.float64), full_matrices=False)[2]
    cos = np.cos(scipy.linalg.subspace_angles(P, Vt[:r].T))
    assert cos.min() > 0.999


def test_right_side_moment_rotation_permutes_columns():
    m, n, r = 300, 64, 32
    cfg = O.Config(m=m, n=n, r=r, seed=5, mom_refresh=2, proj_side=1)
    rng = np.random.default_rng(5)
    st = O.LayerState.create(cfg, np.zeros((m, n), np.int8), np.ones(-(-m * n // 256), np.float32))
    mom = rng.standard_normal((m, r)).astype(np.float32) * 1e-3
    st.Mq, st.sM = O.quant_rowblock_int8(mom, 256)
    st.Vq, st.sV = O.quant_rowblock_int8(np.abs(mom) * 2, 256, unsigned=True)
    m_old, Vq_old = O.dequant_rowblock(st.Mq, st.sM), st.Vq.copy()
    P = synth.orthonormal(n, r, seed=1)
    perm = np.random.default_rng(4).permutation(r)
    O.refresh_moments(st, P[:, perm], P)
    np.testing.assert_allclose(O.dequant_rowblock(st.Mq, st.sM), m_old[:, perm], rtol=0, atol=1e-9)
    assert np.array_equal(st.Vq, Vq_old[:, perm])
