"""The C-ABI library on the CPU: it loads, exports every entry point the header
declares, and its host-only logic (sizes, validation, the refresh schedule)
behaves as specified.  Nothing here launches a kernel."""
import os
import re
from ctypes import byref, c_int32, c_int64, c_void_p

import pytest

import oracle as O
import quantized_rank_gradient_b200 as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgalore.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qg_[a-z0-9_]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = qg.lib()
    names = header_functions()
    assert len(names) >= 20
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(qg.exported_symbols())


def test_library_symbols_via_nm():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", qg.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (qg_[a-z0-9_]+)$", out, flags=re.M))
    assert set(header_functions()) <= exported


def test_status_strings():
    for s in range(8):
        assert isinstance(qg.qg_status_str(s), str) and qg.qg_status_str(s)
    assert qg.qg_status_str(0) == "ok"


def test_config_defaults_and_sizes():
    c = qg.config(4096, 11008, 1024)
    assert (c.m, c.n, c.r, c.w_group, c.p_group, c.mom_block) == (4096, 11008, 1024, 256, 64, 256)
    assert abs(c.gamma - 0.4) < 1e-7 and c.delta0 == 200 and abs(c.alpha - 0.25) < 1e-7
    sb = qg.qg_state_bytes(byref(c))
    # header + 2 x INT4 P + scales + 2 x INT8 moments + moment scales
    mr = 4096 * 1024
    assert sb >= 256 + 2 * (mr // 2 + mr // 64 * 4) + 2 * 1024 * 11008 + 2 * 1024 * 43 * 4
    assert sb % 256 == 0
    ws = qg.qg_step_workspace_bytes(byref(c))
    assert ws >= 4096 * 1024 * 2 + 1024 * 11008 * 2
    bad = qg.config(100, 100, 48)  # r % 32 != 0
    assert qg.qg_state_bytes(byref(bad)) == 0


@pytest.mark.parametrize("field,value,expect", [
    ("r", 48, qg.QG_ESHAPE), ("r", 512, qg.QG_ESHAPE), ("w_group", 128, qg.QG_ESHAPE),
    ("beta1", 1.0, qg.QG_EINVAL), ("eps", 0.0, qg.QG_EINVAL), ("delta0", 0, qg.QG_EINVAL),
    ("mom_refresh", 3, qg.QG_EINVAL), ("mom_refresh", -1, qg.QG_EINVAL),
    ("proj_side", 2, qg.QG_EINVAL), ("w_rescale", 2, qg.QG_EINVAL),
    ("w_rescale", 1, qg.QG_ESHAPE),  # n = 300: a weight group is not one tile row
])
def test_layer_init_rejects_bad_config_before_any_launch(field, value, expect):
    c = qg.config(256, 300, 64)
    setattr(c, field, value)
    h = c_void_p()
    st = qg.qg_layer_init(byref(h), byref(c), 0x100000, 1 << 30, 0x200000, 304, 0x300000, None)
    assert st == expect and not h.value


def test_layer_init_validates_pointers_and_strides():
    c = qg.config(256, 300, 64)
    h = c_void_p()
    n = qg.qg_state_bytes(byref(c))
    assert qg.qg_layer_init(byref(h), byref(c), 0, n, 0x200000, 304, 0x300000, None) == qg.QG_EINVAL
    assert qg.qg_layer_init(byref(h), byref(c), 0x100010, n, 0x200000, 304, 0x300000, None) == qg.QG_EALIGN
    assert qg.qg_layer_init(byref(h), byref(c), 0x100000, n, 0x200000, 300, 0x300000, None) == qg.QG_EALIGN
    assert qg.qg_layer_init(byref(h), byref(c), 0x100000, n, 0x200000, 288, 0x300000, None) == qg.QG_EALIGN
    assert qg.qg_layer_init(byref(h), byref(c), 0x100000, n - 256, 0x200000, 304, 0x300000, None) == qg.QG_ESTATE
    assert qg.qg_step(None, 0x1000, 304, 0x1000, 1 << 20, None) == qg.QG_EINVAL


def test_entry_points_reject_bad_arguments_without_launching():
    assert qg.qg_gemm_bf16(0, 8, 0, 0x1000, 8, 0, 0x2000, 8, 8, 8, 8, None) == qg.QG_EINVAL
    assert qg.qg_gemm_bf16(0x1000, 12, 0, 0x1000, 8, 0, 0x2000, 8, 8, 8, 8, None) == qg.QG_EALIGN
    assert qg.qg_gemm_bf16(0x1008, 8, 0, 0x1000, 8, 0, 0x2000, 8, 8, 8, 8, None) == qg.QG_EALIGN
    assert qg.qg_dequant_projection(0x1000, 0x2000, 64, 48, 0x3000, None) == qg.QG_ESHAPE
    assert qg.qg_cossim(0x1000, 0x2000, 64, 32, 16, 0x3000, 0x4000, 1 << 20, None) == qg.QG_ESHAPE
    assert qg.qg_philox4x32_10(0, 0, 0, 0, 10, 0, 0, 0, None) == qg.QG_EINVAL


def test_fused_forward_rejects_bad_arguments_without_launching():
    f = qg.qg_linear_forward_int8
    X, W, sW, Y = 0x10000, 0x20000, 0x30000, 0x40000
    # (X, ldx, W, ldw, sW, T, m, n, Y, ldy): T in 0..64, m and n positive
    assert f(X, 128, W, 128, sW, 65, 64, 128, Y, 64, None) == qg.QG_ESHAPE
    assert f(X, 128, W, 128, sW, -1, 64, 128, Y, 64, None) == qg.QG_ESHAPE
    assert f(X, 128, W, 128, sW, 4, 0, 128, Y, 64, None) == qg.QG_ESHAPE
    assert f(X, 128, W, 128, sW, 4, 64, 0, Y, 64, None) == qg.QG_ESHAPE
    # W and its scales are required; its stride is a multiple of 16 bytes, at least n
    assert f(X, 128, 0, 128, sW, 4, 64, 128, Y, 64, None) == qg.QG_EINVAL
    assert f(X, 128, W, 128, 0, 4, 64, 128, Y, 64, None) == qg.QG_EINVAL
    assert f(X, 128, W, 136, sW, 4, 64, 128, Y, 64, None) == qg.QG_ESHAPE
    assert f(X, 128, W, 112, sW, 4, 64, 128, Y, 64, None) == qg.QG_ESHAPE
    assert f(X, 128, W + 8, 128, sW, 4, 64, 128, Y, 64, None) == qg.QG_EALIGN
    # bf16 X and Y: strides a multiple of 8 elements and at least a row, 16-byte aligned
    assert f(X, 124, W, 128, sW, 4, 64, 128, Y, 64, None) == qg.QG_ESHAPE
    assert f(X, 128, W, 128, sW, 4, 64, 128, Y, 60, None) == qg.QG_ESHAPE
    assert f(X + 2, 128, W, 128, sW, 4, 64, 128, Y, 64, None) == qg.QG_EALIGN
    assert f(0, 128, W, 128, sW, 4, 64, 128, Y, 64, None) == qg.QG_EINVAL
    # no tokens: nothing to do, nothing launched
    assert f(X, 128, W, 128, sW, 0, 64, 128, Y, 64, None) == qg.QG_OK


def _lib_sched(t, delta, cs, gamma):
    d = c_int32()
    tn = c_int64()
    has = 0 if cs is None else 1
    qg.check(qg.qg_sched_after_refresh(t, delta, has, 0.0 if cs is None else cs, gamma, byref(d), byref(tn)))
    return d.value, tn.value


@pytest.mark.parametrize("gamma", [0.4, 1.5, -1.5, 0.0])
def test_host_schedule_rule_matches_oracle(gamma):
    import numpy as np
    rng = np.random.default_rng(3)
    t, delta = 0, 200
    to, do = 0, 200
    for i in range(12):
        cs = None if i == 0 else float(np.float32(rng.choice([0.4, 0.39, 0.41, 0.9, 0.1, 1.0])))
        delta, t_next = _lib_sched(t, delta, cs, gamma)
        do, tno = O.schedule_after_refresh(to, do, cs, float(np.float32(gamma)))
        assert (delta, t_next) == (do, tno)
        t, to = t_next, tno
