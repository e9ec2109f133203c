"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, draws the same sketch parameters as the oracle's independent Philox, and
rejects bad arguments before touching the device."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle as O
from kernelized_linear_attention_unit_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "slay.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(slay_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = bd.lib()
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(bd.EXPORTS) == set(names)


def test_status_strings():
    L = bd.lib()
    for s in range(6):
        assert L.slay_status_string(s)
    assert L.slay_status_string(99) == b"unknown status"


@pytest.mark.parametrize("D,R,m,seed", [(64, 2, 16, 1234), (64, 4, 64, 1234), (64, 8, 64, 99),
                                        (16, 3, 5, 2 ** 40 + 17)])
def test_sketch_params_match_oracle_bitwise(D, R, m, seed):
    eps = float(np.float32(1e-6))
    om, an, s, w = bd.slay_sketch_params(D, R, m, seed, eps)
    P = O.sketch_params(D, R, m, seed, eps)
    assert np.array_equal(om.astype(np.float64), P.omega)
    assert np.array_equal(an.astype(np.float64), P.anchors)
    # quadrature: Golub-Welsch (library) against Newton/bisection (oracle)
    np.testing.assert_allclose(s, P.s, rtol=1e-13)
    np.testing.assert_allclose(w, P.wt, rtol=1e-11)


@pytest.mark.parametrize("R", list(range(1, 17)))
def test_library_quadrature_against_library_rule(R):
    _, _, s, w = bd.slay_sketch_params(4, R, 1, 0, 1.0)
    tn, wn = np.polynomial.laguerre.laggauss(R)
    np.testing.assert_allclose(s * 3.0, tn, rtol=1e-12)
    np.testing.assert_allclose(w * 3.0, wn, rtol=1e-9, atol=1e-300)


def test_workspace_bytes():
    f = bd.slay_workspace_bytes
    assert f(bd.OP_FEATURE_MAP, bd.SLAY_BF16, 1, 1, 16, 64, 64, 4, 64) == 0
    assert f(bd.OP_DECODE, bd.SLAY_BF16, 1, 1, 16, 64, 64, 4, 64) == 0
    assert f(bd.OP_CAUSAL_FWD, bd.SLAY_F32, 0, 8, 1024, 64, 64, 4, 64) == 0
    for op in (bd.OP_CAUSAL_FWD, bd.OP_BIDIR_FWD, bd.OP_CAUSAL_BWD):
        for dt in (bd.SLAY_F32, bd.SLAY_BF16):
            a = f(op, dt, 1, 2, 1000, 64, 64, 4, 64)
            b = f(op, dt, 1, 2, 2000, 64, 64, 4, 64)
            assert 0 < a <= b
            assert a % 256 == 0
    with pytest.raises(bd.SlayError):
        f(bd.OP_CAUSAL_FWD, bd.SLAY_F32, 1, 1, 16, 32, 64, 4, 64)


@pytest.mark.parametrize("op,dt,B,H,L,R,m,want", [
    ("CAUSAL_FWD", "BF16", 1, 16, 16384, 4, 64, 3),       # the headline: tensor cores
    ("CAUSAL_FWD", "F32", 1, 16, 16384, 4, 64, 0),        # fp32: CUDA cores
    ("CAUSAL_FWD", "BF16", 1, 2, 100, 4, 32, 1),          # m % 64 != 0: CUDA-core contraction
    ("BIDIR_FWD", "BF16", 1, 2, 100, 4, 32, 1),           # after the tensor-core map
    ("CAUSAL_FWD", "BF16", 1, 2, 100, 3, 32, 0),          # F % 128 != 0: no tensor cores
    ("CAUSAL_FWD", "BF16", 2, 16, 8192, 8, 64, 3),        # F = 512 in two chunks
    ("CAUSAL_FWD", "BF16", 1, 2, 100, 16, 64, 0),         # F = 1024 > 512
    ("CAUSAL_FWD", "BF16", 0, 2, 100, 4, 64, 0),          # empty
    ("CAUSAL_STATE", "BF16", 1, 2, 100, 4, 64, 3),
    ("CAUSAL_FWD_SPLIT", "BF16", 1, 2, 100, 4, 64, 3),
    ("BIDIR_FWD", "BF16", 32, 12, 1024, 4, 64, 3),
    ("FEATURE_MAP", "BF16", 1, 1, 1000, 4, 32, 1),        # the map takes m % 32 == 0
    ("FEATURE_MAP", "F32", 1, 1, 1000, 4, 32, 0),
    ("FEATURE_MAP", "BF16", 1, 1, 1000, 3, 64, 0),        # F % 128 != 0
    ("FEATURE_MAP_BWD", "BF16", 1, 1, 1000, 4, 32, 4),
    ("CAUSAL_BWD", "BF16", 2, 16, 8192, 8, 64, 7),
    ("CAUSAL_BWD", "BF16", 1, 2, 100, 2, 64, 7),
    ("CAUSAL_BWD", "BF16", 1, 2, 100, 3, 64, 0),          # F = 192
    ("CAUSAL_BWD", "BF16", 1, 2, 100, 10, 64, 0),         # F = 640
    ("CAUSAL_BWD", "F32", 1, 2, 100, 2, 64, 0),
    ("BIDIR_BWD", "BF16", 32, 12, 1024, 4, 64, 7),
    ("DECODE", "BF16", 256, 16, 1, 8, 64, 0),
    ("LINEAR_ATTN", "BF16", 1, 2, 100, 1, 256, 0),
])
def test_path_query(op, dt, B, H, L, R, m, want):
    # the size rules the header states for the tensor-core kernels; host only
    got = bd.slay_path(getattr(bd, "OP_" + op), getattr(bd, "SLAY_" + dt), B, H, L, 64, 64, R, m)
    assert got == want


def test_path_query_rejects():
    with pytest.raises(bd.SlayError):
        bd.slay_path(bd.OP_CAUSAL_FWD, bd.SLAY_BF16, 1, 1, 16, 32, 64, 4, 64)   # D != 64
    with pytest.raises(bd.SlayError):
        bd.slay_path(99, bd.SLAY_BF16, 1, 1, 16, 64, 64, 4, 64)
    with pytest.raises(bd.SlayError):
        bd.slay_path(bd.OP_CAUSAL_FWD, 7, 1, 1, 16, 64, 64, 4, 64)


def _fake(addr=0x10000):
    return C.c_void_p(addr)


def test_argument_errors_before_any_device_work():
    L = bd.lib()
    f = L.slay_attn_causal_fwd
    good = dict(D=64, Dv=64, R=4, m=64)
    args = lambda q=_fake(), k=_fake(), v=_fake(), out=_fake(), B=1, H=1, Ln=128, D=64, Dv=64, \
        dt=bd.SLAY_BF16, R=4, m=64, eps=1e-6, ws=_fake(0x20000), wsb=1 << 40: \
        (q, k, v, out, None, B, H, Ln, D, Dv, dt, R, m, 1234, eps, ws, wsb, None)
    assert f(*args(q=None)) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(out=None)) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(q=_fake(0x10004))) == bd.SLAY_ERR_INVALID_ARG          # misaligned
    assert f(*args(B=-1)) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(D=32)) == bd.SLAY_ERR_UNSUPPORTED
    assert f(*args(Dv=128)) == bd.SLAY_ERR_UNSUPPORTED
    assert f(*args(R=17)) == bd.SLAY_ERR_UNSUPPORTED
    assert f(*args(m=2048)) == bd.SLAY_ERR_UNSUPPORTED
    assert f(*args(R=0)) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(eps=0.0)) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(eps=float("nan"))) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(dt=7)) == bd.SLAY_ERR_INVALID_ARG
    assert f(*args(ws=None)) == bd.SLAY_ERR_INVALID_ARG                    # workspace missing
    assert f(*args(wsb=16)) == bd.SLAY_ERR_INVALID_ARG                     # workspace too small
    assert f(*args(ws=_fake(0x20010))) == bd.SLAY_ERR_INVALID_ARG          # workspace misaligned
    # empty work is a no-op even with NULL pointers
    assert f(*args(q=None, k=None, v=None, out=None, Ln=0)) == bd.SLAY_OK
    assert f(*args(q=None, k=None, v=None, out=None, B=0)) == bd.SLAY_OK
    # feature map
    fm = L.slay_feature_map
    assert fm(None, _fake(), 10, 64, bd.SLAY_BF16, bd.SLAY_BF16, 4, 64, 1, 1e-6, None) == bd.SLAY_ERR_INVALID_ARG
    assert fm(_fake(), _fake(), 10, 64, bd.SLAY_F32, bd.SLAY_BF16, 4, 64, 1, 1e-6, None) == bd.SLAY_ERR_UNSUPPORTED
    assert fm(_fake(), _fake(), -1, 64, bd.SLAY_F32, bd.SLAY_F32, 4, 64, 1, 1e-6, None) == bd.SLAY_ERR_INVALID_ARG
    assert fm(None, None, 0, 64, bd.SLAY_F32, bd.SLAY_F32, 4, 64, 1, 1e-6, None) == bd.SLAY_OK
    # decode
    dc = L.slay_decode_step
    assert dc(_fake(), _fake(), _fake(), None, _fake(), _fake(), 2, 2, 64, 64, bd.SLAY_BF16, 4, 64,
              1, 1e-6, None) == bd.SLAY_ERR_INVALID_ARG
    assert dc(None, None, None, None, None, None, 0, 16, 64, 64, bd.SLAY_BF16, 4, 64, 1, 1e-6,
              None) == bd.SLAY_OK
    # backward needs den and the gradients
    bw = L.slay_attn_causal_bwd
    assert bw(_fake(), _fake(), _fake(), _fake(), None, _fake(), _fake(), _fake(), _fake(), 1, 1,
              64, 64, 64, bd.SLAY_BF16, 4, 64, 1, 1e-6, _fake(0x20000), 1 << 40,
              None) == bd.SLAY_ERR_INVALID_ARG


def test_two_call_argument_errors_before_any_device_work():
    # the sequence-parallel two-call pairs check their arguments on the host like the rest
    L = bd.lib()
    F, big, ws = _fake(0x30000), 1 << 40, _fake(0x20000)
    sz = [1, 1, 128, 64, 64, bd.SLAY_BF16, 4, 64, 1234, 1e-6]
    fb = L.slay_attn_causal_fwd_begin
    assert fb(_fake(), _fake(), None, None, *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert fb(_fake(), _fake(), _fake(0x30004), _fake(), *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert fb(None, _fake(), F, _fake(), *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert fb(_fake(), _fake(), F, _fake(), *sz, None, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert fb(_fake(), _fake(), F, _fake(), *sz, ws, 256, None) == bd.SLAY_ERR_INVALID_ARG
    assert fb(_fake(), _fake(), F, _fake(), *sz, _fake(0x20010), big, None) == bd.SLAY_ERR_INVALID_ARG
    assert fb(_fake(), _fake(), F, _fake(), 0, *sz[1:], None, 0, None) == bd.SLAY_OK   # B = 0
    ff = L.slay_attn_causal_fwd_finish
    q5 = [_fake()] * 4
    assert ff(None, _fake(), _fake(), _fake(), None, None, None, *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert ff(*q5, None, F, None, *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG          # S_in without z_in
    assert ff(*q5, _fake(0x10002), None, None, *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert ff(*q5, None, None, None, *sz, ws, 256, None) == bd.SLAY_ERR_INVALID_ARG
    sz0 = list(sz)
    sz0[2] = 0
    assert ff(None, None, None, None, None, None, None, *sz0, None, 0, None) == bd.SLAY_OK   # L = 0
    bb = L.slay_attn_causal_bwd_begin
    assert bb(_fake(), _fake(), _fake(), _fake(), None, None, *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert bb(_fake(), _fake(), None, _fake(), F, _fake(), *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG
    assert bb(_fake(), _fake(), _fake(), _fake(), F, _fake(), *sz, ws, 256, None) == bd.SLAY_ERR_INVALID_ARG
    bf = L.slay_attn_causal_bwd_finish
    nine = [_fake()] * 9
    assert bf(*nine, None, None, F, None, *sz, ws, big, None) == bd.SLAY_ERR_INVALID_ARG  # G_in without zg_in
    assert bf(*nine[:6], None, _fake(), _fake(), None, None, None, None, *sz, ws, big,
              None) == bd.SLAY_ERR_INVALID_ARG                                         # dq missing
    assert bf(*nine, None, None, None, None, *sz, ws, 256, None) == bd.SLAY_ERR_INVALID_ARG
    assert bf(*([None] * 13), *sz0, None, 0, None) == bd.SLAY_OK                         # L = 0


def test_sketch_params_rejects_bad_args():
    L = bd.lib()
    assert L.slay_sketch_params(64, 0, 4, 1, 1e-6, None, None, None, None) == bd.SLAY_ERR_INVALID_ARG
    assert L.slay_sketch_params(64, 4, 4, 1, -1.0, None, None, None, None) == bd.SLAY_ERR_INVALID_ARG
    assert L.slay_sketch_params(64, 4, 4, 1, 1e-6, None, None, None, None) == bd.SLAY_OK


def test_noalloc_sizes_the_path_that_runs():
    # bf16 with F = 512 takes the CUDA-core kernels inside the no-allocation entry point
    # (its tensor-core form needs F <= 256); their scratch at B1 H1 L8192 (about 49 MiB)
    # exceeds the 32 MiB array, so the call must be rejected before anything is enqueued,
    # while the regular tensor-core workspace for the same sizes would have fitted.
    L = bd.lib()
    f = L.slay_attn_causal_fwd_noalloc
    tc_ws = bd.slay_workspace_bytes(bd.OP_CAUSAL_FWD, bd.SLAY_BF16, 1, 1, 8192, 64, 64, 8, 64)
    assert tc_ws < (32 << 20)
    for Ln in (8192, 6144):
        assert f(_fake(), _fake(), _fake(), _fake(), None, 1, 1, Ln, 64, 64, bd.SLAY_BF16, 8, 64,
                 1234, 1e-6, None) == bd.SLAY_ERR_UNSUPPORTED
    assert f(_fake(), _fake(), _fake(), _fake(), None, 1, 16, 16384, 64, 64, bd.SLAY_F32, 4, 64,
             1234, 1e-6, None) == bd.SLAY_ERR_UNSUPPORTED


@pytest.mark.parametrize("kind", [0, 1, 2, 3, 4])
def test_variant_sketch_params_match_oracle(kind):
    # the library's draws (its own Philox, modified Gram-Schmidt) against the oracle's (its own
    # Philox, classical Gram-Schmidt): bit for bit where nothing is orthogonalised, to fp32
    # rounding where the two Gram-Schmidt orders round differently
    D, R, m, seed = 16, 3, 20, 91
    eps = float(np.float32(1e-6))
    for head in ((0, 2) if kind == 3 else (0,)):
        om, an, anb, s, w = bd.slay_sketch_params_ex(D, R, m, seed, eps, kind, head)
        P = O.sketch_params_kind(D, R, m, seed, eps, kind, head)
        assert np.array_equal(an.astype(np.float64), P.anchors)
        if kind == 2:
            assert np.array_equal(anb.astype(np.float64), P.anchors_b)
        if kind in (1, 4):
            np.testing.assert_allclose(om.astype(np.float64), P.omega, rtol=2e-6, atol=2e-6)
        else:
            assert np.array_equal(om.astype(np.float64), P.omega)
        np.testing.assert_allclose(s, P.s, rtol=1e-13)
        np.testing.assert_allclose(w, P.wt, rtol=1e-11)


def test_variant_and_contraction_argument_errors():
    L = bd.lib()
    fx = L.slay_feature_map_ex
    assert fx(_fake(), _fake(), 10, 64, bd.SLAY_F32, bd.SLAY_F32, 4, 64, 1, 1e-6, 9, 1, 0, None) \
        == bd.SLAY_ERR_INVALID_ARG                                          # unknown kind
    assert fx(_fake(), _fake(), 10, 64, bd.SLAY_F32, bd.SLAY_F32, 4, 64, 1, 1e-6,
              bd.PHI_PER_HEAD, 2, 3, None) == bd.SLAY_ERR_INVALID_ARG        # 10 % 3 != 0
    assert fx(None, None, 0, 64, bd.SLAY_F32, bd.SLAY_F32, 4, 64, 1, 1e-6, bd.PHI_PERFORMER, 1,
              0, None) == bd.SLAY_OK
    la = L.slay_linear_attn_fwd
    assert la(_fake(), _fake(), _fake(), _fake(), None, 1, 1, 64, 2048, 64, bd.SLAY_F32, 1e-6, 1,
              _fake(0x20000), 1 << 40, None) == bd.SLAY_ERR_UNSUPPORTED     # F > 1024
    assert la(_fake(), _fake(), _fake(), _fake(), None, 1, 1, 64, 256, 64, bd.SLAY_F32, 1e-6, 1,
              None, 0, None) == bd.SLAY_ERR_INVALID_ARG                     # no workspace
    assert bd.slay_workspace_bytes(bd.OP_LINEAR_ATTN, bd.SLAY_F32, 1, 2, 100, 64, 64, 1, 256) > 0
