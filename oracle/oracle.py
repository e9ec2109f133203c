"""ctypes front end of the fp64 C oracle (oracle/slay_oracle.c).

TEST INFRASTRUCTURE ONLY: used by tests/, the package smoke check and the
benchmark's CPU-baseline leg.  Arguments are numpy arrays; everything is
converted to C-contiguous float64 before the call.  The parameter set
(omega, anchors, s, wt) is drawn by the oracle's own Philox from the seed.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        dp = C.POINTER(C.c_double)
        i64p = C.POINTER(C.c_int64)
        u32p = C.POINTER(C.c_uint32)
        L.orc_philox4x32_10.argtypes = [u32p, u32p, u32p]
        L.orc_philox4x32_10.restype = None
        L.orc_gauss_laguerre.argtypes = [C.c_int, dp, dp]
        L.orc_gauss_laguerre.restype = C.c_int
        L.orc_sketch_params.argtypes = [C.c_int, C.c_int, C.c_int, C.c_uint64, C.c_double,
                                        dp, dp, dp, dp]
        L.orc_sketch_params.restype = C.c_int
        L.orc_yat_kernel.argtypes = [C.c_double, C.c_double]
        L.orc_yat_kernel.restype = C.c_double
        L.orc_quad_kernel.argtypes = [C.c_double, C.c_int, C.c_double]
        L.orc_quad_kernel.restype = C.c_double
        par = [dp, dp, dp, dp]
        L.orc_feature_map.argtypes = [dp, C.c_int64, C.c_int, C.c_int, C.c_int] + par + [dp]
        L.orc_feature_map.restype = None
        shp = [C.c_int] * 7
        L.orc_attn_quadratic.argtypes = [dp, dp, dp] + shp + par + [C.c_double, C.c_int, dp, dp]
        L.orc_attn_quadratic.restype = None
        L.orc_attn_quadratic_rows.argtypes = ([dp, dp, dp] + shp + par +
                                              [C.c_double, C.c_int, i64p, C.c_int, dp, dp])
        L.orc_attn_quadratic_rows.restype = None
        L.orc_attn_recurrent.argtypes = [dp, dp, dp] + shp + par + [C.c_double, C.c_int, dp, dp]
        L.orc_attn_recurrent.restype = None
        L.orc_decode_step.argtypes = ([dp, dp, dp, dp, dp, dp] + [C.c_int] * 5 + par +
                                      [C.c_double])
        L.orc_decode_step.restype = None
        L.orc_attn_causal_bwd.argtypes = [dp, dp, dp, dp] + shp + par + [C.c_double, dp, dp, dp]
        L.orc_attn_causal_bwd.restype = None
        L.orc_attn_causal_bwd_rows.argtypes = ([dp, dp, dp, dp] + shp + par +
                                               [C.c_double, i64p, C.c_int, dp, dp, dp])
        L.orc_attn_causal_bwd_rows.restype = None
        L.orc_attn_causal_bwd_given.argtypes = ([dp, dp, dp, dp, dp, dp] + shp + par +
                                                [C.c_double, dp, dp, dp])
        L.orc_attn_causal_bwd_given.restype = None
        L.orc_attn_causal_bwd_given_rows.argtypes = ([dp, dp, dp, dp, dp, dp] + shp + par +
                                                     [C.c_double, i64p, C.c_int, dp, dp, dp])
        L.orc_attn_causal_bwd_given_rows.restype = None
        L.orc_feature_map_bwd.argtypes = [dp, dp, C.c_int64, C.c_int, C.c_int, C.c_int] + par + [dp]
        L.orc_feature_map_bwd.restype = None
        L.orc_attn_bidir_bwd.argtypes = [dp, dp, dp, dp] + shp + par + [C.c_double, dp, dp, dp]
        L.orc_attn_bidir_bwd.restype = None
        L.orc_attn_bidir_bwd_given.argtypes = ([dp, dp, dp, dp, dp, dp] + shp + par +
                                              [C.c_double, dp, dp, dp])
        L.orc_attn_bidir_bwd_given.restype = None
        L.orc_sketch_params_kind.argtypes = [C.c_int, C.c_int, C.c_int, C.c_uint64, C.c_double,
                                             C.c_int, C.c_int, dp, dp, dp, dp, dp]
        L.orc_sketch_params_kind.restype = C.c_int
        L.orc_feature_map_kind.argtypes = [dp, C.c_int64, C.c_int, C.c_int, C.c_int, dp, dp, dp,
                                           dp, dp, C.c_int, dp]
        L.orc_feature_map_kind.restype = None
        L.orc_attn_from_phi.argtypes = [dp, dp, dp] + [C.c_int] * 5 + [C.c_double, C.c_int,
                                                                      dp, dp]
        L.orc_attn_from_phi.restype = None
        L.orc_attn_causal_state.argtypes = [dp, dp, dp, dp, dp] + shp + par + [C.c_double,
                                                                             dp, dp, dp, dp]
        L.orc_attn_causal_state.restype = None
        L.orc_attn_causal_bwd_state.argtypes = ([dp] * 10 + shp + par +
                                                [C.c_double, dp, dp, dp, dp, dp])
        L.orc_attn_causal_bwd_state.restype = None
        L.orc_num_threads.argtypes = []
        L.orc_num_threads.restype = C.c_int
        _lib = L
    return _lib


def _d(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return a.ctypes.data_as(C.POINTER(C.c_double))


def num_threads() -> int:
    return lib().orc_num_threads()


def philox4x32_10(ctr, key):
    c = (C.c_uint32 * 4)(*[int(x) & 0xffffffff for x in ctr])
    k = (C.c_uint32 * 2)(*[int(x) & 0xffffffff for x in key])
    o = (C.c_uint32 * 4)()
    lib().orc_philox4x32_10(c, k, o)
    return [int(x) for x in o]


def gauss_laguerre(R: int):
    t = np.zeros(R)
    w = np.zeros(R)
    if lib().orc_gauss_laguerre(R, _p(t), _p(w)) != 0:
        raise ValueError("gauss_laguerre failed for R=%d" % R)
    return t, w


class Params:
    """Sketch parameters of one (D, R, m, seed, eps) key, drawn by the oracle."""

    def __init__(self, D, R, m, seed, eps):
        F = R * m
        self.D, self.R, self.m, self.seed, self.eps, self.F = D, R, m, seed, eps, F
        self.omega = np.zeros((F, D))
        self.anchors = np.zeros((F, D))
        self.s = np.zeros(R)
        self.wt = np.zeros(R)
        rc = lib().orc_sketch_params(D, R, m, C.c_uint64(seed), eps, _p(self.omega),
                                     _p(self.anchors), _p(self.s), _p(self.wt))
        if rc != 0:
            raise ValueError("sketch_params failed")

    def args(self):
        return [_p(self.omega), _p(self.anchors), _p(self.s), _p(self.wt)]


def sketch_params(D, R, m, seed, eps) -> Params:
    return Params(D, R, m, seed, eps)


def yat_kernel(x, eps):
    return lib().orc_yat_kernel(float(x), float(eps))


def quad_kernel(x, R, eps):
    return lib().orc_quad_kernel(float(x), int(R), float(eps))


def feature_map(x, P: Params):
    x = _d(x)
    n = x.size // P.D
    phi = np.zeros((n, P.F))
    lib().orc_feature_map(_p(x), n, P.D, P.R, P.m, *P.args(), _p(phi))
    return phi.reshape(x.shape[:-1] + (P.F,))


def _shape4(q, v):
    B, H, L, D = q.shape
    return B, H, L, D, v.shape[-1]


def attn_quadratic(q, k, v, P: Params, causal: bool):
    q, k, v = _d(q), _d(k), _d(v)
    B, H, L, D, Dv = _shape4(q, v)
    out = np.zeros((B, H, L, Dv))
    den = np.zeros((B, H, L))
    lib().orc_attn_quadratic(_p(q), _p(k), _p(v), B, H, L, D, Dv, P.R, P.m, *P.args(),
                             P.eps, int(causal), _p(out), _p(den))
    return out, den


def attn_quadratic_rows(q, k, v, P: Params, causal: bool, rows):
    q, k, v = _d(q), _d(k), _d(v)
    B, H, L, D, Dv = _shape4(q, v)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    nr = rows.size
    out = np.zeros((B, H, nr, Dv))
    den = np.zeros((B, H, nr))
    lib().orc_attn_quadratic_rows(_p(q), _p(k), _p(v), B, H, L, D, Dv, P.R, P.m, *P.args(),
                                  P.eps, int(causal),
                                  rows.ctypes.data_as(C.POINTER(C.c_int64)), nr,
                                  _p(out), _p(den))
    return out, den


def attn_recurrent(q, k, v, P: Params, causal: bool):
    q, k, v = _d(q), _d(k), _d(v)
    B, H, L, D, Dv = _shape4(q, v)
    out = np.zeros((B, H, L, Dv))
    den = np.zeros((B, H, L))
    lib().orc_attn_recurrent(_p(q), _p(k), _p(v), B, H, L, D, Dv, P.R, P.m, *P.args(),
                             P.eps, int(causal), _p(out), _p(den))
    return out, den


def decode_step(q, k, v, S, z, P: Params):
    """Returns (out, S_new, z_new); inputs are not modified."""
    q, k, v = _d(q), _d(k), _d(v)
    S = _d(S).copy()
    z = _d(z).copy()
    N = q.size // P.D
    Dv = v.shape[-1]
    out = np.zeros(v.shape)
    lib().orc_decode_step(_p(q), _p(k), _p(v), _p(S), _p(z), _p(out), N, P.D, Dv, P.R, P.m,
                          *P.args(), P.eps)
    return out, S, z


def attn_causal_bwd(q, k, v, dout, P: Params):
    q, k, v, g = _d(q), _d(k), _d(v), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    lib().orc_attn_causal_bwd(_p(q), _p(k), _p(v), _p(g), B, H, L, D, Dv, P.R, P.m, *P.args(),
                              P.eps, _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def attn_causal_bwd_rows(q, k, v, dout, P: Params, rows):
    q, k, v, g = _d(q), _d(k), _d(v), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    nr = rows.size
    dq = np.zeros((B, H, nr, D))
    dk = np.zeros((B, H, nr, D))
    dv = np.zeros((B, H, nr, Dv))
    lib().orc_attn_causal_bwd_rows(_p(q), _p(k), _p(v), _p(g), B, H, L, D, Dv, P.R, P.m,
                                   *P.args(), P.eps,
                                   rows.ctypes.data_as(C.POINTER(C.c_int64)), nr,
                                   _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def attn_causal_bwd_given(q, k, v, out, den, dout, P: Params):
    """Gradients at a given forward output (out [B,H,L,Dv], den [B,H,L]), the inputs the
    library's backward takes; equals attn_causal_bwd when out, den are the exact ones."""
    q, k, v, o, dn, g = _d(q), _d(k), _d(v), _d(out), _d(den), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    lib().orc_attn_causal_bwd_given(_p(q), _p(k), _p(v), _p(o), _p(dn), _p(g), B, H, L, D, Dv,
                                    P.R, P.m, *P.args(), P.eps, _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def attn_causal_bwd_given_rows(q, k, v, out, den, dout, P: Params, rows):
    q, k, v, o, dn, g = _d(q), _d(k), _d(v), _d(out), _d(den), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    nr = rows.size
    dq = np.zeros((B, H, nr, D))
    dk = np.zeros((B, H, nr, D))
    dv = np.zeros((B, H, nr, Dv))
    lib().orc_attn_causal_bwd_given_rows(_p(q), _p(k), _p(v), _p(o), _p(dn), _p(g), B, H, L,
                                         D, Dv, P.R, P.m, *P.args(), P.eps,
                                         rows.ctypes.data_as(C.POINTER(C.c_int64)), nr,
                                         _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def feature_map_bwd(x, dphi, P: Params):
    """dx [..., D] of sum(dphi * phi(x)) (the derivative of feature_map)."""
    x, g = _d(x), _d(dphi)
    n = x.size // P.D
    dx = np.zeros((n, P.D))
    lib().orc_feature_map_bwd(_p(x), _p(g), n, P.D, P.R, P.m, *P.args(), _p(dx))
    return dx.reshape(x.shape)


def attn_bidir_bwd(q, k, v, dout, P: Params):
    """Gradients of sum(dout * out) for the bidirectional forward."""
    q, k, v, g = _d(q), _d(k), _d(v), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    lib().orc_attn_bidir_bwd(_p(q), _p(k), _p(v), _p(g), B, H, L, D, Dv, P.R, P.m, *P.args(),
                             P.eps, _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def attn_bidir_bwd_given(q, k, v, out, den, dout, P: Params):
    """Bidirectional gradients at a given forward output (out, den as inputs)."""
    q, k, v, o, dn, g = _d(q), _d(k), _d(v), _d(out), _d(den), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    lib().orc_attn_bidir_bwd_given(_p(q), _p(k), _p(v), _p(o), _p(dn), _p(g), B, H, L, D, Dv,
                                   P.R, P.m, *P.args(), P.eps, _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


PHI_ANCHOR, PHI_ORTHOGONAL, PHI_SIGNED, PHI_PER_HEAD, PHI_PERFORMER = range(5)


class KindParams:
    """Sketch parameters of one variant (kind) and head: omega, anchors, anchors_b [F, D],
    s, wt [R]; drawn by the oracle's own Philox and Gram-Schmidt."""

    def __init__(self, D, R, m, seed, eps, kind, head=0):
        F = R * m
        self.D, self.R, self.m, self.seed, self.eps, self.F = D, R, m, seed, eps, F
        self.kind, self.head = kind, head
        self.omega = np.zeros((F, D))
        self.anchors = np.zeros((F, D))
        self.anchors_b = np.zeros((F, D))
        self.s = np.zeros(R)
        self.wt = np.zeros(R)
        rc = lib().orc_sketch_params_kind(D, R, m, C.c_uint64(seed), eps, kind, head,
                                          _p(self.omega), _p(self.anchors), _p(self.anchors_b),
                                          _p(self.s), _p(self.wt))
        if rc != 0:
            raise ValueError("sketch_params_kind failed")


def sketch_params_kind(D, R, m, seed, eps, kind, head=0) -> KindParams:
    return KindParams(D, R, m, seed, eps, kind, head)


def feature_map_kind(x, P: KindParams):
    x = _d(x)
    n = x.size // P.D
    phi = np.zeros((n, P.F))
    lib().orc_feature_map_kind(_p(x), n, P.D, P.R, P.m, _p(P.omega), _p(P.anchors),
                               _p(P.anchors_b), _p(P.s), _p(P.wt), P.kind, _p(phi))
    return phi.reshape(x.shape[:-1] + (P.F,))


def attn_from_phi(pq, pk, v, eps, causal):
    """The masked-sum contraction on given features pq, pk [B,H,L,F] and v [B,H,L,Dv]."""
    pq, pk, v = _d(pq), _d(pk), _d(v)
    B, H, L, F = pq.shape
    Dv = v.shape[-1]
    out = np.zeros((B, H, L, Dv))
    den = np.zeros((B, H, L))
    lib().orc_attn_from_phi(_p(pq), _p(pk), _p(v), B, H, L, F, Dv, float(eps), int(causal),
                            _p(out), _p(den))
    return out, den


def attn_causal_state(q, k, v, P: Params, S0=None, z0=None):
    """Causal forward continued from state (S0 [B,H,F,Dv], z0 [B,H,F]; None = zero);
    returns (out, den, S1, z1) with the state after the last token."""
    q, k, v = _d(q), _d(k), _d(v)
    B, H, L, D, Dv = _shape4(q, v)
    F = P.F
    out = np.zeros((B, H, L, Dv))
    den = np.zeros((B, H, L))
    S1 = np.zeros((B, H, F, Dv))
    z1 = np.zeros((B, H, F))
    s0 = None if S0 is None else _d(S0)
    zz0 = None if z0 is None else _d(z0)
    lib().orc_attn_causal_state(_p(q), _p(k), _p(v), None if s0 is None else _p(s0),
                                None if zz0 is None else _p(zz0), B, H, L, D, Dv, P.R, P.m,
                                *P.args(), P.eps, _p(out), _p(den), _p(S1), _p(z1))
    return out, den, S1, z1


def attn_causal_bwd_state(q, k, v, out, den, dout, P: Params, S_in=None, z_in=None, G_in=None,
                          zg_in=None):
    """Backward of one piece of a longer causal sequence at its given forward output: S_in
    [B,H,F,Dv], z_in [B,H,F] sum phi(k)[v, 1] over the tokens before the piece, G_in, zg_in
    sum phi(q)[dn, delta] over the tokens after it (None = zero).  Returns (dq, dk, dv,
    G_out, zg_out), the last two the piece's own sum of phi(q)[dn, delta]."""
    q, k, v, o, dn, g = _d(q), _d(k), _d(v), _d(out), _d(den), _d(dout)
    B, H, L, D, Dv = _shape4(q, v)
    F = P.F
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    G_out = np.zeros((B, H, F, Dv))
    zg_out = np.zeros((B, H, F))
    st = [None if x is None else _d(x) for x in (S_in, z_in, G_in, zg_in)]
    lib().orc_attn_causal_bwd_state(_p(q), _p(k), _p(v), _p(o), _p(dn), _p(g),
                                    *[None if x is None else _p(x) for x in st],
                                    B, H, L, D, Dv, P.R, P.m, *P.args(), P.eps,
                                    _p(dq), _p(dk), _p(dv), _p(G_out), _p(zg_out))
    return dq, dk, dv, G_out, zg_out


__all__ = ["lib", "num_threads", "philox4x32_10", "gauss_laguerre", "Params", "sketch_params",
           "yat_kernel", "quad_kernel", "feature_map", "attn_quadratic", "attn_quadratic_rows",
           "attn_recurrent", "decode_step", "attn_causal_bwd", "attn_causal_bwd_rows",
           "attn_causal_bwd_given", "attn_causal_bwd_given_rows", "feature_map_bwd",
           "attn_bidir_bwd", "attn_bidir_bwd_given", "KindParams", "sketch_params_kind",
           "feature_map_kind", "attn_from_phi", "PHI_ANCHOR", "PHI_ORTHOGONAL", "PHI_SIGNED",
           "PHI_PER_HEAD", "PHI_PERFORMER", "attn_causal_state", "attn_causal_bwd_state"]
