"""GPU parity: every entry point of libslay.so against the fp64 oracle.

Inputs come from the shared seeded recipe (kernelized_linear_attention_unit_b200.workloads)
and are rounded to the mode's dtype before either side sees them, so both compute on the
same values.  Bars (relative L2 error): 1e-5 in fp32 mode and 1.5e-2 in bf16-input /
fp32-accumulate mode for the whole tensor, ten times that for every single row
(tests/parity_check.py).  Small cases are compared over every row; the full-size workloads
on the first and last row of every 128-token tile (every segment the tensor-core kernels
cut a sequence into starts and ends on one) plus random rows, in the launch configuration
the benchmark times.

"Scaled" cases multiply every q and k row by 10^U(-3,3), with a few rows at 10^{+-6} and
10^{+-10}, before rounding (and the "norm range" cases put rows at both ends of the
range the library supports, 1e-12 .. 1e15): the workloads' own rows are unit length, so
without these the kernels' normalisation (the sphere projection of the review's "Proposed
method", step 1) and, in the backward, the projection of the gradient onto the sphere's
tangent space would go unchecked.
"""
import numpy as np
import pytest
import torch

import oracle as O
from kernelized_linear_attention_unit_b200 import binding as bd
from kernelized_linear_attention_unit_b200 import workloads as W
from parity_check import check, gradient_row_scale, rel_l2

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1.5e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _eps(w):
    return float(np.float32(w.eps))


def dev(x, dt):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(TDT[dt])


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def params(w):
    return O.sketch_params(w.D, w.R, w.m, w.sketch_seed, _eps(w))


def small(dt, R, m, L, B=1, H=2, correlated=False, seed=21):
    return W.Workload("small", B=B, H=H, L=L, R=R, m=m, dtype=dt, correlated=correlated,
                      data_seed=seed)


def qkv(w, scaled=False):
    q, k, v = W.gen_qkv(w)
    if scaled:
        q = W.scale_rows(w, q, "q")
        k = W.scale_rows(w, k, "k")
    return q, k, v


def tag(w, what, scaled=False):
    return "%s %s B%dH%dL%d R%d m%d%s" % (what, w.dtype, w.B, w.H, w.L, w.R, w.m,
                                           " scaled" if scaled else "")


# ------------------------------------------------------------- feature map

@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("dt_in,dt_out,R,m,n", [("f32", "f32", 2, 16, 1000),
                                                 ("f32", "f32", 4, 64, 130),
                                                 ("bf16", "bf16", 4, 64, 1000),
                                                 ("bf16", "f32", 8, 64, 333),
                                                 ("bf16", "bf16", 8, 64, 4097),
                                                 ("bf16", "bf16", 2, 64, 40000),
                                                 ("bf16", "bf16", 4, 32, 38001),
                                                 ("bf16", "bf16", 3, 64, 777)])
def test_feature_map(dt_in, dt_out, R, m, n, scaled):
    w = small(dt_in, R, m, n, B=1, H=1)
    q, _, _ = qkv(w, scaled)
    x = q.reshape(n, 64).copy()
    x[3] = 0.0                       # degenerate zero row -> phi = 0
    x[5] = W.to_dtype(x[5] * 37.0, dt_in)   # rescaled row -> same phi
    P = params(w)
    want = O.feature_map(x, P)
    xt = dev(x, dt_in)
    phi = torch.empty((n, R * m), device="cuda", dtype=TDT[dt_out])
    bd.slay_feature_map(xt, phi, R, m, w.sketch_seed, _eps(w))
    bd.slay_kernel_status(None)
    torch.cuda.synchronize()
    got = host(phi)
    tol = TOL["bf16"] if "bf16" in (dt_in, dt_out) else TOL["f32"]
    check("phi %s->%s n%d R%d m%d%s" % (dt_in, dt_out, n, R, m, " scaled" if scaled else ""),
          got, want, tol)
    assert (got[3] == 0).all()
    assert (np.delete(got, 3, axis=0) >= 0).all()


# The ends of the row-norm range the library states it supports (1e-12 .. 1e15): the
# bf16 tensor-core kernels fold 1/|x|^2 into the exponent of phi, which must stay inside
# fp32's exponent range for every feature; the fp32 kernels normalise first.
NORM_ENDS = (15.0, 15.0, 14.0, 13.5, 12.0, -11.0, -11.9, -11.9)


@pytest.mark.parametrize("dt,R,m", [("bf16", 4, 64), ("bf16", 8, 64), ("bf16", 16, 32),
                                    ("f32", 8, 64)])
def test_feature_map_norm_range(dt, R, m):
    w = small(dt, R, m, 2000, B=1, H=1, seed=23)
    q, _, _ = W.gen_qkv(w)
    x = W.scale_rows(w, q.reshape(2000, 64), "q", extremes=NORM_ENDS)
    P = params(w)
    want = O.feature_map(x, P)
    phi = torch.empty((2000, R * m), device="cuda", dtype=TDT[dt])
    bd.slay_feature_map(dev(x, dt), phi, R, m, w.sketch_seed, _eps(w))
    bd.slay_kernel_status(None)
    torch.cuda.synchronize()
    check("phi norm range %s R%d m%d" % (dt, R, m), host(phi), want, TOL[dt])


@pytest.mark.parametrize("dt,R,m,L", [("bf16", 4, 64, 700), ("bf16", 8, 64, 300),
                                      ("f32", 4, 64, 300)])
def test_attn_fwd_norm_range(dt, R, m, L):
    w = small(dt, R, m, L, seed=24)
    q, k, v = W.gen_qkv(w)
    q = W.scale_rows(w, q, "q", extremes=NORM_ENDS)
    k = W.scale_rows(w, k, "k", extremes=NORM_ENDS)
    P = params(w)
    want, wden = O.attn_quadratic(q, k, v, P, True)
    got, gden = _run_fwd(q, k, v, w, True)
    _check_fwd(tag(w, "causal norm range"), got, gden, want, wden, TOL[dt])


# ------------------------------------------------------------ forward

def _run_fwd(q, k, v, w, causal):
    B, H, L, _ = q.shape
    qt, kt, vt = dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype)
    out = torch.empty((B, H, L, w.Dv), device="cuda", dtype=TDT[w.dtype])
    den = torch.empty((B, H, L), device="cuda", dtype=torch.float32)
    fn = bd.slay_attn_causal_fwd if causal else bd.slay_attn_bidir_fwd
    ws = fn(qt, kt, vt, out, den, w.R, w.m, w.sketch_seed, _eps(w))
    bd.slay_kernel_status(ws)          # raises if a kernel stopped on an expired wait
    torch.cuda.synchronize()
    return host(out), host(den)


def _check_fwd(name, got, gden, want, wden, tol):
    check(name + " out", got, want, tol)
    check(name + " den", gden, wden, tol, per_element=True)


FWD_SMALL = [("f32", 2, 16, 256), ("f32", 2, 16, 1), ("f32", 4, 64, 200),
             ("f32", 3, 16, 129), ("bf16", 4, 64, 300),
             ("bf16", 4, 64, 1), ("bf16", 8, 64, 257),
             ("bf16", 2, 16, 64), ("bf16", 2, 64, 129),
             ("bf16", 4, 64, 1000), ("bf16", 2, 64, 2049),
             ("bf16", 4, 64, 128), ("bf16", 6, 64, 300),
             ("bf16", 8, 64, 1000)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dt,R,m,L", FWD_SMALL)
def test_attn_fwd_small(dt, R, m, L, causal):
    w = small(dt, R, m, L)
    q, k, v = W.gen_qkv(w)
    q[0, 1, min(2, L - 1)] = 0.0          # zero query: phi = 0, den = 0, out = 0
    P = params(w)
    want, wden = O.attn_quadratic(q, k, v, P, causal)
    got, gden = _run_fwd(q, k, v, w, causal)
    _check_fwd(tag(w, "causal" if causal else "bidir"), got, gden, want, wden, TOL[dt])
    assert (got[0, 1, min(2, L - 1)] == 0).all()


# q and k rows far from unit length, on every path: fp32 (CUDA cores), bf16 sizes the
# tensor cores take (one feature chunk, two chunks, three 128-feature chunks) and bf16 sizes
# they do not (m % 64 != 0).
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dt,R,m,L", [("f32", 2, 16, 256), ("f32", 4, 64, 200),
                                      ("bf16", 4, 64, 300), ("bf16", 8, 64, 257),
                                      ("bf16", 2, 16, 129), ("bf16", 4, 64, 1000),
                                      ("bf16", 6, 64, 300)])
def test_attn_fwd_scaled_rows(dt, R, m, L, causal):
    w = small(dt, R, m, L, seed=22)
    q, k, v = qkv(w, scaled=True)
    P = params(w)
    want, wden = O.attn_quadratic(q, k, v, P, causal)
    got, gden = _run_fwd(q, k, v, w, causal)
    _check_fwd(tag(w, "causal" if causal else "bidir", True), got, gden, want, wden, TOL[dt])


# Enough (b, h) slices that the sequence is cut into few segments, so one CTA walks
# several 128-token tiles (state carried in tensor memory from tile to tile), with a
# ragged last tile; and B*H >= 148, where a single segment covers the whole sequence.
# F = 512 and 384 run as feature chunks (256 + 256, 3 x 128) summed before the division.
@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("B,H,L,R,m", [(2, 37, 657, 4, 64), (1, 148, 300, 4, 64),
                                       (2, 37, 520, 2, 64), (1, 50, 1111, 4, 64),
                                       (2, 37, 657, 8, 64), (1, 20, 700, 6, 64)])
def test_attn_fwd_multi_tile_segments(B, H, L, R, m, scaled):
    w = W.Workload("multitile", B=B, H=H, L=L, R=R, m=m, dtype="bf16", data_seed=17)
    q, k, v = qkv(w, scaled)
    P = params(w)
    want, wden = O.attn_quadratic(q, k, v, P, True)
    got, gden = _run_fwd(q, k, v, w, True)
    _check_fwd(tag(w, "causal", scaled), got, gden, want, wden, TOL["bf16"])


def test_tiny_workload_both_modes():
    w = W.TINY
    q, k, v = W.gen_qkv(w)
    P = params(w)
    for causal in (True, False):
        want, wden = O.attn_quadratic(q, k, v, P, causal)
        got, gden = _run_fwd(q, k, v, w, causal)
        _check_fwd(tag(w, "tiny causal" if causal else "tiny bidir"), got, gden, want, wden,
                   TOL["f32"])


# (workload, (b, h) slices checked): every slice of the causal workloads, at the first and
# last row of every tile plus random rows; a spread of slices of the wide vision batch.
FULL = [(W.CAUSAL_2K, None), (W.CAUSAL_16K, None), (W.BIDIR_VISION, (4, 3)),
        (W.FWDBWD_8K, None)]


@pytest.mark.parametrize("w,sl", FULL, ids=[x[0].name for x in FULL])
def test_attn_fwd_full_size_sampled(w, sl):
    q, k, v = W.gen_qkv(w)
    got, gden = _run_fwd(q, k, v, w, w.causal)
    assert np.isfinite(got).all() and (gden > 0).all()
    rows = np.union1d(W.tile_border_rows(w.L), W.sample_rows(w.L, 24))
    if sl is None:
        bsel, hsel = slice(0, w.B), slice(0, w.H)
    else:
        bsel = slice(0, w.B, max(1, w.B // sl[0]))
        hsel = slice(0, w.H, max(1, w.H // sl[1]))
    P = params(w)
    want, wden = O.attn_quadratic_rows(q[bsel, hsel], k[bsel, hsel], v[bsel, hsel], P,
                                       w.causal, rows)
    _check_fwd("full " + w.name, got[bsel, hsel][:, :, rows], gden[bsel, hsel][:, :, rows],
               want, wden, TOL[w.dtype])


def test_attn_fwd_full_size_scaled_rows():
    # the headline shape with rows far from unit length (all heads, every tile border)
    w = W.CAUSAL_16K
    q, k, v = qkv(w, scaled=True)
    got, gden = _run_fwd(q, k, v, w, True)
    rows = W.tile_border_rows(w.L)
    P = params(w)
    want, wden = O.attn_quadratic_rows(q, k, v, P, True, rows)
    _check_fwd("full scaled " + w.name, got[:, :, rows], gden[:, :, rows], want, wden,
               TOL["bf16"])


@pytest.mark.parametrize("scaled", [False, True])
def test_bidir_correlated_small(scaled):
    w = small("bf16", 4, 64, 160, B=2, H=3, correlated=True)
    q, k, v = qkv(w, scaled)
    P = params(w)
    want, wden = O.attn_quadratic(q, k, v, P, False)
    got, gden = _run_fwd(q, k, v, w, False)
    _check_fwd(tag(w, "bidir corr", scaled), got, gden, want, wden, TOL["bf16"])


# ------------------------------------------------------------ backward

def _run_bwd(q, k, v, g, w):
    B, H, L, _ = q.shape
    qt, kt, vt, gt = dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype), dev(g, w.dtype)
    out = torch.empty((B, H, L, w.Dv), device="cuda", dtype=TDT[w.dtype])
    den = torch.empty((B, H, L), device="cuda", dtype=torch.float32)
    bd.slay_attn_causal_fwd(qt, kt, vt, out, den, w.R, w.m, w.sketch_seed, _eps(w))
    dq = torch.empty((B, H, L, w.D), device="cuda", dtype=torch.float32)
    dk = torch.empty_like(dq)
    dv = torch.empty((B, H, L, w.Dv), device="cuda", dtype=torch.float32)
    ws = bd.slay_attn_causal_bwd(qt, kt, vt, out, den, gt, dq, dk, dv, w.R, w.m, w.sketch_seed,
                                 _eps(w))
    bd.slay_kernel_status(ws)
    torch.cuda.synchronize()
    return host(dq), host(dk), host(dv)


def _bwd_reference(q, k, v, g, P, dt, rows=None):
    """The oracle's gradients (at every row, or at `rows`) and their per-row scales: the
    same gradients at the oracle's own forward output rounded to dt (the dtype in which the
    backward receives `out`) measure how strongly each row cancels."""
    out, den = O.attn_recurrent(q, k, v, P, True)
    ro, rd = W.to_dtype(out, dt), W.to_dtype(den, "f32")
    if rows is None:
        want = O.attn_causal_bwd(q, k, v, g, P)
        pert = O.attn_causal_bwd_given(q, k, v, ro, rd, g, P)
    else:
        want = O.attn_causal_bwd_rows(q, k, v, g, P, rows)
        pert = O.attn_causal_bwd_given_rows(q, k, v, ro, rd, g, P, rows)
    return want, [gradient_row_scale(a, b, dt) for a, b in zip(want, pert)]


def _check_bwd(name, got, ref, tol, xnorm=None):
    """dq, dk, dv against the oracle.  xnorm: row norms of (q, k) when the rows are far from
    unit length: dq and dk scale as 1/|x|, so rows are weighted by |x| (on both sides) and
    the whole-tensor error is not decided by the smallest rows alone."""
    want, scales = ref
    for i, (nm, g, wv, sc) in enumerate(zip(("dq", "dk", "dv"), got, want, scales)):
        if xnorm is not None and i < 2:
            f = xnorm[i]
            g, wv, sc = g * f[..., None], wv * f[..., None], sc * f
        check("%s %s" % (name, nm), g, wv, tol, row_scale=sc)


def _xnorm(q, k, rows=None):
    nq = np.linalg.norm(np.asarray(q, np.float64), axis=-1)
    nk = np.linalg.norm(np.asarray(k, np.float64), axis=-1)
    if rows is not None:
        nq, nk = nq[..., rows], nk[..., rows]
    return nq, nk


@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("dt,R,m,L", [("f32", 2, 16, 100), ("f32", 4, 64, 130),
                                      ("bf16", 4, 64, 150), ("bf16", 8, 64, 64),
                                      ("bf16", 2, 16, 65), ("bf16", 3, 64, 300)])
def test_attn_bwd_small(dt, R, m, L, scaled):
    w = small(dt, R, m, L)
    q, k, v = qkv(w, scaled)
    g = W.gen_dout(w)
    P = params(w)
    ref = _bwd_reference(q, k, v, g, P, dt)
    got = _run_bwd(q, k, v, g, w)
    _check_bwd(tag(w, "bwd", scaled), got, ref, TOL[dt], _xnorm(q, k) if scaled else None)


# Rows below the 1e-12 norm guard (x^ = x / 1e-12, not a unit vector) and a zero row take the
# guarded derivative; the bf16 path runs the feature map's backward on tensor cores.  The
# guarded rows' gradients are about 1e12 times the others', so they are checked apart: the
# guarded rows on their own, and every other row without them.
@pytest.mark.parametrize("R,m,L", [(4, 64, 200), (8, 64, 130)])
def test_attn_bwd_guarded_rows(R, m, L):
    w = small("bf16", R, m, L)
    q, k, v = W.gen_qkv(w)
    q[0, 0, 3] = W.round_bf16(q[0, 0, 3] * 1e-14)   # inputs stay exact bf16 values
    k[0, 1, 5] = W.round_bf16(k[0, 1, 5] * 1e-14)
    k[0, 0, 7] = 0.0
    g = W.gen_dout(w)
    P = params(w)
    (wq, wk, wv), (sq, sk, sv) = _bwd_reference(q, k, v, g, P, "bf16")
    gq, gk, gv = _run_bwd(q, k, v, g, w)
    name = tag(w, "bwd guarded")
    tol = TOL["bf16"]
    check(name + " dq guarded row", gq[0, 0, 3][None], wq[0, 0, 3][None], tol,
          row_scale=sq[0, 0, 3][None])
    check(name + " dk guarded row", gk[0, 1, 5][None], wk[0, 1, 5][None], tol,
          row_scale=sk[0, 1, 5][None])
    assert (gk[0, 0, 7] == 0).all() and (wk[0, 0, 7] == 0).all()   # zero key: no gradient
    mq = np.ones(gq.shape[:-1], bool)
    mq[0, 0, 3] = False
    mk = np.ones(gk.shape[:-1], bool)
    mk[0, 1, 5] = False
    check(name + " dq other rows", gq[mq], wq[mq], tol, row_scale=sq[mq])
    check(name + " dk other rows", gk[mk], wk[mk], tol, row_scale=sk[mk])
    check(name + " dv", gv, wv, tol, row_scale=sv)


def test_attn_bwd_single_token():
    # L = 1: the only weight is a/(a+eps) ~ 1 - eps/a, so dq and dk are O(eps/a) and come
    # from the cancellation <v, dn> + delta with delta = -<g, out>/Z.  Rounding `out` to
    # bf16 (relative 2^-9) swamps that difference, so the case is checked in fp32, where
    # the same cancellation amplifies fp32 rounding by a/eps: dv to 1e-5, dq and dk to 1e-3.
    w = small("f32", 2, 16, 1)
    q, k, v = W.gen_qkv(w)
    g = W.gen_dout(w)
    P = params(w)
    wq, wk, wv = O.attn_causal_bwd(q, k, v, g, P)
    gq, gk, gv = _run_bwd(q, k, v, g, w)
    check("bwd L1 f32 dv", gv, wv, 1e-5)
    check("bwd L1 f32 dq", gq, wq, 1e-3)
    check("bwd L1 f32 dk", gk, wk, 1e-3)


def test_attn_bwd_many_items():
    # 160 sequences of one tile each: on 148 SMs some CTAs take two (b, h, tile) items in turn
    w = W.Workload("items", B=1, H=160, L=100, R=4, m=64, dtype="bf16", data_seed=23)
    q, k, v = W.gen_qkv(w)
    g = W.gen_dout(w)
    P = params(w)
    ref = _bwd_reference(q, k, v, g, P, "bf16")
    got = _run_bwd(q, k, v, g, w)
    _check_bwd(tag(w, "bwd items"), got, ref, TOL["bf16"])


@pytest.mark.parametrize("scaled", [False, True])
def test_attn_bwd_full_size_sampled(scaled):
    # eight (b, h) slices, the first and last row of every 128-token tile and random rows
    w = W.FWDBWD_8K
    q, k, v = qkv(w, scaled)
    g = W.gen_dout(w)
    gq, gk, gv = _run_bwd(q, k, v, g, w)
    assert np.isfinite(gq).all() and np.isfinite(gk).all() and np.isfinite(gv).all()
    rows = np.union1d(W.tile_border_rows(w.L), W.sample_rows(w.L, 12))
    bsel, hsel = slice(0, 2), slice(0, 16, 4)
    P = params(w)
    qs, ks = q[bsel, hsel], k[bsel, hsel]
    ref = _bwd_reference(qs, ks, v[bsel, hsel], g[bsel, hsel], P, "bf16", rows)
    got = tuple(x[bsel, hsel][:, :, rows] for x in (gq, gk, gv))
    _check_bwd(("full scaled " if scaled else "full ") + w.name + " bwd", got, ref,
               TOL["bf16"], _xnorm(qs, ks, rows) if scaled else None)


# -------------------------------------------------------------- decode

def _run_decode(q, k, v, S, z, w):
    qt, kt, vt = dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype)
    St = torch.from_numpy(S).cuda()
    zt = torch.from_numpy(z).cuda()
    out = torch.empty(v.shape, device="cuda", dtype=TDT[w.dtype])
    bd.slay_decode_step(qt, kt, vt, St, zt, out, w.R, w.m, w.sketch_seed, _eps(w))
    torch.cuda.synchronize()
    return host(out), St.cpu().numpy().astype(np.float64), zt.cpu().numpy().astype(np.float64)


def _check_decode(name, got, want, S, z, dt):
    (go, gS, gz), (wo, wS, wz) = got, want
    tol = TOL[dt]
    check(name + " out", go, wo, tol)
    check(name + " S", gS, wS, 1e-5 if dt == "f32" else tol)
    check(name + " z", gz, wz, 1e-5 if dt == "f32" else tol)
    if dt == "bf16":
        # the increments phi(k) v^T and phi(k) are small next to the states, so they are
        # checked on their own too (whole tensor only: where an increment is far below the
        # state, the fp32 rounding of the stored state decides its row's error); in fp32
        # mode that rounding is of the order of the bar itself, so only S and z are checked
        S0 = S.astype(np.float64)
        z0 = z.astype(np.float64)
        check(name + " dS", gS - S0, wS - S0, tol, row_factor=np.inf)
        check(name + " dz", gz - z0, wz - z0, tol, row_factor=np.inf)


@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("dt,R,m,Bt,H", [("f32", 2, 16, 3, 2), ("f32", 8, 64, 5, 3),
                                         ("bf16", 4, 64, 7, 2), ("bf16", 8, 64, 9, 16)])
def test_decode_small(dt, R, m, Bt, H, scaled):
    w = W.Workload("dec", B=Bt, H=H, L=1, R=R, m=m, dtype=dt, data_seed=31)
    q, k, v, S, z = W.gen_decode(w)
    if scaled:
        q = W.scale_rows(w, q, "q")
        k = W.scale_rows(w, k, "k")
    P = params(w)
    want = O.decode_step(q, k, v, S, z, P)
    got = _run_decode(q, k, v, S, z, w)
    _check_decode("decode %s Bt%dH%d R%d m%d%s" % (dt, Bt, H, R, m, " scaled" if scaled else ""),
                  got, want, S, z, dt)


def test_decode_full_size():
    w = W.DECODE
    q, k, v, S, z = W.gen_decode(w)
    go, gS, gz = _run_decode(q, k, v, S, z, w)
    sel = slice(0, w.B, 8)     # 32 of the 256 sequences, all heads
    P = params(w)
    want = O.decode_step(q[sel], k[sel], v[sel], S[sel], z[sel], P)
    _check_decode("decode full " + w.name, (go[sel], gS[sel], gz[sel]), want, S[sel], z[sel],
                  "bf16")


def test_decode_chain_matches_causal():
    # L decode steps from S = z = 0 reproduce the causal forward rows (GPU vs oracle).
    w = small("f32", 2, 16, 40, B=2, H=2)
    q, k, v = W.gen_qkv(w)
    P = params(w)
    want, _ = O.attn_quadratic(q, k, v, P, True)
    F = w.F
    St = torch.zeros((2, 2, F, 64), device="cuda")
    zt = torch.zeros((2, 2, F), device="cuda")
    outs = []
    for i in range(w.L):
        qi, ki, vi = (dev(np.ascontiguousarray(a[:, :, i]), "f32") for a in (q, k, v))
        o = torch.empty((2, 2, 64), device="cuda")
        bd.slay_decode_step(qi, ki, vi, St, zt, o, w.R, w.m, w.sketch_seed, _eps(w))
        outs.append(o)
    got = torch.stack(outs, dim=2).cpu().numpy()
    check("decode chain f32", got, want, TOL["f32"])


# ------------------------------------------------- bidirectional backward

def _run_bidir_bwd(q, k, v, g, w):
    B, H, L, _ = q.shape
    qt, kt, vt, gt = dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype), dev(g, w.dtype)
    out = torch.empty((B, H, L, w.Dv), device="cuda", dtype=TDT[w.dtype])
    den = torch.empty((B, H, L), device="cuda", dtype=torch.float32)
    bd.slay_attn_bidir_fwd(qt, kt, vt, out, den, w.R, w.m, w.sketch_seed, _eps(w))
    dq = torch.empty((B, H, L, w.D), device="cuda", dtype=torch.float32)
    dk = torch.empty_like(dq)
    dv = torch.empty((B, H, L, w.Dv), device="cuda", dtype=torch.float32)
    ws = bd.slay_attn_bidir_bwd(qt, kt, vt, out, den, gt, dq, dk, dv, w.R, w.m, w.sketch_seed,
                                _eps(w))
    bd.slay_kernel_status(ws)
    bd.slay_kernel_status(None)
    torch.cuda.synchronize()
    return host(dq), host(dk), host(dv)


def _bidir_reference(q, k, v, g, P, dt):
    """The oracle's bidirectional gradients and their per-row cancellation scales (the same
    gradients at the oracle's own forward output rounded to dt; see gradient_row_scale)."""
    out, den = O.attn_quadratic(q, k, v, P, False)
    want = O.attn_bidir_bwd(q, k, v, g, P)
    pert = O.attn_bidir_bwd_given(q, k, v, W.to_dtype(out, dt), W.to_dtype(den, "f32"), g, P)
    return want, [gradient_row_scale(a, b, dt) for a, b in zip(want, pert)]


@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("dt,R,m,L,B,H,corr", [("f32", 2, 16, 100, 1, 2, False),
                                              ("f32", 4, 64, 130, 1, 2, False),
                                              ("bf16", 4, 64, 150, 1, 2, False),
                                              ("bf16", 8, 64, 64, 1, 2, False),
                                              ("bf16", 2, 16, 65, 1, 2, False),
                                              ("bf16", 4, 64, 257, 2, 3, True),
                                              ("bf16", 3, 64, 300, 1, 2, False)])
def test_attn_bidir_bwd_small(dt, R, m, L, B, H, corr, scaled):
    w = small(dt, R, m, L, B=B, H=H, correlated=corr)
    q, k, v = qkv(w, scaled)
    g = W.gen_dout(w)
    P = params(w)
    ref = _bidir_reference(q, k, v, g, P, dt)
    got = _run_bidir_bwd(q, k, v, g, w)
    _check_bwd(tag(w, "bidir bwd" + (" corr" if corr else ""), scaled), got, ref, TOL[dt],
               _xnorm(q, k) if scaled else None)


def test_attn_bidir_bwd_vision_shape_sampled():
    # the vision-shaped workload (32 x 12 sequences of 32 x 32 patches, correlated angles):
    # the whole batch runs, the oracle checks a spread of eight (b, h) sequences in full
    w = W.BIDIR_VISION
    q, k, v = W.gen_qkv(w)
    g = W.gen_dout(w)
    gq, gk, gv = _run_bidir_bwd(q, k, v, g, w)
    assert np.isfinite(gq).all() and np.isfinite(gk).all() and np.isfinite(gv).all()
    bsel, hsel = slice(0, w.B, w.B // 4), slice(0, w.H, w.H // 2)
    P = params(w)
    ref = _bidir_reference(q[bsel, hsel], k[bsel, hsel], v[bsel, hsel], g[bsel, hsel], P, "bf16")
    got = tuple(x[bsel, hsel] for x in (gq, gk, gv))
    _check_bwd("full " + w.name + " bidir bwd", got, ref, TOL["bf16"])


# ------------------------------------------------- feature-map backward

@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("dt_x,dt_g,R,m,n", [("f32", "f32", 2, 16, 1000),
                                             ("f32", "f32", 4, 64, 130),
                                             ("bf16", "bf16", 4, 64, 1000),
                                             ("bf16", "bf16", 8, 64, 4097),
                                             ("bf16", "f32", 4, 64, 333),
                                             ("bf16", "bf16", 2, 16, 777),
                                             ("bf16", "bf16", 4, 32, 38001)])
def test_feature_map_bwd(dt_x, dt_g, R, m, n, scaled):
    w = small(dt_x, R, m, n, B=1, H=1)
    q, _, _ = qkv(w, scaled)
    x = q.reshape(n, 64).copy()
    x[3] = 0.0                                     # zero row: guarded derivative
    x[7] = W.to_dtype(x[7] * 1e-14, dt_x)          # under the 1e-12 norm guard
    gw = W.Workload("g", B=1, H=1, L=n, R=R, m=m, dtype=dt_g, data_seed=w.data_seed)
    G = W.gen_dphi(gw, n)
    P = params(w)
    want = O.feature_map_bwd(x, G, P)
    xt, gt = dev(x, dt_x), dev(G, dt_g)
    dx = torch.empty((n, 64), device="cuda", dtype=torch.float32)
    bd.slay_feature_map_bwd(xt, gt, dx, R, m, w.sketch_seed, _eps(w))
    bd.slay_kernel_status(None)
    torch.cuda.synchronize()
    got = host(dx)
    tol = TOL["bf16"] if "bf16" in (dt_x, dt_g) else TOL["f32"]
    name = "phi bwd %s,%s n%d R%d m%d%s" % (dt_x, dt_g, n, R, m, " scaled" if scaled else "")
    # rows far from unit length have gradients scaled by 1/|x|: weighted by |x| on both sides
    nx = np.linalg.norm(x.astype(np.float64), axis=-1)
    keep = np.ones(n, bool)
    keep[[3, 7]] = False
    check(name, got[keep] * nx[keep, None], want[keep] * nx[keep, None], tol)
    check(name + " guarded row", got[7][None], want[7][None], tol)
    assert np.isfinite(got).all()


# ------------------------------------------ feature-map variants and the contraction

KINDS = {"orthogonal": 1, "signed": 2, "per_head": 3, "performer": 4}


@pytest.mark.parametrize("scaled", [False, True])
@pytest.mark.parametrize("kind", sorted(KINDS))
@pytest.mark.parametrize("dt_in,dt_out,R,m,B,H,L", [("f32", "f32", 2, 16, 1, 3, 100),
                                                   ("bf16", "bf16", 4, 64, 2, 3, 130),
                                                   ("bf16", "f32", 8, 64, 1, 2, 70)])
def test_feature_map_variants(kind, dt_in, dt_out, R, m, B, H, L, scaled):
    w = small(dt_in, R, m, L, B=B, H=H)
    q, _, _ = qkv(w, scaled)
    kd = KINDS[kind]
    F = w.F
    eps = _eps(w)
    if kd == 3:   # per head: the rows of head h use head h's draw
        want = np.concatenate([O.feature_map_kind(q[:, h:h + 1], O.sketch_params_kind(
            64, R, m, w.sketch_seed, eps, kd, h)) for h in range(H)], axis=1)
    else:
        want = O.feature_map_kind(q, O.sketch_params_kind(64, R, m, w.sketch_seed, eps, kd))
    xt = dev(q, dt_in)
    phi = torch.empty((B, H, L, F), device="cuda", dtype=TDT[dt_out])
    bd.slay_feature_map_ex(xt, phi, R, m, w.sketch_seed, eps, kd, heads=H, rows_per_head=L)
    torch.cuda.synchronize()
    tol = TOL["bf16"] if "bf16" in (dt_in, dt_out) else TOL["f32"]
    check("phi %s %s->%s R%d m%d%s" % (kind, dt_in, dt_out, R, m, " scaled" if scaled else ""),
          host(phi), want, tol)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dt,F,L", [("f32", 32, 100), ("f32", 256, 129), ("bf16", 256, 300),
                                    ("bf16", 512, 257), ("bf16", 384, 1)])
def test_linear_attn_on_given_features(dt, F, L, causal):
    # the oracle's features (rounded to the mode's dtype) feed both sides
    w = small(dt, 4, F // 4, L, B=2, H=2)
    q, k, v = W.gen_qkv(w)
    P = O.sketch_params(64, 4, F // 4, w.sketch_seed, _eps(w))
    pq = W.to_dtype(O.feature_map(q, P), dt)
    pk = W.to_dtype(O.feature_map(k, P), dt)
    want, wden = O.attn_from_phi(pq, pk, v, P.eps, causal)
    out = torch.empty(v.shape, device="cuda", dtype=TDT[dt])
    den = torch.empty(v.shape[:-1], device="cuda", dtype=torch.float32)
    ws = bd.slay_linear_attn_fwd(dev(pq, dt), dev(pk, dt), dev(v, dt), out, den, _eps(w), causal)
    bd.slay_kernel_status(ws)
    torch.cuda.synchronize()
    _check_fwd("linear attn %s F%d L%d %s" % (dt, F, L, "causal" if causal else "bidir"),
               host(out), host(den), want, wden, TOL[dt])


@pytest.mark.parametrize("kind", ["performer", "orthogonal"])
def test_variant_attention_composed(kind):
    # a variant's map for q and k, then the contraction, against the oracle's composition
    w = small("bf16", 4, 64, 200, B=1, H=2, seed=24)
    q, k, v = W.gen_qkv(w)
    kd = KINDS[kind]
    P = O.sketch_params_kind(64, 4, 64, w.sketch_seed, _eps(w), kd)
    want, wden = O.attn_from_phi(O.feature_map_kind(q, P), O.feature_map_kind(k, P), v, P.eps,
                                 True)
    pq = torch.empty((1, 2, 200, 256), device="cuda", dtype=torch.bfloat16)
    pk = torch.empty_like(pq)
    bd.slay_feature_map_ex(dev(q, "bf16"), pq, 4, 64, w.sketch_seed, _eps(w), kd)
    bd.slay_feature_map_ex(dev(k, "bf16"), pk, 4, 64, w.sketch_seed, _eps(w), kd)
    out = torch.empty((1, 2, 200, 64), device="cuda", dtype=torch.bfloat16)
    den = torch.empty((1, 2, 200), device="cuda", dtype=torch.float32)
    bd.slay_linear_attn_fwd(pq, pk, dev(v, "bf16"), out, den, _eps(w), True)
    torch.cuda.synchronize()
    _check_fwd("composed %s causal" % kind, host(out), host(den), want, wden, TOL["bf16"])


# ------------------------------------------- state continuation, sequence parallelism

@pytest.mark.parametrize("dt,R,m,L,cuts", [("bf16", 4, 64, 1000, (300, 700)),
                                           ("bf16", 8, 64, 700, (128, 512)),
                                           ("f32", 2, 16, 300, (1, 150)),
                                           ("bf16", 2, 16, 257, (64, 65))])
def test_sequence_pieces_emulating_ranks(dt, R, m, L, cuts):
    # the sequence-parallel decomposition on one GPU: every piece's state, the exclusive
    # prefix over pieces, each piece's forward from that prefix; the pieces' outputs and the
    # last piece's final state against the oracle's whole-sequence forward
    w = small(dt, R, m, L, B=1, H=3, seed=25)
    q, k, v = W.gen_qkv(w)
    P = params(w)
    want, wden, wS, wz = O.attn_causal_state(q, k, v, P)
    bounds = (0,) + tuple(cuts) + (L,)
    pieces = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    F = w.F
    eps = _eps(w)
    Ss, zs = [], []
    for a, b in pieces:
        S = torch.empty((1, 3, F, 64), device="cuda")
        z = torch.empty((1, 3, F), device="cuda")
        ws = bd.slay_causal_state(dev(k[:, :, a:b], dt), dev(v[:, :, a:b], dt), S, z, R, m,
                                  w.sketch_seed, eps)
        bd.slay_kernel_status(ws)
        Ss.append(S)
        zs.append(z)
    S_all, z_all = torch.stack(Ss), torch.stack(zs)
    outs, dens = [], []
    S_fin = torch.empty((1, 3, F, 64), device="cuda")
    z_fin = torch.empty((1, 3, F), device="cuda")
    for r, (a, b) in enumerate(pieces):
        S_in = torch.empty((1, 3, F, 64), device="cuda")
        z_in = torch.empty((1, 3, F), device="cuda")
        bd.slay_state_prefix(S_all, z_all, r, S_in, z_in)
        out = torch.empty((1, 3, b - a, 64), device="cuda", dtype=TDT[dt])
        den = torch.empty((1, 3, b - a), device="cuda")
        last = r == len(pieces) - 1
        ws = bd.slay_attn_causal_fwd_state(dev(q[:, :, a:b], dt), dev(k[:, :, a:b], dt),
                                           dev(v[:, :, a:b], dt), out, den, R, m, w.sketch_seed,
                                           eps, S_in=S_in, z_in=z_in,
                                           S_out=S_fin if last else None,
                                           z_out=z_fin if last else None)
        bd.slay_kernel_status(ws)
        outs.append(host(out))
        dens.append(host(den))
    torch.cuda.synchronize()
    name = "pieces %s R%d m%d L%d %s" % (dt, R, m, L, cuts)
    _check_fwd(name, np.concatenate(outs, axis=2), np.concatenate(dens, axis=2), want, wden,
               TOL[dt])
    # the states are fp32 sums on both sides; in bf16 mode phi(k) is rounded to bf16 first
    check(name + " final S", host(S_fin), wS, TOL[dt])
    check(name + " final z", host(z_fin), wz, TOL[dt])
    check(name + " piece-0 S", host(Ss[0]), O.attn_causal_state(
        q[:, :, :cuts[0]], k[:, :, :cuts[0]], v[:, :, :cuts[0]], P)[2], TOL[dt])


@pytest.mark.parametrize("dt,R,m,L,cuts", [("bf16", 4, 64, 1000, (300, 700)),
                                           ("bf16", 8, 64, 700, (128, 512)),
                                           ("bf16", 4, 64, 600, (0, 600)),
                                           ("f32", 2, 16, 300, (1, 150)),
                                           ("bf16", 2, 16, 257, (64, 65))])
def test_two_call_forward_emulating_ranks(dt, R, m, L, cuts):
    # the two-call forward: every piece's begin (its state, phi(k) kept in its own
    # workspace), the prefix over pieces, every piece's finish; the outputs against the
    # oracle's whole-sequence forward and bit for bit against the one-call continuation on
    # the same prefix (the same output kernel on the same phi(k) and sums)
    w = small(dt, R, m, L, B=1, H=3, seed=27)
    q, k, v = W.gen_qkv(w)
    P = params(w)
    want, wden, _, _ = O.attn_causal_state(q, k, v, P)
    bounds = (0,) + tuple(cuts) + (L,)
    pieces = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    F, eps = w.F, _eps(w)
    qt, kt, vt = dev(q, dt), dev(k, dt), dev(v, dt)

    def piece(t, a, b):
        return t[:, :, a:b].contiguous()

    Ss, zs, wss = [], [], []
    for a, b in pieces:
        S = torch.full((1, 3, F, 64), float("nan"), device="cuda")
        z = torch.full((1, 3, F), float("nan"), device="cuda")
        wss.append(bd.slay_attn_causal_fwd_begin(piece(kt, a, b), piece(vt, a, b), S, z, R, m,
                                                 w.sketch_seed, eps))
        Ss.append(S)
        zs.append(z)
    S_all, z_all = torch.stack(Ss), torch.stack(zs)
    outs, dens = [], []
    for r, (a, b) in enumerate(pieces):
        S_in = torch.empty((1, 3, F, 64), device="cuda")
        z_in = torch.empty((1, 3, F), device="cuda")
        bd.slay_state_prefix(S_all, z_all, r, S_in, z_in)
        out = torch.empty((1, 3, b - a, 64), device="cuda", dtype=TDT[dt])
        den = torch.empty((1, 3, b - a), device="cuda")
        bd.slay_attn_causal_fwd_finish(piece(qt, a, b), piece(kt, a, b), piece(vt, a, b), out,
                                       den, R, m, w.sketch_seed, eps, wss[r], S_in=S_in,
                                       z_in=z_in)
        bd.slay_kernel_status(wss[r])
        ref = torch.empty_like(out)
        rden = torch.empty_like(den)
        bd.slay_attn_causal_fwd_state(piece(qt, a, b), piece(kt, a, b), piece(vt, a, b), ref,
                                      rden, R, m, w.sketch_seed, eps, S_in=S_in, z_in=z_in)
        torch.cuda.synchronize()
        assert torch.equal(out, ref) and torch.equal(den, rden), (r, a, b)
        outs.append(host(out))
        dens.append(host(den))
    name = "two-call %s R%d m%d L%d %s" % (dt, R, m, L, cuts)
    _check_fwd(name, np.concatenate(outs, axis=2), np.concatenate(dens, axis=2), want, wden,
               TOL[dt])
    for (a, b), S, z in zip(pieces, Ss, zs):
        if b == a:   # an empty piece: zero state
            assert not torch.any(S) and not torch.any(z)
            continue
        _, _, wS, wz = O.attn_causal_state(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], P)
        check(name + " piece S", host(S), wS, TOL[dt])
        check(name + " piece z", host(z), wz, TOL[dt])


@pytest.mark.parametrize("dt,R,m,L,cuts", [("bf16", 4, 64, 1000, (300, 700)),
                                           ("bf16", 8, 64, 700, (128, 512)),
                                           ("bf16", 4, 64, 600, (0, 600)),
                                           ("f32", 2, 16, 300, (1, 150)),
                                           ("bf16", 2, 16, 257, (64, 65))])
def test_two_call_backward_emulating_ranks(dt, R, m, L, cuts):
    # the two-call backward: every piece's begin (its phi(q)[dn, delta] sum, phi(q) and the
    # row statistics kept in its own workspace) before any finish; the gradients bit for bit
    # against the one-call piece backward on the same outside sums, and against the oracle's
    # whole-sequence backward
    w = small(dt, R, m, L, B=1, H=3, seed=29)
    q, k, v = W.gen_qkv(w)
    g = W.gen_dout(w)
    P = params(w)
    F, eps = w.F, _eps(w)
    qt, kt, vt, gt = dev(q, dt), dev(k, dt), dev(v, dt), dev(g, dt)
    out = torch.empty((1, 3, L, 64), device="cuda", dtype=TDT[dt])
    den = torch.empty((1, 3, L), device="cuda")
    bd.slay_attn_causal_fwd(qt, kt, vt, out, den, R, m, w.sketch_seed, eps)
    bounds = (0,) + tuple(cuts) + (L,)
    pieces = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]

    def piece(t, a, b):
        return t[:, :, a:b].contiguous()

    def state_pair():
        return torch.empty((1, 3, F, 64), device="cuda"), torch.empty((1, 3, F), device="cuda")

    Ss, zs, Gs, zgs, wss = [], [], [], [], []
    for a, b in pieces:
        S, z = state_pair()
        bd.slay_kernel_status(bd.slay_causal_state(piece(kt, a, b), piece(vt, a, b), S, z, R, m,
                                                    w.sketch_seed, eps))
        G, zg = state_pair()
        wss.append(bd.slay_attn_causal_bwd_begin(piece(qt, a, b), piece(out, a, b),
                                                 piece(den, a, b), piece(gt, a, b), G, zg, R, m,
                                                 w.sketch_seed, eps))
        Ss.append(S)
        zs.append(z)
        Gs.append(G)
        zgs.append(zg)
    S_all, z_all, G_all, zg_all = (torch.stack(x) for x in (Ss, zs, Gs, zgs))
    grads = []
    for r, (a, b) in enumerate(pieces):
        S_in, z_in = state_pair()
        G_in, zg_in = state_pair()
        bd.slay_state_prefix(S_all, z_all, r, S_in, z_in)
        bd.slay_state_suffix(G_all, zg_all, r, G_in, zg_in)
        n = b - a
        args = [piece(t, a, b) for t in (qt, kt, vt, out, den, gt)]
        got = [torch.empty((1, 3, n, 64), device="cuda") for _ in range(3)]
        ref = [torch.empty((1, 3, n, 64), device="cuda") for _ in range(3)]
        bd.slay_attn_causal_bwd_finish(*args, *got, R, m, w.sketch_seed, eps, wss[r], S_in=S_in,
                                       z_in=z_in, G_in=G_in, zg_in=zg_in)
        bd.slay_kernel_status(wss[r])
        bd.slay_kernel_status(bd.slay_attn_causal_bwd_state(*args, *ref, R, m, w.sketch_seed, eps,
                                                            S_in=S_in, z_in=z_in, G_in=G_in,
                                                            zg_in=zg_in))
        torch.cuda.synchronize()
        for x, y in zip(got, ref):
            assert torch.equal(x, y), (r, a, b)
        grads.append(tuple(host(x) for x in got))
    name = "two-call bwd %s R%d m%d L%d %s" % (dt, R, m, L, cuts)
    got = tuple(np.concatenate([x[i] for x in grads], axis=2) for i in range(3))
    _check_bwd(name, got, _bwd_reference(q, k, v, g, P, dt), TOL[dt])


def test_two_call_forward_rejects_small_workspace():
    w = small("bf16", 4, 64, 512, B=1, H=2, seed=28)
    q, k, v = (dev(x, "bf16") for x in W.gen_qkv(w))
    S = torch.empty((1, 2, 256, 64), device="cuda")
    z = torch.empty((1, 2, 256), device="cuda")
    need = bd.slay_workspace_bytes(bd.OP_CAUSAL_FWD_SPLIT, torch.bfloat16, 1, 2, 512, 64, 64, 4, 64)
    # the two-call workspace keeps phi(k): larger than the one-call forward's
    assert need >= bd.slay_workspace_bytes(bd.OP_CAUSAL_FWD, torch.bfloat16, 1, 2, 512, 64, 64,
                                           4, 64)
    small_ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(bd.SlayError):
        bd.slay_attn_causal_fwd_begin(k, v, S, z, 4, 64, w.sketch_seed, _eps(w), workspace=small_ws)
    out = torch.empty((1, 2, 512, 64), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(bd.SlayError):
        bd.slay_attn_causal_fwd_finish(q, k, v, out, None, 4, 64, w.sketch_seed, _eps(w), small_ws)
    with pytest.raises(bd.SlayError):   # the state outputs are required
        bd.slay_attn_causal_fwd_begin(k, v, None, None, 4, 64, w.sketch_seed, _eps(w))


@pytest.mark.parametrize("dt,R,m,L,cuts", [("bf16", 4, 64, 1000, (300, 700)),
                                           ("bf16", 8, 64, 700, (128, 512)),
                                           ("f32", 2, 16, 300, (1, 150)),
                                           ("bf16", 2, 16, 257, (64, 65))])
def test_sequence_pieces_backward_emulating_ranks(dt, R, m, L, cuts):
    # the sequence-parallel backward on one GPU: every piece's forward state (prefix over
    # the pieces before it) and its sum of phi(q)[dn, delta] (suffix over the pieces after
    # it), then each piece's backward from both; the pieces' gradients against the oracle's
    # whole-sequence backward, and a piece's phi(q)[dn, delta] sum against the oracle's
    w = small(dt, R, m, L, B=1, H=3, seed=26)
    q, k, v = W.gen_qkv(w)
    g = W.gen_dout(w)
    P = params(w)
    F, eps = w.F, _eps(w)
    qt, kt, vt, gt = dev(q, dt), dev(k, dt), dev(v, dt), dev(g, dt)
    out = torch.empty((1, 3, L, 64), device="cuda", dtype=TDT[dt])
    den = torch.empty((1, 3, L), device="cuda")
    bd.slay_attn_causal_fwd(qt, kt, vt, out, den, R, m, w.sketch_seed, eps)
    bounds = (0,) + tuple(cuts) + (L,)
    pieces = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]

    def piece(t, a, b):
        return t[:, :, a:b].contiguous()

    def state_pair():
        return torch.empty((1, 3, F, 64), device="cuda"), torch.empty((1, 3, F), device="cuda")

    Ss, zs, Gs, zgs = [], [], [], []
    for a, b in pieces:
        S, z = state_pair()
        bd.slay_kernel_status(bd.slay_causal_state(piece(kt, a, b), piece(vt, a, b), S, z, R, m,
                                                    w.sketch_seed, eps))
        G, zg = state_pair()
        bd.slay_kernel_status(bd.slay_causal_bwd_state(piece(qt, a, b), piece(out, a, b),
                                                       piece(den, a, b), piece(gt, a, b), G, zg,
                                                       R, m, w.sketch_seed, eps))
        Ss.append(S)
        zs.append(z)
        Gs.append(G)
        zgs.append(zg)
    S_all, z_all, G_all, zg_all = (torch.stack(x) for x in (Ss, zs, Gs, zgs))
    grads = []
    for r, (a, b) in enumerate(pieces):
        S_in, z_in = state_pair()
        G_in, zg_in = state_pair()
        bd.slay_state_prefix(S_all, z_all, r, S_in, z_in)
        bd.slay_state_suffix(G_all, zg_all, r, G_in, zg_in)
        n = b - a
        dq = torch.empty((1, 3, n, 64), device="cuda")
        dk = torch.empty_like(dq)
        dv = torch.empty_like(dq)
        ws = bd.slay_attn_causal_bwd_state(piece(qt, a, b), piece(kt, a, b), piece(vt, a, b),
                                           piece(out, a, b), piece(den, a, b), piece(gt, a, b),
                                           dq, dk, dv, R, m, w.sketch_seed, eps, S_in=S_in,
                                           z_in=z_in, G_in=G_in, zg_in=zg_in)
        bd.slay_kernel_status(ws)
        grads.append((host(dq), host(dk), host(dv)))
    torch.cuda.synchronize()
    name = "bwd pieces %s R%d m%d L%d %s" % (dt, R, m, L, cuts)
    got = tuple(np.concatenate([x[i] for x in grads], axis=2) for i in range(3))
    _check_bwd(name, got, _bwd_reference(q, k, v, g, P, dt), TOL[dt])
    # the first piece's sum of phi(q)[dn, delta] at the library's forward output
    a, b = pieces[0]
    ow, dw = host(out)[:, :, a:b], host(den)[:, :, a:b]
    _, _, _, wG, wzg = O.attn_causal_bwd_state(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], ow, dw,
                                                W.to_dtype(g, dt)[:, :, a:b], P)
    check(name + " piece-0 G", host(Gs[0]), wG, TOL[dt])
    check(name + " piece-0 zg", host(zgs[0]), wzg, TOL[dt])
