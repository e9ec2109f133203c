"""Thin ctypes binding of libslay.so (the C ABI declared in include/slay.h).

Argument marshalling only: each function checks the torch tensors it is given
(device, dtype, contiguity, shape), passes their device pointers and the current CUDA
stream to the C entry point of the same name, and raises SlayError on a non-zero
status.  Every step of the computation runs in the library's CUDA kernels; there is no
Python or CPU fallback, and the first call raises if the library is missing.
"""
import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libslay.so")

SLAY_OK, SLAY_ERR_INVALID_ARG, SLAY_ERR_UNSUPPORTED, SLAY_ERR_CUDA, SLAY_ERR_TIMEOUT, \
    SLAY_ERR_NO_MEMORY = range(6)
SLAY_F32, SLAY_BF16 = 0, 1
OP_FEATURE_MAP, OP_CAUSAL_FWD, OP_BIDIR_FWD, OP_CAUSAL_BWD, OP_DECODE, OP_BIDIR_BWD, \
    OP_LINEAR_ATTN, OP_CAUSAL_STATE, OP_CAUSAL_FWD_SPLIT, OP_FEATURE_MAP_BWD = range(10)
PATH_TC_FEATURE_MAP, PATH_TC_CONTRACTION, PATH_TC_PHI_BWD = 1, 2, 4
PHI_ANCHOR, PHI_ORTHOGONAL, PHI_SIGNED, PHI_PER_HEAD, PHI_PERFORMER = range(5)

EXPORTS = ["slay_feature_map", "slay_attn_causal_fwd", "slay_attn_bidir_fwd",
           "slay_attn_causal_bwd", "slay_decode_step", "slay_workspace_bytes", "slay_prepare",
           "slay_sketch_params", "slay_status_string", "slay_last_error", "slay_trace_enable",
           "slay_trace_read", "slay_attn_causal_fwd_noalloc", "slay_kernel_status",
           "slay_debug_expire_wait", "slay_attn_bidir_bwd", "slay_feature_map_bwd",
           "slay_feature_map_ex", "slay_sketch_params_ex", "slay_linear_attn_fwd",
           "slay_attn_causal_fwd_state", "slay_causal_state", "slay_state_prefix",
           "slay_state_suffix", "slay_attn_causal_bwd_state", "slay_causal_bwd_state",
           "slay_attn_causal_fwd_begin", "slay_attn_causal_fwd_finish", "slay_path",
           "slay_attn_causal_bwd_begin", "slay_attn_causal_bwd_finish"]


class SlayError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = "%s: %s" % (where, lib().slay_status_string(status).decode())
        detail = lib().slay_last_error().decode()
        if status in (SLAY_ERR_CUDA, SLAY_ERR_TIMEOUT) and detail:
            msg += " (%s)" % detail
        super().__init__(msg)


_lib = None


def lib():
    """Load libslay.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libslay.so not found at %s: build it with "
                           "`python -m kernelized_linear_attention_unit_b200.build`" % LIB_PATH)
    L = C.CDLL(LIB_PATH)
    vp, i32, i64, u64, f32, sz = C.c_void_p, C.c_int, C.c_int64, C.c_uint64, C.c_float, C.c_size_t
    L.slay_feature_map.argtypes = [vp, vp, i64, i32, i32, i32, i32, i32, u64, f32, vp]
    attn = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, u64, f32, vp, sz, vp]
    L.slay_attn_causal_fwd.argtypes = attn
    L.slay_attn_bidir_fwd.argtypes = attn
    L.slay_attn_causal_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                               i32, i32, u64, f32, vp]
    L.slay_attn_causal_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                       i32, i32, i32, i32, u64, f32, vp, sz, vp]
    L.slay_attn_bidir_bwd.argtypes = L.slay_attn_causal_bwd.argtypes
    L.slay_feature_map_bwd.argtypes = [vp, vp, vp, i64, i32, i32, i32, i32, i32, u64, f32, vp]
    L.slay_feature_map_ex.argtypes = [vp, vp, i64, i32, i32, i32, i32, i32, u64, f32, i32, i32,
                                      i64, vp]
    L.slay_sketch_params_ex.argtypes = [i32, i32, i32, u64, f32, i32, i32, vp, vp, vp, vp, vp]
    L.slay_linear_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32,
                                       i32, vp, sz, vp]
    L.slay_attn_causal_fwd_state.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                             i32, i32, i32, i32, i32, u64, f32, vp, sz, vp]
    L.slay_causal_state.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                    u64, f32, vp, sz, vp]
    L.slay_attn_causal_fwd_begin.argtypes = [vp] * 4 + [i32] * 8 + [u64, f32, vp, sz, vp]
    L.slay_attn_causal_fwd_finish.argtypes = [vp] * 7 + [i32] * 8 + [u64, f32, vp, sz, vp]
    L.slay_state_prefix.argtypes = [vp, vp, i32, i32, vp, vp, i32, i32, i32, vp]
    L.slay_state_suffix.argtypes = L.slay_state_prefix.argtypes
    L.slay_attn_causal_bwd_state.argtypes = [vp] * 13 + [i32] * 8 + [u64, f32, vp, sz, vp]
    L.slay_causal_bwd_state.argtypes = [vp] * 6 + [i32] * 8 + [u64, f32, vp, sz, vp]
    L.slay_attn_causal_bwd_begin.argtypes = L.slay_causal_bwd_state.argtypes
    L.slay_attn_causal_bwd_finish.argtypes = L.slay_attn_causal_bwd_state.argtypes
    L.slay_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                   u64, f32, vp]
    L.slay_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32]
    L.slay_workspace_bytes.restype = sz
    L.slay_path.argtypes = [i32] * 9
    L.slay_path.restype = i32
    L.slay_prepare.argtypes = [i32, i32, i32, u64, f32]
    L.slay_sketch_params.argtypes = [i32, i32, i32, u64, f32, vp, vp, vp, vp]
    L.slay_status_string.argtypes = [i32]
    L.slay_status_string.restype = C.c_char_p
    L.slay_last_error.argtypes = []
    L.slay_last_error.restype = C.c_char_p
    L.slay_kernel_status.argtypes = [vp, vp]
    L.slay_kernel_status.restype = i32
    L.slay_debug_expire_wait.argtypes = [i32]
    L.slay_debug_expire_wait.restype = i32
    L.slay_trace_enable.argtypes = [i32]
    L.slay_trace_enable.restype = i32
    L.slay_trace_read.argtypes = [C.POINTER(C.c_char_p), C.POINTER(C.c_float), i32]
    L.slay_trace_read.restype = i32
    for name in ("slay_feature_map", "slay_attn_causal_fwd", "slay_attn_bidir_fwd",
                 "slay_attn_causal_bwd", "slay_decode_step", "slay_prepare",
                 "slay_attn_bidir_bwd", "slay_feature_map_bwd", "slay_feature_map_ex",
                 "slay_sketch_params_ex", "slay_linear_attn_fwd", "slay_attn_causal_fwd_state",
                 "slay_causal_state", "slay_state_prefix", "slay_state_suffix",
                 "slay_attn_causal_bwd_state", "slay_causal_bwd_state",
                 "slay_attn_causal_fwd_noalloc", "slay_attn_causal_fwd_begin",
                 "slay_attn_causal_fwd_finish", "slay_attn_causal_bwd_begin",
                 "slay_attn_causal_bwd_finish",
                 "slay_sketch_params"):
        getattr(L, name).restype = i32
    _lib = L
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SLAY_F32
    if t.dtype == torch.bfloat16:
        return SLAY_BF16
    raise TypeError("dtype %s not supported (float32 or bfloat16)" % t.dtype)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _check(t, name, dtype=None, shape=None):
    if t is None:
        raise ValueError("%s is required" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _raise(status, where):
    if status != SLAY_OK:
        raise SlayError(status, where)


def slay_workspace_bytes(op, dtype, B, H, L, D, Dv, R, m) -> int:
    dt = dtype if isinstance(dtype, int) else _dt(torch.empty(0, dtype=dtype))
    n = lib().slay_workspace_bytes(op, dt, B, H, L, D, Dv, R, m)
    if n == C.c_size_t(-1).value:
        raise SlayError(SLAY_ERR_UNSUPPORTED, "slay_workspace_bytes")
    return int(n)


def slay_path(op, dtype, B, H, L, D, Dv, R, m) -> int:
    """Mask of PATH_* bits: which steps of `op` run on tensor cores at these sizes (0: all
    on CUDA cores); raises for sizes the op rejects."""
    dt = dtype if isinstance(dtype, int) else _dt(torch.empty(0, dtype=dtype))
    n = lib().slay_path(op, dt, B, H, L, D, Dv, R, m)
    if n < 0:
        raise SlayError(SLAY_ERR_UNSUPPORTED, "slay_path")
    return n


def alloc_workspace(op, dtype, B, H, L, D, Dv, R, m, device=None):
    """Caller-owned workspace of the size the library asks for (torch allocation).  When the
    call needs none (empty work, which enqueues nothing and leaves the workspace as it is),
    a zeroed 256-byte block, so that slay_kernel_status on it reads a clear status word."""
    n = slay_workspace_bytes(op, dtype, B, H, L, D, Dv, R, m)
    if n == 0:
        return torch.zeros(256, dtype=torch.uint8, device=device or "cuda")
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def slay_prepare(D, R, m, seed, eps):
    _raise(lib().slay_prepare(D, R, m, seed, eps), "slay_prepare")


def slay_sketch_params(D, R, m, seed, eps):
    """Host copy of (omega [F,D] f32, anchors [F,D] f32, s [R] f64, wt [R] f64)."""
    import numpy as np
    F = R * m
    om = np.zeros((F, D), dtype=np.float32)
    an = np.zeros((F, D), dtype=np.float32)
    s = np.zeros(R, dtype=np.float64)
    w = np.zeros(R, dtype=np.float64)
    _raise(lib().slay_sketch_params(D, R, m, seed, eps, om.ctypes.data, an.ctypes.data,
                                    s.ctypes.data, w.ctypes.data), "slay_sketch_params")
    return om, an, s, w


def slay_trace_enable(on: bool):
    _raise(lib().slay_trace_enable(1 if on else 0), "slay_trace_enable")


def slay_trace_read(cap: int = 1 << 16):
    """List of (kernel name, milliseconds) for the launches recorded since the last read."""
    names = (C.c_char_p * cap)()
    ms = (C.c_float * cap)()
    n = lib().slay_trace_read(names, ms, cap)
    return [(names[i].decode(), float(ms[i])) for i in range(min(n, cap))]


def slay_feature_map(x, phi, R, m, seed, eps, stream=None):
    """phi[n, R*m] = phi(x[n, D]); x f32 -> phi f32, x bf16 -> phi bf16 or f32."""
    _check(x, "x")
    _check(phi, "phi")
    D = x.shape[-1]
    n = x.numel() // D if D else 0
    if phi.numel() != n * R * m or phi.shape[-1] != R * m:
        raise ValueError("phi must have %d rows of %d features" % (n, R * m))
    _raise(lib().slay_feature_map(_ptr(x), _ptr(phi), n, D, _dt(x), _dt(phi), R, m, seed, eps,
                                  _stream(stream)), "slay_feature_map")


def _attn(fn, name, op, q, k, v, out, den, R, m, seed, eps, workspace, stream):
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    _check(k, "k", q.dtype, (B, H, L, D))
    _check(v, "v", q.dtype, (B, H, L, Dv))
    _check(out, "out", q.dtype, (B, H, L, Dv))
    if den is not None:
        _check(den, "den", torch.float32, (B, H, L))
    dt = _dt(q)
    need = slay_workspace_bytes(op, dt, B, H, L, D, Dv, R, m)
    if workspace is None:
        workspace = alloc_workspace(op, dt, B, H, L, D, Dv, R, m, q.device)
    _check(workspace, "workspace")
    wbytes = workspace.numel() * workspace.element_size()
    if wbytes < need:
        raise ValueError("workspace has %d bytes, %d needed" % (wbytes, need))
    _raise(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(den), B, H, L, D, Dv, dt, R, m, seed,
              eps, _ptr(workspace), wbytes, _stream(stream)), name)
    return workspace


def slay_attn_causal_fwd(q, k, v, out, den, R, m, seed, eps, workspace=None, stream=None):
    """Enqueue the causal forward; returns the workspace it used (see slay_kernel_status)."""
    return _attn(lib().slay_attn_causal_fwd, "slay_attn_causal_fwd", OP_CAUSAL_FWD, q, k, v, out, den,
          R, m, seed, eps, workspace, stream)


def slay_attn_bidir_fwd(q, k, v, out, den, R, m, seed, eps, workspace=None, stream=None):
    """Enqueue the bidirectional forward; returns the workspace it used."""
    return _attn(lib().slay_attn_bidir_fwd, "slay_attn_bidir_fwd", OP_BIDIR_FWD, q, k, v, out, den,
          R, m, seed, eps, workspace, stream)


def slay_attn_causal_fwd_noalloc(q, k, v, out, den, R, m, seed, eps, stream=None):
    """Causal forward that allocates nothing (library-owned static scratch, 32 MiB max)."""
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    _check(k, "k", q.dtype, (B, H, L, D))
    _check(v, "v", q.dtype, (B, H, L, Dv))
    _check(out, "out", q.dtype, (B, H, L, Dv))
    if den is not None:
        _check(den, "den", torch.float32, (B, H, L))
    _raise(lib().slay_attn_causal_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(den), B,
                                              H, L, D, Dv, _dt(q), R, m, seed, eps,
                                              _stream(stream)), "slay_attn_causal_fwd_noalloc")


def _attn_bwd(fn, name, op, q, k, v, out, den, dout, dq, dk, dv, R, m, seed, eps, workspace,
              stream):
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    _check(k, "k", q.dtype, (B, H, L, D))
    _check(v, "v", q.dtype, (B, H, L, Dv))
    _check(out, "out", q.dtype, (B, H, L, Dv))
    _check(den, "den", torch.float32, (B, H, L))
    _check(dout, "dout", q.dtype, (B, H, L, Dv))
    _check(dq, "dq", torch.float32, (B, H, L, D))
    _check(dk, "dk", torch.float32, (B, H, L, D))
    _check(dv, "dv", torch.float32, (B, H, L, Dv))
    dt = _dt(q)
    need = slay_workspace_bytes(op, dt, B, H, L, D, Dv, R, m)
    if workspace is None:
        workspace = alloc_workspace(op, dt, B, H, L, D, Dv, R, m, q.device)
    wbytes = workspace.numel() * workspace.element_size()
    if wbytes < need:
        raise ValueError("workspace has %d bytes, %d needed" % (wbytes, need))
    _raise(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(den), _ptr(dout), _ptr(dq), _ptr(dk),
              _ptr(dv), B, H, L, D, Dv, dt, R, m, seed, eps, _ptr(workspace), wbytes,
              _stream(stream)), name)
    return workspace


def slay_attn_causal_bwd(q, k, v, out, den, dout, dq, dk, dv, R, m, seed, eps, workspace=None,
                         stream=None):
    """Enqueue the causal backward; returns the workspace it used."""
    return _attn_bwd(lib().slay_attn_causal_bwd, "slay_attn_causal_bwd", OP_CAUSAL_BWD, q, k, v,
                     out, den, dout, dq, dk, dv, R, m, seed, eps, workspace, stream)


def slay_attn_bidir_bwd(q, k, v, out, den, dout, dq, dk, dv, R, m, seed, eps, workspace=None,
                        stream=None):
    """Enqueue the bidirectional backward; returns the workspace it used."""
    return _attn_bwd(lib().slay_attn_bidir_bwd, "slay_attn_bidir_bwd", OP_BIDIR_BWD, q, k, v,
                     out, den, dout, dq, dk, dv, R, m, seed, eps, workspace, stream)


def slay_feature_map_ex(x, phi, R, m, seed, eps, kind, heads=1, rows_per_head=0, stream=None):
    """phi of a variant kind (PHI_*); per-head rows are sequences of rows_per_head rows."""
    _check(x, "x")
    _check(phi, "phi")
    D = x.shape[-1]
    n = x.numel() // D if D else 0
    if phi.numel() != n * R * m or phi.shape[-1] != R * m:
        raise ValueError("phi must have %d rows of %d features" % (n, R * m))
    _raise(lib().slay_feature_map_ex(_ptr(x), _ptr(phi), n, D, _dt(x), _dt(phi), R, m, seed,
                                     eps, kind, heads, rows_per_head, _stream(stream)),
           "slay_feature_map_ex")


def slay_sketch_params_ex(D, R, m, seed, eps, kind, head=0):
    """Host copy of a variant's (omega, anchors, anchors_b [F,D] f32, s, wt [R] f64)."""
    import numpy as np
    F = R * m
    om = np.zeros((F, D), np.float32)
    an = np.zeros((F, D), np.float32)
    anb = np.zeros((F, D), np.float32)
    s = np.zeros(R, np.float64)
    w = np.zeros(R, np.float64)
    _raise(lib().slay_sketch_params_ex(D, R, m, seed, eps, kind, head, om.ctypes.data,
                                       an.ctypes.data, anb.ctypes.data, s.ctypes.data,
                                       w.ctypes.data), "slay_sketch_params_ex")
    return om, an, anb, s, w


def slay_linear_attn_fwd(phq, phk, v, out, den, eps, causal, workspace=None, stream=None):
    """The contraction on given features phq, phk [B,H,L,F] (causal or bidirectional)."""
    _check(phq, "phq")
    B, H, L, F = phq.shape
    Dv = v.shape[-1]
    _check(phk, "phk", phq.dtype, (B, H, L, F))
    _check(v, "v", phq.dtype, (B, H, L, Dv))
    _check(out, "out", phq.dtype, (B, H, L, Dv))
    if den is not None:
        _check(den, "den", torch.float32, (B, H, L))
    dt = _dt(phq)
    if workspace is None:
        workspace = alloc_workspace(OP_LINEAR_ATTN, dt, B, H, L, 64, Dv, 1, F, phq.device)
    wbytes = workspace.numel() * workspace.element_size()
    _raise(lib().slay_linear_attn_fwd(_ptr(phq), _ptr(phk), _ptr(v), _ptr(out), _ptr(den), B, H,
                                      L, F, Dv, dt, eps, 1 if causal else 0, _ptr(workspace),
                                      wbytes, _stream(stream)), "slay_linear_attn_fwd")
    return workspace


def _state_ptrs(S, z, BH_shape, F, name):
    if S is None and z is None:
        return None, None
    _check(S, name + " S", torch.float32, BH_shape + (F, 64))
    _check(z, name + " z", torch.float32, BH_shape + (F,))
    return _ptr(S), _ptr(z)


def slay_attn_causal_fwd_state(q, k, v, out, den, R, m, seed, eps, S_in=None, z_in=None,
                               S_out=None, z_out=None, workspace=None, stream=None):
    """Causal forward from state (S_in, z_in) [B,H,F,64], [B,H,F] (None: zero), writing the
    final state into S_out, z_out if given; returns the workspace it used."""
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    _check(k, "k", q.dtype, (B, H, L, D))
    _check(v, "v", q.dtype, (B, H, L, Dv))
    _check(out, "out", q.dtype, (B, H, L, Dv))
    if den is not None:
        _check(den, "den", torch.float32, (B, H, L))
    F = R * m
    si, zi = _state_ptrs(S_in, z_in, (B, H), F, "state in")
    so, zo = _state_ptrs(S_out, z_out, (B, H), F, "state out")
    dt = _dt(q)
    if workspace is None:
        workspace = alloc_workspace(OP_CAUSAL_FWD, dt, B, H, L, D, Dv, R, m, q.device)
    wbytes = workspace.numel() * workspace.element_size()
    _raise(lib().slay_attn_causal_fwd_state(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(den), si, zi,
                                            so, zo, B, H, L, D, Dv, dt, R, m, seed, eps,
                                            _ptr(workspace), wbytes, _stream(stream)),
           "slay_attn_causal_fwd_state")
    return workspace


def slay_causal_state(k, v, S_out, z_out, R, m, seed, eps, S_in=None, z_in=None, workspace=None,
                      stream=None):
    """S_out = S_in + sum phi(k) v^T, z_out = z_in + sum phi(k) over the tokens of k, v."""
    _check(k, "k")
    B, H, L, D = k.shape
    Dv = v.shape[-1]
    _check(v, "v", k.dtype, (B, H, L, Dv))
    F = R * m
    si, zi = _state_ptrs(S_in, z_in, (B, H), F, "state in")
    so, zo = _state_ptrs(S_out, z_out, (B, H), F, "state out")
    dt = _dt(k)
    if workspace is None:
        workspace = alloc_workspace(OP_CAUSAL_STATE, dt, B, H, L, D, Dv, R, m, k.device)
    wbytes = workspace.numel() * workspace.element_size()
    _raise(lib().slay_causal_state(_ptr(k), _ptr(v), si, zi, so, zo, B, H, L, D, Dv, dt, R, m,
                                   seed, eps, _ptr(workspace), wbytes, _stream(stream)),
           "slay_causal_state")
    return workspace


def slay_attn_causal_fwd_begin(k, v, S_out, z_out, R, m, seed, eps, workspace=None,
                               stream=None):
    """First call of the two-call forward: this piece's state S_out = sum phi(k) v^T,
    z_out = sum phi(k) [B,H,F,64], [B,H,F] fp32; the workspace it returns (or the one given)
    carries phi(k) and the segment sums to slay_attn_causal_fwd_finish."""
    _check(k, "k")
    B, H, L, D = k.shape
    Dv = v.shape[-1]
    _check(v, "v", k.dtype, (B, H, L, Dv))
    F = R * m
    so, zo = _state_ptrs(S_out, z_out, (B, H), F, "state out")
    dt = _dt(k)
    if workspace is None:
        workspace = alloc_workspace(OP_CAUSAL_FWD_SPLIT, dt, B, H, L, D, Dv, R, m, k.device)
    wbytes = workspace.numel() * workspace.element_size()
    _raise(lib().slay_attn_causal_fwd_begin(_ptr(k), _ptr(v), so, zo, B, H, L, D, Dv, dt, R, m,
                                            seed, eps, _ptr(workspace), wbytes, _stream(stream)),
           "slay_attn_causal_fwd_begin")
    return workspace


def slay_attn_causal_fwd_finish(q, k, v, out, den, R, m, seed, eps, workspace, S_in=None,
                                z_in=None, stream=None):
    """Second call of the two-call forward: out (and den) of the piece from the state
    (S_in, z_in) (None: zero), on the workspace of slay_attn_causal_fwd_begin for k, v."""
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    _check(k, "k", q.dtype, (B, H, L, D))
    _check(v, "v", q.dtype, (B, H, L, Dv))
    _check(out, "out", q.dtype, (B, H, L, Dv))
    if den is not None:
        _check(den, "den", torch.float32, (B, H, L))
    si, zi = _state_ptrs(S_in, z_in, (B, H), R * m, "state in")
    wbytes = workspace.numel() * workspace.element_size()
    _raise(lib().slay_attn_causal_fwd_finish(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(den),
                                             si, zi, B, H, L, D, Dv, _dt(q), R, m, seed, eps,
                                             _ptr(workspace), wbytes, _stream(stream)),
           "slay_attn_causal_fwd_finish")


def slay_state_prefix(S_all, z_all, rank, S_in, z_in, stream=None):
    """S_in = sum of S_all[r] for r < rank (S_all [N,B,H,F,64], z_all [N,B,H,F])."""
    _check(S_all, "S_all", torch.float32)
    N, B, H, F, Dv = S_all.shape
    _check(z_all, "z_all", torch.float32, (N, B, H, F))
    _check(S_in, "S_in", torch.float32, (B, H, F, Dv))
    _check(z_in, "z_in", torch.float32, (B, H, F))
    _raise(lib().slay_state_prefix(_ptr(S_all), _ptr(z_all), N, rank, _ptr(S_in), _ptr(z_in),
                                   B * H, F, Dv, _stream(stream)), "slay_state_prefix")


def slay_state_suffix(S_all, z_all, rank, S_out, z_out, stream=None):
    """S_out = sum of S_all[r] for r > rank (S_all [N,B,H,F,64], z_all [N,B,H,F])."""
    _check(S_all, "S_all", torch.float32)
    N, B, H, F, Dv = S_all.shape
    _check(z_all, "z_all", torch.float32, (N, B, H, F))
    _check(S_out, "S_out", torch.float32, (B, H, F, Dv))
    _check(z_out, "z_out", torch.float32, (B, H, F))
    _raise(lib().slay_state_suffix(_ptr(S_all), _ptr(z_all), N, rank, _ptr(S_out), _ptr(z_out),
                                   B * H, F, Dv, _stream(stream)), "slay_state_suffix")


def slay_attn_causal_bwd_state(q, k, v, out, den, dout, dq, dk, dv, R, m, seed, eps, S_in=None,
                               z_in=None, G_in=None, zg_in=None, workspace=None, stream=None):
    """Backward of one piece of a causal sequence: S_in, z_in [B,H,F,64], [B,H,F] sum
    phi(k)[v, 1] over the tokens before it, G_in, zg_in sum phi(q)[dn, delta] over the tokens
    after it (None: zero); returns the workspace it used."""
    return _bwd_piece(lib().slay_attn_causal_bwd_state, "slay_attn_causal_bwd_state", q, k, v,
                      out, den, dout, dq, dk, dv, R, m, seed, eps, S_in, z_in, G_in, zg_in,
                      workspace, stream)


def slay_attn_causal_bwd_finish(q, k, v, out, den, dout, dq, dk, dv, R, m, seed, eps, workspace,
                                S_in=None, z_in=None, G_in=None, zg_in=None, stream=None):
    """Second call of the two-call backward: the gradients of slay_attn_causal_bwd_state on
    the workspace of slay_attn_causal_bwd_begin for the same q, out, den, dout."""
    _bwd_piece(lib().slay_attn_causal_bwd_finish, "slay_attn_causal_bwd_finish", q, k, v, out,
               den, dout, dq, dk, dv, R, m, seed, eps, S_in, z_in, G_in, zg_in, workspace, stream)


def _bwd_piece(fn, name, q, k, v, out, den, dout, dq, dk, dv, R, m, seed, eps, S_in, z_in, G_in,
               zg_in, workspace, stream):
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = v.shape[-1]
    for t, name, dt_, shp in ((k, "k", q.dtype, (B, H, L, D)), (v, "v", q.dtype, (B, H, L, Dv)),
                              (out, "out", q.dtype, (B, H, L, Dv)),
                              (den, "den", torch.float32, (B, H, L)),
                              (dout, "dout", q.dtype, (B, H, L, Dv)),
                              (dq, "dq", torch.float32, (B, H, L, D)),
                              (dk, "dk", torch.float32, (B, H, L, D)),
                              (dv, "dv", torch.float32, (B, H, L, Dv))):
        _check(t, name, dt_, shp)
    F = R * m
    si, zi = _state_ptrs(S_in, z_in, (B, H), F, "state before")
    gi, zgi = _state_ptrs(G_in, zg_in, (B, H), F, "state after")
    dt = _dt(q)
    if workspace is None:
        workspace = alloc_workspace(OP_CAUSAL_BWD, dt, B, H, L, D, Dv, R, m, q.device)
    wbytes = workspace.numel() * workspace.element_size()
    _raise(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(den), _ptr(dout), _ptr(dq), _ptr(dk),
              _ptr(dv), si, zi, gi, zgi, B, H, L, D, Dv, dt, R, m, seed, eps, _ptr(workspace),
              wbytes, _stream(stream)), name)
    return workspace


def slay_causal_bwd_state(q, out, den, dout, G_out, zg_out, R, m, seed, eps, workspace=None,
                          stream=None):
    """G_out = sum phi(q) dn^T, zg_out = sum phi(q) delta over the tokens of a piece."""
    return _g_state(lib().slay_causal_bwd_state, "slay_causal_bwd_state", q, out, den, dout,
                    G_out, zg_out, R, m, seed, eps, workspace, stream)


def slay_attn_causal_bwd_begin(q, out, den, dout, G_out, zg_out, R, m, seed, eps, workspace=None,
                               stream=None):
    """First call of the two-call backward: as slay_causal_bwd_state; the workspace it returns
    (or the one given) carries phi(q) and the row statistics to slay_attn_causal_bwd_finish."""
    return _g_state(lib().slay_attn_causal_bwd_begin, "slay_attn_causal_bwd_begin", q, out, den,
                    dout, G_out, zg_out, R, m, seed, eps, workspace, stream)


def _g_state(fn, name, q, out, den, dout, G_out, zg_out, R, m, seed, eps, workspace, stream):
    _check(q, "q")
    B, H, L, D = q.shape
    Dv = out.shape[-1]
    _check(out, "out", q.dtype, (B, H, L, Dv))
    _check(den, "den", torch.float32, (B, H, L))
    _check(dout, "dout", q.dtype, (B, H, L, Dv))
    F = R * m
    go, zgo = _state_ptrs(G_out, zg_out, (B, H), F, "state out")
    dt = _dt(q)
    if workspace is None:
        workspace = alloc_workspace(OP_CAUSAL_BWD, dt, B, H, L, D, Dv, R, m, q.device)
    wbytes = workspace.numel() * workspace.element_size()
    _raise(fn(_ptr(q), _ptr(out), _ptr(den), _ptr(dout), go, zgo, B, H, L, D, Dv, dt, R, m, seed,
              eps, _ptr(workspace), wbytes, _stream(stream)), name)
    return workspace


def slay_feature_map_bwd(x, dphi, dx, R, m, seed, eps, stream=None):
    """dx[n, D] (fp32) = (d phi / d x)^T dphi for x[n, D] (f32 or bf16), dphi[n, R*m]."""
    _check(x, "x")
    _check(dphi, "dphi")
    D = x.shape[-1]
    n = x.numel() // D if D else 0
    if dphi.numel() != n * R * m or dphi.shape[-1] != R * m:
        raise ValueError("dphi must have %d rows of %d features" % (n, R * m))
    _check(dx, "dx", torch.float32, tuple(x.shape))
    _raise(lib().slay_feature_map_bwd(_ptr(x), _ptr(dphi), _ptr(dx), n, D, _dt(x), _dt(dphi), R,
                                      m, seed, eps, _stream(stream)), "slay_feature_map_bwd")


def slay_kernel_status(workspace=None, stream=None):
    """Raise SlayError if a kernel of the last call on `workspace` (None: the last
    no-alloc causal forward on this device) stopped on a wait that ran out; synchronizes
    the stream."""
    if workspace is not None:
        _check(workspace, "workspace")
    _raise(lib().slay_kernel_status(_ptr(workspace), _stream(stream)), "slay_kernel_status")


def slay_decode_step(q, k, v, S, z, out, R, m, seed, eps, stream=None):
    _check(q, "q")
    Bt, H, D = q.shape
    Dv = v.shape[-1]
    F = R * m
    _check(k, "k", q.dtype, (Bt, H, D))
    _check(v, "v", q.dtype, (Bt, H, Dv))
    _check(S, "S", torch.float32, (Bt, H, F, Dv))
    _check(z, "z", torch.float32, (Bt, H, F))
    _check(out, "out", q.dtype, (Bt, H, Dv))
    _raise(lib().slay_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(z), _ptr(out), Bt, H,
                                  D, Dv, _dt(q), R, m, seed, eps, _stream(stream)),
           "slay_decode_step")
