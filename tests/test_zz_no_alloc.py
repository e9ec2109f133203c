"""The causal forward that allocates nothing, against the regular causal forward.

slay_attn_causal_fwd_noalloc serves callers that cannot allocate device memory (a host
that reserves all of HBM for its own pool, a plugin given tensors but no workspace, a
latency-bound loop that must not pay for cudaMalloc's synchronisation).  It keeps its
workspace and one sketch-parameter set in file-scope device arrays instead.  These tests
call it through the C ABI twice in a row -- with different inputs and different
parameter keys, so the second call must reload the parameter slot and reuse the scratch
the first call left behind -- and compare each result with slay_attn_causal_fwd within
the parity tolerances (1e-5 fp32, 1.5e-2 bf16).  This file is named to be collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from kernelized_linear_attention_unit_b200 import binding as bd
from kernelized_linear_attention_unit_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1.5e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).norm() / max(float(b.norm()), 1e-300))


def _inputs(w):
    q, k, v = W.gen_qkv(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(TDT[w.dtype])
    return dev(q), dev(k), dev(v)


def _noalloc_call(q, k, v, out, den, w):
    """Direct C-ABI call (no Python-side marshalling beyond pointers)."""
    B, H, L, D = q.shape
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    dt = bd.SLAY_F32 if w.dtype == "f32" else bd.SLAY_BF16
    return bd.lib().slay_attn_causal_fwd_noalloc(
        C.c_void_p(q.data_ptr()), C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
        C.c_void_p(out.data_ptr()), C.c_void_p(den.data_ptr()), B, H, L, D, v.shape[-1], dt,
        w.R, w.m, w.sketch_seed, float(np.float32(w.eps)), st)


def test_noalloc_matches_causal_fwd_on_two_calls_in_a_row():
    cases = [W.Workload("na_bf16", B=1, H=3, L=300, R=4, m=64, dtype="bf16", data_seed=41),
             W.Workload("na_f32", B=2, H=1, L=129, R=2, m=16, dtype="f32", data_seed=42,
                        sketch_seed=77)]
    for w in cases:
        q, k, v = _inputs(w)
        out_ref = torch.empty(v.shape, device="cuda", dtype=TDT[w.dtype])
        den_ref = torch.empty(v.shape[:-1], device="cuda", dtype=torch.float32)
        bd.slay_attn_causal_fwd(q, k, v, out_ref, den_ref, w.R, w.m, w.sketch_seed,
                                float(np.float32(w.eps)))
        out = torch.full(v.shape, float("nan"), device="cuda", dtype=TDT[w.dtype])
        den = torch.full(v.shape[:-1], float("nan"), device="cuda", dtype=torch.float32)
        assert _noalloc_call(q, k, v, out, den, w) == bd.SLAY_OK
        bd.slay_kernel_status(None)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert _rel(out.float(), out_ref.float()) <= TOL[w.dtype]
        assert _rel(den, den_ref) <= TOL[w.dtype]


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = W.Workload("na_big", B=1, H=16, L=16384, R=4, m=64, dtype="f32", data_seed=43)
    need = bd.slay_workspace_bytes(bd.OP_CAUSAL_FWD, bd.SLAY_F32, w.B, w.H, w.L, 64, 64, w.R, w.m)
    assert need > (32 << 20)
    q = torch.zeros((1, 16, 16384, 64), device="cuda")
    out = torch.empty_like(q)
    den = torch.empty((1, 16, 16384), device="cuda")
    assert _noalloc_call(q, q, q, out, den, w) == bd.SLAY_ERR_UNSUPPORTED
