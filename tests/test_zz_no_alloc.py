"""The causal forward that allocates nothing, against the oracle and the regular forward.

slay_attn_causal_fwd_noalloc serves callers that cannot allocate device memory: a host that
reserves all of HBM for its own pool at start-up, a plugin that is handed tensors but no
workspace, or a latency-bound loop that must not pay for cudaMalloc's implicit
synchronisation.  It keeps its workspace and one sketch-parameter set in file-scope device
arrays instead.  These tests call it through the C ABI twice in a row -- with different
inputs and different parameter keys, so the second call must reload the parameter slot and
reuse the scratch the first call left behind -- and compare each result with the fp64
oracle and with slay_attn_causal_fwd, within the parity bars (relative L2 1e-5 in fp32,
1.5e-2 in bf16; ten times that per row).  The sizes cover the tensor-core form it runs for
bf16 with F <= 256 (with several 128-token tiles per segment) and the CUDA-core kernels it
runs otherwise (fp32, and bf16 with F = 512).  This file is named to be collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as O
from kernelized_linear_attention_unit_b200 import binding as bd
from kernelized_linear_attention_unit_b200 import workloads as W
from parity_check import check

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1.5e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _inputs(w, scaled=False):
    q, k, v = W.gen_qkv(w)
    if scaled:
        q = W.scale_rows(w, q, "q")
        k = W.scale_rows(w, k, "k")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(TDT[w.dtype])
    return (q, k, v), (dev(q), dev(k), dev(v))


def _noalloc_call(q, k, v, out, den, w):
    """Direct C-ABI call (no Python-side marshalling beyond pointers)."""
    B, H, L, D = q.shape
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    dt = bd.SLAY_F32 if w.dtype == "f32" else bd.SLAY_BF16
    return bd.lib().slay_attn_causal_fwd_noalloc(
        C.c_void_p(q.data_ptr()), C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
        C.c_void_p(out.data_ptr()), C.c_void_p(den.data_ptr()), B, H, L, D, v.shape[-1], dt,
        w.R, w.m, w.sketch_seed, float(np.float32(w.eps)), st)


CASES = [
    # tensor-core low-memory form: 74 sequences -> 2 segments of 3 tiles (ragged last tile)
    W.Workload("na_bf16_multitile", B=2, H=37, L=657, R=4, m=64, dtype="bf16", data_seed=41),
    # CUDA-core kernels: fp32, and bf16 with F = 512 (outside the low-memory form)
    W.Workload("na_f32", B=2, H=1, L=129, R=2, m=16, dtype="f32", data_seed=42, sketch_seed=77),
    W.Workload("na_bf16_f512", B=1, H=2, L=300, R=8, m=64, dtype="bf16", data_seed=43),
]


def test_noalloc_matches_oracle_and_causal_fwd_on_calls_in_a_row():
    for i, w in enumerate(CASES):
        (qh, kh, vh), (q, k, v) = _inputs(w, scaled=(i == 0))
        P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
        want, wden = O.attn_quadratic(qh, kh, vh, P, True)
        out_ref = torch.empty(v.shape, device="cuda", dtype=TDT[w.dtype])
        den_ref = torch.empty(v.shape[:-1], device="cuda", dtype=torch.float32)
        bd.slay_attn_causal_fwd(q, k, v, out_ref, den_ref, w.R, w.m, w.sketch_seed,
                                float(np.float32(w.eps)))
        for call in range(2):
            out = torch.full(v.shape, float("nan"), device="cuda", dtype=TDT[w.dtype])
            den = torch.full(v.shape[:-1], float("nan"), device="cuda", dtype=torch.float32)
            assert _noalloc_call(q, k, v, out, den, w) == bd.SLAY_OK
            bd.slay_kernel_status(None)
            torch.cuda.synchronize()
            name = "noalloc %s call %d" % (w.name, call + 1)
            got = out.double().cpu().numpy()
            gden = den.double().cpu().numpy()
            check(name + " out", got, want, TOL[w.dtype])
            check(name + " den", gden, wden, TOL[w.dtype], per_element=True)
            check(name + " out vs slay_attn_causal_fwd", got, out_ref.double().cpu().numpy(),
                  TOL[w.dtype])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = W.Workload("na_big", B=1, H=16, L=16384, R=4, m=64, dtype="f32", data_seed=43)
    need = bd.slay_workspace_bytes(bd.OP_CAUSAL_FWD, bd.SLAY_F32, w.B, w.H, w.L, 64, 64, w.R, w.m)
    assert need > (32 << 20)
    q = torch.zeros((1, 16, 16384, 64), device="cuda")
    out = torch.empty_like(q)
    den = torch.empty((1, 16, 16384), device="cuda")
    assert _noalloc_call(q, q, q, out, den, w) == bd.SLAY_ERR_UNSUPPORTED
