"""The failure path of the kernels' bounded waits, on the GPU, without a fault.

Every mbarrier wait in the tensor-core kernels is bounded in time; a wait that runs out
makes the kernel stop early, drain its own copies, free its tensor memory and set a status
word that slay_kernel_status reports as SLAY_ERR_TIMEOUT.  Here the library's test hook
makes one warp of the feature map withhold one release of a projection buffer (a barrier
that guards no copy or MMA in flight), and bounds that launch's waits at 1 ms: the issuing
thread's wait runs out.  The test checks the reported status, and that the next normal call
in the same process runs clean and matches the oracle.
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


def _feature_map(xt, w):
    phi = torch.zeros((xt.shape[0], w.F), device="cuda", dtype=torch.bfloat16)
    bd.slay_feature_map(xt, phi, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
    return phi


def _status():
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return bd.lib().slay_kernel_status(None, st)


def test_expired_wait_is_reported_and_the_next_call_is_clean():
    w = W.Workload("expiry", B=1, H=1, L=1000, R=4, m=64, dtype="bf16", data_seed=51)
    q, _, _ = W.gen_qkv(w)
    x = q.reshape(w.L, 64)
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda().to(torch.bfloat16)
    torch.cuda.synchronize()
    assert bd.lib().slay_debug_expire_wait(1) == bd.SLAY_OK
    _feature_map(xt, w)
    assert _status() == bd.SLAY_ERR_TIMEOUT
    assert b"bounded wait ran out" in bd.lib().slay_last_error()
    # the hook disarmed itself: the same call again runs clean and is correct
    phi = _feature_map(xt, w)
    assert _status() == bd.SLAY_OK
    P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
    check("phi after an expired wait", phi.float().cpu().numpy(), O.feature_map(x, P), 1.5e-2)
