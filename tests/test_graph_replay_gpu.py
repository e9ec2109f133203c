"""The library's calls inside a CUDA graph: captured once after slay_prepare (the only
synchronous work, the sketch-parameter upload, happens there), then replayed on new inputs
copied into the same buffers.  The replay must give exactly what the same calls give when
launched one by one (same kernels, same inputs, same order), for the bf16 tensor-core causal
forward (two launches, the second a programmatic dependent of the first) and backward."""
import numpy as np
import pytest
import torch

from kernelized_linear_attention_unit_b200 import binding as bd
from kernelized_linear_attention_unit_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def test_forward_and_backward_replay_from_a_cuda_graph():
    w = W.Workload("graph", B=2, H=3, L=700, R=4, m=64, dtype="bf16", data_seed=27)
    eps = float(np.float32(w.eps))
    B, H, L, D = w.B, w.H, w.L, w.D
    bd.slay_prepare(D, w.R, w.m, w.sketch_seed, eps)
    q, k, v, g = (torch.empty((B, H, L, 64), device="cuda", dtype=torch.bfloat16) for _ in range(4))
    out = torch.empty_like(v)
    den = torch.empty((B, H, L), device="cuda")
    dq, dk, dv = (torch.empty((B, H, L, 64), device="cuda") for _ in range(3))
    wsf = bd.alloc_workspace(bd.OP_CAUSAL_FWD, torch.bfloat16, B, H, L, D, 64, w.R, w.m)
    wsb = bd.alloc_workspace(bd.OP_CAUSAL_BWD, torch.bfloat16, B, H, L, D, 64, w.R, w.m)

    def load(seed):
        ww = W.Workload("graph", B=B, H=H, L=L, R=w.R, m=w.m, dtype="bf16", data_seed=seed)
        a, b, c = W.gen_qkv(ww)
        for t, x in zip((q, k, v, g), (a, b, c, W.gen_dout(ww))):
            t.copy_(_dev(x))

    def calls():
        bd.slay_attn_causal_fwd(q, k, v, out, den, w.R, w.m, w.sketch_seed, eps, wsf)
        bd.slay_attn_causal_bwd(q, k, v, out, den, g, dq, dk, dv, w.R, w.m, w.sketch_seed, eps,
                                wsb)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        load(27)
        calls()                     # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        calls()
    load(28)
    graph.replay()
    torch.cuda.synchronize()
    assert bd.lib().slay_kernel_status(bd._ptr(wsb), bd._stream()) == bd.SLAY_OK
    got = [t.clone() for t in (out, den, dq, dk, dv)]
    load(28)
    calls()
    torch.cuda.synchronize()
    for a, b in zip(got, (out, den, dq, dk, dv)):
        assert torch.equal(a, b)
    assert torch.isfinite(got[2]).all() and got[2].abs().sum() > 0
