"""slay_path against the kernels a call actually launches: each call runs with the library's
launch trace on, and the trace names say which steps ran on tensor cores."""
import pytest
import torch

from kernelized_linear_attention_unit_b200 import binding as bd

pytestmark = pytest.mark.gpu

SEED, EPS = 5, 1e-3
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}
FWD_OPS = ("causal", "bidir", "state", "split")


def _rand(shape, dt):
    g = torch.Generator(device="cuda").manual_seed(1)
    return torch.randn(shape, generator=g, device="cuda").to(TDT[dt])


def _run(op, dt, B, H, L, R, m):
    F = R * m
    q, k, v = (_rand((B, H, L, 64), dt) for _ in range(3))
    out = torch.empty_like(v)
    den = torch.empty((B, H, L), device="cuda")
    S = torch.empty((B, H, F, 64), device="cuda")
    z = torch.empty((B, H, F), device="cuda")
    if op == "causal":
        ws = bd.slay_attn_causal_fwd(q, k, v, out, den, R, m, SEED, EPS)
    elif op == "bidir":
        ws = bd.slay_attn_bidir_fwd(q, k, v, out, den, R, m, SEED, EPS)
    elif op == "state":
        ws = bd.slay_causal_state(k, v, S, z, R, m, SEED, EPS)
    elif op == "split":
        ws = bd.slay_attn_causal_fwd_begin(k, v, S, z, R, m, SEED, EPS)
        bd.slay_attn_causal_fwd_finish(q, k, v, out, den, R, m, SEED, EPS, ws)
    elif op in ("causal_bwd", "bidir_bwd"):
        fwd = bd.slay_attn_causal_fwd if op == "causal_bwd" else bd.slay_attn_bidir_fwd
        fwd(q, k, v, out, den, R, m, SEED, EPS)
        torch.cuda.synchronize()
        bd.slay_trace_read()   # the forward's launches are not the backward's
        dq, dk, dv = (torch.empty((B, H, L, 64), device="cuda") for _ in range(3))
        bwd = bd.slay_attn_causal_bwd if op == "causal_bwd" else bd.slay_attn_bidir_bwd
        ws = bwd(q, k, v, out, den, _rand((B, H, L, 64), dt), dq, dk, dv, R, m, SEED, EPS)
    elif op == "fmap":
        x = q.reshape(-1, 64)
        bd.slay_feature_map(x, torch.empty((x.shape[0], F), device="cuda", dtype=TDT[dt]), R, m,
                            SEED, EPS)
        ws = None
    elif op == "fmap_bwd":
        x = q.reshape(-1, 64)
        bd.slay_feature_map_bwd(x, _rand((x.shape[0], F), dt),
                                torch.empty((x.shape[0], 64), device="cuda"), R, m, SEED, EPS)
        ws = None
    if ws is not None:
        bd.slay_kernel_status(ws)
    torch.cuda.synchronize()


OPS = {"causal": bd.OP_CAUSAL_FWD, "bidir": bd.OP_BIDIR_FWD, "state": bd.OP_CAUSAL_STATE,
       "split": bd.OP_CAUSAL_FWD_SPLIT, "causal_bwd": bd.OP_CAUSAL_BWD,
       "bidir_bwd": bd.OP_BIDIR_BWD, "fmap": bd.OP_FEATURE_MAP, "fmap_bwd": bd.OP_FEATURE_MAP_BWD}


# trace names of the fused tensor-core forward kernels (projection and phi inside them)
FWD_TC = {"tc_kphi_state", "tc_qphi_out", "tc_bidir_state", "tc_bidir_out", "tc_state_sums",
          "tc_causal_state", "tc_causal_out", "tc_state_total"}


def _observed(op, names):
    if op in FWD_OPS and any(n in FWD_TC for n in names):
        return bd.PATH_TC_FEATURE_MAP | bd.PATH_TC_CONTRACTION
    mask = 0
    if "tc_feature_map" in names:
        mask |= bd.PATH_TC_FEATURE_MAP
    if "tc_bwd_tile" in names:
        mask |= bd.PATH_TC_CONTRACTION
    if "tc_phi_bwd" in names:
        mask |= bd.PATH_TC_PHI_BWD
    return mask


@pytest.mark.parametrize("op,dt,R,m", [
    ("causal", "bf16", 4, 64), ("causal", "f32", 4, 64), ("causal", "bf16", 4, 32),
    ("causal", "bf16", 8, 64), ("bidir", "bf16", 4, 64), ("bidir", "bf16", 2, 48),
    ("state", "bf16", 4, 64), ("state", "bf16", 2, 16), ("split", "bf16", 4, 64),
    ("split", "f32", 2, 16), ("causal_bwd", "bf16", 2, 64), ("causal_bwd", "bf16", 4, 32),
    ("causal_bwd", "bf16", 3, 64), ("causal_bwd", "f32", 2, 64), ("bidir_bwd", "bf16", 4, 64),
    ("bidir_bwd", "bf16", 3, 64), ("fmap", "bf16", 4, 32), ("fmap", "f32", 4, 32),
    ("fmap", "bf16", 3, 64), ("fmap_bwd", "bf16", 4, 32), ("fmap_bwd", "f32", 4, 32)])
def test_path_query_matches_launched_kernels(op, dt, R, m):
    B, H, L = 1, 2, 300
    want = bd.slay_path(OPS[op], TDT[dt], B, H, L, 64, 64, R, m)
    bd.slay_trace_read()
    bd.slay_trace_enable(True)
    try:
        _run(op, dt, B, H, L, R, m)
        names = [n for n, _ in bd.slay_trace_read()]
    finally:
        bd.slay_trace_enable(False)
    assert names, "no launches traced"
    assert _observed(op, names) == want, (want, sorted(set(names)))
