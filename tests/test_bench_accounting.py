"""bench.py's algorithmic work per launch (CPU): the launches of one step add up to the
per-token-head counts of the method, also when the map is split into feature chunks.

Per token-head, D = Dv = 64, C = 64: causal forward 8DF + 4F Dv + (C+1)(F+Dv) flop,
bidirectional 8DF + 4F Dv flop; the feature map moves 2D + 2F bytes per row.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from kernelized_linear_attention_unit_b200 import workloads as W  # noqa: E402

D = DV = 64
C = 64


def causal_flop(F):
    return 8 * D * F + 4 * F * DV + (C + 1) * (F + DV)


def chunks(F):
    return 1 if F <= 256 else (F // 256 if F % 256 == 0 else F // 128)


@pytest.mark.parametrize("R,m", [(4, 64), (8, 64), (6, 64), (2, 64)])
def test_causal_launches_add_up(R, m):
    w = W.Workload("acct", B=2, H=3, L=1000, R=R, m=m, dtype="bf16")
    th = w.B * w.H * w.L
    n = chunks(w.F)
    per_step = n * (bench.kernel_work("tc_kphi_state", w, "causal")[0] +
                    bench.kernel_work("tc_qphi_out", w, "causal")[0])
    # the masked P.V term (C+1) Dv is counted once although every chunk computes it
    assert per_step == pytest.approx(th * causal_flop(w.F), rel=1e-12, abs=n)


@pytest.mark.parametrize("R,m", [(4, 64), (8, 64)])
def test_bidir_launches_add_up(R, m):
    w = W.Workload("acct", B=2, H=3, L=1000, R=R, m=m, dtype="bf16", causal=False)
    th = w.B * w.H * w.L
    n = chunks(w.F)
    per_step = n * (bench.kernel_work("tc_bidir_state", w, "bidir")[0] +
                    bench.kernel_work("tc_bidir_out", w, "bidir")[0])
    assert per_step == th * (8 * D * w.F + 4 * w.F * DV)


def test_feature_map_bytes():
    w = W.CAUSAL_16K
    th = w.B * w.H * w.L
    amount, unit, bound = bench.kernel_work("tc_feature_map", w, "feature_map")
    assert (unit, bound) == ("byte", "hbm")
    assert amount == 2 * th * (2 * D + 2 * w.F)


def test_backward_kernels_are_not_chunk_split():
    # the backward's tensor-core kernels take the whole map: their counts use the full F
    w = W.FWDBWD_8K
    th = w.B * w.H * w.L
    assert bench.kernel_work("tc_phi_bwd", w, "bwd")[0] == th * (2 * D + 2 * w.F + 4 * D)
    # the feature-map backward workload maps the q and the k rows in one launch
    assert bench.kernel_work("tc_phi_bwd", w, "feature_map_bwd")[0] == \
        2 * th * (2 * D + 2 * w.F + 4 * D)
    tiles = w.B * w.H * ((w.L + 127) // 128)
    # the running sums read phi(q), phi(k), v, dn once and write every tile's operands
    assert bench.kernel_work("tc_bwd_sums", w, "bwd")[0] == \
        th * (4 * w.F + 4 * DV) + tiles * 2 * w.F * (DV * 2 + 4)
    # the contraction by its flops: three products with the scanned sums (2 F Dv each) and
    # the masked intra-tile terms over the C + 1 keys of a causal chunk row on average
    amount, unit, bound = bench.kernel_work("tc_bwd_tile", w, "bwd")
    assert (unit, bound) == ("flop", "tensor")
    assert amount == th * (6 * w.F * DV + 65 * (3 * w.F + 2 * DV))


def test_backward_step_flops_are_the_per_token_head_count():
    # 16 D F + 10 F Dv + (C+1)(3F + 2Dv) per token-head = 960,128 at F = 512: 2.52e11 per step
    w = W.FWDBWD_8K
    per = 16 * D * w.F + 10 * w.F * DV + 65 * (3 * w.F + 2 * DV)
    assert per == 960128
    assert abs(per * w.B * w.H * w.L - 2.517e11) < 1e9


def test_profiled_traffic_needs_the_same_workload_and_sources(tmp_path, monkeypatch):
    # a committed ncu figure is reported only for the workload it was captured on and only
    # while the kernel's sources hash as they did then
    import hashlib
    csrc = tmp_path / "kernelized_linear_attention_unit_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_bytes(b"kernel source one")
    (tmp_path / "profiles").mkdir()
    h = hashlib.sha256(b"kernel source one").hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        "text\ntraffic: tc_x 1234 %s a.cu wl_big\ntraffic: tc_x 99 %s a.cu wl_small\n" % (h, h))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("tc_x", "wl_big") == 1234
    assert bench.profiled_traffic("tc_x", "wl_small") == 99
    assert bench.profiled_traffic("tc_x", "wl_other") is None
    assert bench.profiled_traffic("tc_y", "wl_big") is None
    (csrc / "a.cu").write_bytes(b"kernel source two")
    assert bench.profiled_traffic("tc_x", "wl_big") is None
