"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

The forward shards over independent (b, h) sequences, so the only cross-rank steps are the
barriers around the timed region and the max over ranks of the device time; each rank
draws its own batch.  These tests run those steps with real process groups (gloo over
127.0.0.1), no GPU.
"""
import datetime
import os
import socket
import sys
import tempfile

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from kernelized_linear_attention_unit_b200 import workloads as W  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        dist.barrier()
        slowest = bench.max_over_ranks(local_ms, world)
        value = bench.job_throughput(world, 16384, 4, slowest)
        wr = bench.rank_workload(W.CAUSAL_2K, rank)
        small = W.Workload(**{**wr.__dict__, "B": 1, "H": 2, "L": 16})
        q, _, _ = W.gen_qkv(small)
        np.save(os.path.join(outdir, "r%d.npy" % rank),
                np.array([slowest, value, wr.data_seed, float(q.astype(np.float64).sum())]))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    import torch.multiprocessing as mp
    outdir = tempfile.mkdtemp(prefix="slay_gloo_")
    mp.spawn(_rank_main, args=(2, _free_port(), outdir), nprocs=2, join=True)
    return [np.load(os.path.join(outdir, "r%d.npy" % r)) for r in range(2)]


def test_time_is_the_max_over_ranks(two_ranks):
    for r in two_ranks:
        assert r[0] == 15.0


def test_value_counts_every_rank_over_the_slowest_time(two_ranks):
    # 2 ranks x 16384 tokens x 4 steps in 15 ms
    for r in two_ranks:
        assert r[1] == pytest.approx(2 * 16384 * 4 / 0.015)


def test_each_rank_draws_its_own_batch(two_ranks):
    assert two_ranks[1][2] - two_ranks[0][2] == 1000
    assert two_ranks[0][3] != two_ranks[1][3]


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_throughput(1, 100, 10, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    class Args:
        gpus, steps, warmup = 2, 1, 1
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(Args(), W.TINY, "causal") == 0
    assert capsys.readouterr().out == ""


def _json_lines(out):
    import json
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_gpus_flag_starts_that_many_ranks():
    # `python bench.py --gpus 2` outside torchrun starts two ranks itself; without a GPU they
    # form a gloo group, and rank 0 reports both
    import subprocess
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--check-launch"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout
    assert lines[0]["n_gpus"] == 2
    assert sorted(lines[0]["ranks"]) == [0, 1]
    assert lines[0]["max_over_ranks"] == 1.0


def test_gpus_flag_must_match_the_launcher(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2", "--check-launch"])


class _OracleOps:
    """The sequence-parallel steps computed by the fp64 oracle on CPU tensors (a stand-in
    for the library on ranks without a GPU; the orchestration under test is the package's
    own).  begin's handle records the piece it was made for, and finish checks it was
    handed that handle for the same k, v (the library's workspace contract)."""

    def __init__(self, P):
        self.P = P
        self.begins = 0

    def begin(self, k, v, S_out, z_out, handle=None):
        self.state(k, v, S_out, z_out)
        self.begins += 1
        h = handle if handle is not None else {}
        h.update(k=k, v=v, n=self.begins)
        return h

    def finish(self, q, k, v, out, den, S_in, z_in, handle):
        import oracle as O
        assert handle["k"] is k and handle["v"] is v and handle["n"] == self.begins
        o, d, _, _ = O.attn_causal_state(q.numpy(), k.numpy(), v.numpy(), self.P,
                                         S_in.double().numpy(), z_in.double().numpy())
        out.copy_(torch_from(o))
        den.copy_(torch_from(d))

    def state(self, k, v, S_out, z_out):
        import oracle as O
        _, _, S, z = O.attn_causal_state(k.numpy(), k.numpy(), v.numpy(), self.P)
        S_out.copy_(torch_from(S))
        z_out.copy_(torch_from(z))

    def prefix(self, S_all, z_all, rank, S_in, z_in):
        S_in.copy_(S_all[:rank].sum(0) if rank else torch_zeros_like(S_in))
        z_in.copy_(z_all[:rank].sum(0) if rank else torch_zeros_like(z_in))

    def bwd_begin(self, q, out, den, dout, G_out, zg_out, handle=None):
        import oracle as O
        zeros = np.zeros(q.shape)
        _, _, _, G, zg = O.attn_causal_bwd_state(q.numpy(), zeros, zeros, out.numpy(), den.numpy(),
                                                 dout.numpy(), self.P)
        G_out.copy_(torch_from(G))
        zg_out.copy_(torch_from(zg))
        self.bwd_begins = getattr(self, "bwd_begins", 0) + 1
        h = handle if handle is not None else {}
        h.update(q=q, dout=dout, n=self.bwd_begins)
        return h

    def suffix(self, G_all, zg_all, rank, G_in, zg_in):
        G_in.copy_(G_all[rank + 1:].sum(0) if rank + 1 < G_all.shape[0] else torch_zeros_like(G_in))
        zg_in.copy_(zg_all[rank + 1:].sum(0) if rank + 1 < zg_all.shape[0] else torch_zeros_like(zg_in))

    def bwd_finish(self, q, k, v, out, den, dout, dq, dk, dv, S_in, z_in, G_in, zg_in, handle):
        import oracle as O
        assert handle["q"] is q and handle["dout"] is dout and handle["n"] == self.bwd_begins
        st = [x.double().numpy() for x in (S_in, z_in, G_in, zg_in)]
        a, b, c, _, _ = O.attn_causal_bwd_state(q.numpy(), k.numpy(), v.numpy(), out.numpy(),
                                                den.numpy(), dout.numpy(), self.P, *st)
        dq.copy_(torch_from(a))
        dk.copy_(torch_from(b))
        dv.copy_(torch_from(c))


def torch_from(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).float()


def torch_zeros_like(t):
    import torch
    return torch.zeros_like(t)


def test_seqpar_scratch_reuses_the_handle_only_for_the_same_piece():
    # without a process group (one rank): begin's workspace handle is kept in the scratch and
    # handed back to begin on the next step of the same sizes; a new piece length or dtype
    # starts a new one (the library's workspace size depends on both)
    import torch
    from kernelized_linear_attention_unit_b200 import seqpar

    class CountingOps:
        def __init__(self):
            self.given, self.made = [], 0

        def begin(self, k, v, S_out, z_out, handle=None):
            self.given.append(handle)
            if handle is None:
                self.made += 1
                handle = {"id": self.made}
            S_out.zero_()
            z_out.zero_()
            return handle

        def prefix(self, S_all, z_all, rank, S_in, z_in):
            S_in.zero_()
            z_in.zero_()

        def finish(self, q, k, v, out, den, S_in, z_in, handle):
            out.zero_()

    ops, sc = CountingOps(), {}

    def step(L, dtype=torch.float64):
        q, k, v = (torch.zeros((1, 2, L, 64), dtype=dtype) for _ in range(3))
        seqpar.causal_fwd_seqpar(q, k, v, torch.empty_like(v), torch.empty((1, 2, L)), 16,
                                 ops, scratch=sc)

    step(40)
    step(40)
    step(41)
    step(41, torch.float32)
    assert [h["id"] if h else None for h in ops.given] == [None, 1, None, None]
    assert ops.made == 3


def _seqpar_rank(rank, world, port, outdir):
    import torch
    import torch.distributed as dist
    import oracle as O
    from kernelized_linear_attention_unit_b200 import seqpar
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = W.Workload("sp", B=1, H=2, L=90, R=2, m=8, dtype="f32", data_seed=61)
        q, k, v = W.gen_qkv(w)
        P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
        a, b = rank * w.L // world, (rank + 1) * w.L // world
        piece = [torch.from_numpy(np.ascontiguousarray(x[:, :, a:b])).double() for x in (q, k, v)]
        out = torch.empty((1, 2, b - a, 64))
        den = torch.empty((1, 2, b - a))
        ops, scratch = _OracleOps(P), {}
        seqpar.causal_fwd_seqpar(*piece, out, den, w.F, ops, scratch=scratch)
        first, handle = out.clone(), scratch["handle"]
        # a second step on the same scratch reuses begin's handle
        seqpar.causal_fwd_seqpar(*piece, out, den, w.F, ops, scratch=scratch)
        assert scratch["handle"] is handle and ops.begins == 2
        assert torch.equal(first, out)
        np.save(os.path.join(outdir, "sp%d.npy" % rank), out.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_orchestration(world):
    # gloo ranks each hold a contiguous piece of a sequence; the package's orchestration (piece
    # state, all-gather, prefix over earlier ranks, forward from it) reproduces the whole
    # sequence (with three ranks the middle one starts from a non-zero, non-total prefix)
    import torch.multiprocessing as mp
    import oracle as O
    outdir = tempfile.mkdtemp(prefix="slay_sp_")
    mp.spawn(_seqpar_rank, args=(world, _free_port(), outdir), nprocs=world, join=True)
    got = np.concatenate([np.load(os.path.join(outdir, "sp%d.npy" % r)) for r in range(world)],
                         axis=2)
    w = W.Workload("sp", B=1, H=2, L=90, R=2, m=8, dtype="f32", data_seed=61)
    q, k, v = W.gen_qkv(w)
    P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
    want, _ = O.attn_quadratic(q, k, v, P, True)
    assert np.abs(got - want).max() < 1e-5 * np.abs(want).max()


def _seqpar_bwd_rank(rank, world, port, outdir):
    import torch
    import torch.distributed as dist
    import oracle as O
    from kernelized_linear_attention_unit_b200 import seqpar
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = W.Workload("spb", B=1, H=2, L=60, R=2, m=8, dtype="f32", data_seed=62)
        q, k, v = W.gen_qkv(w)
        g = W.gen_dout(w)
        P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
        a, b = rank * w.L // world, (rank + 1) * w.L // world
        sl = (slice(None), slice(None), slice(a, b))
        piece = [torch.from_numpy(np.ascontiguousarray(x[sl])).double() for x in (q, k, v, g)]
        ops = _OracleOps(P)
        out = torch.empty((1, 2, b - a, 64), dtype=torch.float64)
        den = torch.empty((1, 2, b - a), dtype=torch.float64)
        scratch = {}
        seqpar.causal_fwd_seqpar(piece[0], piece[1], piece[2], out, den, w.F, ops, scratch=scratch)
        res = []
        for reuse in (False, True):   # the forward's state recomputed, or passed in
            dq, dk, dv = (torch.empty((1, 2, b - a, 64), dtype=torch.float64) for _ in range(3))
            seqpar.causal_bwd_seqpar(piece[0], piece[1], piece[2], out, den, piece[3], dq, dk, dv,
                                     w.F, ops, fwd_state=(scratch["S_in"], scratch["z_in"])
                                     if reuse else None)
            res.append(np.stack([dq.numpy(), dk.numpy(), dv.numpy()]))
        np.save(os.path.join(outdir, "spb%d.npy" % rank), np.stack(res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_backward_orchestration(world):
    # gloo ranks each hold a piece of a sequence: forward as above, then each rank's piece
    # state and phi(q)[dn, delta] sum all-gathered, prefix and suffix over ranks, and the
    # piece's backward; together they are the whole sequence's gradients (with three ranks
    # the middle one has both a non-zero prefix and a non-zero suffix)
    import torch.multiprocessing as mp
    import oracle as O
    outdir = tempfile.mkdtemp(prefix="slay_spb_")
    mp.spawn(_seqpar_bwd_rank, args=(world, _free_port(), outdir), nprocs=world, join=True)
    got2 = np.concatenate([np.load(os.path.join(outdir, "spb%d.npy" % r)) for r in range(world)],
                          axis=4)
    np.testing.assert_array_equal(got2[0], got2[1])
    got = got2[0]
    w = W.Workload("spb", B=1, H=2, L=60, R=2, m=8, dtype="f32", data_seed=62)
    q, k, v = W.gen_qkv(w)
    g = W.gen_dout(w)
    P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
    want = O.attn_causal_bwd(q, k, v, g, P)
    for i in range(3):
        assert np.abs(got[i] - want[i]).max() < 1e-4 * np.abs(want[i]).max(), i
