#!/usr/bin/env python
"""Benchmark of the SLAY causal forward (spherical Yat-kernel linear attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload causal_16k|causal_2k|bidir_vision|fwd_8k|bwd_8k|bidir_bwd|decode|
                                feature_map|feature_map_bwd|matched_budget|seqpar_16k|
                                seqpar_bwd_8k]

seqpar_16k splits the headline sequence over the N ranks (strong scaling, one all-gather of
the pieces' states per step), seqpar_bwd_8k the fwd/bwd sequence for its backward (one
all-gather per step, of the pieces' phi(q)[dn, delta] sums; the prefix state comes from the
untimed forward); every other workload gives each rank its own batch (weak).  For those two
the dominant kernel's work is counted over the rank's piece.

With --gpus N > 1 outside torchrun, bench.py starts the N ranks itself (torch.distributed.run
on 127.0.0.1); under torchrun, --gpus must equal WORLD_SIZE.

One step = one pass of the whole forward path (feature map of q and k, causal contraction,
normalisation) over one batch of synthetic inputs already resident in HBM.  Default
workload: B=1, H=16, L=16384, D=Dv=64, R=4 nodes, m=64 features per node (F=256), bf16
inputs, fp32 state.  Multi-GPU (torchrun): every rank runs its own batch (weak scaling,
no collective on the data path); the timed region is bracketed by barriers and the
reported time is the max over ranks.

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle (the only
reference this method has) on the host cores instead.
"""
import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kernelized_linear_attention_unit_b200 import workloads as W  # noqa: E402

METRIC = "SLAY causal fwd tokens/s at L=16k on 1 B200; % of tensor-core/HBM roofline"

WORKLOADS = {
    "causal_16k": (W.CAUSAL_16K, "causal"),
    "causal_2k": (W.CAUSAL_2K, "causal"),
    "bidir_vision": (W.BIDIR_VISION, "bidir"),
    "fwd_8k": (W.FWDBWD_8K, "causal"),
    "bwd_8k": (W.FWDBWD_8K, "bwd"),
    "bidir_bwd": (W.BIDIR_VISION, "bidir_bwd"),
    "feature_map_bwd": (W.CAUSAL_16K, "feature_map_bwd"),
    "matched_budget": (W.CAUSAL_16K, "matched_budget"),
    "seqpar_16k": (W.CAUSAL_16K, "seqpar"),
    "seqpar_bwd_8k": (W.FWDBWD_8K, "seqpar_bwd"),
    "decode": (W.DECODE, "decode"),
    "feature_map": (W.CAUSAL_16K, "feature_map"),
}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
L2_FLUSH_BYTES = 256 << 20
C_CHUNK = 64


# ----------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def alu_peak_tflops(sm_mhz):
    # FP32 FFMA: 148 SMs x 128 lanes x 2 flop per clock
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` in `workload` from the committed ncu summaries under
    profiles/ (lines "traffic: <kernel> <bytes> <sha256[:16] of its sources> <sources>
    <workload>"), or None when no capture of that kernel in that workload exists or the
    kernel's sources changed since it was taken."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "kernelized_linear_attention_unit_b200", "csrc")
    for fn in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(fn):
            parts = line.split()
            if len(parts) != 6 or parts[0] != "traffic:" or parts[1] != kernel or parts[5] != workload:
                continue
            h = hashlib.sha256()
            try:
                for src in parts[4].split("+"):
                    with open(os.path.join(csrc, src), "rb") as f:
                        h.update(f.read())
            except OSError:
                return None
            return int(parts[2]) if h.hexdigest()[:16] == parts[3] else None
    return None


def kernel_work(name, w, op):
    """Algorithmic work of one launch of kernel `name`: (amount, unit, bound).

    Per-unit figures (token-head = one row of one (b, h) slice; D = Dv = 64):
      feature map     bytes: x read (2 B/elem) + phi written in its own dtype, per row
      causal fwd      flop: 8DF + 4F Dv + (C+1)(F+Dv) per token-head, C = 64
      bidir fwd       flop: 8DF + 4F Dv per token-head
    """
    D, Dv, F = w.D, w.Dv, w.F
    th = w.B * w.H * w.L                    # token-heads in the batch
    # The tensor-core kernels take at most 256 features per launch: a wider map runs as
    # nch feature chunks (256 each, or 128 when F is not a multiple of 256), one launch of
    # each kernel per chunk, whose sums meet before the division.  A launch gets its
    # chunk's share; the masked P.V term (C+1) Dv, repeated per chunk, counts once.
    nch = 1 if F <= 256 else (F // 256 if F % 256 == 0 else F // 128)
    if name in ("tc_causal_out", "tc_qphi_out", "tc_causal_state", "tc_kphi_state",
                "tc_bidir_out", "tc_bidir_state"):
        F = F // nch
    if name in ("tc_causal_out", "tc_qphi_out"):
        return (th * (4 * D * F + 4 * F * Dv + (C_CHUNK + 1) * F) +
                th * (C_CHUNK + 1) * Dv // nch +
                (th * 4 * D * F if name == "tc_causal_out" else 0)), "flop", "tensor"
    if name in ("tc_causal_state", "tc_state_sums"):
        return th * (4 * D * F + 2 * F * Dv), "flop", "tensor"
    # stored-phi(k) form: the state kernel maps k (its own segment sums are not algorithmic
    # work), the output kernel does the rest of the causal forward
    if name == "tc_kphi_state":
        return th * (4 * D * F), "flop", "tensor"
    if name in ("tc_bidir_out",):
        return th * (4 * D * F + 2 * F * Dv), "flop", "tensor"
    if name in ("tc_bidir_state",):
        return th * (4 * D * F + 2 * F * Dv), "flop", "tensor"
    # the feature-map workload maps q and k rows (2 th rows, bf16 -> bf16) in one launch;
    # the CUDA-core attention paths map q and k separately (th rows each; bf16 features in
    # bf16 mode through the tensor-core map, fp32 features in fp32 mode)
    if name == "tc_feature_map":
        rows = 2 * th if op == "feature_map" else th
        return rows * (D * 2 + F * 2), "byte", "hbm"
    if name == "simt_feature_map":
        if op == "feature_map":
            return 2 * th * (D * 2 + F * 2), "byte", "hbm"
        return th * (D * 2 + F * 4), "byte", "hbm"
    if name == "simt_chunk_state":
        return th * 2 * F * (Dv + 1), "flop", "alu"
    if name == "simt_chunk_out":
        if op == "bidir":
            return th * 2 * F * (Dv + 1), "flop", "alu"
        return th * ((C_CHUNK + 1) * (F + Dv + 1) + 2 * F * (Dv + 1)), "flop", "alu"
    # the tensor-core backward's running sums: phi(q), phi(k) (bf16) and v, dn read once; the
    # causal form writes every tile's operands (bf16 [F][64] and fp32 z, for S and for G), the
    # bidirectional form the whole-sequence sums only
    if name == "tc_bwd_sums":
        tiles = w.B * w.H * ((w.L + 127) // 128)
        rd = th * (2 * F * 2 + 2 * Dv * 2)
        wr = 2 * (w.B * w.H if op == "bidir_bwd" else tiles) * F * (Dv * 2 + 4)
        return rd + wr, "byte", "hbm"
    if name == "simt_scan":
        nc = (w.L + C_CHUNK - 1) // C_CHUNK
        return w.B * w.H * nc * F * (Dv + 1) * 4 * 2, "byte", "hbm"
    # backward (CUDA cores): of the whole-backward count 16DF + 10F Dv + (C+1)(3F + 2Dv) per
    # token-head, the phi backward takes 8DF per row (projections of x^ and their transpose,
    # q and k launched separately), the two chunk-state launches 2F(Dv+1) each, the chunk
    # kernel the rest; the row statistics read out, g, den and write [dn, delta] (bytes)
    if name == "simt_phi_bwd":
        return th * 8 * D * F, "flop", "alu"
    # the tensor-core chunk contraction of the backward, by its algorithmic flops per
    # token-head: the three products with the scanned sums (dphi(q) = S dn, dphi(k) = G v,
    # dv = G^T phi(k): 2 F Dv each) and the masked intra-tile terms (scores and c_ij, the
    # dphi(q), dphi(k) and dv contractions over the C+1 keys of a causal chunk row on average)
    if name == "tc_bwd_tile":
        return th * (6 * F * Dv + (C_CHUNK + 1) * (3 * F + 2 * Dv)), "flop", "tensor"
    # the tensor-core phi backward is bound by its reads: x (bf16), dphi (bf16), dx (fp32);
    # the feature-map backward workload maps q and k rows (2 th rows) in one launch each
    if name == "tc_phi_bwd":
        rows = 2 * th if op == "feature_map_bwd" else th
        return rows * (2 * D + 2 * F + 4 * D), "byte", "hbm"
    if name == "simt_bwd_chunk":
        if op == "bidir_bwd":   # S [dn; delta], G [v; 1], G^T phi(k): no masked term
            return th * (2 * F * (Dv + 1) * 2 + 2 * F * Dv), "flop", "alu"
        return th * (6 * F * Dv + (C_CHUNK + 1) * (3 * F + 2 * Dv)), "flop", "alu"
    if name == "simt_bwd_rowstats":
        return th * (2 * Dv * 2 + 4 + (Dv + 1) * 4), "byte", "hbm"
    if name == "simt_decode":
        per = F * Dv * 4 * 2 + F * 4 * 2 + (2 * D + 2 * Dv) * 2
        return w.B * w.H * per, "byte", "hbm"
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU is loaded."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="slay_clk_", suffix=".csv")
        os.close(fd)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append((float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags)
                          if f.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ CPU oracle leg

def oracle_sample(w, op, max_heads):
    """Time the fp64 oracle's O(L) form on `h` full-length (b, h) slices.

    Returns (seconds, token-equivalents processed, threads, description)."""
    import oracle as O
    P = O.sketch_params(w.D, w.R, w.m, w.sketch_seed, float(np.float32(w.eps)))
    threads = O.num_threads()
    if op == "decode":
        n = min(w.B * w.H, max(64, 16 * threads))
        q, k, v, S, z = W.gen_decode(w, Bt=1, H=n)
        t0 = time.perf_counter()
        O.decode_step(q, k, v, S, z, P)
        dt = time.perf_counter() - t0
        return dt, n, threads, "%d of %d (b,h) decode states" % (n, w.B * w.H)
    h = max(1, min(w.H, max_heads))
    q, k, v = W.gen_qkv(w, B=1, H=h)
    form = "O(L) fp64 form"
    tokens = h / w.H * w.L          # token-equivalents (a token carries H heads)
    if op in ("bwd", "seqpar_bwd"):
        # the causal backward has no O(L) oracle form: its per-row form on a seeded sample of
        # 32 rows of each head (each row sums over all later queries and earlier keys)
        g = W.gen_dout(w, B=1, H=h)
        rows = np.sort(np.random.default_rng(11).choice(w.L, 32, replace=False))
        t0 = time.perf_counter()
        O.attn_causal_bwd_rows(q, k, v, g, P, rows)
        dt = time.perf_counter() - t0
        tokens = h / w.H * len(rows)
        form = "per-row fp64 backward at 32 rows"
    else:
        t0 = time.perf_counter()
        if op == "feature_map":
            O.feature_map(q, P)
            O.feature_map(k, P)
        elif op == "feature_map_bwd":
            gq = W.gen_dphi(w, w.L * h)
            O.feature_map_bwd(q.reshape(-1, w.D), gq, P)
            O.feature_map_bwd(k.reshape(-1, w.D), gq, P)
            form = "fp64 feature-map backward"
        elif op == "bidir_bwd":
            O.attn_bidir_bwd(q, k, v, W.gen_dout(w, B=1, H=h), P)
            form = "quadratic fp64 backward"
        else:
            O.attn_recurrent(q, k, v, P, op != "bidir")
        dt = time.perf_counter() - t0
    return dt, tokens, threads, "%d of %d heads of one sequence at L=%d, %s" % (h, w.H, w.L, form)


def oracle_baseline(w, op, cores, target_s=10.0, max_reps=30):
    """The CPU baseline: the oracle sample of oracle_sample, repeated until about target_s
    seconds of work have run (at most max_reps times).  Returns (seconds, token-equivalents,
    threads, description)."""
    total_dt, total_u, reps = 0.0, 0.0, 0
    threads, desc = 1, ""
    while reps < max_reps and (reps == 0 or total_dt < target_s):
        dt, u, threads, desc = oracle_sample(w, op, max(1, min(w.H, cores)))
        total_dt += dt
        total_u += u
        reps += 1
    return total_dt, total_u, threads, "%s, %d repetition%s" % (desc, reps, "" if reps == 1 else "s")


def run_reference(args, w, op):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = os.cpu_count() or 1
    max_heads = max(1, min(w.H, cores))
    times, units = [], 0.0
    for i in range(args.warmup + args.steps):
        dt, u, threads, desc = oracle_sample(w, op, max_heads if i else 1)
        if i >= args.warmup:
            times.append(dt)
            units += u
    val = units / sum(times)
    unit = "tokens/s" if op != "decode" else "decode-steps/s"
    line = {"impl": "reference", "metric": metric_of(w, op, unit), "value": val, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, op),
            "cpu_baseline": {"value": val, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


OP_NAMES = {"causal": "causal fwd", "bidir": "bidirectional fwd", "bwd": "causal bwd",
            "bidir_bwd": "bidirectional bwd", "decode": "decode", "feature_map": "feature map",
            "feature_map_bwd": "feature-map bwd", "seqpar": "sequence-parallel causal fwd",
            "seqpar_bwd": "sequence-parallel causal bwd"}


def metric_of(w, op, unit):
    """The headline metric for the L=16k causal forward; a name of its own for every other
    workload bench.py can time."""
    if w.name == W.CAUSAL_16K.name and op == "causal":
        return METRIC
    return "SLAY %s %s on %s; %% of tensor-core/HBM roofline" % (OP_NAMES.get(op, op), unit,
                                                                 w.name)


def config_of(w, op):
    return {"workload": w.name if op in ("causal", "bidir", "decode") else "%s_%s" % (w.name, op),
            "B": w.B, "H": w.H, "L": w.L, "D": w.D, "Dv": w.Dv, "R": w.R, "m": w.m, "F": w.F,
            "op": op, "eps": w.eps, "sketch_seed": w.sketch_seed,
            "l2": "flushed between timed steps (256 MiB write outside the timed events)"}


# ----------------------------------------------------------------- GPU leg

def rank_workload(w, rank):
    """The batch rank `rank` times: same shapes, data seed offset by 1000 * rank (weak
    scaling, independent sequences per rank, no exchange)."""
    return W.Workload(**{**w.__dict__, "data_seed": w.data_seed + 1000 * rank})


def max_over_ranks(x, world, device="cpu"):
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_step, steps, max_total_ms):
    """Whole-job units per second: every rank processed units_per_step per step."""
    return world * units_per_step * steps / (max_total_ms / 1e3)


def run_ours(args, w, op):
    import torch
    import torch.distributed as dist
    from kernelized_linear_attention_unit_b200 import binding as bd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    eps = float(np.float32(w.eps))
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(tdt)

    def pinned(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    # inputs: each rank draws its own batch (data seed offset by rank); the sequence-parallel
    # workload shares one sequence
    wr = w if op in ("seqpar", "seqpar_bwd") else rank_workload(w, rank)
    # the sizes one launch of this rank works on (the sequence-parallel ops: its piece)
    w_launch = w
    if op == "decode":
        qn, kn, vn, Sn, zn = W.gen_decode(wr)
        q, k, v = to_dev(qn), to_dev(kn), to_dev(vn)
        S = torch.from_numpy(Sn).to(dev)
        z = torch.from_numpy(zn).to(dev)
        out = torch.empty(v.shape, device=dev, dtype=tdt)
        host_in = [pinned(x.cpu()) for x in (q, k, v)]
        dev_in = [q, k, v]

        def step():
            bd.slay_decode_step(q, k, v, S, z, out, w.R, w.m, w.sketch_seed, eps)
        units_per_step = w.B * w.H
        unit = "decode-steps/s"
    elif op == "feature_map":
        qn, kn, _ = W.gen_qkv(wr)
        x = to_dev(np.concatenate([qn.reshape(-1, w.D), kn.reshape(-1, w.D)]))
        out = torch.empty((x.shape[0], w.F), device=dev, dtype=tdt)
        host_in, dev_in = [pinned(x.cpu())], [x]

        def step():
            bd.slay_feature_map(x, out, w.R, w.m, w.sketch_seed, eps)
        units_per_step = w.B * w.L
        unit = "tokens/s"
    elif op == "seqpar":
        from kernelized_linear_attention_unit_b200 import seqpar
        # this rank's contiguous piece of the one long sequence (every rank draws the whole
        # sequence from the same seed and keeps its piece)
        qn, kn, vn = W.gen_qkv(w)
        a, b = rank * w.L // world, (rank + 1) * w.L // world
        q, k, v = (to_dev(np.ascontiguousarray(x[:, :, a:b])) for x in (qn, kn, vn))
        out = torch.empty(v.shape, device=dev, dtype=tdt)
        den = torch.empty(v.shape[:-1], device=dev, dtype=torch.float32)
        host_in, dev_in = [pinned(x.cpu()) for x in (q, k, v)], [q, k, v]
        ops = seqpar.LibraryOps(w.R, w.m, w.sketch_seed, eps)
        scratch = {}

        def step():
            seqpar.causal_fwd_seqpar(q, k, v, out, den, w.F, ops, scratch=scratch)
        units_per_step = w.B * (b - a)
        w_launch = dataclasses.replace(w, L=b - a)
        unit = "tokens/s"
    elif op == "seqpar_bwd":
        from kernelized_linear_attention_unit_b200 import seqpar
        # this rank's piece of one long sequence: its forward (once, untimed) gives out and
        # den; the timed step is the piece's backward with its two state exchanges
        qn, kn, vn = W.gen_qkv(w)
        gn = W.gen_dout(w)
        a, b = rank * w.L // world, (rank + 1) * w.L // world
        q, k, v, g = (to_dev(np.ascontiguousarray(x[:, :, a:b])) for x in (qn, kn, vn, gn))
        out = torch.empty(v.shape, device=dev, dtype=tdt)
        den = torch.empty(v.shape[:-1], device=dev, dtype=torch.float32)
        ops = seqpar.LibraryOps(w.R, w.m, w.sketch_seed, eps)
        scratch = {}
        seqpar.causal_fwd_seqpar(q, k, v, out, den, w.F, ops, scratch=scratch)
        dq = torch.empty(q.shape, device=dev, dtype=torch.float32)
        dk = torch.empty_like(dq)
        dv = torch.empty(v.shape, device=dev, dtype=torch.float32)
        host_in, dev_in = [pinned(x.cpu()) for x in (q, k, v, g)], [q, k, v, g]

        # the state this piece's forward started from is the forward's (a training step
        # has it); the backward adds the exchange of the later pieces' phi(q)[dn, delta] sums
        fwd_state = (scratch["S_in"], scratch["z_in"])

        def step():
            seqpar.causal_bwd_seqpar(q, k, v, out, den, g, dq, dk, dv, w.F, ops, scratch=scratch,
                                     fwd_state=fwd_state)
        units_per_step = w.B * (b - a)
        w_launch = dataclasses.replace(w, L=b - a)
        unit = "tokens/s"
    elif op == "feature_map_bwd":
        qn, kn, _ = W.gen_qkv(wr)
        x = to_dev(np.concatenate([qn.reshape(-1, w.D), kn.reshape(-1, w.D)]))
        gphi = to_dev(W.gen_dphi(wr, x.shape[0]))
        out = torch.empty((x.shape[0], w.D), device=dev, dtype=torch.float32)
        host_in, dev_in = [pinned(x.cpu()), pinned(gphi.cpu())], [x, gphi]

        def step():
            bd.slay_feature_map_bwd(x, gphi, out, w.R, w.m, w.sketch_seed, eps)
        units_per_step = w.B * w.L
        unit = "tokens/s"
    else:
        qn, kn, vn = W.gen_qkv(wr)
        q, k, v = to_dev(qn), to_dev(kn), to_dev(vn)
        out = torch.empty(v.shape, device=dev, dtype=tdt)
        den = torch.empty(v.shape[:-1], device=dev, dtype=torch.float32)
        host_in, dev_in = [pinned(x.cpu()) for x in (q, k, v)], [q, k, v]
        if op in ("bwd", "bidir_bwd"):
            causal = op == "bwd"
            g = to_dev(W.gen_dout(wr))
            opb = bd.OP_CAUSAL_BWD if causal else bd.OP_BIDIR_BWD
            opf = bd.OP_CAUSAL_FWD if causal else bd.OP_BIDIR_FWD
            ws = bd.alloc_workspace(opb, tdt, w.B, w.H, w.L, w.D, w.Dv, w.R, w.m, dev)
            wsf = bd.alloc_workspace(opf, tdt, w.B, w.H, w.L, w.D, w.Dv, w.R, w.m, dev)
            fwd = bd.slay_attn_causal_fwd if causal else bd.slay_attn_bidir_fwd
            bwd = bd.slay_attn_causal_bwd if causal else bd.slay_attn_bidir_bwd
            fwd(q, k, v, out, den, w.R, w.m, w.sketch_seed, eps, wsf)
            dq = torch.empty(q.shape, device=dev, dtype=torch.float32)
            dk = torch.empty_like(dq)
            dv = torch.empty(v.shape, device=dev, dtype=torch.float32)
            host_in.append(pinned(g.cpu()))
            dev_in.append(g)

            def step():
                bwd(q, k, v, out, den, g, dq, dk, dv, w.R, w.m, w.sketch_seed, eps, ws)
        else:
            opc = bd.OP_BIDIR_FWD if op == "bidir" else bd.OP_CAUSAL_FWD
            ws = bd.alloc_workspace(opc, tdt, w.B, w.H, w.L, w.D, w.Dv, w.R, w.m, dev)
            fn = bd.slay_attn_bidir_fwd if op == "bidir" else bd.slay_attn_causal_fwd

            def step():
                fn(q, k, v, out, den, w.R, w.m, w.sketch_seed, eps, ws)
        units_per_step = w.B * w.L
        unit = "tokens/s"
    result = dq if op in ("bwd", "bidir_bwd", "seqpar_bwd") else out
    host_out = torch.empty(result.shape, dtype=result.dtype, pin_memory=True)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    bd.slay_prepare(w.D, w.R, w.m, w.sketch_seed, eps)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-timed region: inputs resident in HBM, L2 flushed between steps.  Pass 1
    # gives `value` (the library's calls alone); pass 2 repeats the same steps with the
    # library's per-launch tracing on (CUDA events around each kernel on its stream), which
    # gives the per-kernel durations of the roofline.  Tracing is kept out of pass 1
    # because its events between launches cost about 10 us per step.
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)

    def timed_pass(traced):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        bd.slay_trace_enable(traced)
        bd.slay_trace_read()
        barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        bd.slay_trace_enable(False)
        return [s.elapsed_time(e) for s, e in zip(starts, ends)], bd.slay_trace_read()

    step_ms, _ = timed_pass(False)
    traced_ms, trace = timed_pass(True)
    clocks = clk.stop()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    value = job_throughput(world, units_per_step, args.steps, total_ms)

    # ---- end to end through the same public call: H2D of inputs, the call, D2H of result
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = host_out.numel() * host_out.element_size()
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e_starts[i].record(stream)
        for hsrc, dtgt in zip(host_in, dev_in):
            dtgt.copy_(hsrc, non_blocking=True)
        step()
        host_out.copy_(result, non_blocking=True)
        e_ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends)), world, dev)
    e2e = job_throughput(world, units_per_step, args.steps, e2e_ms)

    # ---- roofline of the dominant kernel (largest total device time in the timed region)
    peaks, peak_src = load_peaks()
    per = {}
    for name, ms in trace:
        per.setdefault(name, []).append(ms)
    roofline = None
    kernels = {n: {"launches": len(v), "total_ms": sum(v), "avg_us": 1e3 * sum(v) / len(v)}
               for n, v in per.items()}
    if per:
        dom = max(per, key=lambda n: sum(per[n]))
        avg_s = sum(per[dom]) / len(per[dom]) / 1e3
        wk = kernel_work(dom, w_launch, op)
        if wk is not None:
            amount, kind, bound = wk
            if bound == "hbm":
                achieved, peak, u = amount / avg_s / 1e9, peaks["hbm_gbs"], "GB/s"
            elif bound == "tensor":
                achieved, peak, u = amount / avg_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
            else:
                achieved = amount / avg_s / 1e12
                peak = alu_peak_tflops(peaks.get("sm_max_mhz", 1965.0))
                u = "TFLOP/s"
            roofline = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak,
                        "unit": u, "frac": achieved / peak,
                        "traffic": profiled_traffic(dom, config_of(w, op)["workload"]),
                        "peak_source": peak_src + (" (fp32 FFMA: 148 SMs x 128 x 2 x max clock)"
                                                   if bound == "alu" else ""),
                        "algorithmic_%s_per_launch" % kind: amount,
                        "avg_launch_us": avg_s * 1e6,
                        "timing": "CUDA events around each launch on its stream, in the "
                                  "second timed pass (%.4f ms per step with them)"
                                  % (sum(traced_ms) / args.steps)}

    # the backward workloads also by the whole step's algorithmic flops (per token-head, D =
    # Dv = 64, C = 64): causal 16 D F + 10 F Dv + (C+1)(3F + 2Dv); bidirectional
    # 16 D F + 10 F Dv (no masked term)
    step_roofline = None
    if op in ("bwd", "bidir_bwd", "seqpar_bwd"):
        D_, Dv_, F_ = w.D, w.Dv, w.F
        per = 16 * D_ * F_ + 10 * F_ * Dv_ + ((C_CHUNK + 1) * (3 * F_ + 2 * Dv_) if op != "bidir_bwd" else 0)
        # (the sequence-parallel backward: this rank's tokens)
        toks = units_per_step if op == "seqpar_bwd" else w.B * w.L
        flop = per * w.H * toks
        tflops = flop / (total_ms / args.steps / 1e3) / 1e12
        step_roofline = {"bound": "tensor", "algorithmic_flop_per_step": flop,
                         "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"], "peak_source": peak_src}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cores = os.cpu_count() or 1
        dt, u, threads, desc = oracle_baseline(w, op, cores)
        cpu = {"value": u / dt, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}

    if rank == 0:
        line = {"metric": metric_of(w, op, unit), "value": value, "unit": unit,
                "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "strong" if op in ("seqpar", "seqpar_bwd") else "weak", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic",
                "config": config_of(w, op),
                "e2e": {"value": e2e, "unit": unit, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": len(trace),
                "roofline": roofline, "kernels": kernels, "clocks": clocks,
                "step_roofline": step_roofline,
                "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------- matched-feature-budget comparison

def run_comparison(args, w):
    """Latency of the causal forward at one feature budget F = R*m with different feature
    maps on the same kernels: the SLAY map (positive anchor) and the Performer FAVOR+ map,
    both by the CUDA-core variant kernel, each followed by the same contraction on the given
    features; the SLAY map on tensor cores followed by that contraction; and the fused
    tensor-core SLAY forward.  Inputs resident in HBM, L2 flushed between steps, CUDA events
    on the launching stream; rank 0 prints one JSON line (a comparison, not the headline)."""
    import torch
    from kernelized_linear_attention_unit_b200 import binding as bd
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    eps = float(np.float32(w.eps))
    qn, kn, vn = W.gen_qkv(w)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev).to(torch.bfloat16)
    q, k, v = to(qn), to(kn), to(vn)
    B, H, L, F = w.B, w.H, w.L, w.F
    pq = torch.empty((B, H, L, F), device=dev, dtype=torch.bfloat16)
    pk = torch.empty_like(pq)
    out = torch.empty_like(v)
    den = torch.empty((B, H, L), device=dev, dtype=torch.float32)
    wl = bd.alloc_workspace(bd.OP_LINEAR_ATTN, bd.SLAY_BF16, B, H, L, 64, 64, 1, F, dev)
    wf = bd.alloc_workspace(bd.OP_CAUSAL_FWD, bd.SLAY_BF16, B, H, L, 64, 64, w.R, w.m, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def maps(kind):
        if kind is None:          # the library's default map (tensor cores for these sizes)
            bd.slay_feature_map(q, pq, w.R, w.m, w.sketch_seed, eps)
            bd.slay_feature_map(k, pk, w.R, w.m, w.sketch_seed, eps)
        else:                     # the CUDA-core variant kernel (per head with one head = SLAY)
            bd.slay_feature_map_ex(q, pq, w.R, w.m, w.sketch_seed, eps, kind, 1, L)
            bd.slay_feature_map_ex(k, pk, w.R, w.m, w.sketch_seed, eps, kind, 1, L)

    def contract():
        bd.slay_linear_attn_fwd(pq, pk, v, out, den, eps, True, wl)

    arms = {
        "slay_anchor_cuda_cores": (lambda: maps(bd.PHI_PER_HEAD), contract),
        "performer_favor_cuda_cores": (lambda: maps(bd.PHI_PERFORMER), contract),
        "slay_anchor_tensor_cores": (lambda: maps(None), contract),
        "slay_fused_tensor_cores": (None, lambda: bd.slay_attn_causal_fwd(
            q, k, v, out, den, w.R, w.m, w.sketch_seed, eps, wf)),
    }

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / args.steps

    res = {}
    for name, (mp_, ct) in arms.items():
        step = (lambda m=mp_, c=ct: (m(), c())) if mp_ else ct
        ms = timed(step)
        entry = {"ms_per_step": ms, "tokens_per_s": B * L / (ms / 1e3)}
        if mp_:
            entry["map_ms"] = timed(mp_)
        res[name] = entry
    base = res["slay_anchor_cuda_cores"]
    perf = res["performer_favor_cuda_cores"]
    if rank == 0:
        line = {"metric": "causal fwd latency at a matched feature budget (F=%d)" % F,
                "value": base["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": base["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {**config_of(w, "causal"), "workload": "matched_budget_" + w.name},
                "comparison": res,
                "map_ratio_performer_over_slay": perf["map_ms"] / base["map_ms"],
                "step_ratio_performer_over_slay": perf["ms_per_step"] / base["ms_per_step"]}
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ rank launch

def free_port():
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_ranks(n, argv):
    """Run this same command line as n ranks under torch.distributed.run on this node
    (rendezvous on 127.0.0.1); returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(n), "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def check_launch(args):
    """--check-launch: start the process group exactly as the benchmark does (NCCL with a
    GPU per rank, gloo without one), run its barrier and max-over-ranks steps on a fixed
    per-rank number, and have rank 0 print which ranks took part.  Times nothing."""
    import datetime
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = "cpu"
    backend = "gloo"
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        device, backend = torch.device("cuda", local), "nccl"
    if world > 1:
        kw = {"device_id": device} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60), **kw)
        dist.barrier()
    slowest = max_over_ranks(float(rank), world, device)
    ranks = [rank]
    if world > 1:
        got = [None] * world
        dist.all_gather_object(got, rank)
        ranks = got
        dist.barrier()
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": world, "ranks": ranks,
                          "backend": backend if world > 1 else None,
                          "max_over_ranks": slowest}), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="causal_16k", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--check-launch", action="store_true",
                    help="start the ranks and the process group, report them, time nothing")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        # not started by torchrun: start the N ranks here, one process per GPU
        return relaunch_ranks(args.gpus, argv)
    if world_env is not None and int(world_env) != args.gpus:
        ap.error("--gpus %d does not match WORLD_SIZE=%s" % (args.gpus, world_env))
    if args.check_launch:
        return check_launch(args)
    w, op = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w, op)
    if op == "matched_budget":
        return run_comparison(args, w)
    return run_ours(args, w, op)


if __name__ == "__main__":
    sys.exit(main())
