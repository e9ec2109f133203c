"""Sequence-parallel causal SLAY forward and backward over the ranks of a process group.

The causal contraction's prefix state carries everything earlier tokens contribute
(review, "Proposed method", step 6), so a long sequence split into contiguous pieces, one
per rank in rank order, needs one exchange: each rank sums its own piece's state
(slay_attn_causal_fwd_begin: sum of phi(k) [v, 1]^T, with phi(k) and the segment sums kept
in its workspace), the ranks all-gather those states (F x (Dv+1) fp32 per (b, h)), each rank
adds up the states of the ranks before it (slay_state_prefix) and runs its piece's causal
forward from that state on the kept phi(k) (slay_attn_causal_fwd_finish).  The
backward also needs, for each piece, the sum of phi(q) [dn, delta]^T over the later ranks'
tokens: one more all-gather of the pieces' such sums (slay_attn_causal_bwd_begin, which keeps
phi(q) and the row statistics in its workspace), a suffix over ranks (slay_state_suffix),
then the piece's backward from both states on the kept values (slay_attn_causal_bwd_finish).  The collective is NCCL's all-gather over NVLink on GPUs (any
backend works: the states are ordinary tensors); no kernel waits on another rank's memory.

Every step of the path runs in the library's kernels; this module orders them and calls the
collective.  The steps are passed in as an object (LibraryOps by default: begin, prefix,
finish for the forward; bwd_begin, suffix, bwd_finish, and state when the forward's prefix
state is not passed in, for the backward), so the same orchestration runs in tests on CPU
ranks.
"""
from typing import Optional

import torch
import torch.distributed as dist

from . import binding as bd


class LibraryOps:
    """The steps through libslay.so (device tensors)."""

    def __init__(self, R, m, seed, eps):
        self.R, self.m, self.seed, self.eps = R, m, seed, eps

    def begin(self, k, v, S_out, z_out, handle=None):
        """The piece's state; returns the workspace that carries phi(k) to finish (handle: a
        workspace of an earlier call on the same sizes, reused)."""
        return bd.slay_attn_causal_fwd_begin(k, v, S_out, z_out, self.R, self.m, self.seed,
                                             self.eps, workspace=handle)

    def finish(self, q, k, v, out, den, S_in, z_in, handle):
        bd.slay_attn_causal_fwd_finish(q, k, v, out, den, self.R, self.m, self.seed, self.eps,
                                       handle, S_in=S_in, z_in=z_in)

    def state(self, k, v, S_out, z_out):
        bd.slay_causal_state(k, v, S_out, z_out, self.R, self.m, self.seed, self.eps)

    def prefix(self, S_all, z_all, rank, S_in, z_in):
        bd.slay_state_prefix(S_all, z_all, rank, S_in, z_in)

    def bwd_begin(self, q, out, den, dout, G_out, zg_out, handle=None):
        """The piece's phi(q)[dn, delta] sum; returns the workspace that carries phi(q) and
        the row statistics to bwd_finish."""
        return bd.slay_attn_causal_bwd_begin(q, out, den, dout, G_out, zg_out, self.R, self.m,
                                             self.seed, self.eps, workspace=handle)

    def suffix(self, G_all, zg_all, rank, G_in, zg_in):
        bd.slay_state_suffix(G_all, zg_all, rank, G_in, zg_in)

    def bwd_finish(self, q, k, v, out, den, dout, dq, dk, dv, S_in, z_in, G_in, zg_in, handle):
        bd.slay_attn_causal_bwd_finish(q, k, v, out, den, dout, dq, dk, dv, self.R, self.m,
                                       self.seed, self.eps, handle, S_in=S_in, z_in=z_in,
                                       G_in=G_in, zg_in=zg_in)


def gather_states(S_loc: torch.Tensor, z_loc: torch.Tensor, group=None):
    """All ranks' piece states stacked in rank order: [N, B, H, F, Dv] and [N, B, H, F]."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return S_loc.unsqueeze(0), z_loc.unsqueeze(0)
    S_list = [torch.empty_like(S_loc) for _ in range(world)]
    z_list = [torch.empty_like(z_loc) for _ in range(world)]
    dist.all_gather(S_list, S_loc.contiguous(), group=group)
    dist.all_gather(z_list, z_loc.contiguous(), group=group)
    return torch.stack(S_list), torch.stack(z_list)


def causal_fwd_seqpar(q, k, v, out, den, F: int, ops, group=None,
                      scratch: Optional[dict] = None):
    """This rank's piece [B, H, Lr, D] of a sequence split over the group in rank order:
    out (and den, if given) of the causal forward of the whole sequence at this piece's rows.

    F = R * m features; ops: LibraryOps (or an object with its begin, prefix and finish
    methods); scratch: optional dict reused across calls for the state buffers and the
    workspace begin hands to finish."""
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, H, Lr = q.shape[0], q.shape[1], q.shape[2]
    Dv = v.shape[-1]
    sc = scratch if scratch is not None else {}
    shape_s, shape_z = (B, H, F, Dv), (B, H, F)
    key = (shape_s, Lr, q.dtype, q.device)
    if sc.get("shape") != key:
        sc.clear()
        sc["shape"] = key
        for name in ("S_loc", "S_in"):
            sc[name] = torch.empty(shape_s, dtype=torch.float32, device=q.device)
        for name in ("z_loc", "z_in"):
            sc[name] = torch.empty(shape_z, dtype=torch.float32, device=q.device)
    sc["handle"] = ops.begin(k, v, sc["S_loc"], sc["z_loc"], sc.get("handle"))
    S_all, z_all = gather_states(sc["S_loc"], sc["z_loc"], group)
    ops.prefix(S_all, z_all, rank, sc["S_in"], sc["z_in"])
    ops.finish(q, k, v, out, den, sc["S_in"], sc["z_in"], sc["handle"])
    return out


def causal_bwd_seqpar(q, k, v, out, den, dout, dq, dk, dv, F: int, ops, group=None,
                      scratch: Optional[dict] = None, fwd_state=None):
    """This rank's piece of the backward of a sequence split over the group in rank order:
    dq, dk, dv of the whole sequence's backward at this piece's rows.  out, den are this
    piece's rows of the forward (causal_fwd_seqpar), dout its upstream gradient.

    Besides the prefix state of the forward (the sum of phi(k)[v, 1] over the earlier
    ranks), the backward needs the sum of phi(q)[dn, delta] over the later ranks' tokens:
    each rank computes its piece's (ops.bwd_begin), the ranks all-gather them and each adds
    up those of the ranks after it (ops.suffix) before its local backward (ops.bwd_finish,
    on what bwd_begin kept).
    fwd_state: the (S_in, z_in) this rank's forward started from (the scratch of
    causal_fwd_seqpar on the same q, k, v), which saves recomputing it."""
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, H = q.shape[0], q.shape[1]
    Dv = v.shape[-1]
    sc = scratch if scratch is not None else {}
    shape_s, shape_z = (B, H, F, Dv), (B, H, F)
    key = (shape_s, q.shape[2], q.dtype, q.device)
    if sc.get("bwd_shape") != key:
        sc["bwd_shape"] = key
        sc.pop("bwd_handle", None)
        for name in ("bS_loc", "bS_in", "bG_loc", "bG_in"):
            sc[name] = torch.empty(shape_s, dtype=torch.float32, device=q.device)
        for name in ("bz_loc", "bz_in", "bzg_loc", "bzg_in"):
            sc[name] = torch.empty(shape_z, dtype=torch.float32, device=q.device)
    if fwd_state is None:
        ops.state(k, v, sc["bS_loc"], sc["bz_loc"])
        S_all, z_all = gather_states(sc["bS_loc"], sc["bz_loc"], group)
        ops.prefix(S_all, z_all, rank, sc["bS_in"], sc["bz_in"])
        S_in, z_in = sc["bS_in"], sc["bz_in"]
    else:
        S_in, z_in = fwd_state
    sc["bwd_handle"] = ops.bwd_begin(q, out, den, dout, sc["bG_loc"], sc["bzg_loc"],
                                     sc.get("bwd_handle"))
    G_all, zg_all = gather_states(sc["bG_loc"], sc["bzg_loc"], group)
    ops.suffix(G_all, zg_all, rank, sc["bG_in"], sc["bzg_in"])
    ops.bwd_finish(q, k, v, out, den, dout, dq, dk, dv, S_in, z_in, sc["bG_in"], sc["bzg_in"],
                   sc["bwd_handle"])
    return dq, dk, dv
