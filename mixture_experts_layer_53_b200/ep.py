"""Expert parallelism: the layer's E experts split over the ranks of a
torch.distributed process group, tokens moved to their experts' rank and
back by two all-to-all exchanges.

Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
loss, aux-free bias", "Going further" (expert parallelism: experts on
different GPUs, tokens moved by all-to-all), on top of its sec. 2.2 sorted
dispatch, which already leaves each expert's rows as one contiguous slice.

Rank r holds experts r * E_r .. (r + 1) * E_r - 1 (E_r = E / world).  Each
rank runs the layer for its own N tokens:

  1. moe_route and moe_dispatch: x_sorted grouped by expert, so the rows for
     each rank's experts form one contiguous block, in rank order;
  2. the per-expert row counts go to the experts' ranks (an all-to-all of
     E_r integers per pair of ranks), then the rows themselves (an
     all-to-all whose split sizes are those counts summed per rank);
  3. the received rows arrive ordered (source rank, local expert); they are
     regrouped to (local expert, source rank) with moe_permute_rows so that
     every local expert has one contiguous slice, and moe_expert_ffn runs
     the local experts over them;
  4. the results go back to the (source rank, local expert) order and to
     their ranks (the reverse all-to-all), and moe_combine weights them in
     token order.  moe_aux_loss gives the rank's Switch loss as in the
     data-parallel layer.

The exchanges are torch.distributed collectives (NCCL between GPUs); every
step between them runs in libmoe.so.  The split sizes are needed on the
host: one device-to-host copy of 2 E integers per forward.  This is the
plain form of the exchange; a kernel that moves the rows over NVLink peer
memory while the expert GEMMs run would replace steps 2 and 4.
"""
from typing import List, NamedTuple, Optional

import numpy as np
import torch
import torch.distributed as dist

from . import (MoeConfig, make_config, moe_aux_loss, moe_combine, moe_dispatch, moe_expert_ffn, moe_permute_rows,
               moe_route)


class EPPlan(NamedTuple):
    send_rows: List[int]  # rows this rank sends to each rank (x_sorted blocks, rank order)
    recv_rows: List[int]  # rows it receives from each rank
    offsets: np.ndarray   # [E_r + 1] int32: the local experts' slices after the regroup
    regroup: np.ndarray   # [R] int32: received row i goes to row regroup[i] of the regrouped rows


def plan(counts: np.ndarray, recv_counts: np.ndarray, world: int) -> EPPlan:
    """Split sizes and the regroup permutation of one exchange.

    counts [E]: this rank's rows per global expert (its dispatch counts);
    recv_counts [world, E_r]: the rows each rank sends for each of this
    rank's local experts (what the counts exchange delivered).
    """
    counts = np.asarray(counts, dtype=np.int64)
    recv_counts = np.asarray(recv_counts, dtype=np.int64)
    E = counts.shape[0]
    if world <= 0 or E % world != 0:
        raise ValueError(f"{E} experts do not split over {world} ranks")
    E_r = E // world
    if recv_counts.shape != (world, E_r):
        raise ValueError(f"recv_counts must be [{world}, {E_r}]")
    send = counts.reshape(world, E_r).sum(axis=1)
    recv = recv_counts.sum(axis=1)
    per_expert = recv_counts.sum(axis=0)
    offsets = np.zeros(E_r + 1, dtype=np.int64)
    np.cumsum(per_expert, out=offsets[1:])
    # rows of (source s, local expert j) start, after the regroup, at
    # offsets[j] + the rows of expert j from sources before s
    start = offsets[:-1][None, :] + np.cumsum(recv_counts, axis=0) - recv_counts
    regroup = np.empty(int(recv.sum()), dtype=np.int64)
    pos = 0
    for s in range(world):
        for j in range(E_r):
            c = int(recv_counts[s, j])
            regroup[pos:pos + c] = np.arange(start[s, j], start[s, j] + c)
            pos += c
    return EPPlan([int(v) for v in send], [int(v) for v in recv], offsets.astype(np.int32),
                  regroup.astype(np.int32))


def exchange(t: torch.Tensor, send_rows: List[int], recv_rows: List[int], group=None) -> torch.Tensor:
    """All-to-all of the leading-axis blocks of t: send_rows[r] rows to rank r,
    recv_rows[r] rows from rank r (concatenated in rank order)."""
    out = t.new_empty((sum(recv_rows),) + tuple(t.shape[1:]))
    dist.all_to_all_single(out, t.contiguous(), recv_rows, send_rows, group=group)
    return out


class DispatchState(NamedTuple):
    """What a rank keeps between its dispatch and its combine."""
    ids: torch.Tensor       # [N, k] int32
    w: torch.Tensor         # [N, k] f32
    probs: torch.Tensor     # [N, E] f32
    x_sorted: torch.Tensor  # [N k, d_model], grouped by expert
    inv_perm: torch.Tensor  # [N k] int32
    counts: torch.Tensor    # [E] int32


class ExpertParallelMoE:
    """One rank's share of an expert-parallel layer (see the module docstring).

    cfg: the layer's configuration with this rank's token count N and all E
    experts.  The rank's expert weights follow the layer layout restricted
    to its experts: W1 / W3 [E_r, d_ff, d_model], W2 [E_r, d_model, d_ff],
    b1 [E_r, d_ff], b2 [E_r, d_model].  ``world`` and ``rank`` default to
    the process group's; given explicitly (with no group), the phases below
    can be driven by a caller that moves the rows itself.
    """

    def __init__(self, cfg: MoeConfig, group=None, world: Optional[int] = None, rank: Optional[int] = None):
        if cfg.d_ff_shared != 0:
            raise ValueError("the shared expert is not part of the expert-parallel exchange")
        self.cfg = cfg
        self.group = group
        self.world = dist.get_world_size(group) if world is None else int(world)
        self.rank = dist.get_rank(group) if rank is None else int(rank)
        if cfg.E % self.world != 0:
            raise ValueError(f"{cfg.E} experts do not split over {self.world} ranks")
        self.E_r = cfg.E // self.world

    def local_config(self, rows: int) -> MoeConfig:
        """The expert FFN's view of the regrouped rows: `rows` rows, k = 1, the local experts."""
        c = self.cfg
        return make_config(rows, c.d_model, c.d_ff, self.E_r, 1, act=("gelu", "swiglu")[c.act],
                           dtype=("f32", "bf16")[c.dtype])

    # -- the three compute phases; the exchanges sit between them

    def dispatch_phase(self, x: torch.Tensor, W_g: torch.Tensor, b_e: Optional[torch.Tensor] = None) -> DispatchState:
        """Step 1: route and dispatch this rank's tokens."""
        ids, w, probs = moe_route(self.cfg, x, W_g, b_e, want_probs=True)
        dsp = moe_dispatch(self.cfg, ids, x)
        return DispatchState(ids, w, probs, dsp["x_sorted"], dsp["inv_perm"], dsp["counts"])

    def expert_phase(self, x_recv: torch.Tensor, p: EPPlan, W1: torch.Tensor, W2: torch.Tensor,
                     W3: Optional[torch.Tensor] = None, b1: Optional[torch.Tensor] = None,
                     b2: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Step 3: the received rows, in (source rank, local expert) order,
        regrouped by local expert, through the local experts and back to the
        received order."""
        rows = x_recv.shape[0]
        y_recv = torch.empty_like(x_recv)
        if rows > 0:
            dev = x_recv.device
            regroup = torch.from_numpy(p.regroup).to(dev)
            back = np.empty_like(p.regroup)
            back[p.regroup] = np.arange(rows, dtype=np.int32)
            x_local = moe_permute_rows(x_recv, regroup)
            y_local = moe_expert_ffn(self.local_config(rows), x_local, torch.from_numpy(p.offsets).to(dev), W1, W2,
                                     b1=b1, W3=W3, b2=b2)
            moe_permute_rows(y_local, torch.from_numpy(back).to(dev), out=y_recv)
        return y_recv

    def combine_phase(self, st: DispatchState, y_sorted: torch.Tensor):
        """Step 4: the rank's rows back in token order, and its Switch loss."""
        y = moe_combine(self.cfg, y_sorted, st.w, st.inv_perm)
        aux, _, _ = moe_aux_loss(self.cfg, st.probs, st.ids)
        return y, aux

    def forward(self, x: torch.Tensor, W_g: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor,
                W3: Optional[torch.Tensor] = None, b1: Optional[torch.Tensor] = None,
                b2: Optional[torch.Tensor] = None, b_e: Optional[torch.Tensor] = None):
        """Returns (y [N, d_model], aux [1] f32: this rank's Switch loss).

        b_e (sigmoid router) selects as in moe_forward; its sign-rule step
        is left to the caller (moe_aux_loss with gamma and b_e, on this
        rank's counts or on counts all-reduced over the group)."""
        cfg, world, E_r, g = self.cfg, self.world, self.E_r, self.group
        st = self.dispatch_phase(x, W_g, b_e)
        recv_counts = exchange(st.counts, [E_r] * world, [E_r] * world, g)
        host = torch.cat([st.counts, recv_counts]).cpu().numpy()
        p = plan(host[:cfg.E], host[cfg.E:].reshape(world, E_r), world)
        x_recv = exchange(st.x_sorted, p.send_rows, p.recv_rows, g)
        y_recv = self.expert_phase(x_recv, p, W1, W2, W3=W3, b1=b1, b2=b2)
        y_sorted = exchange(y_recv, p.recv_rows, p.send_rows, g)
        return self.combine_phase(st, y_sorted)
