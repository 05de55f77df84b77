"""Data parallelism: every rank of a torch.distributed process group runs
the whole layer on its own tokens with replicated weights, and the Switch
loss and the aux-free bias step are taken over the whole batch.

Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
loss, aux-free bias", sec. 2.3 (L = E sum_e f_e P_e with f and P averages
over the batch) and sec. 2.5 (the sign rule on the batch's expert load):
when the batch is split across ranks, both need one exchange of two [E]
vectors, the assignment counts and the probability sums sum_n p_{n,e}.

Per forward, on each rank:

  1. moe_forward_partials: the layer on the rank's tokens, writing y and the
     two partials (the selection bias is read, not moved);
  2. two all-reduce sums (NCCL between GPUs), counts int32 [E] and the
     probability sums float64 [E];
  3. moe_aux_from_partials: the whole batch's L and, with gamma > 0, one
     sign-rule step of b_e on the whole batch's load.  Every rank holds the
     same sums, so every rank computes the same L and the same b_e.

The token path (route, dispatch, expert GEMMs, combine) has no collective;
only the loss and the bias step wait for the exchange.
"""
from typing import Dict, Optional

import torch
import torch.distributed as dist

from . import MoeConfig, forward_outputs, moe_aux_from_partials, moe_forward_partials, workspace


def all_reduce_partials(counts: torch.Tensor, psum: torch.Tensor, group=None) -> None:
    """Sum the Switch-loss partials over the group, in place (counts int32
    [E], psum float64 [E]); the same two collectives in the same order on
    every rank."""
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(psum, op=dist.ReduceOp.SUM, group=group)


class DataParallelMoE:
    """The layer on one rank of a data-parallel group (see the module doc).

    ``forward`` returns (y [N, d_model], aux [1] f32 -- the whole batch's
    Switch loss --, counts [E] int32 -- the whole batch's load).  With
    ``gamma > 0`` and a sigmoid router's ``b_e``, b_e is moved in place by
    one sign-rule step on the whole batch's load after this forward's
    selection, identically on every rank.
    """

    def __init__(self, cfg: MoeConfig, group=None, gamma: float = 0.0, device=None):
        self.cfg = cfg
        self.group = group
        self.gamma = float(gamma)
        dev = torch.device(device or "cuda")
        self.ws = workspace(cfg, dev)
        self.out = forward_outputs(cfg, dev)
        self.out["psum"] = torch.empty(cfg.E, dtype=torch.float64, device=dev)
        self.aux = torch.empty(1, dtype=torch.float32, device=dev)

    def forward(self, x: torch.Tensor, W_g: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor,
                W3: Optional[torch.Tensor] = None, b1: Optional[torch.Tensor] = None,
                b2: Optional[torch.Tensor] = None, b_e: Optional[torch.Tensor] = None,
                shared: Optional[Dict[str, Optional[torch.Tensor]]] = None):
        cfg = self.cfg
        out = moe_forward_partials(cfg, x, W_g, W1, W2, W3=W3, b1=b1, b2=b2, b_e=b_e, ws=self.ws, out=self.out,
                                   shared=shared)
        all_reduce_partials(out["counts"], out["psum"], self.group)
        moe_aux_from_partials(cfg.E, cfg.k, out["counts"], out["psum"], gamma=self.gamma, b_e=b_e, aux=self.aux)
        return out["y"], self.aux, out["counts"]
