"""The multi-rank host logic on CPU, with two gloo ranks.

* bench.py's max-over-ranks reduction of the timed region;
* the layer is token-parallel: tokens sharded over ranks give the same
  outputs as the whole batch, and the data-parallel layer's exchange
  (``dp.all_reduce_partials``: int32 counts and float64 probability sums,
  the inputs of moe_aux_from_partials) gives the whole batch's Switch loss
  (course module sec. 2.3: L = E sum_e f_e P_e over all N tokens).
The layer math here is the fp64 oracle (no GPU on this path).
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        sys.path.insert(0, root)
        import torch
        import bench
        import oracle as O
        import workloads as W

        # timing reduction: every rank sees the slowest rank's time
        got = bench.max_over_ranks(10.0 + rank * 5.0, world)
        assert got == 10.0 + (world - 1) * 5.0

        wl = W.WORKLOADS["gpt2_moe"].scaled(N=96, d_model=64, d_ff=128)
        inp = W.make_inputs(wl)
        x = inp["x"].float().numpy().astype(np.float64)
        Wg = inp["W_g"].float().numpy().astype(np.float64)
        lo, hi = rank * wl.N // world, (rank + 1) * wl.N // world
        r = O.route(x[lo:hi], Wg, wl.k)
        f64 = lambda t: None if t is None else t.float().numpy().astype(np.float64)
        y = O.dense_forward(x[lo:hi], r["ids"], r["w"], f64(inp["W1"]), f64(inp["W2"]), wl.act, None,
                            f64(inp["b1"]), f64(inp["b2"]))
        # the partials moe_forward_partials returns, exchanged by the
        # data-parallel layer's own all-reduce step, then the whole batch's
        # loss from them (the oracle's statement of moe_aux_from_partials)
        from mixture_experts_layer_53_b200 import dp as DP
        counts = torch.from_numpy(np.bincount(r["ids"].reshape(-1), minlength=wl.E).astype(np.int32))
        psum = torch.from_numpy(r["probs"].sum(axis=0))
        DP.all_reduce_partials(counts, psum)
        L = O.aux_from_partials(counts.numpy(), psum.numpy(), wl.k)
        ys = [torch.zeros(0)] * world
        dist.all_gather_object(ys, y)
        if rank == 0:
            full = O.route(x, Wg, wl.k)
            y_full = O.dense_forward(x, full["ids"], full["w"], f64(inp["W1"]), f64(inp["W2"]), wl.act, None,
                                     f64(inp["b1"]), f64(inp["b2"]))
            L_full, counts_full = O.aux_loss(full["probs"], full["ids"])
            results["y_equal"] = bool(np.array_equal(np.concatenate(ys), y_full))
            results["counts_equal"] = bool(np.array_equal(counts.numpy(), counts_full))
            results["L_err"] = abs(L - L_full)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(WORLD, _free_port(), results), nprocs=WORLD, join=True,
                           start_method="spawn")
        assert results["y_equal"], "token shards differ from the whole batch"
        assert results["counts_equal"]
        assert results["L_err"] < 1e-12
