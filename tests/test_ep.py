"""Expert parallelism's host logic on CPU, with gloo ranks.

* ep.plan (split sizes, the regroup permutation and the local slices)
  against brute force;
* the whole expert-parallel forward with two gloo ranks: each rank routes
  and dispatches its own tokens (the fp64 oracle), ep.plan and ep.exchange
  (the library's code) move the rows to their experts' ranks and back, the
  local experts and the combine are the oracle's again.  The result must
  equal the oracle's single-process forward of the rank's tokens (course
  module "Going further": experts on different devices, tokens moved by
  all-to-all; the sec. 2.2 forward is unchanged by where the experts live).

There is no GPU on this path; tests/test_gpu_ep.py runs the same forward
with the library's kernels.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_53_b200 import ep as EP

WORLD = 2


def test_plan_matches_brute_force():
    rng = np.random.default_rng(7)
    for world, E_r in ((1, 3), (2, 2), (3, 4)):
        E = world * E_r
        counts = rng.integers(0, 5, size=E)
        recv = rng.integers(0, 6, size=(world, E_r))
        recv[0, 0] = 0  # an empty (source, expert) block
        p = EP.plan(counts, recv, world)
        assert p.send_rows == [int(v) for v in counts.reshape(world, E_r).sum(1)]
        assert p.recv_rows == [int(v) for v in recv.sum(1)]
        # received rows in (source, local expert, i) order, as the exchange delivers them
        labels = [(s, j, i) for s in range(world) for j in range(E_r) for i in range(recv[s, j])]
        assert sorted(p.regroup.tolist()) == list(range(len(labels)))
        regrouped = [None] * len(labels)
        for src_pos, dst in enumerate(p.regroup):
            regrouped[dst] = labels[src_pos]
        assert regrouped == sorted(labels, key=lambda t: (t[1], t[0], t[2]))  # expert-major, then source
        # each local expert's slice holds exactly its rows
        for j in range(E_r):
            lo, hi = int(p.offsets[j]), int(p.offsets[j + 1])
            assert all(t[1] == j for t in regrouped[lo:hi]) and hi - lo == recv[:, j].sum()


def test_plan_rejects_bad_shapes():
    with pytest.raises(ValueError):
        EP.plan(np.zeros(5), np.zeros((2, 2)), 2)  # 5 experts over 2 ranks
    with pytest.raises(ValueError):
        EP.plan(np.zeros(4), np.zeros((2, 3)), 2)  # recv_counts not [world, E_r]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ep_rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        sys.path.insert(0, root)
        import oracle as O
        import workloads as W
        from mixture_experts_layer_53_b200 import ep

        wl = W.WORKLOADS["mixtral"].scaled(N=37, d_model=16, d_ff=24)  # E 8, k 2, SwiGLU
        inp = W.make_inputs(wl)  # the same seeded weights on every rank
        f64 = lambda t: None if t is None else t.float().numpy().astype(np.float64)
        W1, W2, W3 = f64(inp["W1"]), f64(inp["W2"]), f64(inp["W3"])
        x_all, Wg = f64(inp["x"]), f64(inp["W_g"])
        lo, hi = (0, 20) if rank == 0 else (20, 37)  # uneven token counts per rank
        x = x_all[lo:hi]
        k, E = wl.k, wl.E
        E_r = E // world

        r = O.route(x, Wg, k)
        dsp = O.dispatch(r["ids"], E)
        x_sorted = x[dsp["perm"] // k]
        recv_counts = ep.exchange(torch.from_numpy(dsp["counts"].astype(np.int64)), [E_r] * world, [E_r] * world)
        p = ep.plan(dsp["counts"], recv_counts.numpy().reshape(world, E_r), world)
        x_recv = ep.exchange(torch.from_numpy(x_sorted), p.send_rows, p.recv_rows).numpy()
        x_local = np.empty_like(x_recv)
        x_local[p.regroup] = x_recv
        y_local = np.zeros_like(x_local)
        for j in range(E_r):
            e = rank * E_r + j
            for row in range(int(p.offsets[j]), int(p.offsets[j + 1])):
                y_local[row] = O.expert_ffn(x_local[row], W1[e], W2[e], act=wl.act, W3e=W3[e])
        y_recv = y_local[p.regroup]
        y_sorted = ep.exchange(torch.from_numpy(y_recv), p.recv_rows, p.send_rows).numpy()
        y = O.combine(y_sorted, r["w"], dsp["inv_perm"])
        y_ref = O.dense_forward(x, r["ids"], r["w"], W1, W2, wl.act, W3)
        results[f"err{rank}"] = float(np.max(np.abs(y - y_ref)))
        results[f"rows{rank}"] = int(x_recv.shape[0])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_expert_parallel():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_ep_rank_main, args=(WORLD, _free_port(), results), nprocs=WORLD, join=True,
                           start_method="spawn")
        assert results["rows0"] + results["rows1"] == 37 * 2  # every assignment reached its expert once
        assert results["err0"] < 1e-12 and results["err1"] < 1e-12, dict(results)
