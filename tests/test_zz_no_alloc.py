"""moe_dispatch_noalloc against moe_dispatch, through the C ABI (marked gpu).

moe_dispatch_noalloc serves callers that cannot give the library scratch
memory -- code running under a device-memory plan fixed in advance, or
inside a framework that owns the allocator, where calling cudaMalloc is not
allowed and no workspace is at hand.  Its scratch is a fixed array inside
libmoe.so.  This test calls it twice in a row on different routings (the
second call must not see the first call's leftovers) and requires its
outputs to equal those of moe_dispatch with a caller workspace, bit for
bit, as every dispatch output is integer or a row copy.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_53_b200 as M
from mixture_experts_layer_53_b200 import build

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, cfg, x, ids):
    A = cfg.N * cfg.k
    dev = ids.device
    out = {
        "x_sorted": torch.full((A, cfg.d_model), -7.0, dtype=cfg.torch_dtype, device=dev),
        "perm": torch.full((A,), -1, dtype=torch.int32, device=dev),
        "inv_perm": torch.full((A,), -1, dtype=torch.int32, device=dev),
        "offsets": torch.full((cfg.E + 1,), -1, dtype=torch.int32, device=dev),
        "counts": torch.full((cfg.E,), -1, dtype=torch.int32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.moe_dispatch_noalloc(ctypes.byref(cfg), p(x), p(ids), p(out["x_sorted"]), p(out["perm"]),
                                  p(out["inv_perm"]), p(out["offsets"]), p(out["counts"]), p(out["status"]),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out


def _routing(rng, N, E, k, skew):
    if skew:  # most tokens on a few experts, several experts idle
        pri = np.argsort(rng.standard_normal(E))
        ids = [pri[:k] if rng.random() < 0.7 else rng.permutation(E)[:k] for _ in range(N)]
    else:
        ids = [rng.permutation(E)[:k] for _ in range(N)]
    return torch.from_numpy(np.stack(ids).astype(np.int32)).cuda()


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    build.build()
    lib = M.library()
    rng = np.random.default_rng(2024)
    cases = [(1000, 4096 // 16, 128, 8, False), (3333, 136, 64, 6, True)]
    for N, d, E, k, skew in cases:  # two calls in a row, different sizes and routings
        cfg = M.make_config(N, d, 64, E, k, act="swiglu", dtype="bf16")
        x = torch.randn((N, d), device="cuda").to(torch.bfloat16)
        ids = _routing(rng, N, E, k, skew)
        rc, got = _call_noalloc(lib, cfg, x, ids)
        assert rc == 0, M.STATUS.get(rc, rc)
        want = M.moe_dispatch(cfg, ids, x=x)
        torch.cuda.synchronize()
        for key in ("x_sorted", "perm", "inv_perm", "offsets", "counts", "status"):
            assert torch.equal(got[key], want[key]), key
        assert int(got["status"][0]) == 0


def test_noalloc_dispatch_refuses_sizes_beyond_its_scratch():
    build.build()
    lib = M.library()
    E = 256
    N = (M.NOALLOC_DISPATCH_MAX_SLOTS // E) * 32 + 1  # one chunk too many
    cfg = M.make_config(N, 64, 64, E, 8, dtype="bf16")
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = lib.moe_dispatch_noalloc(ctypes.byref(cfg), None, p, None, None, p, p, p, None, None)
    assert rc == 4  # MOE_ERR_WORKSPACE, nothing enqueued
