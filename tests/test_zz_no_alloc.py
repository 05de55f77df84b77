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


def _outputs(cfg, dev, with_rows):
    """Output buffers pre-filled with marker values, so that entries an entry
    point leaves unwritten compare equal only if both leave them alone."""
    A = cfg.N * cfg.k
    return {
        "x_sorted": torch.full((A, cfg.d_model), -7.0, dtype=cfg.torch_dtype, device=dev) if with_rows else None,
        "perm": torch.full((A,), -5, dtype=torch.int32, device=dev),
        "inv_perm": torch.full((A,), -5, dtype=torch.int32, device=dev),
        "offsets": torch.full((cfg.E + 1,), -5, dtype=torch.int32, device=dev),
        "counts": torch.full((cfg.E,), -5, dtype=torch.int32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }


def _p(t):
    return None if t is None or t.numel() == 0 else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(lib, cfg, x, ids):
    out = _outputs(cfg, ids.device, x is not None)
    rc = lib.moe_dispatch_noalloc(ctypes.byref(cfg), _p(x), _p(ids), _p(out["x_sorted"]), _p(out["perm"]),
                                  _p(out["inv_perm"]), _p(out["offsets"]), _p(out["counts"]), _p(out["status"]),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out


def _call_workspace(lib, cfg, x, ids):
    """moe_dispatch with a caller workspace, into buffers filled like _call_noalloc's."""
    out = _outputs(cfg, ids.device, x is not None)
    ws = M.workspace(cfg, ids.device)
    rc = lib.moe_dispatch(ctypes.byref(cfg), _p(x), _p(ids), _p(out["x_sorted"]), _p(out["perm"]),
                          _p(out["inv_perm"]), _p(out["offsets"]), _p(out["counts"]), _p(out["status"]),
                          _p(ws), ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out


def _assert_same(got, want):
    for key in ("x_sorted", "perm", "inv_perm", "offsets", "counts", "status"):
        if want[key] is None:
            assert got[key] is None, key
        else:
            assert torch.equal(got[key], want[key]), key


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
        rc, want = _call_workspace(lib, cfg, x, ids)
        assert rc == 0, M.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        _assert_same(got, want)
        assert int(got["status"][0]) == 0


@pytest.mark.parametrize("case", ["positions_only", "no_tokens", "bad_ids_with_rows", "bad_ids_positions_only"])
def test_noalloc_dispatch_other_paths(case):
    """The paths besides rows-with-valid-ids: x = NULL (positions only), N = 0
    (the scan alone writes zero counts and offsets), and expert ids outside
    [0, E) (MOE_ERR_BAD_EXPERT_ID; those assignments get inv_perm = -1 and no
    row).  Each is compared bit for bit with moe_dispatch on buffers pre-filled
    with the same marker values, twice in a row."""
    build.build()
    lib = M.library()
    rng = np.random.default_rng(7)
    N = 0 if case == "no_tokens" else 517
    E, k, d = 24, 3, 72
    cfg = M.make_config(N, d, 64, E, k, act="swiglu", dtype="bf16")
    for _ in range(2):
        ids = _routing(rng, N, E, k, skew=True) if N else torch.zeros((0, k), dtype=torch.int32, device="cuda")
        if case.startswith("bad_ids"):
            ids[5, 1] = E
            ids[200, 0] = -3
            ids[N - 1, 2] = 1 << 20
        with_rows = case in ("bad_ids_with_rows",)
        x = torch.randn((N, d), device="cuda").to(torch.bfloat16) if with_rows else None
        rc, got = _call_noalloc(lib, cfg, x, ids)
        assert rc == 0, M.STATUS.get(rc, rc)
        rc, want = _call_workspace(lib, cfg, x, ids)
        assert rc == 0, M.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        _assert_same(got, want)
        if case.startswith("bad_ids"):
            assert int(got["status"][0]) == 6  # MOE_ERR_BAD_EXPERT_ID
            inv = got["inv_perm"].view(N, k).cpu()
            assert inv[5, 1] == -1 and inv[200, 0] == -1 and inv[N - 1, 2] == -1
            assert int(got["counts"].sum()) == N * k - 3
        elif case == "no_tokens":
            assert int(got["status"][0]) == 0
            assert torch.equal(got["counts"].cpu(), torch.zeros(E, dtype=torch.int32))
            assert torch.equal(got["offsets"].cpu(), torch.zeros(E + 1, dtype=torch.int32))
        else:
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
