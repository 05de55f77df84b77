"""Dropless Mixture-of-Experts layer forward on one B200 -- Python binding.

A thin ctypes layer over ``libmoe.so`` (built from ``csrc/`` for sm_100a):
it marshals torch tensors to device pointers, allocates outputs with torch
and passes the current CUDA stream.  Every step of the layer runs in the
library's CUDA kernels; there is no other implementation behind these
functions.  If the library is missing, every call raises.

The functions carry the names of the C entry points in ``include/moe.h``:
``moe_route``, ``moe_dispatch``, ``moe_expert_ffn``, ``moe_combine``,
``moe_aux_loss``, ``moe_forward`` and ``moe_workspace_size``, plus the
shared expert (``moe_shared_ffn``, ``moe_combine_shared``) and the router
z-loss (``moe_router_z_loss``; ``moe_forward`` with ``shared=`` or
``z_loss=True`` calls ``moe_forward_ex``).  Symbols follow
the course module "Mixture of Experts: routing, sorted dispatch, Switch aux
loss, aux-free bias" (sec. 2): N, E, k, d_model, d_ff, W_g, b_e.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

ROUTERS = {"softmax_topk": 0, "topk_softmax": 1, "sigmoid": 2}
ACTS = {"gelu": 0, "swiglu": 1}
DTYPES = {"f32": 0, "bf16": 1}
TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
          4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_BAD_EXPERT_ID"}
NUM_STAGES = 5
STAGE_NAMES = ("route", "dispatch", "gemm1", "gemm2", "combine")
EXPORTS = ("moe_status_string", "moe_last_error", "moe_version", "moe_workspace_size", "moe_route",
           "moe_dispatch", "moe_dispatch_noalloc", "moe_expert_ffn", "moe_combine", "moe_aux_loss",
           "moe_forward", "moe_shared_ffn", "moe_combine_shared", "moe_router_z_loss", "moe_forward_ex",
           "moe_backward_workspace_size", "moe_backward", "moe_permute_rows", "moe_selftest_wait_timeout",
           "moe_forward_partials", "moe_aux_from_partials")
# ceil(N / 32) * E limit of moe_dispatch_noalloc (MOE_NOALLOC_DISPATCH_MAX_SLOTS)
NOALLOC_DISPATCH_MAX_SLOTS = 1 << 19


class MoeConfig(ctypes.Structure):
    """Mirror of ``moe_config`` in include/moe.h."""
    _fields_ = [("N", ctypes.c_int64), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("router", ctypes.c_int32),
                ("norm_topk", ctypes.c_int32), ("routed_scaling", ctypes.c_float),
                ("act", ctypes.c_int32), ("dtype", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32)]

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == 0 else torch.bfloat16


class SharedExpert(ctypes.Structure):
    """Mirror of ``moe_shared_expert`` in include/moe.h (device pointers)."""
    _fields_ = [("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("W3", ctypes.c_void_p),
                ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


class MoeGrads(ctypes.Structure):
    """Mirror of ``moe_grads`` in include/moe.h (fp32 device pointers)."""
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("dx", "dW_g", "dW1", "db1", "dW3", "dW2", "db2", "dWs1", "dbs1", "dWs3", "dWs2", "dbs2")]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


_lib: Optional[ctypes.CDLL] = None


def library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m mixture_experts_layer_53_b200.build`")
    lib = ctypes.CDLL(p)
    vp, cfgp, i32p, f32p = ctypes.c_void_p, ctypes.POINTER(MoeConfig), ctypes.c_void_p, ctypes.c_void_p
    st, sz = ctypes.c_int, ctypes.c_size_t
    lib.moe_status_string.argtypes = [st]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_last_error.argtypes = []
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_version.argtypes = []
    lib.moe_version.restype = ctypes.c_int32
    lib.moe_workspace_size.argtypes = [cfgp]
    lib.moe_workspace_size.restype = sz
    lib.moe_route.argtypes = [cfgp, vp, vp, f32p, i32p, f32p, f32p, vp, sz, vp]
    lib.moe_route.restype = st
    lib.moe_dispatch.argtypes = [cfgp, vp, i32p, vp, i32p, i32p, i32p, i32p, i32p, vp, sz, vp]
    lib.moe_dispatch.restype = st
    lib.moe_dispatch_noalloc.argtypes = [cfgp, vp, i32p, vp, i32p, i32p, i32p, i32p, i32p, vp]
    lib.moe_dispatch_noalloc.restype = st
    lib.moe_expert_ffn.argtypes = [cfgp, vp, i32p, vp, vp, vp, vp, vp, vp, i32p, vp, sz, vp]
    lib.moe_expert_ffn.restype = st
    lib.moe_combine.argtypes = [cfgp, vp, f32p, i32p, vp, vp]
    lib.moe_combine.restype = st
    lib.moe_aux_loss.argtypes = [cfgp, f32p, i32p, f32p, i32p, ctypes.c_float, f32p, i32p, vp, sz, vp]
    lib.moe_aux_loss.restype = st
    lib.moe_forward.argtypes = [cfgp, vp, vp, f32p, ctypes.c_float, vp, vp, vp, vp, vp, vp, i32p, f32p, i32p,
                                f32p, i32p, vp, sz, ctypes.c_void_p, vp]
    lib.moe_forward.restype = st
    shp = ctypes.POINTER(SharedExpert)
    lib.moe_shared_ffn.argtypes = [cfgp, vp, shp, vp, i32p, vp, sz, vp]
    lib.moe_shared_ffn.restype = st
    lib.moe_combine_shared.argtypes = [cfgp, vp, f32p, i32p, vp, vp, vp]
    lib.moe_combine_shared.restype = st
    lib.moe_router_z_loss.argtypes = [cfgp, vp, vp, f32p, i32p, vp, sz, vp]
    lib.moe_router_z_loss.restype = st
    lib.moe_forward_ex.argtypes = [cfgp, vp, vp, f32p, ctypes.c_float, vp, vp, vp, vp, vp, shp, vp, i32p, f32p,
                                   i32p, f32p, f32p, i32p, vp, sz, ctypes.c_void_p, vp]
    lib.moe_forward_ex.restype = st
    lib.moe_forward_partials.argtypes = [cfgp, vp, vp, f32p, vp, vp, vp, vp, vp, shp, vp, i32p, f32p, i32p, vp,
                                         f32p, i32p, vp, sz, vp]
    lib.moe_forward_partials.restype = st
    lib.moe_aux_from_partials.argtypes = [ctypes.c_int32, ctypes.c_int32, i32p, vp, f32p, ctypes.c_float, f32p, vp]
    lib.moe_aux_from_partials.restype = st
    lib.moe_backward_workspace_size.argtypes = [cfgp]
    lib.moe_backward_workspace_size.restype = sz
    lib.moe_backward.argtypes = [cfgp, vp, vp, f32p, vp, vp, vp, vp, vp, shp, vp, ctypes.c_float, ctypes.c_float,
                                 ctypes.POINTER(MoeGrads), i32p, vp, sz, vp]
    lib.moe_backward.restype = st
    lib.moe_permute_rows.argtypes = [ctypes.c_int32, vp, i32p, vp, ctypes.c_int64, ctypes.c_int32, vp]
    lib.moe_permute_rows.restype = st
    lib.moe_selftest_wait_timeout.argtypes = [i32p, vp]
    lib.moe_selftest_wait_timeout.restype = st
    if path is None:
        _lib = lib
    return lib


def make_config(N: int, d_model: int, d_ff: int, E: int, k: int, router: str = "softmax_topk",
                norm_topk: bool = True, routed_scaling: float = 1.0, act: str = "gelu",
                dtype: str = "bf16", d_ff_shared: int = 0) -> MoeConfig:
    return MoeConfig(int(N), int(d_model), int(d_ff), int(E), int(k), ROUTERS[router], int(bool(norm_topk)),
                     float(routed_scaling), ACTS[act], DTYPES[dtype], int(d_ff_shared))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str) -> None:
    if rc != 0:
        detail = library().moe_last_error().decode() if rc == 3 else ""
        raise MoeError(rc, where, detail)


def moe_workspace_size(cfg: MoeConfig) -> int:
    return int(library().moe_workspace_size(ctypes.byref(cfg)))


def workspace(cfg: MoeConfig, device=None) -> torch.Tensor:
    """A device workspace large enough for every entry point (256-byte aligned)."""
    n = moe_workspace_size(cfg)
    if n == 0:
        raise MoeError(1, "moe_workspace_size")
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def moe_route(cfg: MoeConfig, x: torch.Tensor, W_g: torch.Tensor, b_e: Optional[torch.Tensor] = None,
              want_probs: bool = False, ws: Optional[torch.Tensor] = None, stream=None):
    """Returns (topk_ids [N,k] int32, topk_w [N,k] f32, probs [N,E] f32 or None)."""
    dev = x.device
    ws = ws if ws is not None else workspace(cfg, dev)
    ids = torch.empty((cfg.N, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((cfg.N, cfg.k), dtype=torch.float32, device=dev)
    probs = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device=dev) if want_probs else None
    rc = library().moe_route(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(b_e), _ptr(ids), _ptr(w), _ptr(probs),
                             _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_route")
    return ids, w, probs


def moe_dispatch(cfg: MoeConfig, topk_ids: torch.Tensor, x: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None, stream=None) -> Dict[str, torch.Tensor]:
    """Sorted dispatch: x_sorted (if x given), perm, inv_perm, offsets, counts, status."""
    dev = topk_ids.device
    A = cfg.N * cfg.k
    ws = ws if ws is not None else workspace(cfg, dev)
    out = {
        "x_sorted": torch.empty((A, cfg.d_model), dtype=cfg.torch_dtype, device=dev) if x is not None else None,
        "perm": torch.empty(A, dtype=torch.int32, device=dev),
        "inv_perm": torch.empty(A, dtype=torch.int32, device=dev),
        "offsets": torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
        "counts": torch.empty(cfg.E, dtype=torch.int32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    rc = library().moe_dispatch(ctypes.byref(cfg), _ptr(x), _ptr(topk_ids), _ptr(out["x_sorted"]), _ptr(out["perm"]),
                                _ptr(out["inv_perm"]), _ptr(out["offsets"]), _ptr(out["counts"]),
                                _ptr(out["status"]), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_dispatch")
    return out


def moe_dispatch_noalloc(cfg: MoeConfig, topk_ids: torch.Tensor, x: Optional[torch.Tensor] = None,
                         stream=None) -> Dict[str, torch.Tensor]:
    """moe_dispatch for callers that cannot give the library a workspace.

    The scratch is a fixed array inside libmoe.so (ceil(N/32) * E must not
    exceed NOALLOC_DISPATCH_MAX_SLOTS); the library allocates nothing.  This
    wrapper still creates the output tensors with torch; a caller without an
    allocator passes its own buffers to the C entry point instead.
    """
    dev = topk_ids.device
    A = cfg.N * cfg.k
    out = {
        "x_sorted": torch.empty((A, cfg.d_model), dtype=cfg.torch_dtype, device=dev) if x is not None else None,
        "perm": torch.empty(A, dtype=torch.int32, device=dev),
        "inv_perm": torch.empty(A, dtype=torch.int32, device=dev),
        "offsets": torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
        "counts": torch.empty(cfg.E, dtype=torch.int32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    rc = library().moe_dispatch_noalloc(ctypes.byref(cfg), _ptr(x), _ptr(topk_ids), _ptr(out["x_sorted"]),
                                        _ptr(out["perm"]), _ptr(out["inv_perm"]), _ptr(out["offsets"]),
                                        _ptr(out["counts"]), _ptr(out["status"]), _stream(stream))
    _check(rc, "moe_dispatch_noalloc")
    return out


def moe_expert_ffn(cfg: MoeConfig, x_sorted: torch.Tensor, offsets: torch.Tensor, W1: torch.Tensor,
                   W2: torch.Tensor, b1: Optional[torch.Tensor] = None, W3: Optional[torch.Tensor] = None,
                   b2: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    dev = x_sorted.device
    ws = ws if ws is not None else workspace(cfg, dev)
    y_sorted = torch.empty((cfg.N * cfg.k, cfg.d_model), dtype=cfg.torch_dtype, device=dev)
    rc = library().moe_expert_ffn(ctypes.byref(cfg), _ptr(x_sorted), _ptr(offsets), _ptr(W1), _ptr(b1), _ptr(W3),
                                  _ptr(W2), _ptr(b2), _ptr(y_sorted), _ptr(status), _ptr(ws), ws.numel(),
                                  _stream(stream))
    _check(rc, "moe_expert_ffn")
    return y_sorted


def moe_combine(cfg: MoeConfig, y_sorted: torch.Tensor, topk_w: torch.Tensor, inv_perm: torch.Tensor,
                stream=None) -> torch.Tensor:
    y = torch.empty((cfg.N, cfg.d_model), dtype=cfg.torch_dtype, device=y_sorted.device)
    rc = library().moe_combine(ctypes.byref(cfg), _ptr(y_sorted), _ptr(topk_w), _ptr(inv_perm), _ptr(y),
                               _stream(stream))
    _check(rc, "moe_combine")
    return y


def moe_permute_rows(src: torch.Tensor, dst_row: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """out[dst_row[i]] = src[i] for the rows of src [rows, d] (f32 or bf16); dst_row [rows] int32."""
    dtype = {torch.float32: "f32", torch.bfloat16: "bf16"}.get(src.dtype)
    if dtype is None or src.dim() != 2 or dst_row.dtype != torch.int32 or dst_row.numel() != src.shape[0]:
        raise ValueError("moe_permute_rows: src [rows, d] f32/bf16 and dst_row [rows] int32")
    out = out if out is not None else torch.empty_like(src)
    if src.shape[0] == 0:
        return out
    rc = library().moe_permute_rows(DTYPES[dtype], _ptr(src), _ptr(dst_row), _ptr(out), src.shape[0], src.shape[1],
                                    _stream(stream))
    _check(rc, "moe_permute_rows")
    return out


def _shared_struct(shared: Optional[Dict[str, Optional[torch.Tensor]]]):
    """SharedExpert from {"W1", "W2", "W3"?, "b1"?, "b2"?} (None -> None)."""
    if shared is None:
        return None
    ptr = lambda key: _ptr(shared.get(key)).value if shared.get(key) is not None else None
    return SharedExpert(ptr("W1"), ptr("b1"), ptr("W3"), ptr("W2"), ptr("b2"))


def moe_shared_ffn(cfg: MoeConfig, x: torch.Tensor, shared: Dict[str, Optional[torch.Tensor]],
                   ws: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """y_shared [N, d_model] = Shared(x) (weights W1, W2 and W3 / b1 / b2 as the activation needs)."""
    dev = x.device
    ws = ws if ws is not None else workspace(cfg, dev)
    y_shared = torch.empty((cfg.N, cfg.d_model), dtype=cfg.torch_dtype, device=dev)
    sh = _shared_struct(shared)
    rc = library().moe_shared_ffn(ctypes.byref(cfg), _ptr(x), ctypes.byref(sh), _ptr(y_shared), _ptr(status),
                                  _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_shared_ffn")
    return y_shared


def moe_combine_shared(cfg: MoeConfig, y_sorted: torch.Tensor, topk_w: torch.Tensor, inv_perm: torch.Tensor,
                       y_shared: Optional[torch.Tensor], stream=None) -> torch.Tensor:
    y = torch.empty((cfg.N, cfg.d_model), dtype=cfg.torch_dtype, device=y_sorted.device)
    rc = library().moe_combine_shared(ctypes.byref(cfg), _ptr(y_sorted), _ptr(topk_w), _ptr(inv_perm),
                                      _ptr(y_shared), _ptr(y), _stream(stream))
    _check(rc, "moe_combine_shared")
    return y


def moe_router_z_loss(cfg: MoeConfig, x: torch.Tensor, W_g: torch.Tensor, ws: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """Router z-loss [1] f32: mean over tokens of (logsumexp of the router logits)^2."""
    dev = x.device
    ws = ws if ws is not None else workspace(cfg, dev)
    z = torch.empty(1, dtype=torch.float32, device=dev)
    rc = library().moe_router_z_loss(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(z), None, _ptr(ws), ws.numel(),
                                     _stream(stream))
    _check(rc, "moe_router_z_loss")
    return z


def moe_aux_loss(cfg: MoeConfig, probs: torch.Tensor, topk_ids: torch.Tensor, gamma: float = 0.0,
                 b_e: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Returns (aux [1] f32, counts [E] int32, status [1] int32); updates b_e in place if gamma > 0."""
    dev = probs.device
    ws = ws if ws is not None else workspace(cfg, dev)
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = library().moe_aux_loss(ctypes.byref(cfg), _ptr(probs), _ptr(topk_ids), _ptr(aux), _ptr(counts),
                                float(gamma), _ptr(b_e), _ptr(status), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_aux_loss")
    return aux, counts, status


def moe_backward(cfg: MoeConfig, x: torch.Tensor, W_g: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor,
                 dy: torch.Tensor, W3: Optional[torch.Tensor] = None, b1: Optional[torch.Tensor] = None,
                 b2: Optional[torch.Tensor] = None, b_e: Optional[torch.Tensor] = None,
                 shared: Optional[Dict[str, Optional[torch.Tensor]]] = None, aux_coef: float = 0.0,
                 z_coef: float = 0.0, ws: Optional[torch.Tensor] = None,
                 out: Optional[Dict[str, torch.Tensor]] = None, stream=None) -> Dict[str, torch.Tensor]:
    """fp32 gradients of <dy, y> + aux_coef L_aux + z_coef L_z (moe_backward): dx, dW_g, dW1, dW2 and, as
    the layer has them, db1, dW3, db2 and the shared expert's dWs1, dbs1, dWs3, dWs2, dbs2; plus status."""
    dev = x.device
    if ws is None:
        n = int(library().moe_backward_workspace_size(ctypes.byref(cfg)))
        if n == 0:
            raise MoeError(1, "moe_backward_workspace_size")
        raw = torch.empty(n + 256, dtype=torch.uint8, device=dev)
        off = (-raw.data_ptr()) % 256
        ws = raw[off:off + n]
    f32 = dict(dtype=torch.float32, device=dev)
    N, d, F, E, Fs = cfg.N, cfg.d_model, cfg.d_ff, cfg.E, cfg.d_ff_shared
    if out is None:
        out = {"dx": torch.empty((N, d), **f32), "dW_g": torch.empty((E, d), **f32),
               "dW1": torch.empty((E, F, d), **f32), "dW2": torch.empty((E, d, F), **f32),
               "db1": torch.empty((E, F), **f32) if b1 is not None else None,
               "dW3": torch.empty((E, F, d), **f32) if W3 is not None else None,
               "db2": torch.empty((E, d), **f32) if b2 is not None else None}
        if shared is not None:
            out.update({"dWs1": torch.empty((Fs, d), **f32), "dWs2": torch.empty((d, Fs), **f32),
                        "dWs3": torch.empty((Fs, d), **f32) if shared.get("W3") is not None else None,
                        "dbs1": torch.empty(Fs, **f32) if shared.get("b1") is not None else None,
                        "dbs2": torch.empty(d, **f32) if shared.get("b2") is not None else None})
        out["status"] = torch.zeros(1, dtype=torch.int32, device=dev)
    g = MoeGrads(*[(_ptr(out.get(k)).value if out.get(k) is not None else None) for k, _ in MoeGrads._fields_])
    sh = _shared_struct(shared)
    rc = library().moe_backward(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(b_e), _ptr(W1), _ptr(b1), _ptr(W3),
                                _ptr(W2), _ptr(b2), ctypes.byref(sh) if sh else None, _ptr(dy), float(aux_coef),
                                float(z_coef), ctypes.byref(g), _ptr(out["status"]), _ptr(ws), ws.numel(),
                                _stream(stream))
    _check(rc, "moe_backward")
    return out


def moe_selftest_wait_timeout(stream=None) -> int:
    """Runs the library's bounded device wait on a barrier nothing arrives at
    and returns the status word it leaves (5, MOE_ERR_TIMEOUT); synchronises."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = library().moe_selftest_wait_timeout(_ptr(st), _stream(stream))
    _check(rc, "moe_selftest_wait_timeout")
    torch.cuda.synchronize()
    return int(st[0])


class StageEvents:
    """CUDA events that moe_forward records at stage boundaries.

    ``which`` selects the boundaries (0 .. MOE_NUM_STAGES; default all); the
    others are passed as NULL and not recorded.  An event between two of the
    library's kernels stops the second from being scheduled early, so timing
    loops record only the boundaries they need.
    """

    def __init__(self, which: Optional[Sequence[int]] = None):
        which = range(NUM_STAGES + 1) if which is None else which
        self.events = [torch.cuda.Event(enable_timing=True) if i in which else None
                       for i in range(NUM_STAGES + 1)]
        for e in self.events:           # materialise the CUDA event handles
            if e is not None:
                e.record()
        self._arr = (ctypes.c_void_p * (NUM_STAGES + 1))(
            *[e.cuda_event if e is not None else None for e in self.events])

    @property
    def pointer(self):
        return ctypes.cast(self._arr, ctypes.c_void_p)

    def elapsed_ms(self) -> Dict[str, float]:
        """Per-stage milliseconds of the last recorded forward (synchronises);
        only stages whose two boundaries were recorded."""
        last = [e for e in self.events if e is not None][-1]
        last.synchronize()
        return {STAGE_NAMES[i]: self.events[i].elapsed_time(self.events[i + 1]) for i in range(NUM_STAGES)
                if self.events[i] is not None and self.events[i + 1] is not None}


def moe_forward(cfg: MoeConfig, x: torch.Tensor, W_g: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor,
                W3: Optional[torch.Tensor] = None, b1: Optional[torch.Tensor] = None,
                b2: Optional[torch.Tensor] = None, b_e: Optional[torch.Tensor] = None, gamma: float = 0.0,
                ws: Optional[torch.Tensor] = None, out: Optional[Dict[str, torch.Tensor]] = None,
                stage_events: Optional[StageEvents] = None, stream=None,
                shared: Optional[Dict[str, Optional[torch.Tensor]]] = None,
                z_loss: bool = False) -> Dict[str, torch.Tensor]:
    """The whole layer: y, topk_ids, topk_w, counts, aux (Switch loss), z (z-loss), status.

    b_e (sigmoid router) selects only; with gamma > 0 it is moved in place by one
    sign-rule step after the selection.  ``out`` may hold preallocated outputs.
    ``shared`` (weights W1, W2, W3 / b1 / b2 of width cfg.d_ff_shared) adds the
    shared expert; ``z_loss`` fills out["z"] with the router z-loss.  Either
    goes through moe_forward_ex, otherwise moe_forward.
    """
    dev = x.device
    ws = ws if ws is not None else workspace(cfg, dev)
    if out is None:
        out = forward_outputs(cfg, dev)
    events = stage_events.pointer if stage_events else None
    if shared is None and not z_loss:
        rc = library().moe_forward(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(b_e), float(gamma), _ptr(W1),
                                   _ptr(b1), _ptr(W3), _ptr(W2), _ptr(b2), _ptr(out["y"]), _ptr(out["topk_ids"]),
                                   _ptr(out["topk_w"]), _ptr(out["counts"]), _ptr(out["aux"]),
                                   _ptr(out["status"]), _ptr(ws), ws.numel(), events, _stream(stream))
        _check(rc, "moe_forward")
        return out
    sh = _shared_struct(shared)
    rc = library().moe_forward_ex(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(b_e), float(gamma), _ptr(W1),
                                  _ptr(b1), _ptr(W3), _ptr(W2), _ptr(b2), ctypes.byref(sh) if sh else None,
                                  _ptr(out["y"]), _ptr(out["topk_ids"]), _ptr(out["topk_w"]), _ptr(out["counts"]),
                                  _ptr(out["aux"]), _ptr(out["z"]) if z_loss else None, _ptr(out["status"]),
                                  _ptr(ws), ws.numel(), events, _stream(stream))
    _check(rc, "moe_forward_ex")
    return out


class GraphPolicy:
    """Which steady-state calls of HostPipeline replay a CUDA graph.

    ``decide(key)`` returns "replay" for a key that has a graph, "capture"
    for a key met once before while fewer than ``max_graphs`` graphs exist
    (the caller then stores it with ``stored(key, graph)``), and "direct"
    otherwise; a "direct" key is remembered for its next call, at most
    ``max_seen`` of them (the memory is cleared when full)."""

    def __init__(self, max_graphs: int = 8, max_seen: int = 256):
        self.max_graphs = max_graphs
        self.max_seen = max_seen
        self.graphs = {}
        self.seen = set()

    def decide(self, key) -> str:
        if key in self.graphs:
            return "replay"
        if key in self.seen and len(self.graphs) < self.max_graphs:
            return "capture"
        if len(self.seen) >= self.max_seen:
            self.seen.clear()
        self.seen.add(key)
        return "direct"

    def stored(self, key, graph) -> None:
        self.graphs[key] = graph


class HostPipeline:
    """moe_forward over batches that live in pinned host memory.

    Each call of ``step(x_host, y_host, aux_host)`` hands over one batch: its
    upload, the layer and the download of y (and the Switch loss) run on the
    device while later calls proceed.  Uploads and downloads use two copy
    streams of their own and two device buffers of each kind, so one batch's
    upload and another's download overlap a third batch's forward.

    ``graphs=True`` (the default) software-pipelines the calls: call i
    enqueues the upload of batch i, the forward of batch i-1 and the download
    of batch i-2 as three branches of one piece of work (the first two calls
    fill the pipeline).  A parity and set of host buffers met a second time
    gets a CUDA graph of that work, replayed with one launch (at most
    ``GraphPolicy.max_graphs`` graphs); other calls enqueue the same work
    directly.  Batch i's outputs are on the
    host once call i+2 has completed on the device, or after ``flush()``.
    ``graphs=False`` enqueues each batch's upload, forward and download in its
    own call.  ``flush()`` enqueues the work still owed (without waiting);
    ``finish()`` flushes and waits for the last download.  A host buffer must
    stay untouched until its copy has run.  Only torch copies, CUDA events
    and graph launches are added around the library call; the layer is
    ``moe_forward``.
    """

    def __init__(self, cfg: MoeConfig, weights: Dict[str, Optional[torch.Tensor]], gamma: float = 0.0,
                 device=None, graphs: bool = True):
        self.cfg = cfg
        self.w = weights
        self.gamma = gamma
        self.graphs = graphs
        dev = torch.device(device or "cuda")
        self.compute = torch.cuda.current_stream(dev)
        self.upload = torch.cuda.Stream(dev)
        self.download = torch.cuda.Stream(dev)
        self.ws = workspace(cfg, dev)
        self.x = [torch.empty((cfg.N, cfg.d_model), dtype=cfg.torch_dtype, device=dev) for _ in range(2)]
        self.out = [forward_outputs(cfg, dev) for _ in range(2)]
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]
        self.i = 0
        self._owed = []      # (batch, y_host, aux_host) uploaded, not yet downloaded, oldest first
        self.policy = GraphPolicy()  # which calls replay a graph

    def _forward(self, b: int, stream):
        w = self.w
        moe_forward(self.cfg, self.x[b], w["W_g"], w["W1"], w["W2"], W3=w.get("W3"), b1=w.get("b1"),
                    b2=w.get("b2"), b_e=w.get("b_e"), gamma=self.gamma, ws=self.ws, out=self.out[b],
                    stream=stream, shared=w.get("shared"))

    def _upload(self, b: int, x_host: torch.Tensor):
        with torch.cuda.stream(self.upload):
            self.upload.wait_event(self.computed[b])  # x buffer b was last read by the forward two batches ago
            self.x[b].copy_(x_host, non_blocking=True)
            self.uploaded[b].record(self.upload)

    def _run(self, b: int):
        self.compute.wait_event(self.uploaded[b])
        self.compute.wait_event(self.downloaded[b])  # outputs two batches ago are on the host
        self._forward(b, self.compute)
        self.computed[b].record(self.compute)

    def _download(self, b: int, y_host: torch.Tensor, aux_host: Optional[torch.Tensor]):
        with torch.cuda.stream(self.download):
            self.download.wait_event(self.computed[b])
            y_host.copy_(self.out[b]["y"], non_blocking=True)
            if aux_host is not None:
                aux_host.copy_(self.out[b]["aux"], non_blocking=True)
            self.downloaded[b].record(self.download)

    def _steady(self, p: int, x_host, y_host, aux_host, cap):
        """Upload into x[p], forward of x[1-p], download of out[p]: two
        branches forked from stream `cap`, which runs the forward and joins
        them (captured into a graph, or enqueued as it stands)."""
        fork = torch.cuda.Event()
        fork.record(cap)
        self.upload.wait_event(fork)
        with torch.cuda.stream(self.upload):
            self.x[p].copy_(x_host, non_blocking=True)
        self.download.wait_event(fork)
        with torch.cuda.stream(self.download):
            y_host.copy_(self.out[p]["y"], non_blocking=True)
            if aux_host is not None:
                aux_host.copy_(self.out[p]["aux"], non_blocking=True)
        self._forward(1 - p, cap)
        cap.wait_stream(self.upload)
        cap.wait_stream(self.download)

    def _steady_step(self, p: int, x_host, y_host, aux_host):
        """The steady-state call: a graph for a parity and set of host buffers
        met before (captured on its second use; GraphPolicy), so that buffers
        a caller reuses cost one launch; otherwise the same work enqueued
        directly, so that fresh buffers on every call cost no capture."""
        key = (p, x_host.data_ptr(), y_host.data_ptr(), aux_host.data_ptr() if aux_host is not None else 0)
        how = self.policy.decide(key)
        if how == "capture":
            torch.cuda.synchronize()  # no earlier work pending on the streams the capture joins
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                self._steady(p, x_host, y_host, aux_host, torch.cuda.current_stream())
            self.policy.stored(key, g)
        if how != "direct":
            self.policy.graphs[key].replay()
            return
        self._steady(p, x_host, y_host, aux_host, self.compute)

    def step(self, x_host: torch.Tensor, y_host: torch.Tensor, aux_host: Optional[torch.Tensor] = None):
        b = self.i & 1
        if not self.graphs:
            self._upload(b, x_host)
            self._run(b)
            self._download(b, y_host, aux_host)
            self.i += 1
            return
        self._owed.append((b, y_host, aux_host))
        if self.i < 2:  # filling the pipeline: upload (and the first forward) eagerly
            self._upload(b, x_host)
            if self.i == 1:
                self._run(0)
            self.i += 1
            return
        # steady state: batch i up, batch i-1 through the layer, batch i-2 down
        _, y_old, aux_old = self._owed.pop(0)
        self.compute.wait_stream(self.upload)
        self.compute.wait_stream(self.download)
        self._steady_step(b, x_host, y_old, aux_old)
        self.computed[1 - b].record(self.compute)
        self.i += 1

    def flush(self):
        """Enqueues the forward and the downloads still owed (does not wait)."""
        if not self.graphs or not self._owed:
            return
        if self.i >= 2:
            # the graph launches ran on the compute stream: later copies follow them
            self.upload.wait_stream(self.compute)
            self.download.wait_stream(self.compute)
            self.uploaded[(self.i - 1) & 1].record(self.compute)
            self.downloaded[0].record(self.compute)
            self.downloaded[1].record(self.compute)
        last = self._owed[-1][0]
        self._run(last)  # the last uploaded batch
        for b, y_host, aux_host in self._owed:
            self._download(b, y_host, aux_host)
        self._owed = []
        self.i = 0  # the next call starts a new pipeline

    def finish(self):
        self.flush()
        for e in self.downloaded:
            e.synchronize()


def moe_forward_partials(cfg: MoeConfig, x: torch.Tensor, W_g: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor,
                         W3: Optional[torch.Tensor] = None, b1: Optional[torch.Tensor] = None,
                         b2: Optional[torch.Tensor] = None, b_e: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None, out: Optional[Dict[str, torch.Tensor]] = None,
                         stream=None, shared: Optional[Dict[str, Optional[torch.Tensor]]] = None,
                         z_loss: bool = False) -> Dict[str, torch.Tensor]:
    """One data-parallel rank's forward: y, topk_ids, topk_w, status, (z) and
    the Switch-loss partials counts [E] int32 and psum [E] float64 (sum over
    this call's tokens of softmax(z_n)).  b_e selects only and is not moved."""
    dev = x.device
    ws = ws if ws is not None else workspace(cfg, dev)
    if out is None:
        out = forward_outputs(cfg, dev)
    if "psum" not in out:
        out["psum"] = torch.empty(cfg.E, dtype=torch.float64, device=dev)
    sh = _shared_struct(shared)
    rc = library().moe_forward_partials(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(b_e), _ptr(W1), _ptr(b1),
                                        _ptr(W3), _ptr(W2), _ptr(b2), ctypes.byref(sh) if sh else None,
                                        _ptr(out["y"]), _ptr(out["topk_ids"]), _ptr(out["topk_w"]),
                                        _ptr(out["counts"]), _ptr(out["psum"]), _ptr(out["z"]) if z_loss else None,
                                        _ptr(out["status"]), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_forward_partials")
    return out


def moe_aux_from_partials(E: int, k: int, counts: torch.Tensor, psum: torch.Tensor, gamma: float = 0.0,
                          b_e: Optional[torch.Tensor] = None, aux: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Whole-batch Switch loss [1] f32 from summed partials (counts int32 [E],
    psum float64 [E]); with gamma > 0 moves b_e in place by the sign rule on
    the whole batch's load."""
    if counts.dtype != torch.int32 or psum.dtype != torch.float64:
        raise ValueError("moe_aux_from_partials: counts int32 [E] and psum float64 [E]")
    aux = aux if aux is not None else torch.empty(1, dtype=torch.float32, device=counts.device)
    rc = library().moe_aux_from_partials(int(E), int(k), _ptr(counts), _ptr(psum), _ptr(aux), float(gamma),
                                         _ptr(b_e), _stream(stream))
    _check(rc, "moe_aux_from_partials")
    return aux


def forward_outputs(cfg: MoeConfig, device) -> Dict[str, torch.Tensor]:
    return {
        "y": torch.empty((cfg.N, cfg.d_model), dtype=cfg.torch_dtype, device=device),
        "topk_ids": torch.empty((cfg.N, cfg.k), dtype=torch.int32, device=device),
        "topk_w": torch.empty((cfg.N, cfg.k), dtype=torch.float32, device=device),
        "counts": torch.empty(cfg.E, dtype=torch.int32, device=device),
        "aux": torch.empty(1, dtype=torch.float32, device=device),
        "z": torch.empty(1, dtype=torch.float32, device=device),
        "status": torch.zeros(1, dtype=torch.int32, device=device),
    }


__all__ = ["MoeConfig", "SharedExpert", "MoeError", "make_config", "library", "workspace", "moe_workspace_size",
           "moe_route", "moe_dispatch", "moe_dispatch_noalloc", "moe_expert_ffn", "moe_combine", "moe_aux_loss",
           "moe_forward", "moe_shared_ffn", "moe_combine_shared", "moe_router_z_loss", "moe_backward",
           "moe_forward_partials", "moe_aux_from_partials",
           "MoeGrads", "forward_outputs",
           "StageEvents", "HostPipeline", "EXPORTS", "LIB_PATH"]
