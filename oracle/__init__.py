"""fp64 CPU oracle of the dropless MoE layer forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and it
never calls the CUDA library: the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, single thread); this
module only converts numpy arrays to ``float64``/``int32`` and calls it.  The
per-token loop used for sampled tokens of a full-size workload
(``forward_tokens``) also lives here, in plain Python over the C expert FFN.

Sources: "Mixture of Experts: routing, sorted dispatch, Switch aux loss,
aux-free bias" (course module) sec. 2.1-2.5 and sec. 4; "nano-moe" (expert MLP
with exact GELU and biases).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

SOFTMAX_TOPK, TOPK_SOFTMAX, SIGMOID = 0, 1, 2
GELU, SWIGLU = 0, 1
ROUTERS = {"softmax_topk": SOFTMAX_TOPK, "topk_softmax": TOPK_SOFTMAX, "sigmoid": SIGMOID}
ACTS = {"gelu": GELU, "swiglu": SWIGLU}

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with gcc into a shared library (no BLAS, no OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *GCC_FLAGS, src, "-lm", "-o", tmp])
        os.replace(tmp, out)
    return out


_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (building first if needed) an oracle shared library and type it."""
    lib = ctypes.CDLL(path or build())
    i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_route.argtypes = [i64, i32, i32, i32, i32, i32, f64, _dp, _dp, _dp, _ip, _u8p,
                                 _ip, _dp, _dp, _dp, _dp]
    lib.oracle_route.restype = i32
    lib.oracle_expert_ffn.argtypes = [i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
    lib.oracle_expert_ffn.restype = None
    lib.oracle_dense_forward.argtypes = [i64, i32, i32, i32, i32, i32, _dp, _dp, _dp, _dp, _dp,
                                         _dp, _ip, _dp, _dp]
    lib.oracle_dense_forward.restype = i32
    lib.oracle_dispatch.argtypes = [i64, i32, i32, _ip, _ip, _ip, _ip, _ip]
    lib.oracle_dispatch.restype = i32
    lib.oracle_combine.argtypes = [i64, i32, i32, _dp, _dp, _ip, _dp]
    lib.oracle_combine.restype = None
    lib.oracle_sorted_forward.argtypes = [i64, i32, i32, i32, i32, i32, _dp, _dp, _dp, _dp, _dp,
                                          _dp, _ip, _dp, _dp, _dp, _dp]
    lib.oracle_sorted_forward.restype = i32
    lib.oracle_aux_loss.argtypes = [i64, i32, i32, _dp, _ip, _ip]
    lib.oracle_aux_loss.restype = f64
    lib.oracle_aux_from_partials.argtypes = [i32, i32, _ip, _dp]
    lib.oracle_aux_from_partials.restype = f64
    lib.oracle_bias_update.argtypes = [i64, i32, i32, _ip, f64, _dp]
    lib.oracle_bias_update.restype = None
    lib.oracle_z_loss.argtypes = [i64, i32, _dp]
    lib.oracle_z_loss.restype = f64
    lib.oracle_shared_add.argtypes = [i64, i32, i32, i32, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
    lib.oracle_shared_add.restype = i32
    lib.oracle_backward.argtypes = [i64, i32, i32, i32, i32, i32, i32, f64, i32, _dp, _dp, _dp, _dp, _dp, _dp,
                                    _dp, _dp, i32, _dp, _dp, _dp, _dp, _dp, _dp, f64, f64, _ip, _u8p,
                                    _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
    lib.oracle_backward.restype = i32
    return lib


_default: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _default
    if _default is None:
        _default = load()
    return _default


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: Optional[np.ndarray], t):
    if a is None:
        return ctypes.cast(None, t)
    return a.ctypes.data_as(t)


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc == 1:
        raise OracleError(f"{what}: invalid argument")
    if rc == 2:
        raise OracleError(f"{what}: expert id out of range")
    if rc != 0:
        raise OracleError(f"{what}: error {rc}")


def route(x, Wg, k: int, router: str = "softmax_topk", norm_topk: bool = True,
          routed_scaling: float = 1.0, b_sel=None, forced_ids=None, forced=None,
          L: Optional[ctypes.CDLL] = None) -> Dict[str, np.ndarray]:
    """Route N tokens: returns ids [N,k], w [N,k], probs [N,E], logits [N,E], margin [N]."""
    L = L or lib()
    x = _f64(x)
    Wg = _f64(Wg)
    N, d = x.shape
    E = Wg.shape[0]
    assert Wg.shape == (E, d)
    ids = np.zeros((N, k), np.int32)
    w = np.zeros((N, k), np.float64)
    probs = np.zeros((N, E), np.float64)
    logits = np.zeros((N, E), np.float64)
    margin = np.zeros((N,), np.float64)
    b = None if b_sel is None else _f64(b_sel)
    fi = None if forced_ids is None else _i32(forced_ids)
    fm = None if forced is None else np.ascontiguousarray(np.asarray(forced, dtype=np.uint8))
    rc = L.oracle_route(N, d, E, k, ROUTERS[router], int(bool(norm_topk)), float(routed_scaling),
                        _p(x, _dp), _p(Wg, _dp), _p(b, _dp), _p(fi, _ip), _p(fm, _u8p),
                        _p(ids, _ip), _p(w, _dp), _p(probs, _dp), _p(logits, _dp), _p(margin, _dp))
    _check(rc, "oracle_route")
    return {"ids": ids, "w": w, "probs": probs, "logits": logits, "margin": margin}


def expert_ffn(x_row, W1e, W2e, act: str = "gelu", b1e=None, W3e=None, b2e=None,
               L: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """One expert on one token; W1e/W3e are [F, d], W2e is [d, F]."""
    L = L or lib()
    x_row = _f64(x_row)
    W1e = _f64(W1e)
    W2e = _f64(W2e)
    F, d = W1e.shape
    out = np.zeros(d, np.float64)
    h = np.zeros(F, np.float64)
    b1 = None if b1e is None else _f64(b1e)
    W3 = None if W3e is None else _f64(W3e)
    b2 = None if b2e is None else _f64(b2e)
    L.oracle_expert_ffn(d, F, ACTS[act], _p(x_row, _dp), _p(W1e, _dp), _p(b1, _dp), _p(W3, _dp),
                        _p(W2e, _dp), _p(b2, _dp), _p(h, _dp), _p(out, _dp))
    return out


def _weights(W1, W2, W3, b1, b2):
    return (_f64(W1), _f64(W2), None if W3 is None else _f64(W3),
            None if b1 is None else _f64(b1), None if b2 is None else _f64(b2))


def dense_forward(x, ids, w, W1, W2, act="gelu", W3=None, b1=None, b2=None,
                  L: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """Per-token loop y_n = sum_j w_nj Expert_{ids[n,j]}(x_n)."""
    L = L or lib()
    x = _f64(x)
    ids = _i32(ids)
    w = _f64(w)
    W1, W2, W3, b1, b2 = _weights(W1, W2, W3, b1, b2)
    N, d = x.shape
    E, F, _ = W1.shape
    k = ids.shape[1]
    y = np.zeros((N, d), np.float64)
    rc = L.oracle_dense_forward(N, d, F, E, k, ACTS[act], _p(x, _dp), _p(W1, _dp), _p(b1, _dp),
                                _p(W3, _dp), _p(W2, _dp), _p(b2, _dp), _p(ids, _ip), _p(w, _dp),
                                _p(y, _dp))
    _check(rc, "oracle_dense_forward")
    return y


def dispatch(ids, E: int, L: Optional[ctypes.CDLL] = None) -> Dict[str, np.ndarray]:
    """Sorted dispatch of ids [N,k]: perm, inv_perm, offsets [E+1], counts [E]."""
    L = L or lib()
    ids = _i32(ids)
    N, k = ids.shape
    perm = np.zeros(N * k, np.int32)
    inv = np.zeros(N * k, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    counts = np.zeros(E, np.int32)
    rc = L.oracle_dispatch(N, E, k, _p(ids, _ip), _p(perm, _ip), _p(inv, _ip), _p(offsets, _ip),
                           _p(counts, _ip))
    _check(rc, "oracle_dispatch")
    return {"perm": perm, "inv_perm": inv, "offsets": offsets, "counts": counts}


def combine(y_sorted, w, inv_perm, L: Optional[ctypes.CDLL] = None) -> np.ndarray:
    L = L or lib()
    y_sorted = _f64(y_sorted)
    w = _f64(w)
    inv = _i32(inv_perm)
    N, k = w.shape
    d = y_sorted.shape[1]
    y = np.zeros((N, d), np.float64)
    L.oracle_combine(N, d, k, _p(y_sorted, _dp), _p(w, _dp), _p(inv, _ip), _p(y, _dp))
    return y


def sorted_forward(x, ids, w, W1, W2, act="gelu", W3=None, b1=None, b2=None,
                   L: Optional[ctypes.CDLL] = None) -> Dict[str, np.ndarray]:
    """Dispatch, per-expert slices, combine; returns y, x_sorted, y_sorted."""
    L = L or lib()
    x = _f64(x)
    ids = _i32(ids)
    w = _f64(w)
    W1, W2, W3, b1, b2 = _weights(W1, W2, W3, b1, b2)
    N, d = x.shape
    E, F, _ = W1.shape
    k = ids.shape[1]
    y = np.zeros((N, d), np.float64)
    xs = np.zeros((N * k, d), np.float64)
    ys = np.zeros((N * k, d), np.float64)
    rc = L.oracle_sorted_forward(N, d, F, E, k, ACTS[act], _p(x, _dp), _p(W1, _dp), _p(b1, _dp),
                                 _p(W3, _dp), _p(W2, _dp), _p(b2, _dp), _p(ids, _ip), _p(w, _dp),
                                 _p(y, _dp), _p(xs, _dp), _p(ys, _dp))
    _check(rc, "oracle_sorted_forward")
    return {"y": y, "x_sorted": xs, "y_sorted": ys}


def aux_loss(probs, ids, L: Optional[ctypes.CDLL] = None) -> Tuple[float, np.ndarray]:
    """Switch loss E sum_e f_e P_e and the assignment counts."""
    L = L or lib()
    probs = _f64(probs)
    ids = _i32(ids)
    N, E = probs.shape
    k = ids.shape[1]
    counts = np.zeros(E, np.int32)
    val = L.oracle_aux_loss(N, E, k, _p(probs, _dp), _p(ids, _ip), _p(counts, _ip))
    return float(val), counts


def aux_from_partials(counts, psum, k: int, L: Optional[ctypes.CDLL] = None) -> float:
    """Switch loss of a whole batch from its parts' summed counts [E] and
    probability sums [E] (N = sum(counts) / k)."""
    L = L or lib()
    counts = _i32(counts)
    psum = _f64(psum)
    E = counts.shape[0]
    assert psum.shape == (E,)
    return float(L.oracle_aux_from_partials(E, int(k), _p(counts, _ip), _p(psum, _dp)))


def bias_update(b, counts, N: int, k: int, gamma: float,
                L: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """Return b after one sign-rule step (the input is not modified)."""
    L = L or lib()
    out = _f64(b).copy()
    counts = _i32(counts)
    L.oracle_bias_update(N, out.shape[0], k, _p(counts, _ip), float(gamma), _p(out, _dp))
    return out


def z_loss(logits, L: Optional[ctypes.CDLL] = None) -> float:
    """Router z-loss: mean over tokens of (logsumexp of the logits)^2."""
    L = L or lib()
    z = _f64(logits)
    N, E = z.shape
    return float(L.oracle_z_loss(N, E, _p(z, _dp)))


def shared_add(y, x, Ws1, Ws2, act="swiglu", Ws3=None, bs1=None, bs2=None,
               L: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """Return y + Shared(x) (row by row); Ws1/Ws3 [Fs,d], Ws2 [d,Fs]."""
    L = L or lib()
    out = _f64(y).copy()
    x = _f64(x)
    Ws1 = _f64(Ws1)
    Ws2 = _f64(Ws2)
    Ws3 = None if Ws3 is None else _f64(Ws3)
    bs1 = None if bs1 is None else _f64(bs1)
    bs2 = None if bs2 is None else _f64(bs2)
    N, d = x.shape
    Fs = Ws1.shape[0]
    rc = L.oracle_shared_add(N, d, Fs, ACTS[act], _p(x, _dp), _p(Ws1, _dp), _p(bs1, _dp), _p(Ws3, _dp),
                             _p(Ws2, _dp), _p(bs2, _dp), _p(out, _dp))
    _check(rc, "oracle_shared_add")
    return out


def forward_tokens(x_rows, ids, w, expert_weights: Callable[[int], Dict[str, Optional[np.ndarray]]],
                   act: str, L: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """Per-token loop for a few sampled tokens of a large workload.

    x_rows [S, d], ids/w [S, k]; ``expert_weights(e)`` returns that expert's
    {"W1": [F,d], "W3": [F,d] or None, "W2": [d,F], "b1", "b2"} as arrays, so
    that the caller need only hold the experts the sample touches.  Same sum
    order as ``dense_forward``: zero, then + w_j * o_j for j = 0..k-1.
    """
    L = L or lib()
    x_rows = _f64(x_rows)
    ids = _i32(ids)
    w = _f64(w)
    S, d = x_rows.shape
    k = ids.shape[1]
    y = np.zeros((S, d), np.float64)
    by_expert: Dict[int, list] = {}
    for s in range(S):
        for j in range(k):
            by_expert.setdefault(int(ids[s, j]), []).append((s, j))
    outs: Dict[Tuple[int, int], np.ndarray] = {}
    for e in sorted(by_expert):
        ew = expert_weights(e)
        for (s, j) in by_expert[e]:
            outs[(s, j)] = expert_ffn(x_rows[s], ew["W1"], ew["W2"], act=act, b1e=ew.get("b1"),
                                      W3e=ew.get("W3"), b2e=ew.get("b2"), L=L)
    for s in range(S):
        for j in range(k):
            y[s] += w[s, j] * outs[(s, j)]
    return y


def backward(x, Wg, k: int, W1, W2, dy, router: str = "softmax_topk", norm_topk: bool = True,
             routed_scaling: float = 1.0, act: str = "gelu", W3=None, b1=None, b2=None, b_sel=None,
             shared: Optional[Dict[str, Optional[np.ndarray]]] = None, aux_coef: float = 0.0,
             z_coef: float = 0.0, forced_ids=None, forced=None,
             L: Optional[ctypes.CDLL] = None) -> Dict[str, np.ndarray]:
    """Gradients of <dy, y> + aux_coef L_aux + z_coef L_z: dx, dW_g, dW1, db1, dW3, dW2, db2 and, with a
    shared expert ({"W1","W2","W3"?,"b1"?,"b2"?}), dWs1, dbs1, dWs3, dWs2, dbs2."""
    L = L or lib()
    x, Wg, dy = _f64(x), _f64(Wg), _f64(dy)
    W1, W2, W3, b1, b2 = _weights(W1, W2, W3, b1, b2)
    N, d = x.shape
    E = Wg.shape[0]
    F = W1.shape[1]
    b_sel = None if b_sel is None else _f64(b_sel)
    sh = {kk: (None if v is None else _f64(v)) for kk, v in (shared or {}).items()}
    Fs = sh["W1"].shape[0] if sh else 0
    g = {"dx": np.zeros((N, d)), "dWg": np.zeros((E, d)), "dW1": np.zeros((E, F, d)),
         "db1": np.zeros((E, F)) if b1 is not None else None,
         "dW3": np.zeros((E, F, d)) if W3 is not None else None,
         "dW2": np.zeros((E, d, F)), "db2": np.zeros((E, d)) if b2 is not None else None}
    if Fs:
        g.update({"dWs1": np.zeros((Fs, d)), "dbs1": np.zeros(Fs) if sh.get("b1") is not None else None,
                  "dWs3": np.zeros((Fs, d)) if sh.get("W3") is not None else None,
                  "dWs2": np.zeros((d, Fs)), "dbs2": np.zeros(d) if sh.get("b2") is not None else None})
    fi = None if forced_ids is None else _i32(forced_ids)
    fm = None if forced is None else np.ascontiguousarray(np.asarray(forced, dtype=np.uint8))
    rc = L.oracle_backward(N, d, F, E, k, ROUTERS[router], int(bool(norm_topk)), float(routed_scaling), ACTS[act],
                           _p(x, _dp), _p(Wg, _dp), _p(b_sel, _dp), _p(W1, _dp), _p(b1, _dp), _p(W3, _dp),
                           _p(W2, _dp), _p(b2, _dp), Fs, _p(sh.get("W1"), _dp), _p(sh.get("b1"), _dp),
                           _p(sh.get("W3"), _dp), _p(sh.get("W2"), _dp), _p(sh.get("b2"), _dp), _p(dy, _dp),
                           float(aux_coef), float(z_coef), _p(fi, _ip), _p(fm, _u8p),
                           _p(g["dx"], _dp), _p(g["dWg"], _dp), _p(g["dW1"], _dp), _p(g["db1"], _dp),
                           _p(g["dW3"], _dp), _p(g["dW2"], _dp), _p(g["db2"], _dp), _p(g.get("dWs1"), _dp),
                           _p(g.get("dbs1"), _dp), _p(g.get("dWs3"), _dp), _p(g.get("dWs2"), _dp),
                           _p(g.get("dbs2"), _dp))
    _check(rc, "oracle_backward")
    return g
