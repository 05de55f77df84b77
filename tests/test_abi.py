"""The C ABI of libmoe.so on the CPU: exports, struct layout, validation.

No compute call is made here: every call below fails argument validation,
which returns before anything touches CUDA.
"""
import ctypes
import os
import re
import subprocess

import pytest

import mixture_experts_layer_53_b200 as M
from mixture_experts_layer_53_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")
BAD = ctypes.c_void_p(0x1001)  # never dereferenced: every call here fails validation first


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(M.EXPORTS), names
    out = subprocess.check_output(["nm", "-D", "--defined-only", M.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in names:
        assert name in exported, f"{name} declared in moe.h but not exported"
        assert hasattr(lib, name)
    assert all(e.startswith("moe_") for e in exported), sorted(e for e in exported if not e.startswith("moe_"))


def test_config_layout_matches_header(tmp_path):
    src = tmp_path / "probe.c"
    src.write_text("""
#include <stddef.h>
#include <stdio.h>
#include "moe.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(moe_config),
         offsetof(moe_config, N), offsetof(moe_config, d_model), offsetof(moe_config, d_ff),
         offsetof(moe_config, E), offsetof(moe_config, k), offsetof(moe_config, router),
         offsetof(moe_config, norm_topk), offsetof(moe_config, routed_scaling),
         offsetof(moe_config, act), offsetof(moe_config, dtype), offsetof(moe_config, d_ff_shared));
  printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(moe_shared_expert), offsetof(moe_shared_expert, W1),
         offsetof(moe_shared_expert, b1), offsetof(moe_shared_expert, W3), offsetof(moe_shared_expert, W2),
         offsetof(moe_shared_expert, b2));
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(moe_grads), offsetof(moe_grads, dx),
         offsetof(moe_grads, dW_g), offsetof(moe_grads, dW1), offsetof(moe_grads, db1), offsetof(moe_grads, dW3),
         offsetof(moe_grads, dW2), offsetof(moe_grads, db2), offsetof(moe_grads, dWs1), offsetof(moe_grads, dbs1),
         offsetof(moe_grads, dWs3), offsetof(moe_grads, dWs2), offsetof(moe_grads, dbs2));
  return 0;
}
""")
    exe = tmp_path / "probe"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    lines = subprocess.check_output([str(exe)], text=True).splitlines()
    assert len(lines) == 3
    for line, C in zip(lines, (M.MoeConfig, M.SharedExpert, M.MoeGrads)):
        got = [int(v) for v in line.split()]
        want = [ctypes.sizeof(C)] + [getattr(C, f).offset for f, _ in C._fields_]
        assert got == want, C.__name__


def test_status_strings_and_version(lib):
    for code in range(7):
        assert lib.moe_status_string(code)
    assert lib.moe_version() >= 100


def cfg(**kw):
    base = dict(N=64, d_model=64, d_ff=128, E=4, k=2, router="softmax_topk", act="gelu", dtype="f32")
    base.update(kw)
    return M.make_config(**base)


@pytest.mark.parametrize("bad,code", [
    (dict(k=5), 1), (dict(k=0), 1), (dict(E=0), 1), (dict(N=-1), 1), (dict(d_model=0), 1),
    (dict(E=257, k=2), 2), (dict(E=32, k=17), 2), (dict(d_model=60), 2), (dict(d_ff=100), 2),
    (dict(N=2 ** 31, k=2), 2), (dict(d_ff_shared=-8), 1), (dict(d_ff_shared=12), 2),
])
def test_invalid_configs(lib, bad, code):
    c = cfg(**bad)
    assert lib.moe_workspace_size(ctypes.byref(c)) == 0
    rc = lib.moe_route(ctypes.byref(c), BAD, BAD, None, BAD, BAD, None, None, 0, None)
    assert rc == code


def test_invalid_enums(lib):
    for field, value in (("router", 3), ("act", 2), ("dtype", 5), ("norm_topk", 2)):
        c = cfg()
        setattr(c, field, value)
        assert lib.moe_workspace_size(ctypes.byref(c)) == 0
        assert lib.moe_combine(ctypes.byref(c), BAD, BAD, BAD, BAD, None) == 1
    c = cfg()
    c.routed_scaling = float("nan")
    assert lib.moe_workspace_size(ctypes.byref(c)) == 0


def test_null_and_misaligned_pointers(lib):
    c = cfg()
    assert lib.moe_route(ctypes.byref(c), None, BAD, None, BAD, BAD, None, None, 0, None) == 1
    assert lib.moe_route(ctypes.byref(c), ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2008), None,
                         ctypes.c_void_p(0x3000), ctypes.c_void_p(0x4000), None, None, 0, None) == 1
    assert lib.moe_combine(ctypes.byref(c), None, BAD, BAD, BAD, None) == 1
    assert lib.moe_route(None, BAD, BAD, None, BAD, BAD, None, None, 0, None) == 1


def test_bias_only_for_sigmoid_router(lib):
    c = cfg()
    a = ctypes.c_void_p(0x10000)
    assert lib.moe_route(ctypes.byref(c), a, a, a, a, a, None, None, 0, None) == 1
    rc = lib.moe_forward(ctypes.byref(c), a, a, a, ctypes.c_float(0.0), a, a, None, a, a, a, None, None, None,
                         None, None, a, ctypes.c_size_t(1 << 40), None, None)
    assert rc == 1


def test_swiglu_rejects_hidden_bias_and_needs_W3(lib):
    c = cfg(act="swiglu")
    a = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    # b1 given with SwiGLU
    assert lib.moe_expert_ffn(ctypes.byref(c), a, a, a, a, a, a, None, a, None, ws, ctypes.c_size_t(1 << 40),
                              None) == 1
    # W3 missing
    assert lib.moe_expert_ffn(ctypes.byref(c), a, a, a, None, None, a, None, a, None, ws,
                              ctypes.c_size_t(1 << 40), None) == 1


def test_workspace_checks(lib):
    c = cfg()
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert need > 0
    a = ctypes.c_void_p(0x10000)
    ws_misaligned = ctypes.c_void_p(0x100010)
    ws = ctypes.c_void_p(0x100000)
    assert lib.moe_dispatch(ctypes.byref(c), None, a, None, None, a, a, a, None, None, ctypes.c_size_t(need),
                            None) == 4
    assert lib.moe_dispatch(ctypes.byref(c), None, a, None, None, a, a, a, None, ws_misaligned,
                            ctypes.c_size_t(need), None) == 4
    assert lib.moe_dispatch(ctypes.byref(c), None, a, None, None, a, a, a, None, ws, ctypes.c_size_t(need - 1),
                            None) == 4
    # gamma must be finite and >= 0
    assert lib.moe_aux_loss(ctypes.byref(c), a, a, a, None, ctypes.c_float(-1.0), None, None, ws,
                            ctypes.c_size_t(need), None) == 1


def test_workspace_grows_with_tokens(lib):
    sizes = [lib.moe_workspace_size(ctypes.byref(cfg(N=n, dtype="bf16"))) for n in (0, 1, 64, 1000)]
    assert sizes[0] > 0 and sizes == sorted(sizes) and sizes[3] > sizes[2]
    # x_sorted + h + y_sorted dominate: N k (2 d + F) elements
    c = cfg(N=4096, d_model=4096, d_ff=14336, E=8, k=2, act="swiglu", dtype="bf16")
    n = lib.moe_workspace_size(ctypes.byref(c))
    assert n >= 4096 * 2 * (2 * 4096 + 14336) * 2


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        M.library(str(tmp_path / "libmoe.so"))


def test_shared_expert_needs_width_and_weights(lib):
    a = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    sh = M.SharedExpert(0x10000, None, None, 0x10000, None)
    c0, c1 = cfg(), cfg(d_ff_shared=64)
    # moe_forward has no slot for shared weights
    assert lib.moe_forward(ctypes.byref(c1), a, a, None, ctypes.c_float(0.0), a, None, None, a, None, a, None,
                           None, None, None, None, ws, big, None, None) == 1
    # weights without a width, a width without weights
    args = lambda c, shp: (ctypes.byref(c), a, a, None, ctypes.c_float(0.0), a, None, None, a, None, shp, a, None,
                           None, None, None, None, None, ws, big, None, None)
    assert lib.moe_forward_ex(*args(c0, ctypes.byref(sh))) == 1
    assert lib.moe_forward_ex(*args(c1, None)) == 1
    assert lib.moe_shared_ffn(ctypes.byref(c0), a, ctypes.byref(sh), a, None, ws, big, None) == 1
    assert lib.moe_shared_ffn(ctypes.byref(c1), a, None, a, None, ws, big, None) == 1
    # SwiGLU shared expert without W3
    c2 = cfg(act="swiglu", d_ff_shared=64)
    assert lib.moe_shared_ffn(ctypes.byref(c2), a, ctypes.byref(sh), a, None, ws, big, None) == 1
    # misaligned shared weight
    bad = M.SharedExpert(0x10008, None, None, 0x10000, None)
    assert lib.moe_shared_ffn(ctypes.byref(c1), a, ctypes.byref(bad), a, None, ws, big, None) == 1


def test_z_loss_validation(lib):
    a = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    c = cfg()
    assert lib.moe_router_z_loss(ctypes.byref(c), a, a, None, None, ws, big, None) == 1
    assert lib.moe_router_z_loss(ctypes.byref(c), a, None, a, None, ws, big, None) == 1
    assert lib.moe_router_z_loss(ctypes.byref(c), a, a, a, None, None, big, None) == 4
    assert lib.moe_combine_shared(ctypes.byref(c), a, a, a, ctypes.c_void_p(0x10004), a, None) == 1


def test_workspace_holds_the_shared_expert(lib):
    base = dict(N=1024, d_model=256, d_ff=128, E=8, k=2, dtype="bf16")
    n0 = lib.moe_workspace_size(ctypes.byref(cfg(**base)))
    n1 = lib.moe_workspace_size(ctypes.byref(cfg(**base, d_ff_shared=128)))
    n2 = lib.moe_workspace_size(ctypes.byref(cfg(**base, d_ff_shared=1024)))
    assert n1 - n0 >= 1024 * 256 * 2 - 256         # + y_shared [N, d] (an empty region still takes 256 B)
    assert n2 >= n1 + 1024 * (1024 - 2 * 128) * 2  # h grows to N * Fs once that exceeds N k F


def test_backward_validation(lib):
    a = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    c = cfg(act="swiglu")
    assert lib.moe_backward_workspace_size(ctypes.byref(c)) > lib.moe_workspace_size(ctypes.byref(c))
    full = M.MoeGrads(*([0x20000] * 12))
    no_dw3 = M.MoeGrads(0x20000, 0x20000, 0x20000, None, None, 0x20000, None, None, None, None, None, None)
    args = lambda g, dy=a, aux=0.0: (ctypes.byref(c), a, a, None, a, None, a, a, None, None, dy, ctypes.c_float(aux),
                                     ctypes.c_float(0.0), ctypes.byref(g) if g is not None else None, None, ws, big,
                                     None)
    assert lib.moe_backward(*args(no_dw3)) == 1          # SwiGLU needs dW3
    assert lib.moe_backward(*args(None)) == 1            # no gradient struct
    assert lib.moe_backward(*args(full, dy=None)) == 1   # dy missing
    assert lib.moe_backward(*args(full, aux=float("inf"))) == 1
    misaligned = M.MoeGrads(*([0x20000] * 5 + [0x20004] + [0x20000] * 6))  # dW2 off a 16-byte boundary
    assert lib.moe_backward(*args(misaligned)) == 1
    small = ctypes.c_size_t(lib.moe_workspace_size(ctypes.byref(c)))
    assert lib.moe_backward(ctypes.byref(c), a, a, None, a, None, a, a, None, None, a, ctypes.c_float(0.0),
                            ctypes.c_float(0.0), ctypes.byref(full), None, ws, small, None) == 4


def test_permute_rows_validation(lib):
    a = ctypes.c_void_p(0x10000)
    idx = ctypes.cast(ctypes.c_void_p(0x20000), ctypes.POINTER(ctypes.c_int32))
    assert lib.moe_permute_rows(2, a, idx, a, 4, 8, None) == 1                       # no such dtype
    assert lib.moe_permute_rows(1, a, idx, a, 4, 12, None) == 1                      # d not a multiple of 8
    assert lib.moe_permute_rows(1, None, idx, a, 4, 8, None) == 1                    # src missing
    assert lib.moe_permute_rows(1, ctypes.c_void_p(0x10008), idx, a, 4, 8, None) == 1  # src misaligned
    assert lib.moe_permute_rows(1, a, idx, a, -1, 8, None) == 1                      # negative rows
    assert lib.moe_permute_rows(1, None, None, None, 0, 8, None) == 0                # nothing to move


def test_data_parallel_partials_validation(lib):
    """moe_forward_partials needs counts and an 8-byte aligned psum_out;
    moe_aux_from_partials checks E, k, its outputs and gamma -- all before
    any launch."""
    c = M.make_config(64, 64, 128, 8, 2, act="swiglu", dtype="bf16")
    fwd = lambda counts, psum: lib.moe_forward_partials(ctypes.byref(c), BAD, BAD, None, BAD, None, BAD, BAD, None,
                                                        None, BAD, None, None, counts, psum, None, None, BAD, 1 << 30,
                                                        None)
    assert fwd(None, ctypes.c_void_p(0x2000)) == 1                   # counts missing
    assert fwd(ctypes.c_void_p(0x2000), None) == 1                   # psum_out missing
    assert fwd(ctypes.c_void_p(0x2000), ctypes.c_void_p(0x2004)) == 1  # psum_out not 8-byte aligned
    cnt, ps, a = ctypes.c_void_p(0x3000), ctypes.c_void_p(0x4000), ctypes.c_void_p(0x5000)
    fin = lib.moe_aux_from_partials
    assert fin(8, 9, cnt, ps, a, 0.0, None, None) == 1                       # k > E
    assert fin(0, 1, cnt, ps, a, 0.0, None, None) == 1                       # E < 1
    assert fin(512, 2, cnt, ps, a, 0.0, None, None) == 2                     # E > 256
    assert fin(64, 17, cnt, ps, a, 0.0, None, None) == 2                     # k > 16
    assert fin(8, 2, None, ps, a, 0.0, None, None) == 1                      # counts missing
    assert fin(8, 2, cnt, ctypes.c_void_p(0x4004), a, 0.0, None, None) == 1  # psum misaligned
    assert fin(8, 2, cnt, ps, None, 0.0, None, None) == 1                    # no output at all
    assert fin(8, 2, cnt, ps, a, float("nan"), None, None) == 1              # gamma not finite
