"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from oracle.moe_oracle import expert_capacity as oracle_capacity

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def B():
    from mixture_experts_layer_sqrt_b200 import build
    build.build()
    from mixture_experts_layer_sqrt_b200 import binding
    return binding


def test_exports_every_declared_symbol(B):
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(B.lib, n), n
    assert sorted(B.EXPORTS) == names


def test_library_links_no_cuda_shared_object():
    # the CUDA runtime is linked statically: loading needs no libcudart.so
    from mixture_experts_layer_sqrt_b200 import build
    lib = build.build()
    deps = open(lib, "rb").read()
    assert b"libcudart.so" not in deps


def test_status_strings(B):
    for s in range(6):
        assert B.status_string(s).startswith("MOE_")
    assert "sm_100a" in B.version()


@pytest.mark.parametrize("T,k,E,cf", [(8192, 2, 64, "1.2"), (4096, 2, 8, "1.2"), (100, 2, 4, "1.2"),
                                      (10, 1, 3, "1"), (7, 3, 5, "1.25"), (1, 1, 1, "2.5")])
def test_capacity_matches_oracle(B, T, k, E, cf):
    from fractions import Fraction
    f = Fraction(cf)
    assert B.expert_capacity(T, k, E, f.numerator, f.denominator) == oracle_capacity(T, k, E, cf)


def test_capacity_edge(B):
    assert B.expert_capacity(64, 2, 8, 0, 1) == 0
    assert B.expert_capacity(64, 2, 8, 1, 0) == -1


def _cfg(B, **kw):
    base = dict(E=8, k=2, D=128, F=256)
    base.update(kw)
    return B.make_config(**base)


def test_workspace_sizes(B):
    c = _cfg(B, act="bf16")
    assert B.lib.moe_workspace_size(ctypes.byref(c), 64) > 0
    assert B.lib.moe_workspace_size(ctypes.byref(c), 4096) > B.lib.moe_workspace_size(ctypes.byref(c), 64)
    assert B.lib.moe_dispatch_workspace_size(ctypes.byref(c), 4096) >= 256
    bad = _cfg(B, k=9)
    assert B.lib.moe_workspace_size(ctypes.byref(bad), 64) == 0
    fp4 = _cfg(B, expert="nvfp4")
    assert B.lib.moe_expert_workspace_size(ctypes.byref(fp4)) >= 2 * 8 * 256 * 128 * 2


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), 1), (dict(k=9), 1), (dict(E=2000), 2), (dict(D=100), 2), (dict(k=17, E=32), 1),
    (dict(act="f32", expert="bf16"), 2), (dict(act="f32", expert="nvfp4"), 2),
    (dict(expert="nvfp4", F=200), 2), (dict(clamp=-1.0), 1), (dict(capacity=-1), 1),
])
def test_invalid_config_rejected_on_host(B, kw, status):
    c = _cfg(B, **kw)
    w = B.MoEWeights()
    st = B.lib.moe_route_topk(ctypes.byref(c), 4, 16, ctypes.byref(w), None, 16, 16, 16, 256, None)
    assert st == status


def test_null_and_misaligned_pointers_rejected(B):
    c = _cfg(B)
    w = B.MoEWeights(w_router=16)
    assert B.lib.moe_route_topk(ctypes.byref(c), 4, None, ctypes.byref(w), None, 16, 16, 16, 256, None) == B.MOE_ERR_INVALID_ARG
    assert B.lib.moe_route_topk(ctypes.byref(c), 4, 24, ctypes.byref(w), None, 16, 16, 16, 256, None) == B.MOE_ERR_INVALID_ARG
    assert B.lib.moe_route_topk(None, 4, 16, ctypes.byref(w), None, 16, 16, 16, 256, None) == B.MOE_ERR_INVALID_ARG
    assert B.lib.moe_route_topk(ctypes.byref(c), -1, 16, ctypes.byref(w), None, 16, 16, 16, 256, None) == B.MOE_ERR_INVALID_ARG
    # zero tokens: nothing to do, nothing launched
    assert B.lib.moe_route_topk(ctypes.byref(c), 0, None, None, None, None, None, 16, 256, None) == B.MOE_OK
    # workspace missing or too small
    assert B.lib.moe_route_topk(ctypes.byref(c), 4, 16, ctypes.byref(w), None, 16, 16, None, 0, None) == B.MOE_ERR_INVALID_ARG
    assert B.lib.moe_route_topk(ctypes.byref(c), 4, 16, ctypes.byref(w), None, 16, 16, 16, 8, None) == B.MOE_ERR_WORKSPACE
    assert B.lib.moe_combine(ctypes.byref(c), 4, None, 16, None, 16, None) == B.MOE_ERR_INVALID_ARG


def test_workspace_too_small_rejected(B):
    c = _cfg(B)
    need = B.lib.moe_dispatch_workspace_size(ctypes.byref(c), 64)
    st = B.lib.moe_dispatch(ctypes.byref(c), 64, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, need - 1, None)
    assert st == B.MOE_ERR_WORKSPACE
    w = B.MoEWeights(w_router=16, w_gate=16, w_up=16, w_down=16)
    need = B.lib.moe_workspace_size(ctypes.byref(c), 64)
    st = B.lib.moe_forward(ctypes.byref(c), 64, 16, ctypes.byref(w), None, 16, None, None, 16, need - 1, None)
    assert st == B.MOE_ERR_WORKSPACE
    e = B.lib.moe_expert_workspace_size(ctypes.byref(c))
    st = B.lib.moe_expert_gate_up(ctypes.byref(c), 8, 16, 8, None, None, 16, 16, None, None, 16, 16, e - 1,
                                  None)
    assert st == B.MOE_ERR_WORKSPACE


def test_nvfp4_requires_scales(B):
    c = _cfg(B, expert="nvfp4")
    e = B.lib.moe_expert_workspace_size(ctypes.byref(c))
    st = B.lib.moe_expert_gate_up(ctypes.byref(c), 8, 16, 8, None, None, 16, 16, None, 16, 16, 16, e, None)
    assert st == B.MOE_ERR_INVALID_ARG
    st = B.lib.moe_expert_down(ctypes.byref(c), 8, 16, None, 16, None, None, 16, 16, e, None)
    assert st == B.MOE_ERR_INVALID_ARG
    # scales are read by TMA: 16-byte aligned like the codes
    st = B.lib.moe_expert_down(ctypes.byref(c), 8, 16, None, 16, 24, None, 16, 16, e, None)
    assert st == B.MOE_ERR_INVALID_ARG


def test_gather_needs_source_rows(B):
    # a row map without the row count of the source matrix cannot be bounded
    c = _cfg(B, act="bf16")
    e = B.lib.moe_expert_workspace_size(ctypes.byref(c))
    st = B.lib.moe_expert_gate_up(ctypes.byref(c), 8, 16, 0, 16, None, 16, 16, None, None, 16, 16, e, None)
    assert st == B.MOE_ERR_INVALID_ARG


def test_profiled_forward_event_count(B):
    # 0 events (plain forward) or exactly MOE_STAGE_EVENTS; checked before any CUDA work
    c = _cfg(B)
    w = B.MoEWeights(w_router=16, w_gate=16, w_up=16, w_down=16)
    need = B.lib.moe_workspace_size(ctypes.byref(c), 64)
    assert B.STAGE_EVENTS == 8
    ev = (ctypes.c_void_p * 9)()
    for n in (1, 7, 9, -1):
        st = B.lib.moe_forward_profiled(ctypes.byref(c), 64, 16, ctypes.byref(w), None, 16, None, None, 16, need,
                                        None, ctypes.cast(ev, ctypes.c_void_p), n)
        assert st == B.MOE_ERR_INVALID_ARG
    st = B.lib.moe_forward_profiled(ctypes.byref(c), 64, 16, ctypes.byref(w), None, 16, None, None, 16, need,
                                    None, None, 8)
    assert st == B.MOE_ERR_INVALID_ARG


def test_selftest_needs_a_status_word(B):
    assert B.lib.moe_selftest_wait_timeout(None, 256, None) == B.MOE_ERR_INVALID_ARG
    assert B.lib.moe_selftest_wait_timeout(16, 8, None) == B.MOE_ERR_INVALID_ARG


def test_launch_count_starts_at_zero_without_gpu(B):
    assert B.launch_count() >= 0
