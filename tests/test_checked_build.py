"""The bounds-checking build (MOE_CHECKED, libmoe_b200_checked.so).

Its kernels check the indices they read from their inputs before using them
and count violations instead of touching memory out of range.  The CPU test
checks that it builds and exports the whole ABI; the GPU tests check that on
valid inputs it computes exactly what the normal build computes with no
violation, and that indices planted out of range are caught by those checks
(only ever run against the checked build, whose checks precede every access
they guard).
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from mixture_experts_layer_sqrt_b200 import synth
from tests import harness as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_checked():
    try:
        from mixture_experts_layer_sqrt_b200 import build
        return build.build(checked=True)
    except (RuntimeError, OSError) as e:
        pytest.skip(f"cannot build the checked library here: {e}")


def test_checked_library_builds_and_exports_the_abi():
    path = _build_checked()
    lib = ctypes.CDLL(path)
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "moe.h")).read(), flags=re.S)
    for name in sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src))):
        assert hasattr(lib, name), name
    assert lib.moe_checked_build() == 1


@pytest.fixture(scope="module")
def BC():
    """The binding module with its library handle switched to the checked build
    for the duration of the module's tests."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mixture_experts_layer_sqrt_b200 import build
    build.build()
    _build_checked()
    from mixture_experts_layer_sqrt_b200 import binding as B
    normal = B.lib
    checked = B.load_library(B.LIB_CHECKED_PATH)
    assert checked.moe_checked_build() == 1 and normal.moe_checked_build() == 0
    yield B, normal, checked
    B.lib = normal


def _forward(B, lib, p):
    from mixture_experts_layer_sqrt_b200 import workload as W
    B.lib = lib
    a = synth.generate(p)
    cfg = W.config_of(p)
    wt = W.device_weights(p, a)
    ws = B.workspace(B.workspace_size(cfg, p.T))
    out = B.forward(cfg, W.to_torch(a["x"]), B.make_weights(wt), ws, W.to_torch(a.get("image_mask")))
    torch.cuda.synchronize()
    B.check_device_status(ws)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny_f32", "mixtral_bf16", "sqrt_fp4", "finegrained_bf16"])
def test_checked_build_matches_normal_build(BC, name):
    B, normal, checked = BC
    p = H.small(name)
    ref = _forward(B, normal, p)
    got = _forward(B, checked, p)
    assert checked.moe_checked_violations() == 0
    assert torch.equal(got, ref)
    B.lib = normal


@pytest.mark.gpu
def test_checked_combine_skips_slot_rows_out_of_range(BC):
    B, normal, checked = BC
    B.lib = checked
    checked.moe_checked_violations()  # reset
    T, k, D = 64, 2, 128
    cfg = B.make_config(E=4, k=k, D=D, F=128)
    y = torch.randn((T * k, D), dtype=torch.float32, device="cuda")
    slot = torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k).clone()
    slot[5, 1] = T * k + 100      # past the T * k rows y_perm may hold
    slot[9, 0] = 1 << 30
    out = B.combine(cfg, y, slot, T)
    torch.cuda.synchronize()
    assert checked.moe_checked_violations() >= 2
    ref = y.view(T, k, D).sum(dim=1)
    ref[5] = y[10]                # slot 1 skipped
    ref[9] = y[19]                # slot 0 skipped
    torch.testing.assert_close(out, ref, rtol=0, atol=1e-6)
    B.lib = normal


@pytest.mark.gpu
@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_checked_gemm_rejects_bad_expert_offsets(BC, act):
    # offsets that decrease: the grouped GEMM does no work and counts a violation
    B, normal, checked = BC
    B.lib = checked
    checked.moe_checked_violations()
    from mixture_experts_layer_sqrt_b200 import workload as W
    p = synth.MoEProblem("offs", T=64, D=256, F=128, E=4, k=2, act=act, wdtype=act, seed=5)
    a = synth.generate(p)
    cfg = W.config_of(p)
    wt = W.device_weights(p, a)
    rows = p.T * p.k
    h = torch.randn((rows, p.F), device="cuda").to(torch.float32 if act == "f32" else torch.bfloat16)
    offs = torch.tensor([0, 40, 20, 90, rows], dtype=torch.int32, device="cuda")
    y = torch.full((rows, p.D), 7.5, dtype=torch.float32, device="cuda")
    B.expert_down(cfg, h, offs, wt["w_down"], None, None, y=y)
    torch.cuda.synchronize()
    assert checked.moe_checked_violations() >= 1
    assert torch.all(y == 7.5)
    B.lib = normal


@pytest.mark.gpu
def test_checked_gathered_rows_out_of_range(BC):
    # the CUDA-core GEMM's row-map gather: a token index past the source rows is skipped
    B, normal, checked = BC
    B.lib = checked
    checked.moe_checked_violations()
    from mixture_experts_layer_sqrt_b200 import workload as W
    p = synth.PROBLEMS["tiny_f32"]
    a = synth.generate(p)
    cfg = W.config_of(p)
    wt = W.device_weights(p, a)
    x = W.to_torch(a["x"])
    rows = 16
    row_token = torch.arange(rows, dtype=torch.int32, device="cuda")
    row_token[3] = p.T + 3
    h = B.expert_gate_up(cfg, x, None, wt["w_gate"], wt["w_up"], row_token=row_token, rows=rows)
    torch.cuda.synchronize()
    assert checked.moe_checked_violations() >= 1
    assert torch.all(h[3] == 0.0)                  # the skipped row reads as zeros: SiLU(0) * 0
    B.lib = normal
    ref = B.expert_gate_up(cfg, x, None, wt["w_gate"], wt["w_up"], row_token=row_token.clamp(max=p.T - 1),
                           rows=rows)
    torch.cuda.synchronize()
    keep = np.arange(rows) != 3
    assert torch.equal(h[torch.from_numpy(keep).cuda()], ref[torch.from_numpy(keep).cuda()])
