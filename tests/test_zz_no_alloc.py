"""moe_dispatch_noalloc: dispatch for callers that cannot allocate device memory.

Such callers (a plugin inside an inference engine that gives it no
workspace, a serving loop that may not call cudaMalloc, a program whose
memory is all owned by another allocator) get the dispatch stage with its
histogram scratch held in a fixed array inside the library.  This file is
collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from mixture_experts_layer_sqrt_b200 import synth

KEYS = ("expert_counts", "expert_offsets", "slot_row", "row_token", "row_weight", "x_perm")


def _case(p):
    from mixture_experts_layer_sqrt_b200 import binding as B, workload as W
    a = synth.generate(p)
    cfg = W.config_of(p)
    wt = W.device_weights(p, a)
    x = W.to_torch(a["x"])
    idx, w = B.route_topk(cfg, x, B.make_weights(wt), W.to_torch(a.get("image_mask")))
    return B, cfg, x, idx, w


@pytest.mark.gpu
def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    assert torch.cuda.is_available()
    from mixture_experts_layer_sqrt_b200 import build
    build.build()
    # two calls in a row with different shapes: the second finds the first's
    # leftovers in the shared scratch and must not depend on them
    problems = [synth.PROBLEMS["finegrained_bf16"].with_(T=1000, D=512, F=384, E=16, k=4),
                synth.PROBLEMS["capacity_bf16"].with_(T=300, D=512, F=384, E=6)]
    for p in problems:
        B, cfg, x, idx, w = _case(p)
        ref = B.dispatch(cfg, x, idx, w)
        got = B.dispatch_noalloc(cfg, x, idx, w)
        torch.cuda.synchronize()
        R = int(ref["expert_offsets"][-1].item())
        for k in KEYS:
            a, b = ref[k], got[k]
            if k in ("row_token", "row_weight", "x_perm"):
                a, b = a[:R], b[:R]
            assert torch.equal(a, b), k
        # the maps-only form (no x_perm), as with the workspace entry point
        maps = B.dispatch_noalloc(cfg, x, idx, w, gather=False)
        torch.cuda.synchronize()
        assert maps["x_perm"] is None
        for k in KEYS[:-1]:
            a, b = ref[k], maps[k]
            if k in ("row_token", "row_weight"):
                a, b = a[:R], b[:R]
            assert torch.equal(a, b), k


def _host_library():
    # the size check runs on the host: no GPU needed, only the built library
    try:
        from mixture_experts_layer_sqrt_b200 import build
        build.build()
        from mixture_experts_layer_sqrt_b200 import binding
    except (RuntimeError, OSError) as e:
        pytest.skip(f"native library unavailable here: {e}")
    return binding


def test_noalloc_dispatch_rejects_oversize():
    # rejected on the host before any CUDA call: 257 chunks x 1024 experts > 262144 ints
    B = _host_library()
    cfg = B.make_config(E=1024, k=2, D=512, F=384)
    T = 256 * 257
    st = B.lib.moe_dispatch_noalloc(ctypes.byref(cfg), T, 16, 16, 16, 16, 16, 16, 16, 16, 16, None)
    assert st == B.MOE_ERR_UNSUPPORTED
