"""GPU parity: every stage through the C ABI against the float64 oracle.

Small shrunken copies of the five workloads (several tiles, ragged tails) are
checked element by element; the full-size workloads on sampled tokens (routing
and dispatch on every token).  Tolerances: indices, counts, rows and copies
bit-exact (a selection may differ only on a k-th near-tie, and only within
1e-4 of a valid top-k; see harness.check_selection); routing weights 1e-5 relative;
fp32 layer 1e-5 relative; bf16/FP4 layer max|err| <= 2e-2 * rms(oracle).
"""
import math

import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from mixture_experts_layer_sqrt_b200 import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

NAMES = ["tiny_f32", "mixtral_bf16", "capacity_bf16", "finegrained_bf16", "sqrt_fp4"]
SMALL_NAMES = NAMES + ["mixtral_bf16_pair", "sqrt_fp4_pair", "sigmoid_bf16"]


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mixture_experts_layer_sqrt_b200 import build
    build.build()
    from mixture_experts_layer_sqrt_b200 import binding
    return binding


@pytest.fixture(scope="module")
def W(B):
    from mixture_experts_layer_sqrt_b200 import workload
    return workload


class Case:
    """One problem: stored arrays, the device copies and the oracle view."""

    def __init__(self, B, W, p, arrays=None, clamp_mode="preact"):
        self.p = p
        self.a = arrays if arrays is not None else synth.generate(p)
        self.cfg = W.config_of(p, clamp_mode)
        self.clamp_mode = clamp_mode
        self.wt = W.device_weights(p, self.a)
        self.w = B.make_weights(self.wt)
        self.x = W.to_torch(self.a["x"])
        self.mask = W.to_torch(self.a.get("image_mask"))
        self.L = H.oracle_layer(p, self.a)
        self.C = self.cfg.expert_capacity

    def shared_cfg(self, B):
        p = self.p
        return B.make_config(E=1, k=1, D=p.D, F=p.Fs, clamp=p.clamp, clamp_mode=self.clamp_mode,
                             act=p.act, expert=p.act)


def _stages(B, c: Case):
    """Run route, dispatch, gate/up, down, shared expert and combine one by one."""
    p = c.p
    idx, w = B.route_topk(c.cfg, c.x, c.w, c.mask)
    d = B.dispatch(c.cfg, c.x, idx, w)
    s = {k: c.wt.get(k) for k in ("s_gate", "s_up", "s_down")}
    h = B.expert_gate_up(c.cfg, d["x_perm"], d["expert_offsets"], c.wt["w_gate"], c.wt["w_up"], s["s_gate"], s["s_up"])
    # the same projection with the rows gathered from x by the GEMM's own loads
    hg = B.expert_gate_up(c.cfg, c.x, d["expert_offsets"], c.wt["w_gate"], c.wt["w_up"], s["s_gate"], s["s_up"],
                          row_token=d["row_token"])
    y = B.expert_down(c.cfg, h, d["expert_offsets"], c.wt["w_down"], s["s_down"], d["row_weight"])
    sh = None
    if p.Fs:
        sc = c.shared_cfg(B)
        hs = B.expert_gate_up(sc, c.x, None, c.wt["sh_gate"], c.wt["sh_up"])
        sh = B.expert_down(sc, hs, None, c.wt["sh_down"])
    out = B.combine(c.cfg, y, d["slot_row"], p.T, shared_y=sh)
    torch.cuda.synchronize()
    return dict(idx=idx, w=w, h=h, hg=hg, y=y, sh=sh, out=out, **d)


@pytest.mark.parametrize("name", SMALL_NAMES)
def test_stages_small(B, W, name):
    p = H.small(name)
    c = Case(B, W, p)
    g = _stages(B, c)
    idx_g, w_g = H.to_np(g["idx"]), H.to_np(g["w"])

    # a1-a2 route
    logits, idx_o, w_o, keys = H.oracle_route(p, c.L, c.a)
    rc = H.check_route(p, idx_g, w_g, logits, idx_o, keys, c.a.get("bias"))
    print(f"{p.name}: {H.route_report(rc)}")

    # a3-a5 dispatch, conditioned on the GPU's selection: bit-exact
    d = O.dispatch(idx_g.astype(np.int64), p.E, c.C)
    R = int(d["offsets"][-1])
    np.testing.assert_array_equal(H.to_np(g["expert_counts"]), d["counts"])
    np.testing.assert_array_equal(H.to_np(g["expert_offsets"]), d["offsets"])
    np.testing.assert_array_equal(H.to_np(g["slot_row"]), d["slot_row"])
    np.testing.assert_array_equal(H.to_np(g["row_token"])[:R], d["row_token"])
    np.testing.assert_array_equal(H.to_np(g["row_weight"])[:R], w_g[d["row_token"], d["row_slot"]])
    xp = g["x_perm"][:R].cpu()
    assert torch.equal(xp, c.x.cpu()[torch.from_numpy(d["row_token"])])
    if c.C:
        assert d["drops"] > 0 or p.name.startswith("tiny")

    # a6 gate/up + SwiGLU epilogue, per expert on the GPU's rows
    x64 = c.L.x()
    h_g = H.to_np(g["h"][:R])
    h_ref = np.zeros_like(h_g)
    y_ref = np.zeros((R, p.D))
    for e in range(p.E):
        r0, r1 = d["offsets"][e], d["offsets"][e + 1]
        if r1 == r0:
            continue
        wg, wu, wd = c.L.expert(e)
        h_ref[r0:r1] = O.swiglu_hidden(x64[d["row_token"][r0:r1]], wg, wu, p.clamp, c.clamp_mode)
        # a7 down + weight epilogue, fed with the GPU's own h
        y_ref[r0:r1] = w_g[d["row_token"][r0:r1], d["row_slot"][r0:r1], None] * (h_g[r0:r1] @ wd.T)
    H.assert_close_h(p, h_g, h_ref)
    # gathered A rows are the same tile bytes as x_perm's: the same bits
    assert torch.equal(g["hg"][:R], g["h"][:R])
    y_g = H.to_np(g["y"][:R])
    H.assert_close_f32(y_g, y_ref, "y_perm")

    # both projections in one call: the same launches as the staged calls, so the same bits
    y2 = B.grouped_swiglu(c.cfg, g["x_perm"], g["expert_offsets"], c.w, g["row_weight"])
    torch.cuda.synchronize()
    assert torch.equal(y2[:R], g["y"][:R])

    # a8 shared expert
    sh_g = None
    if p.Fs:
        sh_g = H.to_np(g["sh"])
        H.assert_close_layer(p, sh_g, O.swiglu(x64, *c.L.shared(), p.clamp, c.clamp_mode), "shared")

    # a9 combine of the GPU's y (and shared): fp32 sums, one rounding
    ref = np.zeros((p.T, p.D))
    for t in range(p.T):
        for j in range(p.k):
            r = d["slot_row"][t, j]
            if r >= 0:
                ref[t] += y_g[r]
    if sh_g is not None:
        ref += sh_g
    out_g = H.to_np(g["out"])
    H.assert_close_f32(out_g, ref, "combine", rtol=1e-6)

    # whole layer vs the oracle (conditioned on the GPU's selection)
    o = O.moe_forward(x64, logits, idx_g.astype(np.int64), O.route_weights(logits, idx_g.astype(np.int64), p.gate,
                      c.a.get("bias") if p.gate == "softmax" else None), c.L.expert, p.E, c.C, p.clamp,
                      c.clamp_mode, c.L.shared())
    rel = H.assert_close_layer(p, out_g, o["out"], "out")
    print(f"{p.name}: out max|err|/rms = {rel:.3g}")

    # moe_forward gives the staged result bit for bit (same tile shapes)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    out_f = B.forward(c.cfg, c.x, c.w, ws, c.mask)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    if p.name.endswith("_pair"):
        H.assert_close_layer(p, H.to_np(out_f), o["out"], "forward")
    else:
        assert torch.equal(out_f, g["out"])

    # a bf16 output is the fp32 output rounded once (RNE: at most 2^-8 relative)
    c.cfg.out_dtype = B.MOE_BF16
    out_b = B.forward(c.cfg, c.x, c.w, ws, c.mask)
    torch.cuda.synchronize()
    assert out_b.dtype == torch.bfloat16
    assert torch.equal(out_b, out_f.to(torch.bfloat16))


def _full_forward_check(B, W, name, n_sample):
    p = synth.PROBLEMS[name]
    c = Case(B, W, p)
    T = p.T
    ws = B.workspace(B.workspace_size(c.cfg, T))
    idx_t = torch.empty((T, p.k), dtype=torch.int32, device="cuda")
    cnt_t = torch.empty(p.E, dtype=torch.int32, device="cuda")
    out = B.forward(c.cfg, c.x, c.w, ws, c.mask, topk_idx_out=idx_t, expert_counts_out=cnt_t)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    # staged route + dispatch for the per-stage maps
    idx_g_t, w_g_t = B.route_topk(c.cfg, c.x, c.w, c.mask)
    dg = B.dispatch(c.cfg, c.x, idx_g_t, w_g_t)
    torch.cuda.synchronize()
    idx_g, w_g = H.to_np(idx_g_t), H.to_np(w_g_t)
    assert np.array_equal(idx_g, H.to_np(idx_t))

    logits, idx_o, w_o, keys = H.oracle_route(p, c.L, c.a)
    rc = H.check_route(p, idx_g, w_g, logits, idx_o, keys, c.a.get("bias"))
    d = O.dispatch(idx_g.astype(np.int64), p.E, c.C)
    R = int(d["offsets"][-1])
    np.testing.assert_array_equal(H.to_np(cnt_t), d["counts"])
    np.testing.assert_array_equal(H.to_np(dg["expert_offsets"]), d["offsets"])
    np.testing.assert_array_equal(H.to_np(dg["slot_row"]), d["slot_row"])
    np.testing.assert_array_equal(H.to_np(dg["row_token"])[:R], d["row_token"])
    rows = np.random.default_rng(99).choice(R, size=min(R, 512), replace=False)
    xs = dg["x_perm"][torch.from_numpy(rows).cuda()].cpu()
    assert torch.equal(xs, c.x[torch.from_numpy(d["row_token"][rows]).cuda()].cpu())
    if c.C:
        print(f"{name}: capacity {c.C}, drops {d['drops']}")
        assert d["drops"] > 0

    rng = np.random.default_rng(7)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, size=n_sample, replace=False)]))
    w_sel = O.route_weights(logits, idx_g.astype(np.int64), p.gate, c.a.get("bias") if p.gate == "softmax" else None)
    o = O.moe_forward(c.L.x(), logits, idx_g.astype(np.int64), w_sel, c.L.expert, p.E, c.C, p.clamp, "preact",
                      c.L.shared(), tokens=toks)
    got = H.to_np(out[torch.from_numpy(toks).cuda()])
    rel = H.assert_close_layer(p, got, o["out"], "out")
    print(f"{name}: {H.route_report(rc)}, sampled {len(toks)} tokens, max|err|/rms {rel:.3g}")


@pytest.mark.parametrize("name,n_sample", [("tiny_f32", 64), ("mixtral_bf16", 48), ("capacity_bf16", 48),
                                           ("finegrained_bf16", 32), ("sqrt_fp4", 24)])
def test_full_size_sampled(B, W, name, n_sample):
    _full_forward_check(B, W, name, n_sample)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("E,k,gate,bias", [(8, 2, "softmax", "none"), (6, 6, "softmax", "zipf"),
                                           (33, 16, "sqrt_softplus", "uniform"), (48, 4, "softmax", "none"),
                                           (64, 2, "softmax", "zipf"), (128, 16, "softmax", "none"),
                                           (300, 6, "sqrt_softplus", "uniform"), (512, 8, "softmax", "none"),
                                           (8, 2, "sigmoid", "uniform"), (96, 6, "sigmoid", "uniform"),
                                           (16, 4, "softmax", "zipf"), (24, 3, "sqrt_softplus", "uniform"),
                                           (32, 8, "softmax", "none")])
def test_route_many_experts(B, W, E, k, gate, bias):
    # the router on both paths (CUDA cores up to 32 experts, tensor cores
    # above): ragged 128-token tiles, padded expert columns, one or two MMA
    # column blocks, k = E, both gates and both biases
    p = synth.MoEProblem("route", T=300, D=512, F=128, E=E, k=k, gate=gate, bias=bias, seed=21)
    a = synth.generate(p, experts=False)
    cfg = W.config_of(p)
    wt = {n: W.to_torch(a.get(n)) for n in ("w_router", "bias", "bias_vl")}
    x = W.to_torch(a["x"])
    idx, w = B.route_topk(cfg, x, B.make_weights(wt), W.to_torch(a.get("image_mask")))
    torch.cuda.synchronize()
    L = H.oracle_layer(p, a)
    logits, idx_o, w_o, keys = H.oracle_route(p, L, a)
    rc = H.check_route(p, H.to_np(idx), H.to_np(w), logits, idx_o, keys, a.get("bias"))
    print(f"route E={E} k={k} {gate}: {H.route_report(rc)}")


@pytest.mark.parametrize("T,D,E,k", [(77, 1040, 8, 2), (45, 2064, 32, 4), (16, 16, 8, 1), (1, 528, 24, 6)])
def test_route_ring_slices(B, W, T, D, E, k):
    # the streamed router for up to 32 experts: hidden sizes that end in a
    # short slice (the ring moves 512 columns at a time), a single 16-wide
    # step, token counts below and across one 16-token group
    p = synth.MoEProblem("route", T=T, D=D, F=128, E=E, k=k, gate="softmax", bias="zipf", seed=23)
    a = synth.generate(p, experts=False)
    cfg = W.config_of(p)
    wt = {n: W.to_torch(a.get(n)) for n in ("w_router", "bias", "bias_vl")}
    idx, w = B.route_topk(cfg, W.to_torch(a["x"]), B.make_weights(wt), W.to_torch(a.get("image_mask")))
    torch.cuda.synchronize()
    L = H.oracle_layer(p, a)
    logits, idx_o, w_o, keys = H.oracle_route(p, L, a)
    rc = H.check_route(p, H.to_np(idx), H.to_np(w), logits, idx_o, keys, a.get("bias"))
    print(f"route T={T} D={D} E={E} k={k}: {H.route_report(rc)}")


# ---------------------------------------------------------------- edge cases

def _edge_case(B, W, p, bias=None, capacity=None, clamp_mode="preact", x_scale=None):
    a = synth.generate(p)
    if bias is not None:
        a["bias"] = bias.astype(np.float32)
    if x_scale is not None:
        xf = O.decode_act(a["x"], p.act) * x_scale
        a["x"] = xf.astype(np.float32) if p.act == "f32" else synth.f32_to_bf16_bits(xf.astype(np.float32))
    c = Case(B, W, p, a, clamp_mode)
    if capacity is not None:
        c.cfg.expert_capacity = capacity
        c.C = capacity
    g = _stages(B, c)
    idx_g = H.to_np(g["idx"]).astype(np.int64)
    logits, idx_o, w_o, keys = H.oracle_route(p, c.L, a)
    H.check_route(p, idx_g, H.to_np(g["w"]), logits, idx_o, keys, a.get("bias"))
    d = O.dispatch(idx_g, p.E, c.C)
    np.testing.assert_array_equal(H.to_np(g["slot_row"]), d["slot_row"])
    np.testing.assert_array_equal(H.to_np(g["expert_offsets"]), d["offsets"])
    w_sel = O.route_weights(logits, idx_g, p.gate, a.get("bias") if p.gate == "softmax" else None)
    o = O.moe_forward(c.L.x(), logits, idx_g, w_sel, c.L.expert, p.E, c.C, p.clamp, clamp_mode, c.L.shared())
    # tokens with no kept assignment (and no shared expert) output exactly 0;
    # the rms bound is taken over the tokens that receive expert output
    got = H.to_np(g["out"])
    live = (d["slot_row"] >= 0).any(axis=1) | bool(p.Fs)
    assert np.all(got[~live] == 0.0)
    H.assert_close_layer(p, got[live], o["out"][live], "out")
    return g, d


BASE = synth.MoEProblem("edge", T=300, D=512, F=384, E=6, k=2, seed=11)


@pytest.mark.parametrize("T", [1, 2, 37, 129, 257])
def test_ragged_token_counts(B, W, T):
    _edge_case(B, W, BASE.with_(T=T))


def test_expert_with_no_tokens(B, W):
    bias = np.zeros(6)
    bias[3] = -100.0
    g, d = _edge_case(B, W, BASE, bias=bias)
    assert d["counts"][3] == 0


def test_all_tokens_one_expert(B, W):
    bias = np.zeros(6)
    bias[4] = 100.0
    g, d = _edge_case(B, W, BASE.with_(k=1), bias=bias)
    assert d["counts"][4] == BASE.T


def test_capacity_one(B, W):
    g, d = _edge_case(B, W, BASE, capacity=1)
    assert d["drops"] == BASE.T * 2 - 6


def test_k_equals_E(B, W):
    _edge_case(B, W, BASE.with_(E=4, k=4))


def test_shapes_off_the_tile_grid(B, W):
    _edge_case(B, W, BASE.with_(T=77, D=200, F=104))


def test_fp32_shapes_off_the_tile_grid(B, W):
    _edge_case(B, W, synth.PROBLEMS["tiny_f32"].with_(T=45, D=72, F=40, E=5, k=3))


def test_clamp_fires_both_modes(B, W):
    p = synth.PROBLEMS["sqrt_fp4"].with_(T=200, D=256, F=256, E=8, k=2, Fs=128)
    _edge_case(B, W, p, x_scale=20.0, clamp_mode="preact")
    _edge_case(B, W, p, x_scale=20.0, clamp_mode="output")


def test_deterministic_and_canaries(B, W):
    p = H.small("finegrained_bf16")
    c = Case(B, W, p)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    G = 4096  # guard elements on each side of the output
    outs = []
    for _ in range(3):
        buf = torch.full((p.T * p.D + 2 * G,), 7.25, dtype=torch.float32, device="cuda")
        out = buf[G:G + p.T * p.D].view(p.T, p.D)
        idx = torch.full((p.T * p.k + 2 * G,), -77, dtype=torch.int32, device="cuda")
        B.forward(c.cfg, c.x, c.w, ws, c.mask, out=out, topk_idx_out=idx[G:G + p.T * p.k].view(p.T, p.k))
        torch.cuda.synchronize()
        assert torch.all(buf[:G] == 7.25) and torch.all(buf[-G:] == 7.25)
        assert torch.all(idx[:G] == -77) and torch.all(idx[-G:] == -77)
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    B.check_device_status(ws)


def test_binding_rejects_mismatched_out(B, W):
    p = H.small("mixtral_bf16")
    c = Case(B, W, p)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    with pytest.raises(ValueError):
        B.forward(c.cfg, c.x, c.w, ws, out=torch.empty((p.T, p.D), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        B.forward(c.cfg, c.x, c.w, ws, out=torch.empty((p.T - 1, p.D), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("name", ["sqrt_fp4_pair", "sqrt_fp4"])
def test_fp4_direct_matches_expanded_weights(B, W, name):
    # NVFP4 codes converted to bf16 in shared memory give the MMA the same
    # operand bits as weights expanded beforehand (every e2m1 * e4m3 product is
    # exact in bf16): bit for bit the bf16 GEMM (same 128-row tiles) on the
    # expanded weights
    p = H.small(name)
    c = Case(B, W, p)
    idx, w = B.route_topk(c.cfg, c.x, c.w, c.mask)
    d = B.dispatch(c.cfg, c.x, idx, w)
    wt = c.wt
    h4 = B.expert_gate_up(c.cfg, d["x_perm"], d["expert_offsets"], wt["w_gate"], wt["w_up"], wt["s_gate"],
                          wt["s_up"])
    y4 = B.expert_down(c.cfg, h4, d["expert_offsets"], wt["w_down"], wt["s_down"], d["row_weight"])
    torch.cuda.synchronize()
    ex = {}
    for k in ("w_gate", "w_up", "w_down"):
        v = O.dequant_nvfp4(c.a[k], c.a[k + "_scale"])
        assert np.array_equal(v.astype(np.float32).astype(np.float64), v)  # exact in fp32 (and bf16)
        ex[k] = W.to_torch(synth.f32_to_bf16_bits(v.astype(np.float32)))
    cfg16 = W.config_of(p.with_(wdtype="bf16"))
    # few rows per expert: the bf16 GEMMs take single 128-row tiles too
    assert p.T * p.k < 768 * p.E
    h16 = B.expert_gate_up(cfg16, d["x_perm"], d["expert_offsets"], ex["w_gate"], ex["w_up"])
    y16 = B.expert_down(cfg16, h16, d["expert_offsets"], ex["w_down"], None, d["row_weight"])
    torch.cuda.synchronize()
    R = int(d["expert_offsets"][-1])
    assert torch.equal(h4[:R], h16[:R])
    assert torch.equal(y4[:R], y16[:R])


@pytest.mark.parametrize("name", ["mixtral_bf16", "sqrt_fp4"])
def test_profiled_forward_matches(B, W, name):
    # the stage events change nothing in the result; they bracket the stages in order
    p = H.small(name)
    c = Case(B, W, p)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    ref = B.forward(c.cfg, c.x, c.w, ws, c.mask)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(B.STAGE_EVENTS)]
    got = B.forward_profiled(c.cfg, c.x, c.w, ws, ev, c.mask)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    assert torch.equal(got, ref)
    stage = [ev[i].elapsed_time(ev[i + 1]) for i in range(B.STAGE_EVENTS - 1)]
    assert all(t >= 0.0 for t in stage)
    assert abs(sum(stage) - ev[0].elapsed_time(ev[-1])) < 1e-2


def test_fp4_forward_f16_rows_exact(B, W):
    # moe_forward gathers NVFP4 gate/up rows in f16 under a power-of-two scale
    # per row: rows of any magnitude (zero, tiny, large) keep the bf16 path's
    # products, so the layer equals the staged bf16-operand result bit for bit
    p = H.small("sqrt_fp4")
    c = Case(B, W, p)
    x = c.x.float()
    x[0] = 0.0
    x[1] *= 1.0e4
    x[2] *= 1.0e-6
    x[3] *= 3.0e-30
    c.x = x.to(torch.bfloat16)
    g = _stages(B, c)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    out_f = B.forward(c.cfg, c.x, c.w, ws, c.mask)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    assert torch.equal(out_f, g["out"])


@pytest.mark.parametrize("clamp,x_scale", [(10.0, 1.0), (10.0, 20.0), (300.0, 1.0)])
def test_fp4_forward_h_f16(B, W, clamp, x_scale):
    # inside moe_forward an NVFP4 layer whose SwiGLU clamp bounds |h| below
    # f16's range (L <= 255) keeps h in f16 and runs the down projection in
    # f16: the layer meets the oracle, and differs from the staged bf16-h path
    # by no more than bf16's rounding of h; with L > 255 h stays bf16 and the
    # layer equals the staged path bit for bit
    p = synth.PROBLEMS["sqrt_fp4"].with_(name="fp4_hf16", T=333, D=512, F=512, E=8, k=2, Fs=128, clamp=clamp)
    a = synth.generate(p)
    if x_scale != 1.0:
        a["x"] = synth.f32_to_bf16_bits((O.decode_act(a["x"], p.act) * x_scale).astype(np.float32))
    c = Case(B, W, p, a)
    g = _stages(B, c)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    out_f = B.forward(c.cfg, c.x, c.w, ws, c.mask)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    idx_g = H.to_np(g["idx"]).astype(np.int64)
    logits, idx_o, w_o, keys = H.oracle_route(p, c.L, a)
    w_sel = O.route_weights(logits, idx_g, p.gate)
    o = O.moe_forward(c.L.x(), logits, idx_g, w_sel, c.L.expert, p.E, 0, p.clamp, "preact", c.L.shared())
    rel = H.assert_close_layer(p, H.to_np(out_f), o["out"], "forward")
    if clamp > 255.0:
        assert torch.equal(out_f, g["out"])
    else:
        rms = float(np.sqrt(np.mean(o["out"] ** 2)))
        diff = float((out_f - g["out"]).abs().max())
        assert diff <= 2.0 ** -6 * rms, (diff, rms)
        print(f"clamp {clamp}, x*{x_scale}: forward vs oracle {rel:.3g} rms, vs staged bf16-h path {diff / rms:.3g} rms")


def test_bounded_wait_times_out_and_context_survives(B, W):
    # a wait that nothing satisfies gives up after its limit, records the
    # timeout in the status word and returns; the GPU keeps working
    ws = B.workspace(256)
    B.selftest_wait_timeout(ws)
    assert B.lib.moe_check_device_status(B._p(ws), None) == B.MOE_ERR_DEVICE_TIMEOUT
    assert B.lib.moe_check_device_status(B._p(ws), None) == B.MOE_OK  # read and cleared
    p = H.small("mixtral_bf16")
    c = Case(B, W, p)
    wsf = B.workspace(B.workspace_size(c.cfg, p.T))
    out = B.forward(c.cfg, c.x, c.w, wsf, c.mask)
    torch.cuda.synchronize()
    B.check_device_status(wsf)
    assert torch.isfinite(out).all()


def test_host_batches_overlapped_copies(B, W):
    # pinned host batches through the overlapped-copy path give the same
    # outputs as one forward per device batch
    p = H.small("sqrt_fp4")
    c = Case(B, W, p)
    layer = B.MoELayer(c.cfg, c.wt, p.T)
    xs, refs = [], []
    for i in range(3):
        xb = W.to_torch(synth.generate(p.with_(seed=p.seed + 100 + i), experts=False)["x"])
        refs.append(layer.forward(xb, c.mask).cpu())
        xs.append(xb.cpu().pin_memory())
    masks = [c.mask.cpu().pin_memory()] * 3
    outs = [torch.empty((p.T, p.D), dtype=torch.float32).pin_memory() for _ in range(3)]
    layer.forward_host_batches(xs, outs, masks)
    torch.cuda.synchronize()
    B.check_device_status(layer.ws)
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)


def test_zero_tokens(B, W):
    p = H.small("mixtral_bf16")
    c = Case(B, W, p)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    x0 = c.x[:0]
    out = B.forward(c.cfg, x0, c.w, ws)
    assert out.shape == (0, p.D)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_shared_expert_added_once_each_k(B, W, k):
    # at each top-k: the layer matches the oracle, and out(shared) minus
    # out(shared weights zeroed) is the shared expert alone (added once, weight 1)
    import bench
    p = H.small("sqrt_fp4").with_(k=k)
    c = Case(B, W, p)
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    idx = torch.empty((p.T, k), dtype=torch.int32, device="cuda")
    out = B.forward(c.cfg, c.x, c.w, ws, c.mask, topk_idx_out=idx)
    zero = dict(c.wt, sh_gate=torch.zeros_like(c.wt["sh_gate"]), sh_up=torch.zeros_like(c.wt["sh_up"]),
                sh_down=torch.zeros_like(c.wt["sh_down"]))
    out0 = B.forward(c.cfg, c.x, B.make_weights(zero), ws, c.mask)
    sh = bench.shared_expert_alone(B, p, c.x, c.wt)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    # combine adds the shared row last to the same routed sum r: out = fl(r + sh),
    # out0 = r, so out - out0 - sh is two fp32 roundings: <= 2^-22 (|r| + |sh|)
    r, s_ = H.to_np(out0).astype(np.float64), H.to_np(sh).astype(np.float64)
    err = np.abs(H.to_np(out).astype(np.float64) - r - s_)
    assert np.all(err <= 2.0 ** -22 * (np.abs(r) + np.abs(s_)) + 1e-30), "shared expert not added exactly once"
    idx_g = H.to_np(idx).astype(np.int64)
    logits, idx_o, w_o, keys = H.oracle_route(p, c.L, c.a)
    H.check_selection(idx_g, keys, k)
    w_sel = O.route_weights(logits, idx_g, p.gate)
    o = O.moe_forward(c.L.x(), logits, idx_g, w_sel, c.L.expert, p.E, 0, p.clamp, "preact", c.L.shared())
    H.assert_close_layer(p, H.to_np(out), o["out"], "out")
    o0 = O.moe_forward(c.L.x(), logits, idx_g, w_sel, c.L.expert, p.E, 0, p.clamp, "preact", None)
    H.assert_close_layer(p, H.to_np(out0), o0["out"], "out without the shared expert")


def test_fp4_uneven_experts(B, W):
    # the NVFP4 GEMMs with very uneven experts: an empty expert, one expert
    # with most rows (several 128-row tiles) and odd counts elsewhere; both
    # projections read the packed weights (F % 256 == 0)
    p = synth.PROBLEMS["sqrt_fp4"].with_(name="fp4_uneven", T=333, D=512, F=512, E=8, k=2, Fs=256)
    a = synth.generate(p)
    bias = np.zeros(p.E, dtype=np.float32)
    bias[0] = -100.0
    bias[3] = 3.0
    a["bias"] = bias
    a["bias_vl"] = bias
    c = Case(B, W, p, a)
    g = _stages(B, c)
    idx_g = H.to_np(g["idx"]).astype(np.int64)
    d = O.dispatch(idx_g, p.E, 0)
    assert d["counts"][0] == 0 and d["counts"][3] > 256
    logits, idx_o, w_o, keys = H.oracle_route(p, c.L, a)
    H.check_route(p, idx_g, H.to_np(g["w"]), logits, idx_o, keys, bias)
    w_sel = O.route_weights(logits, idx_g, p.gate)
    o = O.moe_forward(c.L.x(), logits, idx_g, w_sel, c.L.expert, p.E, 0, p.clamp, "preact", c.L.shared())
    H.assert_close_layer(p, H.to_np(g["out"]), o["out"], "out")
    ws = B.workspace(B.workspace_size(c.cfg, p.T))
    out_f = B.forward(c.cfg, c.x, c.w, ws, c.mask)
    torch.cuda.synchronize()
    B.check_device_status(ws)
    H.assert_close_layer(p, H.to_np(out_f), o["out"], "forward")
