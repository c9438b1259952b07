"""Helpers for the GPU-vs-oracle parity tests (not a test module).

The GPU side goes through the C ABI (binding); the oracle side through
oracle/moe_oracle.py.  Both read the same stored arrays from synth.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle.moe_oracle as O
from mixture_experts_layer_sqrt_b200 import synth

NEAR_TIE = 1e-4        # selection-key gap below which a token counts as a near-tie
F32_RTOL = 1e-5        # fp32 layer: |err_i| <= 1e-5 * max(|ref_i|, rms(ref))
BF16_RMS_TOL = 2e-2    # bf16 / FP4 layer: max |err| <= 2e-2 * rms(ref)
ROUTE_W_RTOL = 1e-5    # routing weights, every dtype


def small(name: str) -> synth.MoEProblem:
    """A shrunken copy of workload `name` that keeps its features (gate, dtypes,
    capacity, bias, shared expert) and spans several 128x128 tiles with ragged
    tails, small enough for the oracle to finish in seconds.

    A "_pair" suffix gives enough rows per group (>= 2048) for the expert GEMMs
    to take the CTA-pair (256-row tile) path."""
    if name == "mixtral_bf16_pair":
        return synth.PROBLEMS["mixtral_bf16"].with_(name=name, T=4200, D=512, F=384, E=4)
    if name == "sqrt_fp4_pair":
        # F % 256 == 0: both projections read the packed FP4 weights directly
        return synth.PROBLEMS["sqrt_fp4"].with_(name=name, T=2100, D=512, F=512, E=12, k=3, Fs=256)
    if name == "sigmoid_bf16":
        # the sigmoid gate with selection biases, image positions and a shared expert
        return synth.MoEProblem(name, T=300, D=512, F=384, E=16, k=4, gate="sigmoid", bias="uniform", Fs=256,
                                clamp=10.0, seed=7)
    p = synth.PROBLEMS[name]
    if name == "tiny_f32":
        return p
    kw = dict(T=300, D=512, F=384)
    if name == "capacity_bf16":
        kw.update(E=6)
    elif name == "finegrained_bf16":
        kw.update(E=16, k=4)
    elif name == "sqrt_fp4":
        kw.update(E=12, k=3, Fs=256)
    else:
        kw.update(E=6)
    return p.with_(name=name + "_small", **kw)


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    return t.numpy()


def oracle_layer(p: synth.MoEProblem, arrays) -> O.StoredLayer:
    return O.StoredLayer(arrays, p.act, p.wdtype)


def oracle_route(p: synth.MoEProblem, L: O.StoredLayer, arrays):
    logits = O.router_logits(L.x(), L.w_router())
    idx, w, keys = O.route(logits, p.k, p.gate, arrays.get("bias"), arrays.get("bias_vl"), arrays.get("image_mask"))
    return logits, idx, w, keys


def check_selection(idx_g: np.ndarray, keys: np.ndarray, k: int) -> dict:
    """Validate a GPU top-k selection against the oracle's float64 selection keys.

    Rule (the routing tolerance): the expert SET must equal the oracle's unless
    the token's k-th vs (k+1)-th key gap is below NEAR_TIE; the slot ORDER must
    equal the oracle's except for swaps of keys within NEAR_TIE of each other.
    Whatever the exemptions let through must still be a valid top-k within
    NEAR_TIE: k distinct experts in range, every chosen key >= the oracle's
    k-th key - NEAR_TIE, every unchosen key <= the oracle's (k+1)-th key +
    NEAR_TIE, and the slots in descending key order up to NEAR_TIE (every pair).

    Returns counts: set_ties (tokens whose k-th gap is below NEAR_TIE),
    order_ties (tokens with some adjacent gap among their top k below
    NEAR_TIE), set_flips and order_flips (tokens where the GPU's set, or only
    its order, differs from the oracle's).
    """
    T, E = keys.shape
    idx_g = np.asarray(idx_g).astype(np.int64)
    assert idx_g.shape == (T, k), f"selection shape {idx_g.shape} != {(T, k)}"
    assert ((idx_g >= 0) & (idx_g < E)).all(), "expert index out of range"
    srt_i = np.sort(idx_g, axis=1)
    assert (srt_i[:, 1:] != srt_i[:, :-1]).all(), "an expert selected twice for one token"
    idx_o = O.topk_select(keys, k)
    srt = -np.sort(-keys, axis=1)
    kth = srt[:, k - 1]
    nxt = srt[:, k] if k < E else np.full(T, -np.inf)
    set_tie = (kth - nxt) < NEAR_TIE
    same_set = (srt_i == np.sort(idx_o, axis=1)).all(axis=1)
    bad = ~same_set & ~set_tie
    assert not bad.any(), (f"{bad.sum()} tokens select a different expert set with no k-th near-tie, "
                           f"e.g. {np.nonzero(bad)[0][:5]}")
    kg = np.take_along_axis(keys, idx_g, axis=1)
    low = kg < (kth - NEAR_TIE)[:, None]
    assert not low.any(), f"{low.any(axis=1).sum()} tokens select a key below the k-th key - {NEAR_TIE}"
    rest = keys.copy()
    np.put_along_axis(rest, idx_g, -np.inf, axis=1)
    high = rest.max(axis=1) > nxt + NEAR_TIE if k < E else np.zeros(T, bool)
    assert not high.any(), f"{high.sum()} tokens leave out a key above the (k+1)-th key + {NEAR_TIE}"
    inv = kg[:, :, None] < kg[:, None, :] - NEAR_TIE           # slot i holds a key below a later slot's
    inv &= np.triu(np.ones((k, k), bool), 1)[None]
    assert not inv.any(), f"{inv.any(axis=(1, 2)).sum()} tokens order their slots against the keys"
    top = srt[:, :k]
    order_tie = ((top[:, :-1] - top[:, 1:]) < NEAR_TIE).any(axis=1) if k > 1 else np.zeros(T, bool)
    differs = (idx_g != idx_o).any(axis=1)
    return dict(set_ties=int(set_tie.sum()), order_ties=int(order_tie.sum()),
                set_flips=int((~same_set).sum()), order_flips=int((differs & same_set).sum()))


def check_route(p, idx_g: np.ndarray, w_g: np.ndarray, logits, idx_o, keys, bias=None) -> dict:
    """The selection by check_selection; the weights of the GPU's own selection
    within ROUTE_W_RTOL of the oracle's weights for that selection.  Returns
    check_selection's counts."""
    assert np.array_equal(O.topk_select(keys, p.k), idx_o)
    counts = check_selection(idx_g, keys, p.k)
    w_ref = O.route_weights(logits, idx_g.astype(np.int64), p.gate, bias if p.gate == "softmax" else None)
    np.testing.assert_allclose(w_g, w_ref, rtol=ROUTE_W_RTOL, atol=1e-7)
    return counts


def route_report(c: dict) -> str:
    return (f"near-ties set {c['set_ties']} order {c['order_ties']}, "
            f"flipped set {c['set_flips']} order {c['order_flips']}")


def assert_close_h(p, got: np.ndarray, ref: np.ndarray, what: str = "h"):
    """The SwiGLU hidden h is stored in the act dtype: bf16 adds one rounding of
    at most 2^-8 relative (RNE), on top of fp32 accumulation error."""
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    if p.act == "f32":
        lim = F32_RTOL * np.maximum(np.abs(ref), rms)
    else:
        lim = 2.0 ** -8 * np.abs(ref) + 1e-3 * rms
    bad = err > lim
    assert not bad.any(), f"{what}: {bad.sum()} elements out of bound, max ratio {(err / lim).max():.3g}"


def assert_close_f32(got: np.ndarray, ref: np.ndarray, what: str, rtol: float = F32_RTOL):
    """fp32 results computed from the GPU's own (exactly known) inputs."""
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    lim = rtol * np.maximum(np.abs(ref), rms)
    bad = err > lim
    assert not bad.any(), f"{what}: {bad.sum()} elements above {rtol} rel, max ratio {(err / lim).max():.3g}"


def assert_close_layer(p, got: np.ndarray, ref: np.ndarray, what: str):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    if p.act == "f32":
        lim = F32_RTOL * np.maximum(np.abs(ref), rms)
        bad = err > lim
        assert not bad.any(), f"{what}: {bad.sum()} elements above 1e-5 rel, max ratio {(err / lim).max():.3g}"
    else:
        assert err.max() <= BF16_RMS_TOL * rms, f"{what}: max|err| {err.max():.4g} > 2e-2 * rms {rms:.4g}"
    return float(err.max() / max(rms, 1e-30))
