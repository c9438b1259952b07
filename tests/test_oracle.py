"""Pins for the CPU oracle: what the pages and the mathematics fix.

Each check compares an oracle function with something other than itself:
the pages' worked example, closed forms, a library routine (numpy, scipy,
torch CPU), or a brute force on tiny inputs.  The mutation tests at the end
plant plausible mistakes in the oracle and require one of these checks to fail.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as Fnn

import oracle.moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    return np.array(rows)


def _rand_layer(rng, T, D, F, E):
    x = rng.standard_normal((T, D))
    wr = rng.standard_normal((E, D)) / math.sqrt(D)
    ex = [(rng.standard_normal((F, D)) / math.sqrt(D), rng.standard_normal((F, D)) / math.sqrt(D),
           rng.standard_normal((D, F)) / math.sqrt(F)) for _ in range(E)]
    return x, wr, ex


def _torch_swiglu(x, wg, wu, wd):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    h = Fnn.silu(Fnn.linear(t(x), t(wg))) * Fnn.linear(t(x), t(wu))
    return Fnn.linear(h, t(wd)).numpy()


# ---------------------------------------------------------------- checks
# Each check_* raises AssertionError on a mismatch; the tests below call them
# with the real oracle and the mutation tests with a broken one.


def check_worked_example():
    g = _golden("gate_worked_example.txt")
    np.testing.assert_allclose(O.softplus(g[:, 0]), g[:, 1], atol=5e-7)
    np.testing.assert_allclose(O.sqrt_softplus(g[:, 0]), g[:, 2], atol=5e-7)


def check_softplus_library():
    s = np.concatenate([np.linspace(-60, 60, 2001), [-1000.0, -100.0, 0.0, 20.0, 30.0, 100.0, 1000.0]])
    np.testing.assert_allclose(O.softplus(s), np.logaddexp(0.0, s), rtol=1e-15, atol=0)
    assert O.softplus(np.array([0.0]))[0] == pytest.approx(math.log(2.0), rel=1e-15)
    # large-x branch: softplus(x) -> x, overflow free
    assert O.softplus(np.array([1000.0]))[0] == 1000.0
    big = np.array([20.0, 30.0, 40.0])
    assert np.all(O.softplus(big) - big >= 0) and np.all(O.softplus(big) - big <= np.exp(-big))
    # identity softplus(x) - softplus(-x) = x
    np.testing.assert_allclose(O.softplus(s[:2001]) - O.softplus(-s[:2001]), s[:2001], atol=1e-12)


def check_silu_library():
    z = np.linspace(-50, 50, 1001)
    np.testing.assert_allclose(O.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)


def check_softmax_library():
    rng = np.random.default_rng(1)
    l = rng.standard_normal((7, 11)) * 3
    np.testing.assert_allclose(O.softmax_rows(l), scipy.special.softmax(l, axis=1), rtol=1e-14)


def check_topk_bruteforce():
    rng = np.random.default_rng(2)
    for E, k in [(8, 2), (6, 3), (5, 5), (9, 1)]:
        keys = rng.integers(-3, 4, size=(40, E)).astype(np.float64)   # many ties
        idx = O.topk_select(keys, k)
        for t in range(keys.shape[0]):
            # e is selected iff fewer than k experts beat it (larger key, or equal key and lower index)
            beats = lambda e: sum(1 for f in range(E)
                                  if keys[t, f] > keys[t, e] or (keys[t, f] == keys[t, e] and f < e))
            want = sorted(range(E), key=beats)[:k]
            assert [beats(e) for e in want] == list(range(k))
            assert list(idx[t]) == want, (t, keys[t], idx[t], want)


def check_softmax_route():
    rng = np.random.default_rng(3)
    T, E = 50, 8
    l = rng.standard_normal((T, E)) * 2
    for k in (1, 2, 5):
        idx, w, _ = O.route(l, k, "softmax")
        np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-14)
        assert np.all(w > 0)
        # ratios of selected weights follow the logits: w_a / w_b = e^{l_a - l_b}
        la = np.take_along_axis(l, idx, 1)
        np.testing.assert_allclose(w[:, 1:] / w[:, :1], np.exp(la[:, 1:] - la[:, :1]), rtol=1e-12)
        # descending weights
        assert np.all(np.diff(w, axis=1) <= 0)
    # k = E: the full softmax (library), re-ordered
    idx, w, _ = O.route(l, E, "softmax")
    full = scipy.special.softmax(l, axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, idx, 1), rtol=1e-13)
    # logit bias shifts both selection and weights
    b = rng.standard_normal(E)
    idx2, w2, _ = O.route(l, 2, "softmax", bias=b)
    full2 = scipy.special.softmax(l + b, axis=1)
    ps = np.take_along_axis(full2, idx2, 1)
    np.testing.assert_allclose(w2, ps / ps.sum(1, keepdims=True), rtol=1e-13)


def check_sqrt_route():
    rng = np.random.default_rng(4)
    T, E, k = 64, 16, 6
    s = rng.standard_normal((T, E))
    bias = rng.uniform(-0.5, 0.5, E)
    bvl = rng.uniform(-0.5, 0.5, E)
    img = (rng.random(T) < 0.3).astype(np.uint8)
    idx, w, keys = O.route(s, k, "sqrt_softplus", bias, bvl, img)
    # weights are the raw gate of the raw score (worked-example function), unnormalised
    np.testing.assert_allclose(w, np.sqrt(np.logaddexp(0.0, np.take_along_axis(s, idx, 1))), rtol=1e-14)
    # selection uses bias_vl at image rows, bias elsewhere
    for t in range(T):
        b = bvl if img[t] else bias
        want = sorted(range(E), key=lambda e: (-(s[t, e] + b[e]), e))[:k]
        assert list(idx[t]) == want
    # bias_vl = 0: selection may change at image rows only; the gate of any
    # (t, e) chosen in both runs is identical ([DSV] sec. 4 profiling check)
    idx0, w0, _ = O.route(s, k, "sqrt_softplus", bias, np.zeros(E), img)
    for t in range(T):
        if not img[t]:
            assert list(idx0[t]) == list(idx[t])
        common = set(idx0[t]) & set(idx[t])
        for e in common:
            a = w[t, list(idx[t]).index(e)]
            b_ = w0[t, list(idx0[t]).index(e)]
            assert a == b_
    # no bias at all: selection = top-k of the raw score, weights ranked alike
    idxn, wn, _ = O.route(s, k, "sqrt_softplus")
    assert np.all(np.diff(wn, axis=1) <= 0)


def check_capacity_table():
    assert O.expert_capacity(8192, 2, 64, 1.2) == 308      # capacity workload: 307.2 -> 308
    assert O.expert_capacity(4096, 2, 8, 1.2) == 1229      # 1228.8 -> 1229
    assert O.expert_capacity(100, 2, 4, 1.2) == 60         # exact, not rounded up
    assert O.expert_capacity(10, 1, 3, 1.0) == 4           # 3.33 -> 4
    assert O.expert_capacity(64, 2, 8, 0) == 0             # unlimited


def check_dispatch_sort():
    rng = np.random.default_rng(5)
    T, E, k = 97, 6, 2
    keys = rng.standard_normal((T, E)) + np.linspace(0, 2, E)[None, :]   # skewed
    idx = O.topk_select(keys, k)
    # unlimited capacity: rows are the stable sort of assignments by expert
    d = O.dispatch(idx, E, 0)
    perm = np.argsort(idx.reshape(-1), kind="stable")
    np.testing.assert_array_equal(d["row_token"], perm // k)
    np.testing.assert_array_equal(d["row_slot"], perm % k)
    np.testing.assert_array_equal(d["counts"], np.bincount(idx.reshape(-1), minlength=E))
    assert d["drops"] == 0
    flat = d["slot_row"].reshape(-1)
    np.testing.assert_array_equal(np.sort(flat), np.arange(T * k))
    np.testing.assert_array_equal(flat[perm], np.arange(T * k))
    # capacity: kept_e = min(count_e, C), drops = T*k - sum kept, and the kept
    # assignments are exactly the first C of each expert in token order
    C = 20
    dc = O.dispatch(idx, E, C)
    np.testing.assert_array_equal(dc["kept"], np.minimum(dc["counts"], C))
    assert dc["drops"] == T * k - dc["kept"].sum() > 0
    onehot = np.zeros((T, E), dtype=np.int64)
    for j in range(k):
        onehot[np.arange(T), idx[:, j]] = 1
    rank = np.cumsum(onehot, axis=0) - 1
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            assert (dc["slot_row"][t, j] >= 0) == (rank[t, e] < C)
            if rank[t, e] < C:
                assert dc["slot_row"][t, j] == dc["offsets"][e] + rank[t, e]


def check_expert_library():
    rng = np.random.default_rng(6)
    x, _, ex = _rand_layer(rng, 13, 24, 40, 1)
    wg, wu, wd = ex[0]
    np.testing.assert_allclose(O.swiglu(x, wg, wu, wd), _torch_swiglu(x, wg, wu, wd), rtol=1e-12, atol=1e-13)


def check_layer_e1k1():
    # E = 1, k = 1: every token goes to the one expert with weight 1, so the
    # layer is a single SwiGLU FFN (library)
    rng = np.random.default_rng(7)
    x, wr, ex = _rand_layer(rng, 21, 16, 32, 1)
    l = O.router_logits(x, wr)
    idx, w, _ = O.route(l, 1, "softmax")
    np.testing.assert_array_equal(w, 1.0)
    r = O.moe_forward(x, l, idx, w, lambda e: ex[e], 1)
    np.testing.assert_allclose(r["out"], _torch_swiglu(x, *ex[0]), rtol=1e-12, atol=1e-13)


def check_router_library():
    rng = np.random.default_rng(8)
    x, wr, _ = _rand_layer(rng, 9, 12, 4, 5)
    want = Fnn.linear(torch.from_numpy(x), torch.from_numpy(wr)).numpy()
    np.testing.assert_allclose(O.router_logits(x, wr), want, rtol=1e-13, atol=1e-14)


def check_sparse_dense():
    rng = np.random.default_rng(9)
    T, D, F, E = 37, 16, 24, 5
    x, wr, ex = _rand_layer(rng, T, D, F, E)
    l = O.router_logits(x, wr)
    for k, C in [(E, 0), (2, 0), (2, 9), (3, 14)]:
        idx, w, _ = O.route(l, k, "softmax")
        sp = O.moe_forward(x, l, idx, w, lambda e: ex[e], E, capacity=C)["out"]
        de = O.moe_forward_dense(x, l, idx, w, lambda e: ex[e], E, capacity=C)
        np.testing.assert_allclose(sp, de, rtol=1e-12, atol=1e-13)
    # k = E without capacity: the dense softmax mixture of the page's formula
    idx, w, _ = O.route(l, E, "softmax")
    p = scipy.special.softmax(l, axis=1)
    mix = sum(p[:, e:e + 1] * _torch_swiglu(x, *ex[e]) for e in range(E))
    sp = O.moe_forward(x, l, idx, w, lambda e: ex[e], E)["out"]
    np.testing.assert_allclose(sp, mix, rtol=1e-11, atol=1e-13)
    # sampled tokens equal the matching rows of the full output
    idx, w, _ = O.route(l, 2, "softmax")
    full = O.moe_forward(x, l, idx, w, lambda e: ex[e], E, capacity=9)["out"]
    sub = O.moe_forward(x, l, idx, w, lambda e: ex[e], E, capacity=9, tokens=[3, 30, 0])["out"]
    np.testing.assert_allclose(sub, full[[3, 30, 0]], rtol=1e-14, atol=0)


def check_shared_once():
    rng = np.random.default_rng(10)
    T, D, F, E, Fs = 19, 16, 8, 4, 12
    x, wr, ex = _rand_layer(rng, T, D, F, E)
    sh = (rng.standard_normal((Fs, D)) / 4, rng.standard_normal((Fs, D)) / 4, rng.standard_normal((D, Fs)) / 4)
    l = O.router_logits(x, wr)
    idx, w, _ = O.route(l, 2, "sqrt_softplus")
    routed = O.moe_forward(x, l, idx, w, lambda e: ex[e], E)["out"]
    both = O.moe_forward(x, l, idx, w, lambda e: ex[e], E, shared=sh)["out"]
    np.testing.assert_allclose(both - routed, _torch_swiglu(x, *sh), rtol=1e-11, atol=1e-13)
    zero = tuple(np.zeros_like(a) for a in sh)
    np.testing.assert_array_equal(O.moe_forward(x, l, idx, w, lambda e: ex[e], E, shared=zero)["out"], routed)
    dense = O.moe_forward_dense(x, l, idx, w, lambda e: ex[e], E, shared=sh)
    np.testing.assert_allclose(both, dense, rtol=1e-12, atol=1e-13)


def check_clamp():
    rng = np.random.default_rng(11)
    x, _, ex = _rand_layer(rng, 17, 16, 24, 1)
    wg, wu, wd = ex[0]
    xs = 20.0 * x
    free = O.swiglu(xs, wg, wu, wd)
    np.testing.assert_array_equal(O.swiglu(xs, wg, wu, wd, clamp=1e9), free)
    g, u = xs @ wg.T, xs @ wu.T
    assert np.abs(g).max() > 10 and np.abs(u).max() > 10          # the clamp fires
    h = O.swiglu_hidden(xs, wg, wu, clamp=10.0)
    # pre-activation clamp: h = SiLU(clip g) * clip u (library SiLU)
    want = Fnn.silu(torch.from_numpy(np.clip(g, -10, 10))).numpy() * np.clip(u, -10, 10)
    np.testing.assert_allclose(h, want, rtol=1e-13, atol=1e-13)
    assert np.abs(h).max() <= 10.0 * 10.0
    ho = O.swiglu_hidden(xs, wg, wu, clamp=10.0, clamp_mode="output")
    assert np.abs(ho).max() <= 10.0
    assert not np.allclose(O.swiglu(xs, wg, wu, wd, clamp=10.0), free)


def check_e2m1_table():
    g = _golden("e2m1_codes.txt")
    got = O.decode_e2m1(g[:, 0].astype(np.uint8))
    np.testing.assert_array_equal(got, g[:, 1])
    np.testing.assert_array_equal(np.signbit(got), np.signbit(g[:, 1]))


def check_e4m3_library():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.decode_e4m3(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def check_nvfp4_dequant():
    # nibble order and block scale on a hand-built block: byte 0x21 holds
    # code 1 (0.5) at the even index and code 2 (1.0) at the odd index
    packed = np.array([[0x21] + [0x00] * 7 + [0xF7] + [0x00] * 7], dtype=np.uint8)  # K = 32
    scales = np.array([[0x38, 0x40]], dtype=np.uint8)          # e4m3: 1.0, 2.0
    v = O.dequant_nvfp4(packed, scales)
    assert v.shape == (1, 32)
    assert v[0, 0] == 0.5 and v[0, 1] == 1.0 and np.all(v[0, 2:16] == 0)
    assert v[0, 16] == 6.0 * 2.0 and v[0, 17] == -6.0 * 2.0
    # every product e2m1 * e4m3 is exact in bf16 (library round trip)
    rng = np.random.default_rng(12)
    p = rng.integers(0, 256, size=(64, 64), dtype=np.uint8)
    s = rng.integers(0, 127, size=(64, 8), dtype=np.uint8)      # finite scales
    d = O.dequant_nvfp4(p, s)
    rt = torch.from_numpy(d).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(rt, d)


def check_bf16_decode():
    rng = np.random.default_rng(13)
    f = rng.standard_normal(1000).astype(np.float32)
    bits = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    want = torch.from_numpy(f).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.decode_bf16(bits), want)


def check_sigmoid_closed_forms():
    # sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4, sigmoid(-z) = 1 - sigmoid(z);
    # scipy's expit over the whole range, saturating cleanly at both ends
    np.testing.assert_allclose(O.sigmoid(np.array([0.0, math.log(3.0), -math.log(3.0)])), [0.5, 0.75, 0.25],
                               rtol=1e-15)
    z = np.concatenate([np.linspace(-40, 40, 1601), [-800.0, -50.0, 50.0, 800.0]])
    np.testing.assert_allclose(O.sigmoid(z) + O.sigmoid(-z), 1.0, rtol=1e-15)
    np.testing.assert_allclose(O.sigmoid(z), scipy.special.expit(z), rtol=1e-14, atol=0)
    assert O.sigmoid(np.array([-800.0]))[0] == 0.0 and O.sigmoid(np.array([800.0]))[0] == 1.0


def check_sigmoid_route():
    rng = np.random.default_rng(5)
    T, E, k = 64, 16, 4
    s = rng.standard_normal((T, E)) * 3
    bias = rng.uniform(-0.5, 0.5, E)
    bvl = rng.uniform(-0.5, 0.5, E)
    img = (rng.random(T) < 0.3).astype(np.uint8)
    idx, w, keys = O.route(s, k, "sigmoid", bias, bvl, img)
    # weights: the library sigmoid of the raw score, unnormalised (sums are not 1)
    np.testing.assert_allclose(w, scipy.special.expit(np.take_along_axis(s, idx, 1)), rtol=1e-14)
    assert np.all((w > 0) & (w < 1)) and not np.allclose(w.sum(1), 1.0)
    # selection: brute force over s + bias_vl at image rows, s + bias elsewhere
    for t in range(T):
        b = bvl if img[t] else bias
        want = sorted(range(E), key=lambda e: (-(s[t, e] + b[e]), e))[:k]
        assert list(idx[t]) == want
    # without a bias the weights rank like the scores (sigmoid is increasing)
    idxn, wn, _ = O.route(s, k, "sigmoid")
    assert np.all(np.diff(wn, axis=1) <= 0)


CHECKS = [check_worked_example, check_softplus_library, check_silu_library, check_softmax_library,
          check_topk_bruteforce, check_softmax_route, check_sqrt_route, check_capacity_table,
          check_dispatch_sort, check_expert_library, check_layer_e1k1, check_router_library,
          check_sparse_dense, check_shared_once, check_clamp, check_e2m1_table, check_e4m3_library,
          check_nvfp4_dequant, check_bf16_decode, check_sigmoid_closed_forms, check_sigmoid_route]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check()


def test_gap_measure():
    keys = np.array([[3.0, 1.0, 2.0, 2.5], [1.0, 1.0, 1.0, 0.0]])
    np.testing.assert_allclose(O.topk_gap(keys, 2), [0.5, 0.0])
    assert np.isinf(O.topk_gap(keys, 4)).all()


# ------------------------------------------------------------ mutations
# Plausible mistakes planted in the oracle (on the CPU); at least one pin must
# catch each.

def _mut_softplus(s):
    s = np.asarray(s, dtype=np.float64)
    return np.log1p(np.exp(-np.abs(s)))                      # dropped max(s, 0) term


def _mut_sqrt_softplus(s):
    return np.sqrt(O.softplus(s)) * np.sqrt(np.log(2.0))          # a stray constant factor


def _mut_topk_lastwins(keys, k):
    order = np.argsort(-keys[:, ::-1], axis=1, kind="stable")
    return (keys.shape[1] - 1 - order[:, :k]).astype(np.int64)  # ties to the higher index


def _mut_route_weights_norenorm(logits, idx, gate, bias=None):
    if gate == "softmax":
        p = O.softmax_rows(logits + (0.0 if bias is None else bias[None, :]))
        return np.take_along_axis(p, idx, axis=1)                  # not renormalised
    return O.sqrt_softplus(np.take_along_axis(logits, idx, axis=1))


def _mut_route_weights_biased_gate(logits, idx, gate, bias=None):
    if gate == "softmax":
        return _orig["route_weights"](logits, idx, gate, bias)
    return O.sqrt_softplus(np.take_along_axis(logits + 0.1, idx, axis=1))  # bias leaks into gate


def _mut_swiglu_hidden_swap(xr, wg, wu, clamp=0.0, clamp_mode="preact"):
    return _orig["swiglu_hidden"](xr, wu, wg, clamp, clamp_mode)   # gate/up swapped


def _mut_swiglu_hidden_clamp_u_only(xr, wg, wu, clamp=0.0, clamp_mode="preact"):
    g = xr @ wg.T
    u = xr @ wu.T
    if clamp > 0:
        u = np.clip(u, -clamp, clamp)
    return O.silu(g) * u


def _mut_dispatch_reverse(idx, E, capacity):
    # keeps the LAST C tokens of each expert
    T, k = idx.shape
    d = _orig["dispatch"](idx[::-1], E, capacity)
    sr = d["slot_row"][::-1].copy()
    d["slot_row"] = sr
    d["row_token"] = T - 1 - d["row_token"]
    return d


def _mut_capacity_trunc(T, k, E, cf):
    if not cf or cf <= 0:
        return 0
    return int(T * k / E * cf)


def _mut_router_transposed(x, w_router):
    return (x @ w_router.T)[:, ::-1]                               # expert axis reversed


def _mut_decode_e2m1(codes):
    c = codes.astype(np.int64) & 0xF
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = np.ldexp(1.0 + 0.5 * m, e - 1)                           # no subnormal case
    return np.where(s == 1, -mag, mag)


def _mut_dequant_nibbles(packed, scales):
    return _orig["dequant_nvfp4"](((packed & 0xF) << 4) | (packed >> 4), scales)  # nibble order swapped


def _mut_decode_e4m3(b):
    c = b.astype(np.int64) & 0xFF
    s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
    mag = np.ldexp(1.0 + m / 8.0, e - 8)                           # wrong bias
    return np.where(s == 1, -mag, mag)


def _mut_moe_forward_shared_twice(*a, **kw):
    r = _orig["moe_forward"](*a, **kw)
    if kw.get("shared") is not None:
        x = a[0]
        toks = r["tokens"]
        r["out"] = r["out"] + O.swiglu(x[toks], *kw["shared"])
    return r


def _mut_softmax_rows(l):
    ex = np.exp(l)
    return ex / ex.sum(axis=0, keepdims=True)                      # normalised over the wrong axis


def _mut_selection_keys(logits, gate, bias=None, bias_vl=None, image_mask=None):
    if gate == "softmax":
        return _orig["selection_keys"](logits, gate, bias, bias_vl, image_mask)
    return _orig["selection_keys"](logits, gate, bias, None, None)  # bias_vl ignored


def _mut_sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(z))                                 # sign error: sigmoid(-z)


def _mut_route_weights_sigmoid_renorm(logits, idx, gate, bias=None):
    if gate != "sigmoid":
        return _orig["route_weights"](logits, idx, gate, bias)
    w = O.sigmoid(np.take_along_axis(logits, idx, axis=1))
    return w / w.sum(axis=1, keepdims=True)                        # renormalised (not in the reading)


def _mut_silu(z):
    return np.asarray(z, float) / (1.0 + np.exp(np.asarray(z, float)))  # sign error


_orig = {n: getattr(O, n) for n in ("route_weights", "swiglu_hidden", "dispatch", "dequant_nvfp4",
                                     "moe_forward", "selection_keys")}

MUTANTS = {
    "softplus": _mut_softplus,
    "sqrt_softplus": _mut_sqrt_softplus,
    "topk_select": _mut_topk_lastwins,
    "route_weights": _mut_route_weights_norenorm,
    "route_weights#bias": _mut_route_weights_biased_gate,
    "swiglu_hidden": _mut_swiglu_hidden_swap,
    "swiglu_hidden#clamp": _mut_swiglu_hidden_clamp_u_only,
    "dispatch": _mut_dispatch_reverse,
    "expert_capacity": _mut_capacity_trunc,
    "router_logits": _mut_router_transposed,
    "decode_e2m1": _mut_decode_e2m1,
    "dequant_nvfp4": _mut_dequant_nibbles,
    "decode_e4m3": _mut_decode_e4m3,
    "moe_forward": _mut_moe_forward_shared_twice,
    "softmax_rows": _mut_softmax_rows,
    "selection_keys": _mut_selection_keys,
    "silu": _mut_silu,
    "sigmoid": _mut_sigmoid,
    "route_weights#sigmoid": _mut_route_weights_sigmoid_renorm,
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    monkeypatch.setattr(O, name.split("#")[0], MUTANTS[name])
    failed = []
    for c in CHECKS:
        try:
            with np.errstate(all="ignore"):
                c()
        except AssertionError:
            failed.append(c.__name__)
    assert failed, f"no pin catches the planted mistake in {name}"
