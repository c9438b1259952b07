"""CPU oracle for the Mixture-of-Experts SwiGLU forward layer.

TEST INFRASTRUCTURE.  This is the plain, slow, obviously-correct restatement of
what the layer computes, in float64, used only to check the CUDA path.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  It shares no code with
the CUDA library (no kernels, headers, helpers or tables) and imports nothing
from the product package; inputs reach it as the same stored arrays (fp32,
bf16 bit patterns, NVFP4 bytes) the GPU consumes, and it decodes them itself.

Sources (web pages on the subject; cited by title and section):

* [FSM]  "FFN、SwiGLU 与 MoE" (bjdmk.com.cn) -- sec. 2 SwiGLU (formula
  W_down[SiLU(W_gate x) * (W_up x)]), sec. 3 MoE (r = W_r x, p = softmax(r),
  TopK(p), y = sum_i p_i E_i(x); the example module renormalises the top-k
  probabilities by their sum).
* [OPS]  ops-transformer MoE operator walkthrough (gitcode.csdn.net) --
  "MoE的核心思路" (MoEConfig, MoEForward: MatMul -> TopK -> Softmax ->
  per-expert Gather / ExpertForward / Scatter -> WeightedSum), "优化二"
  (partial top-k), "坑一" (expert capacity: overflow tokens dropped, capacity
  = S*top_k/E*1.2), "坑三" (router scores in FP32).
* [DSV]  "5A · MoE fine-grained" (DeepSeek-V4.1-Flash course, openarchlab.com)
  -- sec. 1 Định nghĩa (selection on scores + bias, bias_vl only at image
  positions; multiplier gate = sqrt(softplus(scores)) raw and unnormalised;
  worked example s=[1,2]; SwiGLU clamp +-10), sec. 3 Giải pháp (shared
  expert always on; selection separated from weighting), sec. 4 Profiling
  (bias_vl=0 parity, softplus large-x branch, shared expert added once).
* [ECHO] Echo's MoE quick reference (cybersecurityerial.github.io) -- the four
  stages Router, Dispatch, FFN, Combine.
* [TH]   "กลยุทธ์การกำหนดเส้นทาง MoE: Top-K, Expert-Choice และ Sigmoid Gating"
  (blogdee.com) -- the router scores every expert, keeps the top-scoring
  ones, and a sigmoid gate gives the mixing weights of the selected experts.

Readings where the pages are silent or disagree (each also listed in the
design notes):

1. Softmax then top-k ([FSM] sec. 3) vs top-k then softmax ([OPS] MoEForward):
   identical selections (softmax is monotone); this oracle follows [FSM]:
   softmax over all experts, top-k of p, divide by the selected sum.
2. Ties in the selection key go to the lower expert index; output slots are in
   descending key order.
3. "(s + bias) / bias_vl" in [DSV] sec. 2 means "or": the selection key is
   s + bias_vl[e] at image positions, s + bias[e] elsewhere.  The bias never
   enters the multiplier.  In softmax mode the optional per-expert bias is a
   router *logit* bias: it enters both selection and weights.
4. s is the raw router logit x . W_r[e] (router weights in nn.Linear layout
   [E, D], no router bias).
5. softplus(s) = max(s, 0) + log1p(exp(-|s|)), which equals s to double
   precision above the large-x threshold the profiling note asks for.
6. Clamp (parity unpinned by the pages beyond the +-10 limit): both
   pre-activations g = W_gate x and u = W_up x are clipped to [-L, L] before
   h = SiLU(g) * u (clamp_mode "preact"); "output" clips h instead.  Applies
   to every expert, shared included.
7. Capacity C = ceil(T * k * cf / E) in exact rational arithmetic (cf = 1.2
   gives 308 for T=8192, k=2, E=64); [OPS] "坑一" truncates instead.
8. Within an expert, assignments are ordered by token index; the first C are
   kept, the rest contribute nothing and the surviving weights are not
   renormalised.
9. The shared expert has weight 1 and is added once: out = shared(x) + routed.
10. No Linear biases anywhere (the formulas have none).
11. Sigmoid gate ([TH] names it as the function that gives the selected
    experts' mixing weights, and no more): w_j = sigmoid(s_j) of the raw
    router score, not renormalised; selection is top-k of the score plus the
    selection bias exactly as in the sqrt-softplus gate (bias_vl at image
    positions), the bias never entering the weight.

Function pins (tests/test_oracle.py): every function below is pinned against
the pages' worked example, closed forms, a library routine or a brute force,
except the clamp *location* (reading 6), which is "parity unpinned".
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

# --------------------------------------------------------------------------
# Storage decoding (inputs arrive as the bytes the GPU reads)
# --------------------------------------------------------------------------


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def decode_e2m1(codes: np.ndarray) -> np.ndarray:
    """FP4 e2m1 codes (low 4 bits) -> float64: 1 sign, 2 exponent (bias 1), 1 mantissa bit."""
    c = codes.astype(np.int64) & 0xF
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return np.where(s == 1, -mag, mag)


def decode_e4m3(b: np.ndarray) -> np.ndarray:
    """FP8 e4m3fn bytes -> float64: 1 sign, 4 exponent (bias 7), 3 mantissa; S.1111.111 = NaN."""
    c = b.astype(np.int64) & 0xFF
    s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def dequant_nvfp4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Block-scaled FP4 -> float64.

    packed [..., K/2] holds two e2m1 codes per byte, the even K index in the low
    nibble; scales [..., K/16] holds one e4m3 scale per 16 consecutive K
    elements.  value[..., k] = e2m1(code[k]) * e4m3(scale[k // 16]).
    """
    K = packed.shape[-1] * 2
    codes = np.empty(packed.shape[:-1] + (K,), dtype=np.uint8)
    codes[..., 0::2] = packed & 0xF
    codes[..., 1::2] = packed >> 4
    vals = decode_e2m1(codes).reshape(*packed.shape[:-1], K // 16, 16)
    return (vals * decode_e4m3(scales)[..., None]).reshape(*packed.shape[:-1], K)


def decode_act(a: np.ndarray, fmt: str) -> np.ndarray:
    """Activation / dense-weight storage ('f32' | 'bf16') -> float64."""
    if fmt == "f32":
        return a.astype(np.float64)
    if fmt == "bf16":
        return decode_bf16(a)
    raise ValueError(fmt)


# --------------------------------------------------------------------------
# Elementwise functions
# --------------------------------------------------------------------------


def softplus(s: np.ndarray) -> np.ndarray:
    """softplus(s) = ln(1 + e^s), in the overflow-free form max(s,0) + ln(1 + e^-|s|) ([DSV] sec. 4)."""
    s = np.asarray(s, dtype=np.float64)
    return np.maximum(s, 0.0) + np.log1p(np.exp(-np.abs(s)))


def sqrt_softplus(s: np.ndarray) -> np.ndarray:
    """The raw multiplier gate sqrt(softplus(s)) ([DSV] sec. 1, worked example s=[1,2])."""
    return np.sqrt(softplus(s))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) ([FSM] sec. 2)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def sigmoid(z: np.ndarray) -> np.ndarray:
    """sigmoid(z) = 1 / (1 + e^-z), evaluated without overflow on either side ([TH] "Sigmoid Gating")."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def softmax_rows(l: np.ndarray) -> np.ndarray:
    """Row softmax, p_i = e^{l_i} / sum_j e^{l_j} (max-shifted) ([FSM] sec. 3)."""
    m = l.max(axis=1, keepdims=True)
    ex = np.exp(l - m)
    return ex / ex.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Router: scores, selection, weights
# --------------------------------------------------------------------------


def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """r = W_r x for every token: [T, D] x [E, D]^T -> [T, E] ([FSM] sec. 3; [OPS] 优化一)."""
    return x @ w_router.T


def topk_select(keys: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest keys per row, in descending key order, ties to the lower index ([OPS] 优化二)."""
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def selection_keys(logits: np.ndarray, gate: str, bias: Optional[np.ndarray] = None,
                   bias_vl: Optional[np.ndarray] = None,
                   image_mask: Optional[np.ndarray] = None) -> np.ndarray:
    """The value the top-k compares.

    softmax mode: the (optionally logit-biased) router logit.
    sqrt_softplus and sigmoid modes: s + bias_vl at image positions, s + bias
    elsewhere ([DSV] sec. 1, 3; reading 11 for the sigmoid gate).
    """
    if gate == "softmax":
        return logits + (0.0 if bias is None else bias.astype(np.float64)[None, :])
    T, E = logits.shape
    b = np.zeros((T, E))
    if bias is not None:
        b[:] = bias.astype(np.float64)[None, :]
    if bias_vl is not None and image_mask is not None:
        img = image_mask.astype(bool)
        b[img] = bias_vl.astype(np.float64)[None, :]
    return logits + b


def route_weights(logits: np.ndarray, idx: np.ndarray, gate: str,
                  bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Multipliers of the selected experts idx [T, k].

    softmax: p = softmax over all experts of the (biased) logits, then the
    selected p renormalised to sum 1 ([FSM] sec. 3 example module).
    sqrt_softplus: sqrt(softplus(s)) of the raw logit, unnormalised ([DSV] sec. 1).
    sigmoid: sigmoid(s) of the raw logit, unnormalised ([TH]; reading 11).
    """
    if gate == "softmax":
        l = logits + (0.0 if bias is None else bias.astype(np.float64)[None, :])
        p = softmax_rows(l)
        ps = np.take_along_axis(p, idx, axis=1)
        return ps / ps.sum(axis=1, keepdims=True)
    if gate == "sigmoid":
        return sigmoid(np.take_along_axis(logits, idx, axis=1))
    if gate == "sqrt_softplus":
        return sqrt_softplus(np.take_along_axis(logits, idx, axis=1))
    raise ValueError(gate)


def route(logits: np.ndarray, k: int, gate: str, bias=None, bias_vl=None, image_mask=None):
    """Top-k routing of every token: returns (idx [T,k] int64, w [T,k] float64, keys [T,E])."""
    keys = selection_keys(logits, gate, bias, bias_vl, image_mask)
    idx = topk_select(keys, k)
    w = route_weights(logits, idx, gate, bias if gate == "softmax" else None)
    return idx, w, keys


def topk_gap(keys: np.ndarray, k: int) -> np.ndarray:
    """key_(k) - key_(k+1) per token (inf when k == E): the near-tie measure."""
    T, E = keys.shape
    if k >= E:
        return np.full(T, np.inf)
    srt = -np.sort(-keys, axis=1)
    return srt[:, k - 1] - srt[:, k]


# --------------------------------------------------------------------------
# Dispatch: per-expert token lists, capacity, row maps
# --------------------------------------------------------------------------


def expert_capacity(T: int, k: int, E: int, cf) -> int:
    """C = ceil(T * k / E * cf) exactly (0 = unlimited) ([OPS] 坑一; rounded up, reading 7)."""
    if not cf or float(cf) <= 0:
        return 0
    return math.ceil(Fraction(T * k, E) * Fraction(str(cf)))


def dispatch(idx: np.ndarray, E: int, capacity: int) -> Dict[str, np.ndarray]:
    """Group assignments (t, j) by expert, in token order; keep the first C of each ([OPS] MoEForward step 3, 坑一).

    Returns counts [E] (before capacity), kept [E], offsets [E+1] (prefix of
    kept), slot_row [T, k] (row of x_perm holding (t, j), -1 if dropped),
    row_token [R], row_slot [R], drops.
    """
    T, k = idx.shape
    lists = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            lists[int(idx[t, j])].append((t, j))
    counts = np.array([len(l) for l in lists], dtype=np.int64)
    kept_lists = [l if capacity <= 0 else l[:capacity] for l in lists]
    kept = np.array([len(l) for l in kept_lists], dtype=np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    R = int(offsets[-1])
    slot_row = np.full((T, k), -1, dtype=np.int64)
    row_token = np.zeros(R, dtype=np.int64)
    row_slot = np.zeros(R, dtype=np.int64)
    r = 0
    for e in range(E):
        for (t, j) in kept_lists[e]:
            slot_row[t, j] = r
            row_token[r] = t
            row_slot[r] = j
            r += 1
    return dict(counts=counts, kept=kept, offsets=offsets, slot_row=slot_row,
                row_token=row_token, row_slot=row_slot, drops=int(T * k - R))


# --------------------------------------------------------------------------
# Expert FFN
# --------------------------------------------------------------------------


def swiglu_hidden(xr: np.ndarray, wg: np.ndarray, wu: np.ndarray, clamp: float = 0.0,
                  clamp_mode: str = "preact") -> np.ndarray:
    """h = SiLU(W_gate x) * (W_up x), with the optional +-clamp ([FSM] sec. 2; [DSV] sec. 1, 3)."""
    g = xr @ wg.T
    u = xr @ wu.T
    if clamp > 0 and clamp_mode == "preact":
        g = np.clip(g, -clamp, clamp)
        u = np.clip(u, -clamp, clamp)
    h = silu(g) * u
    if clamp > 0 and clamp_mode == "output":
        h = np.clip(h, -clamp, clamp)
    return h


def swiglu(xr, wg, wu, wd, clamp: float = 0.0, clamp_mode: str = "preact") -> np.ndarray:
    """y = W_down h ([FSM] sec. 2)."""
    return swiglu_hidden(xr, wg, wu, clamp, clamp_mode) @ wd.T


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------

ExpertFn = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def moe_forward(x: np.ndarray, logits: np.ndarray, idx: np.ndarray, w: np.ndarray,
                experts: ExpertFn, E: int, capacity: int = 0, clamp: float = 0.0,
                clamp_mode: str = "preact", shared: Optional[Tuple[np.ndarray, np.ndarray, np.ndarray]] = None,
                tokens: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Sparse forward: dispatch, per-expert SwiGLU on its kept rows, weighted sum back to tokens.

    ([OPS] MoEForward steps 3-4; [ECHO] Dispatch/FFN/Combine; [FSM] sec. 3
    y = sum_{i in TopK} w_i E_i(x); [DSV] sec. 3 shared expert added once.)

    `experts(e)` returns the float64 (W_gate [F,D], W_up [F,D], W_down [D,F]) of
    expert e.  `tokens` restricts the returned outputs to those token indices
    (routing and capacity still use every token).  Returns the dispatch maps,
    `out` [len(tokens), D] and `h_rows` {row: h} for the computed rows.
    """
    T = x.shape[0]
    disp = dispatch(idx, E, capacity)
    toks = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    pos = {int(t): i for i, t in enumerate(toks)}
    out = np.zeros((len(toks), x.shape[1]))
    h_rows = {}
    offs = disp["offsets"]
    for e in range(E):
        rows = [r for r in range(offs[e], offs[e + 1]) if int(disp["row_token"][r]) in pos]
        if not rows:
            continue
        wg, wu, wd = experts(e)
        ts = disp["row_token"][rows]
        h = swiglu_hidden(x[ts], wg, wu, clamp, clamp_mode)
        y = h @ wd.T
        for i, r in enumerate(rows):
            t, j = int(disp["row_token"][r]), int(disp["row_slot"][r])
            out[pos[t]] += w[t, j] * y[i]
            h_rows[r] = h[i]
    if shared is not None:
        sg, su, sd = shared
        out += swiglu(x[toks], sg, su, sd, clamp, clamp_mode)
    disp.update(out=out, h_rows=h_rows, tokens=toks)
    return disp


def moe_forward_dense(x: np.ndarray, logits: np.ndarray, idx: np.ndarray, w: np.ndarray,
                      experts: ExpertFn, E: int, capacity: int = 0, clamp: float = 0.0,
                      clamp_mode: str = "preact", shared=None) -> np.ndarray:
    """Brute force: every expert on every token, mixed by a dense [T, E] weight matrix.

    The weight of (t, e) is w[t, j] when idx[t, j] = e and the assignment is
    among the first C assignments of e in token order (a running count down
    the token axis), else 0.  An independent formulation of the same layer for
    tiny inputs.
    """
    T, k = idx.shape
    sel = np.zeros((T, E))
    for j in range(k):
        sel[np.arange(T), idx[:, j]] = w[:, j]
    chosen = np.zeros((T, E), dtype=np.int64)
    for j in range(k):
        chosen[np.arange(T), idx[:, j]] = 1
    if capacity > 0:
        position = np.cumsum(chosen, axis=0) - 1     # order of (t, e) among e's tokens
        sel = np.where(position < capacity, sel, 0.0)
    out = np.zeros((T, x.shape[1]))
    for e in range(E):
        wg, wu, wd = experts(e)
        out += sel[:, e:e + 1] * swiglu(x, wg, wu, wd, clamp, clamp_mode)
    if shared is not None:
        out += swiglu(x, *shared, clamp, clamp_mode)
    return out


# --------------------------------------------------------------------------
# Convenience: a layer from stored arrays
# --------------------------------------------------------------------------


class StoredLayer:
    """Decodes the stored arrays of one layer on demand (one expert at a time)."""

    def __init__(self, arrays: Dict[str, Optional[np.ndarray]], act: str, wdtype: str):
        self.a = arrays
        self.act = act
        self.wdtype = wdtype

    def x(self) -> np.ndarray:
        return decode_act(self.a["x"], self.act)

    def w_router(self) -> np.ndarray:
        return decode_act(self.a["w_router"], self.act)

    def expert(self, e: int):
        if self.wdtype == "nvfp4":
            return tuple(dequant_nvfp4(self.a[n][e], self.a[n + "_scale"][e])
                         for n in ("w_gate", "w_up", "w_down"))
        return tuple(decode_act(self.a[n][e], self.wdtype) for n in ("w_gate", "w_up", "w_down"))

    def shared(self):
        if self.a.get("sh_gate") is None:
            return None
        return tuple(decode_bf16(self.a[n]) for n in ("sh_gate", "sh_up", "sh_down"))
