"""Seeded synthetic inputs for the MoE SwiGLU forward layer.

This module only draws random tensors and encodes them in the storage formats
the layer consumes (fp32, bf16 bits, NVFP4 = e2m1 codes + e4m3 block scales).
It holds none of the layer's arithmetic: no routing, no gate, no expert math,
no decoding.  Both the CUDA path (through the C-ABI) and the CPU oracle are fed
from the arrays it returns.

Recipe (per tensor, independent counter streams so any slice can be
regenerated without drawing the others):

  stream(seed, tensor_id, expert) = numpy.random.default_rng([seed, tensor_id, expert])

  x        ~ N(0, 1)                 [T, D]
  W_router ~ N(0, 1/D)               [E, D]      (nn.Linear layout: out x in)
  W_gate   ~ N(0, 1/D)               [E, F, D]   (K-major: reduction dim last)
  W_up     ~ N(0, 1/D)               [E, F, D]
  W_down   ~ N(0, 1/F)               [E, D, F]
  shared   ~ N(0, 1/fan_in)          [Fs, D], [Fs, D], [D, Fs]
  bias (capacity workload)  3 * (z_e - min z) / (max z - min z), z_e = r_e^-1.1,
                            r = seeded permutation of 1..E (Zipf s=1.1 ranks)
  bias, bias_vl (sqrt-softplus workload) ~ U(-0.5, 0.5) [E]
  image mask (sqrt-softplus workload)    = U(0,1) < 0.1 [T]

bf16 values are float32 draws rounded to nearest-even.  NVFP4 weights are
quantised per block of 16 along the reduction (last) dimension:
scale = e4m3_rne(amax / 6), q = e2m1_rne(w / scale) (saturating at 6), two
codes per byte with the even index in the low nibble.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np

# tensor ids for the counter streams
_TID = dict(x=1, w_router=2, bias=3, bias_vl=4, w_gate=5, w_up=6, w_down=7,
            sh_gate=8, sh_up=9, sh_down=10, image_mask=11)


@dataclasses.dataclass(frozen=True)
class MoEProblem:
    """One MoE layer workload: sizes, gate mode, dtypes and seed."""
    name: str
    T: int                      # tokens
    D: int                      # hidden_dim
    F: int                      # intermediate_dim of a routed expert
    E: int                      # num_experts
    k: int                      # top_k
    act: str = "bf16"           # activations and router weights: "f32" | "bf16"
    wdtype: str = "bf16"        # routed expert weights: "f32" | "bf16" | "nvfp4"
    gate: str = "softmax"       # "softmax" (renormalised top-k) | "sqrt_softplus" | "sigmoid"
    capacity_factor: float = 0.0  # 0 = unlimited capacity
    clamp: float = 0.0          # SwiGLU clamp limit, 0 = off
    Fs: int = 0                 # shared expert intermediate dim, 0 = none
    bias: str = "none"          # "none" | "zipf" (router logit bias) | "uniform" (selection bias + bias_vl)
    seed: int = 0

    def with_(self, **kw) -> "MoEProblem":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny fp32 layer, the Mixtral-shaped layer, a
# capacity-limited skewed layer, a fine-grained layer and the sqrt-softplus
# gated FP4 layer with a shared expert.
PROBLEMS: Dict[str, MoEProblem] = {
    "tiny_f32": MoEProblem("tiny_f32", T=64, D=128, F=256, E=8, k=2, act="f32", wdtype="f32", seed=0),
    "mixtral_bf16": MoEProblem("mixtral_bf16", T=4096, D=4096, F=14336, E=8, k=2, seed=2),
    "capacity_bf16": MoEProblem("capacity_bf16", T=8192, D=2048, F=8192, E=64, k=2,
                                capacity_factor=1.2, bias="zipf", seed=3),
    "finegrained_bf16": MoEProblem("finegrained_bf16", T=8192, D=4096, F=1536, E=128, k=8, seed=4),
    "sqrt_fp4": MoEProblem("sqrt_fp4", T=8192, D=4096, F=1024, E=384, k=6, wdtype="nvfp4",
                           gate="sqrt_softplus", clamp=10.0, Fs=2048, bias="uniform", seed=5),
}


def _rng(p: MoEProblem, name: str, e: int = 0) -> np.random.Generator:
    return np.random.default_rng([p.seed, _TID[name], e])


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


# e2m1 magnitudes in code order 0..7 and the round-to-nearest-even decision
# points between consecutive codes (a tie goes to the even code).
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def _e2m1_codes(v: np.ndarray) -> np.ndarray:
    """Encode float32 values to e2m1 codes (sign<<3 | magnitude code), RNE, saturating."""
    a = np.abs(v)
    mid = (_E2M1_MAG[1:] + _E2M1_MAG[:-1]) * 0.5          # 7 midpoints
    code = np.searchsorted(mid, a, side="left").astype(np.uint8)  # a <= mid -> lower code
    # exact midpoints: searchsorted(side=left) picked the lower code; move to the
    # upper one when the lower code is odd (ties go to the even code)
    idx = np.minimum(code, 6)
    at_mid = (code < 7) & (a == mid[idx])
    odd_low = (code & 1) == 1
    code = np.where(at_mid & odd_low, code + 1, code).astype(np.uint8)
    sign = (np.signbit(v) & (code != 0)).astype(np.uint8)
    return (sign << 3) | code


def _e4m3_rne(a: np.ndarray) -> np.ndarray:
    """Encode non-negative float32 to e4m3fn bytes, round to nearest-even (via torch)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def quantize_nvfp4(w: np.ndarray):
    """Block-16 NVFP4 encoding along the last axis.

    Returns (packed uint8 [..., K/2], scales uint8 [..., K/16]).
    """
    K = w.shape[-1]
    assert K % 16 == 0
    blocks = w.reshape(*w.shape[:-1], K // 16, 16).astype(np.float32)
    amax = np.abs(blocks).max(axis=-1)
    sbytes = _e4m3_rne(amax / np.float32(6.0))
    import torch
    sval = torch.from_numpy(sbytes).view(torch.float8_e4m3fn).float().numpy()
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(sval[..., None] > 0, blocks / sval[..., None], 0.0).astype(np.float32)
    codes = _e2m1_codes(v).reshape(*w.shape[:-1], K)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, sbytes


def _normal(p: MoEProblem, name: str, shape, std: float, e: int = 0) -> np.ndarray:
    g = _rng(p, name, e)
    a = g.standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(std)
    return a


def _store(a: np.ndarray, fmt: str) -> np.ndarray:
    if fmt == "f32":
        return a.astype(np.float32, copy=False)
    if fmt == "bf16":
        return f32_to_bf16_bits(a)
    raise ValueError(fmt)


def gen_expert_weights(p: MoEProblem, name: str, e: int):
    """One expert's matrix ('w_gate'|'w_up'|'w_down') in its storage format.

    bf16/f32: one array.  nvfp4: (packed, scales).
    """
    if name == "w_down":
        shape, std = (p.D, p.F), 1.0 / math.sqrt(p.F)
    else:
        shape, std = (p.F, p.D), 1.0 / math.sqrt(p.D)
    w = _normal(p, name, shape, std, e)
    if p.wdtype == "nvfp4":
        return quantize_nvfp4(w)
    return _store(w, p.wdtype)


def generate(p: MoEProblem, experts: bool = True, threads: int = 8) -> Dict[str, Optional[np.ndarray]]:
    """All inputs of problem `p` in storage form (numpy, host memory).

    Keys: x, w_router, bias, bias_vl, image_mask, w_gate, w_up, w_down
    (+ *_scale for nvfp4), sh_gate, sh_up, sh_down.  Absent inputs are None.
    """
    out: Dict[str, Optional[np.ndarray]] = {}
    out["x"] = _store(_normal(p, "x", (p.T, p.D), 1.0), p.act)
    out["w_router"] = _store(_normal(p, "w_router", (p.E, p.D), 1.0 / math.sqrt(p.D)), p.act)
    out["bias"] = out["bias_vl"] = out["image_mask"] = None
    if p.bias == "zipf":
        r = _rng(p, "bias").permutation(p.E).astype(np.float64) + 1.0
        z = r ** -1.1
        out["bias"] = (3.0 * (z - z.min()) / (z.max() - z.min())).astype(np.float32)
    elif p.bias == "uniform":
        out["bias"] = _rng(p, "bias").uniform(-0.5, 0.5, size=p.E).astype(np.float32)
        out["bias_vl"] = _rng(p, "bias_vl").uniform(-0.5, 0.5, size=p.E).astype(np.float32)
        out["image_mask"] = (_rng(p, "image_mask").random(p.T) < 0.1).astype(np.uint8)
    if experts:
        jobs = [(n, e) for n in ("w_gate", "w_up", "w_down") for e in range(p.E)]
        with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
            res = list(ex.map(lambda ne: gen_expert_weights(p, ne[0], ne[1]), jobs))
        for n in ("w_gate", "w_up", "w_down"):
            parts = [r for (nn_, _), r in zip(jobs, res) if nn_ == n]
            if p.wdtype == "nvfp4":
                out[n] = np.stack([q for q, _ in parts])
                out[n + "_scale"] = np.stack([s for _, s in parts])
            else:
                out[n] = np.stack(parts)
            del parts
        del res
    out["sh_gate"] = out["sh_up"] = out["sh_down"] = None
    if p.Fs:
        out["sh_gate"] = _store(_normal(p, "sh_gate", (p.Fs, p.D), 1.0 / math.sqrt(p.D)), "bf16")
        out["sh_up"] = _store(_normal(p, "sh_up", (p.Fs, p.D), 1.0 / math.sqrt(p.D)), "bf16")
        out["sh_down"] = _store(_normal(p, "sh_down", (p.D, p.Fs), 1.0 / math.sqrt(p.Fs)), "bf16")
    return out
