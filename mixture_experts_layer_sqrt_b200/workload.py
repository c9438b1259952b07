"""Glue between a synthetic workload (``synth.MoEProblem`` + its stored arrays)
and the C ABI: the layer config and the device tensors.  No layer arithmetic.
"""
from __future__ import annotations

from fractions import Fraction
from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B
from .synth import MoEProblem


def capacity_of(p: MoEProblem) -> int:
    if not p.capacity_factor:
        return 0
    f = Fraction(str(p.capacity_factor))
    return B.expert_capacity(p.T, p.k, p.E, f.numerator, f.denominator)


def config_of(p: MoEProblem, clamp_mode: str = "preact", out: str = "f32") -> B.MoEConfig:
    return B.make_config(E=p.E, k=p.k, D=p.D, F=p.F, capacity=capacity_of(p), Fs=p.Fs, gate=p.gate,
                         clamp=p.clamp, clamp_mode=clamp_mode, act=p.act, expert=p.wdtype, out=out)


def to_torch(a: Optional[np.ndarray], device="cuda", pin=False) -> Optional[torch.Tensor]:
    """Stored array -> tensor: uint16 bit patterns become bfloat16, others keep their dtype."""
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device, non_blocking=False)


def device_weights(p: MoEProblem, arrays: Dict[str, Optional[np.ndarray]], device="cuda") -> Dict[str, Optional[torch.Tensor]]:
    """Device tensors keyed by MoEWeights field names."""
    w = {"w_router": to_torch(arrays["w_router"], device),
         "w_gate": to_torch(arrays["w_gate"], device), "w_up": to_torch(arrays["w_up"], device),
         "w_down": to_torch(arrays["w_down"], device),
         "bias": to_torch(arrays.get("bias"), device), "bias_vl": to_torch(arrays.get("bias_vl"), device),
         "sh_gate": to_torch(arrays.get("sh_gate"), device), "sh_up": to_torch(arrays.get("sh_up"), device),
         "sh_down": to_torch(arrays.get("sh_down"), device)}
    if p.wdtype == "nvfp4":
        w["s_gate"] = to_torch(arrays["w_gate_scale"], device)
        w["s_up"] = to_torch(arrays["w_up_scale"], device)
        w["s_down"] = to_torch(arrays["w_down_scale"], device)
    return w
