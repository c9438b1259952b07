"""Thin ctypes binding of libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the layer runs in the library's kernels.
Importing this module loads the library and raises if it is missing; there is
no fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_size_t, c_uint64, c_void_p
from typing import Dict, Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
# the bounds-checking build (build.py --checked): same ABI, loaded only on request
LIB_CHECKED_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200_checked.so")

# enums (include/moe.h)
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT = range(6)
MOE_F32, MOE_BF16, MOE_NVFP4 = range(3)
MOE_GATE_SOFTMAX_TOPK_RENORM, MOE_GATE_SQRT_SOFTPLUS_RAW, MOE_GATE_SIGMOID_RAW = range(3)
MOE_CLAMP_PREACT, MOE_CLAMP_OUTPUT = range(2)

DTYPES = {"f32": MOE_F32, "bf16": MOE_BF16, "nvfp4": MOE_NVFP4}
GATES = {"softmax": MOE_GATE_SOFTMAX_TOPK_RENORM, "sqrt_softplus": MOE_GATE_SQRT_SOFTPLUS_RAW,
         "sigmoid": MOE_GATE_SIGMOID_RAW}
CLAMP_MODES = {"preact": MOE_CLAMP_PREACT, "output": MOE_CLAMP_OUTPUT}


class MoEConfig(ctypes.Structure):
    _fields_ = [("num_experts", c_int), ("top_k", c_int), ("expert_capacity", c_int),
                ("hidden_dim", c_int), ("intermediate_dim", c_int),
                ("shared_intermediate_dim", c_int), ("gate", c_int), ("swiglu_clamp", c_float),
                ("clamp_mode", c_int), ("act_dtype", c_int), ("expert_dtype", c_int),
                ("out_dtype", c_int)]


class MoEWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("w_router", "w_gate", "w_up", "w_down", "s_gate", "s_up",
                                        "s_down", "sh_gate", "sh_up", "sh_down", "bias", "bias_vl")]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads a build of libmoe_b200.so and declares its C signatures."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m mixture_experts_layer_sqrt_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, I, S = c_void_p, c_int, c_size_t
    cfgp, wp = POINTER(MoEConfig), POINTER(MoEWeights)
    sig = {
        "moe_status_string": (c_char_p, [I]),
        "moe_version": (c_char_p, []),
        "moe_expert_capacity": (I, [I, I, I, I, I]),
        "moe_launch_count": (c_uint64, []),
        "moe_checked_build": (I, []),
        "moe_checked_violations": (c_uint64, []),
        "moe_check_device_status": (I, [P, P]),
        "moe_route_workspace_size": (S, [cfgp, I]),
        "moe_route_topk": (I, [cfgp, I, P, wp, P, P, P, P, S, P]),
        "moe_dispatch_workspace_size": (S, [cfgp, I]),
        "moe_dispatch": (I, [cfgp, I, P, P, P, P, P, P, P, P, P, P, S, P]),
        "moe_dispatch_noalloc": (I, [cfgp, I, P, P, P, P, P, P, P, P, P, P]),
        "moe_grouped_swiglu_workspace_size": (S, [cfgp, I]),
        "moe_expert_workspace_size": (S, [cfgp]),
        "moe_expert_gate_up": (I, [cfgp, I, P, I, P, P, P, P, P, P, P, P, S, P]),
        "moe_expert_down": (I, [cfgp, I, P, P, P, P, P, P, P, S, P]),
        "moe_grouped_swiglu": (I, [cfgp, I, P, P, wp, P, P, P, S, P]),
        "moe_combine": (I, [cfgp, I, P, P, P, P, P]),
        "moe_workspace_size": (S, [cfgp, I]),
        "moe_forward": (I, [cfgp, I, P, wp, P, P, P, P, P, S, P]),
        "moe_forward_profiled": (I, [cfgp, I, P, wp, P, P, P, P, P, S, P, P, I]),
        "moe_selftest_wait_timeout": (I, [P, S, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = load_library()

# Every function the header declares (checked by the tests).
EXPORTS = ("moe_status_string", "moe_version", "moe_expert_capacity", "moe_launch_count", "moe_checked_build",
           "moe_checked_violations",
           "moe_check_device_status", "moe_route_workspace_size", "moe_route_topk", "moe_dispatch_workspace_size",
           "moe_dispatch", "moe_dispatch_noalloc", "moe_grouped_swiglu_workspace_size", "moe_expert_workspace_size",
           "moe_expert_gate_up", "moe_expert_down", "moe_grouped_swiglu", "moe_combine",
           "moe_workspace_size", "moe_forward", "moe_forward_profiled", "moe_selftest_wait_timeout")


def status_string(s: int) -> str:
    return lib.moe_status_string(s).decode()


def version() -> str:
    return lib.moe_version().decode()


def launch_count() -> int:
    return int(lib.moe_launch_count())


def expert_capacity(T: int, k: int, E: int, cf_num: int, cf_den: int) -> int:
    return int(lib.moe_expert_capacity(T, k, E, cf_num, cf_den))


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoEError(st, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _expect(t: Optional[torch.Tensor], shape, dtype, what: str):
    """Buffers handed to the library must match what it will write."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{what}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_config(E: int, k: int, D: int, F: int, capacity: int = 0, Fs: int = 0, gate="softmax",
                clamp: float = 0.0, clamp_mode="preact", act="bf16", expert="bf16", out="f32") -> MoEConfig:
    return MoEConfig(E, k, capacity, D, F, Fs, GATES[gate], clamp, CLAMP_MODES[clamp_mode],
                     DTYPES[act], DTYPES[expert], DTYPES[out])


def out_torch_dtype(cfg: MoEConfig):
    return torch.float32 if cfg.out_dtype == MOE_F32 else torch.bfloat16


def make_weights(t: Dict[str, Optional[torch.Tensor]]) -> MoEWeights:
    """MoEWeights from device tensors keyed like the struct fields (missing = NULL)."""
    return MoEWeights(*[_p(t.get(n)) for n, _ in MoEWeights._fields_])


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed device workspace (the status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ------------------------------------------------------------------ stages

def route_topk(cfg: MoEConfig, x: torch.Tensor, w: MoEWeights, image_mask=None,
               topk_idx=None, topk_w=None, ws=None, stream=None):
    T = x.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty((T, cfg.top_k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, cfg.top_k), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(lib.moe_route_workspace_size(ctypes.byref(cfg), T), x.device)
    _check(lib.moe_route_topk(ctypes.byref(cfg), T, _p(x), ctypes.byref(w), _p(image_mask),
                              _p(topk_idx), _p(topk_w), _p(ws), ws.numel(), _stream(stream)), "moe_route_topk")
    return topk_idx, topk_w


def dispatch(cfg: MoEConfig, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
             out: Optional[Dict[str, torch.Tensor]] = None, ws: Optional[torch.Tensor] = None,
             stream=None, gather: bool = True) -> Dict[str, torch.Tensor]:
    """gather=False builds the row maps only (x_perm None): the gate/up GEMM gathers from x."""
    T, D, E, k = x.shape[0], cfg.hidden_dim, cfg.num_experts, cfg.top_k
    dev = x.device
    o = out or dict(
        expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
        expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
        slot_row=torch.empty((T, k), dtype=torch.int32, device=dev),
        row_token=torch.empty(T * k, dtype=torch.int32, device=dev),
        row_weight=torch.empty(T * k, dtype=torch.float32, device=dev),
        x_perm=torch.empty((T * k, D), dtype=x.dtype, device=dev) if gather else None)
    if ws is None:
        ws = workspace(lib.moe_dispatch_workspace_size(ctypes.byref(cfg), T), dev)
    _check(lib.moe_dispatch(ctypes.byref(cfg), T, _p(topk_idx), _p(topk_w), _p(x),
                            _p(o["expert_counts"]), _p(o["expert_offsets"]), _p(o["slot_row"]),
                            _p(o["row_token"]), _p(o["row_weight"]), _p(o["x_perm"]), _p(ws),
                            ws.numel(), _stream(stream)), "moe_dispatch")
    return o


def dispatch_noalloc(cfg: MoEConfig, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                     out: Optional[Dict[str, torch.Tensor]] = None, stream=None,
                     gather: bool = True) -> Dict[str, torch.Tensor]:
    """moe_dispatch_noalloc: dispatch with the library's own fixed scratch, no
    workspace.  gather=False builds the row maps only (x_perm None)."""
    T, D, E, k = x.shape[0], cfg.hidden_dim, cfg.num_experts, cfg.top_k
    dev = x.device
    o = out or dict(
        expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
        expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
        slot_row=torch.empty((T, k), dtype=torch.int32, device=dev),
        row_token=torch.empty(T * k, dtype=torch.int32, device=dev),
        row_weight=torch.empty(T * k, dtype=torch.float32, device=dev),
        x_perm=torch.empty((T * k, D), dtype=x.dtype, device=dev) if gather else None)
    _check(lib.moe_dispatch_noalloc(ctypes.byref(cfg), T, _p(topk_idx), _p(topk_w), _p(x),
                                    _p(o["expert_counts"]), _p(o["expert_offsets"]), _p(o["slot_row"]),
                                    _p(o["row_token"]), _p(o["row_weight"]), _p(o["x_perm"]),
                                    _stream(stream)), "moe_dispatch_noalloc")
    return o


def expert_gate_up(cfg: MoEConfig, a: torch.Tensor, offsets: Optional[torch.Tensor], w_gate, w_up,
                   s_gate=None, s_up=None, h=None, ws=None, rows=None, row_token=None, stream=None) -> torch.Tensor:
    """a = x_perm (dense rows), or with row_token: a = x and row r is a[row_token[r]]."""
    if rows is None:
        rows = row_token.shape[0] if row_token is not None else a.shape[0]
    if h is None:
        h = torch.empty((rows, cfg.intermediate_dim), dtype=a.dtype, device=a.device)
    if ws is None:
        ws = workspace(lib.moe_expert_workspace_size(ctypes.byref(cfg)), a.device)
    _check(lib.moe_expert_gate_up(ctypes.byref(cfg), rows, _p(a), a.shape[0], _p(row_token), _p(offsets),
                                  _p(w_gate), _p(w_up), _p(s_gate), _p(s_up), _p(h), _p(ws), ws.numel(),
                                  _stream(stream)),
           "moe_expert_gate_up")
    return h


def expert_down(cfg: MoEConfig, h: torch.Tensor, offsets: Optional[torch.Tensor], w_down, s_down=None,
                row_weight=None, y=None, ws=None, rows=None, stream=None) -> torch.Tensor:
    rows = h.shape[0] if rows is None else rows
    if y is None:
        y = torch.empty((rows, cfg.hidden_dim), dtype=torch.float32, device=h.device)
    _expect(y, (y.shape[0], cfg.hidden_dim), torch.float32, "y")
    if y.shape[0] < rows:
        raise ValueError("y has fewer rows than `rows`")
    if ws is None:
        ws = workspace(lib.moe_expert_workspace_size(ctypes.byref(cfg)), h.device)
    _check(lib.moe_expert_down(ctypes.byref(cfg), rows, _p(h), _p(offsets), _p(w_down), _p(s_down),
                               _p(row_weight), _p(y), _p(ws), ws.numel(), _stream(stream)),
           "moe_expert_down")
    return y


def grouped_swiglu(cfg: MoEConfig, x_perm: torch.Tensor, offsets, w: MoEWeights, row_weight=None,
                   y=None, ws=None, stream=None) -> torch.Tensor:
    rows = x_perm.shape[0]
    if y is None:
        y = torch.empty((rows, cfg.hidden_dim), dtype=torch.float32, device=x_perm.device)
    if ws is None:
        ws = workspace(lib.moe_grouped_swiglu_workspace_size(ctypes.byref(cfg), rows), x_perm.device)
    _check(lib.moe_grouped_swiglu(ctypes.byref(cfg), rows, _p(x_perm), _p(offsets), ctypes.byref(w),
                                  _p(row_weight), _p(y), _p(ws), ws.numel(), _stream(stream)),
           "moe_grouped_swiglu")
    return y


def combine(cfg: MoEConfig, y_perm: torch.Tensor, slot_row: torch.Tensor, T: int, shared_y=None,
            out=None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((T, cfg.hidden_dim), dtype=out_torch_dtype(cfg), device=y_perm.device)
    _expect(out, (T, cfg.hidden_dim), out_torch_dtype(cfg), "out")
    _expect(y_perm, (y_perm.shape[0], cfg.hidden_dim), torch.float32, "y_perm")
    _check(lib.moe_combine(ctypes.byref(cfg), T, _p(y_perm), _p(slot_row), _p(shared_y), _p(out),
                           _stream(stream)), "moe_combine")
    return out


def workspace_size(cfg: MoEConfig, T: int) -> int:
    return int(lib.moe_workspace_size(ctypes.byref(cfg), T))


def dispatch_workspace_size(cfg: MoEConfig, T: int) -> int:
    return int(lib.moe_dispatch_workspace_size(ctypes.byref(cfg), T))


def expert_workspace_size(cfg: MoEConfig) -> int:
    return int(lib.moe_expert_workspace_size(ctypes.byref(cfg)))


def route_workspace_size(cfg: MoEConfig, T: int) -> int:
    return int(lib.moe_route_workspace_size(ctypes.byref(cfg), T))


def grouped_swiglu_workspace_size(cfg: MoEConfig, rows: int) -> int:
    return int(lib.moe_grouped_swiglu_workspace_size(ctypes.byref(cfg), rows))


def forward(cfg: MoEConfig, x: torch.Tensor, w: MoEWeights, ws: torch.Tensor, image_mask=None,
            out=None, topk_idx_out=None, expert_counts_out=None, stream=None) -> torch.Tensor:
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, cfg.hidden_dim), dtype=out_torch_dtype(cfg), device=x.device)
    _expect(out, (T, cfg.hidden_dim), out_torch_dtype(cfg), "out")
    _expect(topk_idx_out, (T, cfg.top_k), torch.int32, "topk_idx_out")
    _expect(expert_counts_out, (cfg.num_experts,), torch.int32, "expert_counts_out")
    _check(lib.moe_forward(ctypes.byref(cfg), T, _p(x), ctypes.byref(w), _p(image_mask), _p(out),
                           _p(topk_idx_out), _p(expert_counts_out), _p(ws), ws.numel(), _stream(stream)),
           "moe_forward")
    return out


STAGES = ("route", "dispatch", "gate_up", "down", "shared", "combine")
STAGE_EVENTS = 8


def _event_handles(events):
    hs = []
    for ev in events:
        if ev is None:
            hs.append(None)
            continue
        if not ev.cuda_event:  # torch creates the CUDA event lazily
            ev.record()
        hs.append(ctypes.c_void_p(ev.cuda_event))
    return (ctypes.c_void_p * len(hs))(*hs)


def forward_profiled(cfg: MoEConfig, x: torch.Tensor, w: MoEWeights, ws: torch.Tensor, events, image_mask=None,
                     out=None, topk_idx_out=None, expert_counts_out=None, stream=None) -> torch.Tensor:
    """moe_forward_profiled: `events` are 7 torch.cuda.Event (or None), recorded at the stage
    boundaries: before route, then after route, dispatch, gate/up, down, shared, combine."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, cfg.hidden_dim), dtype=out_torch_dtype(cfg), device=x.device)
    _expect(out, (T, cfg.hidden_dim), out_torch_dtype(cfg), "out")
    _expect(topk_idx_out, (T, cfg.top_k), torch.int32, "topk_idx_out")
    _expect(expert_counts_out, (cfg.num_experts,), torch.int32, "expert_counts_out")
    if len(events) != STAGE_EVENTS:
        raise ValueError(f"forward_profiled needs {STAGE_EVENTS} events")
    _check(lib.moe_forward_profiled(ctypes.byref(cfg), T, _p(x), ctypes.byref(w), _p(image_mask), _p(out),
                                    _p(topk_idx_out), _p(expert_counts_out), _p(ws), ws.numel(), _stream(stream),
                                    ctypes.cast(_event_handles(events), ctypes.c_void_p), STAGE_EVENTS),
           "moe_forward_profiled")
    return out


def selftest_wait_timeout(ws: torch.Tensor, stream=None):
    """Launch the never-satisfied bounded wait (about 2 s); the status word of ws then reads timeout."""
    _check(lib.moe_selftest_wait_timeout(_p(ws), ws.numel(), _stream(stream)), "moe_selftest_wait_timeout")


def check_device_status(ws: torch.Tensor, stream=None):
    _check(lib.moe_check_device_status(_p(ws), _stream(stream)), "device status")


# ------------------------------------------------------------------ layer

class MoELayer:
    """A layer whose weights live on the device; forward() is one moe_forward call.

    ``forward_host`` is the end-to-end path: pinned host tokens in, host
    output back, copies included.
    """

    def __init__(self, cfg: MoEConfig, weights: Dict[str, Optional[torch.Tensor]], max_tokens: int,
                 device="cuda"):
        self.cfg = cfg
        self.weights = weights            # keeps the tensors alive
        self.w = make_weights(weights)
        self.max_tokens = max_tokens
        self.ws = workspace(workspace_size(cfg, max_tokens), device)
        self.device = device

    def forward(self, x: torch.Tensor, image_mask=None, out=None, topk_idx_out=None,
                expert_counts_out=None, stream=None) -> torch.Tensor:
        if x.shape[0] > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        return forward(self.cfg, x, self.w, self.ws, image_mask, out, topk_idx_out, expert_counts_out, stream)

    def forward_host_batches(self, xs_host, outs_host, masks_host=None) -> None:
        """Forward a sequence of pinned host batches, copies overlapped with compute.

        Batch i's host-to-device copy runs on its own stream ahead of the
        compute, and batch i's device-to-host copy on a third stream behind
        it, so while batch i computes, batch i+1 is uploading and batch i-1
        downloading; two device buffers alternate.  Every batch is still
        copied in and out.  Asynchronous: synchronise before reading outs_host.
        """
        n = len(xs_host)
        if n == 0:
            return
        comp = torch.cuda.current_stream()
        if not hasattr(self, "_h2d"):
            self._h2d, self._d2h = torch.cuda.Stream(), torch.cuda.Stream()
        h2d, d2h = self._h2d, self._d2h
        T, D = xs_host[0].shape
        odt = out_torch_dtype(self.cfg)
        x_dev = [torch.empty((T, D), dtype=xs_host[0].dtype, device=self.device) for _ in range(2)]
        o_dev = [torch.empty((T, D), dtype=odt, device=self.device) for _ in range(2)]
        m_dev = [None, None]
        if masks_host is not None:
            m_dev = [torch.empty_like(masks_host[0], device=self.device) for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_free = [torch.cuda.Event() for _ in range(2)]
        for i in range(n):
            b = i % 2
            if i >= 2:
                h2d.wait_event(ev_done[b])          # batch i-2 no longer reads x_dev[b]
            with torch.cuda.stream(h2d):
                x_dev[b].copy_(xs_host[i], non_blocking=True)
                if masks_host is not None:
                    m_dev[b].copy_(masks_host[i], non_blocking=True)
                ev_in[b].record(h2d)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_free[b])         # batch i-2's result has left o_dev[b]
            self.forward(x_dev[b], m_dev[b], o_dev[b])
            ev_done[b].record(comp)
            d2h.wait_event(ev_done[b])
            with torch.cuda.stream(d2h):
                outs_host[i].copy_(o_dev[b], non_blocking=True)
                ev_free[b].record(d2h)
        comp.wait_stream(d2h)

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, image_mask_host=None,
                     x_dev=None, out_dev=None, mask_dev=None) -> torch.Tensor:
        """Host (pinned) x -> device -> moe_forward -> host out, on the current stream."""
        x_dev = x_dev if x_dev is not None else torch.empty_like(x_host, device=self.device)
        x_dev.copy_(x_host, non_blocking=True)
        if image_mask_host is not None:
            mask_dev = mask_dev if mask_dev is not None else torch.empty_like(image_mask_host, device=self.device)
            mask_dev.copy_(image_mask_host, non_blocking=True)
        out_dev = self.forward(x_dev, mask_dev, out_dev)
        out_host.copy_(out_dev, non_blocking=True)
        return out_host
