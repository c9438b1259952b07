"""Expert parallelism: the routed experts split over the ranks of a process
group, tokens exchanged with all-to-all (the expert-parallel alternative to
data parallelism for this layer).

Every rank holds the router (and the shared expert) whole and E / world of the
routed experts: rank r owns experts [r E_l, (r + 1) E_l), E_l = E / world.  A
forward on a rank's own tokens:

  1. route and dispatch its tokens over all E experts (the library's kernels):
     x_perm is grouped by expert, so the rows bound for each owner rank are one
     contiguous block;
  2. exchange the per-(owner, local expert) row counts, then the rows and their
     routing weights (all_to_all_single);
  3. on the owner, the received rows (grouped by source rank, then by expert)
     are dispatched again with top-1 over the local experts, which groups them
     by local expert in a stable order, and run through the grouped SwiGLU
     GEMMs, routing weight applied in the down epilogue;
  4. a top-1 combine (one row per received row) puts the fp32 results back in
     received order, a second all_to_all_single returns them to their source
     rank, where they land exactly in x_perm's row order (y_perm);
  5. the usual combine (slot order, + the shared expert) gives the output.

Each row meets the same weights, accumulation order and routing weight as in
the single-GPU layer, and the combine sums in the same order, so the output
matches moe_forward's (the only possible difference is the expert GEMM's tile
shape when the local row counts make it pick another, which changes no
arithmetic per row).  Expert capacity is not supported here (every rank
would see only its own tokens' positions).

`ops` supplies the device stages; by default the library's kernels through the
binding.  The exchange logic is host code (counts, splits, the owner's row
map) and is the same whatever `ops` is.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

__all__ = ["local_expert_range", "send_counts", "received_expert_ids", "ExpertParallelMoE"]


def local_expert_range(E: int, world: int, rank: int):
    """[first, last) of the experts rank `rank` owns (E must divide evenly)."""
    if world < 1 or E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    el = E // world
    return rank * el, (rank + 1) * el


def send_counts(expert_offsets: np.ndarray, world: int) -> np.ndarray:
    """Rows of each (owner rank, owner's local expert) in this rank's x_perm:
    [world, E_l] from the [E + 1] expert offsets of the dispatch."""
    offs = np.asarray(expert_offsets, dtype=np.int64)
    E = offs.shape[0] - 1
    local_expert_range(E, world, 0)
    return np.diff(offs).reshape(world, E // world)


def received_expert_ids(recv_counts: np.ndarray) -> np.ndarray:
    """The local expert of every received row, in received order: source rank
    by source rank, and within a source in local expert order (the order of
    the sender's x_perm).  recv_counts is [world, E_l]."""
    rc = np.asarray(recv_counts, dtype=np.int64)
    E_l = rc.shape[1]
    reps = rc.reshape(-1)
    ids = np.tile(np.arange(E_l, dtype=np.int32), rc.shape[0])
    return np.repeat(ids, reps)


class _KernelOps:
    """The device stages of the layer through the library's C ABI."""

    y_dtype = torch.float32  # the expert outputs (and the exchange of them)

    def __init__(self):
        from . import binding as B
        self.B = B

    def route(self, cfg, x, w, mask):
        return self.B.route_topk(cfg, x, w, mask)

    def dispatch(self, cfg, x, idx, w):
        return self.B.dispatch(cfg, x, idx, w)

    def grouped_swiglu(self, cfg, x_perm, offsets, w, row_weight):
        return self.B.grouped_swiglu(cfg, x_perm, offsets, w, row_weight)

    def combine(self, cfg, y_perm, slot_row, T, shared_y=None):
        return self.B.combine(cfg, y_perm, slot_row, T, shared_y=shared_y)

    def shared(self, cfg, x, wt):
        B = self.B
        sc = B.make_config(E=1, k=1, D=cfg.hidden_dim, F=cfg.shared_intermediate_dim, clamp=cfg.swiglu_clamp,
                           clamp_mode={v: k for k, v in B.CLAMP_MODES.items()}[cfg.clamp_mode],
                           act={v: k for k, v in B.DTYPES.items()}[cfg.act_dtype],
                           expert={v: k for k, v in B.DTYPES.items()}[cfg.act_dtype])
        hs = B.expert_gate_up(sc, x, None, wt["sh_gate"], wt["sh_up"])
        return B.expert_down(sc, hs, None, wt["sh_down"])

    def make_weights(self, wt):
        return self.B.make_weights(wt)

    def local_config(self, cfg, E_local: int, k: int, out_f32: bool = False):
        c = self.B.MoEConfig.from_buffer_copy(cfg)
        c.num_experts = E_local
        c.top_k = k
        c.expert_capacity = 0
        c.shared_intermediate_dim = 0
        c.gate = self.B.MOE_GATE_SOFTMAX_TOPK_RENORM  # only the dispatch and the GEMMs read it
        if out_f32:
            c.out_dtype = self.B.MOE_F32
        return c


class ExpertParallelMoE:
    """One rank's part of an expert-parallel MoE layer.

    cfg: the whole layer's MoEConfig (all E experts; expert_capacity 0).
    weights: dict of device tensors as MoEWeights names: w_router (whole),
    w_gate / w_up / w_down (and s_* for NVFP4) holding ONLY this rank's E_l
    experts, sh_* (whole) when there is a shared expert, bias / bias_vl.
    group: the torch.distributed process group (NCCL for device tensors).
    """

    def __init__(self, cfg, weights: Dict[str, Optional[torch.Tensor]], group=None, ops=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if cfg.expert_capacity:
            raise ValueError("expert capacity is not supported with expert parallelism")
        self.cfg = cfg
        self.E = cfg.num_experts
        self.e0, self.e1 = local_expert_range(self.E, self.world, self.rank)
        self.E_l = self.e1 - self.e0
        self.ops = ops if ops is not None else _KernelOps()
        self.wt = weights
        self.w_all = self.ops.make_weights(weights)
        self.cfg_local = self.ops.local_config(cfg, self.E_l, 1)
        self.cfg_back = self.ops.local_config(cfg, self.E_l, 1, out_f32=True)

    def _a2a(self, out, inp, out_splits: Sequence[int], in_splits: Sequence[int]):
        self.dist.all_to_all_single(out, inp, output_split_sizes=list(map(int, out_splits)),
                                    input_split_sizes=list(map(int, in_splits)), group=self.group)

    def forward(self, x: torch.Tensor, image_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
        cfg, ops = self.cfg, self.ops
        T, D = x.shape
        dev = x.device
        idx, w = ops.route(cfg, x, self.w_all, image_mask)
        d = ops.dispatch(cfg, x, idx, w)
        counts = send_counts(d["expert_offsets"].cpu().numpy(), self.world)       # [world, E_l]
        send_t = torch.from_numpy(counts.reshape(-1).astype(np.int64)).to(dev)
        recv_t = torch.empty_like(send_t)
        self.dist.all_to_all_single(recv_t, send_t, group=self.group)
        recv_counts = recv_t.cpu().numpy().reshape(self.world, self.E_l)
        send_rows, recv_rows = counts.sum(axis=1), recv_counts.sum(axis=1)
        R, R_in = int(send_rows.sum()), int(recv_rows.sum())
        # rows and routing weights to their owners
        x_in = torch.empty((R_in, D), dtype=x.dtype, device=dev)
        w_in = torch.empty(R_in, dtype=d["row_weight"].dtype, device=dev)
        self._a2a(x_in, d["x_perm"][:R], recv_rows, send_rows)
        self._a2a(w_in, d["row_weight"][:R], recv_rows, send_rows)
        # the owner: group by local expert (top-1 dispatch), the expert GEMMs,
        # then back to received order (top-1 combine)
        y_in = torch.empty((R_in, D), dtype=ops.y_dtype, device=dev)
        if R_in:
            ids = torch.from_numpy(received_expert_ids(recv_counts)).to(dev).view(R_in, 1)
            d2 = ops.dispatch(self.cfg_local, x_in, ids, w_in.view(R_in, 1))
            y2 = ops.grouped_swiglu(self.cfg_local, d2["x_perm"], d2["expert_offsets"], self.w_all,
                                    d2["row_weight"])
            y_in = ops.combine(self.cfg_back, y2, d2["slot_row"], R_in)
        # results home, in x_perm's row order
        y_perm = torch.empty((max(R, 1), D), dtype=ops.y_dtype, device=dev)
        self._a2a(y_perm[:R], y_in, send_rows, recv_rows)
        sh = ops.shared(cfg, x, self.wt) if cfg.shared_intermediate_dim else None
        return ops.combine(cfg, y_perm, d["slot_row"], T, shared_y=sh)
