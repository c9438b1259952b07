"""Expert parallelism (mixture_experts_layer_sqrt_b200.ep).

CPU: the exchange logic (counts, splits, the owner's top-1 regrouping and the
return trip) on two gloo ranks, with the device stages stood in for by the
float64 oracle (test infrastructure only), against the oracle's
single-process layer.  GPU: on one device (a process group of one), the
expert-parallel forward through the library's kernels equals moe_forward.
"""
import os
import types

import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from mixture_experts_layer_sqrt_b200 import ep, synth


def test_plan_helpers():
    offs = np.array([0, 3, 3, 7, 10, 12, 12])      # E = 6 experts
    c = ep.send_counts(offs, 3)                   # 3 ranks, 2 experts each
    np.testing.assert_array_equal(c, [[3, 0], [4, 3], [2, 0]])
    assert ep.local_expert_range(6, 3, 1) == (2, 4)
    with pytest.raises(ValueError):
        ep.local_expert_range(6, 4, 0)
    ids = ep.received_expert_ids(np.array([[2, 1], [0, 3]]))  # from 2 sources, 2 local experts
    np.testing.assert_array_equal(ids, [0, 0, 1, 1, 1, 1])


class OracleOps:
    """The device stages in float64 on the CPU (oracle functions), with the
    binding's tensor shapes: a stand-in for the kernels in this CPU test."""

    y_dtype = torch.float64

    def __init__(self, clamp):
        self.clamp = clamp

    def route(self, cfg, x, w, mask):
        logits = O.router_logits(x.numpy(), w["w_router"].numpy())
        idx, wt, _ = O.route(logits, cfg.top_k, "softmax")
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(wt)

    def dispatch(self, cfg, x, idx, w):
        T, k = idx.shape
        d = O.dispatch(idx.numpy().astype(np.int64), cfg.num_experts, 0)
        R = int(d["offsets"][-1])
        xp = torch.zeros((T * k, x.shape[1]), dtype=x.dtype)
        xp[:R] = x[torch.from_numpy(d["row_token"])]
        rw = torch.zeros(T * k, dtype=w.dtype)
        rw[:R] = w[torch.from_numpy(d["row_token"]), torch.from_numpy(d["row_slot"])]
        return dict(expert_offsets=torch.from_numpy(d["offsets"]), slot_row=torch.from_numpy(d["slot_row"]),
                    x_perm=xp, row_weight=rw)

    def grouped_swiglu(self, cfg, x_perm, offsets, w, row_weight):
        y = np.zeros((x_perm.shape[0], x_perm.shape[1]))
        offs = offsets.numpy()
        for e in range(cfg.num_experts):
            r0, r1 = offs[e], offs[e + 1]
            if r1 > r0:
                y[r0:r1] = row_weight.numpy()[r0:r1, None] * O.swiglu(
                    x_perm.numpy()[r0:r1], w["w_gate"][e].numpy(), w["w_up"][e].numpy(), w["w_down"][e].numpy(),
                    self.clamp)
        return torch.from_numpy(y)

    def combine(self, cfg, y_perm, slot_row, T, shared_y=None):
        sr = slot_row.numpy()
        out = np.zeros((T, y_perm.shape[1]))
        for t in range(T):
            for j in range(sr.shape[1]):
                if sr[t, j] >= 0:
                    out[t] += y_perm.numpy()[sr[t, j]]
        if shared_y is not None:
            out += shared_y.numpy()
        return torch.from_numpy(out)

    def shared(self, cfg, x, wt):
        return torch.from_numpy(O.swiglu(x.numpy(), wt["sh_gate"].numpy(), wt["sh_up"].numpy(),
                                         wt["sh_down"].numpy(), self.clamp))

    def make_weights(self, wt):
        return wt

    def local_config(self, cfg, E_local, k, out_f32=False):
        return types.SimpleNamespace(**dict(vars(cfg), num_experts=E_local, top_k=k, expert_capacity=0,
                                            shared_intermediate_dim=0))


def _layer(E, D, F, Fs, seed):
    rng = np.random.default_rng(seed)
    return dict(w_router=rng.standard_normal((E, D)) / np.sqrt(D),
                w_gate=rng.standard_normal((E, F, D)) / np.sqrt(D), w_up=rng.standard_normal((E, F, D)) / np.sqrt(D),
                w_down=rng.standard_normal((E, D, F)) / np.sqrt(F),
                sh_gate=rng.standard_normal((Fs, D)) / np.sqrt(D), sh_up=rng.standard_normal((Fs, D)) / np.sqrt(D),
                sh_down=rng.standard_normal((D, Fs)) / np.sqrt(Fs))


def _ep_rank(rank, world, port, E, k, T, D, F, Fs, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = _layer(E, D, F, Fs, seed=5)
        e0, e1 = ep.local_expert_range(E, world, rank)
        wt = {n: torch.from_numpy(v) for n, v in L.items()}
        for n in ("w_gate", "w_up", "w_down"):
            wt[n] = wt[n][e0:e1].contiguous()
        x = torch.from_numpy(np.random.default_rng(100 + rank).standard_normal((T + 3 * rank, D)))
        cfg = types.SimpleNamespace(num_experts=E, top_k=k, expert_capacity=0, hidden_dim=D, intermediate_dim=F,
                                    shared_intermediate_dim=Fs, swiglu_clamp=10.0)
        layer = ep.ExpertParallelMoE(cfg, wt, ops=OracleOps(10.0))
        out = layer.forward(x).numpy()
        # the single-process layer on this rank's tokens with every expert
        logits = O.router_logits(x.numpy(), L["w_router"])
        idx, w, _ = O.route(logits, k, "softmax")
        ref = O.moe_forward(x.numpy(), logits, idx, w, lambda e: (L["w_gate"][e], L["w_up"][e], L["w_down"][e]),
                            E, 0, 10.0, "preact", (L["sh_gate"], L["sh_up"], L["sh_down"]))["out"]
        q.put((rank, float(np.abs(out - ref).max()), float(np.abs(ref).max())))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 500)
    procs = [ctx.Process(target=_ep_rank, args=(r, 2, port, 8, 2, 40, 32, 24, 16, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, err, mag in res:
        assert err <= 1e-12 * max(mag, 1.0), (rank, err)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["mixtral_bf16", "sqrt_fp4"])
def test_expert_parallel_one_gpu_matches_forward(name):
    # a process group of one: every row stays local, through both exchanges;
    # the result equals moe_forward bit for bit
    import torch.distributed as dist
    from mixture_experts_layer_sqrt_b200 import build
    build.build()
    from mixture_experts_layer_sqrt_b200 import binding as B, workload as W
    from tests import harness as H
    assert torch.cuda.is_available()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(29700 + (os.getpid() % 200))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        p = H.small(name)
        a = synth.generate(p)
        cfg = W.config_of(p)
        wt = W.device_weights(p, a)
        x = W.to_torch(a["x"])
        mask = W.to_torch(a.get("image_mask"))
        ws = B.workspace(B.workspace_size(cfg, p.T))
        ref = B.forward(cfg, x, B.make_weights(wt), ws, mask)
        layer = ep.ExpertParallelMoE(cfg, wt)
        out = layer.forward(x, mask)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()
