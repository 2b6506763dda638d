"""Expert parallelism for the sparsely-gated MoE layer: each of R ranks holds E / R of the
experts and routes its own batch; every token row goes to the rank that holds its expert
and comes back as that expert's output [Shazeer et al., "Outrageously Large Neural
Networks", section "Kombinierte Daten- und Modellparallelität": the gating network and
the rest of the model are replicated, each device keeps a subset of the experts and
receives, from every device, the examples routed to them].

One rank's forward pass:
  1. moe_route and moe_permute on its T tokens (all E experts; capacity per rank, each
     rank's batch being one group for the capacity rule);
  2. the kept rows, already ordered by expert and so by the rank that holds the expert
     (rank r holds experts [r E/R, (r+1) E/R)), go out with one all-to-all; a first
     all-to-all of the per-expert row counts tells every rank what it receives;
  3. moe_expert_ffn_grouped runs the received rows, source by source, each source's rows
     expert by expert (group g = source * E/R + local expert, weights g mod E/R);
  4. the expert outputs return with the reverse all-to-all into the sender's permuted
     order, and moe_combine forms y from them as on one device.

The exchange helpers here are plain torch.distributed collectives on tensors of any
device (NCCL between GPUs); the compute steps are libmoe's kernels.  This is the NCCL
form of the exchange: the rows cross the links in two collective calls around the expert
products rather than inside them.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import List, Optional

import torch
import torch.distributed as dist


def local_expert_range(E: int, world: int, rank: int):
    """Experts [e0, e1) held by `rank` when E experts are split evenly over `world` ranks."""
    if world <= 0 or E % world != 0:
        raise ValueError("E = %d experts do not split evenly over %d ranks" % (E, world))
    n = E // world
    return rank * n, (rank + 1) * n


@dataclass
class ExchangePlan:
    send_splits: List[int]     # rows this rank sends to each rank
    recv_splits: List[int]     # rows this rank receives from each rank
    recv_counts: torch.Tensor  # [world, E_local]: rows from source s for local expert e
    group_offsets: torch.Tensor  # [world * E_local + 1] int32: row groups, source-major

    @property
    def rows_out(self) -> int:
        return int(sum(self.send_splits))

    @property
    def rows_in(self) -> int:
        return int(sum(self.recv_splits))


def exchange_plan(kept_per_expert: torch.Tensor, world: int, group=None) -> ExchangePlan:
    """Exchange the per-expert kept-row counts [E] (int, on the collective's device) and
    derive the row splits of both all-to-alls and the receiver's group offsets.  The
    split lists are read back to the host (the collectives take them as lists)."""
    E = int(kept_per_expert.numel())
    if E % world != 0:
        raise ValueError("E = %d experts do not split evenly over %d ranks" % (E, world))
    send = kept_per_expert.to(torch.int64).reshape(world, E // world).contiguous()
    recv = torch.empty_like(send)
    if world == 1:
        recv.copy_(send)
    else:
        dist.all_to_all_single(recv, send, group=group)
    send_splits = [int(v) for v in send.sum(dim=1).tolist()]
    recv_splits = [int(v) for v in recv.sum(dim=1).tolist()]
    offsets = torch.zeros(recv.numel() + 1, dtype=torch.int64, device=recv.device)
    torch.cumsum(recv.reshape(-1), dim=0, out=offsets[1:])
    return ExchangePlan(send_splits, recv_splits, recv, offsets.to(torch.int32))


def dispatch_rows(rows: torch.Tensor, plan: ExchangePlan, out: torch.Tensor, group=None):
    """All-to-all of the kept rows [rows_out, d] (in expert order) into out[:rows_in]."""
    dst = out[: plan.rows_in]
    if len(plan.send_splits) == 1:
        dst.copy_(rows[: plan.rows_out])
    else:
        dist.all_to_all_single(dst, rows[: plan.rows_out].contiguous(), plan.recv_splits,
                               plan.send_splits, group=group)
    return dst


def return_rows(rows: torch.Tensor, plan: ExchangePlan, out: torch.Tensor, group=None):
    """The reverse all-to-all: rows [rows_in, d] computed here go back to their senders,
    into out[:rows_out] in the sender's original (expert) order."""
    dst = out[: plan.rows_out]
    if len(plan.send_splits) == 1:
        dst.copy_(rows[: plan.rows_in])
    else:
        dist.all_to_all_single(dst, rows[: plan.rows_in].contiguous(), plan.send_splits,
                               plan.recv_splits, group=group)
    return dst


class ExpertParallelMoE:
    """One rank's share of an expert-parallel layer on its GPU.

    cfg: the layer seen from this rank (T = this rank's tokens, E = all experts; bf16).
    weights: w_gate [E, d] (and w_noise, logit_bias) as for MoELayer, and this rank's
    experts only: w1 [E/R, d_ff, d], w2 [E/R, d, d_ff].  Buffers are sized for the worst
    case: every rank sending all its T*k rows here."""

    def __init__(self, cfg, weights: dict, group=None, device="cuda"):
        import sparsely_gated_mixture_moe_b200 as moe
        self.moe = moe
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        if cfg.dtype != moe.DTYPE["bf16"]:
            raise ValueError("expert parallelism runs bf16 layers")
        E, T, k, d, f = cfg.E, cfg.T, cfg.k, cfg.d_model, cfg.d_ff
        self.e0, self.e1 = local_expert_range(E, self.world, self.rank)
        self.E_local = self.e1 - self.e0
        self.cfg = cfg
        self.cfg_local = moe.MoEConfig.from_buffer_copy(cfg)
        self.cfg_local.E = self.E_local
        self.w = moe.prepare_weights(self.cfg_local, {kk: v for kk, v in weights.items()
                                                      if kk in ("w1", "w2")})
        for kk in ("w_gate", "w_noise", "logit_bias"):
            if weights.get(kk) is not None:
                self.w[kk] = weights[kk]
        if self.w["w1"].shape[0] != self.E_local or self.w["w2"].shape[0] != self.E_local:
            raise ValueError("w1/w2 must hold this rank's %d experts" % self.E_local)
        n, cap = T * k, self.world * T * k
        bf16 = torch.bfloat16
        hdt = torch.float16 if cfg.hidden_f16 else bf16
        self.idx = torch.empty(T, k, dtype=torch.int32, device=device)
        self.gate = torch.empty(T, k, dtype=torch.float32, device=device)
        self.counts = torch.empty(E, dtype=torch.int32, device=device)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=device)
        self.perm_src = torch.empty(max(n, 1), dtype=torch.int32, device=device)
        self.slot_pos = torch.empty(max(n, 1), dtype=torch.int32, device=device)
        self.x_perm = torch.empty(max(n, 1), d, dtype=bf16, device=device)
        self.x_recv = torch.empty(max(cap, 1), d, dtype=bf16, device=device)
        self.h = torch.empty(max(cap, 1), f, dtype=hdt, device=device)
        self.y_recv = torch.empty(max(cap, 1), d, dtype=torch.float32, device=device)
        self.y_back = torch.empty(max(n, 1), d, dtype=torch.float32, device=device)
        self.y = torch.empty(T, d, dtype=bf16 if cfg.y_bf16 else torch.float32, device=device)
        self.ws = moe.workspace(cfg, device)
        self.plan: Optional[ExchangePlan] = None

    def forward(self, x: torch.Tensor, noise: Optional[torch.Tensor] = None):
        moe, w, cfg = self.moe, self.w, self.cfg
        moe.moe_route(cfg, x, w["w_gate"], self.idx, self.gate, self.ws, w_noise=w.get("w_noise"),
                      noise=noise, logit_bias=w.get("logit_bias"))
        moe.moe_permute(cfg, self.idx, x, self.counts, self.offsets, self.perm_src, self.slot_pos,
                        self.x_perm, self.ws)
        kept = self.offsets[1:] - self.offsets[:-1]
        self.plan = plan = exchange_plan(kept, self.world, self.group)
        recv = dispatch_rows(self.x_perm, plan, self.x_recv, self.group)
        del recv  # the grouped FFN reads x_recv by its row capacity
        groups = self.world * self.E_local
        moe.moe_expert_ffn_grouped(self.cfg_local, self.x_recv, plan.group_offsets, groups,
                                   w["w1"], w["w2"], self.h, self.y_recv, self.ws)
        return_rows(self.y_recv, plan, self.y_back, self.group)
        moe.moe_combine(cfg, self.y_back, self.slot_pos, self.gate, self.y, self.ws)
        return self.y


__all__ = ["ExchangePlan", "ExpertParallelMoE", "dispatch_rows", "exchange_plan",
           "local_expert_range", "return_rows"]
