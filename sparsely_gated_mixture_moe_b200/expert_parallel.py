"""Expert parallelism for the sparsely-gated MoE layer: each of R ranks holds E / R of the
experts and routes its own batch; every token row goes to the rank that holds its expert
and comes back as that expert's output [Shazeer et al., "Outrageously Large Neural
Networks", section "Kombinierte Daten- und Modellparallelität": the gating network and
the rest of the model are replicated, each device keeps a subset of the experts and
receives, from every device, the examples routed to them].

One rank's forward pass:
  1. moe_route and moe_permute on its T tokens (all E experts; capacity per rank, each
     rank's batch being one group for the capacity rule);
  2. the kept rows are already ordered by expert, and so by the rank that holds the
     expert (rank r holds experts [r E/R, (r+1) E/R)); an all-to-all of the per-expert row
     counts tells every rank what it receives, then every (source, expert) run of rows
     travels as its own point-to-point message straight to its place in the receiver's
     expert-major layout (expert by expert, each expert's rows source by source);
  3. moe_expert_ffn_grouped runs the received rows with one group per local expert, so a
     rank's expert step is the single-device expert FFN on the rows it holds;
  4. every (source, expert) run of outputs returns the same way to the slot its rows came
     from, and moe_combine forms y from them as on one device.

The exchange helpers here are plain torch.distributed collectives and point-to-point
operations on tensors of any device (NCCL between GPUs); the compute steps are libmoe's
kernels.  This is the NCCL form of the exchange: the rows cross the links in messages
around the expert products rather than inside them.
"""
from __future__ import annotations

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
    send_counts: List[List[int]]  # [world][E_local]: rows sent to rank d for its expert e
    recv_counts: List[List[int]]  # [world][E_local]: rows received from s for expert e
    send_pos: List[List[int]]     # first row of each sent run in the sender's kept rows
    recv_pos: List[List[int]]     # first row of each received run (expert-major layout)
    expert_offsets: torch.Tensor  # [E_local + 1] int32: each local expert's received rows

    @property
    def rows_out(self) -> int:
        return int(sum(sum(r) for r in self.send_counts))

    @property
    def rows_in(self) -> int:
        return int(sum(sum(r) for r in self.recv_counts))


def _staged(t: torch.Tensor, group) -> bool:
    """Device tensors go through host memory when the group's backend cannot move them
    itself (gloo); NCCL moves them directly."""
    return t.is_cuda and dist.is_initialized() and dist.get_backend(group) != "nccl"


def exchange_plan(kept_per_expert: torch.Tensor, world: int, group=None) -> ExchangePlan:
    """Exchange the per-expert kept-row counts [E] (int, on the collective's device) and
    lay out both directions: each (rank, local expert) run's place in the sender's kept
    rows (expert order) and in the receiver's expert-major layout.  The counts are read
    back to the host once (the messages' sizes)."""
    E = int(kept_per_expert.numel())
    if E % world != 0:
        raise ValueError("E = %d experts do not split evenly over %d ranks" % (E, world))
    El = E // world
    send = kept_per_expert.to(torch.int64).reshape(world, El).contiguous()
    if world == 1:
        recv = send.clone()
    else:
        if _staged(send, group):
            send = send.cpu()
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
    sc = [[int(v) for v in row] for row in send.tolist()]
    rc = [[int(v) for v in row] for row in recv.tolist()]
    send_pos, p = [], 0
    for d in range(world):
        send_pos.append([])
        for e in range(El):
            send_pos[d].append(p)
            p += sc[d][e]
    recv_pos = [[0] * El for _ in range(world)]
    eoff, p = [0], 0
    for e in range(El):
        for s_ in range(world):
            recv_pos[s_][e] = p
            p += rc[s_][e]
        eoff.append(p)
    offsets = torch.tensor(eoff, dtype=torch.int32, device=kept_per_expert.device)
    return ExchangePlan(sc, rc, send_pos, recv_pos, offsets)


def _exchange(src: torch.Tensor, dst: torch.Tensor, out_pos, out_counts, in_pos, in_counts,
              group=None):
    """Send run (d, e) = src[out_pos[d][e] : + out_counts[d][e]] to rank d and receive run
    (s, e) into dst[in_pos[s][e] : + in_counts[s][e]], for every rank and local expert in
    the same order on both sides; this rank's own runs are copied."""
    world = len(out_counts)
    rank = dist.get_rank(group) if world > 1 else 0
    staged = world > 1 and _staged(src, group)
    ops, landings = [], []
    for peer in range(world):
        for e in range(len(out_counts[peer])):
            n_out, n_in = out_counts[peer][e], in_counts[peer][e]
            if peer == rank:
                if n_out:
                    a, b = out_pos[peer][e], in_pos[peer][e]
                    dst[b:b + n_out].copy_(src[a:a + n_out])
                continue
            if n_out:
                a = out_pos[peer][e]
                run = src[a:a + n_out]
                run = run.cpu() if staged else run.contiguous()
                ops.append(dist.P2POp(dist.isend, run, peer, group))
            if n_in:
                b = in_pos[peer][e]
                if staged:
                    buf = torch.empty((n_in,) + tuple(dst.shape[1:]), dtype=dst.dtype)
                    landings.append((buf, b))
                    ops.append(dist.P2POp(dist.irecv, buf, peer, group))
                else:
                    ops.append(dist.P2POp(dist.irecv, dst[b:b + n_in], peer, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    for buf, b in landings:
        dst[b:b + buf.shape[0]].copy_(buf)


def dispatch_rows(rows: torch.Tensor, plan: ExchangePlan, out: torch.Tensor, group=None):
    """The kept rows [rows_out, d] (expert order) to the ranks holding their experts, into
    out[:rows_in] in expert-major order."""
    _exchange(rows, out, plan.send_pos, plan.send_counts, plan.recv_pos, plan.recv_counts,
              group)
    return out[: plan.rows_in]


def return_rows(rows: torch.Tensor, plan: ExchangePlan, out: torch.Tensor, group=None):
    """The expert outputs [rows_in, d] back to their senders, into out[:rows_out] at the
    places the rows left from."""
    _exchange(rows, out, plan.recv_pos, plan.recv_counts, plan.send_pos, plan.send_counts,
              group)
    return out[: plan.rows_out]


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
        moe.moe_expert_ffn_grouped(self.cfg_local, self.x_recv, plan.expert_offsets,
                                   self.E_local, w["w1"], w["w2"], self.h, self.y_recv, self.ws)
        return_rows(self.y_recv, plan, self.y_back, self.group)
        moe.moe_combine(cfg, self.y_back, self.slot_pos, self.gate, self.y, self.ws)
        return self.y


__all__ = ["ExchangePlan", "ExpertParallelMoE", "dispatch_rows", "exchange_plan",
           "local_expert_range", "return_rows"]
