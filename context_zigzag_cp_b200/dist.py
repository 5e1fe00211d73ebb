"""Context parallelism across GPUs: one process per GPU, rank r of a
torch.distributed group of cp ranks.

Each rank keeps its own query shard Q_r (and O_r, dO_r, dQ_r) and receives the
K/V shards of the others, as the Accelerate "Context Parallel" concept guide
describes ("So how does it work?": Q_i stays on rank i while every K_j, V_j
visits it; the partial attentions are combined).  The two exchange orders of
its "all-to-all vs all-gather" section:

  * all-gather: one all-gather brings every K/V shard to every rank, then one
    cp_attn_fwd_rank call attends Q_r to all of them in the plan's visit order;
  * ring: cp steps; at step s rank r holds shard (r - s) mod cp, computes that
    step's partial (cp_attn_fwd_step) while it sends the shard on to rank r+1
    and receives the next one from rank r-1, and the cp partials are combined
    by the LSE-merge kernel (cp_lse_merge).

The backward takes the same two orders:

  * all-gather: K/V gathered, dQ_r and rank r's fp32 share of dK/dV for every
    key in one call (cp_attn_bwd_rank), and a reduce-scatter hands rank j the
    sum for its shard j;
  * ring: cp steps (cp_attn_bwd_step); the shard visited at step s comes with
    its fp32 dK/dV sums, the step adds rank r's share into them and into its
    own fp32 dQ, and the sums travel on with the shard (one hop per step; after
    the last step one more hop hands every shard's sums back to its owner).
    No rank ever holds more than one other shard.

Both cast the fp32 sums to bf16 with cp_f32_to_bf16.

The library moves no data between GPUs; this module runs the collectives with
torch.distributed (NCCL on GPUs).  The kernel calls go through a `kernels`
object (LibraryKernels by default), so the exchange and ordering can be tested
with another backend standing in for the CUDA library.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (Plan, Problem, attn_bwd_rank, attn_bwd_step, attn_fwd_rank, attn_fwd_step,
               f32_to_bf16, lse_merge)


class LibraryKernels:
    """The per-rank calls of libcpattn."""

    def fwd_rank(self, prob, plan, rank, q, k_all, v_all):
        return attn_fwd_rank(prob, plan, rank, q, k_all, v_all)

    def fwd_step(self, prob, plan, rank, step, q, k, v):
        return attn_fwd_step(prob, plan, rank, step, q, k, v)

    def merge(self, o_parts, lse_parts):
        return lse_merge(o_parts, lse_parts)

    def bwd_rank(self, prob, plan, rank, q, k_all, v_all, o, lse, do):
        return attn_bwd_rank(prob, plan, rank, q, k_all, v_all, o, lse, do)

    def bwd_step(self, prob, plan, rank, step, q, k, v, o, lse, do, dq_sum, dk_sum, dv_sum):
        attn_bwd_step(prob, plan, rank, step, q, k, v, o, lse, do, dq_sum, dk_sum, dv_sum)

    def to_bf16(self, x):
        return f32_to_bf16(x)


def _gather_shards(x: torch.Tensor, cp: int, group) -> torch.Tensor:
    """[B, H, 2C, D] local shards of every rank -> [B, H, S, D] in shard order (rank j's
    shard at rows j*2C .. (j+1)*2C of each head)."""
    B, H, n2c, D = x.shape
    parts = torch.empty((cp * B, H, n2c, D), dtype=x.dtype, device=x.device)   # rank-major
    dist.all_gather_into_tensor(parts, x.contiguous(), group=group)
    return parts.view(cp, B, H, n2c, D).permute(1, 2, 0, 3, 4).reshape(B, H, cp * n2c, D).contiguous()


def _reduce_scatter_shards(x: torch.Tensor, cp: int, group) -> torch.Tensor:
    """[B, H, S, D] per-rank partial sums -> rank j gets the sum over ranks of its own
    shard's rows [B, H, 2C, D]."""
    B, H, S, D = x.shape
    n2c = S // cp
    chunks = x.view(B, H, cp, n2c, D).permute(2, 0, 1, 3, 4).reshape(cp * B, H, n2c, D).contiguous()
    out = torch.empty((B, H, n2c, D), dtype=x.dtype, device=x.device)
    dist.reduce_scatter_tensor(out, chunks, op=dist.ReduceOp.SUM, group=group)
    return out


class ContextParallel:
    """Rank r's side of context-parallel attention for one problem.

    prob: the whole problem (seq_len S over cp = the group's size); every rank
    builds the same plan.  Tensors passed in are the rank's local shards,
    [B, heads, 2C, D] in shard order (local row t = shard position r*2C + t)."""

    def __init__(self, prob: Problem, group=None, kernels=None, plan=None):
        self.prob = prob
        self.group = group
        self.rank = dist.get_rank(group)
        self.cp = dist.get_world_size(group)
        if self.cp != prob.cp:
            raise ValueError(f"the group has {self.cp} ranks, the problem cp = {prob.cp}")
        self.kernels = kernels if kernels is not None else LibraryKernels()
        self.plan = plan if plan is not None else Plan(prob)

    def forward(self, q, k, v):
        """Rank r's (O_r, LSE_r) from its local q, k, v shards."""
        if self.prob.rotate == "allgather":
            k_all = _gather_shards(k, self.cp, self.group)
            v_all = _gather_shards(v, self.cp, self.group)
            return self.kernels.fwd_rank(self.prob, self.plan, self.rank, q, k_all, v_all)
        return self._ring_forward(q, k, v)

    def _ring_forward(self, q, k, v):
        r, cp = self.rank, self.cp
        kv = torch.stack([k, v]).contiguous()
        parts_o, parts_l = [], []
        for s in range(cp):
            # pass the held shard on while this step computes with it
            pending = self._shift(kv) if s + 1 < cp else None
            o_s, l_s = self.kernels.fwd_step(self.prob, self.plan, r, s, q, kv[0], kv[1])
            parts_o.append(o_s)
            parts_l.append(l_s)
            if pending is not None:
                for w in pending[0]:
                    w.wait()
                kv = pending[1]
        B, H, n2c, D = q.shape
        o_parts = torch.stack(parts_o).reshape(cp, B * H * n2c, D)
        l_parts = torch.stack(parts_l).reshape(cp, B * H * n2c)
        o, lse = self.kernels.merge(o_parts, l_parts)
        return o.view(B, H, n2c, D), lse.view(B, H, n2c)

    def _peer(self, r):
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def _shift(self, x):
        """Send x to rank r+1 and return what rank r-1 sent (the ring's one hop)."""
        recv = torch.empty_like(x)
        ops = [dist.P2POp(dist.isend, x, self._peer((self.rank + 1) % self.cp), self.group),
               dist.P2POp(dist.irecv, recv, self._peer((self.rank - 1) % self.cp), self.group)]
        return dist.batch_isend_irecv(ops), recv

    def backward(self, q, k, v, o, lse, do):
        """Rank r's (dQ_r, dK_r, dV_r) from its local shards and the upstream dO_r."""
        if self.prob.rotate == "ring":
            return self._ring_backward(q, k, v, o, lse, do)
        k_all = _gather_shards(k, self.cp, self.group)
        v_all = _gather_shards(v, self.cp, self.group)
        dq, dk_part, dv_part = self.kernels.bwd_rank(self.prob, self.plan, self.rank, q, k_all,
                                                     v_all, o, lse, do)
        dk = self.kernels.to_bf16(_reduce_scatter_shards(dk_part, self.cp, self.group))
        dv = self.kernels.to_bf16(_reduce_scatter_shards(dv_part, self.cp, self.group))
        return dq, dk, dv

    def _ring_backward(self, q, k, v, o, lse, do):
        # step s: rank r holds shard (r - s) mod cp with that shard's dK/dV sums so far
        r, cp = self.rank, self.cp
        kv = torch.stack([k, v]).contiguous()
        acc = torch.zeros(kv.shape, dtype=torch.float32, device=kv.device)   # dK, dV sums
        dq = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
        for s in range(cp):
            pending = self._shift(kv) if s + 1 < cp else None   # overlaps the step
            self.kernels.bwd_step(self.prob, self.plan, r, s, q, kv[0], kv[1], o, lse, do, dq,
                                  acc[0], acc[1])
            # the sums move on with their shard; after the last step this hop brings
            # rank r its own shard's sums, completed by every rank
            if cp > 1:
                works, acc = self._shift(acc)
                for w in works:
                    w.wait()
            if pending is not None:
                for w in pending[0]:
                    w.wait()
                kv = pending[1]
        return (self.kernels.to_bf16(dq), self.kernels.to_bf16(acc[0].contiguous()),
                self.kernels.to_bf16(acc[1].contiguous()))
