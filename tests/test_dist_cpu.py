"""Context parallelism across processes (context_zigzag_cp_b200.dist) with gloo on
CPU, world sizes 2 and 3: the K/V exchange (all-gather, ring send/recv), the order
of the steps and of the merge, the reduce-scatter of dK/dV (all-gather order)
and the dK/dV sums that travel with their shard (ring order), end to end.  The
per-rank kernels are stood in by the oracle (the library's own per-rank calls
are checked on a GPU by test_rank_gpu.py); each rank ends up with its shard of
O, LSE, dQ, dK, dV, and rank 0 compares the reassembled result with the oracle's
unsharded attention."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

B, HQ, HKV, D = 1, 4, 2, 8


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleKernels:
    """The per-rank calls computed by the oracle from the shards the rank holds.
    Each call only sees what the real call would: the rank's local rows and the
    K/V rows handed to it; they are placed at their original positions (from the
    plan's perm) in otherwise-zero full-length arrays for the oracle."""

    def __init__(self, pl, ds, cp, S):
        import oracle
        self.o, self.pl, self.ds, self.cp, self.S = oracle, pl, ds, cp, S
        self.n2c = S // cp

    def _place(self, x, shard, nheads):
        full = np.zeros((B, nheads, self.S, D))
        pos = self.pl["perm"][shard * self.n2c:(shard + 1) * self.n2c]
        full[:, :, pos] = x.double().numpy()
        return full

    def _all(self, x_all, nheads):
        full = np.zeros((B, nheads, self.S, D))
        full[:, :, self.pl["perm"]] = x_all.double().numpy()
        return full

    def fwd_step(self, prob, plan, rank, step, q, k, v):
        j = int(self.pl["src"][rank * self.cp + step])
        po, pl_ = self.o.partial(self._place(q, rank, HQ), self._place(k, j, HKV),
                                 self._place(v, j, HKV), self.pl["perm"], self.cp, rank, j, self.ds)
        return (torch.from_numpy(po).float().view(B, HQ, self.n2c, D),
                torch.from_numpy(pl_).float().view(B, HQ, self.n2c))

    def merge(self, o_parts, lse_parts):
        o, lse = self.o.lse_merge(o_parts.double().numpy(), lse_parts.double().numpy())
        return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).float()

    def fwd_rank(self, prob, plan, rank, q, k_all, v_all):
        qf, kf, vf = self._place(q, rank, HQ), self._all(k_all, HKV), self._all(v_all, HKV)
        parts = [self.o.partial(qf, kf, vf, self.pl["perm"], self.cp, rank,
                                int(self.pl["src"][rank * self.cp + s]), self.ds)
                 for s in range(self.cp)]
        o, lse = self.o.lse_merge(np.stack([p[0].reshape(-1, D) for p in parts]),
                                  np.stack([p[1].reshape(-1) for p in parts]))
        return (torch.from_numpy(o).to(torch.bfloat16).view(B, HQ, self.n2c, D),
                torch.from_numpy(lse).float().view(B, HQ, self.n2c))

    def bwd_rank(self, prob, plan, rank, q, k_all, v_all, o, lse, do):
        # rows of other ranks carry dO = 0: they add nothing to dK / dV
        qf, of, dof = (self._place(x, rank, HQ) for x in (q, o, do))
        lf = self._place_lse(lse, rank)
        dq, dk, dv = self.o.bwd(qf, self._all(k_all, HKV), self._all(v_all, HKV), of, lf, dof,
                                self.ds)
        pos = self.pl["perm"][rank * self.n2c:(rank + 1) * self.n2c]
        return (torch.from_numpy(dq[:, :, pos]).to(torch.bfloat16),
                torch.from_numpy(dk[:, :, self.pl["perm"]]).float(),
                torch.from_numpy(dv[:, :, self.pl["perm"]]).float())

    def _place_lse(self, lse, rank):
        lf = np.zeros((B, HQ, self.S))
        lf[:, :, self.pl["perm"][rank * self.n2c:(rank + 1) * self.n2c]] = lse.double().numpy()
        return lf

    def bwd_step(self, prob, plan, rank, step, q, k, v, o, lse, do, dq_sum, dk_sum, dv_sum):
        # the oracle's unit backward: rank r's rows against shard j's keys
        j = int(self.pl["src"][rank * self.cp + step])
        dq, dk, dv = self.o.bwd_partial(self._place(q, rank, HQ), self._place(k, j, HKV),
                                        self._place(v, j, HKV), self._place(o, rank, HQ),
                                        self._place_lse(lse, rank), self._place(do, rank, HQ),
                                        self.pl["perm"], self.cp, rank, j, self.ds)
        dq_sum += torch.from_numpy(dq).float()
        dk_sum += torch.from_numpy(dk).float()
        dv_sum += torch.from_numpy(dv).float()

    def to_bf16(self, x):
        return x.to(torch.bfloat16)


# documents for the per-document runs: lengths multiples of 2cp, so every
# document is cut into 2cp chunks of whole rows
CU_DOC = {1: [0, 20, 32, 84, 128], 2: [0, 20, 32, 84, 128], 3: [0, 48, 66, 150, 192]}
SEQ = {1: 128, 2: 128, 3: 192}     # S / 2cp whole rows per chunk


def _worker(rank, world, port, rotate, shard, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import context_zigzag_cp_b200 as cz
    from context_zigzag_cp_b200.dist import ContextParallel
    import oracle
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    cp = world
    S = SEQ[cp]
    cu = CU_DOC[cp] if shard == "doc" else None
    pl = oracle.plan(S, cp, rotate, cu, shard=shard)
    ds = oracle.doc_start(S, cu)
    t = synth.attn_inputs(B, HQ, HKV, S, D, seed=91, with_dout=True)   # the same on every rank
    n2c = S // cp
    local = lambda x: x[:, :, pl["perm"][rank * n2c:(rank + 1) * n2c]].contiguous()
    prob = cz.Problem(B, S, cp, HQ, HKV, D, rotate)
    ctx = ContextParallel(prob, kernels=OracleKernels(pl, ds, cp, S), plan=object())
    o, lse = ctx.forward(local(t["q"]), local(t["k"]), local(t["v"]))
    dq, dk, dv = ctx.backward(local(t["q"]), local(t["k"]), local(t["v"]), o, lse, local(t["do"]))
    outs = [None] * world
    dist.all_gather_object(outs, {n: x.float().numpy() for n, x in
                                  dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()})
    dist.barrier()
    dist.destroy_process_group()
    q_out.put((rank, outs if rank == 0 else None))


# shard "doc": the driver with a per-document plan (the permutation and the
# document mask change; the exchange, the merge order and the reduce-scatter
# are the same)
# world 3: the ring's direction matters (rank r+1 and rank r-1 differ); world 1:
# a ring of one rank has no hop
@pytest.mark.parametrize("world,rotate,shard", [(1, "ring", "sequence"), (1, "allgather", "doc"),
                                                (2, "allgather", "sequence"), (2, "ring", "sequence"),
                                                (2, "ring", "doc"), (3, "ring", "sequence"),
                                                (3, "ring", "doc"), (3, "allgather", "doc")])
def test_ranks_match_unsharded(world, rotate, shard):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rotate, shard, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    outs = res[0]
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    from helpers import assert_bf16_close, assert_lse_close
    S = SEQ[world]
    t = synth.attn_inputs(B, HQ, HKV, S, D, seed=91, with_dout=True)
    f = lambda x: x.double().numpy()
    cu = CU_DOC[world] if shard == "doc" else None
    ds = oracle.doc_start(S, cu)
    ro, rl = oracle.fwd(f(t["q"]), f(t["k"]), f(t["v"]), ds)
    rq, rk, rv = oracle.bwd(f(t["q"]), f(t["k"]), f(t["v"]), ro, rl, f(t["do"]), ds)
    perm = oracle.plan(S, world, rotate, cu, shard=shard)["perm"]
    cat = lambda n: np.concatenate([outs[r][n] for r in range(world)], axis=2).astype(np.float64)
    assert_bf16_close(cat("o"), ro[:, :, perm], f"O {world} ranks {rotate} {shard}")
    assert_lse_close(cat("lse"), rl[:, :, perm], f"LSE {world} ranks {rotate} {shard}")
    assert_bf16_close(cat("dq"), rq[:, :, perm], f"dQ {world} ranks {rotate} {shard}")
    assert_bf16_close(cat("dk"), rk[:, :, perm], f"dK {world} ranks {rotate} {shard}")
    assert_bf16_close(cat("dv"), rv[:, :, perm], f"dV {world} ranks {rotate} {shard}")
