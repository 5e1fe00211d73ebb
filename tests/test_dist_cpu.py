"""Context parallelism across processes (context_zigzag_cp_b200.dist) with gloo on
CPU, world size 2: the K/V exchange (all-gather, ring send/recv), the order of the
steps and of the merge, and the reduce-scatter of dK/dV, end to end.  The
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

B, HQ, HKV, S, D = 1, 4, 2, 128, 8


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

    def __init__(self, pl, ds, cp):
        import oracle
        self.o, self.pl, self.ds, self.cp = oracle, pl, ds, cp
        self.n2c = S // cp

    def _place(self, x, shard, nheads):
        full = np.zeros((B, nheads, S, D))
        pos = self.pl["perm"][shard * self.n2c:(shard + 1) * self.n2c]
        full[:, :, pos] = x.double().numpy()
        return full

    def _all(self, x_all, nheads):
        full = np.zeros((B, nheads, S, D))
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
        lf = np.zeros((B, HQ, S))
        lf[:, :, self.pl["perm"][rank * self.n2c:(rank + 1) * self.n2c]] = lse.double().numpy()
        dq, dk, dv = self.o.bwd(qf, self._all(k_all, HKV), self._all(v_all, HKV), of, lf, dof,
                                self.ds)
        pos = self.pl["perm"][rank * self.n2c:(rank + 1) * self.n2c]
        return (torch.from_numpy(dq[:, :, pos]).to(torch.bfloat16),
                torch.from_numpy(dk[:, :, self.pl["perm"]]).float(),
                torch.from_numpy(dv[:, :, self.pl["perm"]]).float())

    def to_bf16(self, x):
        return x.to(torch.bfloat16)


# documents for the per-document runs: lengths multiples of 2cp = 4, so every
# document is cut into four chunks of whole rows
CU_DOC = [0, 20, 32, 84, 128]


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
    cu = CU_DOC if shard == "doc" else None
    pl = oracle.plan(S, cp, rotate, cu, shard=shard)
    ds = oracle.doc_start(S, cu)
    t = synth.attn_inputs(B, HQ, HKV, S, D, seed=91, with_dout=True)   # the same on every rank
    n2c = S // cp
    local = lambda x: x[:, :, pl["perm"][rank * n2c:(rank + 1) * n2c]].contiguous()
    prob = cz.Problem(B, S, cp, HQ, HKV, D, rotate)
    ctx = ContextParallel(prob, kernels=OracleKernels(pl, ds, cp), plan=object())
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
@pytest.mark.parametrize("rotate,shard", [("allgather", "sequence"), ("ring", "sequence"),
                                          ("ring", "doc")])
def test_two_ranks_match_unsharded(rotate, shard):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, rotate, shard, q)) for r in range(2)]
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
    t = synth.attn_inputs(B, HQ, HKV, S, D, seed=91, with_dout=True)
    f = lambda x: x.double().numpy()
    cu = CU_DOC if shard == "doc" else None
    ds = oracle.doc_start(S, cu)
    ro, rl = oracle.fwd(f(t["q"]), f(t["k"]), f(t["v"]), ds)
    rq, rk, rv = oracle.bwd(f(t["q"]), f(t["k"]), f(t["v"]), ro, rl, f(t["do"]), ds)
    perm = oracle.plan(S, 2, rotate, cu, shard=shard)["perm"]
    cat = lambda n: np.concatenate([outs[r][n] for r in range(2)], axis=2).astype(np.float64)
    assert_bf16_close(cat("o"), ro[:, :, perm], f"O two ranks {rotate} {shard}")
    assert_lse_close(cat("lse"), rl[:, :, perm], f"LSE two ranks {rotate} {shard}")
    assert_bf16_close(cat("dq"), rq[:, :, perm], f"dQ two ranks {rotate} {shard}")
    assert_bf16_close(cat("dk"), rk[:, :, perm], f"dK two ranks {rotate} {shard}")
    assert_bf16_close(cat("dv"), rv[:, :, perm], f"dV two ranks {rotate} {shard}")
