"""The distributed driver (context_zigzag_cp_b200.dist.ContextParallel) with the
library's own kernels (its default LibraryKernels) on one GPU, as a one-rank NCCL
group in both exchange orders.  With one rank the exchange moves nothing, so this
covers what the gloo tests on CPU cannot: the driver's calls into the library
(argument order, shapes and dtypes, the fp32 sums and their casts) on the real
kernels.  The results must equal the whole-sequence calls where those compute
the same values, and match the oracle."""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import context_zigzag_cp_b200 as cz
import oracle
from context_zigzag_cp_b200.dist import ContextParallel
from helpers import assert_bf16_close, assert_lse_close, f64, make_case

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture
def one_rank_group():
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rotate", ["allgather", "ring"])
@pytest.mark.parametrize("D", [128, 256])
def test_one_rank_driver(one_rank_group, rotate, D):
    S = 1024
    case = make_case(1, 4, 2, S, D, 1, 240 + D, with_dout=True)
    prob = cz.Problem(1, S, 1, 4, 2, D, rotate, None, "separate")
    ctx = ContextParallel(prob)
    plan = ctx.plan
    qs, ks, vs, dos = plan.shard([case[n].cuda() for n in ("q", "k", "v", "do")])
    o, lse = ctx.forward(qs, ks, vs)
    dq, dk, dv = ctx.backward(qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    # the forward of one rank is the whole-sequence forward (one step, one merge)
    o_w, l_w = cz.attn_fwd(prob, plan, qs, ks, vs)
    assert torch.equal(o, o_w) and torch.equal(lse, l_w)
    # and so is dQ of the all-gather order (the per-rank call's two passes)
    dq_w, _, _ = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    if rotate == "allgather":
        assert torch.equal(dq, dq_w)
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"], None, case["lk"])
    rq, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"], None, case["lk"])
    perm = plan.perm.cpu().numpy()
    tag = f"one-rank driver D={D} {rotate}"
    assert_bf16_close(f64(o), ro[:, :, perm], "O " + tag)
    assert_lse_close(f64(lse), rl[:, :, perm], "LSE " + tag)
    dq_u, dk_u, dv_u = plan.unshard([dq, dk, dv])
    assert_bf16_close(f64(dq_u), rq, "dQ " + tag)
    assert_bf16_close(f64(dk_u), rk, "dK " + tag)
    assert_bf16_close(f64(dv_u), rv, "dV " + tag)
