"""The attention kernels' bounded waits, made to run out on the GPU.

cp_selftest_stall runs a forward or backward (the two-pass kernels or the
one-pass kernel) in which CTA 0 of the named kernel
never receives its first K/V tile: its MMA warp's wait must give up after the
wait limit, record CP_ERR_TIMEOUT, and the CTA must drain and free its tensor
memory.  The same process then runs a normal forward and backward and must
still match the oracle, which shows the context survived the teardown."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close, f64, make_case, run_fwd

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000          # 20 ms: far above any wait of this tiny problem
DEFAULT_NS = 2_000_000_000


def _parity_after(case, cp, rotate):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    o, dq, dk, dv = plan.unshard([o, dq, dk, dv])
    lse = lse[:, :, plan.inv_perm.long()]
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"])
    rq, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"])
    assert_bf16_close(f64(o), ro, "O after a timed-out kernel")
    assert_lse_close(f64(lse), rl, "LSE after a timed-out kernel")
    assert_bf16_close(f64(dq), rq, "dQ after a timed-out kernel")
    assert_bf16_close(f64(dk), rk, "dK after a timed-out kernel")
    assert_bf16_close(f64(dv), rv, "dV after a timed-out kernel")


# head_dim 256 runs its own kernels (one forward; dV, dK and dQ passes; no one-pass form)
@pytest.mark.parametrize("kernel,D", [("fwd", 128), ("bwd_dkdv", 128), ("bwd_dq", 128), ("bwd_fused", 128),
                                      ("fwd", 256), ("bwd_dkdv", 256), ("bwd_dq", 256)])
def test_stalled_kernel_times_out_and_context_survives(kernel, D):
    case = make_case(1, 4, 2, 1024, D, 2, 31, with_dout=True)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, 2, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    torch.cuda.synchronize()
    cz.set_wait_limit_ns(LIMIT_NS)
    try:
        if kernel == "fwd":
            cz.selftest_stall(kernel, prob, plan, qs, ks, vs, torch.empty_like(o),
                              torch.empty_like(lse))
        else:
            cz.selftest_stall(kernel, prob, plan, qs, ks, vs, o, lse, dos, torch.empty_like(qs),
                              torch.empty_like(ks), torch.empty_like(vs))
        torch.cuda.synchronize()
        status = cz.get_device_status()
    finally:
        cz.set_wait_limit_ns(DEFAULT_NS)
    assert status == cz._lib.CP_ERR_TIMEOUT
    assert cz.get_device_status() == 0          # read-and-clear
    _parity_after(case, 2, "ring")


def test_stall_rejects_other_kernels():
    case = make_case(1, 2, 2, 512, 64, 2, 32)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, 2, "allgather", "fused")
    with pytest.raises(cz.CPError):
        cz.selftest_stall("merge", prob, plan, qs, ks, vs, o, lse)
