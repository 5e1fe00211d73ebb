"""Attention without the causal mask (CP_MASK_FULL: every query sees every key)
on the GPU against the oracle: plan pair counts bit-exact, outputs, LSE and
gradients element by element, at sizes that span several tiles per chunk, an
odd number of tiles per chunk (cp 3), GQA, both head dims, both merges and both
visit orders."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close, f64, make_case, run_fwd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,cp", [(8192, 4), (2304, 3)])
def test_plan_pairs_bit_exact(S, cp):
    ref = oracle.plan(S, cp, "ring", causal=False)
    plan = cz.Plan(cz.Problem(1, S, cp, 2, 1, 64, "ring", causal=False))
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    for key in ("perm", "src", "doc_start", "pairs"):
        assert np.array_equal(getattr(plan, key).cpu().numpy(), ref[key]), key
    assert int(ref["pairs"].sum()) == S * S


def check_fwd(case, cp, rotate, merge, scale=0.0):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge, scale)
    q, k, v = (f64(case[n]) for n in ("q", "k", "v"))
    ro, rl = oracle.fwd(q, k, v, case["ds"], scale or None, case["lk"])
    perm = plan.perm.cpu().numpy()
    tag = f"S={q.shape[2]} cp={cp} no causal mask {rotate} {merge}"
    assert_bf16_close(f64(o), ro[:, :, perm], "O " + tag)
    assert_lse_close(f64(lse), rl[:, :, perm], "LSE " + tag)
    return prob, plan, qs, ks, vs, o, lse


@pytest.mark.parametrize("Hq,Hkv,S,D,cp", [(2, 2, 512, 64, 2), (8, 2, 4096, 128, 4),
                                           (4, 2, 2304, 128, 3), (4, 1, 1024, 64, 1)])
def test_fwd_noncausal(Hq, Hkv, S, D, cp):
    case = make_case(1, Hq, Hkv, S, D, cp, 81 + S, causal=False)
    check_fwd(case, cp, "allgather", "fused")
    check_fwd(case, cp, "ring", "separate")


def test_fwd_noncausal_differs_from_causal():
    """Sanity: the unmasked result is far from the causal one on the same inputs."""
    case = make_case(1, 2, 2, 1024, 128, 2, 85, causal=False)
    _, plan, _, _, _, o, _ = run_fwd(cz, case, 2, "ring", "fused")
    q, k, v = (f64(case[n]) for n in ("q", "k", "v"))
    rc, _ = oracle.fwd(q, k, v)
    assert np.abs(f64(o) - rc[:, :, plan.perm.cpu().numpy()]).max() > 0.1


@pytest.mark.parametrize("Hq,Hkv,S,D,cp,scale", [(8, 2, 4096, 128, 2, 0.0), (4, 4, 2304, 128, 3, 0.07),
                                                 (4, 2, 2048, 64, 4, 0.0)])
def test_bwd_noncausal(Hq, Hkv, S, D, cp, scale):
    case = make_case(1, Hq, Hkv, S, D, cp, 86 + S, with_dout=True, causal=False)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, "ring", "fused", scale)
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dq, dk, dv = plan.unshard([dq, dk, dv])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"], scale or None, case["lk"])
    rq, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"], scale or None, case["lk"])
    tag = f"S={S} cp={cp} D={D} no causal mask"
    assert_bf16_close(f64(dq), rq, "dQ " + tag)
    assert_bf16_close(f64(dk), rk, "dK " + tag)
    assert_bf16_close(f64(dv), rv, "dV " + tag)
