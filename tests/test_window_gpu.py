"""Sliding-window causal attention (the query at q sees keys q - W < k <= q, on
top of the causal and document masks) on the GPU against the oracle: the plan's
pair counts bit-exact, outputs and gradients element by element.  Windows are
chosen to cut tiles at odd places (not multiples of 128), to be narrower than a
tile (including W = 1, where attention is the identity on V) and wider than the
sequence (where the result must equal plain causal attention)."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close, f64, make_case, random_docs, run_fwd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,cp,W,docs", [(8192, 4, 1000, False), (8192, 4, 1, False),
                                         (4096, 2, 333, True), (4096, 2, 9000, True)])
def test_plan_pairs_bit_exact(S, cp, W, docs):
    cu = random_docs(S, 61, 400.0) if docs else None
    ref = oracle.plan(S, cp, "ring", cu, W)
    prob = cz.Problem(1, S, cp, 2, 1, 64, "ring", None if cu is None else torch.from_numpy(cu).cuda(),
                      window=W)
    plan = cz.Plan(prob)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    for key in ("perm", "doc_start", "pairs"):
        assert np.array_equal(getattr(plan, key).cpu().numpy(), ref[key]), key
    assert int(ref["pairs"].sum()) == oracle.causal_pairs(S, cu, W)


def check_fwd(case, cp, rotate, merge):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge)
    q, k, v = (f64(case[n]) for n in ("q", "k", "v"))
    ro, rl = oracle.fwd(q, k, v, case["ds"])
    perm = plan.perm.cpu().numpy()
    tag = f"S={q.shape[2]} cp={cp} W={case['window']} {rotate} {merge}"
    assert_bf16_close(f64(o), ro[:, :, perm], "O " + tag)
    assert_lse_close(f64(lse), rl[:, :, perm], "LSE " + tag)
    return prob, plan, qs, ks, vs, o, lse


@pytest.mark.parametrize("W", [1, 77, 300, 1024, 5000])
def test_fwd_window(W):
    """GQA 8/2, head_dim 128, S 4096 over cp 2; both merges and both orders."""
    case = make_case(1, 8, 2, 4096, 128, 2, 62, window=W)
    check_fwd(case, 2, "allgather", "fused")
    check_fwd(case, 2, "ring", "separate")


def test_fwd_window_docs_d64():
    cu = random_docs(4096, 63, 300.0)
    case = make_case(1, 4, 2, 4096, 64, 4, 64, cu=cu, window=200)
    check_fwd(case, 4, "ring", "fused")
    check_fwd(case, 4, "allgather", "separate")


def test_window_one_is_identity():
    """W = 1: O = V of the query's own position (bf16 V, so within rounding)."""
    case = make_case(1, 4, 2, 2048, 128, 2, 65, window=1)
    _, plan, _, _, _, o, _ = check_fwd(case, 2, "allgather", "fused")
    (ou,) = plan.unshard([o])
    v = f64(case["v"])
    np.testing.assert_allclose(f64(ou)[0, 1], v[0, 0], atol=1e-2)


@pytest.mark.parametrize("W,docs,D,Hkv", [(77, False, 128, 2), (700, True, 128, 2), (1, False, 64, 8),
                                           (3000, False, 64, 2)])
def test_bwd_window(W, docs, D, Hkv):
    """GQA 8/2 except at W = 1, where dV of a key is the sum of its group's dO rows
    (magnitude ~2 for a group of 4, whose bf16 rounding alone averages 2e-3):
    there the heads are MHA, so dV = dO and dK = 0."""
    cu = random_docs(4096, 66, 300.0) if docs else None
    case = make_case(1, 8, Hkv, 4096, D, 2, 67, cu=cu, with_dout=True, window=W)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, 2, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dq, dk, dv = plan.unshard([dq, dk, dv])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"])
    rq, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"])
    tag = f"W={W} docs={docs} D={D}"
    assert_bf16_close(f64(dq), rq, "dQ " + tag)
    assert_bf16_close(f64(dk), rk, "dK " + tag)
    assert_bf16_close(f64(dv), rv, "dV " + tag)
