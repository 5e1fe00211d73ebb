"""head_dim 256 on the GPU against the oracle: the forward (its own kernel, one
128-row query tile per CTA with Q in tensor memory and 64-key K/V tiles) under
every mask, order, merge and sharding, element by element; the per-rank calls."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close, f64, make_case, random_docs, run_fwd

pytestmark = pytest.mark.gpu


def check_fwd(case, cp, rotate, merge, tag):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge)
    q, k, v = (f64(case[n]) for n in ("q", "k", "v"))
    ro, rl = oracle.fwd(q, k, v, case["ds"], None, case["lk"])
    perm = plan.perm.cpu().numpy()
    tag = f"D=256 {tag} S={q.shape[2]} cp={cp} {rotate} {merge}"
    assert_bf16_close(f64(o), ro[:, :, perm], "O " + tag)
    assert_lse_close(f64(lse), rl[:, :, perm], "LSE " + tag)
    return prob, plan, qs, ks, vs, o, lse


@pytest.mark.parametrize("rotate,merge", [("allgather", "fused"), ("ring", "separate"),
                                          ("ring", "fused"), ("allgather", "separate")])
def test_causal_gqa(rotate, merge):
    case = make_case(1, 8, 2, 2048, 256, 2, 201)
    check_fwd(case, 2, rotate, merge, "causal GQA 8/2")


def test_cp4_mha_batch2():
    case = make_case(2, 4, 4, 4096, 256, 4, 202)
    check_fwd(case, 4, "ring", "separate", "causal MHA batch 2")


def test_cp3_ragged_chunks():
    """cp 3: C = 384, three 128-row tiles per chunk (odd tile counts)."""
    case = make_case(1, 4, 2, 2304, 256, 3, 203)
    check_fwd(case, 3, "allgather", "fused", "causal")


def test_documents_and_window():
    cu = random_docs(4096, 204, 300.0)
    case = make_case(1, 4, 2, 4096, 256, 2, 205, cu=cu)
    check_fwd(case, 2, "ring", "fused", "documents")
    case = make_case(1, 4, 2, 4096, 256, 2, 206, cu=cu, window=200)
    check_fwd(case, 2, "allgather", "separate", "documents + window 200")
    case = make_case(1, 4, 4, 2048, 256, 2, 207, window=77)
    check_fwd(case, 2, "ring", "separate", "window 77")


def test_no_causal_mask():
    case = make_case(1, 4, 2, 2048, 256, 2, 208, causal=False)
    check_fwd(case, 2, "allgather", "fused", "no causal mask")
    check_fwd(case, 2, "ring", "separate", "no causal mask")


def test_per_document_sharding():
    cu = random_docs(4096, 209, 900.0, 128, quantum=512)
    case = make_case(1, 4, 2, 4096, 256, 2, 210, cu=cu, shard="doc")
    check_fwd(case, 2, "ring", "fused", "per-doc")
    check_fwd(case, 2, "allgather", "separate", "per-doc")


def test_amplitude_and_single_tile():
    """Larger scores (amp 2, score std 4: the running max moves by more than the
    lazy-rescale threshold) and cp 1 with one query tile."""
    case = make_case(1, 2, 2, 4096, 256, 2, 211, amp=2.0)
    check_fwd(case, 2, "allgather", "fused", "amp 2")
    case = make_case(1, 2, 1, 256, 256, 1, 212)
    check_fwd(case, 1, "allgather", "separate", "S 256 cp 1")


def test_rank_calls_reassemble_whole():
    S, cp, D = 4096, 4, 256
    case = make_case(1, 4, 2, S, D, cp, 213)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, "ring", "fused")
    prob_sep = prob.with_merge("separate")
    o_sep, lse_sep = cz.attn_fwd(prob_sep, plan, qs, ks, vs)
    n2c = S // cp
    src = plan.src.cpu().numpy()
    loc = lambda x, r: x[:, :, r * n2c:(r + 1) * n2c].contiguous()
    for r in range(cp):
        o_r, l_r = cz.attn_fwd_rank(prob, plan, r, loc(qs, r), ks, vs)
        assert torch.equal(o_r, loc(o, r)) and torch.equal(l_r, loc(lse, r))
        parts = [cz.attn_fwd_step(prob, plan, r, s, loc(qs, r), loc(ks, int(src[r * cp + s])),
                                  loc(vs, int(src[r * cp + s]))) for s in range(cp)]
        om, lm = cz.lse_merge(torch.stack([p[0] for p in parts]).view(cp, -1, D),
                              torch.stack([p[1] for p in parts]).view(cp, -1))
        assert torch.equal(om.view_as(o_r), loc(o_sep, r))
        assert torch.equal(lm.view_as(l_r), loc(lse_sep, r))
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0


# ------------------------------------------------------------------ backward
# Three passes at head_dim 256 (dV, dK: 64-row query units against 128-key
# tiles; dQ: 64-key tiles against 128-row query tiles), against the oracle's
# explicit-P gradients in original order.

def check_bwd(case, cp, rotate, tag):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dq, dk, dv = plan.unshard([dq, dk, dv])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"], None, case["lk"])
    rq, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"], None, case["lk"])
    tag = f"D=256 {tag} S={q.shape[2]} cp={cp} {rotate}"
    assert_bf16_close(f64(dq), rq, "dQ " + tag)
    assert_bf16_close(f64(dk), rk, "dK " + tag)
    assert_bf16_close(f64(dv), rv, "dV " + tag)


@pytest.mark.parametrize("rotate", ["allgather", "ring"])
def test_bwd_causal_gqa(rotate):
    case = make_case(1, 8, 2, 2048, 256, 2, 221, with_dout=True)
    check_bwd(case, 2, rotate, "causal GQA 8/2")


def test_bwd_cp3_batch2():
    case = make_case(2, 4, 4, 2304, 256, 3, 222, with_dout=True)
    check_bwd(case, 3, "ring", "causal MHA batch 2")


def test_bwd_documents_window():
    cu = random_docs(4096, 223, 300.0)
    case = make_case(1, 4, 2, 4096, 256, 2, 224, cu=cu, with_dout=True)
    check_bwd(case, 2, "ring", "documents")
    case = make_case(1, 4, 2, 4096, 256, 2, 225, cu=cu, with_dout=True, window=200)
    check_bwd(case, 2, "allgather", "documents + window 200")


def test_bwd_no_causal_mask_and_per_doc():
    case = make_case(1, 4, 2, 2048, 256, 2, 226, with_dout=True, causal=False)
    check_bwd(case, 2, "allgather", "no causal mask")
    cu = random_docs(4096, 227, 900.0, 128, quantum=512)
    case = make_case(1, 4, 2, 4096, 256, 2, 228, cu=cu, with_dout=True, shard="doc")
    check_bwd(case, 2, "ring", "per-doc")


def test_bwd_one_pass_unsupported():
    case = make_case(1, 2, 2, 512, 256, 2, 229, with_dout=True)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, 2, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    with pytest.raises(cz.CPError, match="UNSUPPORTED"):
        cz.attn_bwd(prob.with_one_pass(True), plan, qs, ks, vs, o, lse, dos)


def test_bwd_rank_calls_sum_to_whole():
    S, cp, D = 2048, 2, 256
    case = make_case(1, 4, 2, S, D, cp, 230, with_dout=True)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    n2c = S // cp
    loc = lambda x, r: x[:, :, r * n2c:(r + 1) * n2c].contiguous()
    dk_sum = torch.zeros(ks.shape, dtype=torch.float32, device="cuda")
    dv_sum = torch.zeros_like(dk_sum)
    for r in range(cp):
        dq_r, dkp, dvp = cz.attn_bwd_rank(prob, plan, r, loc(qs, r), ks, vs, loc(o, r), loc(lse, r),
                                          loc(dos, r))
        assert torch.equal(dq_r, loc(dq, r))
        dk_sum += dkp
        dv_sum += dvp
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dk_u, dv_u = plan.unshard([cz.f32_to_bf16(dk_sum), cz.f32_to_bf16(dv_sum)])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"])
    _, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"])
    assert_bf16_close(f64(dk_u), rk, f"dK D=256 S={S} cp={cp} per-rank sum")
    assert_bf16_close(f64(dv_u), rv, f"dV D=256 S={S} cp={cp} per-rank sum")
