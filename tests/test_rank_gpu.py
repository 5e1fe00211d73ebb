"""The per-rank calls (cp_attn_fwd_rank, cp_attn_fwd_step, cp_attn_bwd_rank,
cp_attn_bwd_step, cp_f32_to_bf16) on one GPU: every rank of a cp group run one after another, the
K/V exchange done by slicing (all-gather: the whole shard-order K/V; ring step
s: shard src[r][s]) and the dK/dV reduce-scatter by a sum.  The ranks' results
reassembled must equal the whole-sequence calls (the same kernels restricted to
one rank's rows: bit for bit for the forward and dQ) and the oracle."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close, f64, make_case, random_docs, run_fwd

pytestmark = pytest.mark.gpu


def _local(x, r, n2c):
    return x[:, :, r * n2c:(r + 1) * n2c].contiguous()


# docs: False (no documents), True (packed documents, sequence zigzag) or "per_doc"
# (whole-tile documents, every one cut into 2cp chunks)
@pytest.mark.parametrize("Hq,Hkv,S,D,cp,docs,causal", [
    (8, 2, 4096, 128, 4, False, True), (4, 2, 2304, 128, 3, True, True),
    (4, 4, 2048, 64, 2, False, True), (4, 2, 2048, 128, 4, False, False),
    (8, 2, 6144, 128, 2, "per_doc", True), (4, 2, 6144, 64, 3, "per_doc", True)])
def test_ranks_reassemble_whole(Hq, Hkv, S, D, cp, docs, causal):
    per_doc = docs == "per_doc"
    cu = (random_docs(S, 95, 1500.0, quantum=256 * cp) if per_doc else
          random_docs(S, 95, 300.0) if docs else None)
    case = make_case(1, Hq, Hkv, S, D, cp, 96 + S, cu=cu, with_dout=True, causal=causal,
                     shard="doc" if per_doc else "sequence")
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    # the per-rank backward is the two-pass form: compare with the whole two-pass one
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    prob_sep = prob.with_merge("separate")
    o_sep, lse_sep = cz.attn_fwd(prob_sep, plan, qs, ks, vs)
    n2c = S // cp
    src = plan.src.cpu().numpy()
    ro, rl, rq = [], [], []
    dk_sum = torch.zeros(ks.shape, dtype=torch.float32, device="cuda")
    dv_sum = torch.zeros_like(dk_sum)
    for r in range(cp):
        q_r, do_r = _local(qs, r, n2c), _local(dos, r, n2c)
        # all-gather order: one call against every shard
        o_r, l_r = cz.attn_fwd_rank(prob, plan, r, q_r, ks, vs)
        assert torch.equal(o_r, _local(o, r, n2c)) and torch.equal(l_r, _local(lse, r, n2c))
        o_r2, l_r2 = cz.attn_fwd_rank(prob_sep, plan, r, q_r, ks, vs)
        assert torch.equal(o_r2, _local(o_sep, r, n2c)) and torch.equal(l_r2, _local(lse_sep, r, n2c))
        # ring order: one partial per step against the shard held then, merged in step order
        parts = [cz.attn_fwd_step(prob, plan, r, s, q_r, _local(ks, int(src[r * cp + s]), n2c),
                                  _local(vs, int(src[r * cp + s]), n2c)) for s in range(cp)]
        om, lm = cz.lse_merge(torch.stack([p[0] for p in parts]).view(cp, -1, D),
                              torch.stack([p[1] for p in parts]).view(cp, -1))
        assert torch.equal(om.view_as(o_r), _local(o_sep, r, n2c))
        assert torch.equal(lm.view_as(l_r), _local(lse_sep, r, n2c))
        # backward: dQ of the rank's rows, its fp32 share of dK / dV of every key
        dq_r, dkp, dvp = cz.attn_bwd_rank(prob, plan, r, q_r, ks, vs, o_r, l_r, do_r)
        assert torch.equal(dq_r, _local(dq, r, n2c))
        dk_sum += dkp
        dv_sum += dvp
        ro.append(o_r); rl.append(l_r); rq.append(dq_r)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dk_r, dv_r = cz.f32_to_bf16(dk_sum), cz.f32_to_bf16(dv_sum)
    assert torch.equal(dk_r, dk_sum.to(torch.bfloat16))        # the cast is round-to-nearest-even
    # against the oracle, in original order
    (dk_u, dv_u) = plan.unshard([dk_r, dv_r])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ref_o, ref_l = oracle.fwd(q, k, v, case["ds"], None, case["lk"])
    _, rk, rv = oracle.bwd(q, k, v, ref_o, ref_l, do, case["ds"], None, case["lk"])
    tag = f"S={S} cp={cp} per-rank sum"
    assert_bf16_close(f64(dk_u), rk, "dK " + tag)
    assert_bf16_close(f64(dv_u), rv, "dV " + tag)


def test_rank_calls_reject_bad_rank_and_step():
    case = make_case(1, 2, 2, 512, 64, 2, 97)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, 2, "ring", "fused")
    q0 = _local(qs, 0, 256)
    with pytest.raises(cz.CPError):
        cz.attn_fwd_rank(prob, plan, 2, q0, ks, vs)
    with pytest.raises(cz.CPError):
        cz.attn_fwd_step(prob, plan, 0, 2, q0, _local(ks, 0, 256), _local(vs, 0, 256))


# The ring form of the backward (cp_attn_bwd_step), every rank and step run in
# the ring's order on one GPU: at step s rank r adds its share into its own fp32
# dQ and into the fp32 dK / dV sums of shard src[r][s], which in a ring travel
# with that shard.  The cast sums are compared with the oracle, and with the
# per-rank calls' sums (the same per-rank fp32 shares, added in another order).
@pytest.mark.parametrize("Hq,Hkv,S,D,cp,docs,causal,window", [
    (8, 2, 4096, 128, 4, False, True, 0), (4, 2, 2304, 128, 3, True, True, 0),
    (4, 4, 2048, 64, 2, False, True, 0), (4, 2, 2048, 128, 2, False, False, 0),
    (4, 2, 4096, 128, 2, True, True, 300), (8, 2, 6144, 128, 2, "per_doc", True, 0),
    (8, 2, 2048, 256, 2, False, True, 0), (4, 2, 4096, 256, 2, "per_doc", True, 0)])
def test_ring_backward_steps(Hq, Hkv, S, D, cp, docs, causal, window):
    per_doc = docs == "per_doc"
    cu = (random_docs(S, 98, 1500.0, quantum=256 * cp) if per_doc else
          random_docs(S, 98, 300.0) if docs else None)
    case = make_case(1, Hq, Hkv, S, D, cp, 99 + S + D, cu=cu, with_dout=True, causal=causal,
                     window=window, shard="doc" if per_doc else "sequence")
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    n2c = S // cp
    src = plan.src.cpu().numpy()
    assert all(int(src[r * cp + s]) == (r - s) % cp for r in range(cp) for s in range(cp))
    f32 = dict(dtype=torch.float32, device="cuda")
    dq = [torch.zeros(_local(qs, r, n2c).shape, **f32) for r in range(cp)]
    acc_k = [torch.zeros(_local(ks, j, n2c).shape, **f32) for j in range(cp)]
    acc_v = [torch.zeros_like(a) for a in acc_k]
    for s in range(cp):
        for r in range(cp):
            j = int(src[r * cp + s])
            cz.attn_bwd_step(prob, plan, r, s, _local(qs, r, n2c), _local(ks, j, n2c),
                             _local(vs, j, n2c), _local(o, r, n2c), _local(lse, r, n2c),
                             _local(dos, r, n2c), dq[r], acc_k[j], acc_v[j])
    # the per-rank calls: the same fp32 shares of dK / dV
    pk = torch.zeros(ks.shape, **f32)
    pv = torch.zeros_like(pk)
    for r in range(cp):
        _, dkp, dvp = cz.attn_bwd_rank(prob, plan, r, _local(qs, r, n2c), ks, vs, _local(o, r, n2c),
                                       _local(lse, r, n2c), _local(dos, r, n2c))
        pk += dkp
        pv += dvp
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    ring_k, ring_v = torch.cat(acc_k, dim=2), torch.cat(acc_v, dim=2)
    for a, b, name in ((ring_k, pk, "dK"), (ring_v, pv, "dV")):
        tol = 1e-5 * float(b.abs().max()) + 1e-30
        err = float((a - b).abs().max())
        assert err <= tol, f"{name} ring sums vs per-rank sums: max |diff| {err:.3g} > {tol:.3g}"
    dq_u, dk_u, dv_u = plan.unshard([cz.f32_to_bf16(torch.cat(dq, dim=2)),
                                     cz.f32_to_bf16(ring_k), cz.f32_to_bf16(ring_v)])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ref_o, ref_l = oracle.fwd(q, k, v, case["ds"], None, case["lk"])
    rq, rk, rv = oracle.bwd(q, k, v, ref_o, ref_l, do, case["ds"], None, case["lk"])
    tag = f"ring steps S={S} D={D} cp={cp} docs={docs} causal={causal} window={window}"
    assert_bf16_close(f64(dq_u), rq, "dQ " + tag)
    assert_bf16_close(f64(dk_u), rk, "dK " + tag)
    assert_bf16_close(f64(dv_u), rv, "dV " + tag)


def test_bwd_step_rejects_bad_args():
    case = make_case(1, 2, 2, 512, 64, 2, 97, with_dout=True)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, 2, "ring", "fused")
    (dos,) = plan.shard([case["do"].cuda()])
    loc = lambda x: _local(x, 0, 256)
    f32 = dict(dtype=torch.float32, device="cuda")
    dq = torch.zeros(loc(qs).shape, **f32)
    dk = torch.zeros(loc(ks).shape, **f32)
    dv = torch.zeros_like(dk)
    args = (loc(qs), loc(ks), loc(vs), loc(o), loc(lse), loc(dos))
    with pytest.raises(cz.CPError):
        cz.attn_bwd_step(prob, plan, 0, 2, *args, dq, dk, dv)
    with pytest.raises(cz.CPError):
        cz.attn_bwd_step(prob, plan, -1, 0, *args, dq, dk, dv)
    with pytest.raises(ValueError):     # bf16 where the fp32 sum belongs
        cz.attn_bwd_step(prob, plan, 0, 0, *args, dq.to(torch.bfloat16), dk, dv)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
