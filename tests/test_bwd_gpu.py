"""GPU backward (dQ, dK, dV) against the oracle's explicit-P gradients.

Small and mid sizes: every element.  Full sizes: dQ on sampled rows and dK/dV on
sampled keys (keys near the end of the sequence and of documents, whose rows
the oracle can recompute one by one), plus the identities that hold at any size:
sum_k dV_k = sum of dO over the group's rows, and sum_k dK_k = 0."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
import synth
from helpers import (assert_bf16_close, bf16_operand_attention, f64, make_case, random_docs,
                     run_fwd)

pytestmark = pytest.mark.gpu


def run_bwd(case, cp, rotate="allgather", merge="fused", scale=0.0):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge, scale)
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dq, dk, dv = plan.unshard([dq, dk, dv])
    return prob, plan, dq, dk, dv


def check_full(case, cp, rotate, scale=0.0, emulate=False):
    _, _, dq, dk, dv = run_bwd(case, cp, rotate, scale=scale)
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    o, lse = oracle.fwd(q, k, v, case["ds"], scale or None)
    rq, rk, rv = oracle.bwd(q, k, v, o, lse, do, case["ds"], scale or None)
    tag = f"S={q.shape[2]} cp={cp} {rotate}"
    assert_bf16_close(f64(dq), rq, "dQ " + tag)
    assert_bf16_close(f64(dk), rk, "dK " + tag)
    assert_bf16_close(f64(dv), rv, "dV " + tag)
    if emulate:
        # the kernels carry exactly the rounding of bf16 P / dS operands: their result
        # sits much closer to that emulation than to the fp64 reference
        _, eq, ek, ev = bf16_operand_attention(q, k, v, do, case["ds"],
                                               scale or 1.0 / np.sqrt(q.shape[-1]))
        for name, got, emu, ref in (("dQ", dq, eq, rq), ("dK", dk, ek, rk), ("dV", dv, ev, rv)):
            d_emu = np.abs(f64(got) - emu)
            d_ref = np.abs(f64(got) - ref)
            assert d_emu.mean() < 0.5 * d_ref.mean(), (name, d_emu.mean(), d_ref.mean())


def test_small_d64():
    case = make_case(1, 2, 2, 512, 64, 2, 0, with_dout=True)
    check_full(case, 2, "allgather")


def test_fb8k():
    """S 8192, cp 4, 8 heads MHA, head_dim 128, all-gather order."""
    case = make_case(1, 8, 8, 8192, 128, 4, 1, with_dout=True)
    check_full(case, 4, "allgather")


@pytest.mark.parametrize("D", [64, 128])
def test_gqa_docs_small(D):
    cu = random_docs(4096, 21, 150.0)
    case = make_case(1, 8, 2, 4096, D, 2, 22, cu=cu, with_dout=True)
    check_full(case, 2, "ring", emulate=(D == 128))


def test_batch2_cp3_scale():
    """Batch 2, cp 3 (three query tiles per chunk), GQA 4/2, a non-default scale."""
    case = make_case(2, 4, 2, 2304, 128, 3, 23, with_dout=True)
    check_full(case, 3, "ring", scale=0.07, emulate=True)


# ----------------------------------------------------------------- full sizes, sampled

def check_sampled(name, rotate, n_rows=96, n_keys=24):
    w = synth.WORKLOADS[name]
    t = synth.workload_inputs(w, with_dout=True)
    S, g = w.seq_len, w.num_heads // w.num_kv_heads
    ds = oracle.doc_start(S, t["cu_seqlens"])
    case = dict(q=t["q"], k=t["k"], v=t["v"], do=t["do"], cu_seqlens=t["cu_seqlens"], ds=ds)
    _, _, dq, dk, dv = run_bwd(case, w.cp, rotate)
    rng = np.random.default_rng(w.seed + 200)
    groups = [0, int(rng.integers(1, w.num_kv_heads))]
    qh = [gi * g + i for gi in groups for i in range(g)]
    q, do = f64(t["q"][:, qh]), f64(t["do"][:, qh])
    k, v = f64(t["k"][:, groups]), f64(t["v"][:, groups])
    # dQ on sampled rows
    rows = np.unique(rng.integers(0, S, n_rows))
    flat = np.concatenate([hi * S + rows for hi in range(len(qh))])
    rq = oracle.bwd_dq_rows(q, k, v, do, flat, ds)
    gq = f64(dq[0, qh][:, rows]).reshape(-1, w.head_dim)
    assert_bf16_close(gq, rq, f"dQ {name}")
    # dK / dV on keys whose attending rows are few: the last keys of the sequence
    # and of its documents
    ends = [S - 1 - i for i in range(n_keys // 2)]
    if t["cu_seqlens"] is not None:
        cu = t["cu_seqlens"]
        ends += [int(cu[i + 1]) - 1 - int(rng.integers(0, 64)) for i in range(len(cu) - 1)
                 if cu[i + 1] - cu[i] <= 4096][: n_keys // 2]
    keys = np.unique(np.clip(np.asarray(ends), 0, S - 1))
    flatk = np.concatenate([gi * S + keys for gi in range(len(groups))])
    rk, rv = oracle.bwd_dkv_keys(q, k, v, do, flatk, ds)
    assert_bf16_close(f64(dk[0, groups][:, keys]).reshape(-1, w.head_dim), rk, f"dK {name}")
    assert_bf16_close(f64(dv[0, groups][:, keys]).reshape(-1, w.head_dim), rv, f"dV {name}")
    # identities over the whole sequence (every KV head)
    dv_sum = dv.double().sum(dim=2)[0]                                  # [Hkv, D]
    do_sum = t["do"].cuda().double().sum(dim=2)[0].view(w.num_kv_heads, g, -1).sum(1)
    assert (dv_sum - do_sum).abs().max().item() < 2e-2 * np.sqrt(S)
    dk_sum = dk.double().sum(dim=2)[0]
    assert dk_sum.abs().max().item() < 2e-2 * np.sqrt(S)
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()


def test_gqa32k_ring_sampled():
    check_sampled("gqa32k", "ring")


def test_docs64k_sampled():
    check_sampled("docs64k", "ring")


@pytest.mark.parametrize("rotate", ["allgather", "ring"])
def test_long128k_sampled(rotate):
    check_sampled("long128k", rotate, n_rows=48, n_keys=16)
