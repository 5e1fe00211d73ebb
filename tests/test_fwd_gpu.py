"""GPU forward (plan + gather + per-rank attention + merge) against the oracle.

Small and mid sizes are compared element by element on every output; the
full-size workloads are compared on sampled rows that the oracle computes one
by one (two whole KV groups, a few hundred rows per query head, including every
chunk's first and last rows)."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
import synth
from helpers import (assert_bf16_close, assert_lse_close, f64, make_case, random_docs, run_fwd)

pytestmark = pytest.mark.gpu


def check_full(case, cp, rotate, merge, scale=0.0):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge, scale)
    q, k, v = (f64(case[n]) for n in ("q", "k", "v"))
    ro, rl = oracle.fwd(q, k, v, case["ds"], scale or None)
    perm = plan.perm.cpu().numpy()
    assert np.array_equal(perm, oracle.plan(q.shape[2], cp, rotate, case["cu_seqlens"])["perm"])
    tag = f"S={q.shape[2]} cp={cp} {rotate} {merge}"
    assert_bf16_close(f64(o), ro[:, :, perm], "O " + tag)
    assert_lse_close(f64(lse), rl[:, :, perm], "LSE " + tag)
    return o, lse


@pytest.mark.parametrize("merge", ["fused", "separate"])
def test_tiny(merge):
    """S 512, cp 2 (4 chunks of 128), 2 heads, head_dim 64, all-gather order."""
    w = synth.WORKLOADS["tiny"]
    case = make_case(1, 2, 2, 512, 64, 2, w.seed)
    check_full(case, 2, "allgather", merge)


@pytest.mark.parametrize("rotate,merge", [("allgather", "fused"), ("ring", "separate"),
                                          ("allgather", "separate"), ("ring", "fused")])
def test_fb8k(rotate, merge):
    """S 8192, cp 4 (8 chunks of 1024), 8 heads MHA, head_dim 128."""
    case = make_case(1, 8, 8, 8192, 128, 4, 1)
    check_full(case, 4, rotate, merge)


@pytest.mark.parametrize("D", [64, 128])
def test_gqa_docs_small(D):
    """GQA 8/2 with many short packed documents (lengths down to 1)."""
    cu = random_docs(4096, 11, 150.0)
    case = make_case(1, 8, 2, 4096, D, 2, 12, cu=cu)
    for merge in ("fused", "separate"):
        check_full(case, 2, "ring", merge)


def test_batch2_cp1_scale():
    case = make_case(2, 4, 4, 1024, 128, 1, 13, amp=2.0)
    check_full(case, 1, "allgather", "fused", scale=0.05)
    check_full(case, 1, "allgather", "separate", scale=0.05)


def test_cp3_odd_tiles():
    """cp 3, chunk 384: three query tiles per chunk, the last one unpaired."""
    case = make_case(1, 4, 2, 2304, 128, 3, 14)
    check_full(case, 3, "ring", "fused")
    check_full(case, 3, "allgather", "separate")


def test_local_only_differs():
    """Sanity: the merged result is far from attending the local shard only."""
    case = make_case(1, 2, 2, 2048, 128, 4, 15)
    _, plan, _, _, _, o, _ = run_fwd(cz, case, 4, "ring", "fused")
    q, k, v = (f64(case[n]) for n in ("q", "k", "v"))
    lo, _ = oracle.cp_fwd(q, k, v, 4, "ring", steps=1)
    assert np.abs(f64(o) - lo).max() > 0.1


# ----------------------------------------------------------------- full sizes, sampled

def sampled_rows(S, cp, rng, per_head, cu=None, per_doc=False):
    """Random rows plus the first and last row of every chunk (of the sequence, or
    with per-document sharding, of every document)."""
    if per_doc:
        cu = np.asarray(cu, dtype=np.int64)
        c = np.diff(cu) // (2 * cp)
        starts = (cu[:-1, None] + np.arange(2 * cp)[None, :] * c[:, None]).ravel()
        edges = np.concatenate([starts, starts + np.repeat(c, 2 * cp) - 1])
    else:
        C = S // (2 * cp)
        edges = np.concatenate([np.arange(2 * cp) * C, np.arange(1, 2 * cp + 1) * C - 1])
    return np.unique(np.concatenate([edges, rng.integers(0, S, per_head)]))


def check_sampled(name, rotate, merge="fused", per_head=192):
    w = synth.WORKLOADS[name]
    t = synth.workload_inputs(w, with_dout=False)
    case = dict(q=t["q"], k=t["k"], v=t["v"], cu_seqlens=t["cu_seqlens"],
                ds=oracle.doc_start(w.seq_len, t["cu_seqlens"]), shard=w.shard)
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, w.cp, rotate, merge)
    g = w.num_heads // w.num_kv_heads
    rng = np.random.default_rng(w.seed + 100)
    groups = [0, int(rng.integers(1, w.num_kv_heads))]
    qh = [gi * g + i for gi in groups for i in range(g)]
    q = f64(t["q"][:, qh])
    k = f64(t["k"][:, groups])
    v = f64(t["v"][:, groups])
    rows_orig = sampled_rows(w.seq_len, w.cp, rng, per_head, t["cu_seqlens"], w.shard == "doc")
    S = w.seq_len
    flat = np.concatenate([hi * S + rows_orig for hi in range(len(qh))])
    ro, rl = oracle.fwd_rows(q, k, v, flat, case["ds"])
    inv = plan.inv_perm.cpu().numpy()
    pos = inv[rows_orig]
    go = torch.stack([o[0, h, torch.from_numpy(pos).long().cuda()] for h in qh])
    gl = torch.stack([lse[0, h, torch.from_numpy(pos).long().cuda()] for h in qh])
    assert_bf16_close(f64(go).reshape(-1, w.head_dim), ro, f"O {name} {rotate} {merge}")
    assert_lse_close(f64(gl).reshape(-1), rl, f"LSE {name} {rotate} {merge}")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_gqa32k_ring_sampled():
    check_sampled("gqa32k", "ring")


def test_docs64k_sampled():
    check_sampled("docs64k", "ring", "separate")
    check_sampled("docs64k", "allgather", "fused")


def test_gqa32k_d256_sampled():
    """gqa32k at head_dim 256 (its own forward kernel)."""
    check_sampled("gqa32k_d256", "ring", "separate")
    check_sampled("gqa32k_d256", "allgather", "fused", per_head=96)


def test_docs64k_perdoc_sampled():
    """The docs64k length mix in whole-tile multiples, every document cut into 2cp chunks."""
    check_sampled("docs64k_perdoc", "ring", "fused")
    check_sampled("docs64k_perdoc", "allgather", "separate")


@pytest.mark.parametrize("rotate", ["allgather", "ring"])
def test_long128k_sampled(rotate):
    check_sampled("long128k", rotate, per_head=96)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_one_kv_head_eight_query_heads(D):
    """GQA group of 8 (one KV head), both merges."""
    case = make_case(1, 8, 1, 2048, D, 2, 250 + D)
    check_full(case, 2, "ring", "fused")
    check_full(case, 2, "allgather", "separate")
