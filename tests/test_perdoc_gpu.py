"""Per-document zigzag sharding on the GPU (FlashCP abstract, "Per-Doc" sharding:
every packed document is cut into 2cp chunks and rank r holds, document after
document, its chunk r and its chunk 2cp-1-r).

The attention is the same document-masked causal attention as with sequence
sharding, only the rows sit in another order, so the forward is compared with
the oracle's unsharded forward permuted by the oracle's per-document plan, and
the gradients, restored to the original order, with the oracle's backward."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close, f64, make_case, random_docs, run_fwd

pytestmark = pytest.mark.gpu


def per_doc_case(B, Hq, Hkv, S, D, cp, seed, median, window=0, amp=1.0):
    cu = random_docs(S, seed, median, 128, quantum=256 * cp)
    return make_case(B, Hq, Hkv, S, D, cp, seed + 1, amp=amp, cu=cu, with_dout=True,
                     window=window, shard="doc")


def check_fwd_bwd(case, cp, rotate, merge, one_pass=False):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge)
    S = qs.shape[2]
    pl = oracle.plan(S, cp, rotate, case["cu_seqlens"], case["window"], shard="doc")
    perm = plan.perm.cpu().numpy()
    assert np.array_equal(perm, pl["perm"])
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    ro, rl = oracle.fwd(q, k, v, case["ds"])
    tag = f"per-doc S={S} cp={cp} D={q.shape[-1]} {rotate} {merge}" + \
          (f" window {case['window']}" if case["window"] else "")
    assert_bf16_close(f64(o), ro[:, :, perm], "O " + tag)
    assert_lse_close(f64(lse), rl[:, :, perm], "LSE " + tag)
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob.with_one_pass(one_pass), plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    dq, dk, dv = plan.unshard([dq, dk, dv])
    rq, rk, rv = oracle.bwd(q, k, v, ro, rl, do, case["ds"])
    tag += " one-pass" if one_pass else ""
    assert_bf16_close(f64(dq), rq, "dQ " + tag)
    assert_bf16_close(f64(dk), rk, "dK " + tag)
    assert_bf16_close(f64(dv), rv, "dV " + tag)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("rotate,merge", [("ring", "fused"), ("allgather", "separate")])
def test_gqa_cp2(D, rotate, merge):
    """GQA 8/2, S 4096, cp 2: documents of 512-row multiples (chunks of 128 rows up)."""
    check_fwd_bwd(per_doc_case(1, 8, 2, 4096, D, 2, 40, 700.0), 2, rotate, merge)


@pytest.mark.parametrize("one_pass", [False, True])
def test_cp4_many_documents(one_pass):
    """cp 4 over 8192 rows: 1024-row document quanta, so single-tile chunks."""
    check_fwd_bwd(per_doc_case(1, 4, 2, 8192, 128, 4, 41, 1200.0), 4, "ring", "fused",
                  one_pass=one_pass)


def test_cp3_batch2_window():
    """cp 3, two sequences sharing one document list, a sliding window of 700."""
    check_fwd_bwd(per_doc_case(2, 4, 4, 6144, 64, 3, 42, 1500.0, window=700), 3, "allgather",
                  "fused")


def test_single_document_is_sequence_sharding():
    """One document: per-document and sequence sharding hold the same rows, and the
    two runs agree with the oracle (and closely with each other)."""
    S, cp = 4096, 4
    cu = np.array([0, S], np.int32)
    base = make_case(1, 4, 2, S, 128, cp, 43, cu=cu, with_dout=True)
    per = dict(base, shard="doc")
    _, pa, _, _, _, oa, la = run_fwd(cz, base, cp, "ring", "fused")
    _, pb, _, _, _, ob, lb = run_fwd(cz, per, cp, "ring", "fused")
    assert torch.equal(pa.perm, pb.perm) and torch.equal(pa.doc_start, pb.doc_start)
    assert torch.equal(pa.tile_orig, pb.tile_orig)
    assert (oa.float() - ob.float()).abs().max().item() <= 2 ** -7
    assert (la - lb).abs().max().item() <= 1e-5
    check_fwd_bwd(per, cp, "allgather", "separate")
