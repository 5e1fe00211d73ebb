"""Pins for the CPU oracle: each test checks it against something other than itself
(closed forms, invariants the pages fix, brute force on tiny inputs, independent
library routines, finite differences).  No GPU."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, amp=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * amp


# ----------------------------------------------------------------------------- plan

def test_plan_golden_small():
    """Hand-derived plans for S=8, cp=2 and S=12, cp=3 (golden file, derivation in it)."""
    with open(os.path.join(GOLDEN, "plan_small.json")) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        p = oracle.plan(case["S"], case["cp"], case["rotate"], case.get("cu_seqlens"))
        for key in ("perm", "inv_perm", "src", "doc_start", "rank_cu_off", "rank_cu", "pairs"):
            assert p[key].tolist() == case[key], (case["name"], key)


@pytest.mark.parametrize("S,cp", [(512, 2), (8192, 4), (32768, 8), (65536, 8), (131072, 8),
                                  (96, 3), (40, 5), (4, 1)])
def test_plan_equal_causal_work(S, cp):
    """Head/tail pairing gives every rank the same causal pair count:
    C^2 (2cp-1) + C (C+1), and the ranks together hold S(S+1)/2 pairs."""
    p = oracle.plan(S, cp)
    C = S // (2 * cp)
    assert (p["pairs"] == C * C * (2 * cp - 1) + C * (C + 1)).all()
    assert int(p["pairs"].sum()) == S * (S + 1) // 2
    perm, inv = p["perm"], p["inv_perm"]
    assert sorted(perm.tolist()) == list(range(S))            # a bijection
    assert (perm[inv] == np.arange(S)).all() and (inv[perm] == np.arange(S)).all()


def test_plan_cp1_identity():
    p = oracle.plan(64, 1)
    assert p["perm"].tolist() == list(range(64))
    assert p["src"].tolist() == [0]


@pytest.mark.parametrize("cp", [2, 3, 4, 8])
def test_plan_ring_and_allgather_orders(cp):
    """Ring: step 0 is local and each step takes the left neighbour's shard, so every
    shard is visited once; all-gather visits shards in rank order."""
    S = 2 * cp * 4
    ring = oracle.plan(S, cp, "ring")["src"].reshape(cp, cp)
    ag = oracle.plan(S, cp, "allgather")["src"].reshape(cp, cp)
    for r in range(cp):
        assert ag[r].tolist() == list(range(cp))
        assert ring[r, 0] == r
        assert sorted(ring[r].tolist()) == list(range(cp))
        for s in range(1, cp):
            # what rank r sees at step s is what its left neighbour saw at step s-1
            assert ring[r, s] == ring[(r - 1) % cp, s - 1]


def test_plan_rejects_bad_configs():
    with pytest.raises(ValueError):
        oracle.plan(100, 3)          # 100 % 6 != 0
    with pytest.raises(ValueError):
        oracle.plan(64, 0)
    with pytest.raises(ValueError):
        oracle.plan(64, 2, "allgather", np.array([0, 10, 60], np.int32))   # last != S
    with pytest.raises(ValueError):
        oracle.plan(64, 2, "allgather", np.array([0, 30, 30, 64], np.int32))  # empty doc


def test_plan_docs_pairs_and_segments():
    lens = synth.doc_lengths(65536, 3)
    cu = synth.cu_seqlens(lens)
    p = oracle.plan(65536, 8, "ring", cu)
    L = np.asarray(lens, dtype=np.int64)
    assert int(p["pairs"].sum()) == int((L * (L + 1) // 2).sum())
    # every local segment lies inside one chunk and one document
    C = 65536 // 16
    for r in range(8):
        seg = p["rank_cu"][p["rank_cu_off"][r]:p["rank_cu_off"][r + 1]]
        assert seg[0] == 0 and seg[-1] == 2 * C and C in seg
        for a, b in zip(seg[:-1], seg[1:]):
            assert b > a
            orig = p["perm"][r * 2 * C + a:r * 2 * C + b]
            assert (np.diff(orig) == 1).all()
            assert len(set(p["doc_start"][r * 2 * C + a:r * 2 * C + b].tolist())) == 1


def test_doc_lengths_recipe():
    lens = synth.doc_lengths(65536, 3)
    assert sum(lens) == 65536
    assert all(128 <= n <= 32768 for n in lens[:-1]) and lens[-1] >= 1
    # the median of a long draw sits near 2048
    many = synth.doc_lengths(10_000_000, 11)
    assert 1800 < float(np.median(many[:-1])) < 2300


# -------------------------------------------------------------------- forward pins

def brute_force(q, k, v, ds, scale):
    """Materialised masked score matrix and an explicit softmax (tiny inputs only)."""
    B, Hq, S, D = q.shape
    g = Hq // k.shape[1]
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, S))
    qi = np.arange(S)[:, None]
    ki = np.arange(S)[None, :]
    mask = (ki <= qi) & (ki >= ds[:, None])
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, h] @ k[b, h // g].T
            s = np.where(mask, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / e.sum(axis=1, keepdims=True)
            o[b, h] = p @ v[b, h // g]
            lse[b, h] = (m[:, 0] + np.log(e.sum(axis=1)))
    return o, lse


@pytest.mark.parametrize("Hq,Hkv,S,D,docs", [(2, 2, 16, 8, None), (4, 2, 24, 4, [0, 5, 6, 24]),
                                             (3, 1, 33, 5, [0, 20, 33])])
def test_fwd_brute_force(Hq, Hkv, S, D, docs):
    q, k, v = rnd((2, Hq, S, D), 1), rnd((2, Hkv, S, D), 2), rnd((2, Hkv, S, D), 3)
    cu = None if docs is None else np.array(docs, np.int32)
    ds = oracle.doc_start(S, cu)
    o, lse = oracle.fwd(q, k, v, ds)
    bo, bl = brute_force(q, k, v, ds, 1 / math.sqrt(D))
    np.testing.assert_allclose(o, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)


def test_fwd_closed_forms():
    """Row 0 sees only key 0: O = V[0], LSE = scale q0.k0.  With K = 0 every admitted
    score is 0: O is the running mean of V and LSE = ln(#admitted keys)."""
    S, D = 40, 16
    q, k, v = rnd((1, 2, S, D), 4), rnd((1, 2, S, D), 5), rnd((1, 2, S, D), 6)
    o, lse = oracle.fwd(q, k, v)
    sc = 1 / math.sqrt(D)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-14)
    np.testing.assert_allclose(lse[:, :, 0], sc * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-14)
    cu = np.array([0, 7, 19, 40], np.int32)
    ds = oracle.doc_start(S, cu)
    o, lse = oracle.fwd(q, np.zeros_like(k), v, ds)
    for t in range(S):
        np.testing.assert_allclose(o[:, :, t], v[:, :, ds[t]:t + 1].mean(axis=2), atol=1e-13)
        np.testing.assert_allclose(lse[:, :, t], math.log(t - ds[t] + 1), atol=1e-13)


def test_fwd_rows_sum_to_one():
    """Softmax rows sum to 1: with V = 1 every output element is exactly 1."""
    S, D = 64, 8
    q, k = rnd((1, 2, S, D), 7, 3.0), rnd((1, 2, S, D), 8, 3.0)
    o, _ = oracle.fwd(q, k, np.ones((1, 2, S, D)), oracle.doc_start(S, [0, 10, 64]))
    np.testing.assert_allclose(o, 1.0, atol=1e-13)


def test_fwd_matches_torch_sdpa_gqa():
    """Independent library routine: torch SDPA (fp64, causal, GQA by head groups)."""
    B, Hq, Hkv, S, D = 1, 8, 2, 96, 32
    q, k, v = rnd((B, Hq, S, D), 9), rnd((B, Hkv, S, D), 10), rnd((B, Hkv, S, D), 11)
    o, _ = oracle.fwd(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True,
        enable_gqa=True).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


def test_fwd_doc_mask_matches_per_document_sdpa():
    """Packed documents: each document is causal attention on its own slice."""
    S, D = 80, 16
    q, k, v = rnd((1, 4, S, D), 12), rnd((1, 2, S, D), 13), rnd((1, 2, S, D), 14)
    cu = np.array([0, 9, 10, 41, 80], np.int32)
    o, _ = oracle.fwd(q, k, v, oracle.doc_start(S, cu))
    for a, b in zip(cu[:-1], cu[1:]):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, :, a:b]), torch.from_numpy(k[:, :, a:b]),
            torch.from_numpy(v[:, :, a:b]), is_causal=True, enable_gqa=True).numpy()
        np.testing.assert_allclose(o[:, :, a:b], ref, atol=1e-12)


def test_fwd_rows_equals_full():
    S, D = 50, 8
    q, k, v = rnd((2, 4, S, D), 15), rnd((2, 2, S, D), 16), rnd((2, 2, S, D), 17)
    ds = oracle.doc_start(S, [0, 20, 50])
    o, lse = oracle.fwd(q, k, v, ds)
    rows = np.array([0, 3, 49, 2 * S + 21, 7 * S + 49])
    ro, rl = oracle.fwd_rows(q, k, v, rows, ds)
    np.testing.assert_allclose(ro, o.reshape(-1, D)[rows], atol=1e-14)
    np.testing.assert_allclose(rl, lse.reshape(-1)[rows], atol=1e-14)


# ------------------------------------------------------------- sharding + merge pins

@pytest.mark.parametrize("cp,rotate,docs", [(2, "allgather", None), (2, "ring", None),
                                            (4, "ring", None), (4, "allgather", [0, 3, 40, 41, 64]),
                                            (8, "ring", [0, 17, 64]), (1, "allgather", None)])
def test_sharded_merged_equals_unsharded(cp, rotate, docs):
    """The principle the method rests on: attending Q_i to every K_j,V_j and combining
    the partials gives exactly unsharded attention (to rounding)."""
    S, D = 64, 8
    q, k, v = rnd((1, 4, S, D), 18), rnd((1, 2, S, D), 19), rnd((1, 2, S, D), 20)
    cu = None if docs is None else np.array(docs, np.int32)
    o, lse = oracle.fwd(q, k, v, oracle.doc_start(S, cu))
    so, sl = oracle.cp_fwd(q, k, v, cp, rotate, cu)
    perm = oracle.plan(S, cp, rotate, cu)["perm"]
    np.testing.assert_allclose(so, o[:, :, perm], atol=1e-12)
    np.testing.assert_allclose(sl, lse[:, :, perm], atol=1e-12)


@pytest.mark.parametrize("cp,S,rotate,docs,shard,window,causal", [
    (3, 72, "ring", None, "sequence", 0, True), (4, 64, "allgather", None, "sequence", 0, True),
    (2, 64, "ring", [0, 3, 40, 41, 64], "sequence", 0, True),
    (2, 64, "ring", [0, 16, 24, 64], "doc", 0, True), (2, 64, "allgather", None, "sequence", 9, True),
    (2, 64, "ring", None, "sequence", 0, False)])
def test_sharded_bwd_equals_unsharded(cp, S, rotate, docs, shard, window, causal):
    """The backward unit by unit (rank r's queries against shard src[r][s], P from
    the final LSE): dQ_r summed over the steps and dK_j / dV_j over the ranks give
    the unsharded gradients, and stopping one step short does not."""
    D = 8
    q, k, v, do = rnd((1, 4, S, D), 24), rnd((1, 2, S, D), 25), rnd((1, 2, S, D), 26), rnd((1, 4, S, D), 27)
    cu = None if docs is None else np.array(docs, np.int32)
    ds, lk = oracle.first_key(S, cu, window), oracle.last_key(S, cu, causal)
    o, lse = oracle.fwd(q, k, v, ds, None, lk)
    rq, rk, rv = oracle.bwd(q, k, v, o, lse, do, ds, None, lk)
    perm = oracle.plan(S, cp, rotate, cu, window, causal, shard)["perm"]
    kw = dict(window=window, causal=causal, shard=shard)
    got = oracle.cp_bwd(q, k, v, o, lse, do, cp, rotate, cu, **kw)
    for g, ref in zip(got, (rq, rk, rv)):
        np.testing.assert_allclose(g, ref[:, :, perm], atol=1e-12)
    short = oracle.cp_bwd(q, k, v, o, lse, do, cp, rotate, cu, steps=cp - 1, **kw)
    assert max(np.abs(g - ref[:, :, perm]).max() for g, ref in zip(short, (rq, rk, rv))) > 1e-2


def test_bwd_partial_is_the_masked_full_backward():
    """One unit by another route: the full backward with every row outside rank r's
    queries and every key outside shard j zeroed (P from the final LSE, so zero K, V
    rows add nothing to dQ) read back at rank r's and shard j's rows."""
    S, D, cp, r, j = 64, 8, 4, 1, 2
    q, k, v, do = rnd((1, 4, S, D), 28), rnd((1, 2, S, D), 29), rnd((1, 2, S, D), 30), rnd((1, 4, S, D), 31)
    cu = np.array([0, 5, 33, 64], np.int32)
    ds = oracle.doc_start(S, cu)
    o, lse = oracle.fwd(q, k, v, ds)
    perm = oracle.plan(S, cp, "ring", cu)["perm"]
    rows = lambda x: perm[x * (S // cp):(x + 1) * (S // cp)]
    on = lambda p: np.isin(np.arange(S), p)
    keep = lambda x, p: np.where(on(p)[None, None, :, None], x, 0.0)
    fq, fk, fv = oracle.bwd(keep(q, rows(r)), keep(k, rows(j)), keep(v, rows(j)), keep(o, rows(r)),
                            np.where(on(rows(r))[None, None, :], lse, 0.0), keep(do, rows(r)), ds)
    pq, pk, pv = oracle.bwd_partial(q, k, v, o, lse, do, perm, cp, r, j, ds)
    np.testing.assert_allclose(pq, fq[:, :, rows(r)], atol=1e-13)
    np.testing.assert_allclose(pk, fk[:, :, rows(j)], atol=1e-13)
    np.testing.assert_allclose(pv, fv[:, :, rows(j)], atol=1e-13)
    assert np.abs(pk).max() > 1e-3


def test_local_only_attention_breaks_parity():
    """If only the local shard is attended (CP communication silently off), the result
    is wrong: dropping steps s > 0 must fail parity."""
    S, D, cp = 64, 8, 4
    q, k, v = rnd((1, 2, S, D), 21), rnd((1, 2, S, D), 22), rnd((1, 2, S, D), 23)
    o, _ = oracle.fwd(q, k, v)
    lo, _ = oracle.cp_fwd(q, k, v, cp, "ring", steps=1)
    perm = oracle.plan(S, cp)["perm"]
    assert np.abs(lo - o[:, :, perm]).max() > 0.1


def test_merge_identity_and_halves():
    R, D = 30, 8
    S = 40
    q, k, v = rnd((1, 1, S, D), 24), rnd((1, 1, S, D), 25), rnd((1, 1, S, D), 26)
    o, lse = oracle.fwd(q, k, v)
    # identity: merging with an all-(-inf) partial
    po = rnd((1, R, D), 27)
    pl = rnd((1, R), 28)
    mo, ml = oracle.lse_merge(np.concatenate([po, np.zeros((1, R, D))]),
                              np.concatenate([pl, np.full((1, R), -np.inf)]))
    np.testing.assert_allclose(mo, po[0], atol=1e-15)
    np.testing.assert_allclose(ml, pl[0], atol=1e-15)
    # halves of each row's key set: with the identity permutation and cp=2, "rank" 1
    # holds rows 20..39 and the two "shards" are keys [0,20) and [20,40)
    perm = np.arange(S, dtype=np.int32)
    ds = np.zeros(S, np.int32)
    first = oracle.partial(q, k, v, perm, 2, 1, 0, ds)
    second = oracle.partial(q, k, v, perm, 2, 1, 1, ds)
    mo, ml = oracle.lse_merge(np.stack([first[0][0], second[0][0]]),
                              np.stack([first[1][0], second[1][0]]))
    np.testing.assert_allclose(mo, o[0, 0, 20:], atol=1e-13)
    np.testing.assert_allclose(ml, lse[0, 0, 20:], atol=1e-13)
    # rows 0..19 against keys 20..39: every row empty -> (0, -inf)
    empty = oracle.partial(q, k, v, perm, 2, 0, 1, ds)
    assert np.isneginf(empty[1]).all() and (empty[0] == 0).all()


def test_merge_associative():
    P, R, D = 3, 20, 4
    po, pl = rnd((P, R, D), 29), rnd((P, R), 30)
    pl[1, :5] = -np.inf
    full = oracle.lse_merge(po, pl)
    ab = oracle.lse_merge(po[:2], pl[:2])
    nested = oracle.lse_merge(np.stack([ab[0], po[2]]), np.stack([ab[1], pl[2]]))
    np.testing.assert_allclose(full[0], nested[0], atol=1e-13)
    np.testing.assert_allclose(full[1], nested[1], atol=1e-13)


# ------------------------------------------------------------------- backward pins

def _loss(q, k, v, dout, ds):
    o, _ = oracle.fwd(q, k, v, ds)
    return float((o * dout).sum())


def test_bwd_finite_differences():
    """Central differences in fp64 of L = sum(O * dO) on a tiny GQA + doc-mask case."""
    B, Hq, Hkv, S, D = 1, 4, 2, 16, 8
    q, k, v = rnd((B, Hq, S, D), 31), rnd((B, Hkv, S, D), 32), rnd((B, Hkv, S, D), 33)
    dout = rnd((B, Hq, S, D), 34)
    ds = oracle.doc_start(S, [0, 6, 16])
    o, lse = oracle.fwd(q, k, v, ds)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds)
    eps = 1e-6
    g = np.random.default_rng(35)
    for name, x, gx in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(g.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], dout, ds)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], dout, ds)
            assert abs((lp - lm) / (2 * eps) - gx[idx]) < 1e-6, (name, idx)


def test_bwd_matches_torch_autograd():
    B, Hq, Hkv, S, D = 1, 4, 2, 48, 16
    q, k, v = rnd((B, Hq, S, D), 36), rnd((B, Hkv, S, D), 37), rnd((B, Hkv, S, D), 38)
    dout = rnd((B, Hq, S, D), 39)
    o, lse = oracle.fwd(q, k, v)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                          enable_gqa=True)
    to.backward(torch.from_numpy(dout))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def test_bwd_sum_properties():
    """Rows of P sum to 1, so sum_k dV_k = sum of dO over the group's rows, and
    sum_k dK_k = 0 (since sum_k P dP = Dq)."""
    B, Hq, Hkv, S, D = 1, 6, 2, 40, 8
    q, k, v = rnd((B, Hq, S, D), 40), rnd((B, Hkv, S, D), 41), rnd((B, Hkv, S, D), 42)
    dout = rnd((B, Hq, S, D), 43)
    ds = oracle.doc_start(S, [0, 13, 40])
    o, lse = oracle.fwd(q, k, v, ds)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds)
    g = Hq // Hkv
    for hk in range(Hkv):
        np.testing.assert_allclose(dv[0, hk].sum(0), dout[0, hk * g:(hk + 1) * g].sum((0, 1)),
                                   atol=1e-12)
        np.testing.assert_allclose(dk[0, hk].sum(0), 0.0, atol=1e-12)


def test_bwd_sampled_equals_full():
    B, Hq, Hkv, S, D = 1, 4, 2, 36, 8
    q, k, v = rnd((B, Hq, S, D), 44), rnd((B, Hkv, S, D), 45), rnd((B, Hkv, S, D), 46)
    dout = rnd((B, Hq, S, D), 47)
    ds = oracle.doc_start(S, [0, 11, 36])
    o, lse = oracle.fwd(q, k, v, ds)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds)
    rows = np.array([0, 5, 35, S + 12, 3 * S + 35])
    np.testing.assert_allclose(oracle.bwd_dq_rows(q, k, v, dout, rows, ds),
                               dq.reshape(-1, D)[rows], atol=1e-13)
    keys = np.array([0, 10, 11, 35, S + 20])
    sk, sv = oracle.bwd_dkv_keys(q, k, v, dout, keys, ds)
    np.testing.assert_allclose(sk, dk.reshape(-1, D)[keys], atol=1e-13)
    np.testing.assert_allclose(sv, dv.reshape(-1, D)[keys], atol=1e-13)
    # the keys-only form that reads the forward's O / LSE instead of recomputing rows
    fk, fv = oracle.bwd_dkv_keys_fwd(q, k, v, o, lse, dout, keys, ds)
    np.testing.assert_allclose(fk, dk.reshape(-1, D)[keys], atol=1e-13)
    np.testing.assert_allclose(fv, dv.reshape(-1, D)[keys], atol=1e-13)


def test_bwd_keys_from_forward_batch2():
    """bwd_dkv_keys_fwd indexes batch and KV head: batch 2, GQA 3:1, keys of every
    (batch, KV head), against the full backward."""
    B, Hq, Hkv, S, D = 2, 6, 2, 30, 8
    q, k, v = rnd((B, Hq, S, D), 48), rnd((B, Hkv, S, D), 49), rnd((B, Hkv, S, D), 50)
    dout = rnd((B, Hq, S, D), 51)
    ds = oracle.first_key(S, [0, 7, 30], window=9)
    o, lse = oracle.fwd(q, k, v, ds)
    _, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds)
    keys = np.array([0, 6, 7, S + 3, 2 * S + 29, 3 * S + 0, 3 * S + 15])
    fk, fv = oracle.bwd_dkv_keys_fwd(q, k, v, o, lse, dout, keys, ds)
    np.testing.assert_allclose(fk, dk.reshape(-1, D)[keys], atol=1e-13)
    np.testing.assert_allclose(fv, dv.reshape(-1, D)[keys], atol=1e-13)
    with pytest.raises(ValueError):
        oracle.bwd_dkv_keys_fwd(q, k, v, o, lse, dout, np.array([4 * S]), ds)


# --------------------------------------------------------------- arithmetic pins

def test_flop_convention_and_memory_estimate():
    # 4*D*Hq per unmasked pair; the table's fwd FLOPs
    assert abs(oracle.flops(2, 64, oracle.causal_pairs(512)) - 6.72e7) / 6.72e7 < 1e-3
    assert abs(oracle.flops(32, 128, oracle.causal_pairs(131072)) - 1.407e14) / 1.407e14 < 1e-3
    assert oracle.flops(8, 128, 100, backward=True) == 3 * oracle.flops(8, 128, 100)
    # the concept guide's vanilla attention-matrix estimate: 128k*128k*2 B = 32 GiB per head
    assert 131072 * 131072 * 2 == 32 * 2 ** 30


def test_bf16_ulp_helper():
    """The tolerance helper's bf16 spacing: 2^-7 at 1, 2^-4 at 8..16, and exact for
    values that bf16 represents."""
    from helpers import bf16_ulp
    assert bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert bf16_ulp(np.array([8.159]))[0] == 2.0 ** -4
    assert bf16_ulp(np.array([-3.0]))[0] == 2.0 ** -6
    x = torch.tensor([8.159, 1.2345, -0.3]).to(torch.bfloat16).double().numpy()
    ref = np.array([8.159, 1.2345, -0.3])
    assert (np.abs(x - ref) <= bf16_ulp(ref) / 2 + 1e-12).all()


# ------------------------------------------------------------- sliding-window pins
# A sliding window of W keys on top of the causal (and document) mask: the query
# at q sees keys q - W < k <= q.  The oracle takes it as first_key(q) = max(doc
# start, q - W + 1); these pins check that array and everything built on it
# against the band mask written out directly.

def band_brute_force(q, k, v, cu, window, scale):
    """Explicit softmax over the mask k <= q, k > q - W, k in q's document."""
    B, Hq, S, D = q.shape
    g = Hq // k.shape[1]
    qi = np.arange(S)[:, None]
    ki = np.arange(S)[None, :]
    doc = np.zeros(S, np.int64) if cu is None else np.searchsorted(np.asarray(cu), np.arange(S), side="right") - 1
    mask = (ki <= qi) & (ki > qi - window) & (doc[ki] == doc[qi])
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            s = np.where(mask, scale * q[b, h] @ k[b, h // g].T, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            o[b, h] = (e / e.sum(axis=1, keepdims=True)) @ v[b, h // g]
            lse[b, h] = m[:, 0] + np.log(e.sum(axis=1))
    return o, lse, int(mask.sum())


@pytest.mark.parametrize("Hq,Hkv,S,D,W,docs", [(2, 2, 32, 8, 5, None), (4, 2, 48, 4, 13, [0, 9, 10, 48]),
                                               (3, 1, 33, 5, 1, [0, 20, 33]), (2, 1, 40, 8, 40, None)])
def test_window_brute_force(Hq, Hkv, S, D, W, docs):
    q, k, v = rnd((1, Hq, S, D), 41), rnd((1, Hkv, S, D), 42), rnd((1, Hkv, S, D), 43)
    cu = None if docs is None else np.array(docs, np.int32)
    o, lse = oracle.fwd(q, k, v, oracle.first_key(S, cu, W))
    bo, bl, npairs = band_brute_force(q, k, v, cu, W, 1 / math.sqrt(D))
    np.testing.assert_allclose(o, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)
    assert oracle.causal_pairs(S, cu, W) == npairs
    if S % 2 == 0:   # the zigzag plan needs S divisible by 2 * cp
        assert int(oracle.plan(S, 1, "allgather", cu, W)["pairs"].sum()) == npairs


def test_window_one_closed_form():
    """W = 1: every query sees only itself, so O = V[q] and LSE = scale * q.k_q."""
    S, D = 64, 16
    q, k, v = rnd((1, 4, S, D), 44), rnd((1, 2, S, D), 45), rnd((1, 2, S, D), 46)
    o, lse = oracle.fwd(q, k, v, oracle.first_key(S, None, 1))
    sc = 1 / math.sqrt(D)
    for h in range(4):
        np.testing.assert_allclose(o[0, h], v[0, h // 2], atol=1e-14)
        np.testing.assert_allclose(lse[0, h], sc * (q[0, h] * k[0, h // 2]).sum(-1), atol=1e-13)


def test_window_wider_than_sequence_is_causal():
    cu = np.array([0, 100, 256], np.int32)
    assert np.array_equal(oracle.first_key(256, cu, 256), oracle.doc_start(256, cu))
    assert np.array_equal(oracle.plan(256, 4, "ring", cu, 300)["pairs"], oracle.plan(256, 4, "ring", cu)["pairs"])


@pytest.mark.parametrize("cp,rotate,W", [(2, "allgather", 37), (4, "ring", 100)])
def test_window_sharded_equals_unsharded(cp, rotate, W):
    S, D = 256, 8
    cu = np.array([0, 70, 71, 256], np.int32)
    q, k, v = rnd((1, 4, S, D), 47), rnd((1, 2, S, D), 48), rnd((1, 2, S, D), 49)
    o, lse = oracle.fwd(q, k, v, oracle.first_key(S, cu, W))
    so, sl = oracle.cp_fwd(q, k, v, cp, rotate, cu, window=W)
    perm = oracle.plan(S, cp, rotate, cu, W)["perm"]
    np.testing.assert_allclose(so, o[:, :, perm], atol=1e-12)
    np.testing.assert_allclose(sl, lse[:, :, perm], atol=1e-12)


def test_window_bwd_finite_differences():
    B, Hq, Hkv, S, D, W = 1, 2, 1, 16, 8, 4
    q, k, v = rnd((B, Hq, S, D), 51), rnd((B, Hkv, S, D), 52), rnd((B, Hkv, S, D), 53)
    dout = rnd((B, Hq, S, D), 54)
    ds = oracle.first_key(S, [0, 9, 16], W)
    o, lse = oracle.fwd(q, k, v, ds)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds)
    eps = 1e-6
    g = np.random.default_rng(55)
    for name, x, gx in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(10):
            idx = tuple(int(g.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], dout, ds)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], dout, ds)
            assert abs((lp - lm) / (2 * eps) - gx[idx]) < 1e-6, (name, idx)


# ------------------------------------------------- attention without the causal mask
# (the bidirectional variant: every query sees every key of its document)

def full_brute_force(q, k, v, cu, scale):
    """Materialised score matrix with only the block-diagonal document mask (or none)
    and an explicit softmax, written out here without the oracle's key ranges."""
    B, Hq, S, D = q.shape
    g = Hq // k.shape[1]
    doc = np.zeros(S, np.int64) if cu is None else np.repeat(np.arange(len(cu) - 1), np.diff(cu))
    mask = doc[:, None] == doc[None, :]
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            s = np.where(mask, scale * q[b, h] @ k[b, h // g].T, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            o[b, h] = (e / e.sum(axis=1, keepdims=True)) @ v[b, h // g]
            lse[b, h] = m[:, 0] + np.log(e.sum(axis=1))
    return o, lse


def test_last_key():
    assert np.array_equal(oracle.last_key(5), np.arange(5))
    assert np.array_equal(oracle.last_key(5, causal=False), [4] * 5)
    assert np.array_equal(oracle.last_key(7, [0, 2, 7], causal=False), [1, 1, 6, 6, 6, 6, 6])


@pytest.mark.parametrize("Hq,Hkv,S,D,docs", [(2, 2, 16, 8, None), (4, 2, 24, 4, [0, 5, 6, 24])])
def test_noncausal_fwd_brute_force(Hq, Hkv, S, D, docs):
    q, k, v = rnd((2, Hq, S, D), 61), rnd((2, Hkv, S, D), 62), rnd((2, Hkv, S, D), 63)
    ds, lk = oracle.first_key(S, docs), oracle.last_key(S, docs, causal=False)
    o, lse = oracle.fwd(q, k, v, ds, None, lk)
    ro, rl = full_brute_force(q, k, v, docs, 1 / np.sqrt(D))
    np.testing.assert_allclose(o, ro, atol=1e-12)
    np.testing.assert_allclose(lse, rl, atol=1e-12)


def test_noncausal_matches_torch_sdpa_and_closed_form():
    B, Hq, Hkv, S, D = 1, 4, 2, 40, 8
    q, k, v = rnd((B, Hq, S, D), 64), rnd((B, Hkv, S, D), 65), rnd((B, Hkv, S, D), 66)
    o, lse = oracle.fwd(q, k, v, None, None, oracle.last_key(S, causal=False))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)), is_causal=False, enable_gqa=True).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)
    # K = 0: every row is the mean of all V and LSE = ln S
    o0, l0 = oracle.fwd(q, np.zeros_like(k), v, None, None, oracle.last_key(S, causal=False))
    np.testing.assert_allclose(o0[0, 0], np.broadcast_to(v[0, 0].mean(0), (S, D)), atol=1e-12)
    np.testing.assert_allclose(l0, np.log(S), atol=1e-12)


@pytest.mark.parametrize("cp,rotate,docs", [(2, "allgather", None), (3, "ring", None),
                                            (2, "ring", [0, 7, 30, 48])])
def test_noncausal_sharded_merged_equals_unsharded(cp, rotate, docs):
    S = 48
    q, k, v = rnd((1, 2, S, 8), 67), rnd((1, 2, S, 8), 68), rnd((1, 2, S, 8), 69)
    so, sl = oracle.cp_fwd(q, k, v, cp, rotate, docs, causal=False)
    o, lse = oracle.fwd(q, k, v, oracle.first_key(S, docs), None,
                        oracle.last_key(S, docs, causal=False))
    perm = oracle.plan(S, cp, rotate, docs, causal=False)["perm"]
    np.testing.assert_allclose(so, o[:, :, perm], atol=1e-12)
    np.testing.assert_allclose(sl, lse[:, :, perm], atol=1e-12)


def test_noncausal_plan_pairs():
    """Every rank's 2C queries see all S keys: 2C*S pairs each (the zigzag changes
    nothing); with documents, the pairs are the sum of L^2 over each rank's rows."""
    for S, cp in ((512, 2), (8192, 4)):
        pl = oracle.plan(S, cp, causal=False)
        assert (pl["pairs"] == (S // cp) * S).all()
        assert pl["pairs"].sum() == oracle.causal_pairs(S, causal=False) == S * S
    cu = [0, 7, 30, 48]
    pl = oracle.plan(48, 2, "ring", cu, causal=False)
    L = np.repeat(np.diff(cu), np.diff(cu))                 # document length per position
    per_rank = [int(L[pl["perm"][r * 24:(r + 1) * 24]].sum()) for r in range(2)]
    assert list(pl["pairs"]) == per_rank
    with pytest.raises(ValueError):
        oracle.plan(48, 2, "ring", None, window=4, causal=False)


def test_noncausal_bwd_finite_differences_and_autograd():
    B, Hq, Hkv, S, D = 1, 4, 2, 16, 8
    q, k, v = rnd((B, Hq, S, D), 70), rnd((B, Hkv, S, D), 71), rnd((B, Hkv, S, D), 72)
    dout = rnd((B, Hq, S, D), 73)
    cu = [0, 6, 16]
    ds, lk = oracle.first_key(S, cu), oracle.last_key(S, cu, causal=False)
    o, lse = oracle.fwd(q, k, v, ds, None, lk)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds, None, lk)
    eps = 1e-6
    g = np.random.default_rng(74)
    for name, x, gx in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(10):
            idx = tuple(int(g.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = float((oracle.fwd(args["q"], args["k"], args["v"], ds, None, lk)[0] * dout).sum())
            args[name] = xm
            lm = float((oracle.fwd(args["q"], args["k"], args["v"], ds, None, lk)[0] * dout).sum())
            assert abs((lp - lm) / (2 * eps) - gx[idx]) < 1e-6, (name, idx)
    # one document: torch autograd of non-causal SDPA
    o, lse = oracle.fwd(q, k, v, None, None, oracle.last_key(S, causal=False))
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, None, None, oracle.last_key(S, causal=False))
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=False,
                                                     enable_gqa=True).backward(torch.from_numpy(dout))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def test_noncausal_sampled_equals_full():
    B, Hq, Hkv, S, D = 1, 4, 2, 30, 8
    q, k, v = rnd((B, Hq, S, D), 75), rnd((B, Hkv, S, D), 76), rnd((B, Hkv, S, D), 77)
    dout = rnd((B, Hq, S, D), 78)
    cu = [0, 11, 30]
    ds, lk = oracle.first_key(S, cu), oracle.last_key(S, cu, causal=False)
    o, lse = oracle.fwd(q, k, v, ds, None, lk)
    dq, dk, dv = oracle.bwd(q, k, v, o, lse, dout, ds, None, lk)
    rows = np.array([0, 5, 29, S + 12, 3 * S + 2])
    np.testing.assert_allclose(oracle.bwd_dq_rows(q, k, v, dout, rows, ds, None, lk),
                               dq.reshape(-1, D)[rows], atol=1e-13)
    ro, rl = oracle.fwd_rows(q, k, v, rows, ds, None, lk)
    np.testing.assert_allclose(ro, o.reshape(-1, D)[rows], atol=1e-13)
    keys = np.array([0, 10, 11, 29, S + 3])
    for fn in (lambda: oracle.bwd_dkv_keys(q, k, v, dout, keys, ds, None, lk),
               lambda: oracle.bwd_dkv_keys_fwd(q, k, v, o, lse, dout, keys, ds, None, lk)):
        sk, sv = fn()
        np.testing.assert_allclose(sk, dk.reshape(-1, D)[keys], atol=1e-13)
        np.testing.assert_allclose(sv, dv.reshape(-1, D)[keys], atol=1e-13)


# ------------------------------------------------------- per-document zigzag sharding
# (FlashCP abstract, "Per-Doc" sharding: every document, not only the sequence, is
# split so each rank gets an equal share of its causal work)

def test_per_doc_plan_golden():
    """S 16, cp 2, two documents of 8: each cut into 4 chunks of 2 tokens; rank 0
    holds chunks 0 and 3 of each document, rank 1 chunks 1 and 2 (worked by hand)."""
    pl = oracle.plan(16, 2, "allgather", [0, 8, 16], shard="doc")
    assert list(pl["perm"]) == [0, 1, 6, 7, 8, 9, 14, 15, 2, 3, 4, 5, 10, 11, 12, 13]
    assert list(pl["inv_perm"][pl["perm"]]) == list(range(16))
    assert list(pl["doc_start"]) == [0, 0, 0, 0, 8, 8, 8, 8, 0, 0, 0, 0, 8, 8, 8, 8]
    assert list(pl["rank_cu_off"]) == [0, 5, 10]
    assert list(pl["rank_cu"]) == [0, 2, 4, 6, 8, 0, 2, 4, 6, 8]
    # causal pairs: rank 0 rows 0,1,6,7 | 8,9,14,15 -> (1+2+7+8) * 2; rank 1 -> (3+4+5+6) * 2
    assert list(pl["pairs"]) == [36, 36]


def test_per_doc_single_document_is_the_sequence_plan():
    for S, cp in ((512, 2), (4096, 4), (2304, 3)):
        a = oracle.plan(S, cp, "ring", [0, S], shard="doc")
        b = oracle.plan(S, cp, "ring", [0, S])
        for key in ("perm", "inv_perm", "src", "doc_start", "rank_cu_off", "rank_cu", "pairs"):
            assert np.array_equal(a[key], b[key]), key


def test_per_doc_balances_causal_work():
    """Per document of length L = 2cp*c, rank r's two chunks carry c^2 (2cp-1) + c(c+1)
    causal pairs whatever r is, so every rank gets the same work; the sequence-level
    zigzag over the same documents does not."""
    cp = 8
    lens = synth.doc_lengths(65536, 3, 2048.0, 1.0, (128, 32768))
    lens = [max(2 * cp, (n // (2 * cp)) * 2 * cp) for n in lens]
    lens[-1] += 65536 - sum(lens)
    assert lens[-1] > 0 and lens[-1] % (2 * cp) == 0
    cu = synth.cu_seqlens(lens)
    pd = oracle.plan(65536, cp, "ring", cu, shard="doc")
    sq = oracle.plan(65536, cp, "ring", cu)
    c = np.asarray(lens, dtype=np.int64) // (2 * cp)
    assert (pd["pairs"] == (c * c * (2 * cp - 1) + c * (c + 1)).sum()).all()
    assert pd["pairs"].sum() == sq["pairs"].sum() == oracle.causal_pairs(65536, cu)
    assert sq["pairs"].max() / sq["pairs"].mean() > 1.5
    assert np.array_equal(np.sort(pd["perm"]), np.arange(65536))


def test_per_doc_sharded_merged_equals_unsharded():
    S, cp, cu = 96, 2, [0, 24, 32, 96]
    q, k, v = rnd((1, 2, S, 8), 81), rnd((1, 2, S, 8), 82), rnd((1, 2, S, 8), 83)
    so, sl = oracle.cp_fwd(q, k, v, cp, "ring", cu, shard="doc")
    o, lse = oracle.fwd(q, k, v, oracle.doc_start(S, cu))
    perm = oracle.plan(S, cp, "ring", cu, shard="doc")["perm"]
    np.testing.assert_allclose(so, o[:, :, perm], atol=1e-12)
    np.testing.assert_allclose(sl, lse[:, :, perm], atol=1e-12)


def test_per_doc_rejects_uneven_documents():
    with pytest.raises(ValueError):
        oracle.plan(16, 2, "allgather", [0, 6, 16], shard="doc")   # 6 is not a multiple of 4
    with pytest.raises(ValueError):
        oracle.plan(16, 2, "allgather", None, shard="doc")         # needs documents


def test_per_doc_cp1_is_identity():
    """cp 1: every document is cut into its two halves and rank 0 holds them in
    order, so the per-document plan is the identity (as the sequence plan is)."""
    cu = [0, 8, 24, 64]
    pl = oracle.plan(64, 1, "allgather", cu, shard="doc")
    assert list(pl["perm"]) == list(range(64))
    assert list(pl["rank_cu"]) == [0, 4, 8, 16, 24, 44, 64]
    assert int(pl["pairs"][0]) == oracle.causal_pairs(64, cu)
