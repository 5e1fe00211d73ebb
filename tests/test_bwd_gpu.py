"""GPU backward (dQ, dK, dV) against the oracle's explicit-P gradients.

Small and mid sizes: every element.  Full sizes: dQ on sampled rows; dK/dV on
keys near the end of the sequence and of documents (few attending rows) and, at
32k and 64k, on whole early key tiles of one KV group (the keys that collect
over the most rows); plus the identities that hold at any size: sum_k dV_k =
sum of dO over the group's rows, and sum_k dK_k = 0, to within the rounding
noise of the bf16 outputs."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
import synth
from helpers import (assert_bf16_close, bf16_operand_attention, f64, make_case, random_docs,
                     run_fwd)

pytestmark = pytest.mark.gpu


def run_bwd(case, cp, rotate="allgather", merge="fused", scale=0.0, with_o=False,
            one_pass=False):
    prob, plan, qs, ks, vs, o, lse = run_fwd(cz, case, cp, rotate, merge, scale)
    (dos,) = plan.shard([case["do"].cuda()])
    dq, dk, dv = cz.attn_bwd(prob.with_one_pass(one_pass), plan, qs, ks, vs, o, lse, dos)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    if with_o:
        dq, dk, dv, o = plan.unshard([dq, dk, dv, o])
        return prob, plan, dq, dk, dv, o
    dq, dk, dv = plan.unshard([dq, dk, dv])
    return prob, plan, dq, dk, dv


def check_full(case, cp, rotate, scale=0.0, emulate=False, one_pass=False):
    _, _, dq, dk, dv = run_bwd(case, cp, rotate, scale=scale, one_pass=one_pass)
    q, k, v, do = (f64(case[n]) for n in ("q", "k", "v", "do"))
    o, lse = oracle.fwd(q, k, v, case["ds"], scale or None)
    rq, rk, rv = oracle.bwd(q, k, v, o, lse, do, case["ds"], scale or None)
    tag = f"S={q.shape[2]} cp={cp} {rotate}" + (" one-pass" if one_pass else "")
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


# one_pass: the one-pass backward (dQ partials reduced into an fp32 accumulator);
# otherwise the default two-pass backward (a dK/dV pass and a dQ pass)
@pytest.mark.parametrize("one_pass", [False, True])
def test_small_d64(one_pass):
    case = make_case(1, 2, 2, 512, 64, 2, 0, with_dout=True)
    check_full(case, 2, "allgather", one_pass=one_pass)


@pytest.mark.parametrize("one_pass", [False, True])
def test_fb8k(one_pass):
    """S 8192, cp 4, 8 heads MHA, head_dim 128, all-gather order."""
    case = make_case(1, 8, 8, 8192, 128, 4, 1, with_dout=True)
    check_full(case, 4, "allgather", one_pass=one_pass)


@pytest.mark.parametrize("D,one_pass", [(64, False), (128, False), (64, True), (128, True)])
def test_gqa_docs_small(D, one_pass):
    cu = random_docs(4096, 21, 150.0)
    case = make_case(1, 8, 2, 4096, D, 2, 22, cu=cu, with_dout=True)
    check_full(case, 2, "ring", emulate=(D == 128), one_pass=one_pass)


def test_one_pass_matches_two_pass():
    """The two backward forms compute the same sums in different orders: dK / dV
    are bit-identical (same per-key accumulation order), dQ differs only by the
    fp32 summation order of its partials."""
    case = make_case(1, 8, 2, 4096, 128, 4, 24, with_dout=True)
    _, _, dq1, dk1, dv1 = run_bwd(case, 4, "ring", one_pass=True)
    _, _, dq2, dk2, dv2 = run_bwd(case, 4, "ring")
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    ulp = torch.exp2(torch.floor(torch.log2(dq2.double().abs().clamp_min(2.0 ** -126))) - 7)
    assert ((dq1.double() - dq2.double()).abs() <= ulp + 1e-6).all()


def test_batch2_cp3_scale():
    """Batch 2, cp 3 (three query tiles per chunk), GQA 4/2, a non-default scale."""
    case = make_case(2, 4, 2, 2304, 128, 3, 23, with_dout=True)
    check_full(case, 3, "ring", scale=0.07, emulate=True)


# ----------------------------------------------------------------- full sizes, sampled

def key_tiles_early(S, cu, rng):
    """Whole 128-key tiles whose keys collect over the most query rows: the first
    tile, the two tiles around the middle (the first and second halves of the
    zigzag key-tile pairs meet there), a random one and the last.  With documents:
    the first and a middle tile of the longest document instead of the middle."""
    nkt = S // 128
    tiles = {0, nkt - 1, int(rng.integers(1, nkt - 1))}
    if cu is None:
        tiles |= {nkt // 2 - 1, nkt // 2}
    else:
        lens = np.diff(cu)
        d = int(np.argmax(lens))
        first, last = (int(cu[d]) + 127) // 128, int(cu[d + 1]) // 128 - 1
        tiles |= {first, (first + last) // 2}
    return np.concatenate([np.arange(t * 128, t * 128 + 128) for t in sorted(tiles)])


def check_identities(name, S, g, Hkv, scale, cu, dq, dk, dv, q, o, do):
    """Whole-sequence identities, per KV head and column: sum_k dV_k equals the sum of
    dO over the group's rows (every row's P sums to 1), and sum_k dK_k = 0 (every
    row's dS sums to 0).  The GPU's sums differ from these by three effects, each
    bounded here:
      * output rounding: every gradient is a bf16 value rounded to nearest, an
        independent error of variance ulp^2 / 12, so the sum over S keys carries
        noise of standard deviation sigma_out = sqrt(sum ulp^2 / 12); 6 sigma;
      * accumulation: dK_k and dV_k are fp32 tensor-core accumulations over m_k
        = g * n_k / 16 MMA steps (n_k rows attend key k, 16 rows per step); each
        step may be biased by up to 2^-24 of the accumulator (its rounding), so
        |bias_k| <= m_k 2^-22 |grad_k| with a factor-4 margin (measured: the
        deviation grows as S^2, 0.10 at 32k and 1.47 at 128k);
      * dK only: the backward takes D_q = dO_q . O_q from the bf16 O, so row q's dS
        sums to dO_q . (O_exact - O_q), at most delta_q = sum_d |dO_qd| ulp(O_qd)/2;
        summed as independent terms over the rows: 6 scale sqrt(sum_q Q_qd^2 delta_q^2)."""
    dvd, dkd = dv.double()[0], dk.double()[0]                          # [Hkv, S, D]
    ulp = lambda x: torch.exp2(torch.floor(torch.log2(x.abs().clamp_min(2.0 ** -126))) - 7)
    pos = torch.arange(S, device=dvd.device, dtype=torch.float64)
    if cu is None:
        n_k = S - pos                                                   # rows q >= k
    else:
        ends = torch.from_numpy(np.repeat(np.asarray(cu[1:]), np.diff(cu))).to(dvd.device)
        n_k = ends.double() - pos                                       # rows of k's document
    m_k = (g * n_k / 16.0)[None, :, None]
    sig_v = (ulp(dvd) ** 2 / 12).sum(dim=1).sqrt()
    sig_k = (ulp(dkd) ** 2 / 12).sum(dim=1).sqrt()
    acc_v = (m_k * dvd.abs()).sum(dim=1) * 2.0 ** -22
    acc_k = (m_k * dkd.abs()).sum(dim=1) * 2.0 ** -22
    qd, od, dod = (x.cuda().double()[0] for x in (q, o, do))            # [Hq, S, D]
    delta = (dod.abs() * ulp(od) / 2).sum(dim=2, keepdim=True)          # [Hq, S, 1]
    sig_d = scale * ((qd * delta) ** 2).sum(dim=1).view(Hkv, g, -1).sum(1).sqrt()
    dv_sum = dvd.sum(dim=1)
    do_sum = dod.sum(dim=1).view(Hkv, g, -1).sum(1)
    ev = (dv_sum - do_sum).abs()
    ek = dkd.sum(dim=1).abs()
    bv = 6 * sig_v + acc_v
    bk = 6 * (sig_k ** 2 + sig_d ** 2).sqrt() + acc_k
    assert (ev <= bv).all(), (name, "dV", ev.max().item(), (ev / bv).max().item())
    assert (ek <= bk).all(), (name, "dK", ek.max().item(), (ek / bk).max().item())
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    return (ev / bv).max().item(), (ek / bk).max().item()


def check_sampled(name, rotate, n_rows=96, n_keys=24, early=True, one_pass=False):
    w = synth.WORKLOADS[name]
    t = synth.workload_inputs(w, with_dout=True)
    S, g = w.seq_len, w.num_heads // w.num_kv_heads
    cu = t["cu_seqlens"]
    ds = oracle.doc_start(S, cu)
    case = dict(q=t["q"], k=t["k"], v=t["v"], do=t["do"], cu_seqlens=cu, ds=ds, shard=w.shard)
    _, _, dq, dk, dv, o_gpu = run_bwd(case, w.cp, rotate, with_o=True, one_pass=one_pass)
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
    tag = f"{name} {rotate}" + (" one-pass" if one_pass else "")
    assert_bf16_close(gq, rq, f"dQ {tag} sampled rows")
    # dK / dV on keys whose attending rows are few: the last keys of the sequence
    # and of its documents
    ends = [S - 1 - i for i in range(n_keys // 2)]
    if cu is not None:
        ends += [int(cu[i + 1]) - 1 - int(rng.integers(0, 64)) for i in range(len(cu) - 1)
                 if cu[i + 1] - cu[i] <= 4096][: n_keys // 2]
    keys = np.unique(np.clip(np.asarray(ends), 0, S - 1))
    flatk = np.concatenate([gi * S + keys for gi in range(len(groups))])
    rk, rv = oracle.bwd_dkv_keys(q, k, v, do, flatk, ds)
    assert_bf16_close(f64(dk[0, groups][:, keys]).reshape(-1, w.head_dim), rk,
                      f"dK {tag} late keys")
    assert_bf16_close(f64(dv[0, groups][:, keys]).reshape(-1, w.head_dim), rv,
                      f"dV {tag} late keys")
    if early:
        # dK / dV on whole key tiles that collect over the most query rows (every
        # row after them), for one KV group: the oracle's forward of that group's
        # rows is computed once and read by the keys-only backward
        gi = groups[1]
        hq = slice(gi * g, (gi + 1) * g)
        q1, do1 = f64(t["q"][:, hq]), f64(t["do"][:, hq])
        k1, v1 = f64(t["k"][:, gi:gi + 1]), f64(t["v"][:, gi:gi + 1])
        o1, l1 = oracle.fwd(q1, k1, v1, ds)
        ek = key_tiles_early(S, cu, rng)
        fk, fv = oracle.bwd_dkv_keys_fwd(q1, k1, v1, o1, l1, do1, ek, ds)
        assert_bf16_close(f64(dk[0, gi][ek]), fk, f"dK {tag} early key tiles")
        assert_bf16_close(f64(dv[0, gi][ek]), fv, f"dV {tag} early key tiles")
    check_identities(name, S, g, w.num_kv_heads, 1.0 / np.sqrt(w.head_dim), cu, dq, dk, dv,
                     t["q"], o_gpu, t["do"])


@pytest.mark.parametrize("one_pass", [False, True])
def test_gqa32k_ring_sampled(one_pass):
    check_sampled("gqa32k", "ring", one_pass=one_pass)


def test_docs64k_sampled():
    check_sampled("docs64k", "ring")


def test_gqa32k_d256_sampled():
    """gqa32k at head_dim 256: the three-pass backward."""
    check_sampled("gqa32k_d256", "ring")


@pytest.mark.parametrize("one_pass", [False, True])
def test_docs64k_perdoc_sampled(one_pass):
    check_sampled("docs64k_perdoc", "ring", one_pass=one_pass)


@pytest.mark.parametrize("rotate,one_pass", [("allgather", False), ("ring", True)])
def test_long128k_sampled(rotate, one_pass):
    # the oracle forward of a whole KV group at 128k is too slow for a test: early
    # key tiles are covered at 32k and 64k
    check_sampled("long128k", rotate, n_rows=48, n_keys=16, early=False, one_pass=one_pass)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_one_kv_head_eight_query_heads(D):
    """GQA group of 8 (one KV head): dK / dV sum over eight query heads."""
    case = make_case(1, 8, 1, 2048, D, 2, 240 + D, with_dout=True)
    check_full(case, 2, "ring")
