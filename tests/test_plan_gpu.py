"""GPU shard planner and gather against the oracle's plan: bit-exact."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
import synth
from helpers import random_docs

pytestmark = pytest.mark.gpu

CASES = [
    # (S, cp, rotate, docs)
    (512, 2, "allgather", None),
    (8192, 4, "allgather", None),
    (32768, 8, "ring", None),
    (65536, 8, "ring", "lognormal"),
    (65536, 8, "allgather", "lognormal"),
    (131072, 8, "allgather", None),
    (131072, 8, "ring", None),
    (96, 3, "ring", None),               # C = 16: planner works for any chunk length
    (64, 1, "allgather", None),
    (4096, 2, "ring", "small"),          # many short documents, some of length 1
    (4096, 4, "allgather", "one"),       # a single document = plain causal
    # per-document zigzag: every document cut into 2cp chunks of whole 128-row tiles
    (65536, 8, "ring", "perdoc"),
    (6144, 3, "allgather", "perdoc"),
    (4096, 2, "ring", "perdoc_one"),
]


def cu_for(S, cp, docs, seed):
    if docs is None:
        return None
    if docs == "lognormal":
        return synth.cu_seqlens(synth.doc_lengths(S, 3))
    if docs == "small":
        return random_docs(S, seed, 20.0)
    if docs == "perdoc":
        return random_docs(S, seed, 2048.0, 128, quantum=256 * cp)
    return np.array([0, S], np.int32)


@pytest.mark.parametrize("S,cp,rotate,docs", CASES)
def test_plan_bit_exact(S, cp, rotate, docs):
    cu = cu_for(S, cp, docs, 5)
    shard = "doc" if docs is not None and docs.startswith("perdoc") else "sequence"
    ref = oracle.plan(S, cp, rotate, cu, shard=shard)
    prob = cz.Problem(1, S, cp, 2, 1, 64, rotate,
                      None if cu is None else torch.from_numpy(cu).cuda(), shard=shard)
    plan = cz.Plan(prob)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    for key in ("perm", "inv_perm", "src", "doc_start", "rank_cu_off", "pairs"):
        got = getattr(plan, key).cpu().numpy()
        assert np.array_equal(got, ref[key]), key
    n = int(ref["rank_cu_off"][-1])
    assert n <= plan.rank_cu.numel()
    assert np.array_equal(plan.rank_cu.cpu().numpy()[:n], ref["rank_cu"])
    if (S // (2 * cp)) % 128 == 0 and (shard == "doc" or S % 128 == 0):
        # tile tables: the start of every shard tile, and its inverse
        perm, inv = ref["perm"], ref["inv_perm"]
        assert np.array_equal(plan.tile_orig.cpu().numpy(), perm[::128])
        assert np.array_equal(plan.tile_shard.cpu().numpy(), inv[::128] // 128)


def test_per_doc_uneven_documents_flagged_on_device():
    """Per-document chunks must be whole tiles: any other length records
    CP_ERR_UNSUPPORTED, and every table still holds indices inside the sequence."""
    S, cp = 4096, 2
    for cu in (np.array([0, 1000, 4096], np.int32), np.array([0, 512, 2048, 4096], np.int32),
               np.array([0, 4000, 4096], np.int32)):
        prob = cz.Problem(1, S, cp, 2, 2, 64, "ring", torch.from_numpy(cu).cuda(), shard="doc")
        plan = cz.Plan(prob)
        torch.cuda.synchronize()
        st = cz.get_device_status()
        bad = any(n % (256 * cp) for n in np.diff(cu))
        assert st == (2 if bad else 0), (cu, st)       # CP_ERR_UNSUPPORTED
        for t in (plan.perm, plan.inv_perm):
            a = t.cpu().numpy()
            assert a.min() >= 0 and a.max() < S
        for t in (plan.tile_orig, plan.tile_shard):
            a = t.cpu().numpy()
            assert a.min() >= 0 and a.max() < S
    bad_cu = torch.tensor([0, 600, 4096], dtype=torch.int32, device="cuda")
    cz.Plan(cz.Problem(1, S, cp, 2, 2, 64, "ring", bad_cu, shard="doc"))
    assert cz.get_device_status() == 2


def test_per_doc_gather_and_restore_bit_exact():
    S, cp = 6144, 3
    cu = random_docs(S, 9, 1500.0, 128, quantum=256 * cp)
    g = torch.Generator().manual_seed(8)
    q = torch.randn(2, 3, S, 64, generator=g).to(torch.bfloat16)
    x = torch.randint(0, 2 ** 31, (2, S, 4), generator=g, dtype=torch.int32)
    prob = cz.Problem(2, S, cp, 3, 3, 64, "ring", torch.from_numpy(cu).cuda(), shard="doc")
    plan = cz.Plan(prob)
    sh = plan.shard([q.cuda(), x.cuda()])
    perm = torch.from_numpy(oracle.plan(S, cp, "ring", cu, shard="doc")["perm"]).long()
    for a, b in zip((q, x), sh):
        assert torch.equal(b.cpu(), a[..., perm, :])
    for a, b in zip((q, x), plan.unshard(sh)):
        assert torch.equal(b.cpu(), a)


@pytest.mark.parametrize("S,cp", [(8192, 4), (131072, 8), (96, 3)])
def test_gather_and_restore_bit_exact(S, cp):
    g = torch.Generator().manual_seed(7)
    q = torch.randn(1, 4, S, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(2, 2, S, 64, generator=g).to(torch.bfloat16)
    x = torch.randint(0, 2 ** 31, (3, S, 12), generator=g, dtype=torch.int32)   # 48-byte rows
    prob = cz.Problem(1, S, cp, 4, 2, 128)
    plan = cz.Plan(prob)
    dev = [t.cuda() for t in (q, k, x)]
    sh = plan.shard(dev)
    perm = torch.from_numpy(oracle.plan(S, cp)["perm"]).long()
    for a, b in zip((q, k, x), sh):
        assert torch.equal(b.cpu(), a[..., perm, :])
    back = plan.unshard(sh)
    for a, b in zip((q, k, x), back):
        assert torch.equal(b.cpu(), a)


def test_bad_cu_seqlens_flagged_on_device():
    S = 1024
    for cu in (np.array([0, 500, 400, 1024], np.int32), np.array([0, 500, 1000], np.int32),
               np.array([3, 500, 1024], np.int32)):
        prob = cz.Problem(1, S, 2, 2, 2, 64, "allgather", torch.from_numpy(cu).cuda())
        cz.Plan(prob)
        assert cz.get_device_status() == 1      # CP_ERR_INVALID_ARG
    cz.Plan(cz.Problem(1, S, 2, 2, 2, 64))
    assert cz.get_device_status() == 0
