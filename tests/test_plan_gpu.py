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
]


def cu_for(S, docs, seed):
    if docs is None:
        return None
    if docs == "lognormal":
        return synth.cu_seqlens(synth.doc_lengths(S, 3))
    if docs == "small":
        return random_docs(S, seed, 20.0)
    return np.array([0, S], np.int32)


@pytest.mark.parametrize("S,cp,rotate,docs", CASES)
def test_plan_bit_exact(S, cp, rotate, docs):
    cu = cu_for(S, docs, 5)
    ref = oracle.plan(S, cp, rotate, cu)
    prob = cz.Problem(1, S, cp, 2, 1, 64, rotate,
                      None if cu is None else torch.from_numpy(cu).cuda())
    plan = cz.Plan(prob)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    for key in ("perm", "inv_perm", "src", "doc_start", "rank_cu_off", "pairs"):
        got = getattr(plan, key).cpu().numpy()
        assert np.array_equal(got, ref[key]), key
    n = int(ref["rank_cu_off"][-1])
    assert np.array_equal(plan.rank_cu.cpu().numpy()[:n], ref["rank_cu"])


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
