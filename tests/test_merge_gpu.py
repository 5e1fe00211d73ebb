"""GPU LSE merge kernel against the oracle's combine."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
import oracle
from helpers import assert_bf16_close, assert_lse_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,rows,D", [(1, 100, 64), (2, 3000, 128), (8, 5000, 128), (3, 777, 4),
                                      (5, 1000, 256), (33, 300, 128), (64, 129, 64)])
def test_merge_matches_oracle(n, rows, D):
    g = np.random.default_rng(n * 1000 + D)
    o = g.standard_normal((n, rows, D)).astype(np.float32)
    lse = (g.standard_normal((n, rows)) * 3).astype(np.float32)
    # rows with no key in some parts, and rows with no key at all
    lse[g.random((n, rows)) < 0.3] = -np.inf
    lse[:, :7] = -np.inf
    o[np.isneginf(lse)] = np.nan          # a -inf part's O must never be read
    oo, ol = cz.lse_merge(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.lse_merge(np.nan_to_num(o.astype(np.float64)), lse.astype(np.float64))
    assert_bf16_close(oo.float().cpu().numpy().astype(np.float64), ref_o, f"merge O n={n}")
    assert_lse_close(ol.cpu().numpy().astype(np.float64), ref_l, f"merge LSE n={n}", tol=1e-5)
    assert (oo[:7].float() == 0).all()


def test_merge_of_attention_halves():
    """Two partial attentions over halves of each row's keys merge into the whole."""
    S, D = 256, 128
    g = np.random.default_rng(3)
    q, k, v = (g.standard_normal((1, 1, S, D)) for _ in range(3))
    o, lse = oracle.fwd(q, k, v)
    perm = np.arange(S, dtype=np.int32)
    a = oracle.partial(q, k, v, perm, 2, 1, 0)
    b = oracle.partial(q, k, v, perm, 2, 1, 1)
    po = np.stack([a[0][0], b[0][0]]).astype(np.float32)
    pl = np.stack([a[1][0], b[1][0]]).astype(np.float32)
    oo, ol = cz.lse_merge(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda())
    assert_bf16_close(oo.float().cpu().numpy().astype(np.float64), o[0, 0, S // 2:], "halves O")
    assert_lse_close(ol.cpu().numpy().astype(np.float64), lse[0, 0, S // 2:], "halves LSE", 1e-5)
