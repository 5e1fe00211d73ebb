"""The forward kernel's software exp2 (Cody-Waite reduction + Remez degree-3
polynomial) against CUDA's ex2 and against exp2 in float64."""
import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz

pytestmark = pytest.mark.gpu


def test_software_exp2_error_bound():
    x = torch.cat([torch.linspace(-124.0, 8.0, 2_000_001), torch.tensor([-125.0, 0.0, 0.5, -0.5])])
    xs = x.cuda()
    ys, yh = cz.selftest_exp2(xs)
    ref = np.exp2(x.double().numpy())
    rel = np.abs(ys.double().cpu().numpy() / ref - 1.0)
    assert rel.max() < 1.0e-4                      # 7.5e-5 by construction (Remez fit)
    relh = np.abs(yh.double().cpu().numpy() / ref - 1.0)
    assert relh.max() < 1e-5                       # the hardware ex2 for comparison
    # far below bf16's half-ulp, so P rounded to bf16 is unaffected almost everywhere
    assert rel.max() < 2.0 ** -9 / 20
