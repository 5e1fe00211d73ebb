"""cp_attn_bwd_noalloc: the backward for callers that cannot allocate device memory
(for example while a CUDA graph is being captured, or under an allocator that
hands out no scratch).  It must give the same gradients as cp_attn_bwd, call
after call, using only the library's fixed scratch array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import context_zigzag_cp_b200 as cz
from context_zigzag_cp_b200 import _lib
from helpers import assert_bf16_close, f64, make_case

pytestmark = pytest.mark.gpu


def _call_noalloc(prob, plan, qs, ks, vs, o, lse, dos, dq, dk, dv):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return cz.lib().cp_attn_bwd_noalloc(prob.ref, plan.ref, p(qs), p(ks), p(vs), p(o), p(lse),
                                        p(dos), p(dq), p(dk), p(dv),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("D", [128, 256])
def test_noalloc_matches_workspace_backward_twice(D):
    case = make_case(1, 8, 2, 4096, D, 4, 31, with_dout=True)
    dev = "cuda"
    q, k, v, do = (case[n].to(dev) for n in ("q", "k", "v", "do"))
    prob = cz.Problem(1, 4096, 4, 8, 2, D, "ring")
    plan = cz.Plan(prob)
    qs, ks, vs, dos = plan.shard([q, k, v, do])
    o, lse = cz.attn_fwd(prob, plan, qs, ks, vs)
    ref = cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos)      # caller-provided workspace
    torch.cuda.synchronize()
    ref = [f64(t) for t in ref]
    for call in range(2):                                          # the array is reused
        outs = [torch.full_like(t, float("nan")) for t in (qs, ks, vs)]
        st = _call_noalloc(prob, plan, qs, ks, vs, o, lse, dos, *outs)
        assert st == _lib.CP_OK, st
        torch.cuda.synchronize()
        assert cz.get_device_status() == 0
        for name, got, want in zip(("dQ", "dK", "dV"), outs, ref):
            assert_bf16_close(f64(got), want, f"{name} no-alloc D={D} call {call}")


def test_noalloc_rejects_problems_beyond_the_array():
    rows_over = _lib.NOALLOC_MAX_ROWS // 4096 + 1      # heads so that rows exceed the limit
    prob = cz.Problem(1, 4096, 2, rows_over, 1, 128)
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    st = cz.lib().cp_attn_bwd_noalloc(prob.ref, ctypes.byref(plan), d, d, d, d, d, d, d, d, d,
                                      None)
    assert st == _lib.CP_ERR_WORKSPACE
