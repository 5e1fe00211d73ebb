"""Shared helpers for the parity tests: run the library through its C ABI and
compare against the oracle.  Tolerances are the ones the path is held to:
bf16 outputs and gradients max-abs 2e-2 and mean-abs 2e-3, fp32 LSE 1e-3."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_bf16_close(gpu: np.ndarray, ref: np.ndarray, what: str, max_abs=O_MAX, mean_abs=O_MEAN):
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    mx, mn = float(err.max()), float(err.mean())
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max {mx:.3e} mean {mn:.3e}"
    return mx, mn


def assert_lse_close(gpu: np.ndarray, ref: np.ndarray, what: str, tol=LSE_MAX):
    assert gpu.shape == ref.shape
    fin = np.isfinite(ref)
    assert (np.isfinite(gpu) == fin).all(), f"{what}: -inf pattern differs"
    err = float(np.abs(gpu[fin] - ref[fin]).max()) if fin.any() else 0.0
    assert err <= tol, f"{what}: max {err:.3e}"
    return err


def random_docs(seq_len: int, seed: int, median: float, lo: int = 1, hi: int | None = None):
    return synth.cu_seqlens(synth.doc_lengths(seq_len, seed, median, 1.0,
                                              (lo, hi or seq_len)))


def make_case(B, Hq, Hkv, S, D, cp, seed, amp=1.0, cu=None, with_dout=False):
    """Seeded inputs on the CPU (original order) plus the doc-start array."""
    t = synth.attn_inputs(B, Hq, Hkv, S, D, seed, amp=amp, with_dout=with_dout)
    t["cu_seqlens"] = cu
    t["ds"] = oracle.doc_start(S, cu)
    return t


def run_fwd(cz, case, cp, rotate="allgather", merge="fused", scale=0.0, dev="cuda"):
    """Plan + gather + forward on the GPU through the C ABI; returns (prob, plan,
    shard-order q/k/v on device, o, lse)."""
    q, k, v = (case[n].to(dev) for n in ("q", "k", "v"))
    B, Hq, S, D = q.shape
    cu = None if case["cu_seqlens"] is None else torch.from_numpy(case["cu_seqlens"]).to(dev)
    prob = cz.Problem(B, S, cp, Hq, k.shape[1], D, rotate, cu, merge, scale)
    plan = cz.Plan(prob)
    qs, ks, vs = plan.shard([q, k, v])
    o, lse = cz.attn_fwd(prob, plan, qs, ks, vs)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    return prob, plan, qs, ks, vs, o, lse
