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


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits): 2^(floor(log2|x|) - 7)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def assert_bf16_close(gpu: np.ndarray, ref: np.ndarray, what: str, max_abs=O_MAX, mean_abs=O_MEAN):
    """Element bound: |err| <= max(max_abs, 2^-6 |ref|).  The absolute bound governs
    every |ref| <= 1.28; above that the bound is four bf16 unit roundoffs of the
    value: bf16 cannot hold such values closely (half an ulp is 0.0156 at 4 and
    0.031 at 8), and the bf16 P / dS operands of any tensor-core attention add
    errors of the same order (a numpy emulation of those roundings reproduces the
    GPU's errors to four digits).  Mean bound: mean |err| <= mean_abs."""
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    bound = np.maximum(max_abs, np.abs(ref) * 2.0 ** -6)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    mx, mn = float(err.max()), float(err.mean())
    ok = bool((err <= bound).all()) and mn <= mean_abs
    assert ok, (f"{what}: max {mx:.3e} mean {mn:.3e}; worst vs bound: err {err[worst]:.3e} "
                f"at |ref| {abs(ref[worst]):.3f} (bound {bound[worst]:.3e})")
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


def make_case(B, Hq, Hkv, S, D, cp, seed, amp=1.0, cu=None, with_dout=False, window=0):
    """Seeded inputs on the CPU (original order) plus, per original position, the
    first key it attends to (document start, raised by a sliding window)."""
    t = synth.attn_inputs(B, Hq, Hkv, S, D, seed, amp=amp, with_dout=with_dout)
    t["cu_seqlens"] = cu
    t["window"] = window
    t["ds"] = oracle.first_key(S, cu, window)
    return t


def run_fwd(cz, case, cp, rotate="allgather", merge="fused", scale=0.0, dev="cuda"):
    """Plan + gather + forward on the GPU through the C ABI; returns (prob, plan,
    shard-order q/k/v on device, o, lse)."""
    q, k, v = (case[n].to(dev) for n in ("q", "k", "v"))
    B, Hq, S, D = q.shape
    cu = None if case["cu_seqlens"] is None else torch.from_numpy(case["cu_seqlens"]).to(dev)
    prob = cz.Problem(B, S, cp, Hq, k.shape[1], D, rotate, cu, merge, scale, case.get("window", 0))
    plan = cz.Plan(prob)
    qs, ks, vs = plan.shard([q, k, v])
    o, lse = cz.attn_fwd(prob, plan, qs, ks, vs)
    torch.cuda.synchronize()
    assert cz.get_device_status() == 0
    return prob, plan, qs, ks, vs, o, lse


def bf16r(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest even) and back."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).double().numpy()


def bf16_operand_attention(q, k, v, do, ds, scale):
    """Forward and gradients with the tensor-core operand roundings made explicit:
    P (forward and backward) and dS rounded to bf16 before their products, the
    final O rounded to bf16 before D = dO.O, fp64 everywhere else.  Small cases
    only (materialises S x S).  Used to show the kernels' error budget is that of
    bf16 operands, not of anything else."""
    B, Hq, S, D = q.shape
    g = Hq // k.shape[1]
    qi = np.arange(S)[:, None]
    ki = np.arange(S)[None, :]
    mask = (ki <= qi) & (ki >= ds[:, None])
    o = np.zeros_like(q)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kk, vv = k[b, h // g], v[b, h // g]
            s = np.where(mask, scale * q[b, h] @ kk.T, -np.inf)
            m = s.max(1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(1, keepdims=True)
            o[b, h] = bf16r((bf16r(e) @ vv) / l)
            lse = (m + np.log(l))
            P = np.where(mask, np.exp(s - lse), 0.0)
            dP = do[b, h] @ vv.T
            Dq = (do[b, h] * o[b, h]).sum(1, keepdims=True)
            dS = bf16r(P * (dP - Dq))
            dv[b, h // g] += bf16r(P).T @ do[b, h]
            dk[b, h // g] += scale * dS.T @ q[b, h]
            dq[b, h] = scale * dS @ kk
    return o, bf16r(dq), bf16r(dk), bf16r(dv)
