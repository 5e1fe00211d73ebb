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


# Every comparison made through assert_bf16_close, for the per-configuration
# error report (written by conftest.py when CP_PARITY_REPORT names a file).
PARITY_LOG: list = []


def bf16_bound(ref: np.ndarray, max_abs: float = O_MAX) -> np.ndarray:
    """Per-element bound: the stated 2e-2 plus half a bf16 ulp of the reference value.
    A bf16 output cannot land closer to the exact value than half an ulp (its own
    rounding), so this is the 2e-2 budget on top of what the output format forces,
    and nothing more: 0.0217 at |ref| 0.5, 0.0278 at 3, 0.0513 at 8."""
    return max_abs + 0.5 * bf16_ulp(ref)


def parity_stats(gpu: np.ndarray, ref: np.ndarray, max_abs: float = O_MAX) -> dict:
    """Error summary of one comparison: max / mean error, how many elements exceed the
    plain 2e-2, and the worst element measured against its bound, in bf16 ulps of
    the reference value."""
    err = np.abs(gpu - ref)
    bound = bf16_bound(ref, max_abs)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    over = err > max_abs
    # of the elements beyond the plain 2e-2, the one farthest from its reference in ulps
    ulps_over = (err / bf16_ulp(ref))[over]
    k = int(np.argmax(ulps_over)) if over.any() else -1
    return dict(n=int(err.size), max=float(err.max()), mean=float(err.mean()),
                n_over_abs=int(over.sum()), n_over_bound=int((err > bound).sum()),
                worst_err=float(err[worst]), worst_ref=float(abs(ref[worst])),
                worst_bound=float(bound[worst]),
                worst_ulps=float(err[worst] / bf16_ulp(np.asarray(ref[worst]))),
                over_abs_max_ulps=float(ulps_over[k]) if k >= 0 else 0.0,
                over_abs_ref=float(np.abs(ref)[over][k]) if k >= 0 else 0.0)


def assert_bf16_close(gpu: np.ndarray, ref: np.ndarray, what: str, max_abs=O_MAX, mean_abs=O_MEAN):
    """Element bound |err| <= 2e-2 + ulp_bf16(ref)/2 (bf16_bound); mean bound
    mean |err| <= 2e-3."""
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    st = parity_stats(gpu, ref, max_abs)
    PARITY_LOG.append(dict(what=what, **st))
    ok = st["n_over_bound"] == 0 and st["mean"] <= mean_abs
    assert ok, (f"{what}: max {st['max']:.3e} mean {st['mean']:.3e}; {st['n_over_bound']} of "
                f"{st['n']} over the bound; worst: err {st['worst_err']:.3e} at |ref| "
                f"{st['worst_ref']:.3f} (bound {st['worst_bound']:.3e})")
    return st["max"], st["mean"]


def assert_lse_close(gpu: np.ndarray, ref: np.ndarray, what: str, tol=LSE_MAX):
    assert gpu.shape == ref.shape
    fin = np.isfinite(ref)
    assert (np.isfinite(gpu) == fin).all(), f"{what}: -inf pattern differs"
    err = float(np.abs(gpu[fin] - ref[fin]).max()) if fin.any() else 0.0
    assert err <= tol, f"{what}: max {err:.3e}"
    return err


def random_docs(seq_len: int, seed: int, median: float, lo: int = 1, hi: int | None = None,
                quantum: int = 1):
    return synth.cu_seqlens(synth.doc_lengths(seq_len, seed, median, 1.0,
                                              (lo, hi or seq_len), quantum))


def make_case(B, Hq, Hkv, S, D, cp, seed, amp=1.0, cu=None, with_dout=False, window=0,
              causal=True, shard="sequence"):
    """Seeded inputs on the CPU (original order) plus, per original position, the
    first key it attends to (document start, raised by a sliding window) and the
    last (itself under the causal mask, else the end of its document)."""
    t = synth.attn_inputs(B, Hq, Hkv, S, D, seed, amp=amp, with_dout=with_dout)
    t["cu_seqlens"] = cu
    t["window"] = window
    t["causal"] = causal
    t["shard"] = shard
    t["ds"] = oracle.first_key(S, cu, window)
    t["lk"] = oracle.last_key(S, cu, causal)
    return t


def run_fwd(cz, case, cp, rotate="allgather", merge="fused", scale=0.0, dev="cuda"):
    """Plan + gather + forward on the GPU through the C ABI; returns (prob, plan,
    shard-order q/k/v on device, o, lse)."""
    q, k, v = (case[n].to(dev) for n in ("q", "k", "v"))
    B, Hq, S, D = q.shape
    cu = None if case["cu_seqlens"] is None else torch.from_numpy(case["cu_seqlens"]).to(dev)
    prob = cz.Problem(B, S, cp, Hq, k.shape[1], D, rotate, cu, merge, scale, case.get("window", 0),
                      case.get("causal", True), shard=case.get("shard", "sequence"))
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
