"""Zigzag context-parallel causal attention on one B200.

A thin binding over libcpattn (include/cp_attn.h): every step of the path
(plan, gather, forward, merge, backward) runs in the library's CUDA kernels;
this module only marshals torch tensors (device memory and streams) into the
C ABI.  There is no CPU fallback: without the built library every call raises.

Typical use (all tensors on one CUDA device, bf16 BHSD in original order):

    prob = Problem(batch=1, seq_len=S, cp=8, num_heads=32, num_kv_heads=8, head_dim=128,
                   rotate="ring")
    plan = Plan(prob)
    qs, ks, vs = plan.shard([q, k, v])            # original -> shard order
    o, lse = attn_fwd(prob, plan, qs, ks, vs)     # shard order
    dq, dk, dv = attn_bwd(prob, plan, qs, ks, vs, o, lse, plan.shard([do])[0])
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import CpPlan, CpProblem, STATUS_NAMES

__all__ = ["CPError", "Problem", "Plan", "attn_fwd", "attn_bwd", "lse_merge",
           "fwd_workspace_bytes", "bwd_workspace_bytes", "get_device_status",
           "set_wait_limit_ns", "selftest_wait_timeout", "version", "lib", "launch_count",
           "LaunchTrace", "attn_bwd_noalloc", "selftest_stall", "attn_fwd_rank", "attn_fwd_step",
           "attn_bwd_rank", "attn_bwd_step", "f32_to_bf16"]


class CPError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    return _lib.load()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise CPError(status, what)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _on_device(t, dev) -> bool:
    """True when tensor t lives on CUDA device dev."""
    return t.device.type == "cuda" and t.device == dev


def _validate(*specs) -> None:
    """Refuse tensors the kernels would read or write out of bounds before any
    pointer reaches the library.  ``specs``: (tensor or None, shape, dtype, name);
    None entries are outputs the binding allocates itself.  Shapes and dtypes are
    checked first, then that every tensor is contiguous and on one CUDA device."""
    given = [sp for sp in specs if sp[0] is not None]
    for t, shape, dtype, name in given:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
        if t.dtype != dtype:
            raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    dev = given[0][0].device
    for t, _, _, name in given:
        if not _on_device(t, dev):
            raise ValueError(f"{name}: on {t.device}; every tensor must be on one CUDA device "
                             f"(the first is on {dev})")
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")


def _check_plan(prob: "Problem", plan: "Plan", dev) -> None:
    """The plan's arrays are sized and filled for the problem it was built from;
    the kernels index them by the problem's seq_len and cp, so a plan built for
    another problem (or living on another device) is refused here."""
    if not isinstance(plan, Plan):
        raise TypeError(f"plan: expected a Plan, got {type(plan).__name__}")
    pp = plan.prob
    if (pp.seq_len, pp.cp, pp.rotate) != (prob.seq_len, prob.cp, prob.rotate):
        raise ValueError(f"plan: built for seq_len {pp.seq_len}, cp {pp.cp}, {pp.rotate}; the "
                         f"problem has seq_len {prob.seq_len}, cp {prob.cp}, {prob.rotate}")
    if getattr(pp, "causal", True) != getattr(prob, "causal", True):
        raise ValueError("plan: built for the other mask (causal / no causal mask)")
    if getattr(pp, "shard", "sequence") != getattr(prob, "shard", "sequence"):
        raise ValueError(f"plan: built for {pp.shard!r} sharding; the problem has {prob.shard!r}")
    if getattr(pp, "window", 0) != getattr(prob, "window", 0):
        raise ValueError(f"plan: built for window {pp.window}; the problem has {prob.window}")
    if pp.cu_seqlens is not prob.cu_seqlens:
        same = (pp.cu_seqlens is not None and prob.cu_seqlens is not None
                and pp.cu_seqlens.shape == prob.cu_seqlens.shape
                and bool(torch.equal(pp.cu_seqlens, prob.cu_seqlens)))
        if not same:
            raise ValueError("plan: built for other documents (cu_seqlens) than the problem's")
    if not _on_device(plan.perm, dev):
        raise ValueError(f"plan: on {plan.perm.device}, the tensors are on {dev}")
    if prob.cu_seqlens is not None and not _on_device(prob.cu_seqlens, dev):
        raise ValueError(f"cu_seqlens: on {prob.cu_seqlens.device}, the tensors are on {dev}")


def _attn_shapes(prob: "Problem"):
    q = (prob.batch, prob.num_heads, prob.seq_len, prob.head_dim)
    kv = (prob.batch, prob.num_kv_heads, prob.seq_len, prob.head_dim)
    return q, kv, q[:-1]


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def version() -> int:
    return int(lib().cp_version())


class Problem:
    """cp_problem_t.  ``cu_seqlens`` (int32, original order, device) turns on the
    packed-document mask; ``window`` > 0 adds a sliding window (the query at q
    sees keys q - window < k <= q); ``causal=False`` drops the causal mask (every
    query sees every key; no documents or window then); ``bwd_one_pass=True``
    selects the one-pass backward (dQ by fp32 atomic reductions; the default is the
    two deterministic passes); ``shard="doc"`` cuts every document, not the whole
    sequence, into 2*cp zigzag chunks (needs ``cu_seqlens``, and every document's
    length a multiple of 256*cp)."""

    def __init__(self, batch: int, seq_len: int, cp: int, num_heads: int, num_kv_heads: int,
                 head_dim: int, rotate: str = "allgather", cu_seqlens: torch.Tensor | None = None,
                 merge: str = "fused", softmax_scale: float = 0.0, window: int = 0,
                 causal: bool = True, bwd_one_pass: bool = False, shard: str = "sequence"):
        if not causal and (cu_seqlens is not None or window):
            raise ValueError("causal=False takes no cu_seqlens and no window")
        if shard not in _lib.SHARD:
            raise ValueError(f"shard: expected one of {sorted(_lib.SHARD)}, got {shard!r}")
        if shard == "doc" and cu_seqlens is None:
            raise ValueError("shard='doc' needs cu_seqlens")
        if cu_seqlens is not None:
            if not isinstance(cu_seqlens, torch.Tensor):
                raise TypeError("cu_seqlens: expected a torch.Tensor")
            if cu_seqlens.dtype != torch.int32 or cu_seqlens.device.type != "cuda":
                raise ValueError(f"cu_seqlens: must be an int32 CUDA tensor, got "
                                 f"{cu_seqlens.dtype} on {cu_seqlens.device}")
            if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2 or not cu_seqlens.is_contiguous():
                raise ValueError("cu_seqlens: must be a contiguous 1-D tensor of num_docs + 1 >= 2 "
                                 "offsets")
        self.cu_seqlens = cu_seqlens
        self.window = window
        self.batch, self.seq_len, self.cp = batch, seq_len, cp
        self.num_heads, self.num_kv_heads, self.head_dim = num_heads, num_kv_heads, head_dim
        self.rotate, self.merge, self.causal = rotate, merge, causal
        self.bwd_one_pass = bwd_one_pass
        self.shard = shard
        self.softmax_scale = float(softmax_scale)
        self.num_docs = 0 if cu_seqlens is None else int(cu_seqlens.numel()) - 1
        mask = "full" if not causal else ("causal" if cu_seqlens is None else "doc")
        self.c = CpProblem(batch, seq_len, cp, num_heads, num_kv_heads, head_dim,
                           _lib.ROTATE[rotate], _lib.MASK[mask],
                           _lib.MERGE[merge], self.softmax_scale, self.num_docs, int(window),
                           int(bool(bwd_one_pass)), _lib.SHARD[shard],
                           None if cu_seqlens is None else cu_seqlens.data_ptr())

    def _replace(self, **kw) -> "Problem":
        args = dict(batch=self.batch, seq_len=self.seq_len, cp=self.cp, num_heads=self.num_heads,
                    num_kv_heads=self.num_kv_heads, head_dim=self.head_dim, rotate=self.rotate,
                    cu_seqlens=self.cu_seqlens, merge=self.merge,
                    softmax_scale=self.softmax_scale, window=self.window, causal=self.causal,
                    bwd_one_pass=self.bwd_one_pass, shard=self.shard)
        args.update(kw)
        return Problem(**args)

    def with_merge(self, merge: str) -> "Problem":
        return self._replace(merge=merge)

    def with_one_pass(self, bwd_one_pass: bool) -> "Problem":
        return self._replace(bwd_one_pass=bwd_one_pass)

    def rank_cu_len(self) -> int:
        """Entries of the plan's per-rank segment list (cp_plan_t.rank_cu)."""
        if self.shard == "doc":
            return self.cp * (2 * self.num_docs + 1)
        return 3 * self.cp + max(self.num_docs, 1)

    @property
    def ref(self):
        return ctypes.byref(self.c)


class Plan:
    """Caller-owned plan buffers (cp_plan_t) filled by cp_plan_shards."""

    def __init__(self, prob: Problem, device=None, stream=None):
        dev = torch.device("cuda") if device is None else torch.device(device)
        S, cp = prob.seq_len, prob.cp
        i32 = dict(dtype=torch.int32, device=dev)
        self.prob = prob
        self.perm = torch.empty(S, **i32)
        self.inv_perm = torch.empty(S, **i32)
        self.src = torch.empty(cp * cp, **i32)
        self.doc_start = torch.empty(S, **i32)
        self.rank_cu_off = torch.empty(cp + 1, **i32)
        self.rank_cu = torch.empty(prob.rank_cu_len(), **i32)
        self.pairs = torch.empty(cp, dtype=torch.int64, device=dev)
        self.tile_orig = torch.empty((S + 127) // 128, **i32)
        self.tile_shard = torch.empty((S + 127) // 128, **i32)
        self.c = CpPlan(*(t.data_ptr() for t in (self.perm, self.inv_perm, self.src,
                                                  self.doc_start, self.rank_cu_off,
                                                  self.rank_cu, self.pairs, self.tile_orig,
                                                  self.tile_shard)))
        self.build(stream=stream)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def _bufs(self, tensors, outs):
        n = len(tensors)
        if len(outs) != n:
            raise ValueError(f"{n} input buffers but {len(outs)} output buffers")
        for i, (t, u) in enumerate(zip(tensors, outs)):
            if not isinstance(t, torch.Tensor) or not isinstance(u, torch.Tensor):
                raise TypeError(f"buffer {i}: expected torch.Tensor inputs and outputs")
            if t.dim() < 2 or t.shape[-2] != self.prob.seq_len:
                raise ValueError(f"buffer {i}: shape {tuple(t.shape)} is not [..., seq_len, row]")
            _validate((t, t.shape, t.dtype, f"buffer {i}"), (u, t.shape, t.dtype, f"output {i}"))
            if not _on_device(t, self.perm.device):
                raise ValueError(f"buffer {i}: on {t.device}, the plan is on {self.perm.device}")
        outer = (ctypes.c_int64 * max(n, 1))(*[t[..., 0, 0].numel() for t in tensors])
        row = (ctypes.c_int64 * max(n, 1))(*[t.shape[-1] * t.element_size() for t in tensors])
        return n, outer, row

    def build(self, bufs_in=(), bufs_out=(), stream=None):
        n, outer, row = self._bufs(list(bufs_in), list(bufs_out))
        pin = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in bufs_in])
        pout = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in bufs_out])
        _check(lib().cp_plan_shards(self.prob.ref, self.ref, n, pin, pout, outer, row, None,
                                    None, _stream(stream)), "cp_plan_shards")

    def shard(self, tensors, stream=None):
        """Gather tensors [..., S, row] from original into shard order (new tensors)."""
        outs = [torch.empty_like(t) for t in tensors]
        self.build(tensors, outs, stream)
        return outs

    def unshard(self, tensors, stream=None):
        """Scatter tensors [..., S, row] from shard back into original order."""
        outs = [torch.empty_like(t) for t in tensors]
        n, outer, row = self._bufs(list(tensors), outs)
        pin = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in tensors])
        pout = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in outs])
        _check(lib().cp_unshard(self.prob.ref, self.ref, n, pin, pout, outer, row,
                                _stream(stream)), "cp_unshard")
        return outs


def fwd_workspace_bytes(prob: Problem) -> int:
    n = ctypes.c_size_t(0)
    dummy = ctypes.c_void_p(256)
    plan = CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    _check(lib().cp_attn_fwd(prob.ref, ctypes.byref(plan), dummy, dummy, dummy, dummy, dummy,
                             None, ctypes.byref(n), None), "cp_attn_fwd(workspace query)")
    return n.value


def bwd_workspace_bytes(prob: Problem) -> int:
    n = ctypes.c_size_t(0)
    d = ctypes.c_void_p(256)
    plan = CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    _check(lib().cp_attn_bwd(prob.ref, ctypes.byref(plan), d, d, d, d, d, d, d, d, d, None,
                             ctypes.byref(n), None), "cp_attn_bwd(workspace query)")
    return n.value


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return None
    if ws is not None and (ws.device != device or not ws.is_contiguous()):
        raise ValueError(f"ws: must be a contiguous tensor on {device}")
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def attn_fwd(prob: Problem, plan: Plan, q, k, v, o=None, lse=None, ws=None, stream=None):
    """cp_attn_fwd on shard-order q [B,Hq,S,D], k/v [B,Hkv,S,D]; returns (o, lse)."""
    qs, kvs, ls = _attn_shapes(prob)
    bf16 = torch.bfloat16
    _validate((q, qs, bf16, "q"), (k, kvs, bf16, "k"), (v, kvs, bf16, "v"), (o, qs, bf16, "o"),
              (lse, ls, torch.float32, "lse"))
    _check_plan(prob, plan, q.device)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    nbytes = fwd_workspace_bytes(prob)
    w = _workspace(nbytes, q.device, ws)
    n = ctypes.c_size_t(nbytes)
    _check(lib().cp_attn_fwd(prob.ref, plan.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                             _ptr(w), ctypes.byref(n) if w is not None else None,
                             _stream(stream)), "cp_attn_fwd")
    return o, lse


def _validate_bwd(prob, plan, q, k, v, o, lse, do, dq, dk, dv):
    qs, kvs, ls = _attn_shapes(prob)
    bf16 = torch.bfloat16
    _validate((q, qs, bf16, "q"), (k, kvs, bf16, "k"), (v, kvs, bf16, "v"), (o, qs, bf16, "o"),
              (lse, ls, torch.float32, "lse"), (do, qs, bf16, "do"), (dq, qs, bf16, "dq"),
              (dk, kvs, bf16, "dk"), (dv, kvs, bf16, "dv"))
    _check_plan(prob, plan, q.device)


def attn_bwd(prob: Problem, plan: Plan, q, k, v, o, lse, do, dq=None, dk=None, dv=None,
             ws=None, stream=None):
    """cp_attn_bwd; returns (dq, dk, dv) in shard order."""
    _validate_bwd(prob, plan, q, k, v, o, lse, do, dq, dk, dv)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = bwd_workspace_bytes(prob)
    w = _workspace(nbytes, q.device, ws)
    n = ctypes.c_size_t(nbytes)
    _check(lib().cp_attn_bwd(prob.ref, plan.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                             _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(w),
                             ctypes.byref(n) if w is not None else None, _stream(stream)),
           "cp_attn_bwd")
    return dq, dk, dv


def attn_bwd_noalloc(prob: Problem, plan: Plan, q, k, v, o, lse, do, dq, dk, dv, stream=None):
    """cp_attn_bwd_noalloc: the backward without a workspace, for callers that cannot
    allocate device memory at this point (inside a CUDA graph capture, or under an
    allocator that hands out no scratch).  Its scratch lives in a fixed 32 MiB array
    inside the library (batch * heads * seq_len <= 4,194,304 rows); calls that could
    overlap on the GPU must be serialised, and the first call on a device must come
    before any stream capture.  The caller passes every output; nothing is allocated."""
    if dq is None or dk is None or dv is None:
        raise ValueError("attn_bwd_noalloc: dq, dk and dv must be given")
    _validate_bwd(prob, plan, q, k, v, o, lse, do, dq, dk, dv)
    _check(lib().cp_attn_bwd_noalloc(prob.ref, plan.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                     _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                                     _stream(stream)), "cp_attn_bwd_noalloc")
    return dq, dk, dv


# ------------------------------------------------------------------ per-rank calls
# One process per GPU: rank r holds its local query shard (2C = S / cp rows per
# head, local row t = shard position r*2C + t); the K/V shards of the other ranks
# arrive by collectives run outside the library (see context_zigzag_cp_b200.dist).

def _rank_shapes(prob: "Problem"):
    n2c = prob.seq_len // prob.cp
    q = (prob.batch, prob.num_heads, n2c, prob.head_dim)
    kv_all = (prob.batch, prob.num_kv_heads, prob.seq_len, prob.head_dim)
    kv_one = (prob.batch, prob.num_kv_heads, n2c, prob.head_dim)
    return q, kv_all, kv_one, q[:-1]


def _ws_query(fn, *args) -> int:
    n = ctypes.c_size_t(0)
    _check(fn(*args, None, ctypes.byref(n), None), "workspace query")
    return n.value


def attn_fwd_rank(prob: Problem, plan: Plan, rank: int, q, k, v, o=None, lse=None, ws=None,
                  stream=None):
    """cp_attn_fwd_rank: rank's local q [B,Hq,2C,D] against gathered k/v [B,Hkv,S,D]
    (shard order); returns the rank's (o [B,Hq,2C,D] bf16, lse [B,Hq,2C] fp32)."""
    qs, kva, _, ls = _rank_shapes(prob)
    bf16 = torch.bfloat16
    _validate((q, qs, bf16, "q"), (k, kva, bf16, "k"), (v, kva, bf16, "v"), (o, qs, bf16, "o"),
              (lse, ls, torch.float32, "lse"))
    _check_plan(prob, plan, q.device)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty(ls, dtype=torch.float32, device=q.device) if lse is None else lse
    d = ctypes.c_void_p(256)
    nbytes = _ws_query(lib().cp_attn_fwd_rank, prob.ref, plan.ref, int(rank), d, d, d, d, d)
    w = _workspace(nbytes, q.device, ws)
    n = ctypes.c_size_t(nbytes)
    _check(lib().cp_attn_fwd_rank(prob.ref, plan.ref, int(rank), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                  _ptr(lse), _ptr(w), ctypes.byref(n) if w is not None else None,
                                  _stream(stream)), "cp_attn_fwd_rank")
    return o, lse


def attn_fwd_step(prob: Problem, plan: Plan, rank: int, step: int, q, k, v, o_part=None,
                  lse_part=None, stream=None):
    """cp_attn_fwd_step: rank's local q against the one K/V shard it holds at ring step
    `step` (k/v [B,Hkv,2C,D]); returns the step's fp32 partial (o [B,Hq,2C,D],
    lse [B,Hq,2C]; lse = -inf where no key of the shard is visible)."""
    qs, _, kv1, ls = _rank_shapes(prob)
    bf16, f32 = torch.bfloat16, torch.float32
    _validate((q, qs, bf16, "q"), (k, kv1, bf16, "k"), (v, kv1, bf16, "v"),
              (o_part, qs, f32, "o_part"), (lse_part, ls, f32, "lse_part"))
    _check_plan(prob, plan, q.device)
    o_part = torch.empty(qs, dtype=f32, device=q.device) if o_part is None else o_part
    lse_part = torch.empty(ls, dtype=f32, device=q.device) if lse_part is None else lse_part
    _check(lib().cp_attn_fwd_step(prob.ref, plan.ref, int(rank), int(step), _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(o_part), _ptr(lse_part), _stream(stream)),
           "cp_attn_fwd_step")
    return o_part, lse_part


def attn_bwd_rank(prob: Problem, plan: Plan, rank: int, q, k, v, o, lse, do, dq=None,
                  dk_part=None, dv_part=None, ws=None, stream=None):
    """cp_attn_bwd_rank: the rank's dQ [B,Hq,2C,D] and its fp32 share of dK/dV for every
    key [B,Hkv,S,D] (to be summed over the ranks by a reduce-scatter)."""
    qs, kva, _, ls = _rank_shapes(prob)
    bf16, f32 = torch.bfloat16, torch.float32
    _validate((q, qs, bf16, "q"), (k, kva, bf16, "k"), (v, kva, bf16, "v"), (o, qs, bf16, "o"),
              (lse, ls, f32, "lse"), (do, qs, bf16, "do"), (dq, qs, bf16, "dq"),
              (dk_part, kva, f32, "dk_part"), (dv_part, kva, f32, "dv_part"))
    _check_plan(prob, plan, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk_part = torch.empty(kva, dtype=f32, device=q.device) if dk_part is None else dk_part
    dv_part = torch.empty(kva, dtype=f32, device=q.device) if dv_part is None else dv_part
    d = ctypes.c_void_p(256)
    nbytes = _ws_query(lib().cp_attn_bwd_rank, prob.ref, plan.ref, int(rank), d, d, d, d, d, d, d,
                       d, d)
    w = _workspace(nbytes, q.device, ws)
    n = ctypes.c_size_t(nbytes)
    _check(lib().cp_attn_bwd_rank(prob.ref, plan.ref, int(rank), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk_part),
                                  _ptr(dv_part), _ptr(w), ctypes.byref(n) if w is not None else None,
                                  _stream(stream)), "cp_attn_bwd_rank")
    return dq, dk_part, dv_part


def attn_bwd_step(prob: Problem, plan: Plan, rank: int, step: int, q, k, v, o, lse, do,
                  dq_sum, dk_sum, dv_sum, ws=None, stream=None):
    """cp_attn_bwd_step: one ring step of the backward.  Adds the step's share of the
    rank's dQ into dq_sum [B,Hq,2C,D] and of shard src[rank][step]'s dK / dV into
    dk_sum / dv_sum [B,Hkv,2C,D] (fp32, zeroed by the caller before the first step)."""
    qs, _, kv1, ls = _rank_shapes(prob)
    bf16, f32 = torch.bfloat16, torch.float32
    for t, name in ((dq_sum, "dq_sum"), (dk_sum, "dk_sum"), (dv_sum, "dv_sum")):
        if t is None:
            raise ValueError(f"{name}: the fp32 sum to add into is required")
    _validate((q, qs, bf16, "q"), (k, kv1, bf16, "k"), (v, kv1, bf16, "v"), (o, qs, bf16, "o"),
              (lse, ls, f32, "lse"), (do, qs, bf16, "do"), (dq_sum, qs, f32, "dq_sum"),
              (dk_sum, kv1, f32, "dk_sum"), (dv_sum, kv1, f32, "dv_sum"))
    _check_plan(prob, plan, q.device)
    d = ctypes.c_void_p(256)
    nbytes = _ws_query(lib().cp_attn_bwd_step, prob.ref, plan.ref, int(rank), int(step), d, d, d, d, d,
                       d, d, d, d)
    w = _workspace(nbytes, q.device, ws)
    n = ctypes.c_size_t(nbytes)
    _check(lib().cp_attn_bwd_step(prob.ref, plan.ref, int(rank), int(step), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(o), _ptr(lse), _ptr(do), _ptr(dq_sum), _ptr(dk_sum),
                                  _ptr(dv_sum), _ptr(w), ctypes.byref(n) if w is not None else None,
                                  _stream(stream)), "cp_attn_bwd_step")
    return dq_sum, dk_sum, dv_sum


def f32_to_bf16(x, out=None, stream=None):
    """cp_f32_to_bf16 on a contiguous fp32 CUDA tensor (numel a multiple of 4)."""
    _validate((x, tuple(x.shape), torch.float32, "x"), (out, tuple(x.shape), torch.bfloat16, "out"))
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if out is None else out
    _check(lib().cp_f32_to_bf16(_ptr(x), _ptr(out), x.numel(), _stream(stream)), "cp_f32_to_bf16")
    return out


def lse_merge(o_parts, lse_parts, o_out=None, lse_out=None, stream=None):
    """cp_lse_merge on o_parts fp32 [n, rows, D], lse_parts fp32 [n, rows]."""
    if not isinstance(o_parts, torch.Tensor) or o_parts.dim() != 3:
        raise ValueError("o_parts: expected a [n, rows, head_dim] tensor")
    n, rows, D = o_parts.shape
    _validate((o_parts, (n, rows, D), torch.float32, "o_parts"),
              (lse_parts, (n, rows), torch.float32, "lse_parts"),
              (o_out, (rows, D), torch.bfloat16, "o_out"), (lse_out, (rows,), torch.float32, "lse_out"))
    if o_out is None:
        o_out = torch.empty((rows, D), dtype=torch.bfloat16, device=o_parts.device)
    if lse_out is None:
        lse_out = torch.empty(rows, dtype=torch.float32, device=o_parts.device)
    _check(lib().cp_lse_merge(rows, D, n, _ptr(o_parts), _ptr(lse_parts), _ptr(o_out),
                              _ptr(lse_out), _stream(stream)), "cp_lse_merge")
    return o_out, lse_out


def get_device_status(stream=None) -> int:
    st = ctypes.c_int32(0)
    _check(lib().cp_get_device_status(ctypes.byref(st), _stream(stream)), "cp_get_device_status")
    return st.value


def set_wait_limit_ns(limit_ns: int) -> None:
    _check(lib().cp_set_wait_limit_ns(int(limit_ns)), "cp_set_wait_limit_ns")


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib().cp_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "cp_selftest_wait_timeout")


def selftest_stall(kernel: str, prob: Problem, plan: Plan, q, k, v, o, lse, do=None, dq=None,
                   dk=None, dv=None, stream=None) -> None:
    """cp_selftest_stall: run the forward (kernel "fwd") or the backward ("bwd_dkdv",
    "bwd_dq") with CTA 0 of the named kernel never receiving its first K/V tile, so
    that its bounded wait runs out (the test of the kernels' timeout teardown).
    For "fwd", o and lse are outputs; for the backward they are inputs."""
    kid = _lib.KERNEL_IDS.get(kernel, -1)
    if kernel == "fwd":
        qs, kvs, ls = _attn_shapes(prob)
        _validate((q, qs, torch.bfloat16, "q"), (k, kvs, torch.bfloat16, "k"),
                  (v, kvs, torch.bfloat16, "v"), (o, qs, torch.bfloat16, "o"),
                  (lse, ls, torch.float32, "lse"))
        _check_plan(prob, plan, q.device)
        nbytes = fwd_workspace_bytes(prob)
    else:
        _validate_bwd(prob, plan, q, k, v, o, lse, do, dq, dk, dv)
        # the stalled kernel picks the backward form: the one-pass kernel needs its dQ
        # accumulator whatever the problem's default form is
        nbytes = bwd_workspace_bytes(prob.with_one_pass(kernel == "bwd_fused"))
    w = _workspace(nbytes, q.device, None)
    n = ctypes.c_size_t(nbytes)
    _check(lib().cp_selftest_stall(kid, prob.ref, plan.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                   _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(w),
                                   ctypes.byref(n) if w is not None else None, _stream(stream)),
           "cp_selftest_stall")


def selftest_exp2(x: torch.Tensor, stream=None):
    """(software exp2, hardware ex2) of a float32 CUDA tensor."""
    ys, yh = torch.empty_like(x), torch.empty_like(x)
    _check(lib().cp_selftest_exp2(_ptr(x), _ptr(ys), _ptr(yh), x.numel(), _stream(stream)),
           "cp_selftest_exp2")
    return ys, yh


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().cp_launch_count())


class LaunchTrace:
    """Context manager around cp_trace_begin / cp_trace_end: CUDA events recorded
    on the launching stream just before and after each library kernel launch."""

    def __init__(self, capacity: int = 512):
        self.cap = capacity
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:          # torch creates the CUDA event on first record
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self._ids = (ctypes.c_int32 * capacity)()
        self.n = 0

    def __enter__(self):
        _check(lib().cp_trace_begin(self._handles, self.cap), "cp_trace_begin")
        return self

    def __exit__(self, *exc):
        n = ctypes.c_int32(0)
        _check(lib().cp_trace_end(ctypes.byref(n), self._ids), "cp_trace_end")
        self.n = n.value
        return False

    def launches(self):
        """[(kernel name, milliseconds)] for the traced launches (synchronises)."""
        torch.cuda.synchronize()
        out = []
        for i in range(min(self.n, self.cap)):
            name = _lib.KERNEL_NAMES.get(self._ids[i], str(self._ids[i]))
            out.append((name, self.events[2 * i].elapsed_time(self.events[2 * i + 1])))
        return out
