"""CPU oracle for zigzag context-parallel causal attention (fp64, plain C + OpenMP).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use it; the product path never does.  It
shares no code with the CUDA library (``context_zigzag_cp_b200``) and imports
nothing from it.

What it computes, and where each step is defined:
  * the shard plan: 2*cp chunks, rank r owns chunks r and 2*cp-1-r, with
    seq_len % (2*cp) == 0 (NeMo "Hierarchical Context Parallel Skill",
    "Required constraints"; head/tail pairing for equal causal work);
  * visit orders: all-gather (one gather, shards in rank order) and ring
    ("all-to-all": receive the neighbour's shard cp-1 times)
    (Accelerate "Context Parallel" concept guide, "all-to-all vs all-gather");
  * per-(rank, step) partial attention and the combine of the partials
    (concept guide, "So how does it work?", pseudocode), read as the exact
    log-sum-exp merge;
  * unsharded attention and its explicit-P backward (the definition of scaled
    dot-product attention with the causal / packed-document mask), and that
    backward unit by unit in the visit order: rank r's queries against shard j,
    dQ_r summed over the steps and dK_j / dV_j over the ranks.

Inputs are numpy float64 arrays [B, H, S, D] in original token order.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, portable x86-64 flags)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        I32, I64, F64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.orc_doc_start.argtypes = [I32, I32, _i32p, _i32p]
        lib.orc_plan.argtypes = [I32, I32, I32, I32, _i32p, I32, I32, I32, _i32p, _i32p, _i32p,
                                 _i32p, _i32p, _i32p, _i64p]
        lib.orc_fwd_rows.argtypes = [I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p, _i32p,
                                     _i32p, I64, _i64p, _f64p, _f64p]
        lib.orc_fwd.argtypes = [I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p, _i32p, _i32p,
                                _f64p, _f64p]
        lib.orc_partial.argtypes = [I32, I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p,
                                    _i32p, _i32p, _i32p, I32, I32, _f64p, _f64p]
        lib.orc_lse_merge.argtypes = [I64, I32, I32, _f64p, _f64p, _f64p, _f64p]
        lib.orc_lse_merge.restype = None
        lib.orc_bwd.argtypes = [I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p, _f64p,
                                _f64p, _f64p, _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.orc_bwd_dq_rows.argtypes = [I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p,
                                        _f64p, _i32p, _i32p, I64, _i64p, _f64p]
        lib.orc_bwd_dkv_keys.argtypes = [I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p,
                                         _f64p, _i32p, _i32p, I64, _i64p, _f64p, _f64p]
        lib.orc_bwd_dkv_keys_fwd.argtypes = [I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p,
                                             _f64p, _f64p, _f64p, _i32p, _i32p, I64, _i64p, _f64p,
                                             _f64p]
        lib.orc_bwd_partial.argtypes = [I32, I32, I32, I32, I32, I32, F64, _f64p, _f64p, _f64p,
                                        _f64p, _f64p, _f64p, _i32p, _i32p, _i32p, I32, I32,
                                        _f64p, _f64p, _f64p]
        lib.orc_num_threads.argtypes = []
        for name in ("orc_doc_start", "orc_plan", "orc_fwd_rows", "orc_fwd", "orc_partial",
                     "orc_bwd", "orc_bwd_dq_rows", "orc_bwd_dkv_keys", "orc_bwd_dkv_keys_fwd",
                     "orc_bwd_partial", "orc_num_threads"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def num_threads() -> int:
    return int(_load().orc_num_threads())


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


ROTATE = {"allgather": 0, "ring": 1}


def doc_start(seq_len: int, cu_seqlens=None) -> np.ndarray:
    """Per original position, the first position of its document (zeros: one document)."""
    ds = np.zeros(seq_len, dtype=np.int32)
    cu = (np.zeros(1, dtype=np.int32) if cu_seqlens is None
          else np.ascontiguousarray(cu_seqlens, dtype=np.int32))
    nd = 0 if cu_seqlens is None else len(cu) - 1
    _check(_load().orc_doc_start(seq_len, nd, cu, ds), "doc_start")
    return ds


def plan(seq_len: int, cp: int, rotate: str = "allgather", cu_seqlens=None, window: int = 0,
         causal: bool = True, shard: str = "sequence") -> dict:
    """The zigzag plan: perm, inv_perm, src, doc_start (shard order), rank_cu_off,
    rank_cu and pairs (int64), exactly as the library's planner must produce them.
    ``window`` > 0 counts pairs under a sliding window (keys q-W < k <= q);
    ``causal`` False counts every key of the query's document.  ``shard`` "doc"
    cuts every document (not the sequence) into 2cp chunks, rank r taking chunks r
    and 2cp-1-r of each document in turn (document lengths multiples of 2cp)."""
    lib = _load()
    cu = (np.zeros(1, dtype=np.int32) if cu_seqlens is None
          else np.ascontiguousarray(cu_seqlens, dtype=np.int32))
    nd = 0 if cu_seqlens is None else len(cu) - 1
    S = seq_len
    out = dict(perm=np.zeros(S, np.int32), inv_perm=np.zeros(S, np.int32),
               src=np.zeros(cp * cp, np.int32), doc_start=np.zeros(S, np.int32),
               rank_cu_off=np.zeros(cp + 1, np.int32),
               rank_cu=np.zeros(cp * (2 * max(nd, 1) + 3), np.int32), pairs=np.zeros(cp, np.int64))
    _check(lib.orc_plan(S, cp, ROTATE[rotate], nd, cu, int(window), int(bool(causal)),
                        {"sequence": 0, "doc": 1}[shard], out["perm"], out["inv_perm"],
                        out["src"], out["doc_start"], out["rank_cu_off"], out["rank_cu"],
                        out["pairs"]), "plan")
    out["rank_cu"] = out["rank_cu"][: out["rank_cu_off"][cp]].copy()
    return out


def first_key(seq_len: int, cu_seqlens=None, window: int = 0) -> np.ndarray:
    """Per original position q, the first key q attends to: its document's start,
    raised to q - W + 1 under a sliding window of W keys (window 0: none).  Every
    attention function here takes this array as ``ds_orig`` (keys
    first(q) <= k <= q are unmasked)."""
    ds = doc_start(seq_len, cu_seqlens)
    if window and window > 0:
        ds = np.maximum(ds, np.arange(seq_len, dtype=np.int64) - (window - 1)).astype(np.int32)
    return ds


def last_key(seq_len: int, cu_seqlens=None, causal: bool = True) -> np.ndarray:
    """Per original position q, the last key q attends to: q itself under the causal
    mask; without it, the last position of q's document (S - 1 with one document).
    Every attention function here takes this array as ``lk_orig`` (None: causal)."""
    if causal:
        return np.arange(seq_len, dtype=np.int32)
    if cu_seqlens is None:
        return np.full(seq_len, seq_len - 1, dtype=np.int32)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return np.repeat(cu[1:] - 1, np.diff(cu)).astype(np.int32)


def _lk(S, lk_orig):
    return (np.arange(S, dtype=np.int32) if lk_orig is None
            else np.ascontiguousarray(lk_orig, np.int32))


def _dims(q, k):
    B, Hq, S, D = q.shape
    assert k.shape[0] == B and k.shape[2] == S and k.shape[3] == D
    return B, Hq, k.shape[1], S, D


def _scale(D, scale):
    return 1.0 / math.sqrt(D) if not scale else float(scale)


def fwd(q, k, v, ds_orig=None, scale=None, lk_orig=None):
    """Unsharded attention: O [B,Hq,S,D], LSE [B,Hq,S] (natural log), original order."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    o = np.zeros(q.shape, np.float64)
    lse = np.zeros((B, Hq, S), np.float64)
    _check(_load().orc_fwd(B, Hq, Hkv, S, D, _scale(D, scale), q, k, v, ds, _lk(S, lk_orig), o,
                           lse), "fwd")
    return o, lse


def fwd_rows(q, k, v, rows, ds_orig=None, scale=None, lk_orig=None):
    """Unsharded attention at selected flat rows (bh*S + q_orig): O [n,D], LSE [n]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    o = np.zeros((len(rows), D), np.float64)
    lse = np.zeros(len(rows), np.float64)
    _check(_load().orc_fwd_rows(B, Hq, Hkv, S, D, _scale(D, scale), q, k, v, ds, _lk(S, lk_orig),
                                len(rows), rows, o, lse), "fwd_rows")
    return o, lse


def partial(q, k, v, perm, cp, r, j, ds_orig=None, scale=None, lk_orig=None):
    """Partial attention of rank r's queries against rank j's keys:
    O [B*Hq, 2C, D], LSE [B*Hq, 2C] (rank-local shard order)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    n2c = S // cp
    o = np.zeros((B * Hq, n2c, D), np.float64)
    lse = np.zeros((B * Hq, n2c), np.float64)
    _check(_load().orc_partial(B, Hq, Hkv, S, D, cp, _scale(D, scale), q, k, v, ds,
                               _lk(S, lk_orig), np.ascontiguousarray(perm, np.int32), r, j, o, lse),
           "partial")
    return o, lse


def lse_merge(o_parts, lse_parts):
    """combine(): fold partials [P][rows][D] / [P][rows] in order -> O [rows,D], LSE [rows]."""
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    P, R, D = o_parts.shape
    o = np.zeros((R, D), np.float64)
    lse = np.zeros(R, np.float64)
    _load().orc_lse_merge(R, D, P, o_parts, lse_parts, o, lse)
    return o, lse


def cp_fwd(q, k, v, cp, rotate="allgather", cu_seqlens=None, scale=None, steps=None, window=0,
           causal=True, shard="sequence"):
    """The sharded computation: for every rank r, the partials against K/V shard
    src[r][s] for each step s (all steps unless ``steps`` limits them), merged in
    visit order.  Returns O [B,Hq,S,D] and LSE [B,Hq,S] in SHARD order."""
    q = _f64(q)
    B, Hq, S, D = q.shape
    pl = plan(S, cp, rotate, cu_seqlens, window, causal, shard)
    ds = first_key(S, cu_seqlens, window)
    lk = last_key(S, cu_seqlens, causal)
    n2c = S // cp
    o = np.zeros((B * Hq, S, D), np.float64)
    lse = np.zeros((B * Hq, S), np.float64)
    nsteps = cp if steps is None else steps
    for r in range(cp):
        parts_o, parts_l = [], []
        for s in range(nsteps):
            j = int(pl["src"][r * cp + s])
            po, pl_ = partial(q, k, v, pl["perm"], cp, r, j, ds, scale, lk)
            parts_o.append(po.reshape(-1, D))
            parts_l.append(pl_.reshape(-1))
        mo, ml = lse_merge(np.stack(parts_o), np.stack(parts_l))
        o[:, r * n2c:(r + 1) * n2c] = mo.reshape(B * Hq, n2c, D)
        lse[:, r * n2c:(r + 1) * n2c] = ml.reshape(B * Hq, n2c)
    return o.reshape(B, Hq, S, D), lse.reshape(B, Hq, S)


def bwd(q, k, v, o, lse, dout, ds_orig=None, scale=None, lk_orig=None):
    """Explicit-P gradients: dQ [B,Hq,S,D], dK/dV [B,Hkv,S,D], original order."""
    q, k, v, o, lse, dout = map(_f64, (q, k, v, o, lse, dout))
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    dq = np.zeros(q.shape, np.float64)
    dk = np.zeros(k.shape, np.float64)
    dv = np.zeros(k.shape, np.float64)
    _check(_load().orc_bwd(B, Hq, Hkv, S, D, _scale(D, scale), q, k, v, o, lse, dout, ds,
                           _lk(S, lk_orig), dq, dk, dv), "bwd")
    return dq, dk, dv


def bwd_partial(q, k, v, o, lse, dout, perm, cp, r, j, ds_orig=None, scale=None, lk_orig=None):
    """The backward of unit (rank r, shard j) with the final o [B,Hq,S,D] / lse
    [B,Hq,S] (original order): dQ [B,Hq,2C,D] of rank r's rows, dK / dV
    [B,Hkv,2C,D] of shard j's rows (local shard order)."""
    q, k, v, o, lse, dout = map(_f64, (q, k, v, o, lse, dout))
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    n2c = S // cp
    dq = np.zeros((B, Hq, n2c, D), np.float64)
    dk = np.zeros((B, Hkv, n2c, D), np.float64)
    dv = np.zeros((B, Hkv, n2c, D), np.float64)
    _check(_load().orc_bwd_partial(B, Hq, Hkv, S, D, cp, _scale(D, scale), q, k, v, o, lse, dout,
                                   ds, _lk(S, lk_orig), np.ascontiguousarray(perm, np.int32), r, j,
                                   dq, dk, dv), "bwd_partial")
    return dq, dk, dv


def cp_bwd(q, k, v, o, lse, dout, cp, rotate="allgather", cu_seqlens=None, scale=None,
           steps=None, window=0, causal=True, shard="sequence"):
    """The sharded backward, unit by unit in visit order: at step s rank r's
    pieces against shard src[r][s] add into its dQ and into that shard's dK / dV
    (all steps unless ``steps`` limits them).  o / lse: the final forward results
    in original order.  Returns dQ [B,Hq,S,D], dK / dV [B,Hkv,S,D] in SHARD order."""
    q, k = _f64(q), _f64(k)
    B, Hq, Hkv, S, D = _dims(q, k)
    pl = plan(S, cp, rotate, cu_seqlens, window, causal, shard)
    ds = first_key(S, cu_seqlens, window)
    lk = last_key(S, cu_seqlens, causal)
    n2c = S // cp
    dq = np.zeros((B, Hq, S, D), np.float64)
    dk = np.zeros((B, Hkv, S, D), np.float64)
    dv = np.zeros((B, Hkv, S, D), np.float64)
    for s in range(cp if steps is None else steps):
        for r in range(cp):
            j = int(pl["src"][r * cp + s])
            gq, gk, gv = bwd_partial(q, k, v, o, lse, dout, pl["perm"], cp, r, j, ds, scale, lk)
            dq[:, :, r * n2c:(r + 1) * n2c] += gq
            dk[:, :, j * n2c:(j + 1) * n2c] += gk
            dv[:, :, j * n2c:(j + 1) * n2c] += gv
    return dq, dk, dv


def bwd_dq_rows(q, k, v, dout, rows, ds_orig=None, scale=None, lk_orig=None):
    """dQ at selected flat rows (bh*S + q_orig), each from its own forward: [n, D]."""
    q, k, v, dout = map(_f64, (q, k, v, dout))
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    dq = np.zeros((len(rows), D), np.float64)
    _check(_load().orc_bwd_dq_rows(B, Hq, Hkv, S, D, _scale(D, scale), q, k, v, dout, ds,
                                   _lk(S, lk_orig), len(rows), rows, dq), "bwd_dq_rows")
    return dq


def bwd_dkv_keys(q, k, v, dout, keys, ds_orig=None, scale=None, lk_orig=None):
    """dK, dV at selected flat keys (bkv*S + k_orig): [n, D] each."""
    q, k, v, dout = map(_f64, (q, k, v, dout))
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    keys = np.ascontiguousarray(keys, np.int64)
    dk = np.zeros((len(keys), D), np.float64)
    dv = np.zeros((len(keys), D), np.float64)
    _check(_load().orc_bwd_dkv_keys(B, Hq, Hkv, S, D, _scale(D, scale), q, k, v, dout, ds,
                                    _lk(S, lk_orig), len(keys), keys, dk, dv), "bwd_dkv_keys")
    return dk, dv


def bwd_dkv_keys_fwd(q, k, v, o, lse, dout, keys, ds_orig=None, scale=None, lk_orig=None):
    """dK, dV at selected flat keys (bkv*S + k_orig) from the oracle's own forward
    results o [B,Hq,S,D] / lse [B,Hq,S] of every row: [n, D] each.  The same sums
    as ``bwd``, restricted to the selected keys; each row's forward is read once
    instead of being recomputed per key, so early keys (attended by almost every
    row) cost O(S D) each."""
    q, k, v, o, lse, dout = map(_f64, (q, k, v, o, lse, dout))
    B, Hq, Hkv, S, D = _dims(q, k)
    ds = np.zeros(S, np.int32) if ds_orig is None else np.ascontiguousarray(ds_orig, np.int32)
    keys = np.ascontiguousarray(keys, np.int64)
    dk = np.zeros((len(keys), D), np.float64)
    dv = np.zeros((len(keys), D), np.float64)
    _check(_load().orc_bwd_dkv_keys_fwd(B, Hq, Hkv, S, D, _scale(D, scale), q, k, v, o, lse,
                                        dout, ds, _lk(S, lk_orig), len(keys), keys, dk, dv),
           "bwd_dkv_keys_fwd")
    return dk, dv


def causal_pairs(seq_len: int, cu_seqlens=None, window: int = 0, causal: bool = True) -> int:
    """Number of unmasked (q, k) pairs per head: sum over documents of L(L+1)/2
    (with a sliding window: sum over q of q - first_key(q) + 1); without the
    causal mask, sum over documents of L^2."""
    if not causal:
        L = (np.array([seq_len], dtype=np.int64) if cu_seqlens is None
             else np.diff(np.asarray(cu_seqlens, dtype=np.int64)))
        return int((L * L).sum())
    if window and window > 0:
        fk = first_key(seq_len, cu_seqlens, window).astype(np.int64)
        return int((np.arange(seq_len, dtype=np.int64) - fk + 1).sum())
    if cu_seqlens is None:
        return seq_len * (seq_len + 1) // 2
    L = np.diff(np.asarray(cu_seqlens, dtype=np.int64))
    return int((L * (L + 1) // 2).sum())


def flops(num_heads: int, head_dim: int, pairs: int, backward: bool = False) -> float:
    """FLOP convention: 4*D*Hq per unmasked pair forward (two matmuls, 2 FLOP per
    multiply-add), backward twice that, so fwd+bwd = 3x fwd (the attention term of
    the Accelerate example's model-FLOPs helper, ``get_model_flops_per_token``,
    counts 12*Hq*D per token-pair for fwd+bwd)."""
    f = 4.0 * head_dim * num_heads * pairs
    return 3.0 * f if backward else f
