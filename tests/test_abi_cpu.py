"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import context_zigzag_cp_b200 as cz
from context_zigzag_cp_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cp_attn.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from context_zigzag_cp_b200 import build
        build.build()
    return cz.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"CP_API\s+\w+\s+(cp_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("cp_plan_shards", "cp_attn_fwd", "cp_attn_bwd", "cp_lse_merge"):
        assert name in fns
    assert sorted(_lib.EXPORTED) == fns


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert cz.version() >= 100


def prob(**kw):
    base = dict(batch=1, seq_len=512, cp=2, num_heads=2, num_kv_heads=2, head_dim=64)
    base.update(kw)
    return cz.Problem(**base)


def fwd_query(p):
    n = ctypes.c_size_t(0)
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    st = cz.lib().cp_attn_fwd(p.ref, ctypes.byref(plan), d, d, d, d, d, None, ctypes.byref(n),
                              None)
    return st, n.value


@pytest.mark.parametrize("kw,status", [
    (dict(seq_len=510), _lib.CP_ERR_INVALID_ARG),          # 510 % 4 != 0
    (dict(cp=0), _lib.CP_ERR_INVALID_ARG),
    (dict(num_heads=3, num_kv_heads=2), _lib.CP_ERR_INVALID_ARG),
    (dict(head_dim=96), _lib.CP_ERR_UNSUPPORTED),
    (dict(seq_len=384, cp=3), _lib.CP_ERR_UNSUPPORTED),   # C = 64, not a multiple of 128
    (dict(seq_len=2050, cp=1025), _lib.CP_ERR_UNSUPPORTED),  # more virtual ranks than the planner holds
    (dict(batch=1024, num_heads=1024, num_kv_heads=1024, seq_len=4096),
     _lib.CP_ERR_UNSUPPORTED),                            # 2^32 rows: beyond int32 row indices
    (dict(), _lib.CP_OK),
])
def test_fwd_host_checks(lib, kw, status):
    st, _ = fwd_query(prob(**kw))
    assert st == status


def test_bad_enums_and_scale(lib):
    p = prob()
    p.c.rotate = 7
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.mask = 1                     # doc mask without cu_seqlens
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.softmax_scale = float("nan")
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.merge = 5
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.window = -1                  # a sliding window is 0 (none) or positive
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.window = 37
    assert fwd_query(p)[0] == _lib.CP_OK


def test_workspace_query(lib):
    st, n = fwd_query(prob(merge="fused"))
    assert st == 0 and n == 0
    st, n = fwd_query(prob(merge="separate"))
    # cp partial O (fp32) + partial LSE (fp32), each rounded up to 256 B
    rows = 1 * 2 * 512
    assert st == 0 and n == 2 * rows * 64 * 4 + 2 * rows * 4
    # backward: per-row dot(dO, O) and LSE*log2(e), fp32 each; the one-pass form adds an
    # fp32 dQ accumulator of head_dim values per row
    assert cz.bwd_workspace_bytes(prob()) == 2 * rows * 4
    assert cz.bwd_workspace_bytes(prob(bwd_one_pass=True)) == 2 * rows * 4 + rows * 64 * 4


def test_workspace_too_small_and_null_pointers(lib):
    p = prob(merge="separate")
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    n = ctypes.c_size_t(16)
    assert cz.lib().cp_attn_fwd(p.ref, ctypes.byref(plan), d, d, d, d, d, d, ctypes.byref(n),
                                None) == _lib.CP_ERR_WORKSPACE
    assert cz.lib().cp_attn_fwd(p.ref, ctypes.byref(plan), None, d, d, d, d, None,
                                ctypes.byref(n), None) == _lib.CP_ERR_INVALID_ARG
    assert cz.lib().cp_attn_fwd(None, ctypes.byref(plan), d, d, d, d, d, None, ctypes.byref(n),
                                None) == _lib.CP_ERR_INVALID_ARG
    bad_plan = _lib.CpPlan(256, 256, None, 256, 256, 256, 256, 256, 256)
    assert cz.lib().cp_attn_fwd(p.ref, ctypes.byref(bad_plan), d, d, d, d, d, None,
                                ctypes.byref(n), None) == _lib.CP_ERR_INVALID_ARG


def test_plan_host_checks(lib):
    p = prob(seq_len=102)       # 102 % 4 != 0
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    assert cz.lib().cp_plan_shards(p.ref, ctypes.byref(plan), 0, None, None, None, None, None,
                                   None, None) == _lib.CP_ERR_INVALID_ARG
    p = prob()
    assert cz.lib().cp_plan_shards(p.ref, ctypes.byref(plan), 17, None, None, None, None, None,
                                   None, None) == _lib.CP_ERR_INVALID_ARG
    # row bytes not a multiple of 16
    n = 1
    ptrs = (ctypes.c_void_p * 1)(256)
    outs = (ctypes.c_void_p * 1)(1 << 20)
    outer = (ctypes.c_int64 * 1)(2)
    row = (ctypes.c_int64 * 1)(24)
    assert cz.lib().cp_plan_shards(p.ref, ctypes.byref(plan), n, ptrs, outs, outer, row, None,
                                   None, None) == _lib.CP_ERR_INVALID_ARG
    # overlapping in/out
    row = (ctypes.c_int64 * 1)(128)
    outs = (ctypes.c_void_p * 1)(256 + 1024)
    assert cz.lib().cp_plan_shards(p.ref, ctypes.byref(plan), n, ptrs, outs, outer, row, None,
                                   None, None) == _lib.CP_ERR_INVALID_ARG


def test_merge_host_checks(lib):
    d = ctypes.c_void_p(256)
    L = cz.lib()
    assert L.cp_lse_merge(10, 6, 2, d, d, d, d, None) == _lib.CP_ERR_INVALID_ARG    # D % 4
    assert L.cp_lse_merge(10, 512, 2, d, d, d, d, None) == _lib.CP_ERR_INVALID_ARG  # D > 256
    assert L.cp_lse_merge(10, 64, 0, d, d, d, d, None) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_lse_merge(10, 64, 65, d, d, d, d, None) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_lse_merge(-1, 64, 2, d, d, d, d, None) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_lse_merge(0, 64, 2, None, None, None, None, None) == _lib.CP_OK     # empty
    assert L.cp_lse_merge(10, 64, 2, None, d, d, d, None) == _lib.CP_ERR_INVALID_ARG


def test_misc_host_checks(lib):
    L = cz.lib()
    assert L.cp_get_device_status(None, None) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_set_wait_limit_ns(0) == _lib.CP_ERR_INVALID_ARG
    assert L.cp_selftest_wait_timeout(0, None) == _lib.CP_ERR_INVALID_ARG


def test_product_has_no_cpu_fallback():
    """The package never imports the oracle and raises when the library is absent."""
    pkg = os.path.join(ROOT, "context_zigzag_cp_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            text = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in text and "from oracle" not in text, fn


def test_noalloc_limit_checked_on_host(lib):
    """Beyond the fixed scratch array the no-alloc backward refuses before any CUDA call."""
    p = prob(seq_len=4096, cp=2, num_heads=_lib.NOALLOC_MAX_ROWS // 4096 + 1, num_kv_heads=1,
             head_dim=128)
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    assert cz.lib().cp_attn_bwd_noalloc(p.ref, ctypes.byref(plan), d, d, d, d, d, d, d, d, d,
                                        None) == _lib.CP_ERR_WORKSPACE
    assert cz.lib().cp_attn_bwd_noalloc(p.ref, ctypes.byref(plan), None, d, d, d, d, d, d, d, d,
                                        None) == _lib.CP_ERR_INVALID_ARG


def test_full_mask_host_checks(lib):
    """CP_MASK_FULL (no causal mask) takes no documents and no window."""
    p = prob(causal=False)
    assert p.c.mask == 2 and fwd_query(p)[0] == _lib.CP_OK
    p.c.window = 5
    assert fwd_query(p)[0] == _lib.CP_ERR_UNSUPPORTED
    p = prob(causal=False)
    p.c.num_docs = 2
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob(causal=False)
    p.c.cu_seqlens = 256
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.mask = 3                     # no such mask
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    with pytest.raises(ValueError, match="causal=False"):
        prob(causal=False, window=4)


def test_shard_host_checks(lib):
    """cp_problem_t.shard: CP_SHARD_SEQUENCE or CP_SHARD_PER_DOC, the latter only with
    the document mask; a per-document plan must carry its tile tables."""
    p = prob()
    p.c.shard = 2                    # no such sharding
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.shard = 1                    # per-document sharding without documents
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob(causal=False)
    p.c.shard = 1
    assert fwd_query(p)[0] == _lib.CP_ERR_INVALID_ARG
    p = prob()
    p.c.mask, p.c.num_docs, p.c.cu_seqlens, p.c.shard = 1, 2, 256, 1
    assert fwd_query(p)[0] == _lib.CP_OK
    d = ctypes.c_void_p(256)
    n = ctypes.c_size_t(0)
    no_tables = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, None, None)
    assert cz.lib().cp_attn_fwd(p.ref, ctypes.byref(no_tables), d, d, d, d, d, None,
                                ctypes.byref(n), None) == _lib.CP_ERR_INVALID_ARG
    assert cz.lib().cp_plan_shards(p.ref, ctypes.byref(no_tables), 0, None, None, None, None,
                                   None, None, None) == _lib.CP_ERR_INVALID_ARG
    no_inv = _lib.CpPlan(256, None, 256, 256, 256, 256, 256, 256, 256)
    ptrs = (ctypes.c_void_p * 1)(256)
    outs = (ctypes.c_void_p * 1)(1 << 20)
    outer = (ctypes.c_int64 * 1)(1)
    row = (ctypes.c_int64 * 1)(128)
    assert cz.lib().cp_unshard(p.ref, ctypes.byref(no_inv), 1, ptrs, outs, outer, row,
                               None) == _lib.CP_ERR_INVALID_ARG


def test_head_dim_256(lib):
    """head_dim 256 has its own forward and three-pass backward; no one-pass form."""
    st, n = fwd_query(prob(head_dim=256, merge="separate"))
    rows = 1 * 2 * 512
    assert st == _lib.CP_OK and n == 2 * rows * 256 * 4 + 2 * rows * 4
    assert cz.bwd_workspace_bytes(prob(head_dim=256)) == 2 * rows * 4
    with pytest.raises(cz.CPError, match="UNSUPPORTED"):
        cz.bwd_workspace_bytes(prob(head_dim=256, bwd_one_pass=True))
    assert fwd_query(prob(head_dim=192))[0] == _lib.CP_ERR_UNSUPPORTED



def _rank_calls(p, rank, step, ws_bytes):
    """The three per-rank entry points that take a workspace, with dummy aligned
    device pointers and ws = NULL (a workspace query when the arguments pass, so
    nothing launches): their statuses; the byte counts go to ws_bytes."""
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    pl = ctypes.byref(plan)
    L = cz.lib()
    n = [ctypes.c_size_t(0) for _ in range(3)]
    st = [L.cp_attn_fwd_rank(p.ref, pl, rank, d, d, d, d, d, None, ctypes.byref(n[0]), None),
          L.cp_attn_bwd_rank(p.ref, pl, rank, d, d, d, d, d, d, d, d, d, None, ctypes.byref(n[1]), None),
          L.cp_attn_bwd_step(p.ref, pl, rank, step, d, d, d, d, d, d, d, d, d, None, ctypes.byref(n[2]),
                             None)]
    ws_bytes.extend(x.value for x in n)
    return st


def test_rank_calls_host_checks(lib):
    """Rank and step must lie in [0, cp) (refused on the host, before any launch);
    the workspace query of a good call reports the per-row scratch: the step
    backward needs two fp32 values per local query row, like the per-rank one."""
    p = prob()
    sizes = []
    assert _rank_calls(p, 0, 1, sizes) == [_lib.CP_OK] * 3
    rows = 1 * 2 * (512 // 2)                           # batch x heads x 2C local rows
    assert sizes[1] == sizes[2] and sizes[2] >= 2 * rows * 4
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    for rank, step in ((2, 0), (-1, 0), (0, 2), (0, -1)):
        st = _rank_calls(p, rank, step, [])
        assert st[2] == _lib.CP_ERR_INVALID_ARG, (rank, step, st)
        assert cz.lib().cp_attn_fwd_step(p.ref, ctypes.byref(plan), rank, step, d, d, d, d, d,
                                         None) == _lib.CP_ERR_INVALID_ARG, (rank, step)
        if rank not in (0, 1):
            assert st[0] == _lib.CP_ERR_INVALID_ARG and st[1] == _lib.CP_ERR_INVALID_ARG


def test_bwd_step_null_pointers(lib):
    p = prob()
    d = ctypes.c_void_p(256)
    plan = _lib.CpPlan(256, 256, 256, 256, 256, 256, 256, 256, 256)
    n = ctypes.c_size_t(0)
    for i in range(9):                                  # q k v o lse dout dq_sum dk_sum dv_sum
        args = [d] * 9
        args[i] = None
        st = cz.lib().cp_attn_bwd_step(p.ref, ctypes.byref(plan), 0, 0, *args, None,
                                       ctypes.byref(n), None)
        assert st == _lib.CP_ERR_INVALID_ARG, i
