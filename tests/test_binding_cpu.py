"""The Python binding refuses, before any pointer reaches the library, tensors the
kernels would read or write out of bounds: wrong shape or dtype, not contiguous,
not on one CUDA device.  Runs on CPU: correctly shaped CPU tensors pass every
shape and dtype check and stop at the device check."""
import pytest
import torch

import context_zigzag_cp_b200 as cz

B, Hq, Hkv, S, D, CP = 1, 4, 2, 512, 64, 2
bf16, f32 = torch.bfloat16, torch.float32


def prob():
    return cz.Problem(B, S, CP, Hq, Hkv, D)


def tensors():
    q = torch.zeros(B, Hq, S, D, dtype=bf16)
    k = torch.zeros(B, Hkv, S, D, dtype=bf16)
    return dict(q=q, k=k, v=k.clone(), o=q.clone(), lse=torch.zeros(B, Hq, S, dtype=f32),
                do=q.clone(), dq=q.clone(), dk=k.clone(), dv=k.clone())


def fwd(t):
    return cz.attn_fwd(prob(), None, t["q"], t["k"], t["v"], t["o"], t["lse"])


def bwd(t):
    return cz.attn_bwd(prob(), None, t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"],
                       t["dq"], t["dk"], t["dv"])


def test_right_shapes_stop_at_the_device_check():
    for call in (fwd, bwd):
        with pytest.raises(ValueError, match="CUDA device"):
            call(tensors())
    t = tensors()
    with pytest.raises(ValueError, match="CUDA device"):
        cz.attn_fwd(prob(), None, t["q"], t["k"], t["v"])          # outputs allocated later


@pytest.mark.parametrize("name,bad,what", [
    ("q", torch.zeros(B, Hq, S, D + 8, dtype=bf16), "shape"),
    ("k", torch.zeros(B, Hq, S, D, dtype=bf16), "shape"),       # Hq heads where Hkv are expected
    ("v", torch.zeros(B, Hkv, S, D, dtype=f32), "dtype"),
    ("o", torch.zeros(B, Hq, S // 2, D, dtype=bf16), "shape"),
    ("lse", torch.zeros(B, Hq, S, dtype=bf16), "dtype"),
])
def test_forward_rejects(name, bad, what):
    t = tensors()
    t[name] = bad
    with pytest.raises(ValueError, match=what):
        fwd(t)


@pytest.mark.parametrize("name,bad,what", [
    ("do", torch.zeros(B, Hq, S, D, dtype=f32), "dtype"),
    ("lse", torch.zeros(B, Hq, S, 1, dtype=f32), "shape"),
    ("dq", torch.zeros(B, Hkv, S, D, dtype=bf16), "shape"),
    ("dk", torch.zeros(B, Hkv, S, D, dtype=torch.float16), "dtype"),
    ("dv", torch.zeros(2, Hkv, S, D, dtype=bf16), "shape"),
])
def test_backward_rejects(name, bad, what):
    t = tensors()
    t[name] = bad
    with pytest.raises(ValueError, match=what):
        bwd(t)


def test_non_tensor_rejected():
    t = tensors()
    t["k"] = [0.0]
    with pytest.raises(TypeError):
        fwd(t)


def test_noalloc_needs_every_output():
    t = tensors()
    with pytest.raises(ValueError, match="must be given"):
        cz.attn_bwd_noalloc(prob(), None, t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"],
                            None, t["dk"], t["dv"])
    with pytest.raises(ValueError, match="CUDA device"):
        cz.attn_bwd_noalloc(prob(), None, t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"],
                            t["dq"], t["dk"], t["dv"])


def test_merge_rejects():
    n, rows = 3, 100
    po, pl = torch.zeros(n, rows, D, dtype=f32), torch.zeros(n, rows, dtype=f32)
    with pytest.raises(ValueError, match="head_dim"):
        cz.lse_merge(po[0], pl)
    with pytest.raises(ValueError, match="shape"):
        cz.lse_merge(po, pl[:, :50])
    with pytest.raises(ValueError, match="dtype"):
        cz.lse_merge(po, pl, o_out=torch.zeros(rows, D, dtype=f32))
    with pytest.raises(ValueError, match="CUDA device"):
        cz.lse_merge(po, pl)


def test_gather_buffers_checked():
    plan = object.__new__(cz.Plan)            # the buffer checks only, no device plan
    plan.prob = prob()
    plan.perm = torch.zeros(S, dtype=torch.int32)
    x = torch.zeros(2, S, 16, dtype=bf16)
    with pytest.raises(ValueError, match="output buffers"):
        plan._bufs([x], [])
    with pytest.raises(ValueError, match="seq_len"):
        plan._bufs([torch.zeros(2, S + 4, 16, dtype=bf16)], [x])
    with pytest.raises(ValueError, match="shape"):
        plan._bufs([x], [torch.zeros(2, S, 8, dtype=bf16)])
    with pytest.raises(ValueError, match="dtype"):
        plan._bufs([x], [torch.zeros(2, S, 16, dtype=f32)])
    with pytest.raises(ValueError, match="CUDA device"):
        plan._bufs([x], [x.clone()])


class _FakeLib:
    """Stands in for libcpattn so the binding's own steps run on CPU: every entry
    point reports success and writes nothing (workspace queries report 0 bytes)."""

    def __getattr__(self, name):
        return lambda *args: 0


@pytest.fixture
def cpu_binding(monkeypatch):
    """The binding with CPU tensors treated as device tensors and a fake library:
    checks that the argument validation accepts every call pattern the tests, the
    smoke check and the benchmark make."""
    import ctypes
    monkeypatch.setattr(cz, "_on_device", lambda t, dev: t.device == dev)
    monkeypatch.setattr(cz, "lib", lambda: _FakeLib())
    monkeypatch.setattr(cz, "_stream", lambda s: ctypes.c_void_p(0))
    return cz


def _cpu_plan(p):
    plan = object.__new__(cz.Plan)
    plan.prob = p
    plan.perm = torch.zeros(p.seq_len, dtype=torch.int32)
    plan.c = cz.CpPlan(0, 0, 0, 0, 0, 0, 0, 0, 0)
    return plan


@pytest.mark.parametrize("b,hq,hkv,s,d", [(1, 4, 2, 512, 64), (2, 8, 8, 1024, 128)])
def test_call_patterns_pass_validation(cpu_binding, b, hq, hkv, s, d):
    p = cz.Problem(b, s, 2, hq, hkv, d)
    plan = _cpu_plan(p)
    q = torch.zeros(b, hq, s, d, dtype=bf16)
    k, v, do = torch.zeros(b, hkv, s, d, dtype=bf16), torch.zeros(b, hkv, s, d, dtype=bf16), q.clone()
    # plan + gather, forward, backward, restore (tests and smoke check)
    qs, ks, vs = plan.shard([q, k, v])
    o, lse = cz.attn_fwd(p, plan, qs, ks, vs)
    (dos,) = plan.shard([do])
    dq, dk, dv = cz.attn_bwd(p, plan, qs, ks, vs, o, lse, dos)
    plan.unshard([o, dq, dk, dv])
    # the benchmark's step: caller-owned outputs and workspaces, one gather of four
    dos2 = torch.empty_like(do)
    plan.build([q, k, v, do], [qs, ks, vs, dos2])
    ws = torch.empty(256, dtype=torch.uint8)
    cz.attn_fwd(p, plan, qs, ks, vs, o, lse, ws=ws)
    cz.attn_bwd(p, plan, qs, ks, vs, o, lse, dos, dq, dk, dv, ws=ws)
    cz.attn_bwd_noalloc(p, plan, qs, ks, vs, o, lse, dos, dq, dk, dv)
    # gathers of unrelated row tensors through the same plan
    x = torch.zeros(3, s, 12, dtype=torch.int32)
    plan.unshard(plan.shard([q, torch.zeros(2, hkv, s, 64, dtype=bf16), x]))
    cz.lse_merge(torch.zeros(3, 100, d, dtype=f32), torch.zeros(3, 100, dtype=f32))


def test_workspace_taken_when_large_enough():
    ws = torch.empty(512, dtype=torch.uint8)
    assert cz._workspace(0, ws.device, ws) is None                 # nothing needed
    assert cz._workspace(512, ws.device, ws) is ws
    small = cz._workspace(1024, ws.device, ws)                    # too small: a new one
    assert small is not ws and small.numel() == 1024
    with pytest.raises(ValueError, match="ws"):
        cz._workspace(100, torch.device("meta"), ws)              # on another device


def test_problem_checks_cu_seqlens():
    """cu_seqlens reaches the kernels as a raw int32 device pointer: anything else
    (a host tensor, int64, strided, too short) is refused when the Problem is made."""
    with pytest.raises(ValueError, match="int32 CUDA"):
        cz.Problem(B, S, CP, Hq, Hkv, D, cu_seqlens=torch.tensor([0, S], dtype=torch.int32))
    with pytest.raises(ValueError, match="int32 CUDA"):
        cz.Problem(B, S, CP, Hq, Hkv, D, cu_seqlens=torch.tensor([0, S], dtype=torch.int64))
    with pytest.raises(TypeError):
        cz.Problem(B, S, CP, Hq, Hkv, D, cu_seqlens=[0, S])


class _DevTensor:
    """Just enough of a CUDA int32 tensor for Problem's checks (CPU machine)."""

    def __init__(self, n):
        self.t = torch.arange(n, dtype=torch.int32)
        self.dtype, self.device = torch.int32, torch.device("cuda", 0)
        self.shape = self.t.shape

    def dim(self):
        return 1

    def numel(self):
        return self.t.numel()

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return 0


def test_problem_cu_seqlens_shape_checked(monkeypatch):
    monkeypatch.setattr(torch, "Tensor", (torch.Tensor, _DevTensor))
    with pytest.raises(ValueError, match="num_docs"):
        cz.Problem(B, S, CP, Hq, Hkv, D, cu_seqlens=_DevTensor(1))


def test_plan_must_fit_problem(cpu_binding):
    """A plan built for another seq_len, cp, order or document list is refused
    before the kernels index its arrays with the problem's sizes."""
    t = tensors()
    args = (t["q"], t["k"], t["v"], t["o"], t["lse"])
    p = prob()
    for other in (cz.Problem(B, 2 * S, CP, Hq, Hkv, D), cz.Problem(B, S, 2 * CP, Hq, Hkv, D),
                  cz.Problem(B, S, CP, Hq, Hkv, D, rotate="ring")):
        with pytest.raises(ValueError, match="plan: built for"):
            cz.attn_fwd(p, _cpu_plan(other), *args)
        with pytest.raises(ValueError, match="plan: built for"):
            cz.attn_bwd(p, _cpu_plan(other), *args, t["do"], t["dq"], t["dk"], t["dv"])
        with pytest.raises(ValueError, match="plan: built for"):
            cz.attn_bwd_noalloc(p, _cpu_plan(other), *args, t["do"], t["dq"], t["dk"], t["dv"])
    with pytest.raises(TypeError, match="Plan"):
        cz.attn_fwd(p, None, *args)
    # documents: a plan made without them does not serve a problem that has them
    docs = object.__new__(cz.Problem)
    docs.__dict__.update(p.__dict__)
    docs.cu_seqlens = torch.tensor([0, 100, S], dtype=torch.int32)
    with pytest.raises(ValueError, match="other documents"):
        cz.attn_fwd(docs, _cpu_plan(p), *args)
    # and a plan on another device
    plan = _cpu_plan(p)
    plan.perm = torch.zeros(S, dtype=torch.int32, device="meta")
    with pytest.raises(ValueError, match="plan: on"):
        cz.attn_fwd(p, plan, *args)


def test_problem_shard_option(cpu_binding):
    """shard: "sequence" (default) or "doc"; per-document sharding needs documents, and
    a plan made for one sharding does not serve the other."""
    with pytest.raises(ValueError, match="shard"):
        cz.Problem(B, S, CP, Hq, Hkv, D, shard="tile")
    with pytest.raises(ValueError, match="needs cu_seqlens"):
        cz.Problem(B, S, CP, Hq, Hkv, D, shard="doc")
    p = cz.Problem(B, S, CP, Hq, Hkv, D)
    assert p.c.shard == 0 and p.rank_cu_len() == 3 * CP + 1
    assert p.with_merge("separate").shard == "sequence"
    doc = object.__new__(cz.Problem)
    doc.__dict__.update(p.__dict__)
    doc.shard, doc.num_docs = "doc", 5
    assert doc.rank_cu_len() == CP * 11
    t = tensors()
    args = (t["q"], t["k"], t["v"], t["o"], t["lse"])
    with pytest.raises(ValueError, match="'sequence' sharding"):
        cz.attn_fwd(doc, _cpu_plan(p), *args)
    windowed = cz.Problem(B, S, CP, Hq, Hkv, D, window=64)
    with pytest.raises(ValueError, match="window"):
        cz.attn_fwd(windowed, _cpu_plan(p), *args)


def _rank_tensors():
    n2c = S // CP
    q = torch.zeros(B, Hq, n2c, D, dtype=bf16)
    k = torch.zeros(B, Hkv, n2c, D, dtype=bf16)
    return dict(q=q, k=k, v=k.clone(), o=q.clone(), lse=torch.zeros(B, Hq, n2c, dtype=f32),
                do=q.clone(), dq_sum=torch.zeros(q.shape, dtype=f32),
                dk_sum=torch.zeros(k.shape, dtype=f32), dv_sum=torch.zeros(k.shape, dtype=f32))


def _bwd_step(t):
    return cz.attn_bwd_step(prob(), None, 0, 0, t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"],
                            t["dq_sum"], t["dk_sum"], t["dv_sum"])


@pytest.mark.parametrize("name,bad,what", [
    ("dq_sum", lambda t: t["dq_sum"].to(bf16), "dtype"),            # the sums are fp32
    ("dk_sum", lambda t: torch.zeros(B, Hkv, S, D, dtype=f32), "shape"),   # one shard, not all S
    ("k", lambda t: torch.zeros(B, Hkv, S, D, dtype=bf16), "shape"),       # the one shard held
    ("lse", lambda t: t["lse"].to(bf16), "dtype"),
    ("o", lambda t: torch.zeros(B, Hq, S, D, dtype=bf16), "shape")])
def test_bwd_step_rejects(name, bad, what):
    """cp_attn_bwd_step: rank-local q/o/do/lse, one K/V shard, fp32 sums of the same shapes."""
    t = _rank_tensors()
    t[name] = bad(t)
    with pytest.raises(ValueError, match=what):
        _bwd_step(t)


def test_bwd_step_needs_every_sum():
    t = _rank_tensors()
    t["dv_sum"] = None
    with pytest.raises(ValueError, match="dv_sum"):
        _bwd_step(t)
    with pytest.raises(ValueError, match="CUDA device"):   # right shapes: stops at the device check
        _bwd_step(_rank_tensors())
