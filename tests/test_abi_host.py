"""Host-side tests of libmfattn: exported symbols, the pack planner and argument
checks. No GPU is touched: every call here returns before any CUDA work."""
import ctypes
import os
import re

import numpy as np
import pytest

import packed_attention_b200 as pa
from packed_attention_b200 import _native
from packed_attention_b200.build import build
from packed_attention_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _native.lib()


def header_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(mf_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert "mf_pack_plan" in names and "mf_joint_attn_fwd" in names
    for n in names:
        assert hasattr(lib, n), n
    # and the binding covers exactly the declared API
    assert sorted(_native.SIGNATURES) == names


# The boundary's calls, by name: the operation's own (plan, schedule, workspace
# query, the two stages and the joint forward), its 3D-rotation, training and
# sub-layer variants, the allocation-free variant, and the diagnostics.
DOCUMENTED_ABI = sorted([
    "mf_abi_version", "mf_status_string",
    "mf_pack_plan", "mf_schedule_work", "mf_joint_attn_workspace_bytes",
    "mf_qk_prologue", "mf_packed_attention", "mf_joint_attn_fwd",
    "mf_qk_prologue_3d", "mf_joint_attn_fwd_3d",
    "mf_joint_attn_fwd_lse", "mf_bwd_workspace_bytes", "mf_joint_attn_bwd",
    "mf_block_workspace_bytes", "mf_attn_block_fwd",
    "mf_joint_attn_fwd_static_scratch",
    "mf_selftest_exp2", "mf_selftest_timeout", "mf_get_device_error",
])


def test_header_declares_the_documented_calls():
    assert header_functions() == DOCUMENTED_ABI


def test_checked_build_exports_the_same_calls():
    """libmfattn_checked.so (-DMF_CHECKED) exports every declared call and
    knows the status its range checks report."""
    build(checked=True)
    with _native.checked_build() as checked:
        for n in header_functions():
            assert hasattr(checked, n), n
        assert checked.mf_status_string(-8).decode() == "MF_ERR_BOUNDS"
        assert _native.lib() is checked
    assert _native.lib() is not checked


def test_status_strings(lib):
    assert lib.mf_abi_version() == 4
    for code, name in _native.STATUS.items():
        assert lib.mf_status_string(code).decode() == name


def test_struct_sizes_match_header():
    assert ctypes.sizeof(_native.Segment) == 24
    assert ctypes.sizeof(_native.WorkItem) == 16


@pytest.mark.parametrize("cfg,cu", [
    (0, [0, 80, 152]),
    (1, [0, 1152, 2304, 3456, 4608]),
    (2, [0, 1101, 4373, 8725, 9789, 12989, 14688]),
    (3, [0, 8704]),
    (4, [0, 16896, 21248]),
])
def test_plan_offsets_by_hand(lib, cfg, cu):
    w = WORKLOADS[cfg]
    p = pa.pack_plan(w.samples, w.heads, w.head_dim, w.token_budget)
    assert p["cu_seqlens"].tolist() == cu
    assert p["total_tokens"] == cu[-1]  # no padding, no rounding to tiles
    segs = p["segs"]
    for i, (nt, gh, gw, fr) in enumerate(w.samples):
        assert segs[i].tolist() == [cu[i], cu[i + 1] - cu[i], nt, gh, gw, fr]


@pytest.mark.parametrize("cfg,n_work", [(0, 4), (1, 480), (2, 1440), (3, 816), (4, 1992)])
def test_plan_work_list(lib, cfg, n_work):
    w = WORKLOADS[cfg]
    p = pa.pack_plan(w.samples, w.heads, w.head_dim, w.token_budget)
    work = p["work"]
    assert work.shape == (n_work, 4)
    lens = p["segs"][:, 1]
    # every (segment, head, q_tile) exactly once
    want = {(s, h, t) for s in range(len(lens)) for h in range(w.heads)
            for t in range((lens[s] + pa.MF_TILE_M - 1) // pa.MF_TILE_M)}
    got = {tuple(x) for x in work[:, :3].tolist()}
    assert got == want and len(got) == n_work
    # kv_len is the segment length; ordered by cost = length x query sub-tiles
    # (a last tile of at most 128 rows has one), largest first; ties by
    # sample index, then head, then q_tile
    assert np.array_equal(work[:, 3], lens[work[:, 0]])
    def cost(s, t, L):
        rows = min(pa.MF_TILE_M, L - t * pa.MF_TILE_M)
        return L * (2 if rows > pa.MF_TILE_M // 2 else 1)
    keys = [(-cost(s, t, L), int(s), int(h), int(t)) for s, h, t, L in work.tolist()]
    assert keys == sorted(keys)


def test_plan_budget_and_validation(lib):
    w = WORKLOADS[2]
    assert pa.pack_plan(w.samples, 24, 128, 15400)["total_tokens"] == 14688
    with pytest.raises(pa.MfError) as e:
        pa.pack_plan(w.samples, 24, 128, 14687)
    assert e.value.status == -5
    for bad in ([(1, 0, 4, 1)], [(-1, 2, 2, 1)], [(0, 2, 2, 0)]):
        with pytest.raises(pa.MfError) as e:
            pa.pack_plan(bad, 2, 64)
        assert e.value.status == -1
    with pytest.raises(pa.MfError) as e:
        pa.pack_plan([(1, 2, 2, 1)], 2, 96)
    assert e.value.status == -2
    with pytest.raises(pa.MfError):  # total beyond int32
        pa.pack_plan([(0, 46341, 46341, 1)], 1, 64)
    with pytest.raises(pa.MfError):
        pa.pack_plan([(0, 1, 1, 1)], 0, 64)


def test_plan_two_call_capacity(lib):
    n_text = (ctypes.c_int32 * 1)(5)
    gh = (ctypes.c_int32 * 1)(3)
    gw = (ctypes.c_int32 * 1)(100)
    n_work = ctypes.c_int32(0)
    assert lib.mf_pack_plan(1, n_text, gh, gw, None, 2, 64, 0, None, None, None,
                            ctypes.byref(n_work), None) == 0
    assert n_work.value == 2 * 2  # 305 tokens -> two 256-row items per head
    small = (ctypes.c_int32 * 8)()
    n_work.value = 1  # capacity too small
    assert lib.mf_pack_plan(1, n_text, gh, gw, None, 2, 64, 0, None, None, small,
                            ctypes.byref(n_work), None) == -1
    assert lib.mf_pack_plan(1, n_text, gh, gw, None, 2, 64, 0, None, None, small, None, None) == -1


def test_workspace_size(lib):
    assert pa.workspace_bytes(152, 2, 64) == 2 * ((152 * 2 * 64 * 2 + 255) // 256 * 256)
    assert pa.workspace_bytes(0, 2, 64) == 0
    assert pa.workspace_bytes(10, 2, 96) == 0


def _fwd(lib, **over):
    """mf_joint_attn_fwd with fake (never dereferenced) pointers."""
    a = dict(q=0x10000, k=0x20000, v=0x30000, gqt=0x40000, gqi=0x40100, gkt=0x40200,
             gki=0x40300, cu=0x50000, segs=0x60000, n=2, work=0x70000, n_work=4, T=152, H=2,
             d=64, eps=1e-6, scale=0.0, out=0x80000, ws=0x100000, ws_bytes=1 << 20)
    a.update(over)
    P = ctypes.c_void_p
    return lib.mf_joint_attn_fwd(P(a["q"]), P(a["k"]), P(a["v"]), P(a["gqt"]), P(a["gqi"]),
                                 P(a["gkt"]), P(a["gki"]), P(a["cu"]), P(a["segs"]), a["n"],
                                 P(a["work"]), a["n_work"], a["T"], a["H"], a["d"], a["eps"],
                                 a["scale"], P(a["out"]), P(a["ws"]), a["ws_bytes"], None)


def test_forward_argument_checks(lib):
    assert _fwd(lib, d=96) == -2
    assert _fwd(lib, q=0x10008) == -3
    assert _fwd(lib, v=0x30004) == -3
    assert _fwd(lib, out=0x80002) == -3
    assert _fwd(lib, ws=0x100010) == -3
    assert _fwd(lib, ws_bytes=100) == -4
    assert _fwd(lib, q=0) == -1
    assert _fwd(lib, work=0) == -1
    assert _fwd(lib, n_work=0) == -1
    assert _fwd(lib, T=0) == -1
    assert _fwd(lib, eps=-1.0) == -1
    assert _fwd(lib, eps=float("nan")) == -1
    assert _fwd(lib, scale=float("inf")) == -1
    assert _fwd(lib, out=0x10000) == -1        # out aliases q
    assert _fwd(lib, ws=0x10000 - 0x100) == -1  # workspace overlaps q


def test_frame_dims_checked_before_any_launch(lib):
    """mf_joint_attn_fwd_3d / mf_qk_prologue_3d refuse a split of head_dim that
    does not give every axis whole pairs; everything else as in the 2D call."""
    P = ctypes.c_void_p
    base = (P(0x10000), P(0x20000), P(0x30000), P(0x40000), P(0x40100), P(0x40200), P(0x40300),
            P(0x50000), P(0x60000), 2, P(0x70000), 4, 152, 2, 64, 1e-6)
    tail = (0.0, P(0x80000), P(0x100000), 1 << 20, None)
    for F in (-4, 2, 6, 62, 64, 1000):
        assert lib.mf_joint_attn_fwd_3d(*base, F, *tail) == -1, F
    pro = (P(0x10000), P(0x20000), P(0x40000), P(0x40100), P(0x40200), P(0x40300), P(0x50000),
           P(0x60000), 2, 152, 2, 128, 1e-6)
    for F in (-4, 2, 126, 128):
        assert lib.mf_qk_prologue_3d(*pro, F, P(0x100000), 1 << 20, None) == -1, F
    # the shared checks still come first: unsupported head_dim, misaligned input
    assert lib.mf_joint_attn_fwd_3d(*base[:14], 96, 1e-6, 2, *tail) == -2
    assert lib.mf_joint_attn_fwd_3d(P(0x10008), *base[1:], 16, *tail) == -3


def _bwd(lib, **over):
    """mf_joint_attn_bwd with fake (never dereferenced) pointers."""
    # Spaced so that nothing overlaps: every test below changes one argument
    # into an invalid one, and the call must return before any CUDA work.
    a = dict(q=0x10000, k=0x20000, v=0x30000, gqt=0x40000, gqi=0x40100, gkt=0x40200,
             gki=0x40300, out=0x50000, dout=0x60000, lse=0x70000, cu=0x71000, segs=0x72000,
             n=2, work=0x73000, n_work=4, T=152, H=2, d=64, eps=1e-6, F=0, scale=0.0,
             dq=0x80000, dk=0x90000, dv=0xa0000, dg=0xb0000, ws=0x200000, ws_bytes=1 << 22)
    a.update(over)
    P = ctypes.c_void_p
    return lib.mf_joint_attn_bwd(
        P(a["q"]), P(a["k"]), P(a["v"]), P(a["gqt"]), P(a["gqi"]), P(a["gkt"]), P(a["gki"]),
        P(a["out"]), P(a["dout"]), P(a["lse"]), P(a["cu"]), P(a["segs"]), a["n"], P(a["work"]),
        a["n_work"], a["T"], a["H"], a["d"], a["eps"], a["F"], a["scale"], P(a["dq"]),
        P(a["dk"]), P(a["dv"]), P(a["dg"]), P(a["ws"]), a["ws_bytes"], None)


def test_backward_argument_checks(lib):
    T, H, d = 152, 2, 64
    need = lib.mf_bwd_workspace_bytes(T, H, d)
    rows = T * H
    r256 = lambda x: (x + 255) // 256 * 256
    fwd = lib.mf_joint_attn_workspace_bytes(T, H, d)
    blocks = (T + 31) // 32  # 256 threads, 8 per token at d = 64
    assert need == r256(fwd) + r256(rows * 4) + 2 * r256(rows * d * 4) + r256(blocks * 4 * d * 4)
    assert lib.mf_bwd_workspace_bytes(T, H, 96) == 0
    assert _bwd(lib, d=96) == -2
    assert _bwd(lib, F=6) == -1
    assert _bwd(lib, eps=-1.0) == -1
    assert _bwd(lib, dout=0) == -1
    assert _bwd(lib, q=0x10008) == -3
    assert _bwd(lib, dout=0x60004) == -3
    assert _bwd(lib, lse=0x70002) == -3
    assert _bwd(lib, dq=0x80008) == -3
    assert _bwd(lib, ws=0x200010) == -3
    assert _bwd(lib, ws_bytes=need - 1) == -4
    assert _bwd(lib, dq=0x10000) == -1          # dq aliases q
    assert _bwd(lib, dv=0x90000) == -1          # dv aliases dk
    assert _bwd(lib, dg=0x200100) == -1         # dgamma inside the workspace


def test_diagnostic_entry_points_reject_bad_arguments(lib):
    assert lib.mf_selftest_timeout(0, None) == -1
    assert lib.mf_selftest_timeout(2_000_000_000, None) == -1
    assert lib.mf_selftest_exp2(None, None, 4, None) == -1
    assert lib.mf_selftest_exp2(ctypes.c_void_p(16), ctypes.c_void_p(32), -1, None) == -1


# ------------------------------------------------------- mf_schedule_work ---

def _lpt_by_hand(work, ctas):
    """Longest processing time first, written out: cost = key steps x (20 with
    two query sub-tiles, 19 with one), stable in the input order; each item to
    the least-loaded CTA, lowest index on ties."""
    def cost(item):
        s, h, t, L = item
        rows = min(pa.MF_TILE_M, L - t * pa.MF_TILE_M)
        return -(-L // pa.MF_TILE_N) * (20 if rows > pa.MF_TILE_M // 2 else 19)
    order = sorted(range(len(work)), key=lambda i: -cost(work[i]))
    load = [0] * ctas
    lists = [[] for _ in range(ctas)]
    for i in order:
        c = min(range(ctas), key=lambda k: (load[k], k))
        lists[c].append(tuple(work[i]))
        load[c] += cost(work[i])
    return lists, load


@pytest.mark.parametrize("cfg", [0, 1, 2, 4])
@pytest.mark.parametrize("ctas", [1, 3, 148])
def test_schedule_is_lpt_laid_out_for_the_stride(lib, cfg, ctas):
    w = WORKLOADS[cfg]
    work = pa.pack_plan(w.samples, w.heads, w.head_dim, w.token_budget)["work"]
    sched = _native.schedule_work(work, ctas)
    g = min(ctas, len(work))
    assert len(sched) % g == 0
    # every item exactly once; the rest is padding {0, 0, -1, 0}
    real = sched[sched[:, 2] >= 0]
    assert sorted(map(tuple, real.tolist())) == sorted(map(tuple, work.tolist()))
    pad = sched[sched[:, 2] < 0]
    assert (pad == np.array([0, 0, -1, 0])).all()
    # CTA c's items sit at c, c + g, ...: its LPT list, then padding only
    lists, load = _lpt_by_hand(work.tolist(), g)
    for c in range(g):
        col = [tuple(x) for x in sched[c::g].tolist()]
        n = len(lists[c])
        assert col[:n] == lists[c]
        assert all(x[2] < 0 for x in col[n:])
    # never worse than the plain round-robin of the cost-ordered list
    rr = [0] * g
    def cost(item):
        s, h, t, L = item
        rows = min(pa.MF_TILE_M, L - t * pa.MF_TILE_M)
        return -(-L // pa.MF_TILE_N) * (20 if rows > pa.MF_TILE_M // 2 else 19)
    for i, item in enumerate(work.tolist()):
        rr[i % g] += cost(item)
    assert max(load) <= max(rr)


def test_schedule_arguments(lib):
    work = pa.pack_plan([(3, 4, 5)], 2, 128)["work"]
    wp = work.ctypes.data_as(ctypes.c_void_p)
    n = ctypes.c_int32(0)
    assert lib.mf_schedule_work(None, len(work), 4, None, ctypes.byref(n)) == -1
    assert lib.mf_schedule_work(wp, 0, 4, None, ctypes.byref(n)) == -1
    assert lib.mf_schedule_work(wp, len(work), 0, None, ctypes.byref(n)) == -1
    assert lib.mf_schedule_work(wp, len(work), 4, None, None) == -1
    assert lib.mf_schedule_work(wp, len(work), 4, None, ctypes.byref(n)) == 0
    assert n.value == 2  # 2 items, CTAs capped at 2: one round
    out = np.zeros((1, 4), dtype=np.int32)
    small = ctypes.c_int32(1)
    assert lib.mf_schedule_work(wp, len(work), 4, out.ctypes.data_as(ctypes.c_void_p),
                                ctypes.byref(small)) == -1
    bad = work.copy()
    bad[1, 2] = -1  # a padding entry is not an input item
    assert lib.mf_schedule_work(bad.ctypes.data_as(ctypes.c_void_p), len(bad), 4, None,
                                ctypes.byref(n)) == -1
