"""ctypes binding of libmfattn.so (argument marshalling only).

Every computation happens in the library's CUDA kernels; this module only
passes pointers, sizes and the current CUDA stream. If the library is missing
the calls raise: there is no fallback path.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmfattn.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libmfattn_checked.so")

MF_TILE_M = 256
MF_TILE_N = 128

STATUS = {
    0: "MF_OK", -1: "MF_ERR_INVALID_ARG", -2: "MF_ERR_UNSUPPORTED", -3: "MF_ERR_ALIGNMENT",
    -4: "MF_ERR_WORKSPACE", -5: "MF_ERR_BUDGET", -6: "MF_ERR_CUDA", -7: "MF_ERR_TIMEOUT",
    -8: "MF_ERR_BOUNDS",
}


class MfError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        super().__init__(f"{func} failed: {STATUS.get(status, status)}")


class Segment(ctypes.Structure):
    _fields_ = [("start", ctypes.c_int32), ("len", ctypes.c_int32), ("n_text", ctypes.c_int32),
                ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32), ("frames", ctypes.c_int32)]


class WorkItem(ctypes.Structure):
    _fields_ = [("seg", ctypes.c_int32), ("head", ctypes.c_int32), ("q_tile", ctypes.c_int32),
                ("kv_len", ctypes.c_int32)]


_lock = threading.Lock()
_libs = {}
_use_checked = False

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
F32 = ctypes.c_float
SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/mf_attn.h
SIGNATURES = {
    "mf_abi_version": (I32, []),
    "mf_status_string": (ctypes.c_char_p, [I32]),
    "mf_pack_plan": (I32, [I32, P, P, P, P, I32, I32, I64, P, P, P, P, P]),
    "mf_schedule_work": (I32, [P, I32, I32, P, P]),
    "mf_joint_attn_workspace_bytes": (SZ, [I32, I32, I32]),
    "mf_qk_prologue": (I32, [P, P, P, P, P, P, P, P, I32, I32, I32, I32, F32, P, SZ, P]),
    "mf_qk_prologue_3d": (I32, [P, P, P, P, P, P, P, P, I32, I32, I32, I32, F32, I32, P, SZ, P]),
    "mf_packed_attention": (I32, [P, P, I32, P, I32, I32, I32, I32, F32, P, P, SZ, P]),
    "mf_joint_attn_fwd": (I32, [P, P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, F32, F32, P,
                                P, SZ, P]),
    "mf_joint_attn_fwd_3d": (I32, [P, P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, F32, I32,
                                   F32, P, P, SZ, P]),
    "mf_joint_attn_fwd_lse": (I32, [P, P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, F32,
                                    I32, F32, P, P, P, SZ, P]),
    "mf_bwd_workspace_bytes": (SZ, [I32, I32, I32]),
    "mf_joint_attn_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, F32,
                                I32, F32, P, P, P, P, P, SZ, P]),
    "mf_block_workspace_bytes": (SZ, [I32, I32, I32]),
    "mf_attn_block_fwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32,
                                F32, F32, I32, F32, P, P, SZ, P]),
    "mf_joint_attn_fwd_static_scratch": (I32, [P, P, P, P, P, P, P, P, P, I32, P, I32, I32, I32,
                                               I32, F32, F32, P, P]),
    "mf_selftest_exp2": (I32, [P, P, I32, P]),
    "mf_selftest_timeout": (I32, [I64, P]),
    "mf_get_device_error": (I32, [P]),
}

MF_STATIC_SCRATCH_BYTES = 64 * 1024 * 1024


def _load(path):
    with _lock:
        if path not in _libs:
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with "
                                   "`python -m packed_attention_b200.build`")
            handle = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(handle, name)
                f.restype = res
                f.argtypes = args
            _libs[path] = handle
    return _libs[path]


def lib():
    """The loaded library (the checked build inside ``checked_build()``);
    raises if it has not been built."""
    return _load(CHECKED_LIB_PATH if _use_checked else LIB_PATH)


@contextlib.contextmanager
def checked_build():
    """Route every call of the package through libmfattn_checked.so, the
    build whose kernels range-check each global index they compute and
    report a bad one as MF_ERR_BOUNDS (not thread-safe: for tests)."""
    global _use_checked
    prev = _use_checked
    _use_checked = True
    try:
        yield _load(CHECKED_LIB_PATH)
    finally:
        _use_checked = prev


def check(func: str, status: int):
    if status != 0:
        raise MfError(func, status)


def pack_plan(samples, heads: int, head_dim: int, token_budget: int = 0):
    """Host plan: returns dict(cu_seqlens, segs, work, total_tokens) as numpy arrays.

    ``samples`` is a sequence of (n_text, grid_h, grid_w[, frames]).
    """
    s = [tuple(x) + (1,) * (4 - len(x)) for x in samples]
    arr = np.asarray(s, dtype=np.int32).reshape(-1, 4)
    n = len(arr)
    cols = [np.ascontiguousarray(arr[:, i]) for i in range(4)]
    ptrs = [c.ctypes.data_as(P) for c in cols]
    n_work = ctypes.c_int32(0)
    total = ctypes.c_int32(0)
    L = lib()
    check("mf_pack_plan", L.mf_pack_plan(n, *ptrs, heads, head_dim, token_budget, None, None, None,
                                         ctypes.byref(n_work), ctypes.byref(total)))
    cu = np.zeros(n + 1, dtype=np.int32)
    segs = np.zeros((n, 6), dtype=np.int32)
    work = np.zeros((n_work.value, 4), dtype=np.int32)
    check("mf_pack_plan", L.mf_pack_plan(n, *ptrs, heads, head_dim, token_budget,
                                         cu.ctypes.data_as(P), segs.ctypes.data_as(P),
                                         work.ctypes.data_as(P), ctypes.byref(n_work),
                                         ctypes.byref(total)))
    return {"cu_seqlens": cu, "segs": segs, "work": work, "total_tokens": int(total.value),
            "n_samples": n, "heads": heads, "head_dim": head_dim}


def schedule_work(work, n_ctas: int):
    """``work`` ([n, 4] int32, from pack_plan) laid out for ``n_ctas`` CTAs by
    ``mf_schedule_work``: [rounds * n_ctas, 4], padding rows have q_tile -1."""
    work = np.ascontiguousarray(work, dtype=np.int32).reshape(-1, 4)
    n_sched = ctypes.c_int32(0)
    L = lib()
    check("mf_schedule_work", L.mf_schedule_work(work.ctypes.data_as(P), len(work), n_ctas, None,
                                                 ctypes.byref(n_sched)))
    sched = np.zeros((n_sched.value, 4), dtype=np.int32)
    check("mf_schedule_work", L.mf_schedule_work(work.ctypes.data_as(P), len(work), n_ctas,
                                                 sched.ctypes.data_as(P), ctypes.byref(n_sched)))
    return sched[:n_sched.value]


def workspace_bytes(total_tokens: int, heads: int, head_dim: int) -> int:
    return int(lib().mf_joint_attn_workspace_bytes(total_tokens, heads, head_dim))
