"""fp64 CPU oracle for the packed joint text+image attention forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use this package; the product path
(``packed_attention_b200``) never imports it. The arithmetic lives in
``oracle.cpp`` (plain C++, fp64); this module only builds it with g++ and
marshals numpy arrays through ctypes.

Parity status: every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (closed forms, invariants and a dense
brute-force formulation), for the gradients of :func:`attn_grad`,
``tests/test_oracle_grad_pins.py`` (central finite differences, closed forms
and invariants), and for the sub-layer around the path (``oracle.block``),
``tests/test_oracle_block_pins.py``; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.cpp`` into ``liboracle.so`` (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_total_tokens.restype = i64
            lib.oracle_total_tokens.argtypes = [i32, P, P, P, P]
            lib.oracle_qk_prologue.restype = i32
            lib.oracle_qk_prologue.argtypes = [P, i64, i32, i32, P, P, i32, P, P, P, P, dbl, i32,
                                               P]
            lib.oracle_joint_attn.restype = i32
            lib.oracle_joint_attn.argtypes = [P, P, P, P, P, P, P, i32, P, P, P, P, i32, i32, dbl,
                                              i32, dbl, i64, P, P, i32]
            lib.oracle_attn_grad.restype = i32
            lib.oracle_attn_grad.argtypes = [P, P, P, P, P, P, P, P, i32, P, P, P, P, i32, i32, dbl,
                                             i32, dbl, P, P, P, P, P, P, i32]
            lib.oracle_dense_attn.restype = i32
            lib.oracle_dense_attn.argtypes = [P, P, P, P, P, P, P, i32, P, P, P, P, i32, i32, dbl,
                                              i32, dbl, P]
            _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _samples(samples):
    s = np.asarray(samples, dtype=np.int32).reshape(-1, 4)
    return (len(s), np.ascontiguousarray(s[:, 0]), np.ascontiguousarray(s[:, 1]),
            np.ascontiguousarray(s[:, 2]), np.ascontiguousarray(s[:, 3]))


def _u16(x):
    return np.ascontiguousarray(x, dtype=np.uint16)


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def total_tokens(samples) -> int:
    n, nt, gh, gw, fr = _samples(samples)
    return int(_load().oracle_total_tokens(n, _ptr(nt), _ptr(gh), _ptr(gw), _ptr(fr)))


def qk_prologue(x_bits, samples, g_text, g_img, eps=1e-6, frame_dims=0):
    """Normalised, rotated q or k as fp64 ``[T, H, d]`` from bf16 bits ``[T, H, d]``.

    ``frame_dims`` > 0 selects the 3D rotation (frame, row, column)."""
    x = _u16(x_bits)
    T, H, d = x.shape
    n, nt, gh, gw, fr = _samples(samples)
    out = np.empty((T, H, d), dtype=np.float64)
    gt, gi = _f32(g_text), _f32(g_img)
    rc = _load().oracle_qk_prologue(_ptr(x), T, H, d, _ptr(gt), _ptr(gi), n, _ptr(nt), _ptr(gh),
                                    _ptr(gw), _ptr(fr), float(eps), int(frame_dims), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_qk_prologue rejected its arguments")
    return out


def _attn_args(q, k, v, gammas, samples):
    q, k, v = _u16(q), _u16(k), _u16(v)
    if q.shape != k.shape or q.shape != v.shape or q.ndim != 3:
        raise ValueError("q, k, v must share one [T, H, d] shape")
    g = [_f32(gammas[name]) for name in ("g_q_text", "g_q_img", "g_k_text", "g_k_img")]
    return q, k, v, g, _samples(samples)


def joint_attn(q, k, v, gammas, samples, eps=1e-6, scale=None, rows=None, n_threads=0,
               frame_dims=0):
    """Attention output, fp64.

    ``rows`` (optional, int64) selects flat rows ``token * H + head``; the
    result is then ``[len(rows), d]``, otherwise ``[T, H, d]``.
    """
    q, k, v, g, (n, nt, gh, gw, fr) = _attn_args(q, k, v, gammas, samples)
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is None:
        out = np.empty((T, H, d), dtype=np.float64)
        n_rows, rp = T * H, None
    else:
        rp = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty((len(rp), d), dtype=np.float64)
        n_rows = len(rp)
    rc = _load().oracle_joint_attn(_ptr(q), _ptr(k), _ptr(v), *[_ptr(x) for x in g], n, _ptr(nt),
                                   _ptr(gh), _ptr(gw), _ptr(fr), H, d, float(eps),
                                   int(frame_dims), float(scale), n_rows, _ptr(rp), _ptr(out),
                                   int(n_threads))
    if rc != 0:
        raise ValueError("oracle_joint_attn rejected its arguments")
    return out


def dense_attn(q, k, v, gammas, samples, eps=1e-6, scale=None, frame_dims=0):
    """Brute-force dense formulation (small packs only), fp64 ``[T, H, d]``."""
    q, k, v, g, (n, nt, gh, gw, fr) = _attn_args(q, k, v, gammas, samples)
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((T, H, d), dtype=np.float64)
    rc = _load().oracle_dense_attn(_ptr(q), _ptr(k), _ptr(v), *[_ptr(x) for x in g], n, _ptr(nt),
                                   _ptr(gh), _ptr(gw), _ptr(fr), H, d, float(eps),
                                   int(frame_dims), float(scale), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dense_attn rejected its arguments")
    return out


def attn_grad(q, k, v, gammas, samples, dout=None, eps=1e-6, scale=None, frame_dims=0,
              n_threads=0):
    """Forward output, the per-row log-normaliser ``lse`` (``[T, H]``, natural
    log of sum_u exp(s_tu)) and, given ``dout`` = dL/dout, the gradients, all fp64.

    q, k, v, dout: float64 ``[T, H, d]`` values (not bf16 bits); gammas: dict of
    the four ``[d]`` vectors. Returns a dict with ``out`` and, with ``dout``,
    ``dq``, ``dk``, ``dv`` (``[T, H, d]``) and ``dgamma`` (a dict keyed like
    the gammas).
    """
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    if q.shape != k.shape or q.shape != v.shape or q.ndim != 3:
        raise ValueError("q, k, v must share one [T, H, d] shape")
    T, H, d = q.shape
    names = ("g_q_text", "g_q_img", "g_k_text", "g_k_img")
    g = [np.ascontiguousarray(gammas[nm], dtype=np.float64) for nm in names]
    n, nt, gh, gw, fr = _samples(samples)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((T, H, d), dtype=np.float64)
    lse = np.empty((T, H), dtype=np.float64)
    res = {"out": out, "lse": lse}
    go = dq = dk = dv = dg = None
    if dout is not None:
        go = np.ascontiguousarray(dout, dtype=np.float64)
        if go.shape != q.shape:
            raise ValueError("dout must have the shape of q")
        dq, dk, dv = (np.empty((T, H, d), dtype=np.float64) for _ in range(3))
        dg = np.empty((4, d), dtype=np.float64)
    rc = _load().oracle_attn_grad(_ptr(q), _ptr(k), _ptr(v), *[_ptr(x) for x in g], _ptr(go), n,
                                  _ptr(nt), _ptr(gh), _ptr(gw), _ptr(fr), H, d, float(eps),
                                  int(frame_dims), float(scale), _ptr(out), _ptr(lse), _ptr(dq),
                                  _ptr(dk),
                                  _ptr(dv), _ptr(dg), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_attn_grad rejected its arguments")
    if dout is not None:
        res.update(dq=dq, dk=dk, dv=dv, dgamma={nm: dg[i] for i, nm in enumerate(names)})
    return res
