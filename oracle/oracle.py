"""ctypes wrapper of the C oracle (``jl_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library and never imports it.

Arrays are numpy arrays.  bf16 tensors are passed as their raw ``uint16`` bit
patterns (``tensor.view(torch.int16).numpy().view(np.uint16)``) and are upcast
to fp64 inside the oracle, which is exact.  All results are fp64.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

F64, BF16, F32 = 0, 1, 2


class View(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("stride_pos", ctypes.c_int64),
        ("stride_head", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
        _lib.jlo_group_size.restype = i64
        _lib.jlo_group_size.argtypes = [i64, i64]
        _lib.jlo_remote_pos.restype = i64
        _lib.jlo_remote_pos.argtypes = [i64, i64]
        _lib.jlo_inv_freq.restype = None
        _lib.jlo_inv_freq.argtypes = [i32, dbl, vp]
        _lib.jlo_rope_cos_sin.restype = None
        _lib.jlo_rope_cos_sin.argtypes = [i64, i32, dbl, vp, vp]
        _lib.jlo_rotate_rows.restype = None
        _lib.jlo_rotate_rows.argtypes = [vp, vp, i64, i32, dbl, vp]
        _lib.jlo_rotate.restype = None
        _lib.jlo_rotate.argtypes = [vp, i32, i64, dbl, vp]
        rows_args = [View, View, View, i64, i32, i32, i32, vp, vp, i64, i64, i64, dbl, dbl]
        _lib.jlo_bifocal_rows.restype = ctypes.c_int
        _lib.jlo_bifocal_rows.argtypes = rows_args + [ctypes.c_int, vp, vp]
        _lib.jlo_bifocal_rows_three_pass.restype = ctypes.c_int
        _lib.jlo_bifocal_rows_three_pass.argtypes = rows_args + [vp, vp, vp]
        _lib.jlo_interp_rows.restype = ctypes.c_int
        _lib.jlo_interp_rows.argtypes = [View, View, View, i64, i32, i32, i32, vp, vp, i64, i64, dbl, vp, dbl, vp, vp]
        _lib.jlo_decode_step.restype = ctypes.c_int
        _lib.jlo_decode_step.argtypes = [View, View, View, i64, i32, i32, i32, i64, i64, dbl, dbl,
                                         ctypes.c_int, vp, vp]
        _lib.jlo_num_threads.restype = ctypes.c_int
        _lib.jlo_num_threads.argtypes = []
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def view(a: np.ndarray) -> tuple[View, np.ndarray]:
    """View of a contiguous [positions][heads][d] array (fp64, fp32 or uint16 bf16 bits)."""
    a = np.ascontiguousarray(a)
    if a.ndim == 2:
        a = a[:, None, :]
    assert a.ndim == 3
    dt = {np.dtype(np.float64): F64, np.dtype(np.float32): F32, np.dtype(np.uint16): BF16}[a.dtype]
    v = View(_ptr(a), a.shape[1] * a.shape[2], a.shape[2], dt, 0)
    return v, a  # keep the array alive with the view


def group_size(L: int, w_pretrained: int) -> int:
    return int(lib().jlo_group_size(L, w_pretrained))


def remote_pos(x: int, G: int) -> int:
    return int(lib().jlo_remote_pos(x, G))


def inv_freq(d: int, base: float) -> np.ndarray:
    t = np.zeros(d // 2, np.float64)
    lib().jlo_inv_freq(d, base, _ptr(t))
    return t


def rope_cos_sin(n_pos: int, d: int, base: float) -> tuple[np.ndarray, np.ndarray]:
    c = np.zeros((n_pos, d // 2), np.float64)
    s = np.zeros((n_pos, d // 2), np.float64)
    lib().jlo_rope_cos_sin(n_pos, d, base, _ptr(c), _ptr(s))
    return c, s


def rotate(x: np.ndarray, pos: int, base: float) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    y = np.zeros_like(x)
    lib().jlo_rotate(_ptr(x), x.shape[-1], pos, base, _ptr(y))
    return y


def rotate_rows(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """R(pos[r]) x[r] for x [n][d] (any float dtype, upcast to fp64)."""
    x = np.ascontiguousarray(x, np.float64)
    n, d = x.shape
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, np.int64), (n,)))
    y = np.empty_like(x)
    lib().jlo_rotate_rows(_ptr(x), _ptr(p), n, d, base, _ptr(y))
    return y


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def bifocal_rows(q, k, v, L, row_pos, row_head, *, w0, w_pretrained, rope_base, scale=None,
                 plain=False, three_pass=False):
    """Direct-definition rows (or the three-pass merge) for one sequence.

    q: [L][Hq][d], k, v: [L][Hkv][d] (raw, un-rotated), any of fp64/fp32/uint16-bf16.
    Returns (out [n][d], lse [n]) in fp64, plus pass_lse [n][3] when three_pass.
    """
    qv, qa = view(q)
    kv, ka = view(k)
    vv, va = view(v)
    d = qa.shape[2]
    hq, hkv = qa.shape[1], ka.shape[1]
    rp = np.ascontiguousarray(row_pos, np.int64)
    rh = np.ascontiguousarray(row_head, np.int32)
    n = rp.shape[0]
    out = np.zeros((n, d), np.float64)
    lse = np.zeros(n, np.float64)
    sc = default_scale(d) if scale is None else scale
    if three_pass:
        pl = np.zeros((n, 3), np.float64)
        rc = lib().jlo_bifocal_rows_three_pass(qv, kv, vv, L, d, hq, hkv, _ptr(rp), _ptr(rh), n, w0,
                                               w_pretrained, rope_base, sc, _ptr(out), _ptr(lse), _ptr(pl))
        if rc != 0:
            raise ValueError(f"oracle three-pass rejected arguments ({rc})")
        return out, lse, pl
    rc = lib().jlo_bifocal_rows(qv, kv, vv, L, d, hq, hkv, _ptr(rp), _ptr(rh), n, w0, w_pretrained,
                                rope_base, sc, int(plain), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments ({rc})")
    return out, lse


def interp_rows(q, k, v, L, row_pos, row_head, *, w0, rope_base, freq_scale, scale=None):
    """Frequency-interpolation variant: local pairs base RoPE, remote pairs rotated by
    p * theta_c * freq_scale[c].  Returns (out [n][d], lse [n]) in fp64."""
    qv, qa = view(q)
    kv, ka = view(k)
    vv, va = view(v)
    d = qa.shape[2]
    hq, hkv = qa.shape[1], ka.shape[1]
    rp = np.ascontiguousarray(row_pos, np.int64)
    rh = np.ascontiguousarray(row_head, np.int32)
    lam = np.ascontiguousarray(freq_scale, np.float64)
    assert lam.shape == (d // 2,)
    n = rp.shape[0]
    out = np.zeros((n, d), np.float64)
    lse = np.zeros(n, np.float64)
    sc = default_scale(d) if scale is None else scale
    rc = lib().jlo_interp_rows(qv, kv, vv, L, d, hq, hkv, _ptr(rp), _ptr(rh), n, w0, rope_base, _ptr(lam), sc,
                               _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments ({rc})")
    return out, lse


def decode_step(q_tilde, k_cache, v_cache, L, *, w0, w_pretrained, rope_base, scale=None, plain=False):
    """One decode step on a base-RoPE cache.

    q_tilde: [Hq][d] (already rotated by R(L-1)); k_cache, v_cache: [>=L][Hkv][d].
    Returns (out [Hq][d], lse [Hq]) in fp64.
    """
    q3 = np.ascontiguousarray(q_tilde)[None]
    qv, qa = view(q3)
    kv, ka = view(k_cache)
    vv, va = view(v_cache)
    d = qa.shape[2]
    hq, hkv = qa.shape[1], ka.shape[1]
    out = np.zeros((hq, d), np.float64)
    lse = np.zeros(hq, np.float64)
    sc = default_scale(d) if scale is None else scale
    rc = lib().jlo_decode_step(qv, kv, vv, L, d, hq, hkv, w0, w_pretrained, rope_base, sc, int(plain),
                               _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments ({rc})")
    return out, lse


def num_threads() -> int:
    return int(lib().jlo_num_threads())
