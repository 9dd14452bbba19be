"""CPU oracle for the DBSA attention engine -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The product path (the C-ABI library
and its Python binding in ``many_shot_icl_b200``) never does; it shares no
code with it.

This module is argument marshalling (numpy <-> ctypes) around
``dbsa_oracle.c``, which holds all of the arithmetic in plain fp64 C.  The
page it follows is "Efficient Many-Shot In-Context Learning with Dynamic
Block-Sparse Attention" (ACL 2025 paper notes): §Stage 1 items 1-4 and
§Stage 2 items 1-4; see the C file for the per-function citations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dbsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# A prebuilt variant of the oracle may be substituted (the mutation test of
# tests/test_oracle_mutants.py uses this to check that the pins catch
# planted mistakes).
_LIB_OVERRIDE = os.environ.get("DBSA_ORACLE_LIB")

PATTERN_SINK_PREV_SELF = 0
PATTERN_FULL = 1
PATTERN_SINK_SELF = 2
PATTERN_SELF = 3


def build(force: bool = False) -> str:
    """Compile dbsa_oracle.c with gcc into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_LIB_OVERRIDE or build())
        i32, i64, f64, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.orc_group_blocks.argtypes = [vp, i32, i32, vp]
        lib.orc_group_blocks.restype = i32
        lib.orc_stage1_allowed.argtypes = [vp, i32, i32, i32, i64, i64]
        lib.orc_stage1_allowed.restype = i32
        lib.orc_rope.argtypes = [vp, i32, f64, f64, vp]
        lib.orc_rope.restype = None
        lib.orc_stage1_rows.argtypes = [i32, i32, i32, f64, f64, i32, i32, vp, vp, vp, i64,
                                        vp, i32, vp, vp, i64, vp, i32]
        lib.orc_stage1_rows.restype = i32
        lib.orc_stage2_gather_map.argtypes = [vp, i32, vp, i32, vp]
        lib.orc_stage2_gather_map.restype = i64
        lib.orc_stage2_rows.argtypes = [i32, i32, i32, f64, f64, vp, vp, i64, vp, i32, vp, i32,
                                        vp, i32, vp, vp, i32, vp, vp, i32, vp, i32]
        lib.orc_stage2_rows.restype = i32
        lib.orc_stage1_allowed_counts.argtypes = [vp, i32, i32, i32, i64, vp]
        lib.orc_stage1_allowed_counts.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def group_blocks(demo_len, k: int) -> np.ndarray:
    """Block offset table offs[0..nb] from demonstration lengths (k demos per block)."""
    dl = _c(demo_len, np.int32)
    nb = (len(dl) + k - 1) // k
    offs = np.zeros(nb + 1, dtype=np.int32)
    r = _load().orc_group_blocks(_ptr(dl), len(dl), k, _ptr(offs))
    if r < 0:
        raise ValueError("invalid demo lengths / k")
    return offs


def stage1_allowed(offs, j: int, t: int, s: int, pattern: int = PATTERN_SINK_PREV_SELF) -> bool:
    o = _c(offs, np.int32)
    return bool(_load().orc_stage1_allowed(_ptr(o), len(o) - 1, j, pattern, t, s))


def stage1_allowed_counts(offs, j: int, pattern: int = PATTERN_SINK_PREV_SELF) -> np.ndarray:
    o = _c(offs, np.int32)
    T = int(o[-1])
    cnt = np.zeros(T, dtype=np.int64)
    _load().orc_stage1_allowed_counts(_ptr(o), len(o) - 1, j, pattern, T, _ptr(cnt))
    return cnt


def rope(x, pos: float, theta: float) -> np.ndarray:
    xx = _c(x, np.float64)
    y = np.empty_like(xx)
    _load().orc_rope(_ptr(xx), xx.shape[-1], float(pos), float(theta), _ptr(y))
    return y


def stage1_rows(q, k, v, offs, j: int, theta: float, rows_head, rows_tok, *,
                scale: float = 0.0, pattern: int = PATTERN_SINK_PREV_SELF,
                threads: int | None = None) -> np.ndarray:
    """Stage-1 output rows (fp64) for the requested (head, token) pairs.

    q: [T, Hq, d], k/v: [T, Hkv, d] (float32 holding the exact input values).
    Returns [nrows, d]."""
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    o = _c(offs, np.int32)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    rh = _c(rows_head, np.int32)
    rt = _c(rows_tok, np.int64)
    out = np.zeros((len(rh), d), dtype=np.float64)
    r = _load().orc_stage1_rows(Hq, Hkv, d, float(theta), float(scale), j, pattern,
                                _ptr(q), _ptr(k), _ptr(v), T, _ptr(o), len(o) - 1,
                                _ptr(rh), _ptr(rt), len(rh), _ptr(out),
                                threads or default_threads())
    if r != 0:
        raise ValueError("orc_stage1_rows: invalid arguments")
    return out


def stage1_all(q, k, v, offs, j: int, theta: float, **kw) -> np.ndarray:
    """Every Stage-1 output row, as [T, Hq, d]."""
    T, Hq, d = q.shape
    hh, tt = np.meshgrid(np.arange(Hq), np.arange(T))
    out = stage1_rows(q, k, v, offs, j, theta, hh.ravel(), tt.ravel(), **kw)
    return out.reshape(T, Hq, d)


def stage2_gather_map(offs, sel) -> np.ndarray:
    """[T', 2] int32 map (cache row, fresh position) of one query's gathered tokens."""
    o = _c(offs, np.int32)
    s = _c(sel, np.int32)
    lib = _load()
    n = lib.orc_stage2_gather_map(_ptr(o), len(o) - 1, _ptr(s), len(s), None)
    if n < 0:
        raise ValueError("invalid selection")
    m = np.zeros((max(n, 1), 2), dtype=np.int32)
    lib.orc_stage2_gather_map(_ptr(o), len(o) - 1, _ptr(s), len(s), _ptr(m))
    return m[:n]


def stage2_rows(kc, vc, offs, sel, q_new, k_tail, v_tail, theta: float, rows_head, rows_u, *,
                scale: float = 0.0, threads: int | None = None) -> np.ndarray:
    """Stage-2 output rows (fp64) of ONE query for the requested (head, u) pairs.

    kc/vc: [Hkv, cap, d]; q_new: [n_new, Hq, d]; k_tail/v_tail: [tail_len, Hkv, d].
    Returns [nrows, d]."""
    kc = _c(kc, np.float32)
    vc = _c(vc, np.float32)
    o = _c(offs, np.int32)
    s = _c(sel, np.int32)
    qn = _c(q_new, np.float32)
    kt = _c(k_tail, np.float32)
    vt = _c(v_tail, np.float32)
    Hkv, cap, d = kc.shape
    n_new, Hq, _ = qn.shape
    rh = _c(rows_head, np.int32)
    ru = _c(rows_u, np.int32)
    out = np.zeros((len(rh), d), dtype=np.float64)
    r = _load().orc_stage2_rows(Hq, Hkv, d, float(theta), float(scale), _ptr(kc), _ptr(vc), cap,
                                _ptr(o), len(o) - 1, _ptr(s), len(s), _ptr(qn), n_new,
                                _ptr(kt), _ptr(vt), kt.shape[0], _ptr(rh), _ptr(ru), len(rh),
                                _ptr(out), threads or default_threads())
    if r != 0:
        raise ValueError("orc_stage2_rows: invalid arguments")
    return out


def stage2_all(kc, vc, offs, sel, q_new, k_tail, v_tail, theta: float, **kw) -> np.ndarray:
    """Every Stage-2 output row of one query, as [n_new, Hq, d]."""
    n_new, Hq, d = np.shape(q_new)
    hh, uu = np.meshgrid(np.arange(Hq), np.arange(n_new))
    out = stage2_rows(kc, vc, offs, sel, q_new, k_tail, v_tail, theta, hh.ravel(), uu.ravel(), **kw)
    return out.reshape(n_new, Hq, d)
