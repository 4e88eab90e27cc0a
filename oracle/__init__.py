"""CPU oracle for blocked attention with softmax thresholding (fp64, plain C).

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module. The CUDA library never
calls it and shares no code with it.

The arithmetic lives in ``blasst_oracle.c`` (see its header for the passages
of the pages it follows). This file only compiles it with gcc and marshals
numpy arrays through ctypes.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against brute-force dense softmax attention, closed-form bounds and exact
invariants of the method; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "blasst_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MASK_COMPUTED, MASK_SKIPPED, MASK_NOT_VISITED = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC,
             "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class _PrefillArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p),
        ("dtype", C.c_int),
        ("B", C.c_int64), ("Hq", C.c_int64), ("Hkv", C.c_int64),
        ("Lq", C.c_int64), ("Lkv", C.c_int64), ("d", C.c_int64),
        ("causal", C.c_int), ("lam", C.c_double),
        ("Br", C.c_int64), ("Bc", C.c_int64), ("scale", C.c_double),
        ("ref_mode", C.c_int), ("ref_param", C.c_double),
        ("items", C.c_void_p), ("n_items", C.c_int64), ("static_mask", C.c_void_p),
        ("o", C.c_void_p), ("lse", C.c_void_p), ("mask", C.c_void_p),
        ("margin", C.c_void_p), ("nthreads", C.c_int),
    ]


class _DecodeArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p),
        ("dtype", C.c_int),
        ("B", C.c_int64), ("Hq", C.c_int64), ("Hkv", C.c_int64),
        ("Lkv", C.c_int64), ("d", C.c_int64), ("lam", C.c_double),
        ("Bc", C.c_int64), ("num_splits", C.c_int64), ("scale", C.c_double),
        ("o_parts", C.c_void_p), ("lse_parts", C.c_void_p),
        ("mask", C.c_void_p), ("margin", C.c_void_p),
        ("o", C.c_void_p), ("lse", C.c_void_p), ("nthreads", C.c_int),
    ]


class _BackwardArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("dout", C.c_void_p),
        ("dtype", C.c_int),
        ("B", C.c_int64), ("Hq", C.c_int64), ("Hkv", C.c_int64),
        ("Lq", C.c_int64), ("Lkv", C.c_int64), ("d", C.c_int64),
        ("causal", C.c_int), ("Br", C.c_int64), ("Bc", C.c_int64), ("scale", C.c_double),
        ("tile_mask", C.c_void_p),
        ("dq", C.c_void_p), ("dk", C.c_void_p), ("dv", C.c_void_p), ("nthreads", C.c_int),
    ]


class _BackwardRowsArgs(C.Structure):
    _fields_ = [
        ("base", _BackwardArgs),
        ("n_rows", C.c_int64), ("rows", C.c_void_p), ("dq_rows", C.c_void_p),
        ("kv_b", C.c_int64), ("kv_h", C.c_int64), ("key_lo", C.c_int64), ("key_hi", C.c_int64),
        ("dk_part", C.c_void_p), ("dv_part", C.c_void_p), ("nthreads", C.c_int),
    ]


class _SelectArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p), ("dtype", C.c_int),
        ("B", C.c_int64), ("Hq", C.c_int64), ("Hkv", C.c_int64),
        ("Lq", C.c_int64), ("Lkv", C.c_int64), ("d", C.c_int64),
        ("causal", C.c_int), ("Br", C.c_int64), ("Bc", C.c_int64),
        ("scale", C.c_double), ("tau", C.c_double), ("gamma", C.c_double),
        ("mask_out", C.c_void_p), ("cstruct_out", C.c_void_p), ("amap_out", C.c_void_p),
        ("nthreads", C.c_int),
    ]


class Oracle:
    """Handle on one compiled copy of the oracle (``path`` defaults to the
    library built from ``blasst_oracle.c``; the tests also load copies with a
    deliberately planted mistake to show that the pins catch it)."""

    def __init__(self, path: str | None = None):
        lib = C.CDLL(path or build())
        lib.oracle_prefill.argtypes = [C.POINTER(_PrefillArgs)]
        lib.oracle_prefill.restype = C.c_int
        lib.oracle_decode.argtypes = [C.POINTER(_DecodeArgs)]
        lib.oracle_decode.restype = C.c_int
        lib.oracle_lse_merge.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64,
                                         C.c_int64, C.c_void_p, C.c_void_p]
        lib.oracle_lse_merge.restype = None
        lib.oracle_split_len.argtypes = [C.c_int64, C.c_int64, C.c_int64]
        lib.oracle_split_len.restype = C.c_int64
        lib.oracle_select.argtypes = [C.POINTER(_SelectArgs)]
        lib.oracle_select.restype = C.c_int
        lib.oracle_backward_rows.argtypes = [C.POINTER(_BackwardRowsArgs)]
        lib.oracle_backward_rows.restype = C.c_int
        lib.oracle_backward.argtypes = [C.POINTER(_BackwardArgs)]
        lib.oracle_backward.restype = C.c_int
        self.lib = lib

    def prefill(self, *a, **kw):
        return prefill(*a, _lib=self.lib, **kw)

    def decode(self, *a, **kw):
        return decode(*a, _lib=self.lib, **kw)

    def lse_merge(self, *a, **kw):
        return lse_merge(*a, _lib=self.lib, **kw)

    def split_len(self, *a, **kw):
        return split_len(*a, _lib=self.lib, **kw)

    def backward(self, *a, **kw):
        return backward(*a, _lib=self.lib, **kw)

    def backward_rows(self, *a, **kw):
        return backward_rows(*a, _lib=self.lib, **kw)

    def select(self, *a, **kw):
        return select(*a, _lib=self.lib, **kw)


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle().lib
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return 0  # bf16 bit patterns
    if a.dtype == np.float32:
        return 1
    if a.dtype == np.float64:
        return 2
    raise TypeError(f"oracle inputs must be bf16 bits (uint16), float32 or float64, got {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data


def prefill(q, k, v, *, causal: bool, lam: float, Br: int, Bc: int, scale: float | None = None,
            items=None, ref_mode: int = 0, ref_param: float = 0.0, nthreads: int = 0,
            static_mask=None, _lib=None) -> dict:
    """Blocked attention with the threshold skip, per query tile.

    q: [B, Hq, Lq, d]; k, v: [B, Hkv, Lkv, d]; all the same dtype (uint16 bf16
    bits, float32 or float64), C-contiguous. ``items`` selects flat tile ids
    ``(b*Hq + hq)*nQt + qt`` (default: every tile). ``static_mask``: optional
    uint8 [B, Hq, nQt, nKt], nonzero = the (query tile, KV block) pair is
    excluded before any computation. Returns per-item arrays:
    o [n, Br, d], lse [n, Br], mask [n, nKt] (0 computed, 1 skipped, 2 not
    visited), margin [n, nKt] (mu in natural units, NaN where not visited),
    plus the geometry.
    """
    q, k, v = (np.ascontiguousarray(t) for t in (q, k, v))
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    B, Hq, Lq, d = q.shape
    Bk, Hkv, Lkv, dk = k.shape
    assert Bk == B and dk == d and v.shape == k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    nQt = -(-Lq // Br)
    nKt = -(-Lkv // Bc)
    if items is None:
        items_arr = None
        n = B * Hq * nQt
    else:
        items_arr = np.ascontiguousarray(np.asarray(items, dtype=np.int64))
        n = int(items_arr.size)
    smask = None
    if static_mask is not None:
        smask = np.ascontiguousarray(np.asarray(static_mask, dtype=np.uint8))
        assert smask.shape == (B, Hq, nQt, nKt), smask.shape
    o = np.zeros((n, Br, d), np.float64)
    lse = np.zeros((n, Br), np.float64)
    mask = np.zeros((n, nKt), np.uint8)
    margin = np.zeros((n, nKt), np.float64)
    args = _PrefillArgs(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, code, B, Hq, Hkv, Lq, Lkv, d,
        int(bool(causal)), float(lam), Br, Bc, float(scale), int(ref_mode), float(ref_param),
        _ptr(items_arr), n, _ptr(smask), o.ctypes.data, lse.ctypes.data, mask.ctypes.data,
        margin.ctypes.data, int(nthreads))
    rc = (_lib or _load()).oracle_prefill(C.byref(args))
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    return dict(o=o, lse=lse, mask=mask, margin=margin, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lkv=Lkv,
                d=d, Br=Br, Bc=Bc, nQt=nQt, nKt=nKt,
                items=items_arr if items_arr is not None else np.arange(n, dtype=np.int64))


def prefill_dense(res: dict):
    """Scatter a full (all-items) ``prefill`` result to [B,Hq,Lq,d], [B,Hq,Lq],
    [B,Hq,nQt,nKt] mask and margin."""
    B, Hq, Lq, d, Br, nQt, nKt = (res[x] for x in ("B", "Hq", "Lq", "d", "Br", "nQt", "nKt"))
    assert res["o"].shape[0] == B * Hq * nQt
    o = res["o"].reshape(B, Hq, nQt * Br, d)[:, :, :Lq]
    lse = res["lse"].reshape(B, Hq, nQt * Br)[:, :, :Lq]
    return o, lse, res["mask"].reshape(B, Hq, nQt, nKt), res["margin"].reshape(B, Hq, nQt, nKt)


def split_len(Lkv: int, Bc: int, num_splits: int, _lib=None) -> int:
    """Keys per decode split: ceil(Lkv/S) rounded up to whole Bc blocks."""
    return int((_lib or _load()).oracle_split_len(Lkv, Bc, num_splits))


def decode(q, k, v, *, lam: float, Bc: int, num_splits: int, scale: float | None = None,
           nthreads: int = 0, _lib=None) -> dict:
    """Split-KV decode: q [B, Hq, 1, d] (or [B, Hq, d]); k, v [B, Hkv, Lkv, d].

    Returns o [B,Hq,d], lse [B,Hq], o_parts [B,Hq,S,d], lse_parts [B,Hq,S],
    mask [B,Hq,nKt], margin [B,Hq,nKt].
    """
    q, k, v = (np.ascontiguousarray(t) for t in (q, k, v))
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    B, Hq = q.shape[0], q.shape[1]
    d = q.shape[-1]
    assert q.size == B * Hq * d
    _, Hkv, Lkv, dk = k.shape
    assert dk == d and v.shape == k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    S = int(num_splits)
    nKt = -(-Lkv // Bc)
    o_parts = np.zeros((B, Hq, S, d), np.float64)
    lse_parts = np.zeros((B, Hq, S), np.float64)
    mask = np.zeros((B, Hq, nKt), np.uint8)
    margin = np.zeros((B, Hq, nKt), np.float64)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    args = _DecodeArgs(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, code, B, Hq, Hkv, Lkv, d, float(lam), Bc, S,
        float(scale), o_parts.ctypes.data, lse_parts.ctypes.data, mask.ctypes.data,
        margin.ctypes.data, o.ctypes.data, lse.ctypes.data, int(nthreads))
    rc = (_lib or _load()).oracle_decode(C.byref(args))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return dict(o=o, lse=lse, o_parts=o_parts, lse_parts=lse_parts, mask=mask, margin=margin)


def lse_merge(o_parts, lse_parts, _lib=None):
    """Log-sum-exp merge of split partials: o_parts [..., S, d], lse_parts [..., S]."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    S, d = o_parts.shape[-2], o_parts.shape[-1]
    lead = lse_parts.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (d,), np.float64)
    lse = np.zeros(lead, np.float64)
    (_lib or _load()).oracle_lse_merge(o_parts.ctypes.data, lse_parts.ctypes.data, n, S, d, o.ctypes.data,
                             lse.ctypes.data)
    return o, lse


def backward(q, k, v, dout, *, causal: bool, Br: int, Bc: int, scale: float | None = None,
             tile_mask=None, nthreads: int = 0, _lib=None):
    """Gradients (dq, dk, dv) of softmax attention over the kept keys, the
    forward's decisions held fixed. ``tile_mask``: uint8 [B, Hq, nQt, nKt] in
    the layout of the forward's skip mask (0 = the pair was computed and is
    kept); None keeps every causally visible key. Inputs as for ``prefill``;
    ``dout`` is dL/dO in the same dtype. Returns float64 arrays."""
    q, k, v, dout = (np.ascontiguousarray(t) for t in (q, k, v, dout))
    code = _dtype_code(q)
    assert all(_dtype_code(t) == code for t in (k, v, dout))
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    tm = None
    if tile_mask is not None:
        tm = np.ascontiguousarray(np.asarray(tile_mask, dtype=np.uint8))
        assert tm.shape == (B, Hq, -(-Lq // Br), -(-Lkv // Bc)), tm.shape
    dq = np.zeros((B, Hq, Lq, d), np.float64)
    dk = np.zeros((B, Hkv, Lkv, d), np.float64)
    dv = np.zeros((B, Hkv, Lkv, d), np.float64)
    args = _BackwardArgs(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, code,
                         B, Hq, Hkv, Lq, Lkv, d, int(bool(causal)), Br, Bc, float(scale),
                         _ptr(tm), dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(nthreads))
    rc = (_lib or _load()).oracle_backward(C.byref(args))
    if rc != 0:
        raise ValueError("oracle_backward rejected its arguments")
    return dq, dk, dv


def backward_rows(q, k, v, dout, *, causal: bool, Br: int, Bc: int, rows, scale: float | None = None,
                  tile_mask=None, kv_keys=None, nthreads: int = 0, _lib=None):
    """Sampled rows of ``backward``: dq of the query rows ``rows`` (flat ids
    ``(b*Hq + hq)*Lq + i``) as [n, d], and, with ``kv_keys = (b, hk, lo, hi)``,
    the terms those rows add to dk and dv of keys [lo, hi) of KV head (b, hk)
    as two [hi - lo, d] arrays (complete when ``rows`` holds every row that
    keeps one of those keys). Returns (dq_rows, dk_part, dv_part), float64."""
    q, k, v, dout = (np.ascontiguousarray(t) for t in (q, k, v, dout))
    code = _dtype_code(q)
    assert all(_dtype_code(t) == code for t in (k, v, dout))
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    tm = None
    if tile_mask is not None:
        tm = np.ascontiguousarray(np.asarray(tile_mask, dtype=np.uint8))
        assert tm.shape == (B, Hq, -(-Lq // Br), -(-Lkv // Bc)), tm.shape
    rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dq_rows = np.zeros((rows_arr.size, d), np.float64)
    kb, kh, lo, hi = kv_keys if kv_keys is not None else (0, 0, 0, 0)
    dk_part = np.zeros((hi - lo, d), np.float64)
    dv_part = np.zeros((hi - lo, d), np.float64)
    base = _BackwardArgs(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, code,
                         B, Hq, Hkv, Lq, Lkv, d, int(bool(causal)), Br, Bc, float(scale),
                         _ptr(tm), None, None, None, 0)
    args = _BackwardRowsArgs(base, rows_arr.size, _ptr(rows_arr), dq_rows.ctypes.data,
                             kb, kh, lo, hi, dk_part.ctypes.data if hi > lo else None,
                             dv_part.ctypes.data if hi > lo else None, int(nthreads))
    rc = (_lib or _load()).oracle_backward_rows(C.byref(args))
    if rc != 0:
        raise ValueError("oracle_backward_rows rejected its arguments")
    return dq_rows, dk_part, dv_part


def select(q, k, *, causal: bool, Br: int, Bc: int, tau: float, gamma: float,
           scale: float | None = None, with_map: bool = True, nthreads: int = 0, _lib=None) -> dict:
    """Pre-pass block selector (CRISP-style, on the block-pooled attention
    estimate). Returns mask uint8 [B, Hq, nQt, nKt] (0 = selected, 1 = not;
    the forward's static-mask convention), cstruct [B, Hq] and, with
    ``with_map``, the estimated map amap [B, Hq, nQt, nKt] (NaN where not
    visible)."""
    q, k = (np.ascontiguousarray(t) for t in (q, k))
    code = _dtype_code(q)
    assert _dtype_code(k) == code
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    nQt, nKt = -(-Lq // Br), -(-Lkv // Bc)
    mask = np.zeros((B, Hq, nQt, nKt), np.uint8)
    cs = np.zeros((B, Hq), np.float64)
    amap = np.zeros((B, Hq, nQt, nKt), np.float64) if with_map else None
    args = _SelectArgs(q.ctypes.data, k.ctypes.data, code, B, Hq, Hkv, Lq, Lkv, d,
                       int(bool(causal)), Br, Bc, float(scale), float(tau), float(gamma),
                       mask.ctypes.data, cs.ctypes.data, _ptr(amap), int(nthreads))
    rc = (_lib or _load()).oracle_select(C.byref(args))
    if rc != 0:
        raise ValueError("oracle_select rejected its arguments")
    return dict(mask=mask, cstruct=cs, amap=amap, nQt=nQt, nKt=nKt)
