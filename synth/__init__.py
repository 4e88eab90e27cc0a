"""Seeded synthetic workloads for blocked attention with softmax thresholding.

This module is the one piece that both the CPU oracle side and the CUDA side
use: it produces the input tensors (Q, K, V) and nothing else. It holds no
attention arithmetic. The random numbers come from ``synth.c`` (SplitMix64 in
counter mode, Box-Muller normals); this file only lays out the planted
structure.

Planted structure (per batch entry b and KV head hk; query heads of a GQA
group share their KV head's directions):

* ``u``: a random unit direction. Query rows get ``+amp*u``; key rows get
  ``+amp*u`` on the first ``sink_len`` keys, on ``n_rand`` random
  ``rand_len``-key blocks and on ``n_needles`` random ``needle_len``-key
  "needle" blocks (block sets are unions: a key is lifted once).
* prefill local window (``window > 0``): positions are cut into aligned
  segments of ``window`` keys, each with its own unit direction ``w_s``
  orthogonal to ``u``; query i gets ``+window_q_amp*w_{s(i)}`` and key j gets
  ``+window_k_amp*w_{s(j)}``, so a query favours keys of its own segment.
* decode window (``decode_window > 0``): the last ``decode_window`` keys get
  ``+window_k_amp*u`` (the single decode query sits at position Lkv-1).
* ``diffuse_heads='upper_half'``: KV heads hk >= Hkv/2 (and their query
  heads) get no planted structure at all: i.i.d. N(0,1) Q and K.
* V is i.i.d. N(0,1).
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

# stream ids of the counter-based generator
STREAM_Q, STREAM_K, STREAM_V, STREAM_U, STREAM_W, STREAM_BLOCKS = 1, 2, 3, 4, 5, 6
STREAM_DO = 7


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-o", tmp,
                               _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class _FillArgs(C.Structure):
    _fields_ = [
        ("B", C.c_int64), ("H", C.c_int64), ("L", C.c_int64), ("d", C.c_int64),
        ("Hkv", C.c_int64), ("seed", C.c_uint64), ("stream", C.c_uint64),
        ("amp_u", C.c_void_p), ("u", C.c_void_p), ("seg_len", C.c_int64),
        ("amp_w", C.c_double), ("w", C.c_void_p), ("seg_pos_offset", C.c_int64),
        ("nseg", C.c_int64),
        ("out_f32", C.c_void_p), ("out_bf16", C.c_void_p), ("nthreads", C.c_int),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            lib.synth_u64.argtypes = [C.c_uint64, C.c_uint64, C.c_uint64, C.c_int64, C.c_void_p]
            lib.synth_u64.restype = None
            lib.synth_normal.argtypes = [C.c_uint64, C.c_uint64, C.c_uint64, C.c_int64, C.c_void_p]
            lib.synth_normal.restype = None
            lib.synth_fill.argtypes = [C.POINTER(_FillArgs)]
            lib.synth_fill.restype = C.c_int
            lib.synth_mix64.argtypes = [C.c_uint64]
            lib.synth_mix64.restype = C.c_uint64
            _lib = lib
    return _lib


def mix64(x: int) -> int:
    return int(_load().synth_mix64(C.c_uint64(x & (2**64 - 1))))


def draws_u64(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint64)
    _load().synth_u64(seed, stream, start, n, out.ctypes.data)
    return out


def normals(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    _load().synth_normal(seed, stream, start, n, out.ctypes.data)
    return out


@dataclass(frozen=True)
class Workload:
    """One synthetic attention problem (shapes, tiles, thresholds, structure)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lkv: int
    d: int
    dtype: str = "bf16"          # 'bf16' | 'fp32'
    causal: bool = True
    Br: int = 128
    Bc: int = 128
    lambdas: tuple = (0.0, 1e-3)
    num_splits: int = 0          # > 0: split-KV decode (Lq == 1, non-causal)
    amp: float = 3.0
    sink_len: int = 64
    n_rand: int = 2
    rand_len: int = 64
    n_needles: int = 0
    needle_len: int = 128
    window: int = 0
    window_q_amp: float = 3.0
    window_k_amp: float = 1.5
    decode_window: int = 0
    diffuse_heads: str = "none"  # 'none' | 'upper_half'
    seed: int = 0

    @property
    def is_decode(self) -> bool:
        return self.num_splits > 0

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the benchmark (shapes of Llama-3.1-8B attention and
# 32K-256K contexts), literal amplitude 3, plus labelled calibrated variants.
CONFIGS = {
    "tiny_fp32_1k": Workload("tiny_fp32_1k", B=1, Hq=2, Hkv=2, Lq=1024, Lkv=1024, d=64,
                             dtype="fp32", Br=64, Bc=64, lambdas=(0.0, 1e-3, 1e-2)),
    "prefill_32k": Workload("prefill_32k", B=1, Hq=32, Hkv=8, Lq=32768, Lkv=32768, d=128,
                            lambdas=(0.0, 1e-3), n_needles=8, window=1024),
    "prefill_128k": Workload("prefill_128k", B=1, Hq=32, Hkv=8, Lq=131072, Lkv=131072, d=128,
                             lambdas=(0.0, 1e-4, 1e-3, 1e-2), n_needles=8, window=1024),
    "decode_64k": Workload("decode_64k", B=16, Hq=32, Hkv=8, Lq=1, Lkv=65536, d=128,
                           causal=False, Br=1, Bc=128, lambdas=(1e-3,), num_splits=64,
                           n_needles=4, decode_window=1024),
    "prefill_256k": Workload("prefill_256k", B=1, Hq=8, Hkv=8, Lq=262144, Lkv=262144, d=128,
                             lambdas=(1e-3,), n_needles=8, window=1024,
                             diffuse_heads="upper_half"),
}
# MLA-shaped decode (one latent KV head of 576-wide rows, 128 query heads, values
# = the first 512 dims of the rows; the cache is K, V is not used). 9 splits:
# the library's wave-filling choice on 148 SMs (blasst_decode_mla_splits).
CONFIGS["decode_mla_64k"] = Workload("decode_mla_64k", B=8, Hq=128, Hkv=1, Lq=1, Lkv=65536, d=576,
                                     causal=False, Br=1, Bc=64, lambdas=(1e-3,), num_splits=9,
                                     n_needles=4, decode_window=1024)
# Calibrated "structured" variants: amplitude 12 on the planted direction (the
# literal amplitude 3 leaves almost no block below the threshold).
for _k in ("prefill_32k", "prefill_128k", "decode_64k", "prefill_256k", "decode_mla_64k"):
    CONFIGS[_k + "_a12"] = CONFIGS[_k].replace(name=_k + "_a12", amp=12.0)


@dataclass
class Inputs:
    workload: Workload
    q: np.ndarray      # [B, Hq, Lq, d]  uint16 (bf16 bits) or float32
    k: np.ndarray      # [B, Hkv, Lkv, d]
    v: np.ndarray
    u: np.ndarray      # [B, Hkv, d]
    planted_blocks: dict


def _pick_blocks(seed, b, hk, Hkv, kind, n_cand, n_pick):
    """n_pick distinct block indices from [1, n_cand), by smallest draw."""
    if n_pick <= 0 or n_cand <= 1:
        return np.zeros(0, np.int64)
    base = (((b * Hkv + hk) * 4 + kind) << 32)
    r = draws_u64(seed, STREAM_BLOCKS, base, n_cand - 1)
    order = np.argsort(r, kind="stable")[: min(n_pick, n_cand - 1)]
    return np.sort(order + 1).astype(np.int64)


def _unit(vecs):
    return vecs / np.linalg.norm(vecs, axis=-1, keepdims=True)


def structure(w: Workload):
    """Directions and per-row amplitudes of the planted structure."""
    B, Hkv, d = w.B, w.Hkv, w.d
    u = _unit(normals(w.seed, STREAM_U, 0, B * Hkv * d).reshape(B, Hkv, d))
    structured = np.ones((B, Hkv), bool)
    if w.diffuse_heads == "upper_half":
        structured[:, Hkv // 2:] = False
    elif w.diffuse_heads != "none":
        raise ValueError(w.diffuse_heads)

    amp_q = np.zeros((B, Hkv, w.Lq), np.float32)
    amp_k = np.zeros((B, Hkv, w.Lkv), np.float32)
    planted = {}
    for b in range(B):
        for hk in range(Hkv):
            if not structured[b, hk]:
                continue
            amp_q[b, hk, :] = w.amp
            lift = np.zeros(w.Lkv, bool)
            lift[: min(w.sink_len, w.Lkv)] = True
            rb = _pick_blocks(w.seed, b, hk, Hkv, 0, w.Lkv // w.rand_len, w.n_rand) if w.rand_len else []
            for blk in rb:
                lift[blk * w.rand_len:(blk + 1) * w.rand_len] = True
            nb = _pick_blocks(w.seed, b, hk, Hkv, 1, w.Lkv // w.needle_len, w.n_needles)
            for blk in nb:
                lift[blk * w.needle_len:(blk + 1) * w.needle_len] = True
            amp_k[b, hk, lift] = w.amp
            if w.decode_window > 0:
                amp_k[b, hk, max(0, w.Lkv - w.decode_window):] += w.window_k_amp
            planted[(b, hk)] = dict(rand_blocks=list(map(int, rb)), needles=list(map(int, nb)))

    wdir = None
    if w.window > 0:
        L = max(w.Lq, w.Lkv)
        nseg = -(-L // w.window)
        raw = normals(w.seed, STREAM_W, 0, B * Hkv * nseg * d).reshape(B, Hkv, nseg, d)
        raw = raw - np.einsum("bhsd,bhd->bhs", raw, u)[..., None] * u[:, :, None, :]
        wdir = _unit(raw)
        wdir[~structured] = 0.0
    return u, amp_q, amp_k, wdir, planted


def _fill(w, H, L, stream, amp, u, wdir, amp_w, seg_off, out, nthreads):
    bf16 = out.dtype == np.uint16
    args = _FillArgs(
        w.B, H, L, w.d, w.Hkv, w.seed, stream,
        None if amp is None else amp.ctypes.data, None if u is None else u.ctypes.data,
        w.window if (wdir is not None and amp_w != 0.0) else 0, float(amp_w),
        None if wdir is None else wdir.ctypes.data, seg_off,
        0 if wdir is None else wdir.shape[2],
        None if bf16 else out.ctypes.data, out.ctypes.data if bf16 else None, int(nthreads))
    if _load().synth_fill(C.byref(args)) != 0:
        raise ValueError("synth_fill rejected its arguments")


def generate(w: Workload, out_q=None, out_k=None, out_v=None, nthreads: int = 0) -> Inputs:
    """Fill Q, K, V for workload ``w``. bf16 tensors come back as uint16 bit
    patterns, fp32 as float32. ``out_*`` may be preallocated C-contiguous numpy
    arrays of the right shape and dtype (for example views of pinned host
    memory)."""
    dt = np.uint16 if w.dtype == "bf16" else np.float32
    if w.dtype not in ("bf16", "fp32"):
        raise ValueError(w.dtype)
    shp_q = (w.B, w.Hq, w.Lq, w.d)
    shp_kv = (w.B, w.Hkv, w.Lkv, w.d)
    q = np.empty(shp_q, dt) if out_q is None else out_q
    k = np.empty(shp_kv, dt) if out_k is None else out_k
    v = np.empty(shp_kv, dt) if out_v is None else out_v
    for t, shp in ((q, shp_q), (k, shp_kv), (v, shp_kv)):
        assert t.shape == shp and t.dtype == dt and t.flags.c_contiguous
    u, amp_q, amp_k, wdir, planted = structure(w)
    u = np.ascontiguousarray(u)
    wd = None if wdir is None else np.ascontiguousarray(wdir)
    off = w.Lkv - w.Lq if w.causal else 0
    _fill(w, w.Hq, w.Lq, STREAM_Q, amp_q, u, wd, w.window_q_amp, off, q, nthreads)
    _fill(w, w.Hkv, w.Lkv, STREAM_K, amp_k, u, wd, w.window_k_amp, 0, k, nthreads)
    _fill(w, w.Hkv, w.Lkv, STREAM_V, None, None, None, 0.0, 0, v, nthreads)
    return Inputs(w, q, k, v, u, planted)


def grad_output(w: Workload, out=None) -> np.ndarray:
    """dL/dO for the backward pass: i.i.d. N(0, 1) entries of shape
    [B, Hq, Lq, d] (the gradient of a random linear loss), as bf16 bit
    patterns (round to nearest even) or float32, like ``generate``."""
    shp = (w.B, w.Hq, w.Lq, w.d)
    x = normals(w.seed, STREAM_DO, 0, int(np.prod(shp))).astype(np.float32).reshape(shp)
    if w.dtype == "fp32":
        res = x
    else:
        bits = x.view(np.uint32)
        res = ((bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1)))
               >> np.uint32(16)).astype(np.uint16)
    if out is None:
        return res
    out[...] = res
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32)
