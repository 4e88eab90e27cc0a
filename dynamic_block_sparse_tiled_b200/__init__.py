"""Blocked attention with softmax thresholding on B200 (sm_100a).

Thin Python binding of the C ABI in ``include/blasst.h`` (``libblasst.so``,
built in-tree by ``dynamic_block_sparse_tiled_b200.build``). The functions
below only marshal torch tensors and streams into pointers and sizes; every
step of the computation runs in the library's CUDA kernels. There is no CPU
path: if the library is missing or the tensors are not on a CUDA device, the
call raises.

The method (skip a KV block when exp(m_blk - m_run) < lambda on every row of
the query tile; the first block is always computed; a skipped block's V is
never read) follows "BLASST: Dynamic BLocked Attention Sparsity via Softmax
Thresholding" (Telegram channel seeallochnaya, post 3655, paragraphs 2-6
after the headline) and the authors' announcement in "BLASST wins Best Paper
at MLSys 2026 ..." (digg.com/ai/al6mgdew).
"""
from __future__ import annotations

import ctypes as C
import os
import threading

__all__ = [
    "BlasstError", "Stats", "lib_path", "load_library",
    "blasst_fwd", "blasst_fwd_ex", "blasst_decode", "blasst_decode_workspace_bytes",
    "blasst_lse_merge", "blasst_check", "blasst_selftest_exp2", "blasst_selftest_timeout",
    "blasst_decode_noalloc", "blasst_decode_noalloc_max_bytes", "blasst_status_string", "blasst_version",
    "blasst_bwd", "blasst_bwd_workspace_bytes", "blasst_select_blocks",
    "blasst_select_workspace_bytes", "select_blocks", "blasst_decode_mla",
    "blasst_decode_mla_workspace_bytes", "attention_decode_mla",
    "attention_prefill", "attention_backward", "attention_decode", "new_stats", "stats_dict",
    "BLASST_OK", "BLASST_EINVAL", "BLASST_EUNSUPPORTED", "BLASST_ECUDA", "BLASST_ETIMEOUT",
    "BLASST_EWORKSPACE", "BLASST_BF16", "BLASST_FP32",
]

BLASST_OK, BLASST_EINVAL, BLASST_EUNSUPPORTED, BLASST_ECUDA, BLASST_ETIMEOUT, BLASST_EWORKSPACE = (
    0, -1, -2, -3, -4, -5)
BLASST_BF16, BLASST_FP32 = 0, 1

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libblasst.so")
_lock = threading.Lock()
_lib = None


def lib_path() -> str:
    return _LIB_PATH


class BlasstError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {blasst_status_string(status)} ({status})" if where else
                         f"{blasst_status_string(status)} ({status})")


class Stats(C.Structure):
    _fields_ = [("tiles_visited", C.c_ulonglong), ("tiles_skipped", C.c_ulonglong),
                ("v_blocks_loaded", C.c_ulonglong), ("mma_flops", C.c_ulonglong),
                ("bytes_loaded", C.c_ulonglong), ("sm_cycles", C.c_ulonglong),
                ("sm_ns", C.c_ulonglong)]


class _FwdArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("o", C.c_void_p),
        ("lse", C.c_void_p),
        ("B", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("Lq", C.c_int), ("Lkv", C.c_int),
        ("d", C.c_int), ("causal", C.c_int), ("lam", C.c_float), ("Br", C.c_int), ("Bc", C.c_int),
        ("skip_mask_out", C.c_void_p), ("dtype", C.c_int), ("scale", C.c_float),
        ("stream", C.c_void_p), ("stats_out", C.c_void_p), ("block_mask_in", C.c_void_p),
    ]


class _BwdArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("o", C.c_void_p),
        ("dout", C.c_void_p), ("lse", C.c_void_p),
        ("dq", C.c_void_p), ("dk", C.c_void_p), ("dv", C.c_void_p),
        ("B", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("Lq", C.c_int), ("Lkv", C.c_int),
        ("d", C.c_int), ("causal", C.c_int), ("Br", C.c_int), ("Bc", C.c_int),
        ("skip_mask", C.c_void_p), ("scale", C.c_float),
        ("workspace", C.c_void_p), ("workspace_bytes", C.c_size_t), ("stream", C.c_void_p),
    ]


class _SelectArgs(C.Structure):
    _fields_ = [
        ("q", C.c_void_p), ("k", C.c_void_p),
        ("B", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("Lq", C.c_int), ("Lkv", C.c_int),
        ("d", C.c_int), ("causal", C.c_int), ("Br", C.c_int), ("Bc", C.c_int),
        ("scale", C.c_float), ("tau", C.c_float), ("gamma", C.c_float),
        ("mask_out", C.c_void_p), ("cstruct_out", C.c_void_p),
        ("workspace", C.c_void_p), ("workspace_bytes", C.c_size_t), ("stream", C.c_void_p),
    ]


def load_library(path: str | None = None):
    """Load ``libblasst.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or _LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                f"CUDA library {p} is missing; build it with `python -m "
                "dynamic_block_sparse_tiled_b200.build` (there is no CPU fallback)")
        lib = C.CDLL(p)
        vp, i, f, sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t
        lib.blasst_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, vp]
        lib.blasst_fwd.restype = i
        lib.blasst_fwd_ex.argtypes = [C.POINTER(_FwdArgs)]
        lib.blasst_fwd_ex.restype = i
        lib.blasst_decode_mla.argtypes = [vp, vp, vp, vp, i, i, i, f, i, i, f, vp, sz, vp, vp, vp]
        lib.blasst_decode_mla.restype = i
        lib.blasst_decode_mla_workspace_bytes.argtypes = [i, i, i]
        lib.blasst_decode_mla_workspace_bytes.restype = sz
        lib.blasst_decode_mla_splits.argtypes = [i, i, i, i]
        lib.blasst_decode_mla_splits.restype = i
        lib.blasst_select_blocks.argtypes = [C.POINTER(_SelectArgs)]
        lib.blasst_select_blocks.restype = i
        lib.blasst_select_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
        lib.blasst_select_workspace_bytes.restype = sz
        lib.blasst_bwd.argtypes = [C.POINTER(_BwdArgs)]
        lib.blasst_bwd.restype = i
        lib.blasst_bwd_workspace_bytes.argtypes = [i, i, i]
        lib.blasst_bwd_workspace_bytes.restype = sz
        lib.blasst_decode_workspace_bytes.argtypes = [i, i, i, i]
        lib.blasst_decode_workspace_bytes.restype = sz
        lib.blasst_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp, vp, vp]
        lib.blasst_decode.restype = i
        lib.blasst_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, vp, vp]
        lib.blasst_decode_noalloc.restype = i
        lib.blasst_decode_noalloc_max_bytes.argtypes = []
        lib.blasst_decode_noalloc_max_bytes.restype = sz
        lib.blasst_lse_merge.argtypes = [vp, vp, vp, vp, i, i, i, i, vp]
        lib.blasst_lse_merge.restype = i
        lib.blasst_selftest_timeout.argtypes = [C.c_ulonglong, vp]
        lib.blasst_selftest_timeout.restype = i
        lib.blasst_check.argtypes = [vp]
        lib.blasst_check.restype = i
        lib.blasst_status_string.argtypes = [i]
        lib.blasst_status_string.restype = C.c_char_p
        lib.blasst_selftest_exp2.argtypes = [vp, vp, vp, i, vp]
        lib.blasst_selftest_exp2.restype = i
        lib.blasst_last_cuda_error.argtypes = []
        lib.blasst_last_cuda_error.restype = C.c_char_p
        lib.blasst_version.argtypes = []
        lib.blasst_version.restype = i
        if path is None:
            _lib = lib
        return lib


def blasst_status_string(status: int) -> str:
    try:
        return load_library().blasst_status_string(int(status)).decode()
    except RuntimeError:
        return f"status {status}"


def blasst_version() -> int:
    return int(load_library().blasst_version())


# ----------------------------------------------------------------- marshalling
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensors passed to the CUDA library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != 0:
        if rc == BLASST_ECUDA:
            where = f"{where} [{load_library().blasst_last_cuda_error().decode()}]"
        raise BlasstError(rc, where)


def blasst_fwd(q, k, v, o, lse, B, Hq, Hkv, Lq, Lkv, d, causal, lam, Br, Bc, skip_mask_out=None):
    """The C entry point of the same name (bf16, legacy default stream)."""
    rc = load_library().blasst_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq,
                                   Lkv, d, int(causal), float(lam), Br, Bc, _ptr(skip_mask_out))
    _check(rc, "blasst_fwd")


def blasst_fwd_ex(q, k, v, o, lse, *, causal: bool, lam: float, Br: int, Bc: int,
                  skip_mask_out=None, scale: float = 0.0, stream=None, stats_out=None, dtype=None,
                  block_mask_in=None):
    """The C entry point of the same name. q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d], o like q,
    lse [B,Hq,Lq] fp32, skip_mask_out uint8 [B,Hq,ceil(Lq/Br),ceil(Lkv/Bc)] or None,
    stats_out a ``new_stats()`` tensor or None, block_mask_in an optional uint8
    [B,Hq,ceil(Lq/Br),ceil(Lkv/Bc)] static block mask (nonzero = excluded)."""
    import torch
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    if dtype is None:
        dtype = BLASST_BF16 if q.dtype == torch.bfloat16 else BLASST_FP32
    args = _FwdArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lkv, d,
                    int(bool(causal)), float(lam), Br, Bc, _ptr(skip_mask_out), int(dtype),
                    float(scale), _stream(stream), _ptr(stats_out), _ptr(block_mask_in))
    _check(load_library().blasst_fwd_ex(C.byref(args)), "blasst_fwd_ex")


def blasst_bwd_workspace_bytes(B: int, Hq: int, Lq: int) -> int:
    return int(load_library().blasst_bwd_workspace_bytes(B, Hq, Lq))


def blasst_bwd(q, k, v, o, dout, lse, dq, dk, dv, *, causal: bool, Br: int, Bc: int,
               workspace, skip_mask=None, scale: float = 0.0, stream=None):
    """The C entry point of the same name. q, o, dout [B,Hq,Lq,d] bf16; k, v
    [B,Hkv,Lkv,d] bf16; lse [B,Hq,Lq] fp32; dq [B,Hq,Lq,d], dk/dv [B,Hkv,Lkv,d]
    fp32 outputs; skip_mask the forward's uint8 decisions or None; workspace a
    uint8 CUDA tensor of blasst_bwd_workspace_bytes() bytes."""
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    args = _BwdArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                    _ptr(dv), B, Hq, Hkv, Lq, Lkv, d, int(bool(causal)), Br, Bc, _ptr(skip_mask),
                    float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                    _stream(stream))
    _check(load_library().blasst_bwd(C.byref(args)), "blasst_bwd")


def blasst_decode_mla_workspace_bytes(B: int, H: int, num_splits: int) -> int:
    return int(load_library().blasst_decode_mla_workspace_bytes(B, H, num_splits))


def blasst_decode_mla_splits(B: int, H: int, L: int, num_sms: int = 0) -> int:
    """The C entry point of the same name: a split count that fills whole
    waves of `num_sms` SMs (<= 0: the current device's count)."""
    S = int(load_library().blasst_decode_mla_splits(B, H, L, num_sms))
    if S <= 0:
        _check(S, "blasst_decode_mla_splits")
    return S


def blasst_decode_mla(q, cache, o, lse, *, lam: float, Bc: int, num_splits: int, workspace,
                      scale: float = 0.0, skip_mask_out=None, stats_out=None, stream=None):
    """The C entry point of the same name. q [B,H,576], cache [B,L,576] bf16;
    o [B,H,512] bf16, lse [B,H] fp32; workspace a uint8 CUDA tensor."""
    B, H = q.shape[0], q.shape[1]
    L = cache.shape[1]
    rc = load_library().blasst_decode_mla(
        _ptr(q), _ptr(cache), _ptr(o), _ptr(lse), B, H, L, float(lam), Bc, num_splits, float(scale),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(skip_mask_out),
        _ptr(stats_out), _stream(stream))
    _check(rc, "blasst_decode_mla")


def blasst_select_workspace_bytes(B, Hq, Hkv, Lq, Lkv, d, Br, Bc) -> int:
    return int(load_library().blasst_select_workspace_bytes(B, Hq, Hkv, Lq, Lkv, d, Br, Bc))


def blasst_select_blocks(q, k, mask_out, *, causal: bool, Br: int, Bc: int, tau: float,
                         gamma: float, workspace, scale: float = 0.0, cstruct_out=None,
                         stream=None):
    """The C entry point of the same name. q [B,Hq,Lq,d], k [B,Hkv,Lkv,d] bf16;
    mask_out uint8 [B,Hq,ceil(Lq/Br),ceil(Lkv/Bc)]; cstruct_out fp32 [B,Hq] or
    None; workspace a uint8 CUDA tensor of blasst_select_workspace_bytes()."""
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    args = _SelectArgs(_ptr(q), _ptr(k), B, Hq, Hkv, Lq, Lkv, d, int(bool(causal)), Br, Bc,
                       float(scale), float(tau), float(gamma), _ptr(mask_out), _ptr(cstruct_out),
                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                       _stream(stream))
    _check(load_library().blasst_select_blocks(C.byref(args)), "blasst_select_blocks")


def blasst_decode_workspace_bytes(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(load_library().blasst_decode_workspace_bytes(B, Hq, d, num_splits))


def blasst_decode(q, k_cache, v_cache, o, lse, *, lam: float, Bc: int, num_splits: int,
                  workspace, skip_mask_out=None, stats_out=None, stream=None):
    """The C entry point of the same name. q [B,Hq,1,d], caches [B,Hkv,Lkv,d] bf16,
    o [B,Hq,1,d] bf16, lse [B,Hq] fp32, workspace a uint8 CUDA tensor."""
    B, Hq = q.shape[0], q.shape[1]
    d = q.shape[-1]
    _, Hkv, Lkv, _ = k_cache.shape
    rc = load_library().blasst_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), B, Hq, Hkv, Lkv, d,
        float(lam), Bc, num_splits, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(skip_mask_out), _ptr(stats_out), _stream(stream))
    _check(rc, "blasst_decode")


def blasst_decode_noalloc(q, k_cache, v_cache, o, lse, *, lam: float, Bc: int, num_splits: int,
                          skip_mask_out=None, stats_out=None, stream=None):
    """The C entry point of the same name: blasst_decode without a caller
    workspace (the split partials live in a fixed array inside the library)."""
    B, Hq = q.shape[0], q.shape[1]
    d = q.shape[-1]
    _, Hkv, Lkv, _ = k_cache.shape
    rc = load_library().blasst_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), B, Hq, Hkv, Lkv, d,
        float(lam), Bc, num_splits, _ptr(skip_mask_out), _ptr(stats_out), _stream(stream))
    _check(rc, "blasst_decode_noalloc")


def blasst_decode_noalloc_max_bytes() -> int:
    return int(load_library().blasst_decode_noalloc_max_bytes())


def blasst_lse_merge(o_parts, lse_parts, o, lse, *, n_rows: int, d: int, num_splits: int,
                     out_dtype: int = BLASST_BF16, stream=None):
    rc = load_library().blasst_lse_merge(_ptr(o_parts), _ptr(lse_parts), _ptr(o), _ptr(lse),
                                         n_rows, d, num_splits, out_dtype, _stream(stream))
    _check(rc, "blasst_lse_merge")


def blasst_selftest_exp2(x, y_mufu, y_poly, stream=None):
    """The C self-test of the two exp2 paths (fp32 CUDA tensors of equal size)."""
    _check(load_library().blasst_selftest_exp2(_ptr(x), _ptr(y_mufu), _ptr(y_poly), x.numel(),
                                               _stream(stream)), "blasst_selftest_exp2")


def blasst_selftest_timeout(limit_ns: int, stream=None):
    """The C self-test of the bounded-wait failure path (see blasst.h)."""
    _check(load_library().blasst_selftest_timeout(int(limit_ns), _stream(stream)),
           "blasst_selftest_timeout")


def blasst_check(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    return int(load_library().blasst_check(_stream(stream)))


# -------------------------------------------------------------- conveniences
def new_stats(device="cuda"):
    """A zeroed device-side blasst_stats (uint64 fields, as an int64 tensor)."""
    import torch
    return torch.zeros(len(Stats._fields_), dtype=torch.int64, device=device)


def stats_dict(st) -> dict:
    vals = [int(x) for x in st.cpu().tolist()]
    return dict(zip([f[0] for f in Stats._fields_], vals))


def attention_prefill(q, k, v, *, causal=True, lam=0.0, Br=128, Bc=128, scale=0.0,
                      with_mask=False, stats=None, stream=None, block_mask=None):
    """Allocate outputs with torch and run blasst_fwd_ex. Returns (o, lse, mask)."""
    import torch
    B, Hq, Lq, d = q.shape
    Lkv = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    mask = None
    if with_mask:
        mask = torch.empty((B, Hq, -(-Lq // Br), -(-Lkv // Bc)), dtype=torch.uint8, device=q.device)
    blasst_fwd_ex(q, k, v, o, lse, causal=causal, lam=lam, Br=Br, Bc=Bc, skip_mask_out=mask,
                  scale=scale, stream=stream, stats_out=stats, block_mask_in=block_mask)
    return o, lse, mask


def attention_backward(q, k, v, o, lse, dout, *, causal=True, Br=128, Bc=128, skip_mask=None,
                       scale=0.0, stream=None, workspace=None):
    """Allocate fp32 gradients (and the workspace) with torch and run
    blasst_bwd with the forward's decisions ``skip_mask``. Returns (dq, dk, dv)."""
    import torch
    B, Hq, Lq, d = q.shape
    dq = torch.empty((B, Hq, Lq, d), dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(blasst_bwd_workspace_bytes(B, Hq, Lq), dtype=torch.uint8,
                                device=q.device)
    blasst_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal=causal, Br=Br, Bc=Bc, workspace=workspace,
               skip_mask=skip_mask, scale=scale, stream=stream)
    return dq, dk, dv


def select_blocks(q, k, *, causal=True, Br=128, Bc=128, tau=0.2, gamma=0.9, scale=0.0,
                  stream=None, workspace=None):
    """Allocate the mask (and the workspace) with torch and run
    blasst_select_blocks. Returns (mask, cstruct): mask uint8
    [B,Hq,nQt,nKt] (0 = selected), ready for attention_prefill(block_mask=...)."""
    import torch
    B, Hq, Lq, d = q.shape
    _, Hkv, Lkv, _ = k.shape
    mask = torch.empty((B, Hq, -(-Lq // Br), -(-Lkv // Bc)), dtype=torch.uint8, device=q.device)
    cs = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(blasst_select_workspace_bytes(B, Hq, Hkv, Lq, Lkv, d, Br, Bc),
                                dtype=torch.uint8, device=q.device)
    blasst_select_blocks(q, k, mask, causal=causal, Br=Br, Bc=Bc, tau=tau, gamma=gamma,
                         workspace=workspace, scale=scale, cstruct_out=cs, stream=stream)
    return mask, cs


def attention_decode_mla(q, cache, *, lam=0.0, num_splits=0, Bc=None, scale=0.0, with_mask=False,
                         stats=None, stream=None, workspace=None):
    """MLA-shaped decode (one latent KV head, 576-wide rows, 512-wide values):
    allocate outputs and workspace with torch and run blasst_decode_mla
    (64-key decision blocks; the tensor-core kernel when H is a multiple of
    128; num_splits <= 0 takes blasst_decode_mla_splits' choice for this
    device). Returns (o [B,H,512] bf16, lse [B,H], mask [B,H,ceil(L/64)] or None)."""
    import torch
    B, H = q.shape[0], q.shape[1]
    L = cache.shape[1]
    if Bc is None:
        Bc = 64
    if num_splits <= 0:
        num_splits = blasst_decode_mla_splits(B, H, L)
    o = torch.empty((B, H, 512), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(blasst_decode_mla_workspace_bytes(B, H, num_splits),
                                dtype=torch.uint8, device=q.device)
    mask = None
    if with_mask:
        mask = torch.empty((B, H, -(-L // Bc)), dtype=torch.uint8, device=q.device)
    blasst_decode_mla(q, cache, o, lse, lam=lam, Bc=Bc, num_splits=num_splits, workspace=workspace,
                      scale=scale, skip_mask_out=mask, stats_out=stats, stream=stream)
    return o, lse, mask


def attention_decode(q, k_cache, v_cache, *, lam=0.0, Bc=128, num_splits=64, with_mask=False,
                     stats=None, stream=None, workspace=None):
    """Allocate outputs (and the workspace) with torch and run blasst_decode.
    Returns (o, lse, mask)."""
    import torch
    B, Hq = q.shape[0], q.shape[1]
    d = q.shape[-1]
    Lkv = k_cache.shape[2]
    o = torch.empty((B, Hq, 1, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = blasst_decode_workspace_bytes(B, Hq, d, num_splits)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    mask = None
    if with_mask:
        mask = torch.empty((B, Hq, -(-Lkv // Bc)), dtype=torch.uint8, device=q.device)
    blasst_decode(q, k_cache, v_cache, o, lse, lam=lam, Bc=Bc, num_splits=num_splits,
                  workspace=workspace, skip_mask_out=mask, stats_out=stats, stream=stream)
    return o, lse, mask
