"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/blasst.h declares, and rejects bad arguments before
touching the device."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "blasst.h")


@pytest.fixture(scope="module")
def lib():
    from dynamic_block_sparse_tiled_b200 import build
    build.build()
    import dynamic_block_sparse_tiled_b200 as bl
    return bl.load_library()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"BLASST_API\s+[\w\s\*]+?\b(blasst_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("blasst_fwd", "blasst_fwd_ex", "blasst_decode", "blasst_decode_workspace_bytes",
              "blasst_lse_merge", "blasst_check", "blasst_status_string", "blasst_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in blasst.h but not exported"


def test_status_strings(lib):
    import dynamic_block_sparse_tiled_b200 as bl
    for code in (0, -1, -2, -3, -4, -5):
        assert bl.blasst_status_string(code).startswith("BLASST")
    assert bl.blasst_version() >= 100


def _fwd(lib, **kw):
    import dynamic_block_sparse_tiled_b200 as bl
    base = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0x50000, B=1, Hq=4, Hkv=2,
                Lq=256, Lkv=256, d=128, causal=1, lam=1e-3, Br=128, Bc=128, skip_mask_out=None,
                dtype=0, scale=0.0, stream=None, stats_out=None, block_mask_in=None)
    base.update(kw)
    args = bl._FwdArgs(*[base[f[0]] for f in bl._FwdArgs._fields_])
    return lib.blasst_fwd_ex(C.byref(args))


@pytest.mark.parametrize("bad,code", [
    (dict(q=None), -1),
    (dict(q=0x10008), -1),          # misaligned
    (dict(lse=0x50004), -1),        # misaligned lse
    (dict(B=0), -1),
    (dict(Hq=3, Hkv=2), -1),        # Hq % Hkv
    (dict(lam=1.0), -1),
    (dict(lam=-0.1), -1),
    (dict(lam=float("nan")), -1),
    (dict(d=96), -2),
    (dict(Br=32), -2),
    (dict(Bc=256), -2),
    (dict(Lq=300, Lkv=256), -2),    # causal with Lq > Lkv
    (dict(dtype=7), -2),
    (dict(dtype=1, d=128, Bc=64), -2),   # fp32 is d = 64 only
    (dict(dtype=1, d=64, Bc=128), -2),   # fp32 is Bc = 64 only
    (dict(Lq=4096 * 128 + 1, Lkv=4096 * 128 + 1, block_mask_in=0x60000), -2),  # list too long
])
def test_fwd_rejects_bad_arguments_without_a_gpu(lib, bad, code):
    assert _fwd(lib, **bad) == code


def _bwd(lib, **kw):
    import dynamic_block_sparse_tiled_b200 as bl
    base = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, dout=0x50000, lse=0x60000,
                dq=0x70000, dk=0x80000, dv=0x90000, B=1, Hq=4, Hkv=2, Lq=256, Lkv=256, d=128,
                causal=1, Br=128, Bc=128, skip_mask=None, scale=0.0, workspace=0xA0000,
                workspace_bytes=1 << 20, stream=None)
    base.update(kw)
    args = bl._BwdArgs(*[base[f[0]] for f in bl._BwdArgs._fields_])
    return lib.blasst_bwd(C.byref(args))


def test_bwd_workspace_bytes(lib):
    assert lib.blasst_bwd_workspace_bytes(2, 4, 100) == 2 * 2 * 4 * 128 * 4
    assert lib.blasst_bwd_workspace_bytes(1, 32, 32768) == 2 * 32 * 32768 * 4
    assert lib.blasst_bwd_workspace_bytes(0, 4, 100) == 0


@pytest.mark.parametrize("bad,code", [
    (None, -1),
    (dict(dout=None), -1),
    (dict(dq=0x70004), -1),         # misaligned
    (dict(Hq=3, Hkv=2), -1),
    (dict(Lq=0), -1),
    (dict(d=64), -2),               # the backward is d = 128 only
    (dict(Br=32), -2),
    (dict(Bc=256), -2),
    (dict(Lq=300, Lkv=256), -2),    # causal with Lq > Lkv
    (dict(workspace=None), -5),
    (dict(workspace_bytes=2 * 4 * 256 * 4 - 16), -5),
    (dict(workspace=0xA0008), -5),  # misaligned workspace
])
def test_bwd_rejects_bad_arguments_without_a_gpu(lib, bad, code):
    if bad is None:
        assert lib.blasst_bwd(None) == code
    else:
        assert _bwd(lib, **bad) == code


def _sel(lib, **kw):
    import dynamic_block_sparse_tiled_b200 as bl
    base = dict(q=0x10000, k=0x20000, B=1, Hq=4, Hkv=2, Lq=256, Lkv=256, d=128, causal=1,
                Br=128, Bc=128, scale=0.0, tau=0.2, gamma=0.9, mask_out=0x30000,
                cstruct_out=None, workspace=0x40000, workspace_bytes=1 << 20, stream=None)
    base.update(kw)
    args = bl._SelectArgs(*[base[f[0]] for f in bl._SelectArgs._fields_])
    return lib.blasst_select_blocks(C.byref(args))


def test_select_workspace_bytes(lib):
    # qbar 4*2*128 + kbar 2*2*128 + row statistics 4*2*3 + scores 4*2*2, fp32
    assert lib.blasst_select_workspace_bytes(1, 4, 2, 256, 256, 128, 128, 128) == \
        (4 * 2 * 128 + 2 * 2 * 128 + 4 * 2 * 3 + 4 * 2 * 2) * 4
    assert lib.blasst_select_workspace_bytes(0, 4, 2, 256, 256, 128, 128, 128) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(q=None), -1),
    (dict(mask_out=None), -1),
    (dict(k=0x20008), -1),
    (dict(Hq=3), -1),
    (dict(gamma=0.0), -1),
    (dict(gamma=1.5), -1),
    (dict(tau=float("nan")), -1),
    (dict(d=96), -2),
    (dict(Bc=32), -2),
    (dict(Lq=300), -2),                               # causal with Lq > Lkv
    (dict(Lq=2049 * 128, Lkv=2049 * 128), -2),        # more than 2048 KV blocks
    (dict(workspace=None), -5),
    (dict(workspace_bytes=64), -5),
])
def test_select_rejects_bad_arguments_without_a_gpu(lib, bad, code):
    assert _sel(lib, **bad) == code


def test_decode_mla_workspace_and_rejections(lib):
    ws = lib.blasst_decode_mla_workspace_bytes(8, 128, 32)
    assert ws == 8 * 128 * 32 * (512 + 1) * 4
    vp = 0x10000
    f = C.c_float
    # decision blocks other than 64
    assert lib.blasst_decode_mla(vp, vp, vp, vp, 2, 128, 4096, f(1e-3), 128, 4, f(0.0), vp, 1 << 30,
                                 None, None, None) == -2
    assert lib.blasst_decode_mla(vp, vp, vp, vp, 2, 128, 4096, f(1e-3), 32, 4, f(0.0), vp, 1 << 30,
                                 None, None, None) == -2
    # heads not a multiple of 16
    assert lib.blasst_decode_mla(vp, vp, vp, vp, 2, 24, 4096, f(1e-3), 64, 4, f(0.0), vp, 1 << 30,
                                 None, None, None) == -2
    # lambda out of range, bad sizes, misaligned pointers
    assert lib.blasst_decode_mla(vp, vp, vp, vp, 2, 32, 4096, f(1.0), 64, 4, f(0.0), vp, 1 << 30,
                                 None, None, None) == -1
    assert lib.blasst_decode_mla(vp, vp, vp, vp, 0, 32, 4096, f(1e-3), 64, 4, f(0.0), vp, 1 << 30,
                                 None, None, None) == -1
    assert lib.blasst_decode_mla(vp + 8, vp, vp, vp, 2, 32, 4096, f(1e-3), 64, 4, f(0.0), vp, 1 << 30,
                                 None, None, None) == -1
    # workspace too small
    need = lib.blasst_decode_mla_workspace_bytes(2, 32, 4)
    assert lib.blasst_decode_mla(vp, vp, vp, vp, 2, 32, 4096, f(1e-3), 64, 4, f(0.0), vp, need - 16,
                                 None, None, None) == -5


def _mla_split_cost(B, H, L, S, sms):
    per_split = 2 * B * (H // 128) if H % 128 == 0 else B * (H // 16)
    blocks = -(-(-(-L // S)) // 64)
    return -(-(per_split * S) // sms) * blocks


@pytest.mark.parametrize("B,H,L,sms", [(8, 128, 65536, 148), (1, 128, 4096, 148), (3, 256, 100000, 132),
                                       (2, 112, 65536, 148), (64, 128, 8192, 148), (1, 16, 64, 148)])
def test_decode_mla_splits_fill_waves(lib, B, H, L, sms):
    """The split count is the smallest within 3 % of the best wave-filling
    estimate (brute force over every split count)."""
    S = lib.blasst_decode_mla_splits(B, H, L, sms)
    nb = -(-L // 64)
    costs = {s: _mla_split_cost(B, H, L, s, sms) for s in range(1, min(nb, 1024) + 1)}
    best = min(costs.values())
    assert 1 <= S <= min(nb, 1024)
    assert costs[S] <= 1.03 * best
    assert all(costs[s] > 1.03 * best for s in range(1, S))


def test_decode_mla_splits_values_and_rejections(lib):
    # the MLA decode workload on 148 SMs: 144 CTAs of 114 blocks, one wave
    assert lib.blasst_decode_mla_splits(8, 128, 65536, 148) == 9
    assert lib.blasst_decode_mla_splits(0, 128, 65536, 148) == -1
    assert lib.blasst_decode_mla_splits(8, 24, 65536, 148) == -1
    assert lib.blasst_decode_mla_splits(8, 128, 0, 148) == -1


def test_decode_workspace_and_rejections(lib):
    ws = lib.blasst_decode_workspace_bytes(16, 32, 128, 64)
    assert ws == 16 * 32 * 64 * (128 + 1) * 4
    assert lib.blasst_decode_workspace_bytes(0, 32, 128, 64) == 0
    vp = 0x10000
    # too-small workspace
    rc = lib.blasst_decode(vp, vp, vp, vp, vp, 16, 32, 8, 65536, 128, C.c_float(1e-3), 128, 64,
                           vp, ws - 16, None, None, None)
    assert rc == -5
    # GQA group of 3 is not built
    rc = lib.blasst_decode(vp, vp, vp, vp, vp, 1, 6, 2, 1024, 128, C.c_float(1e-3), 128, 4,
                           vp, 1 << 30, None, None, None)
    assert rc == -2
    # lambda out of range
    rc = lib.blasst_decode(vp, vp, vp, vp, vp, 1, 4, 1, 1024, 128, C.c_float(2.0), 128, 4,
                           vp, 1 << 30, None, None, None)
    assert rc == -1


def test_decode_noalloc_checks_the_shape_before_the_size(lib):
    """The allocation-free decode reports an unsupported or invalid shape as
    such, even when its partials would not fit the fixed array either."""
    vp = 0x10000
    cap = lib.blasst_decode_noalloc_max_bytes()
    # d = 256 is not built: EUNSUPPORTED, although 64*32*64*257*4 bytes > 32 MiB
    assert lib.blasst_decode_workspace_bytes(64, 32, 256, 64) > cap
    rc = lib.blasst_decode_noalloc(vp, vp, vp, vp, vp, 64, 32, 8, 65536, 256, C.c_float(1e-3), 128,
                                   64, None, None, None)
    assert rc == -2
    # Hq not a multiple of Hkv: EINVAL
    rc = lib.blasst_decode_noalloc(vp, vp, vp, vp, vp, 64, 32, 7, 65536, 128, C.c_float(1e-3), 128,
                                   64, None, None, None)
    assert rc == -1
    # a misaligned pointer: EINVAL
    rc = lib.blasst_decode_noalloc(vp + 2, vp, vp, vp, vp, 1, 32, 8, 1024, 128, C.c_float(1e-3),
                                   128, 4, None, None, None)
    assert rc == -1
    # a valid shape that does not fit: EWORKSPACE (before any device call)
    rc = lib.blasst_decode_noalloc(vp, vp, vp, vp, vp, 64, 32, 8, 65536, 128, C.c_float(1e-3), 128,
                                   64, None, None, None)
    assert rc == -5


def test_merge_rejects_bad_arguments(lib):
    assert lib.blasst_lse_merge(None, None, None, None, 1, 128, 2, 0, None) == -1
    assert lib.blasst_lse_merge(0x1000, 0x2000, 0x3000, 0x4000, 4, 128, 2, 9, None) == -1


def test_python_binding_fails_loudly_without_cuda_tensors():
    import numpy as np
    import torch
    import dynamic_block_sparse_tiled_b200 as bl
    q = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bl.attention_prefill(q, q, q)
    del np


def test_stats_struct_matches_the_header():
    """The binding's blasst_stats has the header's fields, in order (the
    device writes them by offset)."""
    import dynamic_block_sparse_tiled_b200 as bl
    hdr = open(HEADER).read()
    body = re.search(r"typedef struct blasst_stats \{(.*?)\} blasst_stats;", hdr, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"unsigned long long (\w+);", body)
    assert fields == [f[0] for f in bl.Stats._fields_]
    assert C.sizeof(bl.Stats) == 8 * len(fields)
