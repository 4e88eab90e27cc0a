"""The allocation-free decode entry point (blasst_decode_noalloc), called
through the C ABI, against the workspace entry point (blasst_decode).

Some callers cannot allocate device memory where they run decode (a plugin
whose framework owns every allocation, a serving loop with a fixed memory
plan); blasst_decode_noalloc keeps the split partials in a fixed array inside
the library instead. This file is collected last on purpose, and it passes
both on its own in a fresh process and after the other tests.
"""
import ctypes as C

import numpy as np
import pytest

import parity
import synth

pytestmark = pytest.mark.gpu


def _inputs(seed, amp):
    w = synth.CONFIGS["decode_64k"].replace(name=f"noalloc_{seed}", B=3, Lkv=6000, num_splits=7,
                                            amp=amp, n_needles=2, seed=seed)
    inp = synth.generate(w)
    return w, tuple(parity.to_device(a) for a in (inp.q, inp.k, inp.v))


def _out(w):
    import torch
    o = torch.empty((w.B, w.Hq, 1, w.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    mask = torch.empty((w.B, w.Hq, -(-w.Lkv // w.Bc)), dtype=torch.uint8, device="cuda")
    return o, lse, mask


def test_decode_noalloc_matches_workspace_entry_point_twice():
    import torch
    import dynamic_block_sparse_tiled_b200 as bl
    lib = bl.load_library()
    lam = float(np.float32(1e-3))
    stream = torch.cuda.current_stream().cuda_stream
    for call, (seed, amp) in enumerate(((0, 12.0), (1, 3.0))):
        w, (q, k, v) = _inputs(seed, amp)
        # reference: the entry point with a caller-owned workspace
        o_ref, lse_ref, mask_ref = _out(w)
        ws = torch.empty(bl.blasst_decode_workspace_bytes(w.B, w.Hq, w.d, w.num_splits),
                         dtype=torch.uint8, device="cuda")
        rc = lib.blasst_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_ref.data_ptr(),
                               lse_ref.data_ptr(), w.B, w.Hq, w.Hkv, w.Lkv, w.d, C.c_float(lam),
                               w.Bc, w.num_splits, ws.data_ptr(), ws.numel(), mask_ref.data_ptr(),
                               None, stream)
        assert rc == 0, bl.blasst_status_string(rc)
        # the allocation-free entry point, straight through the C ABI
        o, lse, mask = _out(w)
        rc = lib.blasst_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                       lse.data_ptr(), w.B, w.Hq, w.Hkv, w.Lkv, w.d,
                                       C.c_float(lam), w.Bc, w.num_splits, mask.data_ptr(), None,
                                       stream)
        assert rc == 0, bl.blasst_status_string(rc)
        assert lib.blasst_check(stream) == 0
        torch.cuda.synchronize()
        stats = parity.compare_outputs(parity.bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64),
                                       parity.bf16_tensor_to_f64(o_ref),
                                       lse_ref.cpu().numpy().astype(np.float64))
        parity.assert_within(stats, f"call {call + 1}")
        assert torch.equal(mask, mask_ref), f"call {call + 1}: skip masks differ"


def test_decode_noalloc_rejects_oversize_requests():
    import dynamic_block_sparse_tiled_b200 as bl
    lib = bl.load_library()
    cap = lib.blasst_decode_noalloc_max_bytes()
    assert cap == 32 << 20
    # B=64, Hq=32, S=64, d=128 needs 64*32*64*129*4 bytes (> 32 MiB): refused before any launch
    assert bl.blasst_decode_workspace_bytes(64, 32, 128, 64) > cap
    p = 0x10000
    rc = lib.blasst_decode_noalloc(p, p, p, p, p, 64, 32, 8, 65536, 128, C.c_float(1e-3), 128, 64,
                                   None, None, None)
    assert rc == bl.BLASST_EWORKSPACE


def test_decode_noalloc_empty_splits_after_a_larger_call():
    """Trailing empty splits (Lkv = 600 in 7 splits of 128 keys: splits 5
    and 6 hold no key) must not merge what an earlier call left in the shared
    array: the split kernel writes o = 0, lse = -inf for them, and the merge
    ignores them. The earlier, larger call fills the array first; the
    reference is the workspace entry point with its workspace filled with NaN,
    so any partial that is read without being written shows up there too."""
    import torch
    import dynamic_block_sparse_tiled_b200 as bl
    lib = bl.load_library()
    lam = float(np.float32(1e-3))
    stream = torch.cuda.current_stream().cuda_stream
    # 1) a larger call fills the shared array with its partials
    w_big, (qb, kb, vb) = _inputs(5, 12.0)
    ob, lseb, mb = _out(w_big)
    rc = lib.blasst_decode_noalloc(qb.data_ptr(), kb.data_ptr(), vb.data_ptr(), ob.data_ptr(),
                                   lseb.data_ptr(), w_big.B, w_big.Hq, w_big.Hkv, w_big.Lkv,
                                   w_big.d, C.c_float(lam), w_big.Bc, w_big.num_splits,
                                   mb.data_ptr(), None, stream)
    assert rc == 0, bl.blasst_status_string(rc)
    # 2) a small call whose last two splits are empty
    w = synth.CONFIGS["decode_64k"].replace(name="noalloc_empty", B=2, Lkv=600, num_splits=7,
                                            amp=12.0, n_needles=1, seed=6)
    per = -(-w.Lkv // w.num_splits)
    Ls = -(-per // w.Bc) * w.Bc
    assert Ls == 128 and 5 * Ls >= w.Lkv  # splits 5 and 6 are empty
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    o, lse, mask = _out(w)
    rc = lib.blasst_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), w.B, w.Hq, w.Hkv, w.Lkv, w.d, C.c_float(lam),
                                   w.Bc, w.num_splits, mask.data_ptr(), None, stream)
    assert rc == 0, bl.blasst_status_string(rc)
    o_ref, lse_ref, mask_ref = _out(w)
    nbytes = bl.blasst_decode_workspace_bytes(w.B, w.Hq, w.d, w.num_splits)
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.blasst_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_ref.data_ptr(),
                           lse_ref.data_ptr(), w.B, w.Hq, w.Hkv, w.Lkv, w.d, C.c_float(lam), w.Bc,
                           w.num_splits, ws.data_ptr(), nbytes, mask_ref.data_ptr(), None, stream)
    assert rc == 0, bl.blasst_status_string(rc)
    assert lib.blasst_check(stream) == 0
    torch.cuda.synchronize()
    o64, o_ref64 = parity.bf16_tensor_to_f64(o), parity.bf16_tensor_to_f64(o_ref)
    l64, l_ref64 = (lse.cpu().numpy().astype(np.float64), lse_ref.cpu().numpy().astype(np.float64))
    assert np.isfinite(o64).all() and np.isfinite(o_ref64).all()
    assert np.isfinite(l64).all() and np.isfinite(l_ref64).all()
    parity.assert_within(parity.compare_outputs(o64, l64, o_ref64, l_ref64), "empty splits")
    assert torch.equal(mask, mask_ref)
    # the empty splits' partials were written: lse = -inf at splits 5 and 6
    rows = w.B * w.Hq
    lse_parts = ws[rows * w.num_splits * w.d:].view(rows, w.num_splits).cpu().numpy()
    assert np.all(lse_parts[:, 5:] == -np.inf) and np.isfinite(lse_parts[:, :5]).all()
