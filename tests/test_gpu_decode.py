"""GPU split-KV decode and LSE merge vs the CPU oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import parity
import synth

pytestmark = pytest.mark.gpu


def _lib():
    import dynamic_block_sparse_tiled_b200 as bl
    return bl


def run_decode(w, lam):
    import torch
    bl = _lib()
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    lam32 = float(np.float32(lam))
    st = bl.new_stats()
    o, lse, mask = bl.attention_decode(q, k, v, lam=lam32, Bc=w.Bc, num_splits=w.num_splits,
                                       with_mask=True, stats=st)
    assert bl.blasst_check() == 0
    torch.cuda.synchronize()
    ref = oracle.decode(inp.q, inp.k, inp.v, lam=lam32, Bc=w.Bc, num_splits=w.num_splits)
    mask_g = mask.cpu().numpy()
    n_vis, n_dis, ok, dis = parity.compare_masks(mask_g, ref["mask"], ref["margin"], lam32)
    assert ok, f"decode mask: {n_dis}/{n_vis} disagree outside the tie band"
    o_g = parity.bf16_tensor_to_f64(o)[:, :, 0, :]
    lse_g = lse.cpu().numpy().astype(np.float64)
    stats = parity.compare_outputs(o_g, lse_g, ref["o"], ref["lse"], None, dis.any(axis=-1),
                                   max_tie_rows=n_dis)
    parity.assert_within(stats, w.name)
    sd = bl.stats_dict(st)
    assert sd["tiles_visited"] == mask_g.size
    assert sd["tiles_skipped"] == int((mask_g == 1).sum())
    return dict(stats, skip=float((ref["mask"] == 1).mean()))


DEC = synth.CONFIGS["decode_64k"]

SMALL = [
    ("dec_8k_a12", dict(B=2, Lkv=8192, num_splits=8, amp=12.0, n_needles=2)),
    ("dec_8k_literal", dict(B=2, Lkv=8192, num_splits=8)),
    ("dec_ragged", dict(B=2, Lkv=5000, num_splits=7, amp=12.0)),
    ("dec_bc64", dict(B=1, Lkv=4096, num_splits=5, Bc=64, amp=12.0)),
    ("dec_d64_g8", dict(B=1, Hq=16, Hkv=2, d=64, Lkv=3000, num_splits=4, amp=12.0)),
    ("dec_g1", dict(B=1, Hq=4, Hkv=4, Lkv=2048, num_splits=3, amp=12.0)),
    ("dec_empty_splits", dict(B=1, Lkv=300, num_splits=16, amp=12.0)),
]


@pytest.mark.parametrize("name,over", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("lam", [0.0, 1e-3, 1e-2])
def test_decode_parity_small(name, over, lam):
    run_decode(DEC.replace(name=name, **over), lam)


@pytest.mark.parametrize("cfg", ["decode_64k", "decode_64k_a12"])
def test_decode_full_size(cfg):
    """Full decode workload (B=16, 64K keys, 64 splits) in the benchmark's
    launch configuration, every row checked."""
    w = synth.CONFIGS[cfg]
    for lam in (0.0,) + tuple(w.lambdas):
        run_decode(w, lam)


def test_lse_merge_kernel():
    import torch
    bl = _lib()
    rng = np.random.default_rng(3)
    n_rows, S, d = 37, 9, 128
    o_parts = rng.standard_normal((n_rows, S, d)).astype(np.float32)
    lse_parts = (rng.standard_normal((n_rows, S)) * 3).astype(np.float32)
    lse_parts[3, :4] = -np.inf
    lse_parts[5, :] = -np.inf
    o_parts[5] = 0.0
    ref_o, ref_l = oracle.lse_merge(o_parts.astype(np.float64), lse_parts.astype(np.float64))
    op = torch.from_numpy(o_parts).cuda()
    lp = torch.from_numpy(lse_parts).cuda()
    for dt, tdt, tol in ((bl.BLASST_FP32, torch.float32, 1e-5), (bl.BLASST_BF16, torch.bfloat16, 1e-2)):
        o = torch.empty((n_rows, d), dtype=tdt, device="cuda")
        lse = torch.empty((n_rows,), dtype=torch.float32, device="cuda")
        bl.blasst_lse_merge(op, lp, o, lse, n_rows=n_rows, d=d, num_splits=S, out_dtype=dt)
        torch.cuda.synchronize()
        og = o.float().cpu().numpy()
        lg = lse.cpu().numpy()
        ok = np.isfinite(ref_l)
        assert np.abs(og[ok] - ref_o[ok]).max() < tol
        assert np.abs(lg[ok] - ref_l[ok]).max() < 1e-4
        assert np.all(lg[~ok] == -np.inf)
