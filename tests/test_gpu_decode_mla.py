"""GPU MLA-shaped decode (blasst_decode_mla) vs the CPU oracle.

MLA attention in the absorbed form is softmax attention with one KV head whose
keys are the cached 576-wide rows c and whose values are c[:, 0:512]. The
oracle's decode computes exactly that when given v = c with the 64 rotary
columns set to zero: its output's first 512 columns are the MLA output and the
last 64 are zero. Tolerances and the mask rule are the decode ones
(tests/parity.py)."""
import numpy as np
import pytest

import oracle
import parity
import synth

pytestmark = pytest.mark.gpu

MLA = synth.CONFIGS["decode_mla_64k"]


def _lib():
    from dynamic_block_sparse_tiled_b200 import build
    build.build()
    import dynamic_block_sparse_tiled_b200 as bl
    return bl


def _oracle_v(k):
    v = k.copy()
    v[..., 512:] = 0
    return v


def run_mla(w, lam, seqs=None, heads=None, Bc=64):
    """Run the GPU kernel on the whole workload (the tensor-core kernel when
    the head count is a multiple of 128, else the mma.sync one); compare
    sequences ``seqs`` and heads ``heads`` (default all) with the oracle run
    with the same 64-key decision blocks."""
    bl = _lib()
    inp = synth.generate(w)
    qd = parity.to_device(inp.q[:, :, 0, :].copy())   # [B, H, 576]
    cd = parity.to_device(inp.k[:, 0].copy())         # [B, L, 576]
    lam32 = float(np.float32(lam))
    st = bl.new_stats()
    o, lse, mask = bl.attention_decode_mla(qd, cd, lam=lam32, num_splits=w.num_splits, Bc=Bc,
                                           with_mask=True, stats=st)
    assert bl.blasst_check() == 0
    seqs = range(w.B) if seqs is None else seqs
    heads = slice(None) if heads is None else heads
    o_g = parity.bf16_tensor_to_f64(o)
    lse_g = lse.cpu().numpy().astype(np.float64)
    mask_g = mask.cpu().numpy()
    worst = dict(o_max=0.0, o_mean=0.0, lse_max=0.0)
    skip = []
    for b in seqs:
        qb = np.ascontiguousarray(inp.q[b:b + 1, heads])
        kb = np.ascontiguousarray(inp.k[b:b + 1])
        ref = oracle.decode(qb, kb, _oracle_v(kb), lam=lam32, Bc=Bc, num_splits=w.num_splits)
        assert np.all(ref["o"][..., 512:] == 0.0)
        n_vis, n_dis, ok, dis = parity.compare_masks(mask_g[b:b + 1, heads], ref["mask"],
                                                     ref["margin"], lam32)
        assert ok, f"MLA mask: {n_dis}/{n_vis} disagree outside the tie band"
        stats = parity.compare_outputs(o_g[b:b + 1, heads], lse_g[b:b + 1, heads],
                                       ref["o"][..., :512], ref["lse"], None, dis.any(axis=-1),
                                       max_tie_rows=n_dis)
        parity.assert_within(stats, f"{w.name} seq {b}")
        worst = {k_: max(worst[k_], stats[k_]) for k_ in worst}
        skip.append(float((ref["mask"] == 1).mean()))
    sd = bl.stats_dict(st)
    assert sd["tiles_visited"] == mask_g.size
    assert sd["tiles_skipped"] == int((mask_g == 1).sum())
    print(w.name, f"Bc={Bc}", lam, {k_: f"{v_:.2e}" for k_, v_ in worst.items()}, "skip", np.round(skip, 3))
    return worst


SMALL = [
    # name, overrides, decision block (64; 128-head multiples run the tensor-core kernel)
    ("mla_4k_a12", dict(B=2, Hq=32, Lkv=4096, num_splits=4, amp=12.0, n_needles=2), 64),
    ("mla_4k_literal", dict(B=2, Hq=16, Lkv=4096, num_splits=4), 64),
    ("mla_ragged", dict(B=2, Hq=16, Lkv=3000, num_splits=5, amp=12.0), 64),
    ("mla_empty_splits", dict(B=1, Hq=16, Lkv=200, num_splits=8, amp=12.0), 64),
    ("mla_h112", dict(B=1, Hq=112, Lkv=2048, num_splits=2, amp=12.0, n_needles=2), 64),
    ("mla_h128_tc", dict(B=1, Hq=128, Lkv=2048, num_splits=2, amp=12.0, n_needles=2), 64),
    ("mla_h128_tc_ragged", dict(B=2, Hq=128, Lkv=3000, num_splits=5, amp=12.0), 64),
    ("mla_h128_tc_empty_splits", dict(B=1, Hq=128, Lkv=100, num_splits=8, amp=12.0), 64),
    ("mla_h256_tc", dict(B=1, Hq=256, Lkv=1024, num_splits=2, amp=12.0), 64),
]


@pytest.mark.parametrize("name,over,Bc", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("lam", [0.0, 1e-3, 1e-2])
def test_mla_parity_small(name, over, Bc, lam):
    run_mla(MLA.replace(name=name, **over), lam, Bc=Bc)


@pytest.mark.parametrize("cfg", ["decode_mla_64k", "decode_mla_64k_a12"])
def test_mla_full_size_sampled(cfg):
    """The benchmark's workload (B = 8, 128 heads, 64K keys, 9 splits),
    launched whole; two sequences and 32 of their heads compared with the
    oracle, the telemetry over everything."""
    w = synth.CONFIGS[cfg]
    run_mla(w, 1e-3, seqs=(0, w.B - 1), heads=slice(48, 80))


def test_mla_full_size_mma_sync_kernel():
    """The mma.sync kernel (head counts that are not multiples of 128) at the
    workload's length: 112 heads."""
    w = synth.CONFIGS["decode_mla_64k"].replace(name="decode_mla_64k_h112", B=2, Hq=112)
    run_mla(w, 1e-3, seqs=(1,), heads=slice(0, 32))


def test_mla_workload_splits_are_the_library_choice():
    """The benchmark's split count is what blasst_decode_mla_splits picks for
    this device (on a 148-SM B200)."""
    import torch
    bl = _lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = synth.CONFIGS["decode_mla_64k"]
    S = bl.blasst_decode_mla_splits(w.B, w.Hq, w.Lkv)
    assert S == bl.blasst_decode_mla_splits(w.B, w.Hq, w.Lkv, sms)
    if sms == 148:
        assert S == w.num_splits
