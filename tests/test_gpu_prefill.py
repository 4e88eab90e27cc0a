"""GPU prefill kernel vs the CPU oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import parity
import synth

pytestmark = pytest.mark.gpu


def _lib():
    import dynamic_block_sparse_tiled_b200 as bl
    return bl


def run_case(w, lam, items=None, check_stats=True, static_mask=None):
    """Run GPU and oracle on workload ``w`` at threshold ``lam`` and compare
    (optionally with a static block mask, uint8 [B, Hq, nQt, nKt])."""
    import torch
    bl = _lib()
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    st = bl.new_stats()
    lam32 = float(np.float32(lam))
    sm_dev = None if static_mask is None else torch.from_numpy(static_mask).cuda()
    o, lse, mask = bl.attention_prefill(q, k, v, causal=w.causal, lam=lam32, Br=w.Br, Bc=w.Bc,
                                        with_mask=True, stats=st, block_mask=sm_dev)
    assert bl.blasst_check() == 0
    torch.cuda.synchronize()
    ref = oracle.prefill(inp.q, inp.k, inp.v, causal=w.causal, lam=lam32, Br=w.Br, Bc=w.Bc,
                         items=items, static_mask=static_mask)
    nQt, nKt = ref["nQt"], ref["nKt"]
    mask_g = mask.cpu().numpy()
    items_arr = ref["items"]
    bh = items_arr // nQt
    qt = items_arr % nQt
    b, hq = bh // w.Hq, bh % w.Hq
    # gather the GPU rows of the listed tiles on the device: [n, Br, d]
    rows = qt[:, None] * w.Br + np.arange(w.Br)[None, :]
    valid = rows < w.Lq
    rows_c = np.minimum(rows, w.Lq - 1)
    ib, ih, ir = (torch.from_numpy(np.ascontiguousarray(x)).to(o.device)
                  for x in (np.broadcast_to(b[:, None], rows.shape),
                            np.broadcast_to(hq[:, None], rows.shape), rows_c))
    o_gt = parity.bf16_tensor_to_f64(o[ib, ih, ir])
    lse_gt = lse[ib, ih, ir].cpu().numpy().astype(np.float64)
    mask_gt = mask_g.reshape(w.B * w.Hq, nQt, nKt)[bh, qt]
    n_vis, n_dis, ok, dis = parity.compare_masks(mask_gt, ref["mask"], ref["margin"], lam32)
    assert ok, f"mask: {n_dis} of {n_vis} visited tiles disagree outside the tie band"
    tie_rows = np.broadcast_to(dis.any(axis=1)[:, None], valid.shape)
    # rows left with no key at all (a static mask can do that): O = 0, lse = -inf
    empty = valid & ~tie_rows & np.isneginf(ref["lse"])
    assert np.all(np.isneginf(lse_gt[empty])) and np.all(o_gt[empty] == 0.0)
    stats = parity.compare_outputs(o_gt, lse_gt, ref["o"], ref["lse"], valid & ~empty, tie_rows,
                                   max_tie_rows=n_dis * w.Br)
    parity.assert_within(stats, w.name, parity.FP32_TOL if w.dtype == "fp32" else None)
    if check_stats and items is None:
        sd = bl.stats_dict(st)
        assert sd["tiles_visited"] == int((mask_g != 2).sum())
        assert sd["tiles_skipped"] == int((mask_g == 1).sum())
        if w.dtype != "fp32":
            # the bf16 kernel's own cycle and time spans: a plausible SM clock
            assert sd["sm_cycles"] > 0 and sd["sm_ns"] > 0
            assert 300.0 < sd["sm_cycles"] / sd["sm_ns"] * 1e3 < 2500.0
    return dict(stats, n_vis=n_vis, n_dis=n_dis, skip=float((ref["mask"] == 1).sum()) / max(n_vis, 1))


BASE = synth.CONFIGS["prefill_32k"]

SMALL = [
    # name, overrides
    ("gqa_2k_a12", dict(Hq=4, Hkv=2, Lq=2048, Lkv=2048, amp=12.0, window=256, n_needles=2)),
    ("gqa_1k_literal", dict(Hq=4, Hkv=2, Lq=1024, Lkv=1024, window=256)),
    ("ragged_1000", dict(Hq=2, Hkv=1, Lq=1000, Lkv=1000, amp=12.0, window=256, n_needles=2)),
    ("br64", dict(Hq=2, Hkv=2, Lq=1024, Lkv=1024, Br=64, amp=12.0, window=256, n_needles=2)),
    ("bc64", dict(Hq=2, Hkv=2, Lq=1024, Lkv=1024, Bc=64, amp=12.0, window=256, n_needles=2)),
    ("br64_bc64_ragged", dict(Hq=2, Hkv=1, Lq=777, Lkv=777, Br=64, Bc=64, amp=12.0, window=256, n_needles=2)),
    ("d64", dict(Hq=2, Hkv=2, Lq=1024, Lkv=1024, d=64, amp=12.0, window=256, n_needles=2)),
    ("d64_br64_bc64", dict(Hq=2, Hkv=2, Lq=640, Lkv=640, d=64, Br=64, Bc=64, amp=12.0, window=256, n_needles=2)),
    ("noncausal", dict(Hq=2, Hkv=2, Lq=512, Lkv=900, causal=False, amp=12.0, window=256, n_needles=2)),
    ("bottom_right", dict(Hq=2, Hkv=1, Lq=300, Lkv=1100, amp=12.0, window=256, n_needles=2)),
    ("batch2", dict(B=2, Hq=4, Hkv=1, Lq=768, Lkv=768, amp=12.0, window=256, n_needles=2)),
    ("one_row", dict(Hq=2, Hkv=2, Lq=1, Lkv=700, causal=False, amp=12.0, n_needles=1)),
    ("tiny_L", dict(Hq=1, Hkv=1, Lq=70, Lkv=70, amp=12.0)),
]


@pytest.mark.parametrize("name,over", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("lam", [0.0, 1e-3, 1e-2])
def test_prefill_parity_small(name, over, lam):
    w = BASE.replace(name=name, **over)
    r = run_case(w, lam)
    if lam >= 1e-3 and w.amp > 3 and w.Lkv >= 4 * w.Bc and w.causal:
        assert r["skip"] > 0.05, f"skip path not exercised: {r}"


TINY = synth.CONFIGS["tiny_fp32_1k"]

FP32 = [
    ("tiny_fp32_1k", {}),
    ("tiny_fp32_1k_a12", dict(amp=12.0, window=128, n_needles=2)),
    ("fp32_br128", dict(Br=128, amp=12.0, window=128, n_needles=2)),
    ("fp32_gqa_ragged", dict(Hq=4, Hkv=2, Lq=1000, Lkv=1000, amp=12.0, window=128, n_needles=2)),
    ("fp32_noncausal", dict(Lq=333, Lkv=1100, causal=False, amp=12.0, window=128, n_needles=2)),
    ("fp32_bottom_right", dict(Lq=200, Lkv=1000, amp=12.0, window=128, n_needles=2)),
    ("fp32_tiny_L", dict(Hq=1, Hkv=1, Lq=50, Lkv=50)),
]


@pytest.mark.parametrize("name,over", FP32, ids=[s[0] for s in FP32])
@pytest.mark.parametrize("lam", [0.0, 1e-3, 1e-2])
def test_prefill_fp32_parity(name, over, lam):
    """fp32 in / fp32 out, d = 64, Bc = 64: the small fp32 workload and
    variations of it, at fp32-level tolerances."""
    w = TINY.replace(name=name, **over)
    r = run_case(w, lam)
    if lam >= 1e-3 and w.amp > 3 and w.causal:
        assert r["skip"] > 0.05, f"skip path not exercised: {r}"


def _static_mask_for(w, seed, frac=0.4):
    """Seeded static block mask with the awkward cases forced in: tiles that
    lose block 0, and one tile that loses every block."""
    nQt, nKt = -(-w.Lq // w.Br), -(-w.Lkv // w.Bc)
    rng = np.random.default_rng(seed)
    sm = (rng.random((w.B, w.Hq, nQt, nKt)) < frac).astype(np.uint8)
    sm[:, :, 1::3, 0] = 1
    sm[0, -1, nQt // 2, :] = 1
    return sm


STATIC = [
    ("gqa_2k_a12", BASE.replace(name="s1", Hq=4, Hkv=2, Lq=2048, Lkv=2048, amp=12.0, window=256,
                                n_needles=2)),
    ("br64_ragged", BASE.replace(name="s2", Hq=2, Hkv=1, Lq=777, Lkv=777, Br=64, amp=12.0,
                                 window=256, n_needles=2)),
    ("d64_bc64", BASE.replace(name="s3", Hq=2, Hkv=2, Lq=640, Lkv=640, d=64, Br=64, Bc=64,
                              amp=12.0, window=256, n_needles=2)),
    ("noncausal", BASE.replace(name="s4", Hq=2, Hkv=2, Lq=512, Lkv=900, causal=False, amp=12.0,
                               window=256, n_needles=2)),
    ("fp32_tiny", synth.CONFIGS["tiny_fp32_1k"].replace(name="s5", amp=12.0, window=128,
                                                         n_needles=2)),
]


@pytest.mark.parametrize("name,w", STATIC, ids=[s[0] for s in STATIC])
@pytest.mark.parametrize("lam", [0.0, 1e-3])
def test_prefill_static_block_mask(name, w, lam):
    """Caller-supplied static block mask: excluded pairs are not visited, the
    first block left is computed, the rest against the oracle as usual."""
    sm = _static_mask_for(w, 11)
    r = run_case(w, lam, static_mask=sm)
    assert r["n_vis"] > 0


def test_prefill_static_mask_all_zero_is_no_mask():
    """An all-zero static mask gives the same bits as no mask."""
    import torch
    bl = _lib()
    w = BASE.replace(name="z", Hq=2, Hkv=1, Lq=1024, Lkv=1024, amp=12.0, window=256, n_needles=2)
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    zero = torch.zeros((1, 2, 8, 8), dtype=torch.uint8, device="cuda")
    a = bl.attention_prefill(q, k, v, causal=True, lam=1e-3, with_mask=True)
    b = bl.attention_prefill(q, k, v, causal=True, lam=1e-3, with_mask=True, block_mask=zero)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


@pytest.mark.parametrize("cfg", ["prefill_32k", "prefill_32k_a12"])
def test_prefill_full_size_sampled(cfg):
    """Full 32K, GQA 32/8, in the launch configuration the benchmark times;
    the oracle computes a seeded sample of query tiles (first, last, random)."""
    w = synth.CONFIGS[cfg]
    nQt = -(-w.Lq // w.Br)
    rng = np.random.default_rng(0)
    items = set()
    for bh in range(w.B * w.Hq):
        items.add(bh * nQt + 0)
        items.add(bh * nQt + nQt - 1)
    items.update(int(x) for x in rng.integers(0, w.B * w.Hq * nQt, size=24))
    items = sorted(items)[:80]
    for lam in w.lambdas:
        run_case(w, lam, items=items, check_stats=False)


def _sampled_items(w, n_heads, n_random, seed=0):
    """First and last query tile of `n_heads` seeded heads (all heads when
    there are no more) plus `n_random` seeded random tiles."""
    nQt = -(-w.Lq // w.Br)
    nbh = w.B * w.Hq
    rng = np.random.default_rng(seed)
    heads = range(nbh) if nbh <= n_heads else rng.choice(nbh, size=n_heads, replace=False)
    items = set()
    for bh in heads:
        items.add(int(bh) * nQt + 0)
        items.add(int(bh) * nQt + nQt - 1)
    items.update(int(x) for x in rng.integers(0, nbh * nQt, size=n_random))
    return sorted(items)


@pytest.mark.parametrize("cfg", ["prefill_128k", "prefill_128k_a12"])
def test_prefill_128k_sampled(cfg):
    """Full 128K, GQA 32/8, every lambda of the workload, sampled tiles (the
    last tile of a head sees all 131072 keys)."""
    w = synth.CONFIGS[cfg]
    items = _sampled_items(w, 8, 16)
    lams = w.lambdas if cfg.endswith("_a12") else (0.0, 1e-3)
    for lam in lams:
        run_case(w, lam, items=items, check_stats=False)


def test_prefill_256k_sampled_with_diffuse_heads():
    """Full 256K, 8 heads of which 4 carry no structure: sampled tiles of
    both kinds at lambda = 1e-3 (calibrated amplitude, so the structured
    heads skip and the diffuse ones keep most blocks)."""
    w = synth.CONFIGS["prefill_256k_a12"]
    nQt = -(-w.Lq // w.Br)
    items = _sampled_items(w, 8, 8)
    hs = sorted({i // nQt for i in items})
    assert any(h < 4 for h in hs) and any(h >= 4 for h in hs)
    r = run_case(w, 1e-3, items=items, check_stats=False)
    assert 0.0 < r["skip"] < 1.0, r


def test_prefill_lambda_monotone_full_size():
    """Property at full size: the set of skipped tiles grows with lambda and
    lambda = 0 skips nothing (the margins do not depend on lambda)."""
    import torch
    bl = _lib()
    w = synth.CONFIGS["prefill_32k_a12"]
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    prev = None
    for lam in (0.0, 1e-4, 1e-3, 1e-2):
        _, _, mask = bl.attention_prefill(q, k, v, causal=True, lam=lam, Br=128, Bc=128,
                                          with_mask=True)
        m = mask.cpu().numpy()
        if lam == 0.0:
            assert not np.any(m == 1)
        assert np.all(m[..., 0] == 0)
        if prev is not None:
            # allow tie-band flips: at most 0.1 % of tiles may go the other way
            assert np.mean((prev == 1) & (m != 1)) < 1e-3
        prev = m
    torch.cuda.synchronize()


def test_prefill_stats_and_skip_fraction():
    bl = _lib()
    w = BASE.replace(name="stats", Hq=4, Hkv=1, Lq=2048, Lkv=2048, amp=12.0, window=256, n_needles=2)
    r = run_case(w, 1e-3)
    assert r["skip"] > 0.3, r


def test_c_entry_point_blasst_fwd_legacy_stream():
    """The plain entry point blasst_fwd (bf16, legacy default stream) gives the same bits as blasst_fwd_ex."""
    import torch
    bl = _lib()
    w = BASE.replace(name="legacy", Hq=2, Hkv=1, Lq=512, Lkv=512, amp=12.0, window=128)
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 512), dtype=torch.float32, device="cuda")
    mask = torch.empty((1, 2, 4, 4), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    bl.blasst_fwd(q, k, v, o, lse, 1, 2, 1, 512, 512, 128, 1, float(np.float32(1e-3)), 128, 128,
                  mask)
    torch.cuda.synchronize()
    o2, lse2, mask2 = bl.attention_prefill(q, k, v, causal=True, lam=float(np.float32(1e-3)),
                                           Br=128, Bc=128, with_mask=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2) and torch.equal(mask, mask2)


def test_exp2_paths_against_float64():
    """The hardware exp2 and the FMA-pipe polynomial used for one in eight of the
    softmax exponentials, against float64 2^x over the range where both give
    normal floats (the kernel feeds x <= 8, the lazy-rescale slack)."""
    import torch
    bl = _lib()
    x = np.concatenate([np.linspace(-125.0, 64.0, 200001), np.linspace(-1, 1, 20001),
                        np.arange(-125, 65, dtype=np.float64)]).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    ym = torch.empty_like(xt)
    yp = torch.empty_like(xt)
    bl.blasst_selftest_exp2(xt, ym, yp)
    torch.cuda.synchronize()
    ref = np.exp2(x.astype(np.float64))
    rel_p = np.abs(yp.cpu().numpy().astype(np.float64) / ref - 1.0)
    rel_m = np.abs(ym.cpu().numpy().astype(np.float64) / ref - 1.0)
    assert rel_p.max() < 1.1e-4, rel_p.max()
    assert rel_m.max() < 1e-5, rel_m.max()


@pytest.mark.gpu
def test_bounded_wait_failure_path_keeps_the_context_usable():
    """A wait that nothing satisfies gives up after its bound, the kernel
    records BLASST_ETIMEOUT, blasst_check returns it once and clears it, and
    the next launch runs normally (no fault, no trap)."""
    import dynamic_block_sparse_tiled_b200 as bl
    bl.blasst_selftest_timeout(2_000_000)  # 2 ms
    assert bl.blasst_check() == bl.BLASST_ETIMEOUT
    assert bl.blasst_check() == 0
    w = BASE.replace(name="after_timeout", Hq=2, Hkv=1, Lq=512, Lkv=512, amp=12.0, window=256,
                     n_needles=2)
    run_case(w, 1e-3)
    assert bl.blasst_check() == 0
