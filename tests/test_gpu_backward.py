"""GPU parity of the backward pass (blasst_bwd) against the fp64 oracle.

The forward's decisions are held fixed. To give both sides the same decision
set without feeding anything from the CUDA path into the oracle, the decisions
come from the oracle's forward (its skip mask at the case's lambda, or a
seeded static mask); the GPU forward then runs with lambda = 0 and those
decisions as its static block mask, so its O and lse cover exactly the pairs
the oracle kept, and the GPU backward reads the same mask. One case runs the
GPU forward with the threshold itself and checks that its mask equals the
oracle's before comparing gradients.
"""
import numpy as np
import pytest

import oracle
import parity
import synth

BASE = synth.CONFIGS["prefill_32k"]


def _lib():
    from dynamic_block_sparse_tiled_b200 import build
    build.build()
    import dynamic_block_sparse_tiled_b200 as bl
    return bl


def _static_mask(w, seed, p_excl, empty_tiles=()):
    """Seeded static mask: each (tile, block) pair excluded with probability
    p_excl; the listed (b, hq, qt) tiles lose every block."""
    nQt, nKt = -(-w.Lq // w.Br), -(-w.Lkv // w.Bc)
    r = synth.draws_u64(seed, 11, 0, w.B * w.Hq * nQt * nKt).astype(np.float64) / 2.0 ** 64
    m = (r < p_excl).astype(np.uint8).reshape(w.B, w.Hq, nQt, nKt)
    for (b, hq, qt) in empty_tiles:
        m[b, hq, qt, :] = 1
    return m


def _structural_zeros(w, fmask):
    """Rows no kept pair reaches: query rows with no kept key (their dq is
    exactly 0) and keys that no query row of their GQA group keeps (their dk
    and dv are exactly 0). Returns bool [B, Hq, Lq], bool [B, Hkv, Lkv]."""
    B, Hq, Hkv, Lq, Lkv, Br, Bc = w.B, w.Hq, w.Hkv, w.Lq, w.Lkv, w.Br, w.Bc
    nQt, nKt = -(-Lq // Br), -(-Lkv // Bc)
    keep_t = np.ones((B, Hq, nQt, nKt), bool) if fmask is None else (fmask == 0)
    off = Lkv - Lq
    rows = np.arange(Lq)
    keys = np.arange(Lkv)
    q_zero = np.ones((B, Hq, Lq), bool)
    k_zero = np.ones((B, Hkv, Lkv), bool)
    for b in range(B):
        for hq in range(Hq):
            kt_of_key = keys // Bc
            for qt in range(nQt):
                r = rows[qt * Br:(qt + 1) * Br]
                kept_blocks = keep_t[b, hq, qt]
                vis = kept_blocks[kt_of_key][None, :] & (
                    (keys[None, :] <= r[:, None] + off) if w.causal else True)
                q_zero[b, hq, r] &= ~vis.any(axis=1)
                k_zero[b, hq // (Hq // Hkv)] &= ~vis.any(axis=0)
    return q_zero, k_zero


def run_bwd_case(w, lam, static=None, gpu_decisions=False):
    import torch
    bl = _lib()
    inp = synth.generate(w)
    dout = synth.grad_output(w)
    q, k, v, do = (parity.to_device(a) for a in (inp.q, inp.k, inp.v, dout))
    if lam > 0 or static is not None:
        ref_f = oracle.prefill(inp.q, inp.k, inp.v, causal=w.causal, lam=float(np.float32(lam)),
                               Br=w.Br, Bc=w.Bc, static_mask=static)
        _, _, fmask, _ = oracle.prefill_dense(ref_f)
        fmask = np.ascontiguousarray(fmask)
    else:
        fmask = None
    if gpu_decisions:
        o, lse, gmask = bl.attention_prefill(q, k, v, causal=w.causal, lam=float(np.float32(lam)),
                                             Br=w.Br, Bc=w.Bc, with_mask=True)
        assert np.array_equal(gmask.cpu().numpy(), fmask), "GPU and oracle decisions differ"
        mask_dev = gmask
    else:
        excl = None if fmask is None else torch.from_numpy((fmask != 0).astype(np.uint8)).cuda()
        o, lse, _ = bl.attention_prefill(q, k, v, causal=w.causal, lam=0.0, Br=w.Br, Bc=w.Bc,
                                         block_mask=excl)
        mask_dev = None if fmask is None else torch.from_numpy(fmask).cuda()
    dq, dk, dv = bl.attention_backward(q, k, v, o, lse, do, causal=w.causal, Br=w.Br, Bc=w.Bc,
                                       skip_mask=mask_dev)
    assert bl.blasst_check() == 0
    rq, rk, rv = oracle.backward(inp.q, inp.k, inp.v, dout, causal=w.causal, Br=w.Br, Bc=w.Bc,
                                 tile_mask=fmask)
    gq, gk, gv = (t.cpu().numpy().astype(np.float64) for t in (dq, dk, dv))
    q_zero, k_zero = _structural_zeros(w, fmask)
    scale = 1.0 / np.sqrt(w.d)
    aq, ak, av = parity.grad_abs_scales(inp.q, inp.k, inp.v, dout, causal=w.causal, scale=scale,
                                        tile_mask=fmask, Br=w.Br, Bc=w.Bc)
    errs = {}
    for name, g, r, z, a in (("dq", gq, rq, q_zero, aq), ("dk", gk, rk, k_zero, ak),
                             ("dv", gv, rv, k_zero, av)):
        assert np.all(np.isfinite(g)), f"{w.name} {name} not finite"
        errs[name] = parity.assert_grad_within(g, r, f"{w.name} {name}", abs_scale=a)
        # rows that no kept pair reaches are exact zeros on both sides
        assert np.all(r[z] == 0.0)
        assert np.all(g[z] == 0.0), f"{w.name} {name}: nonzero rows that no kept pair reaches"
    print(w.name, {k: {m: f"{x:.2e}" for m, x in e.items()} for k, e in errs.items()},
          "empty rows", int(q_zero.sum()), "unreached keys", int(k_zero.sum()))
    _gate_rejects_perturbations(w.name, (gq, rq, aq), (gk, rk, ak))
    return errs


def _gate_rejects_perturbations(what, dq_set, dk_set):
    """The gates are tight enough to see small mistakes: the GPU's dk scaled
    by 1.02 must fail, and so must one dq element moved by 4u of its
    componentwise scale (twice the allowance)."""
    gq, rq, aq = dq_set
    gk, rk, ak = dk_set
    if not np.any(rk):
        return
    with pytest.raises(AssertionError):
        parity.assert_grad_within(gk * 1.02, rk, f"{what} dk x 1.02", abs_scale=ak)
    flat = gq.reshape(-1).copy()
    a = np.asarray(aq, np.float64).reshape(-1)
    i = int(np.argmax(a))
    flat[i] += 2 * parity.GRAD_ABS_FACTOR * a[i]
    with pytest.raises(AssertionError):
        parity.assert_grad_within(flat.reshape(gq.shape), rq, f"{what} dq element", abs_scale=aq)


CASES = [
    # name, overrides, lambda, static-mask spec
    ("dense_gqa_1k", dict(Hq=4, Hkv=2, Lq=1024, Lkv=1024, window=256, n_needles=2), 0.0, None),
    ("a12_gqa_2k_lam", dict(Hq=4, Hkv=2, Lq=2048, Lkv=2048, amp=12.0, window=256, n_needles=2),
     1e-3, None),
    ("ragged_1000_br64_bc64", dict(Hq=2, Hkv=1, Lq=1000, Lkv=1000, Br=64, Bc=64, amp=12.0,
                                   window=256, n_needles=2), 1e-2, None),
    ("br64_bc128", dict(Hq=2, Hkv=2, Lq=1024, Lkv=1024, Br=64, amp=12.0, window=256, n_needles=2),
     1e-3, None),
    ("br128_bc64", dict(Hq=2, Hkv=2, Lq=1024, Lkv=1024, Bc=64, amp=12.0, window=256, n_needles=2),
     1e-3, None),
    ("noncausal_512x900", dict(Hq=2, Hkv=2, Lq=512, Lkv=900, causal=False, amp=12.0, window=256,
                               n_needles=2), 1e-3, None),
    ("causal_300x1000", dict(Hq=2, Hkv=1, Lq=300, Lkv=1000, amp=12.0, window=256, n_needles=2),
     1e-3, None),
    ("g8_512", dict(Hq=8, Hkv=1, Lq=512, Lkv=512, amp=12.0, window=128, n_needles=2), 1e-3, None),
    ("static_with_empty_rows", dict(Hq=2, Hkv=2, Lq=768, Lkv=768, amp=12.0, window=256,
                                    n_needles=2), 1e-3, (5, 0.3, ((0, 1, 2), (0, 0, 5)))),
    ("all_excluded", dict(Hq=2, Hkv=1, Lq=384, Lkv=384), 0.0, (6, 1.1, ())),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,over,lam,spec", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(name, over, lam, spec):
    w = BASE.replace(name=name, **over)
    static = None
    if spec is not None:
        seed, p_excl, empty = spec
        static = _static_mask(w, seed, p_excl, empty)
    run_bwd_case(w, lam, static=static)


@pytest.mark.gpu
def test_backward_with_the_gpu_forward_decisions():
    """End to end as a caller runs it: the GPU forward's own skip mask feeds
    the GPU backward (the seeded case has no decision in the tie band)."""
    w = BASE.replace(name="e2e_gqa_1k", Hq=4, Hkv=2, Lq=1024, Lkv=1024, amp=12.0, window=256,
                     n_needles=2)
    run_bwd_case(w, 1e-3, gpu_decisions=True)


@pytest.mark.gpu
def test_backward_all_excluded_gives_zeros():
    import torch
    bl = _lib()
    w = BASE.replace(name="zeros", Hq=2, Hkv=1, Lq=256, Lkv=256)
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    do = parity.to_device(synth.grad_output(w))
    mask = torch.ones((1, 2, 2, 2), dtype=torch.uint8, device="cuda")
    o, lse, _ = bl.attention_prefill(q, k, v, causal=True, block_mask=mask)
    dq, dk, dv = bl.attention_backward(q, k, v, o, lse, do, causal=True, skip_mask=mask)
    assert bl.blasst_check() == 0
    for t in (dq, dk, dv):
        assert int(torch.count_nonzero(t)) == 0


@pytest.mark.gpu
def test_backward_full_size_sampled():
    """The 32K prefill workload as the benchmark runs it (GPU forward at
    lambda = 1e-3, its decisions into the GPU backward), checked on outputs
    the oracle computes one by one: dq of seeded rows plus the last rows of
    one GQA group, and dk, dv of the last key block of that group's KV head
    (under the causal mask only those last rows keep those keys, so the
    oracle's dk, dv rows there are complete). Decisions of the sampled tiles
    come from the oracle's own forward and must match the GPU's."""
    bl = _lib()
    w = BASE
    lam = float(np.float32(1e-3))
    inp = synth.generate(w)
    dout = synth.grad_output(w)
    q, k, v, do = (parity.to_device(a) for a in (inp.q, inp.k, inp.v, dout))
    o, lse, gmask = bl.attention_prefill(q, k, v, causal=True, lam=lam, Br=w.Br, Bc=w.Bc,
                                         with_mask=True)
    dq, dk, dv = bl.attention_backward(q, k, v, o, lse, do, causal=True, Br=w.Br, Bc=w.Bc,
                                       skip_mask=gmask)
    assert bl.blasst_check() == 0
    nQt, nKt = -(-w.Lq // w.Br), -(-w.Lkv // w.Bc)
    g = w.Hq // w.Hkv
    hk = 3
    r = synth.draws_u64(17, 12, 0, 32)
    rows = [(int(r[2 * n]) % w.Hq) * w.Lq + int(r[2 * n + 1]) % w.Lq for n in range(16)]
    rows += [(hk * g + hh) * w.Lq + i for hh in range(g) for i in range(w.Lq - w.Bc, w.Lq)]
    rows = np.array(rows, np.int64)
    tiles = np.unique((rows // w.Lq) * nQt + (rows % w.Lq) // w.Br)
    ref_f = oracle.prefill(inp.q, inp.k, inp.v, causal=True, lam=lam, Br=w.Br, Bc=w.Bc,
                           items=tiles)
    gm = gmask.cpu().numpy().reshape(w.Hq * nQt, nKt)[tiles]
    n_vis, n_dis, ok, dis = parity.compare_masks(gm, ref_f["mask"], ref_f["margin"], lam)
    assert ok and n_dis == 0, f"{n_dis} sampled tiles decided differently"
    tm = np.full((w.B, w.Hq, nQt, nKt), 2, np.uint8)
    tm.reshape(w.Hq * nQt, nKt)[tiles] = ref_f["mask"]
    rq, rk, rv = oracle.backward_rows(inp.q, inp.k, inp.v, dout, causal=True, Br=w.Br, Bc=w.Bc,
                                      tile_mask=tm, rows=rows,
                                      kv_keys=(0, hk, w.Lkv - w.Bc, w.Lkv))
    gq = dq.reshape(-1, w.d)[rows].cpu().numpy().astype(np.float64)
    gk = dk[0, hk, w.Lkv - w.Bc:].cpu().numpy().astype(np.float64)
    gv = dv[0, hk, w.Lkv - w.Bc:].cpu().numpy().astype(np.float64)
    aq, ak, av = parity.grad_abs_scales(inp.q, inp.k, inp.v, dout, causal=True,
                                        scale=1.0 / np.sqrt(w.d), tile_mask=tm, Br=w.Br, Bc=w.Bc,
                                        rows=rows, key_range=(0, hk, w.Lkv - w.Bc, w.Lkv))
    e = {n: parity.assert_grad_within(a, b_, f"32K {n}", abs_scale=s_)
         for n, a, b_, s_ in (("dq", gq, rq, aq), ("dk", gk, rk, ak), ("dv", gv, rv, av))}
    print("32K sampled", {k_: {m: f"{x:.2e}" for m, x in v_.items()} for k_, v_ in e.items()})
    _gate_rejects_perturbations("32K sampled", (gq, rq, aq), (gk, rk, ak))
