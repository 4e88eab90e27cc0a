"""GPU parity of the pre-pass block selector (blasst_select_blocks) against
the fp64 oracle, on the same seeded inputs.

The selector's decisions are comparisons of floating-point map values (fp32
on the GPU, fp64 in the oracle), so a decision may differ where the value
sits on its threshold: a route where C_struct is within 1e-4 of tau, a
block whose map value is within 1e-5 of its row's background mean
(structured path) or of the row's cumulative threshold, or whose row crosses
gamma within 1e-5 at that value (pooled path). Everything else must agree
exactly; C_struct itself within 1e-4.
"""
import numpy as np
import pytest

import oracle
import parity
import synth

BASE = synth.CONFIGS["prefill_32k"]
CS_TOL = 1e-4
A_TOL = 1e-5


def _lib():
    from dynamic_block_sparse_tiled_b200 import build
    build.build()
    import dynamic_block_sparse_tiled_b200 as bl
    return bl


def _borderline(amap_row, kept_ref, j, structured, gamma):
    """Is block j of this oracle map row on its row's decision threshold?"""
    vis = ~np.isnan(amap_row)
    a = amap_row[vis]
    jl = int(np.flatnonzero(vis)[-1])
    v = amap_row[j]
    if structured:
        if j == 0 or j == jl or jl < 2:
            return False
        bg = amap_row[1:jl].mean()
        return abs(v - bg) <= A_TOL
    theta = amap_row[kept_ref].min()
    mass_at_v = a[a >= v].sum()
    return abs(v - theta) <= A_TOL or abs(mass_at_v - gamma) <= A_TOL


def run_select_case(w, tau, gamma):
    bl = _lib()
    inp = synth.generate(w)
    q, k = parity.to_device(inp.q), parity.to_device(inp.k)
    mask, cs = bl.select_blocks(q, k, causal=w.causal, Br=w.Br, Bc=w.Bc, tau=tau, gamma=gamma)
    assert bl.blasst_check() == 0
    ref = oracle.select(inp.q, inp.k, causal=w.causal, Br=w.Br, Bc=w.Bc, tau=tau, gamma=gamma)
    gm, gcs = mask.cpu().numpy(), cs.cpu().numpy().astype(np.float64)
    assert np.abs(gcs - ref["cstruct"]).max() <= CS_TOL, np.abs(gcs - ref["cstruct"]).max()
    n_vis = int((~np.isnan(ref["amap"])).sum())
    n_dis = 0
    for b in range(w.B):
        for hq in range(w.Hq):
            rcs = ref["cstruct"][b, hq]
            structured = rcs >= tau
            if abs(rcs - tau) <= CS_TOL:
                continue  # route on its threshold: either result is right
            diff_rows = np.flatnonzero(np.any(gm[b, hq] != ref["mask"][b, hq], axis=1))
            for t in diff_rows:
                kept_ref = ref["mask"][b, hq, t] == 0
                for j in np.flatnonzero(gm[b, hq, t] != ref["mask"][b, hq, t]):
                    n_dis += 1
                    assert _borderline(ref["amap"][b, hq, t], kept_ref, j, structured, gamma), \
                        (w.name, b, hq, t, j, ref["amap"][b, hq, t, j])
    assert n_dis <= 1e-3 * max(n_vis, 1), (n_dis, n_vis)
    sel = float((ref["mask"] == 0).sum()) / max(n_vis, 1)
    print(w.name, f"tau={tau} gamma={gamma}", "cstruct", np.round(ref["cstruct"].ravel()[:4], 4),
          f"selected {sel:.3f}", "borderline differences", n_dis)
    return ref


SMALL = [
    ("gqa_4k_literal", dict(Hq=4, Hkv=2, Lq=4096, Lkv=4096, window=512, n_needles=2), 0.2, 0.9),
    ("gqa_4k_a12_structured", dict(Hq=4, Hkv=2, Lq=4096, Lkv=4096, amp=12.0, window=512,
                                    n_needles=2), 0.0, 0.9),
    ("gqa_4k_a12_pooled", dict(Hq=4, Hkv=2, Lq=4096, Lkv=4096, amp=12.0, window=512,
                                n_needles=2), 3.0, 0.9),
    ("ragged_1000_b64", dict(Hq=2, Hkv=1, Lq=1000, Lkv=1000, Br=64, Bc=64, amp=12.0, window=256,
                             n_needles=2), 0.2, 0.8),
    ("noncausal_512x900", dict(Hq=2, Hkv=2, Lq=512, Lkv=900, causal=False, amp=12.0, window=256,
                               n_needles=2), 0.2, 0.95),
    ("d64", dict(Hq=2, Hkv=2, Lq=2048, Lkv=2048, d=64, amp=12.0, window=256, n_needles=2), 0.2, 0.9),
    ("causal_300x1000", dict(Hq=2, Hkv=1, Lq=300, Lkv=1000, amp=12.0, window=256, n_needles=2),
     0.2, 0.9),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,over,tau,gamma", SMALL, ids=[c[0] for c in SMALL])
def test_select_matches_oracle(name, over, tau, gamma):
    run_select_case(BASE.replace(name=name, **over), tau, gamma)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["prefill_32k", "prefill_32k_a12", "prefill_256k"])
def test_select_full_size(name):
    """The benchmark workloads at full size, every head and tile."""
    run_select_case(synth.CONFIGS[name], 0.2, 0.9)


@pytest.mark.gpu
def test_selected_mask_feeds_the_forward():
    """The selector's mask is a valid block_mask_in: the forward then visits
    exactly the selected pairs (skip mask 2 everywhere else)."""
    bl = _lib()
    w = BASE.replace(name="sel_fwd", Hq=4, Hkv=2, Lq=2048, Lkv=2048, amp=12.0, window=256,
                     n_needles=2)
    inp = synth.generate(w)
    q, k, v = (parity.to_device(a) for a in (inp.q, inp.k, inp.v))
    mask, _ = bl.select_blocks(q, k, causal=True, tau=0.2, gamma=0.9)
    o, lse, smask = bl.attention_prefill(q, k, v, causal=True, lam=float(np.float32(1e-3)),
                                         with_mask=True, block_mask=mask)
    assert bl.blasst_check() == 0
    m, s = mask.cpu().numpy(), smask.cpu().numpy()
    assert np.array_equal(s == 2, m != 0)
