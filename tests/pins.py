"""Pins for the CPU oracle: checks against things the oracle does not compute
itself (brute-force dense softmax attention written independently in numpy,
closed-form error bounds, exact invariants of the method, a hand-worked
example). Each ``pin_*`` raises AssertionError on failure; they take an
``oracle.Oracle`` handle so the mutation test can run them against copies of
the oracle with a planted mistake.

Method statements these pins rest on ("BLASST: Dynamic BLocked Attention
Sparsity via Softmax Thresholding", Telegram channel seeallochnaya, post 3655;
paragraphs counted after the headline):
  para 2/3 - blocked online softmax is exact once the last block is processed
             (so lambda = 0 must give dense softmax attention);
  para 2/4 - softmax is shift invariant, lazy rescaling keeps the result exact;
  para 5   - a dropped block contributes nothing, its V is never used;
  para 6   - the first block is always processed.
"""
from __future__ import annotations

import json
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# Independent brute force: full score matrix, dense softmax, in float64.
# --------------------------------------------------------------------------
def dense_attention(q, k, v, causal, scale=None, keep=None):
    """softmax(scale*Q K^T + mask) V over the full matrix. ``keep`` [B,Hq,Lq,Lkv]
    optionally removes keys per row. Returns (o, lse)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kk = np.repeat(k, g, axis=1)
    vv = np.repeat(v, g, axis=1)
    s = scale * np.einsum("bhid,bhjd->bhij", q, kk)
    allowed = np.ones((Lq, Lkv), bool)
    if causal:
        i = np.arange(Lq)[:, None]
        j = np.arange(Lkv)[None, :]
        allowed = j <= i + (Lkv - Lq)
    allowed = np.broadcast_to(allowed, s.shape)
    if keep is not None:
        allowed = allowed & keep
    s = np.where(allowed, s, -np.inf)
    m = s.max(-1, keepdims=True)
    p = np.where(allowed, np.exp(s - m), 0.0)
    lsum = p.sum(-1)
    o = np.einsum("bhij,bhjd->bhid", p, vv) / lsum[..., None]
    lse = m[..., 0] + np.log(lsum)
    return o, lse


def _dense_from(res):
    import oracle
    return oracle.prefill_dense(res)


def rand_qkv(seed, B, Hq, Hkv, Lq, Lkv, d, planted=0.0, planted_blocks=(), Bc=16):
    """fp64 inputs; optional planted direction on the query rows and on some
    key blocks (to make the threshold skip actually fire)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, Lq, d))
    k = rng.standard_normal((B, Hkv, Lkv, d))
    v = rng.standard_normal((B, Hkv, Lkv, d))
    if planted:
        u = rng.standard_normal((B, Hkv, d))
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        g = Hq // Hkv
        q += planted * np.repeat(u, g, axis=1)[:, :, None, :]
        for blk in planted_blocks:
            k[:, :, blk * Bc:(blk + 1) * Bc, :] += planted * u[:, :, None, :]
    return q, k, v


GEOMETRIES = [
    # B, Hq, Hkv, Lq, Lkv, d, causal, Br, Bc
    (1, 2, 2, 64, 64, 8, True, 16, 16),
    (2, 4, 2, 100, 100, 8, True, 32, 16),     # GQA, ragged tail
    (1, 2, 1, 37, 90, 8, True, 16, 32),       # Lq < Lkv, bottom-right causal
    (1, 3, 3, 70, 130, 64, False, 32, 64),    # non-causal, ragged
    (1, 2, 2, 256, 256, 64, True, 64, 64),
    (1, 2, 2, 200, 200, 8, True, 64, 32),     # Br > Bc
    (1, 2, 2, 1, 77, 8, False, 1, 16),        # one query row
]


def pin_lambda0_is_dense(orc):
    """lambda = 0 never skips; blocked online softmax is then exactly dense
    softmax attention (paras 2-3)."""
    for n, (B, Hq, Hkv, Lq, Lkv, d, causal, Br, Bc) in enumerate(GEOMETRIES):
        q, k, v = rand_qkv(100 + n, B, Hq, Hkv, Lq, Lkv, d, planted=2.0, planted_blocks=(0, 2), Bc=Bc)
        res = orc.prefill(q, k, v, causal=causal, lam=0.0, Br=Br, Bc=Bc)
        o, lse, mask, _ = _dense_from(res)
        o_ref, lse_ref = dense_attention(q, k, v, causal)
        assert np.all(mask != 1), "lambda=0 skipped a block"
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def _skipping_case(seed=7, d=16, L=256, Bc=16, Br=16, B=1, Hq=4, Hkv=2, causal=True, amp=6.0):
    blocks = (0, 5, 11)
    q, k, v = rand_qkv(seed, B, Hq, Hkv, L, L, d, planted=amp, planted_blocks=blocks, Bc=Bc)
    return q, k, v, dict(causal=causal, Br=Br, Bc=Bc)


def pin_first_block_always_computed(orc):
    """para 6: block 0 of every query tile is processed, whatever lambda."""
    q, k, v, kw = _skipping_case()
    for lam in (1e-3, 0.5, 0.999):
        res = orc.prefill(q, k, v, lam=lam, **kw)
        assert np.all(res["mask"][:, 0] == 0)
        assert np.any(res["mask"] == 1), "case did not skip anything"
    # decode: every split starts with a computed block
    qd = q[:, :, -1:, :]
    S, Bc = 4, 16
    out = orc.decode(qd, k, v, lam=0.5, Bc=Bc, num_splits=S)
    Ls = orc.split_len(k.shape[2], Bc, S)
    starts = [s * Ls // Bc for s in range(S) if s * Ls < k.shape[2]]
    assert np.all(out["mask"][:, :, starts] == 0)
    assert np.any(out["mask"] == 1)


def _kept_keys(res, Lq, Lkv):
    """Per-row key set implied by the oracle's own tile mask."""
    B, Hq, Br, Bc, nQt, nKt = (res[x] for x in ("B", "Hq", "Br", "Bc", "nQt", "nKt"))
    mask = res["mask"].reshape(B, Hq, nQt, nKt)
    keep = np.zeros((B, Hq, Lq, Lkv), bool)
    for qt in range(nQt):
        for kt in range(nKt):
            keep[:, :, qt * Br:(qt + 1) * Br, kt * Bc:(kt + 1) * Bc] = \
                (mask[:, :, qt, kt] == 0)[:, :, None, None]
    return keep


def pin_kept_set_equivalence(orc):
    """para 5: a skipped block contributes nothing. The output equals dense
    softmax attention restricted to the kept blocks, exactly."""
    for causal in (True, False):
        q, k, v, kw = _skipping_case(causal=causal)
        for lam in (1e-3, 1e-2, 0.2):
            res = orc.prefill(q, k, v, lam=lam, **kw)
            o, lse, mask, _ = _dense_from(res)
            assert np.any(mask == 1)
            keep = _kept_keys(res, q.shape[2], k.shape[2])
            o_ref, lse_ref = dense_attention(q, k, v, causal, keep=keep)
            np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def pin_margins_independent_of_lambda(orc):
    """A skipped block has m_blk < m_run on every row, so it would not have
    moved the running max: the per-tile margins are the same for every lambda
    in [0, 1) and the mask is [margin < ln lambda] (block 0 excepted), hence
    monotone in lambda."""
    q, k, v, kw = _skipping_case(seed=11)
    base = orc.prefill(q, k, v, lam=0.0, **kw)
    prev = None
    for lam in (1e-6, 1e-4, 1e-3, 1e-2, 0.1, 0.5):
        res = orc.prefill(q, k, v, lam=lam, **kw)
        np.testing.assert_array_equal(res["margin"], base["margin"])
        vis = res["mask"] != 2
        pred = np.zeros_like(res["mask"])
        mu = np.where(vis, base["margin"], 0.0)
        pred[vis & (mu < np.log(lam))] = 1
        pred[:, 0] = 0
        pred[~vis] = 2
        np.testing.assert_array_equal(res["mask"], pred)
        if prev is not None:
            assert np.all((prev == 1) <= (res["mask"] == 1)), "mask not monotone in lambda"
        prev = res["mask"]


def pin_running_max_is_prefix_max(orc):
    """A skipped block leaves the running max unchanged (its block max lies
    below it on every row), so the running max before block j is the prefix
    max of the visited blocks' row maxima, whatever was skipped. The margins
    mu_j = max_r (m_blk - m_run) recomputed here from that prefix max alone,
    with the oracle's conventions for rows without keys, must equal the
    oracle's (which updates m_run only on computed blocks) while it skips."""
    for causal in (True, False):
        q, k, v, kw = _skipping_case(seed=23, causal=causal)
        Br, Bc = kw["Br"], kw["Bc"]
        B, Hq, Lq, d = q.shape
        Hkv, Lkv = k.shape[1], k.shape[2]
        g = Hq // Hkv
        s = np.einsum("bhid,bhjd->bhij", q, np.repeat(k, g, axis=1)) / np.sqrt(d)
        if causal:
            s = np.where(np.arange(Lkv)[None, :] <= np.arange(Lq)[:, None] + (Lkv - Lq), s, -np.inf)
        nQt, nKt = -(-Lq // Br), -(-Lkv // Bc)
        res = orc.prefill(q, k, v, lam=1e-2, **kw)
        _, _, mask, margin = _dense_from(res)
        assert np.any(mask == 1), "case did not skip anything"
        for qt in range(nQt):
            rows = s[:, :, qt * Br:min((qt + 1) * Br, Lq), :]
            run = np.full(rows.shape[:3], -np.inf)
            for kt in range(nKt):
                vis = mask[:, :, qt, kt] != 2
                mb = rows[..., kt * Bc:min((kt + 1) * Bc, Lkv)].max(-1)
                dr = np.where(mb == -np.inf, -np.inf, np.where(run == -np.inf, np.inf, mb - run))
                mu = dr.max(-1)
                got = margin[:, :, qt, kt]
                np.testing.assert_allclose(np.where(vis, got, 0.0), np.where(vis, mu, 0.0),
                                           rtol=0, atol=1e-9)
                run = np.where(vis[..., None], np.maximum(run, mb), run)


def pin_shift_invariance(orc):
    """paras 2/4: the reference point of the exponentials does not change the
    result (lazy rescale with a large slack, or one fixed reference), and the
    skip decisions are identical because they use the exact running max."""
    q, k, v, kw = _skipping_case(seed=13)
    for lam in (0.0, 1e-2):
        a = orc.prefill(q, k, v, lam=lam, **kw)
        for mode, par in ((1, 3.0), (1, 8.0), (2, 4.0)):
            b = orc.prefill(q, k, v, lam=lam, ref_mode=mode, ref_param=par, **kw)
            np.testing.assert_array_equal(a["mask"], b["mask"])
            np.testing.assert_allclose(b["o"], a["o"], rtol=0, atol=1e-11)
            np.testing.assert_allclose(b["lse"], a["lse"], rtol=0, atol=1e-11)


def pin_permutation_invariance(orc):
    """Reordering keys inside a block (with their values) or query rows
    inside a tile (non-causal) changes nothing: the block max and the block's
    sums do not depend on the order."""
    q, k, v, kw = _skipping_case(seed=17, causal=False)
    Bc, Br = kw["Bc"], kw["Br"]
    rng = np.random.default_rng(5)
    lam = 1e-2
    a = orc.prefill(q, k, v, lam=lam, **kw)
    perm = np.concatenate([blk * Bc + rng.permutation(Bc) for blk in range(k.shape[2] // Bc)])
    b = orc.prefill(q, k[:, :, perm], v[:, :, perm], lam=lam, **kw)
    np.testing.assert_array_equal(a["mask"], b["mask"])
    np.testing.assert_allclose(b["o"], a["o"], rtol=0, atol=1e-12)
    rperm = np.concatenate([t * Br + rng.permutation(Br) for t in range(q.shape[2] // Br)])
    c = orc.prefill(q[:, :, rperm], k, v, lam=lam, **kw)
    np.testing.assert_array_equal(a["mask"], c["mask"])
    oa = _dense_from(a)[0]
    oc = _dense_from(c)[0]
    np.testing.assert_allclose(oc, oa[:, :, rperm], rtol=0, atol=1e-12)


def pin_error_bound(orc):
    """Every skipped score satisfies exp(s - m_final) <= exp(m_blk - m_run) <
    lambda and the global row max lies in a kept block, so with n_skip(r)
    skipped blocks of Bc keys: |O_lambda - O_exact| <= 2 max|v| lambda Bc
    n_skip(r) and 0 <= lse_exact - lse_lambda <= -ln(1 - lambda Bc n_skip)."""
    for causal in (True, False):
        q, k, v, kw = _skipping_case(seed=19, causal=causal, amp=5.0)
        o_ex, lse_ex = dense_attention(q, k, v, causal)
        vmax = np.abs(v).max()
        for lam in (1e-4, 1e-3, 1e-2):
            res = orc.prefill(q, k, v, lam=lam, **kw)
            o, lse, mask, _ = _dense_from(res)
            Br = kw["Br"]
            nskip = np.repeat((mask == 1).sum(-1), Br, axis=2)[:, :, : q.shape[2]]
            bound = 2 * vmax * lam * kw["Bc"] * nskip
            err = np.abs(o - o_ex).max(-1)
            assert np.all(err <= bound + 1e-12), float((err - bound).max())
            dl = lse_ex - lse
            assert np.all(dl >= -1e-12)
            frac = lam * kw["Bc"] * nskip
            ok = frac < 1
            assert np.all(dl[ok] <= -np.log1p(-frac[ok]) + 1e-12)


def pin_gqa_replication(orc):
    """Hq = g*Hkv with contiguous groups equals Hq = Hkv with each KV head
    repeated g times (masks included)."""
    q, k, v, kw = _skipping_case(seed=23, Hq=6, Hkv=2)
    for lam in (0.0, 1e-2):
        a = orc.prefill(q, k, v, lam=lam, **kw)
        b = orc.prefill(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), lam=lam, **kw)
        np.testing.assert_array_equal(a["mask"], b["mask"])
        np.testing.assert_allclose(a["o"], b["o"], rtol=0, atol=0)


def pin_decode_split_merge(orc):
    """Split-KV decode: one split equals the single-row prefill pass; at
    lambda = 0 any number of splits gives dense attention; merged partials
    equal attention over the union of the splits' keys."""
    q, k, v = rand_qkv(29, 2, 4, 2, 1, 300, 16, planted=5.0, planted_blocks=(0, 7, 12), Bc=16)
    for lam in (0.0, 1e-3, 1e-1):
        one = orc.decode(q, k, v, lam=lam, Bc=16, num_splits=1)
        pre = orc.prefill(q, k, v, causal=False, lam=lam, Br=1, Bc=16)
        np.testing.assert_array_equal(one["mask"].reshape(pre["mask"].shape), pre["mask"])
        np.testing.assert_allclose(one["o"].reshape(-1, 16), pre["o"].reshape(-1, 16), rtol=0, atol=1e-12)
        np.testing.assert_allclose(one["lse"].reshape(-1), pre["lse"].reshape(-1), rtol=0, atol=1e-12)
    o_ref, lse_ref = dense_attention(q, k, v, causal=False)
    for S in (2, 3, 5, 19, 40):
        out = orc.decode(q, k, v, lam=0.0, Bc=16, num_splits=S)
        np.testing.assert_allclose(out["o"], o_ref[:, :, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(out["lse"], lse_ref[:, :, 0], rtol=0, atol=1e-12)
        # each partial is dense attention over its own key range
        Ls = orc.split_len(300, 16, S)
        for s in range(S):
            k0, k1 = s * Ls, min((s + 1) * Ls, 300)
            if k0 >= k1:
                assert np.all(out["lse_parts"][:, :, s] == -np.inf)
                continue
            op, lp = dense_attention(q, k[:, :, k0:k1], v[:, :, k0:k1], causal=False)
            np.testing.assert_allclose(out["o_parts"][:, :, s], op[:, :, 0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(out["lse_parts"][:, :, s], lp[:, :, 0], rtol=0, atol=1e-12)
    # decode at lambda > 0: kept-set equivalence per split
    S = 4
    out = orc.decode(q, k, v, lam=1e-2, Bc=16, num_splits=S)
    assert np.any(out["mask"] == 1)
    keep = np.repeat(out["mask"] == 0, 16, axis=-1)[:, :, None, :300]
    o_ref, lse_ref = dense_attention(q, k, v, causal=False, keep=keep)
    # the merge over kept keys equals attention over all kept keys
    np.testing.assert_allclose(out["o"], o_ref[:, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse_ref[:, :, 0], rtol=0, atol=1e-12)


def pin_lse_merge(orc):
    """The log-sum-exp merge of partial softmax results over disjoint key sets
    equals the softmax result over their union; empty parts (-inf) are ignored."""
    rng = np.random.default_rng(31)
    q, k, v = rand_qkv(37, 1, 3, 3, 1, 90, 8)
    cuts = [0, 10, 10, 45, 90]
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        if a == b:
            parts_o.append(np.zeros((1, 3, 8)))
            parts_l.append(np.full((1, 3), -np.inf))
            continue
        o, l = dense_attention(q, k[:, :, a:b], v[:, :, a:b], causal=False)
        parts_o.append(o[:, :, 0])
        parts_l.append(l[:, :, 0])
    o_parts = np.stack(parts_o, axis=2)
    lse_parts = np.stack(parts_l, axis=2)
    o, lse = orc.lse_merge(o_parts, lse_parts)
    o_ref, lse_ref = dense_attention(q, k, v, causal=False)
    np.testing.assert_allclose(o, o_ref[:, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref[:, :, 0], rtol=0, atol=1e-12)
    del rng


def pin_worked_example(orc):
    """Hand-worked examples (tests/golden/skip_rule_worked_example.json): one
    query row, d = 1, scores chosen by hand, expected masks derived on paper
    from the rule, including an exact tie (a tie is computed: the test is
    strict) and a row whose scores are all negative."""
    with open(os.path.join(GOLDEN, "skip_rule_worked_example.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        lam = case["lambda"]
        keys = np.array(case["key_scores"], np.float64)
        tie = case["tie_block"]
        if tie:
            # the tie block's max equals m_run + ln(lambda) exactly in double
            keys[tie["index"] * case["Bc"]] = tie["running_max"] + np.log(lam)
        L = keys.size
        q = np.full((1, 1, 1, 1), 2.0)
        k = keys.reshape(1, 1, L, 1)
        v = np.array(case["values"], np.float64).reshape(1, 1, L, 1)
        res = orc.prefill(q, k, v, causal=False, lam=lam, Br=1, Bc=case["Bc"], scale=0.5)
        assert res["mask"][0].tolist() == case["expected_mask"], (case["name"], res["mask"][0].tolist())
        kept = np.repeat(np.array(case["expected_mask"]) == 0, case["Bc"])
        w = np.exp(keys[kept] - keys[kept].max())
        o_ref = (w * v[0, 0, kept, 0]).sum() / w.sum()
        lse_ref = keys[kept].max() + np.log(w.sum())
        assert abs(res["o"][0, 0, 0] - o_ref) < 1e-14
        assert abs(res["lse"][0, 0] - lse_ref) < 1e-14


# --------------------------------------------------------------------------
# Static block-sparse input: a caller-supplied mask excludes (query tile, KV
# block) pairs before anything is computed.
# --------------------------------------------------------------------------
def _static_mask(seed, B, Hq, nQt, nKt, frac):
    rng = np.random.default_rng(seed)
    return (rng.random((B, Hq, nQt, nKt)) < frac).astype(np.uint8)


def _allowed_from_static(smask, Br, Bc, Lq, Lkv):
    B, Hq, nQt, nKt = smask.shape
    allowed = np.ones((B, Hq, Lq, Lkv), bool)
    for qt in range(nQt):
        for kt in range(nKt):
            allowed[:, :, qt * Br:(qt + 1) * Br, kt * Bc:(kt + 1) * Bc] = \
                (smask[:, :, qt, kt] == 0)[:, :, None, None]
    return allowed


def _compare_with_empty_rows(o, lse, o_ref, lse_ref, any_key):
    """Rows with no allowed key must give O = 0 and lse = -inf; the rest
    must match the dense reference."""
    assert np.all(o[~any_key] == 0.0) and np.all(np.isneginf(lse[~any_key]))
    np.testing.assert_allclose(o[any_key], o_ref[any_key], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[any_key], lse_ref[any_key], rtol=0, atol=1e-12)


def _row_has_key(allowed, causal, Lq, Lkv):
    if causal:
        i = np.arange(Lq)[:, None]
        j = np.arange(Lkv)[None, :]
        allowed = allowed & (j <= i + (Lkv - Lq))
    return allowed.any(-1)


def pin_static_mask_is_restriction(orc):
    """With a static block mask and lambda = 0 the result is dense softmax
    attention over the allowed blocks only (the excluded pairs contribute
    nothing, as a skipped block does, para 5); an all-zero mask changes
    nothing; a tile with every block excluded gives O = 0 and lse = -inf;
    excluded pairs are reported as not visited."""
    geos = [(1, 4, 2, 200, 200, 16, True, 16, 16), (1, 2, 2, 96, 150, 8, False, 32, 16),
            (2, 2, 1, 130, 130, 8, True, 32, 32)]
    for n, (B, Hq, Hkv, Lq, Lkv, d, causal, Br, Bc) in enumerate(geos):
        q, k, v = rand_qkv(300 + n, B, Hq, Hkv, Lq, Lkv, d, planted=2.0, planted_blocks=(0, 3), Bc=Bc)
        nQt, nKt = -(-Lq // Br), -(-Lkv // Bc)
        smask = _static_mask(400 + n, B, Hq, nQt, nKt, 0.35)
        smask[0, 0, 0, 0] = 1          # the first visited block is not block 0
        smask[0, -1, nQt // 2, :] = 1  # a tile with every block excluded
        res = orc.prefill(q, k, v, causal=causal, lam=0.0, Br=Br, Bc=Bc, static_mask=smask)
        o, lse, mask, _ = _dense_from(res)
        allowed = _allowed_from_static(smask, Br, Bc, Lq, Lkv)
        with np.errstate(invalid="ignore", divide="ignore"):
            o_ref, lse_ref = dense_attention(q, k, v, causal, keep=allowed)
        _compare_with_empty_rows(o, lse, o_ref, lse_ref, _row_has_key(allowed, causal, Lq, Lkv))
        m4 = mask.reshape(B, Hq, nQt, nKt)
        assert np.all(m4[smask != 0] == 2), "an excluded pair was visited"
        assert not np.any(m4 == 1), "lambda = 0 skipped a block"
        zero = orc.prefill(q, k, v, causal=causal, lam=0.0, Br=Br, Bc=Bc,
                           static_mask=np.zeros_like(smask))
        none = orc.prefill(q, k, v, causal=causal, lam=0.0, Br=Br, Bc=Bc)
        assert np.array_equal(zero["o"], none["o"]) and np.array_equal(zero["lse"], none["lse"])
        assert np.array_equal(zero["mask"], none["mask"])


def pin_static_mask_with_threshold(orc):
    """Static mask and lambda > 0 together: the first visited block of every
    tile is computed (para 6, read as the first block the mask leaves), and
    the output is dense attention over the blocks that are both allowed and
    kept, exactly."""
    q, k, v, kw = _skipping_case()
    B, Hq, L = q.shape[0], q.shape[1], q.shape[2]
    Br, Bc = kw["Br"], kw["Bc"]
    nQt, nKt = -(-L // Br), -(-L // Bc)
    smask = _static_mask(17, B, Hq, nQt, nKt, 0.3)
    smask[:, :, 3:6, 0] = 1  # some tiles lose block 0
    for lam in (1e-3, 0.2):
        res = orc.prefill(q, k, v, lam=lam, static_mask=smask, **kw)
        o, lse, mask, _ = _dense_from(res)
        m4 = mask.reshape(B, Hq, nQt, nKt)
        assert np.any(m4 == 1), "case did not skip anything"
        for b in range(B):
            for h in range(Hq):
                for qt in range(nQt):
                    vis = np.nonzero(m4[b, h, qt] != 2)[0]
                    if vis.size:
                        assert m4[b, h, qt, vis[0]] == 0, "first visited block was skipped"
        keep = _kept_keys(res, L, L)
        with np.errstate(invalid="ignore", divide="ignore"):
            o_ref, lse_ref = dense_attention(q, k, v, kw["causal"], keep=keep)
        _compare_with_empty_rows(o, lse, o_ref, lse_ref, _row_has_key(keep, kw["causal"], L, L))
    # Worked by hand (d = 1, one query, three one-key blocks, scale 1): the
    # excluded block 0 holds the largest score, 10, which must not enter the
    # running max. Block 1 (score 0) is the first visited block, computed;
    # block 2 (score -1) has exp(-1 - 0) = 0.37 >= lambda = 0.1, computed.
    # Had block 0 raised the running max, block 2 would be dropped.
    qh = np.ones((1, 1, 1, 1))
    kh = np.array([10.0, 0.0, -1.0]).reshape(1, 1, 3, 1)
    vh = np.array([100.0, 1.0, 2.0]).reshape(1, 1, 3, 1)
    sm = np.array([1, 0, 0], np.uint8).reshape(1, 1, 1, 3)
    res = orc.prefill(qh, kh, vh, causal=False, lam=0.1, Br=1, Bc=1, scale=1.0, static_mask=sm)
    assert list(res["mask"][0]) == [2, 0, 0], res["mask"]
    w1, w2 = 1.0, np.exp(-1.0)
    assert abs(res["o"][0, 0, 0] - (w1 * 1.0 + w2 * 2.0) / (w1 + w2)) < 1e-14
    assert abs(res["lse"][0, 0] - np.log(w1 + w2)) < 1e-14


# --------------------------------------------------------------------------
# Backward pass with the forward's decisions held fixed: checked against
# central finite differences of the independent dense brute force.
# --------------------------------------------------------------------------
def _fd_grads(q, k, v, dout, causal, keep, h=1e-6):
    """dL/dq, dL/dk, dL/dv of L = sum(dout * O) by central differences."""
    def loss(qq, kk, vv):
        o, _ = dense_attention(qq, kk, vv, causal, keep=keep)
        return float(np.nansum(dout * np.nan_to_num(o)))
    grads = []
    for t_idx in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        gr = np.zeros_like(base[t_idx])
        it = np.nditer(base[t_idx], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[t_idx][idx] += h
            minus[t_idx][idx] -= h
            gr[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(gr)
    return grads


def pin_backward_matches_finite_differences(orc):
    """The gradient of softmax attention over the kept keys (a dropped block
    contributes nothing, para 5, and the decisions are held fixed) agrees with
    central differences of the dense brute force: dense, causal and
    non-causal, and with a tile mask removing some (query tile, KV block)
    pairs, including a whole tile."""
    B, Hq, Hkv, L, d, Br, Bc = 1, 2, 1, 20, 4, 4, 4
    for causal in (True, False):
        for masked in (False, True):
            rng = np.random.default_rng(21 + 2 * causal + masked)
            q, k, v = (rng.standard_normal(sh) for sh in
                       ((B, Hq, L, d), (B, Hkv, L, d), (B, Hkv, L, d)))
            dout = rng.standard_normal((B, Hq, L, d))
            nT = -(-L // Br)
            tm = None
            keep = None
            if masked:
                tm = (rng.random((B, Hq, nT, nT)) < 0.3).astype(np.uint8)
                tm[..., 0] = 0
                tm[0, 1, 2, :] = 2  # a tile with nothing kept
                keep = _allowed_from_static(tm, Br, Bc, L, L)
            dq, dk, dv = orc.backward(q, k, v, dout, causal=causal, Br=Br, Bc=Bc, tile_mask=tm)
            with np.errstate(invalid="ignore", divide="ignore"):
                fq, fk, fv = _fd_grads(q, k, v, dout, causal, keep)
            for got, ref in ((dq, fq), (dk, fk), (dv, fv)):
                np.testing.assert_allclose(got, ref, rtol=0, atol=2e-7)


def pin_backward_gqa_replication(orc):
    """Query heads sharing a KV head: dq equals the run with the KV heads
    replicated, and dk, dv are the sums over the replicas."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, L, d = 1, 4, 2, 24, 8
    q = rng.standard_normal((B, Hq, L, d))
    k = rng.standard_normal((B, Hkv, L, d))
    v = rng.standard_normal((B, Hkv, L, d))
    dout = rng.standard_normal((B, Hq, L, d))
    dq, dk, dv = orc.backward(q, k, v, dout, causal=True, Br=8, Bc=8)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dq2, dk2, dv2 = orc.backward(q, kr, vr, dout, causal=True, Br=8, Bc=8)
    np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, 2, L, d).sum(2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, 2, L, d).sum(2), rtol=0, atol=1e-12)


def pin_backward_rows_agree_with_full(orc):
    """The sampled-rows entry (used at sizes the full backward cannot reach)
    returns the full backward's dq rows, and its dk, dv of a key range are
    the full ones once every row that keeps those keys is listed."""
    rng = np.random.default_rng(8)
    B, Hq, Hkv, L, d = 2, 4, 2, 48, 8
    q = rng.standard_normal((B, Hq, L, d))
    k = rng.standard_normal((B, Hkv, L, d))
    v = rng.standard_normal((B, Hkv, L, d))
    dout = rng.standard_normal((B, Hq, L, d))
    tm = (rng.random((B, Hq, 6, 6)) < 0.3).astype(np.uint8)
    tm[..., 0] = 0
    dq, dk, dv = orc.backward(q, k, v, dout, causal=True, Br=8, Bc=8, tile_mask=tm)
    b, hk, lo, hi = 1, 1, 20, 35
    rows = [(b * Hq + hq) * L + i for hq in (2, 3) for i in range(L)]
    rq, rk, rv = orc.backward_rows(q, k, v, dout, causal=True, Br=8, Bc=8, tile_mask=tm,
                                   rows=rows, kv_keys=(b, hk, lo, hi))
    np.testing.assert_allclose(rq, dq[b, 2:4].reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(rk, dk[b, hk, lo:hi], rtol=0, atol=1e-12)
    np.testing.assert_allclose(rv, dv[b, hk, lo:hi], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Pre-pass block selector (CRISP-style) feeding the static block mask.
# --------------------------------------------------------------------------
def pin_select_worked_example(orc):
    """Hand-worked C_struct, structured-path and pooled-path masks
    (tests/golden/selector_worked_example.json): d = 1, one row per tile and
    one key per block, so the pooled map is a normalised weight prefix."""
    with open(os.path.join(GOLDEN, "selector_worked_example.json")) as f:
        fx = json.load(f)
    w = np.array(fx["weights"], np.float64)
    L = w.size
    q = np.ones((1, 1, L, 1))
    k = np.log(w).reshape(1, 1, L, 1)
    for route in ("structured", "pooled"):
        c = fx[route]
        r = orc.select(q, k, causal=True, Br=1, Bc=1, tau=c["tau"], gamma=c.get("gamma", 0.9),
                       scale=1.0)
        assert abs(r["cstruct"][0, 0] - fx["cstruct_value"]) < 1e-14
        assert r["mask"][0, 0].tolist() == c["mask"], (route, r["mask"][0, 0].tolist())
        for t in range(L):
            row = w[:t + 1] / w[:t + 1].sum()
            np.testing.assert_allclose(r["amap"][0, 0, t, :t + 1], row, rtol=0, atol=1e-15)
            assert np.all(np.isnan(r["amap"][0, 0, t, t + 1:]))


def pin_select_map_is_block_mass(orc):
    """With every query row of a tile equal and every key row of a block
    equal, the pooled map is exactly the share of dense softmax attention
    (numpy brute force over all keys) that falls in each block; non-causal,
    a ragged last tile and a ragged last block, GQA."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, Lq, Lkv, d, Br, Bc = 1, 4, 2, 44, 52, 8, 8, 16
    nQt, nKt = -(-Lq // Br), -(-Lkv // Bc)
    qt = rng.standard_normal((B, Hq, nQt, d))
    kb = rng.standard_normal((B, Hkv, nKt, d))
    q = np.repeat(qt, Br, axis=2)[:, :, :Lq]
    k = np.repeat(kb, Bc, axis=2)[:, :, :Lkv]
    r = orc.select(q, k, causal=False, Br=Br, Bc=Bc, tau=0.5, gamma=0.9)
    scale = 1.0 / np.sqrt(d)
    g = Hq // Hkv
    for hq in range(Hq):
        s = scale * q[0, hq] @ k[0, hq // g].T
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for t in range(nQt):
            mass = np.array([p[t * Br, j * Bc:(j + 1) * Bc].sum() for j in range(nKt)])
            # the pooled map weights a block by its key count only through its
            # mean: with equal key rows a block's mass is count * exp(s) / Z,
            # the map's is exp(s) / Z'; compare after dividing out the counts
            counts = np.array([min(Bc, Lkv - j * Bc) for j in range(nKt)], np.float64)
            per_key = mass / counts
            np.testing.assert_allclose(r["amap"][0, hq, t], per_key / per_key.sum(), rtol=1e-13,
                                       atol=0)


def pin_select_extremes(orc):
    """gamma = 1 keeps every visible block on the pooled path; tau = 0 puts
    every head on the structured path and tau = 3 none; a uniform map keeps
    only the first and last block on the structured path; causally invisible
    blocks are never selected."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, L, d = 1, 2, 1, 96, 8
    q = rng.standard_normal((B, Hq, L, d))
    k = rng.standard_normal((B, Hkv, L, d))
    nT = L // 16
    vis = np.tril(np.ones((nT, nT), bool))
    r = orc.select(q, k, causal=True, Br=16, Bc=16, tau=3.0, gamma=1.0)
    assert np.array_equal(r["mask"][0, 0] == 0, vis) and np.array_equal(r["mask"][0, 1] == 0, vis)
    r0 = orc.select(q, k, causal=True, Br=16, Bc=16, tau=0.0, gamma=0.5)
    assert np.all((r0["mask"] == 0) <= vis)
    for t in range(nT):
        assert r0["mask"][0, 0, t, 0] == 0 and r0["mask"][0, 0, t, t] == 0
    kz = np.zeros_like(k)  # every score equal: a uniform map
    ru = orc.select(q, kz, causal=True, Br=16, Bc=16, tau=0.0, gamma=0.5)
    for t in range(nT):
        exp_row = np.ones(nT, np.uint8)
        exp_row[0] = 0
        exp_row[t] = 0
        assert ru["mask"][0, 0, t].tolist() == exp_row.tolist()
    n = np.arange(1, nT + 1)
    cs_uniform = np.mean(np.where(n > 1, 2.0 / n, 1.0))
    assert abs(ru["cstruct"][0, 0] - cs_uniform) < 1e-14


def pin_select_permutation(orc):
    """Non-causal: permuting the key blocks other than the first and the last
    permutes the selected blocks of every tile the same way, on both paths."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, L, d, Bc = 1, 2, 1, 128, 8, 16
    q = rng.standard_normal((B, Hq, 64, d))
    k = rng.standard_normal((B, Hkv, L, d)) * 2.0
    nKt = L // Bc
    perm = np.concatenate([[0], rng.permutation(np.arange(1, nKt - 1)), [nKt - 1]])
    kp = k.reshape(B, Hkv, nKt, Bc, d)[:, :, perm].reshape(B, Hkv, L, d)
    for tau in (0.0, 3.0):
        a = orc.select(q, k, causal=False, Br=16, Bc=Bc, tau=tau, gamma=0.8)
        b = orc.select(q, kp, causal=False, Br=16, Bc=Bc, tau=tau, gamma=0.8)
        assert np.array_equal(a["mask"][..., perm], b["mask"])


ALL_PINS = [
    pin_lambda0_is_dense,
    pin_first_block_always_computed,
    pin_kept_set_equivalence,
    pin_margins_independent_of_lambda,
    pin_running_max_is_prefix_max,
    pin_shift_invariance,
    pin_permutation_invariance,
    pin_error_bound,
    pin_gqa_replication,
    pin_decode_split_merge,
    pin_lse_merge,
    pin_worked_example,
    pin_static_mask_is_restriction,
    pin_static_mask_with_threshold,
    pin_backward_matches_finite_differences,
    pin_backward_gqa_replication,
    pin_backward_rows_agree_with_full,
    pin_select_worked_example,
    pin_select_map_is_block_mass,
    pin_select_extremes,
    pin_select_permutation,
]


def synth_small(name, **kw):
    """A synthetic workload from the generator, shrunk for the CPU."""
    return synth.CONFIGS[name].replace(**kw)
