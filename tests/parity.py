"""Helpers shared by the GPU parity tests: host<->device marshalling of the
synthetic inputs and the comparison rules.

Tolerances (bf16 inputs, fp32 accumulation, compared in float64 against the
fp64 oracle run with the same Br/Bc/lambda):
  O:    max |err| <= 2e-2 and mean |err| <= 2e-3
  lse:  max |err| <= 1e-3
  mask: >= 99.9 % of visited tiles agree, and every disagreement lies in the
        tie band |mu - ln(lambda)| < 1e-3 (mu = the oracle's tile margin).
Rows of a tile whose decision legitimately differs (tie band) are left out of
the O/lse comparison: both decisions are correct results of the method. They
are counted, and their number may not exceed the disagreeing tiles' rows.

fp32 inputs (the three-product tf32 split on both contractions, relative
product error near 2^-20; scores of magnitude <= 30 in log2 units and
|v| <= 5 give O errors near 1e-4 at worst):
  O:    max |err| <= 5e-4 and mean |err| <= 5e-5
  lse:  max |err| <= 2e-4

Gradients of the backward pass (bf16 Q, K, V, dO, O; P and dS rounded to
bf16 before their products, fp32 accumulation; compared against the fp64
oracle on the same bf16 inputs). With u = 2^-8 the bf16 spacing, one
round-to-nearest-even rounding has relative error at most u/2, uniform in
[-u/2, u/2]. Every gradient element is a sum of product terms:
dv[j] = sum_r P[r,j] dO[r] (P rounded once), dk[j] = scale sum_r dS[r,j] q[r]
and dq[r] = scale sum_j dS[r,j] k[j] (dS rounded once; P inside dS is formed in
fp32 from the GPU forward's lse, D = rowsum(dO * O) from its bf16 O). The
products are exact and the fp32 sums add at most n 2^-24 relative, so each
term carries at most about two half-ulp roundings, and
  componentwise  |g - g_ref| <= 2u A,   A = the same sums over |terms|
(A_dv = sum_r P |dO|; A_dk, A_dq the same with |dS| taken as
P (|dO|.|v| + |dO|.|O|), so that the roundings inside dP - D count even where
the difference cancels; computed from the definition in float64 by
`grad_abs_scales`), the classic bound for sums of rounded terms with a
factor 2 of margin. With random signs
the errors add like a random walk, about u/sqrt(3) of the gradient (measured
1.4e-3 to 4.2e-3 norm-wise), so two global gates sit at twice that:
  norm-wise      ||g - g_ref||_F <= 2u ||g_ref||_F           (2u = 7.8e-3)
  element-wise   max |g - g_ref| <= 4u max |g_ref|           (4u = 1.6e-2)
and exact zeros where nothing reaches a gradient row (a row with no kept key,
a key no row kept). A gradient scaled by 1.02 fails the norm-wise gate; an
error above the rounding envelope anywhere fails the componentwise one.
"""
from __future__ import annotations

import numpy as np

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
MASK_AGREE = 0.999
TIE_BAND = 1e-3
FP32_TOL = dict(o_max=5e-4, o_mean=5e-5, lse_max=2e-4)
BF16_TOL = dict(o_max=O_MAX_ABS, o_mean=O_MEAN_ABS, lse_max=LSE_MAX_ABS)
BF16_U = 2.0 ** -8
GRAD_REL_FRO = 2 * BF16_U
GRAD_MAX_REL = 4 * BF16_U
GRAD_ABS_FACTOR = 2 * BF16_U


def to_device(arr, device="cuda"):
    import torch
    if arr.dtype == np.uint16:
        return torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(arr).to(device)


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def compare_masks(gpu_mask: np.ndarray, ref_mask: np.ndarray, ref_margin: np.ndarray, lam: float):
    """Returns (n_visited, n_disagree, ok, tiles_disagreeing_bool_array)."""
    gpu_mask = np.asarray(gpu_mask)
    ref_mask = np.asarray(ref_mask)
    vis_ref = ref_mask != 2
    # not-visited tiles are geometry: they must agree exactly
    assert np.array_equal(gpu_mask == 2, ref_mask == 2), "visited/not-visited pattern differs"
    dis = (gpu_mask != ref_mask) & vis_ref
    n_vis = int(vis_ref.sum())
    n_dis = int(dis.sum())
    if n_dis:
        band = np.abs(ref_margin[dis] - np.log(lam)) < TIE_BAND if lam > 0 else np.zeros(n_dis, bool)
        in_band = bool(np.all(band))
    else:
        in_band = True
    ok = in_band and (n_vis == 0 or (n_vis - n_dis) / n_vis >= MASK_AGREE)
    return n_vis, n_dis, ok, dis


def compare_outputs(o_gpu, lse_gpu, o_ref, lse_ref, row_ok=None, tie_rows=None, max_tie_rows=0):
    """o_*: [..., rows, d]; lse_*: [..., rows].
    row_ok: bool [..., rows], the rows that exist (padding and rows with no
    key are checked separately by the caller).
    tie_rows: bool [..., rows], rows of tiles whose skip decision differs from
    the oracle's inside the tie band: both decisions are correct results, so
    these rows are left out, counted, and their number must not exceed
    `max_tie_rows` (the disagreeing tiles times the rows of a tile, which the
    mask rule already bounds to 0.1 % of the visited tiles)."""
    err = np.abs(o_gpu - o_ref)
    lerr = np.abs(lse_gpu - lse_ref)
    sel = np.ones(lerr.shape, bool) if row_ok is None else np.asarray(row_ok, bool)
    n_tie = 0
    if tie_rows is not None:
        tie = sel & np.asarray(tie_rows, bool)
        n_tie = int(tie.sum())
        assert n_tie <= max_tie_rows, f"{n_tie} rows left out of the comparison (allowed {max_tie_rows})"
        sel = sel & ~tie
    err = err[sel]
    lerr = lerr[sel]
    return dict(o_max=float(err.max()) if err.size else 0.0,
                o_mean=float(err.mean()) if err.size else 0.0,
                lse_max=float(lerr.max()) if lerr.size else 0.0,
                n_rows=int(sel.sum()), n_tie_rows=n_tie)


def assert_within(stats: dict, what="", tol=None):
    tol = BF16_TOL if tol is None else tol
    assert stats["o_max"] <= tol["o_max"], f"{what} O max-abs {stats['o_max']:.3e}"
    assert stats["o_mean"] <= tol["o_mean"], f"{what} O mean-abs {stats['o_mean']:.3e}"
    assert stats["lse_max"] <= tol["lse_max"], f"{what} lse max-abs {stats['lse_max']:.3e}"


def grad_errors(g, ref) -> dict:
    """Norm-wise and max errors of a gradient against the oracle's."""
    g = np.asarray(g, np.float64)
    ref = np.asarray(ref, np.float64)
    nref = float(np.linalg.norm(ref))
    mref = float(np.abs(ref).max()) if ref.size else 0.0
    err = g - ref
    return dict(rel_fro=float(np.linalg.norm(err)) / nref if nref > 0 else float(np.linalg.norm(err)),
                max_rel=float(np.abs(err).max()) / mref if mref > 0 else float(np.abs(err).max()))


def grad_abs_scales(q, k, v, dout, *, causal, scale, tile_mask, Br, Bc, rows=None,
                    key_range=None):
    """The componentwise scales A of the gradients' error bound (the sums of
    the absolute values of each gradient element's product terms), from the
    definition of the gradient with the decisions held fixed, in float64, on
    the same inputs (bf16 as uint16 bit patterns, or fp32):
      P[r,j] = exp(scale q_r.k_j - lse_r) on kept pairs (0 elsewhere),
      lse_r = log sum over kept j of exp(scale q_r.k_j),  O = P V,
      |dS|[r,j] = P[r,j] (|dO_r|.|v_j| + |dO_r|.|O_r|)   (dS = P (dO.v - D) with
                  D = dO.O, every inner sum over absolute values),
      A_dq[r] = scale sum_j |dS|[r,j] |k_j|, A_dk[j] = scale sum_r |dS|[r,j] |q_r|,
      A_dv[j] = sum_r P[r,j] |dO_r|   (dk, dv summed over the GQA group).
    tile_mask: uint8 [B, Hq, nQt, nKt] (0 = kept) or None (every visible key).
    Without `rows`: A_dq [B, Hq, Lq, d], A_dk and A_dv [B, Hkv, Lkv, d].
    With `rows` (flat (b*Hq + h)*Lq + i): A_dq of those rows [n, d], and with
    `key_range` (b, hk, j0, j1) A_dk, A_dv of those keys [j1-j0, d] (else None).
    It is only a tolerance scale: nothing here is compared as a value."""
    if q.dtype == np.uint16:
        f = lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    else:
        f = lambda a: np.asarray(a, np.float64)
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    off = Lkv - Lq
    keys = np.arange(Lkv)
    kv_cache = {}

    def terms(b, h, rr):
        hk = h // g
        if (b, hk) not in kv_cache:
            kv_cache.clear()
            kv_cache[(b, hk)] = (f(k[b, hk]), f(v[b, hk]))
        kk, vv = kv_cache[(b, hk)]
        qq, do = f(q[b, h][rr]), f(dout[b, h][rr])
        s = scale * (qq @ kk.T)
        keep = np.ones(s.shape, bool)
        if causal:
            keep &= keys[None, :] <= rr[:, None] + off
        if tile_mask is not None:
            keep &= tile_mask[b, h][(rr // Br)[:, None], (keys // Bc)[None, :]] == 0
        s = np.where(keep, s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        mx = np.where(np.isfinite(mx), mx, 0.0)
        ex = np.where(keep, np.exp(s - mx), 0.0)
        tot = ex.sum(axis=1, keepdims=True)
        pm = np.divide(ex, tot, out=np.zeros_like(ex), where=tot > 0)
        # |dS| with every inner sum taken over absolute values: the rounding of
        # dP = dO.v and of D = dO.O (O rounded to bf16) enters before the
        # difference, so the scale is P (|dO|.|v| + |dO|.|O|), not |dS|
        eabs = np.sum(np.abs(do) * np.abs(pm @ vv), axis=1, keepdims=True)
        ds = pm * (np.abs(do) @ np.abs(vv).T + eabs)
        return qq, do, kk, pm, ds

    if rows is None:
        aq = np.zeros((B, Hq, Lq, d))
        ak = np.zeros((B, Hkv, Lkv, d))
        av = np.zeros((B, Hkv, Lkv, d))
        for b in range(B):
            for h in range(Hq):
                qq, do, kk, pm, ds = terms(b, h, np.arange(Lq))
                aq[b, h] = scale * (np.abs(ds) @ np.abs(kk))
                ak[b, h // g] += scale * (np.abs(ds).T @ np.abs(qq))
                av[b, h // g] += pm.T @ np.abs(do)
        return aq, ak, av
    rows = np.asarray(rows, np.int64)
    aq = np.zeros((len(rows), d))
    order = np.argsort(rows // Lq, kind="stable")  # group rows by head (K/V reuse)
    for n in order:
        bh, i = divmod(int(rows[n]), Lq)
        b, h = divmod(bh, Hq)
        _, _, kk, _, ds = terms(b, h, np.array([i]))
        aq[n] = scale * (np.abs(ds) @ np.abs(kk))[0]
    ak = av = None
    if key_range is not None:
        b, hk, j0, j1 = key_range
        ak = np.zeros((j1 - j0, d))
        av = np.zeros((j1 - j0, d))
        rr = np.arange(max(0, j0 - off), Lq) if causal else np.arange(Lq)
        for h in range(hk * g, hk * g + g):
            qq, do, _, pm, ds = terms(b, h, rr)
            ak += scale * (np.abs(ds[:, j0:j1]).T @ np.abs(qq))
            av += pm[:, j0:j1].T @ np.abs(do)
    return aq, ak, av


def assert_grad_within(g, ref, what="", abs_scale=None):
    e = grad_errors(g, ref)
    assert e["rel_fro"] <= GRAD_REL_FRO, f"{what}: relative Frobenius error {e['rel_fro']:.3e}"
    assert e["max_rel"] <= GRAD_MAX_REL, f"{what}: max error {e['max_rel']:.3e} of max |ref|"
    if abs_scale is not None:
        g = np.asarray(g, np.float64)
        ref = np.asarray(ref, np.float64)
        allow = GRAD_ABS_FACTOR * np.asarray(abs_scale, np.float64).reshape(g.shape)
        err = np.abs(g - ref)
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = np.where(allow > 0, err / np.where(allow > 0, allow, 1.0),
                             np.where(err > 0, np.inf, 0.0))
        worst = float(ratio.max()) if ratio.size else 0.0
        assert worst <= 1.0, (f"{what}: element {int(ratio.argmax())} error is {worst:.2f}x its "
                              f"componentwise bound ({int((ratio > 1).sum())} elements over)")
        e["abs_excess"] = worst
    return e
