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
[-u/2, u/2] (standard deviation u/(2 sqrt 3)). Each gradient element is a sum
of product terms: dv = sum_r P dO (P rounded once), dk = scale sum_r dS q and
dq = scale sum_j dS k (dS rounded once, and P inside dS carries the GPU
forward's lse and its bf16 O through D = rowsum(dO * O)). The products and
sums themselves are exact or fp32 (relative 2^-24 per add), so the error of an
element is the sum of at most two roundings per term, with random signs over
many terms: about u/sqrt(3) of the element's size (measured 1.4e-3 to 4.2e-3
norm-wise, dq the largest through the shared D and lse terms). The gates take
twice the worst case of two full roundings:
  norm-wise      ||g - g_ref||_F <= 2u ||g_ref||_F           (2u = 7.8e-3)
  element-wise   max |g - g_ref| <= 4u max |g_ref|           (4u = 1.6e-2)
  per row        ||g_i - g_ref_i|| <= 4u ||g_ref_i|| + u rms_i ||g_ref_i||
                 (the floor, u times the root-mean-square row norm, covers rows
                 whose terms cancel to a small norm)
and exact zeros where nothing reaches a gradient row (a row with no kept key,
a key no row kept). A gradient scaled by 1.02, or one row off by 5 %, fails.
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
GRAD_ROW_REL = 4 * BF16_U
GRAD_ROW_FLOOR = BF16_U


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


def grad_row_excess(g, ref):
    """Per gradient row i (last axis = the head dims): the row error's norm
    over its allowance GRAD_ROW_REL ||ref_i|| + GRAD_ROW_FLOOR rms(||ref||);
    values above 1 break the per-row gate."""
    g = np.asarray(g, np.float64).reshape(-1, np.shape(g)[-1])
    ref = np.asarray(ref, np.float64).reshape(g.shape)
    rn = np.linalg.norm(ref, axis=1)
    rms = float(np.sqrt(np.mean(rn ** 2))) if rn.size else 0.0
    allow = GRAD_ROW_REL * rn + GRAD_ROW_FLOOR * rms
    en = np.linalg.norm(g - ref, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(allow > 0, en / np.where(allow > 0, allow, 1.0), np.where(en > 0, np.inf, 0.0))


def assert_grad_within(g, ref, what=""):
    e = grad_errors(g, ref)
    assert e["rel_fro"] <= GRAD_REL_FRO, f"{what}: relative Frobenius error {e['rel_fro']:.3e}"
    assert e["max_rel"] <= GRAD_MAX_REL, f"{what}: max error {e['max_rel']:.3e} of max |ref|"
    ex = grad_row_excess(g, ref)
    worst = float(ex.max()) if ex.size else 0.0
    assert worst <= 1.0, (f"{what}: row {int(ex.argmax())} error is {worst:.2f}x its allowance "
                          f"({int((ex > 1).sum())} rows over)")
    e["row_excess"] = worst
    return e
