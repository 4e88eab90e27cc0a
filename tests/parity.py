"""Helpers shared by the GPU parity tests: host<->device marshalling of the
synthetic inputs and the comparison rules.

Tolerances (bf16 inputs, fp32 accumulation, compared in float64 against the
fp64 oracle run with the same Br/Bc/lambda):
  O:    max |err| <= 2e-2 and mean |err| <= 2e-3
  lse:  max |err| <= 1e-3
  mask: >= 99.9 % of visited tiles agree, and every disagreement lies in the
        tie band |mu - ln(lambda)| < 1e-3 (mu = the oracle's tile margin).
Rows of a tile whose decision legitimately differs (tie band) are left out of
the O/lse comparison: both decisions are correct results of the method.

fp32 inputs (the three-product tf32 split on both contractions, relative
product error near 2^-20; scores of magnitude <= 30 in log2 units and
|v| <= 5 give O errors near 1e-4 at worst):
  O:    max |err| <= 5e-4 and mean |err| <= 5e-5
  lse:  max |err| <= 2e-4

Gradients of the backward pass (bf16 Q, K, V, dO, O; P and dS rounded to
bf16 before their products, fp32 accumulation; compared against the fp64
oracle on the same bf16 inputs). Each product term carries at most two bf16
roundings (unit roundoff u = 2^-8), and D = rowsum(dO * O) uses the bf16 O, so
the error of a gradient is near u times the size of its terms; norm-wise, with
signs mixed, about 2u/sqrt(3) = 4.5e-3 of the gradient's norm at worst:
  ||g - g_ref||_F <= 1.5e-2 ||g_ref||_F  and  max |g - g_ref| <= 5e-2 max |g_ref|,
and exact zeros where nothing reaches a gradient row (a row with no kept key,
a key no row kept).
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
GRAD_REL_FRO = 1.5e-2
GRAD_MAX_REL = 5e-2


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


def compare_outputs(o_gpu, lse_gpu, o_ref, lse_ref, row_ok=None):
    """o_*: [..., rows, d]; lse_*: [..., rows]; row_ok: bool [..., rows] rows to compare."""
    err = np.abs(o_gpu - o_ref)
    lerr = np.abs(lse_gpu - lse_ref)
    if row_ok is not None:
        err = err[row_ok]
        lerr = lerr[row_ok]
    return dict(o_max=float(err.max()) if err.size else 0.0,
                o_mean=float(err.mean()) if err.size else 0.0,
                lse_max=float(lerr.max()) if lerr.size else 0.0)


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


def assert_grad_within(g, ref, what=""):
    e = grad_errors(g, ref)
    assert e["rel_fro"] <= GRAD_REL_FRO, f"{what}: relative Frobenius error {e['rel_fro']:.3e}"
    assert e["max_rel"] <= GRAD_MAX_REL, f"{what}: max error {e['max_rel']:.3e} of max |ref|"
    return e
