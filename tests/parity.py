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
