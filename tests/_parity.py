"""Comparison helpers shared by the GPU parity tests and the smoke check.

Tolerances (the layer's stated bar): expert ids identical to the oracle except
where the oracle's fp64 margin between the last chosen and the first rejected
candidate (or between two chosen experts whose order differs, or between the
last kept and first dropped group) is below 1e-6; weights within 1e-5 * alpha;
outputs within max|y - y_oracle| / max|y_oracle| <= 2e-2 for bf16 and 1e-5 for fp32.
"""

from __future__ import annotations

import numpy as np
import torch

TIE = 1e-6
W_TOL = 1e-5
Y_TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-5}


def compare_routing(idx_gpu: torch.Tensor, w_gpu: torch.Tensor, orc: dict, b: torch.Tensor,
                    alpha: float) -> dict:
    gi = idx_gpu.cpu().numpy().astype(np.int64)
    gw = w_gpu.cpu().numpy().astype(np.float64)
    oi = orc["idx"].astype(np.int64)
    ow = orc["w"]
    sp = orc["s"] + b.detach().cpu().double().numpy()[None, :]
    N, k = oi.shape
    # smallest gap between consecutive chosen experts (order ties) per token
    chosen = np.take_along_axis(sp, oi, axis=1)
    order_gap = np.min(chosen[:, :-1] - chosen[:, 1:], axis=1) if k > 1 else np.full(N, np.inf)
    near = (orc["margin_exp"] < TIE) | (orc["margin_grp"] < TIE)
    rows_diff = np.any(gi != oi, axis=1)
    set_diff = np.array([set(gi[n]) != set(oi[n]) for n in range(N)]) if rows_diff.any() else rows_diff
    order_only = rows_diff & ~set_diff
    unexplained = (set_diff & ~near) | (order_only & ~(order_gap < TIE) & ~near)
    # weights, matched by expert id, on tokens whose chosen set agrees
    same = ~set_diff
    werr = 0.0
    if same.any():
        for n in np.nonzero(same)[0]:
            if not rows_diff[n]:
                werr = max(werr, float(np.max(np.abs(gw[n] - ow[n]))))
            else:
                od = dict(zip(oi[n], ow[n]))
                werr = max(werr, max(abs(gw[n][j] - od[gi[n][j]]) for j in range(k)))
    return {"tokens": int(N), "id_mismatch_tokens": int(rows_diff.sum()),
            "near_tie_tokens": int(near.sum()), "unexplained": int(unexplained.sum()),
            "max_w_err_over_alpha": werr / alpha, "near_tie_mask": near | (order_gap < TIE)}


def rel_err(y: np.ndarray, ref: np.ndarray) -> dict:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref))
    row_ref = np.linalg.norm(ref, axis=1)
    row_err = np.linalg.norm(y - ref, axis=1)
    return {"max_rel": float(np.max(np.abs(y - ref)) / scale) if scale > 0 else float(np.max(np.abs(y))),
            "max_row_l2_rel": float(np.max(row_err / np.maximum(row_ref, 1e-300))),
            "finite": bool(np.all(np.isfinite(y)))}
