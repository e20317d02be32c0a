"""The pass rule of the dataset card "wan2.2_production_values", section
"Scoring / loss (the rule)", restated: a candidate output passes against a
reference iff every element is finite, the smallest per-(batch, head) cosine
over the flattened (S, D) slice is at least 0.9999, and the absolute
difference has max <= 3e-2 and mean <= 1e-4.  Statistics are taken in FP32
(the card casts both sides with ``.float()``).
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

_RULE = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scoring_rule.json")))
MIN_COS = _RULE["min_head_cosine"]
MAX_ABS = _RULE["max_abs_diff"]
MEAN_ABS = _RULE["mean_abs_diff"]


def per_head_cos(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """a, b: [B, S, H, D] -> cosine per (b, h), shape [B*H]."""
    a = a.float().permute(0, 2, 1, 3).reshape(a.shape[0] * a.shape[2], -1)
    b = b.float().permute(0, 2, 1, 3).reshape(b.shape[0] * b.shape[2], -1)
    return torch.nn.functional.cosine_similarity(a, b, dim=1)


def score(o: torch.Tensor, o_ref: torch.Tensor) -> dict:
    o = o.float()
    o_ref = o_ref.float()
    finite = bool(torch.isfinite(o).all())
    cos = per_head_cos(o, o_ref)
    diff = (o - o_ref).abs()
    res = {
        "finite": finite,
        "min_head_cos": float(cos.min()),
        "max_abs": float(diff.max()),
        "mean_abs": float(diff.mean()),
    }
    res["ok"] = bool(finite and res["min_head_cos"] >= MIN_COS and res["max_abs"] <= MAX_ABS
                     and res["mean_abs"] <= MEAN_ABS)
    return res


def score_np(o: np.ndarray, o_ref: np.ndarray) -> dict:
    return score(torch.from_numpy(np.asarray(o, dtype=np.float32)),
                 torch.from_numpy(np.asarray(o_ref, dtype=np.float32)))
