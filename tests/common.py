"""Shared helpers of the GPU parity tests: seeded inputs, oracle references,
and the comparison rule.

Inputs come from ``synth`` (random draws only); every expected value comes
from the FP64 oracle on the same inputs; the CUDA path is reached only
through the C-ABI binding.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
import synth
from tests import scoring


def dev(bits: np.ndarray) -> torch.Tensor:
    return synth.bits_to_torch(bits).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return synth.torch_to_bits(t)


@dataclasses.dataclass
class Prepared:
    cfg: synth.Config
    qt: np.ndarray  # tiled bf16 bits [B, S, H, D]
    kt: np.ndarray
    vt: np.ndarray
    vbs: np.ndarray  # int32 [Nq] (after any override)
    idx: np.ndarray  # int32 [B, H, Nq, topk], from the oracle router
    grid_q: np.ndarray | None = None

    @property
    def nq(self):
        return len(self.vbs)


def prepare(name: str, keep_grid: bool = False, **overrides) -> Prepared:
    """Draw a configuration, tile and route it with the oracle."""
    cfg = synth.CONFIGS[name]
    if overrides:
        cfg = dataclasses.replace(cfg, **overrides)
    T, Hh, W = cfg.grid
    q, k, v = synth.grid_qkv(cfg)
    qt, kt, vt = (oracle.tile(x, T, Hh, W) for x in (q, k, v))
    vbs = oracle.cube_counts(T, Hh, W)
    idx = oracle.route(qt, kt, vbs, cfg.topk)
    if cfg.adversarial:
        ov = synth.adversarial_override(cfg, len(vbs))
        vbs = vbs.copy()
        vbs[ov.cubes] = np.minimum(vbs[ov.cubes], ov.counts)
        # re-route with the overridden counts, then force the cubes into the chosen head's lists
        idx = oracle.route(qt, kt, vbs, cfg.topk)
        forced = set(ov.cubes.tolist())
        for b in range(cfg.B):
            for i in range(len(vbs)):
                rest = [j for j in idx[b, ov.head, i].tolist() if j not in forced][: cfg.topk - len(forced)]
                idx[b, ov.head, i] = np.array(ov.cubes.tolist() + rest, np.int32)
    return Prepared(cfg, qt, kt, vt, vbs, idx, q if keep_grid else None)


def sample_items(B: int, H: int, nq: int, n: int, seed: int = 0, must=()) -> np.ndarray:
    g = np.random.default_rng(seed)
    total = B * H * nq
    pick = set(g.choice(total, size=min(n, total), replace=False).tolist())
    for (b, h, i) in must:
        pick.add((b * H + h) * nq + i)
    pick.update({0, total - 1})
    flat = np.array(sorted(pick), np.int64)
    return np.stack([flat // (H * nq), (flat // nq) % H, flat % nq], axis=1).astype(np.int32)


def gather_items(x: torch.Tensor, items: np.ndarray) -> np.ndarray:
    """x [B, S, H, D] (device) -> float32 [n, 64, D] rows of the listed items."""
    out = []
    for b, h, i in items:
        out.append(x[b, 64 * i: 64 * i + 64, h].float().cpu().numpy())
    return np.stack(out)


def near_tie_reference(gpu: np.ndarray, o64: np.ndarray, frac: float = 1.0 / 32, bound=None):
    """The bf16 reference of the pass rule: bf16_rne(oracle), except where the
    GPU value is the other bf16 neighbour of the exact value and the exact
    value lies within `frac` of an ulp (plus `bound`, the evaluation's stated
    per-element error bound, if given) of the midpoint between the two.
    There both roundings are correct results of an evaluation that meets its
    error bound, so the GPU value is taken as the reference (a 'several
    results are correct' case).  Returns (reference as float32, number of
    elements adjusted)."""
    ideal_bits = oracle.f64_to_bf16(o64)
    ideal = oracle.bf16_to_f64(ideal_bits)
    gpu_bits = oracle.f64_to_bf16(gpu.astype(np.float64))  # exact: gpu holds bf16 values
    diff = gpu_bits != ideal_bits
    ref = ideal.copy()
    n_adj = 0
    if diff.any():
        gb = gpu_bits[diff].astype(np.int64)
        ib = ideal_bits[diff].astype(np.int64)
        adjacent = (np.abs(gb - ib) == 1) & ((gb >> 15) == (ib >> 15))
        g = gpu.astype(np.float64)[diff]
        i = ideal[diff]
        window = frac * np.abs(g - i)
        if bound is not None:
            window = window + np.broadcast_to(bound, o64.shape)[diff]
        near = np.abs(o64[diff] - 0.5 * (g + i)) <= window
        ok = adjacent & near
        sub = ref[diff]
        sub[ok] = g[ok]
        ref[diff] = sub
        n_adj = int(ok.sum())
    return ref.astype(np.float32), n_adj


# Default forward mode rounds each softmax weight to bf16 before the P.V
# product (relative error <= 2^-9 per weight); the sum of weights is kept
# in fp32.  The output before its own rounding is then within
# 2^-9 * sum_u w_u |v_u| (+ fp32 accumulation, covered by a factor 2) of exact.
BF16_WEIGHT_BOUND = 2.0 ** -8


def compare(gpu_rows: np.ndarray, o64: np.ndarray, heads: np.ndarray, wabs=None) -> dict:
    """The dataset card's pass rule, per head, against bf16_rne(oracle) with the
    near-midpoint reading (gate), and against the unrounded FP64 oracle
    (reported).  wabs (oracle's sum_u w_u |v_u|) widens the near-midpoint
    window by the default mode's weight-rounding bound."""
    bound = None if wabs is None else BF16_WEIGHT_BOUND * wabs
    ref, n_adj = near_tie_reference(gpu_rows, o64, bound=bound)
    res = {"gate": _rule(gpu_rows, ref, heads), "fp64": _rule(gpu_rows, o64.astype(np.float32), heads)}
    res["gate"]["near_tie_adjusted"] = n_adj
    if wabs is None:
        # plain near-midpoint reading: such ties are rare, so many of them flag a bias
        res["gate"]["ok"] = bool(res["gate"]["ok"] and n_adj <= max(4, 1e-3 * gpu_rows.size))
    return res


def _rule(a: np.ndarray, b: np.ndarray, heads: np.ndarray) -> dict:
    finite = bool(np.isfinite(a).all())
    cos = []
    for h in np.unique(heads):
        sel = heads == h
        x = torch.from_numpy(a[sel].reshape(-1).astype(np.float32))
        y = torch.from_numpy(b[sel].reshape(-1).astype(np.float32))
        cos.append(float(torch.nn.functional.cosine_similarity(x, y, dim=0)))
    diff = np.abs(a.astype(np.float32) - b.astype(np.float32))
    r = {"finite": finite, "min_head_cos": min(cos), "max_abs": float(diff.max()), "mean_abs": float(diff.mean())}
    r["ok"] = bool(finite and r["min_head_cos"] >= scoring.MIN_COS and r["max_abs"] <= scoring.MAX_ABS
                   and r["mean_abs"] <= scoring.MEAN_ABS)
    return r


def lse_bound(qt, kt, items, sm_scale):
    """Per-row bound on the fp32 error of the log-sum-exp: the logits' dot
    products accumulate in fp32 over 128 terms (error <= ~1e-5 of the sum of
    |products|) plus a small absolute term for the fp32 sum of weights."""
    sigma = float(np.float32(sm_scale))
    out = []
    kmax = None
    for b, h, i in items:
        q = oracle.bf16_to_f64(qt[b, 64 * i: 64 * i + 64, h])  # [64, D]
        if kmax is None or kmax[0] != (b, h):
            kabs = np.abs(oracle.bf16_to_f64(kt[b, :, h]))  # [S, D]
            kmax = ((b, h), kabs.max(axis=0))
        out.append(1e-4 + 2e-5 * sigma * (np.abs(q) @ kmax[1]))
    return np.stack(out)
