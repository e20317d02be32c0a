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
    """x [B, S, H, D] (device) -> float32 [n, 64, D] rows of the listed items
    (one device-to-host copy per (b, h) run of the list)."""
    out = np.empty((len(items), 64, x.shape[-1]), np.float32)
    key, head = None, None
    for n, (b, h, i) in enumerate(items):
        if key != (b, h):
            key, head = (b, h), x[b, :, h].float().cpu().numpy()
        out[n] = head[64 * i: 64 * i + 64]
    return out


def gather_lse(lse: torch.Tensor, items: np.ndarray) -> np.ndarray:
    """lse [B, H, S] (device) -> float64 [n, 64] rows of the listed items."""
    out = np.empty((len(items), 64), np.float64)
    key, head = None, None
    for n, (b, h, i) in enumerate(items):
        if key != (b, h):
            key, head = (b, h), lse[b, h].cpu().numpy().astype(np.float64)
        out[n] = head[64 * i: 64 * i + 64]
    return out


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


def compare(gpu_rows: np.ndarray, o64: np.ndarray, heads: np.ndarray) -> dict:
    """The dataset card's pass rule, per head, against bf16_rne(oracle) with the
    1/32-ulp near-midpoint reading (gate; many such ties would flag a bias, so
    at most 1e-3 of the elements may be taken that way), and against the
    unrounded FP64 oracle (reported)."""
    ref, n_adj = near_tie_reference(gpu_rows, o64)
    res = {"gate": _rule(gpu_rows, ref, heads), "fp64": _rule(gpu_rows, o64.astype(np.float32), heads)}
    res["gate"]["near_tie_adjusted"] = n_adj
    res["gate"]["ok"] = bool(res["gate"]["ok"] and n_adj <= max(4, 1e-3 * gpu_rows.size))
    return res


# The default forward mode rounds each softmax weight to bf16 before the P.V
# product and sums the same rounded weights.  bf16 keeps 8 significant bits,
# so a rounded weight is w (1 + d) with |d| <= u = 2^-8, and the output before
# its final rounding is a weighted mean with perturbed weights: within
# u / (1 - u) * sum_u w_u |v_u - out| <= 2 u / (1 - u) * sum_u w_u |v_u| of
# exact, and 2 u / (1 - u) < 2^-7 (1 + 2^-7).
DEFAULT_WEIGHT_BOUND = 2.0 ** -7 * (1.0 + 2.0 ** -7)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


# The precise mode's weights are hi + lo, within u = 2^-17 of P: by the same argument
# as above, 2 u / (1 - u) < 2^-15.
PRECISE_WEIGHT_BOUND = 2.0 ** -15


def within_default_bound(gpu_rows: np.ndarray, o64: np.ndarray, wabs: np.ndarray, coeff: float | None = None
                         ) -> dict:
    """The default mode's stated per-element error bound (not the card's rule):
    |gpu - exact| <= half a bf16 ulp + 2^-7 * sum_u w_u |v_u| (+ 2^-20 |exact|
    for the fp32 accumulation).  coeff replaces the 2^-7 (another mode's weight
    bound, plus any accumulation term a caller states in units of sum w |v|)."""
    coeff = DEFAULT_WEIGHT_BOUND if coeff is None else coeff
    g = gpu_rows.astype(np.float64)
    err = np.abs(g - o64)
    lim = bf16_half_ulp(np.maximum(np.abs(g), np.abs(o64))) + coeff * wabs + 2.0 ** -20 * np.abs(o64)
    worst = float(np.max(err - lim))
    return {"ok": bool(np.isfinite(g).all() and worst <= 0), "worst_excess": worst,
            "max_err": float(err.max())}


def head_cosine(x: np.ndarray, y: np.ndarray) -> float:
    """Cosine of two FP32 vectors with the sums taken in FP64.  A head holds
    64 * 128 * Nq values (5.1 M at Wan 832x480); torch's fp32 cosine on the
    CPU is off by ~1e-3 at that length (cos(a, a) = 1.0018 on such a vector),
    larger than the 1e-4 the rule tests for."""
    x = x.reshape(-1).astype(np.float32).astype(np.float64)
    y = y.reshape(-1).astype(np.float32).astype(np.float64)
    den = np.sqrt(float(x @ x) * float(y @ y))
    return float(x @ y) / max(den, 1e-300)


def _rule(a: np.ndarray, b: np.ndarray, heads: np.ndarray) -> dict:
    finite = bool(np.isfinite(a).all())
    cos = []
    for h in np.unique(heads):
        sel = heads == h
        cos.append(head_cosine(a[sel], b[sel]))
    diff = np.abs(a.astype(np.float32) - b.astype(np.float32))
    r = {"finite": finite, "min_head_cos": min(cos), "max_abs": float(diff.max()), "mean_abs": float(diff.mean())}
    r["ok"] = bool(finite and r["min_head_cos"] >= scoring.MIN_COS and r["max_abs"] <= scoring.MAX_ABS
                   and r["mean_abs"] <= scoring.MEAN_ABS)
    return r


def lse_bound(qt, kt, items, sm_scale, default_mode=True):
    """Per-row bound on the fp32 error of the log-sum-exp: the logits' dot
    products accumulate in fp32 over 128 terms (error <= ~1e-5 of the sum of
    |products|) plus a small absolute term for the fp32 sum of weights.  The
    default mode's row sum adds the bf16-rounded weights (each within 2^-8 of
    its value: bf16 keeps 8 significant bits), the sum that also normalises
    its output: that adds up to -ln(1 - 2^-8) < 4e-3."""
    extra = 4e-3 if default_mode else 0.0
    sigma = float(np.float32(sm_scale))
    out = []
    kmax = None
    for b, h, i in items:
        q = oracle.bf16_to_f64(qt[b, 64 * i: 64 * i + 64, h])  # [64, D]
        if kmax is None or kmax[0] != (b, h):
            kabs = np.abs(oracle.bf16_to_f64(kt[b, :, h]))  # [S, D]
            kmax = ((b, h), kabs.max(axis=0))
        out.append(1e-4 + extra + 2e-5 * sigma * (np.abs(q) @ kmax[1]))
    return np.stack(out)
