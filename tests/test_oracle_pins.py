"""Pins for the FP64 oracle, against things other than the oracle itself:
the pages' printed shapes, exact rational arithmetic, textbook library
routines (torch float64 softmax / SDPA / logsumexp), closed forms and
invariants.  CPU only."""
from __future__ import annotations

import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from tests import exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_bits(x: float) -> int:
    return struct.unpack("<I", struct.pack("<f", x))[0] >> 16


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_special_values(oracle_lib):
    o = oracle_lib
    cases = [
        (1.0, 0x3F80),
        (-2.0, 0xC000),
        (1.0 + 2.0 ** -8, 0x3F80),  # tie -> even (1.0)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),  # tie -> even (1 + 2^-6)
        (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),  # above the tie; a float32 detour would give 0x3F80
        (2.0 ** -133, 0x0001),  # smallest bf16 subnormal
        (0.5 * 2.0 ** -133, 0x0000),  # tie between 0 and 2^-133 -> even
        (1.5 * 2.0 ** -133, 0x0002),  # tie -> even
        (3.3895313892515355e38, 0x7F7F),  # largest finite bf16
        (3.40e38, 0x7F80),  # rounds past the largest finite -> inf
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (math.inf, 0x7F80),
        (-math.inf, 0xFF80),
    ]
    xs = np.array([c[0] for c in cases], dtype=np.float64)
    got = o.f64_to_bf16(xs)
    for (x, want), g in zip(cases, got):
        assert int(g) == want, (x, hex(int(g)), hex(want))
    assert int(o.f64_to_bf16(np.array([math.nan]))[0]) & 0x7FFF > 0x7F80


def test_bf16_rounding_matches_library_cast_on_float32(oracle_lib):
    """On float32 inputs a single rounding step is what torch's cast does."""
    g = np.random.default_rng(1)
    x = (g.standard_normal(200000) * np.exp(g.uniform(-60, 60, 200000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle_lib.f64_to_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_bf16_rounding_matches_exact_rational(oracle_lib):
    g = np.random.default_rng(2)
    xs = g.standard_normal(3000) * np.exp(g.uniform(-30, 30, 3000))
    got = oracle_lib.f64_to_bf16(xs)
    for x, b in zip(xs, got):
        assert int(b) == exact.fraction_to_bf16_bits(Fraction(float(x)))


# ---------------------------------------------------------------- layout

def test_wan480_shapes_match_pages(oracle_lib):
    gold = json.load(open(os.path.join(GOLDEN, "wan480_shapes.json")))
    T, Hh, W = gold["latent_grid"]
    vbs = oracle_lib.cube_counts(T, Hh, W)
    assert len(vbs) == gold["num_cubes"] == int(np.prod(gold["cubes_per_axis"]))
    assert int(vbs.sum()) == gold["real_tokens"] == T * Hh * W
    assert 64 * len(vbs) == gold["S_padded"]
    assert 1.0 - gold["topk"] / len(vbs) == pytest.approx(gold["sparsity"])
    # per-axis extents 21 = 5*4+1, 30 = 7*4+2, 52 = 13*4 give these cube sizes
    vals, counts = np.unique(vbs, return_counts=True)
    assert dict(zip(vals.tolist(), counts.tolist())) == {64: 455, 32: 65, 16: 91, 8: 13}


def test_tiny_cube_counts(oracle_lib):
    vbs = oracle_lib.cube_counts(5, 6, 7)
    assert vbs.tolist() == [64, 48, 32, 24, 16, 12, 8, 6]
    assert int(vbs.sum()) == 210
    assert oracle_lib.cube_counts(24, 32, 52).tolist() == [64] * 624
    vbs720 = oracle_lib.cube_counts(21, 45, 80)
    assert len(vbs720) == 1440 and int(vbs720.sum()) == 21 * 45 * 80


@pytest.mark.parametrize("grid", [(5, 6, 7), (1, 1, 1), (4, 4, 4), (9, 3, 5), (8, 8, 1)])
def test_tile_by_brute_force(oracle_lib, grid):
    """Each cube holds the raster tokens that fall inside it, in raster order,
    followed by zero pads: derived here by filtering all tokens per cube."""
    T, Hh, W = grid
    H, D = 2, 8  # narrow rows suffice for the layout
    L = T * Hh * W
    g = np.random.default_rng(3)
    x = g.integers(1, 60000, size=(2, L, H, D)).astype(np.uint16)
    tiled = oracle_lib.tile(x, T, Hh, W)
    nct, nch, ncw = -(-T // 4), -(-Hh // 4), -(-W // 4)
    coords = [(t, h, w) for t in range(T) for h in range(Hh) for w in range(W)]  # raster order
    expect = np.zeros((2, 64 * nct * nch * ncw, H, D), dtype=np.uint16)
    for c, (ct, ch, cw) in enumerate((a, b, d) for a in range(nct) for b in range(nch) for d in range(ncw)):
        members = [r for r, (t, h, w) in enumerate(coords) if t // 4 == ct and h // 4 == ch and w // 4 == cw]
        expect[:, 64 * c: 64 * c + len(members)] = x[:, members]
    np.testing.assert_array_equal(tiled, expect)
    back = oracle_lib.untile(tiled, T, Hh, W)
    np.testing.assert_array_equal(back, x)


# ---------------------------------------------------------------- routing

def test_cube_means_exact_rational(oracle_lib):
    cfg = synth.CONFIGS["tiny"]
    T, Hh, W = cfg.grid
    q, _, _ = synth.grid_qkv(cfg)
    qt = oracle_lib.tile(q, T, Hh, W)
    vbs = oracle_lib.cube_counts(T, Hh, W)
    means = oracle_lib.cube_means(qt, vbs)
    for h in range(cfg.H):
        for c in range(len(vbs)):
            for d in range(0, 128, 7):
                want = exact.exact_cube_mean_bits(qt[0, 64 * c: 64 * c + 64, h, d], int(vbs[c]))
                assert int(means[0, h, c, d]) == want, (h, c, d)


def test_cube_means_ignore_pads_and_empty_cube(oracle_lib):
    g = np.random.default_rng(4)
    x = synth.f32_to_bf16_bits(g.standard_normal((1, 3 * 64, 1, 128)).astype(np.float32))
    vbs = np.array([64, 5, 0], dtype=np.int32)
    m1 = oracle_lib.cube_means(x, vbs)
    x2 = x.copy()
    x2[0, 64 + 5: 128] = synth.f32_to_bf16_bits(np.full((59, 1, 128), 1e30, np.float32))
    x2[0, 128:] = 0x7FC0  # NaN everywhere in the empty cube
    m2 = oracle_lib.cube_means(x2, vbs)
    np.testing.assert_array_equal(m1, m2)
    assert np.all(m1[0, 0, 2] == 0)


def test_route_planted_order(oracle_lib):
    """Constant cubes along one channel: score = a_i * b_j in closed form, so the
    selection is the topk largest (a_i > 0) or smallest (a_i < 0) b_j,
    equal b_j ordered by lower index first."""
    nq, topk = 12, 5
    b_vals = np.array([3, -1, 7, 7, 0.5, 2, -8, 7, 1, 0.25, 4, 2], dtype=np.float32)
    a_vals = np.array([1, -1, 2, -0.5, 1, 1, -3, 0.75, 1, -1, 1, 2], dtype=np.float32)
    q = np.zeros((1, 64 * nq, 1, 128), np.float32)
    k = np.zeros_like(q)
    for c in range(nq):
        q[0, 64 * c: 64 * c + 64, 0, 9] = a_vals[c]
        k[0, 64 * c: 64 * c + 64, 0, 9] = b_vals[c]
    vbs = np.full(nq, 64, np.int32)
    vbs[3] = 17
    idx, sc = oracle_lib.route(synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k), vbs, topk, want_scores=True)
    np.testing.assert_array_equal(sc[0, 0], np.outer(a_vals, b_vals).astype(np.float64))
    for i in range(nq):
        order = sorted(range(nq), key=lambda j: (-(a_vals[i] * b_vals[j]), j))
        assert idx[0, 0, i].tolist() == order[:topk], i


def test_route_exact_scores_small(oracle_lib):
    """Scores equal the exact rational dot products of the bf16 means, and the
    selection is the exact top-k (ties by lower index)."""
    cfg = synth.CONFIGS["tiny"]
    T, Hh, W = cfg.grid
    q, k, _ = synth.grid_qkv(cfg)
    qt, kt = oracle_lib.tile(q, T, Hh, W), oracle_lib.tile(k, T, Hh, W)
    vbs = oracle_lib.cube_counts(T, Hh, W)
    nq = len(vbs)
    idx, sc = oracle_lib.route(qt, kt, vbs, 3, want_scores=True)
    qc = np.array([[[exact.exact_cube_mean_bits(qt[0, 64 * c: 64 * c + 64, h, d], int(vbs[c]))
                     for d in range(128)] for c in range(nq)] for h in range(cfg.H)])
    kc = np.array([[[exact.exact_cube_mean_bits(kt[0, 64 * c: 64 * c + 64, h, d], int(vbs[c]))
                     for d in range(128)] for c in range(nq)] for h in range(cfg.H)])
    for h in range(cfg.H):
        for i in range(nq):
            ex = []
            for j in range(nq):
                s = sum((exact.bf16_bits_to_fraction(a) * exact.bf16_bits_to_fraction(b)
                         for a, b in zip(qc[h, i], kc[h, j])), Fraction(0))
                ex.append(s)
                assert abs(Fraction(sc[0, h, i, j]) - s) <= abs(s) * Fraction(1, 2 ** 45) + Fraction(1, 2 ** 100)
            order = sorted(range(nq), key=lambda j: (-ex[j], j))
            assert idx[0, h, i].tolist() == order[:3]


def test_route_wan480_lists_distinct_and_valid(oracle_lib):
    """On the Wan shape every list is a set of distinct valid cubes and the lists
    differ across heads and query cubes (the dataset card's 'not banded')."""
    cfg = synth.CONFIGS["wan480"]
    T, Hh, W = cfg.grid
    # three heads are enough for the property and keep the test short
    q, k, _ = synth.grid_qkv(dataclasses_replace(cfg, H=3))
    qt, kt = oracle_lib.tile(q, T, Hh, W), oracle_lib.tile(k, T, Hh, W)
    vbs = oracle_lib.cube_counts(T, Hh, W)
    idx = oracle_lib.route(qt, kt, vbs, cfg.topk)
    assert idx.shape == (1, 3, 624, 78)
    assert idx.min() >= 0 and idx.max() < 624
    srt = np.sort(idx, axis=-1)
    assert np.all(srt[..., 1:] != srt[..., :-1])
    rows = {tuple(r) for r in srt.reshape(-1, 78).tolist()}
    assert len(rows) > 0.99 * 3 * 624


def dataclasses_replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


# ---------------------------------------------------------------- fine forward

def _dense_reference(q, k, v, idx, vbs, sm_scale):
    """Textbook masked attention in torch float64: logits + log(multiplicity)
    for selected valid keys, -inf elsewhere, softmax, times V; plus logsumexp."""
    B, S, H, D = q.shape
    nq = S // 64
    qd = torch.from_numpy(exact_bits_to_f64(q))
    kd = torch.from_numpy(exact_bits_to_f64(k))
    vd = torch.from_numpy(exact_bits_to_f64(v))
    sigma = float(np.float32(sm_scale))
    out = torch.zeros(B, S, H, D, dtype=torch.float64)
    lse = torch.zeros(B, H, S, dtype=torch.float64)
    valid = torch.zeros(S, dtype=torch.bool)
    for c in range(nq):
        valid[64 * c: 64 * c + int(vbs[c])] = True
    for b in range(B):
        for h in range(H):
            logits = sigma * (qd[b, :, h] @ kd[b, :, h].T)  # [S, S]
            bias = torch.full((S, S), -math.inf, dtype=torch.float64)
            for i in range(nq):
                cnt = np.bincount(idx[b, h, i], minlength=nq)
                for j in np.nonzero(cnt)[0]:
                    cols = torch.arange(64 * j, 64 * j + 64)
                    cols = cols[valid[cols]]
                    bias[64 * i: 64 * i + 64, cols] = math.log(cnt[j])
            z = logits + bias
            lse[b, h] = torch.logsumexp(z, dim=1)
            p = torch.softmax(z, dim=1)
            p = torch.nan_to_num(p, nan=0.0)  # rows with no key at all
            out[b, :, h] = p @ vd[b, :, h]
    return out.numpy(), lse.numpy()


def exact_bits_to_f64(x):
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _random_case(seed, B, H, nq, topk, vbs=None, dup=False, scale=2.0):
    g = np.random.default_rng(seed)
    S = 64 * nq
    q, k, v = (synth.f32_to_bf16_bits((g.standard_normal((B, S, H, 128)) * scale).astype(np.float32))
               for _ in range(3))
    if vbs is None:
        vbs = g.integers(0, 65, size=nq).astype(np.int32)
        vbs[0] = 64
    idx = synth.random_topk(seed, B, H, nq, topk, distinct=not dup)
    return q, k, v, idx, np.asarray(vbs, np.int32)


@pytest.mark.parametrize("seed,B,H,nq,topk,dup", [(0, 1, 2, 4, 2, False), (1, 2, 1, 5, 3, True),
                                                   (2, 1, 1, 3, 3, False), (3, 1, 2, 6, 1, False)])
def test_fwd_matches_masked_dense_attention(oracle_lib, seed, B, H, nq, topk, dup):
    q, k, v, idx, vbs = _random_case(seed, B, H, nq, topk, dup=dup)
    out, lse = oracle_lib.fwd(q, k, v, idx, vbs, 1 / math.sqrt(128))
    ref, ref_lse = _dense_reference(q, k, v, idx, vbs, 1 / math.sqrt(128))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    finite = np.isfinite(ref_lse)
    assert np.array_equal(finite, np.isfinite(lse))
    np.testing.assert_allclose(lse[finite], ref_lse[finite], rtol=1e-13, atol=0)


def test_fwd_weighted_abs_v_matches_dense_weights(oracle_lib):
    """wabs = sum_u softmax_u |v_u|: the dense textbook softmax weights applied to |v|."""
    q, k, v, idx, vbs = _random_case(21, 1, 2, 4, 2, dup=True)
    items = oracle_lib.all_items(1, 2, 4)
    _, _, wabs = oracle_lib.fwd_items(q, k, v, idx, vbs, 1 / math.sqrt(128), items, want_wabs=True)
    v_abs = synth.f32_to_bf16_bits(np.abs(exact_bits_to_f64(v)).astype(np.float32))  # |bf16| is exact
    ref, _ = _dense_reference(q, k, v_abs, idx, vbs, 1 / math.sqrt(128))
    ref_items = np.stack([ref[b, 64 * i: 64 * i + 64, h] for b, h, i in items])
    np.testing.assert_allclose(wabs, ref_items, rtol=0, atol=1e-12)
    assert np.all(wabs >= 0)


def test_fwd_tiny_config_matches_masked_dense(oracle_lib):
    cfg = synth.CONFIGS["tiny"]
    T, Hh, W = cfg.grid
    q, k, v = synth.grid_qkv(cfg)
    qt, kt, vt = (oracle_lib.tile(x, T, Hh, W) for x in (q, k, v))
    vbs = oracle_lib.cube_counts(T, Hh, W)
    idx = oracle_lib.route(qt, kt, vbs, cfg.topk)
    out, lse = oracle_lib.fwd(qt, kt, vt, idx, vbs, cfg.sm_scale)
    ref, ref_lse = _dense_reference(qt, kt, vt, idx, vbs, cfg.sm_scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)


def test_fwd_full_selection_is_dense_attention(oracle_lib):
    """topk = Nq with every cube full: plain dense attention (torch SDPA)."""
    nq = 4
    q, k, v, _, _ = _random_case(5, 1, 2, nq, nq, vbs=[64] * nq)
    idx = np.broadcast_to(np.arange(nq, dtype=np.int32), (1, 2, nq, nq)).copy()
    out, _ = oracle_lib.fwd(q, k, v, idx, np.full(nq, 64, np.int32), 1 / math.sqrt(128))
    qd, kd, vd = (torch.from_numpy(exact_bits_to_f64(x)).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qd, kd, vd, scale=float(np.float32(1 / math.sqrt(128)))).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_fwd_constant_v(oracle_lib):
    q, k, v, idx, vbs = _random_case(6, 1, 2, 5, 3)
    vbs[:] = np.maximum(vbs, 1)
    v[:] = f32_bits(1.0)
    out, _ = oracle_lib.fwd(q, k, v, idx, vbs, 1 / math.sqrt(128))
    assert np.all(out == 1.0)  # sum(p * 1) / sum(p) in the same order: exactly 1
    v[:] = f32_bits(-1.625)
    out, _ = oracle_lib.fwd(q, k, v, idx, vbs, 1 / math.sqrt(128))
    np.testing.assert_allclose(out, -1.625, rtol=1e-14, atol=0)


def test_fwd_permuted_selection(oracle_lib):
    q, k, v, idx, vbs = _random_case(7, 1, 2, 6, 4)
    out, lse = oracle_lib.fwd(q, k, v, idx, vbs, 0.1)
    perm = idx[..., ::-1].copy()
    out2, lse2 = oracle_lib.fwd(q, k, v, perm, vbs, 0.1)
    # only the summation order changes: a few FP64 ulps of the largest |v|
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-14 * np.abs(out).max())
    np.testing.assert_allclose(lse2, lse, rtol=1e-15)


def test_fwd_single_token_selection(oracle_lib):
    """One selected cube with one valid token: every row is that v row exactly."""
    q, k, v, _, _ = _random_case(8, 1, 2, 4, 1)
    vbs = np.array([64, 1, 30, 64], np.int32)
    idx = np.full((1, 2, 4, 1), 1, np.int32)
    out, lse = oracle_lib.fwd(q, k, v, idx, vbs, 1 / math.sqrt(128))
    vrow = exact_bits_to_f64(v[0, 64, :, :])  # [H, D]
    for h in range(2):
        np.testing.assert_array_equal(out[0, :, h, :], np.broadcast_to(vrow[h], (256, 128)))
    qd, kd = exact_bits_to_f64(q), exact_bits_to_f64(k)
    sigma = float(np.float32(1 / math.sqrt(128)))
    np.testing.assert_allclose(lse[0, 0], sigma * (qd[0, :, 0] @ kd[0, 64, 0]), rtol=1e-13)


def test_fwd_all_masked_rows(oracle_lib):
    q, k, v, _, _ = _random_case(9, 1, 1, 3, 2)
    vbs = np.array([0, 0, 64], np.int32)
    idx = np.array([[[[0, 1], [2, 0], [1, 1]]]], np.int32)
    out, lse = oracle_lib.fwd(q, k, v, idx, vbs, 0.2)
    assert np.all(out[0, 0:64] == 0) and np.all(lse[0, 0, 0:64] == -np.inf)
    assert np.all(out[0, 128:] == 0) and np.all(lse[0, 0, 128:] == -np.inf)
    assert np.all(np.isfinite(lse[0, 0, 64:128]))


def test_fwd_nan_in_pads_is_ignored(oracle_lib):
    q, k, v, idx, vbs = _random_case(10, 1, 2, 5, 3)
    vbs[:] = [64, 10, 33, 1, 0]
    out, lse = oracle_lib.fwd(q, k, v, idx, vbs, 1 / math.sqrt(128))
    k2, v2 = k.copy(), v.copy()
    for c in range(5):
        k2[0, 64 * c + vbs[c]: 64 * c + 64] = 0x7FC0
        v2[0, 64 * c + vbs[c]: 64 * c + 64] = 0xFF80
    out2, lse2 = oracle_lib.fwd(q, k2, v2, idx, vbs, 1 / math.sqrt(128))
    np.testing.assert_array_equal(out2, out)
    np.testing.assert_array_equal(lse2, lse)


def test_fwd_items_subset_equals_full(oracle_lib):
    q, k, v, idx, vbs = _random_case(11, 2, 2, 4, 2)
    out, lse = oracle_lib.fwd(q, k, v, idx, vbs, 0.3)
    items = np.array([[1, 0, 3], [0, 1, 0], [1, 1, 2]], np.int32)
    o, l = oracle_lib.fwd_items(q, k, v, idx, vbs, 0.3, items)
    for n, (b, h, i) in enumerate(items):
        np.testing.assert_array_equal(o[n], out[b, 64 * i: 64 * i + 64, h])
        np.testing.assert_array_equal(l[n], lse[b, h, 64 * i: 64 * i + 64])


def test_oracle_rejects_bad_arguments(oracle_lib):
    q, k, v, idx, vbs = _random_case(12, 1, 1, 3, 2)
    bad = idx.copy()
    bad[0, 0, 0, 0] = 3
    with pytest.raises(ValueError):
        oracle_lib.fwd(q, k, v, bad, vbs, 0.1)
    with pytest.raises(ValueError):
        oracle_lib.fwd(q, k, v, idx, np.array([65, 1, 1], np.int32), 0.1)


# ---------------------------------------------------------------- comparator

def test_near_tie_reference_accepts_only_midpoint_flips():
    """The parity comparator accepts the other bf16 neighbour only when the exact
    value sits within 1/32 ulp of the midpoint; any other difference stays."""
    from tests import common

    ulp = 2.0 ** -5  # bf16 spacing in [4, 8)
    exact = np.array([4.0 + 0.5 * ulp + 1e-4 * ulp,   # just above the midpoint: ideal = 4 + ulp
                      4.0 + 0.5 * ulp + 0.2 * ulp,    # well above: ideal = 4 + ulp
                      4.0 + 0.5 * ulp + 1e-4 * ulp])  # just above, but the GPU is 2 ulps off
    gpu = np.array([4.0, 4.0, 4.0 - ulp], dtype=np.float32)
    ref, n = common.near_tie_reference(gpu, exact)
    assert n == 1
    assert ref[0] == 4.0 and ref[1] == np.float32(4.0 + ulp) and ref[2] == np.float32(4.0 + ulp)
    # a stated error bound widens the window by exactly that bound, never to a 2-ulp flip
    ref, n = common.near_tie_reference(gpu, exact, bound=np.array([0.25 * ulp, 0.25 * ulp, 10 * ulp]))
    assert n == 2
    assert ref[0] == 4.0 and ref[1] == 4.0 and ref[2] == np.float32(4.0 + ulp)


# ---------------------------------------------------------------- tile plan

def _check_pairing(plan, nq):
    """Every cube of every (b, h) in exactly one tile; tiles ordered by their
    smaller cube; a single cube only as the last leftover of an odd count."""
    for row in plan:
        seen = []
        for a, b in row:
            assert b == -1 or a < b
            seen += [a] + ([b] if b >= 0 else [])
        assert sorted(seen) == list(range(nq))
        firsts = [a for a, _ in row]
        assert firsts == sorted(firsts)
        assert sum(1 for _, b in row if b < 0) == nq % 2


def test_plan_hand_example(oracle_lib):
    """Five cubes: 0 and 2 share both cubes, 1 and 3 share both, 4 shares one
    with 0 and 2.  Round 1 pairs (0,2) and (1,3) by mutual choice; 4 has no
    unpaired candidate left and is the odd one out."""
    idx = np.array([[[[0, 1], [2, 3], [0, 1], [2, 3], [4, 0]]]], np.int32)
    assert oracle_lib.plan(idx).tolist() == [[[0, 2], [1, 3], [4, -1]]]


def test_plan_refills_candidates_of_leftovers(oracle_lib):
    """Sixteen hubs in eight twin pairs (lists: the core cubes 0-7 plus one cube
    of their own) and four cubes 16-19 that each hold two core cubes and one
    shared cube: 16 and 18 share cube 16, 17 and 19 share cube 17.  Every hub
    overlaps a leftover cube by 2 and its twin by 9, so round 1 pairs the twins
    and the four others, whose 8 candidates are all hubs, are left unpaired.
    The refill recomputes their candidates among themselves and pairs them by
    overlap, (16, 18) and (17, 19), not in index order (16, 17), (18, 19)."""
    nq, topk = 20, 10
    idx = np.empty((1, 1, nq, topk), np.int32)
    core = list(range(8))
    for h in range(16):
        lst = core + [8 + h // 2]
        idx[0, 0, h] = lst + lst[:topk - len(lst)]  # duplicates are ignored
    for c, own in ((16, [0, 1, 16]), (17, [4, 5, 17]), (18, [2, 3, 16]), (19, [6, 7, 17])):
        idx[0, 0, c] = (own * topk)[:topk]
    plan = oracle_lib.plan(idx)
    _check_pairing(plan, nq)
    assert plan[0].tolist() == [[2 * p, 2 * p + 1] for p in range(8)] + [[16, 18], [17, 19]]


def test_plan_pairs_planted_twins(oracle_lib):
    """Cubes planted in pairs with identical lists (and lists that share
    nothing across pairs) are paired with their twin, whatever their order."""
    g = np.random.default_rng(8)
    nq, topk = 12, 2
    perm = g.permutation(nq)
    idx = np.empty((1, 1, nq, topk), np.int32)
    for p in range(nq // 2):
        a, b = perm[2 * p], perm[2 * p + 1]
        idx[0, 0, a] = idx[0, 0, b] = [2 * p, 2 * p + 1]
    plan = oracle_lib.plan(idx)
    _check_pairing(plan, nq)
    want = sorted(tuple(sorted((perm[2 * p], perm[2 * p + 1]))) for p in range(nq // 2))
    assert sorted(tuple(t) for t in plan[0].tolist()) == want


@pytest.mark.parametrize("nq,topk,seed", [(7, 3, 0), (10, 4, 1), (33, 5, 2), (64, 8, 3)])
def test_plan_is_a_pairing_and_beats_index_order(oracle_lib, nq, topk, seed):
    """Random lists: the plan pairs every cube once, and its total overlap is at
    least that of pairing cubes in index order (the greedy choice never loses
    to an arbitrary pairing by more than a factor 2; on these inputs it wins)."""
    idx = synth.random_topk(seed, 2, 2, nq, topk)
    plan = oracle_lib.plan(idx)
    _check_pairing(plan, nq)
    for bh in range(4):
        L = idx.reshape(4, nq, topk)[bh]
        ov = lambda a, b: len(set(L[a].tolist()) & set(L[b].tolist()))
        planned = sum(ov(a, b) for a, b in plan[bh] if b >= 0)
        ordered = sum(ov(2 * p, 2 * p + 1) for p in range(nq // 2))
        assert planned >= ordered


def _plan_restated(lists, nq, ncand=8, rounds=64, refills=64):
    """The pairing rule as stated (proposal rounds over the ncand best candidates,
    refills among the unpaired cubes, leftovers in index order), written from the
    statement with sets and an overlap matrix."""
    sets = [set(int(x) for x in row if 0 <= x < nq) for row in lists]
    ov = np.array([[len(a & b) for b in sets] for a in sets])
    partner = [-1] * nq
    for refill in range(refills + 1):
        free = [i for i in range(nq) if partner[i] < 0]
        if refill > 0 and len(free) < 2:
            break
        cand = {}
        for i in free:
            others = [j for j in free if j != i]
            cand[i] = sorted(others, key=lambda j: (-ov[i, j], j))[:ncand]
        formed = False
        for _ in range(rounds):
            prop = {i: next((j for j in cand[i] if partner[j] < 0), -1) for i in range(nq) if partner[i] < 0}
            pairs = [(i, j) for i, j in prop.items() if j >= 0 and prop.get(j) == i and i < j]
            if not pairs:
                break
            for i, j in pairs:
                partner[i], partner[j] = j, i
            formed = True
        if not formed:
            break
    left = [i for i in range(nq) if partner[i] < 0]
    for a in range(0, len(left) - 1, 2):
        partner[left[a]], partner[left[a + 1]] = left[a + 1], left[a]
    odd = left[-1] if len(left) % 2 else -1
    return [[i, -1 if i == odd else partner[i]] for i in range(nq) if partner[i] > i or i == odd]


@pytest.mark.parametrize("seed", range(12))
def test_plan_matches_the_restated_rule(oracle_lib, seed):
    """Random lists (with duplicates and out-of-range ids half the time): the
    oracle's plan equals the rule restated with sets."""
    g = np.random.default_rng(500 + seed)
    nq = int(g.integers(2, 48))
    topk = int(g.integers(1, min(9, nq) + 1))
    idx = synth.random_topk(500 + seed, 1, 2, nq, topk, distinct=bool(seed % 2))
    if seed % 3 == 0:
        idx[0, 0, 0, 0] = nq + 3  # ignored by the rule
    plan = oracle_lib.plan(idx).tolist()
    for bh in range(2):
        assert plan[bh] == _plan_restated(idx[0, bh], nq)


def test_plan_ignores_duplicates_and_bad_ids(oracle_lib):
    """Overlaps count distinct cubes; ids outside [0, Nq) are ignored."""
    idx = np.array([[[[1, 1, 2], [1, 2, 9], [3, 3, 3], [-1, 3, 0]]]], np.int32)
    # distinct sets: {1,2}, {1,2}, {3}, {3,0}: 0-1 overlap 2, 2-3 overlap 1
    assert oracle_lib.plan(idx).tolist() == [[[0, 1], [2, 3]]]


# ------------------------------------------------------------------ proxy compensation
# TensorRT-LLM PR #7 (FlashInfer PR "support proxy-compensated block-sparse attention") and
# TensorRT-Edge-LLM "Video Sparse Attention Runner": omitted blocks contribute through their
# mean key and summed value, the denominator weighted by the tokens each proxy stands for.

def _proxy_case(seed, nq=6, H=2, topk=2, vbs=None, scale=1.5):
    g = np.random.default_rng(seed)
    x = [synth.f32_to_bf16_bits((g.standard_normal((1, 64 * nq, H, 128)) * scale).astype(np.float32)) for _ in range(3)]
    if vbs is None:
        vbs = g.integers(0, 65, size=nq).astype(np.int32)
        vbs[0] = 64
    vbs = np.asarray(vbs, np.int32)
    idx = synth.random_topk(seed, 1, H, nq, topk)
    return x[0], x[1], x[2], vbs, idx


def test_cube_sums_exact(oracle_lib):
    """Sums of small integers are exact in FP64 and in bf16 (below 256); pads and empty cubes add nothing."""
    g = np.random.default_rng(4)
    v = g.integers(-3, 4, size=(1, 64 * 3, 2, 128)).astype(np.float32)
    vbs = np.array([64, 17, 0], np.int32)
    vb = synth.f32_to_bf16_bits(v)
    got = oracle_lib.bf16_to_f64(oracle_lib.cube_sums(vb, vbs))
    for c in range(3):
        want = v[0, 64 * c: 64 * c + vbs[c]].sum(axis=0)  # [H, D]
        np.testing.assert_array_equal(got[0, :, c], want)


def test_proxy_equals_softmax_over_exact_and_proxy_keys(oracle_lib):
    """The same result from a library softmax over the exact tokens and one key per
    omitted cube (its mean key, log-weight log vbs[j], value vc_j / vbs[j])."""
    q, k, v, vbs, idx = _proxy_case(11)
    nq, H = len(vbs), q.shape[2]
    kc, vc = oracle_lib.cube_means(k, vbs), oracle_lib.cube_sums(v, vbs)
    sigma = float(np.float32(0.125))
    items = oracle_lib.all_items(1, H, nq)
    out, lse = oracle_lib.fwd_proxy_items(q, k, v, kc, vc, idx, vbs, 0.125, items)
    f = lambda a: torch.from_numpy(oracle_lib.bf16_to_f64(a))
    Q, K, V, KC, VC = f(q)[0], f(k)[0], f(v)[0], f(kc)[0], f(vc)[0]
    for n, (b, h, i) in enumerate(items):
        sel = idx[0, h, i].tolist()
        toks = [64 * j + u for j in sel for u in range(vbs[j])]
        om = [j for j in range(nq) if j not in sel and vbs[j] > 0]
        qs = Q[64 * i: 64 * i + 64, h]
        logits = torch.cat([sigma * qs @ K[toks, h].T,
                            sigma * qs @ KC[h, om].T + torch.log(torch.tensor(vbs[om], dtype=torch.float64))], dim=1)
        vals = torch.cat([V[toks, h], VC[h, om] / torch.tensor(vbs[om], dtype=torch.float64)[:, None]], dim=0)
        want = torch.softmax(logits, dim=1) @ vals
        assert np.allclose(out[n], want.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[n], torch.logsumexp(logits, dim=1).numpy(), rtol=0, atol=1e-12)


def test_proxy_with_every_cube_selected_is_the_plain_forward(oracle_lib):
    q, k, v, vbs, _ = _proxy_case(12, nq=5, topk=5)
    idx = np.broadcast_to(np.arange(5, dtype=np.int32), (1, 2, 5, 5)).copy()
    kc, vc = oracle_lib.cube_means(k, vbs), oracle_lib.cube_sums(v, vbs)
    items = oracle_lib.all_items(1, 2, 5)
    o1, l1 = oracle_lib.fwd_proxy_items(q, k, v, kc, vc, idx, vbs, 0.1, items)
    o2, l2 = oracle_lib.fwd_items(q, k, v, idx, vbs, 0.1, items)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_proxy_is_exact_when_every_cube_is_constant(oracle_lib):
    """When the keys of each cube are all equal (its mean is that key) and the value
    sums are exact, proxies reproduce the omitted cubes exactly: the result equals
    dense attention over every cube, for any selection."""
    g = np.random.default_rng(13)
    nq, H = 6, 2
    vbs = np.array([64, 40, 1, 64, 17, 33], np.int32)
    q = synth.f32_to_bf16_bits((g.standard_normal((1, 64 * nq, H, 128))).astype(np.float32))
    kcube = g.standard_normal((nq, H, 128)).astype(np.float32)
    k = synth.f32_to_bf16_bits(np.repeat(kcube, 64, axis=0)[None])
    v = synth.f32_to_bf16_bits(g.integers(-2, 3, size=(1, 64 * nq, H, 128)).astype(np.float32))
    kc, vc = oracle_lib.cube_means(k, vbs), oracle_lib.cube_sums(v, vbs)
    items = oracle_lib.all_items(1, H, nq)
    dense = np.broadcast_to(np.arange(nq, dtype=np.int32), (1, H, nq, nq)).copy()
    o_dense, l_dense = oracle_lib.fwd_items(q, k, v, dense, vbs, 0.2, items)
    for topk in (1, 3):
        idx = synth.random_topk(topk, 1, H, nq, topk)
        o, l = oracle_lib.fwd_proxy_items(q, k, v, kc, vc, idx, vbs, 0.2, items)
        assert np.allclose(o, o_dense, rtol=0, atol=1e-12)
        assert np.allclose(l, l_dense, rtol=0, atol=1e-12)


def test_proxy_uniform_logits_closed_form(oracle_lib):
    """q = 0: every weight is equal, so out = (sum of the selected values + the omitted
    cubes' summed values) / (selected tokens + omitted tokens) and lse = log of that count."""
    _, k, v, vbs, idx = _proxy_case(14, nq=7, topk=3)
    q = np.zeros_like(k)
    kc, vc = oracle_lib.cube_means(k, vbs), oracle_lib.cube_sums(v, vbs)
    items = oracle_lib.all_items(1, 2, 7)
    out, lse = oracle_lib.fwd_proxy_items(q, k, v, kc, vc, idx, vbs, 0.3, items)
    V, VC = oracle_lib.bf16_to_f64(v)[0], oracle_lib.bf16_to_f64(vc)[0]
    for n, (b, h, i) in enumerate(items):
        sel = idx[0, h, i].tolist()
        om = [j for j in range(7) if j not in sel and vbs[j] > 0]
        num = sum(V[64 * j: 64 * j + vbs[j], h].sum(axis=0) for j in sel) + sum(VC[h, j] for j in om)
        cnt = sum(int(vbs[j]) for j in sel) + sum(int(vbs[j]) for j in om)
        assert np.allclose(out[n], np.broadcast_to(num / cnt, (64, 128)), rtol=0, atol=1e-13)
        assert np.allclose(lse[n], math.log(cnt), rtol=0, atol=1e-13)


# ------------------------------------------------------------------ route formats
# TensorRT-LLM PR #7 (the embedded FlashInfer PR, "Bitmask format"): canonical BSR rows and
# packed UInt32 exact-block bitmaps per (batch, head, query block); padding bits in the last
# word are ignored.

def _bsr_case(seed, nq=7, H=2, max_len=5, dup=True):
    g = np.random.default_rng(seed)
    x = [synth.f32_to_bf16_bits((g.standard_normal((1, 64 * nq, H, 128)) * 1.5).astype(np.float32))
         for _ in range(3)]
    vbs = g.integers(0, 65, size=nq).astype(np.int32)
    vbs[0] = 64
    indptr, indices = [0], []
    for r in range(H * nq):
        n = int(g.integers(0, max_len + 1)) if r % 5 else 0  # some rows empty
        row = g.choice(nq, size=n, replace=dup).tolist()
        indices.extend(row)
        indptr.append(len(indices))
    return x[0], x[1], x[2], vbs, np.asarray(indptr, np.int32), np.asarray(indices, np.int32)


def test_bsr_rows_equal_softmax_over_listed_tokens(oracle_lib):
    """Variable-length rows, repeats and empty rows: the softmax over exactly the listed
    tokens (a cube named twice counts twice), written out with torch in float64."""
    q, k, v, vbs, indptr, indices = _bsr_case(21)
    nq, H = len(vbs), q.shape[2]
    items = oracle_lib.all_items(1, H, nq)
    out, lse, wabs = oracle_lib.fwd_bsr_items(q, k, v, indptr, indices, vbs, 0.125, items, want_wabs=True)
    sigma = float(np.float32(0.125))
    f = lambda a: torch.from_numpy(oracle_lib.bf16_to_f64(a))
    Q, K, V = f(q)[0], f(k)[0], f(v)[0]
    for n, (b, h, i) in enumerate(items):
        r = h * nq + i
        toks = [64 * j + u for j in indices[indptr[r]:indptr[r + 1]].tolist() for u in range(vbs[j])]
        if not toks:
            assert np.all(out[n] == 0.0) and np.all(np.isneginf(lse[n])) and np.all(wabs[n] == 0.0)
            continue
        logits = sigma * Q[64 * i: 64 * i + 64, h] @ K[toks, h].T
        w = torch.softmax(logits, dim=1)
        assert np.allclose(out[n], (w @ V[toks, h]).numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[n], torch.logsumexp(logits, dim=1).numpy(), rtol=0, atol=1e-12)
        assert np.allclose(wabs[n], (w @ V[toks, h].abs()).numpy(), rtol=0, atol=1e-12)


def test_bsr_rows_with_proxies_equal_softmax_with_proxy_keys(oracle_lib):
    """Proxies over the cubes a row does not list: the softmax over the listed tokens and
    one key per other cube with valid tokens (mean key, log-weight log vbs[j], value
    vc_j / vbs[j])."""
    q, k, v, vbs, indptr, indices = _bsr_case(22, dup=False)
    nq, H = len(vbs), q.shape[2]
    kc, vc = oracle_lib.cube_means(k, vbs), oracle_lib.cube_sums(v, vbs)
    items = oracle_lib.all_items(1, H, nq)
    out, lse = oracle_lib.fwd_bsr_items(q, k, v, indptr, indices, vbs, 0.25, items, kc=kc, vc=vc)
    sigma = 0.25
    f = lambda a: torch.from_numpy(oracle_lib.bf16_to_f64(a))
    Q, K, V, KC, VC = f(q)[0], f(k)[0], f(v)[0], f(kc)[0], f(vc)[0]
    for n, (b, h, i) in enumerate(items):
        r = h * nq + i
        sel = indices[indptr[r]:indptr[r + 1]].tolist()
        toks = [64 * j + u for j in sel for u in range(vbs[j])]
        om = [j for j in range(nq) if j not in sel and vbs[j] > 0]
        qs = Q[64 * i: 64 * i + 64, h]
        logits = torch.cat([sigma * qs @ K[toks, h].T,
                            sigma * qs @ KC[h, om].T + torch.log(torch.tensor(vbs[om], dtype=torch.float64))], dim=1)
        vals = torch.cat([V[toks, h], VC[h, om] / torch.tensor(vbs[om], dtype=torch.float64)[:, None]], dim=0)
        assert np.allclose(out[n], (torch.softmax(logits, dim=1) @ vals).numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[n], torch.logsumexp(logits, dim=1).numpy(), rtol=0, atol=1e-12)


def test_bitmask_bit_order_and_padding(oracle_lib):
    """A hand-worked 37-cube row: bit c % 32 of word c / 32 selects cube c, and the
    27 bits past cube 36 in the last word are ignored."""
    nq = 37
    mask = np.zeros((1, 1, nq, 2), np.uint32)
    mask[0, 0, 3] = [(1 << 0) | (1 << 5) | (1 << 31), (1 << 0) | (1 << 4) | np.uint32(0xFFFFFFE0)]
    indptr, indices = oracle_lib.bitmask_to_bsr(mask, nq)
    assert indptr[3] == 0 and indptr[4] == 5 and indptr[-1] == 5
    assert indices.tolist() == [0, 5, 31, 32, 36]
    back = oracle_lib.bsr_to_bitmask(indptr, indices, 1, 1, nq)
    assert back[0, 0, 3].tolist() == [(1 << 0) | (1 << 5) | (1 << 31), (1 << 0) | (1 << 4)]
    assert int(back.sum()) == int(back[0, 0, 3].sum())


def test_route_formats_describe_the_same_selection(oracle_lib):
    """Distinct lists in ascending order, their BSR rows and their bitmaps give the same
    forward; the BSR rows of fixed lists are the lists in order."""
    q, k, v, vbs, _ = _proxy_case(23, nq=6, topk=3)
    idx = np.sort(synth.random_topk(23, 1, 2, 6, 3), axis=-1).astype(np.int32)
    indptr, indices = oracle_lib.lists_to_bsr(idx)
    assert indptr.tolist() == list(range(0, 3 * 12 + 1, 3)) and indices.tolist() == idx.reshape(-1).tolist()
    ip2, ix2 = oracle_lib.bitmask_to_bsr(oracle_lib.bsr_to_bitmask(indptr, indices, 1, 2, 6), 6)
    assert ip2.tolist() == indptr.tolist() and ix2.tolist() == indices.tolist()
    items = oracle_lib.all_items(1, 2, 6)
    o1, l1 = oracle_lib.fwd_items(q, k, v, idx, vbs, 0.1, items)
    o2, l2 = oracle_lib.fwd_bsr_items(q, k, v, indptr, indices, vbs, 0.1, items)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ------------------------------------------------------------------ short-KV cross-attention
# maxdiffusion PR #509: every query row over every key of a short text key/value sequence,
# one exact softmax, no mask.

def _cross_case(seed, nblk=3, S_kv=77, H=2, scale=1.5):
    g = np.random.default_rng(seed)
    q = synth.f32_to_bf16_bits((g.standard_normal((1, 64 * nblk, H, 128)) * scale).astype(np.float32))
    k = synth.f32_to_bf16_bits((g.standard_normal((1, S_kv, H, 128)) * scale).astype(np.float32))
    v = synth.f32_to_bf16_bits(g.standard_normal((1, S_kv, H, 128)).astype(np.float32))
    return q, k, v


def test_cross_over_its_own_sequence_is_the_dense_fine_forward(oracle_lib):
    """K/V the query sequence itself (S_kv = S) and every cube listed with 64 valid
    tokens: the fine-stage forward, already pinned to dense attention."""
    q, k, v = _cross_case(50, nblk=4, S_kv=256)
    items = oracle_lib.all_items(1, 2, 4)
    o1, l1 = oracle_lib.cross_items(q, k, v, 0.125, items)
    dense = np.broadcast_to(np.arange(4, dtype=np.int32), (1, 2, 4, 4)).copy()
    o2, l2 = oracle_lib.fwd_items(q, k, v, dense, np.full(4, 64, np.int32), 0.125, items)
    assert np.allclose(o1, o2, rtol=0, atol=1e-13) and np.allclose(l1, l2, rtol=0, atol=1e-13)


def test_cross_closed_forms(oracle_lib):
    """q = 0: the mean of v and lse = log S_kv; one key: its value and its logit."""
    q, k, v = _cross_case(51, S_kv=77)
    items = oracle_lib.all_items(1, 2, 3)
    out, lse, wabs = oracle_lib.cross_items(np.zeros_like(q), k, v, 0.3, items, want_wabs=True)
    V = oracle_lib.bf16_to_f64(v)[0]
    for n, (b, h, i) in enumerate(items):
        assert np.allclose(out[n], np.broadcast_to(V[:, h].mean(axis=0), (64, 128)), rtol=0, atol=1e-13)
        assert np.allclose(lse[n], math.log(77), rtol=0, atol=1e-13)
        assert np.allclose(wabs[n], np.broadcast_to(np.abs(V[:, h]).mean(axis=0), (64, 128)), rtol=0, atol=1e-13)
    q, k, v = _cross_case(52, S_kv=1)
    out, lse = oracle_lib.cross_items(q, k, v, 0.25, items)
    Q, K, V = (oracle_lib.bf16_to_f64(a)[0] for a in (q, k, v))
    for n, (b, h, i) in enumerate(items):
        assert np.array_equal(out[n], np.broadcast_to(V[0, h], (64, 128)))
        assert np.allclose(lse[n], 0.25 * (Q[64 * i: 64 * i + 64, h] @ K[0, h]), rtol=0, atol=1e-12)


def test_cross_ignores_the_order_of_keys(oracle_lib):
    q, k, v = _cross_case(53, S_kv=130)
    perm = np.random.default_rng(54).permutation(130)
    items = oracle_lib.all_items(1, 2, 3)
    o1, l1 = oracle_lib.cross_items(q, k, v, 0.2, items)
    o2, l2 = oracle_lib.cross_items(q, k[:, perm], v[:, perm], 0.2, items)
    assert np.allclose(o1, o2, rtol=0, atol=1e-13) and np.allclose(l1, l2, rtol=0, atol=1e-13)
