"""GPU parity: the CUDA path through the C ABI against the FP64 oracle on the
same seeded inputs.  Integer and layout work must be bit-exact; the forward
output must meet the dataset card's pass rule (per-head cosine >= 0.9999,
max |d| <= 3e-2, mean |d| <= 1e-4, all finite) against the oracle's output
rounded to bf16; lse is checked against a derived fp32 error bound."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import common

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_block_sparse_b200 import build

    build.build()
    import video_block_sparse_b200 as m

    return m


def _no_device_error(vsa):
    rc, detail = vsa.device_status()
    assert rc == 0, (rc, detail)


# ------------------------------------------------------------------ tiling

@pytest.mark.parametrize("grid,B,H", [((5, 6, 7), 1, 2), ((9, 3, 5), 2, 3), ((1, 1, 1), 1, 1), ((21, 30, 52), 1, 40)])
def test_tile_untile_bit_exact(vsa, grid, B, H):
    g = np.random.default_rng(1)
    L = int(np.prod(grid))
    x = g.integers(0, 65536, size=(B, L, H, 128), dtype=np.uint16)
    xt = vsa.tile(common.dev(x), grid)
    want = oracle.tile(x, *grid)
    np.testing.assert_array_equal(common.host_bits(xt), want)
    back = vsa.untile(xt, grid)
    np.testing.assert_array_equal(common.host_bits(back), x)
    _no_device_error(vsa)


@pytest.mark.parametrize("grid,B,H", [((5, 6, 7), 1, 2), ((9, 3, 5), 2, 3), ((21, 30, 52), 1, 40)])
def test_tile_qkv_and_means_bit_exact(vsa, grid, B, H):
    """One launch tiles q, k, v exactly as vsa_tile does and forms the cube
    means of q and k exactly as the routing does from the tiled tensors
    (including counts below a cube's real extent, above it, and zero); the
    routing finished from those means equals the oracle's."""
    g = np.random.default_rng(7)
    L = int(np.prod(grid))
    xs = [synth.f32_to_bf16_bits((g.standard_normal((B, L, H, 128)) * 3).astype(np.float32)) for _ in range(3)]
    vbs = oracle.cube_counts(*grid).copy()
    nq = len(vbs)
    vbs[0] = 0
    vbs[nq - 1] = 64  # a partial cube averaged over its pads as well
    if nq > 2:
        vbs[1] = max(1, vbs[1] // 3)
    dvbs = torch.from_numpy(vbs).cuda()
    qt, kt, vt, qc, kc = vsa.tile_qkv(*(common.dev(x) for x in xs), grid, dvbs)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    tiled = [oracle.tile(x, *grid) for x in xs]
    for got, want in zip((qt, kt, vt), tiled):
        np.testing.assert_array_equal(common.host_bits(got), want)
    np.testing.assert_array_equal(common.host_bits(qc), oracle.cube_means(tiled[0], vbs))
    np.testing.assert_array_equal(common.host_bits(kc), oracle.cube_means(tiled[1], vbs))
    *_, vc = vsa.tile_qkv(*(common.dev(x) for x in xs), grid, dvbs, means=False, sums=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(common.host_bits(vc), oracle.cube_sums(tiled[2], vbs))
    topk = min(nq, 78)
    got_idx = vsa.route_means(qc, kc, topk)
    np.testing.assert_array_equal(got_idx.cpu().numpy(), oracle.route(tiled[0], tiled[1], vbs, topk))
    only = vsa.tile_qkv(*(common.dev(x) for x in xs), grid, means=False)
    for got, want in zip(only[:3], tiled):
        np.testing.assert_array_equal(common.host_bits(got), want)
    _no_device_error(vsa)


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("name", ["tiny", "wan480", "adversarial", "wan720"])
def test_route_bit_exact(vsa, name):
    cfg = synth.CONFIGS[name]
    T, Hh, W = cfg.grid
    q, k, _ = synth.grid_qkv(cfg)
    qt, kt = oracle.tile(q, T, Hh, W), oracle.tile(k, T, Hh, W)
    vbs = oracle.cube_counts(T, Hh, W)
    if cfg.adversarial:
        ov = synth.adversarial_override(cfg, len(vbs))
        vbs[ov.cubes] = np.minimum(vbs[ov.cubes], ov.counts)
    want = oracle.route(qt, kt, vbs, cfg.topk)
    got = vsa.route(common.dev(qt), common.dev(kt), torch.from_numpy(vbs).cuda(), cfg.topk)
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    _no_device_error(vsa)


def test_route_ties_and_empty_cubes(vsa):
    """Planted equal scores are ordered by cube index; an empty cube has mean 0."""
    nq, topk = 12, 6
    b_vals = np.array([3, -1, 7, 7, 0.5, 2, -8, 7, 1, 0.25, 4, 2], dtype=np.float32)
    q = np.zeros((1, 64 * nq, 2, 128), np.float32)
    k = np.zeros_like(q)
    q[:, :, :, 9] = 1.0
    for c in range(nq):
        k[0, 64 * c: 64 * c + 64, :, 9] = b_vals[c]
    vbs = np.full(nq, 64, np.int32)
    vbs[5] = 0
    qb, kb = synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k)
    want = oracle.route(qb, kb, vbs, topk)
    got = vsa.route(common.dev(qb), common.dev(kb), torch.from_numpy(vbs).cuda(), topk)
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    assert want[0, 0, 0].tolist() == [2, 3, 7, 10, 0, 11]  # cube 5 is empty: score 0


# ------------------------------------------------------------------ forward

def _run_fwd(vsa, p: common.Prepared, flags=0):
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx = torch.from_numpy(p.idx).cuda()
    vbs = torch.from_numpy(p.vbs).cuda()
    out, lse = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, flags=flags)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    return out, lse


def _check_items(p: common.Prepared, out, lse, items, tag, rule=True, precise=False):
    """rule=True: the card's pass rule against bf16_rne(oracle) with only the
    1/32-ulp near-midpoint reading (the gate of every Wan-shaped case, in both
    precision modes).  rule=False: the default mode's stated per-element error
    bound instead (small cases whose softmax rows are spread out and whose
    outputs reach |out| >= 4, where the default's weight rounding can move an
    element by one bf16 ulp; the precise mode meets the rule there).
    precise: the output came from the precise mode (tighter lse bound)."""
    got = oracle.fwd_items(p.qt, p.kt, p.vt, p.idx, p.vbs, p.cfg.sm_scale, items, want_wabs=not rule)
    o64, l64, wabs = got if not rule else (*got, None)
    rows = common.gather_items(out, items)
    hid = items[:, 1] + 1000 * items[:, 0]
    res = common.compare(rows, o64, hid)
    print(f"\n[{tag}] gate {res['gate']}\n[{tag}] vs fp64 {res['fp64']}")
    if rule:
        assert res["gate"]["ok"], res
    else:
        bnd = common.within_default_bound(rows, o64, wabs)
        print(f"[{tag}] default-mode bound {bnd}")
        assert bnd["ok"], bnd
    assert res["fp64"]["finite"] and res["fp64"]["min_head_cos"] >= 0.9999, res["fp64"]
    got_lse = common.gather_lse(lse, items)
    fin = np.isfinite(l64)
    assert np.array_equal(fin, np.isfinite(got_lse))
    bound = common.lse_bound(p.qt, p.kt, items, p.cfg.sm_scale, default_mode=not precise)
    assert np.all(np.abs(got_lse[fin] - l64[fin]) <= bound[fin]), float(np.max(np.abs(got_lse[fin] - l64[fin])))


def _head_items(p: common.Prepared, heads, batches=None):
    it = oracle.all_items(p.cfg.B, p.cfg.H, p.nq)
    keep = np.isin(it[:, 1], heads)
    if batches is not None:
        keep &= np.isin(it[:, 0], batches)
    return it[keep]


def test_fwd_tiny_precise_all_rows(vsa):
    p = common.prepare("tiny")
    out, lse = _run_fwd(vsa, p, flags=vsa.FWD_PRECISE_P)
    _check_items(p, out, lse, oracle.all_items(p.cfg.B, p.cfg.H, p.nq), "tiny/precise", precise=True)


def test_fwd_tiny_default_within_its_bound(vsa):
    """The tiny configuration (U[0.5, 4] value scales, softmax spread over up to
    128 keys) is the one case the default mode does not meet the rule on: one
    bf16 ulp at |out| >= 4 is 0.031.  It stays within its stated bound."""
    p = common.prepare("tiny")
    out, lse = _run_fwd(vsa, p)
    _check_items(p, out, lse, oracle.all_items(p.cfg.B, p.cfg.H, p.nq), "tiny/default", rule=False)


def test_fwd_mid_ragged_all_rows(vsa):
    """Several tiles and ragged cubes on every axis, every row checked."""
    p = common.prepare("wan480", H=3, grid=(9, 10, 11), topk=7, B=2)
    for flags in (0, vsa.FWD_PRECISE_P):
        out, lse = _run_fwd(vsa, p, flags=flags)
        items = oracle.all_items(p.cfg.B, p.cfg.H, p.nq)
        _check_items(p, out, lse, items, f"mid/flags{flags}", precise=flags != 0)


def _run_fwd_both_pairings(vsa, p):
    """The default mode with the consecutive pairing and with vsa_plan's."""
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx = torch.from_numpy(p.idx).cuda()
    vbs = torch.from_numpy(p.vbs).cuda()
    res = {}
    for planned in (False, True):
        pl = vsa.plan(idx) if planned else None
        out, lse = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, plan=pl)
        torch.cuda.synchronize()
        _no_device_error(vsa)
        assert bool(torch.isfinite(out).all())
        res[planned] = (out, lse)
    return res


@pytest.mark.parametrize("name,heads", [
    ("wan480", [0, 17]),
    ("adversarial", list(synth.ADV_T_HEADS) + [synth.ADV_FORCED_HEAD, 1]),
    ("sweep32", [3]),
    ("sweep156", [3]),
])
def test_fwd_full_size_whole_heads(vsa, name, heads):
    """Every row of whole heads at full size (the adversarial config: its three
    Student-t heads, the head with the forced low-count cubes and a clean head),
    with the consecutive and the planned pairing."""
    p = common.prepare(name)
    items = _head_items(p, heads)
    for planned, (out, lse) in _run_fwd_both_pairings(vsa, p).items():
        _check_items(p, out, lse, items, f"{name}/planned{int(planned)}")


@pytest.mark.slow
@pytest.mark.parametrize("name,heads", [("wan720", [0]), ("sweep312", [5]), ("dense624", [2])])
def test_fwd_large_whole_heads(vsa, name, heads):
    p = common.prepare(name)
    items = _head_items(p, heads)
    for planned, (out, lse) in _run_fwd_both_pairings(vsa, p).items():
        _check_items(p, out, lse, items, f"{name}/planned{int(planned)}")


@pytest.mark.slow
def test_fwd_wan480_every_row(vsa):
    """Every row of the whole Wan 832x480 output, as the bench computes it
    (planned pairing), element by element against the oracle."""
    p = common.prepare("wan480")
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    out, lse = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, plan=vsa.plan(idx))
    torch.cuda.synchronize()
    _no_device_error(vsa)
    _check_items(p, out, lse, oracle.all_items(p.cfg.B, p.cfg.H, p.nq), "wan480/all")


def test_fwd_dense_matches_library_attention(vsa):
    """topk = Nq with every cube full is dense attention: cross-check with torch SDPA."""
    g = np.random.default_rng(5)
    nq, H = 6, 2
    x = [synth.f32_to_bf16_bits(g.standard_normal((1, 64 * nq, H, 128)).astype(np.float32)) for _ in range(3)]
    q, k, v = (common.dev(a) for a in x)
    idx = torch.arange(nq, dtype=torch.int32).repeat(1, H, nq, 1).cuda().contiguous()
    vbs = torch.full((nq,), 64, dtype=torch.int32).cuda()
    out = vsa.fwd(q, k, v, idx, vbs, 128 ** -0.5, flags=vsa.FWD_PRECISE_P)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.permute(0, 2, 1, 3).float(), k.permute(0, 2, 1, 3).float(), v.permute(0, 2, 1, 3).float(),
        scale=128 ** -0.5).permute(0, 2, 1, 3)
    assert float((out.float() - ref).abs().max()) < 1e-2


# ------------------------------------------------------------------ edge cases

def _small(seed, nq=5, H=2, topk=3, B=1, vbs=None, dup=False):
    g = np.random.default_rng(seed)
    x = [synth.f32_to_bf16_bits((g.standard_normal((B, 64 * nq, H, 128)) * 2).astype(np.float32)) for _ in range(3)]
    if vbs is None:
        vbs = g.integers(0, 65, size=nq).astype(np.int32)
    idx = synth.random_topk(seed, B, H, nq, topk, distinct=not dup)
    cfg = synth.Config("edge", B=B, H=H, grid=(4, 4, 4 * nq), topk=topk, kind="tiny")
    return common.Prepared(cfg, x[0], x[1], x[2], np.asarray(vbs, np.int32), idx)


@pytest.mark.parametrize("seed,topk,dup", [(0, 1, False), (1, 3, False), (2, 5, True), (3, 4, True)])
def test_fwd_edge_lists(vsa, seed, topk, dup):
    p = _small(seed, topk=topk, dup=dup, vbs=[64, 1, 17, 33, 48][:5])
    for flags in (0, vsa.FWD_PRECISE_P):
        out, lse = _run_fwd(vsa, p, flags)
        _check_items(p, out, lse, oracle.all_items(1, 2, 5), f"edge{seed}/{flags}", rule=flags != 0,
                     precise=flags != 0)


@pytest.mark.parametrize("seed,topk,plan", [(20, 1, False), (21, 2, False), (22, 3, True)])
def test_fwd_many_short_tiles(vsa, seed, topk, plan):
    """More tiles than SMs, each of one to three steps (two to six KV cubes), some
    cubes empty: every CTA walks several tiles, so the step rings, the two-tile
    hand-off of row sums to the epilogue and the end-of-stream signalling run with
    very short tiles.  Every row is checked."""
    p = _small(seed, nq=9, H=80, topk=topk)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx = torch.from_numpy(p.idx).cuda()
    vbs = torch.from_numpy(p.vbs).cuda()
    pl = vsa.plan(idx) if plan else None
    out, lse = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, plan=pl)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    _check_items(p, out, lse, oracle.all_items(1, 80, 9), f"short{seed}", rule=False)


def test_fwd_all_masked_rows(vsa):
    p = _small(10, nq=3, H=1, topk=2, vbs=[0, 0, 64])
    p.idx[:] = np.array([[[[0, 1], [2, 0], [1, 1]]]], np.int32)
    out, lse = _run_fwd(vsa, p)
    o = out.float().cpu().numpy()
    ls = lse.cpu().numpy()
    assert np.all(o[0, 0:64] == 0) and np.all(ls[0, 0, 0:64] == -np.inf)
    assert np.all(o[0, 128:] == 0) and np.all(ls[0, 0, 128:] == -np.inf)
    assert np.all(np.isfinite(ls[0, 0, 64:128]))


def test_fwd_nan_pads_do_not_leak(vsa):
    p = _small(11, vbs=[64, 10, 33, 1, 0])
    out0, lse0 = _run_fwd(vsa, p)
    for c in range(5):
        p.kt[0, 64 * c + p.vbs[c]: 64 * c + 64] = 0x7FC0  # NaN
        p.vt[0, 64 * c + p.vbs[c]: 64 * c + 64] = 0xFF80  # -inf
    out1, lse1 = _run_fwd(vsa, p)
    assert torch.equal(out0.view(torch.int16), out1.view(torch.int16))
    assert torch.equal(lse0, lse1)


def test_fwd_nonfinite_real_v_row(vsa):
    """An Inf in a real V row (the contract asks for finite real rows): every
    query cube that selected that KV cube gets a non-finite value in that
    column, as the definition does; its tile partner, which did not select
    the cube, gets NaN there (weight 0 times Inf: the documented deviation of
    paired tiles); every other element still matches the oracle."""
    p = _small(19, nq=4, H=1, topk=2, vbs=[64, 64, 64, 64])
    p.idx[0, 0] = np.array([[0, 2], [1, 3], [0, 1], [3, 1]], np.int32)
    j, r, d = 2, 5, 7
    p.vt[0, 64 * j + r, 0, d] = 0x7F80  # +inf in a real row of cube 2 (selected by query cube 0 only)
    plan = torch.tensor([[[0, 1], [2, 3]]], dtype=torch.int32).cuda()
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    out = vsa.fwd(q, k, v, torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda(), p.cfg.sm_scale, plan=plan)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    items = oracle.all_items(1, 1, 4)
    o64, _, wabs = oracle.fwd_items(p.qt, p.kt, p.vt, p.idx, p.vbs, p.cfg.sm_scale, items, want_wabs=True)
    rows = common.gather_items(out, items)
    col = np.zeros(rows.shape, bool)
    col[..., d] = True
    assert not np.isfinite(rows[0][col[0]]).any() and not np.isfinite(o64[0][col[0]]).any()  # selected it
    assert np.isnan(rows[1][col[1]]).all() and np.isfinite(o64[1]).all()  # partner: the deviation
    finite = np.isfinite(o64)
    finite[1] &= ~col[1]
    bnd = common.within_default_bound(np.where(finite, rows, 0), np.where(finite, o64, 0), np.where(finite, wabs, 0))
    assert bnd["ok"], bnd
    assert np.isfinite(rows[2:]).all()  # the other tile never saw cube 2


def test_fwd_deterministic(vsa):
    p = _small(12, nq=8, H=3, topk=4)
    a, la = _run_fwd(vsa, p)
    b, lb = _run_fwd(vsa, p)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb)


def test_fwd_permuted_lists_agree(vsa):
    p = _small(13, nq=6, H=2, topk=4)
    a, _ = _run_fwd(vsa, p)
    p.idx = p.idx[..., ::-1].copy()
    b, _ = _run_fwd(vsa, p)
    assert float((a.float() - b.float()).abs().max()) <= 2 ** -7 * float(a.float().abs().max())


def test_fwd_bad_index_latches_device_error(vsa):
    p = _small(14, nq=4, H=1, topk=2, vbs=[64, 64, 64, 64])
    p.idx[0, 0, 1, 1] = 7  # out of range: the kernel skips it and latches error 1
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    vsa.fwd(q, k, v, torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda(), 0.1)
    rc, detail = vsa.device_status()
    assert rc == -7 and detail == 1
    assert vsa.device_status() == (0, 0)  # reading clears the word
    vbs = torch.tensor([64, 65, 64, 64], dtype=torch.int32).cuda()
    p.idx[0, 0, 1, 1] = 1
    vsa.fwd(q, k, v, torch.from_numpy(p.idx).cuda(), vbs, 0.1)
    rc, detail = vsa.device_status()
    assert rc == -7 and detail == 2


def test_stalled_pipeline_wait_ends_with_error_status(vsa):
    """A bounded pipeline wait that nothing completes gives up (~2 s of clock),
    latches code 3, raises the abort flag and returns; the context stays usable."""
    import time

    assert vsa.device_status() == (0, 0)
    t0 = time.perf_counter()
    bits = vsa.stall_check()
    elapsed = time.perf_counter() - t0
    assert bits == 2  # the wait reported failure and raised the abort flag
    assert vsa.device_status() == (-7, 3)
    assert 0.2 < elapsed < 60.0
    p = _small(16, nq=4, H=1, topk=2, vbs=[64, 40, 64, 9])
    out, lse = _run_fwd(vsa, p)
    _check_items(p, out, lse, oracle.all_items(1, 1, 4), "after-stall", rule=False)
    assert vsa.device_status() == (0, 0)


def test_fwd_rejects_bad_calls(vsa):
    p = _small(15, nq=4, H=1, topk=2)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    with pytest.raises(vsa.VSAError):
        vsa.fwd(q[:, :, :, :64].contiguous(), k, v, idx, vbs)
    with pytest.raises(ValueError):
        vsa.fwd(q.float(), k, v, idx, vbs)


def test_fwd_negative_scale(vsa):
    """A negative logit scale flips which key dominates; the contract holds for any sign."""
    p = _small(16, nq=6, H=2, topk=4, vbs=[64, 7, 64, 33, 64, 1])
    p.cfg = synth.Config("neg", B=1, H=2, grid=(4, 4, 24), topk=4, kind="tiny")
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    items = oracle.all_items(1, 2, 6)
    o64, l64, wabs = oracle.fwd_items(p.qt, p.kt, p.vt, p.idx, p.vbs, -0.3, items, want_wabs=True)
    for flags in (vsa.FWD_PRECISE_P, 0):
        out, lse = vsa.fwd(q, k, v, idx, vbs, -0.3, want_lse=True, flags=flags)
        torch.cuda.synchronize()
        _no_device_error(vsa)
        rows = common.gather_items(out, items)
        if flags:
            res = common.compare(rows, o64, items[:, 1])
            assert res["gate"]["ok"], res
        else:
            bnd = common.within_default_bound(rows, o64, wabs)
            assert bnd["ok"], bnd
        got_lse = common.gather_lse(lse, items)
        # default mode: the row sum of bf16-rounded weights, within -ln(1 - 2^-8) < 4e-3
        assert np.allclose(got_lse, l64, rtol=1e-5, atol=1e-3 if flags else 5e-3)


# ------------------------------------------------------------------ tile plan

@pytest.mark.parametrize("case", ["tiny", "random33", "wan480"])
def test_plan_bit_exact(vsa, case):
    if case == "random33":
        idx = synth.random_topk(21, 2, 2, 33, 5)
    else:
        p = common.prepare(case)
        idx = p.idx
    want = oracle.plan(idx)
    got = vsa.plan(torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    _no_device_error(vsa)
    np.testing.assert_array_equal(got.cpu().numpy(), want)


def test_fwd_with_plan_mid(vsa):
    """The paired kernel on the planner's pairing: every row checked (both modes)."""
    p = common.prepare("wan480", H=3, grid=(9, 10, 11), topk=7, B=2)
    plan = oracle.plan(p.idx)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    for flags in (0, vsa.FWD_PRECISE_P):
        out, lse = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, flags=flags,
                           plan=torch.from_numpy(plan).cuda())
        torch.cuda.synchronize()
        _no_device_error(vsa)
        _check_items(p, out, lse, oracle.all_items(p.cfg.B, p.cfg.H, p.nq), f"plan-mid/{flags}", precise=flags != 0)


def test_fwd_with_arbitrary_pairing(vsa):
    """Any valid pairing gives the same results: a random one, singles included."""
    p = _small(17, nq=9, H=2, topk=4, vbs=[64, 7, 64, 33, 64, 1, 16, 0, 48])
    g = np.random.default_rng(17)
    plan = np.empty((2, 5, 2), np.int32)
    for bh in range(2):
        perm = g.permutation(9).tolist()
        tiles = [sorted(perm[2 * t: 2 * t + 2]) for t in range(4)] + [[perm[8], -1]]
        plan[bh] = np.array(sorted(tiles), np.int32)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    out, lse = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, plan=torch.from_numpy(plan).cuda())
    torch.cuda.synchronize()
    _no_device_error(vsa)
    _check_items(p, out, lse, oracle.all_items(1, 2, 9), "arbitrary-pairing", rule=False)


def test_fwd_plan_bad_entry_latches_error(vsa):
    p = _small(18, nq=4, H=1, topk=2, vbs=[64, 64, 64, 64])
    plan = np.array([[[0, 1], [2, 9]]], np.int32)  # 9 is not a cube: the kernel drops it, error 4
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    vsa.fwd(q, k, v, torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda(), 0.1,
            plan=torch.from_numpy(plan).cuda())
    rc, detail = vsa.device_status()
    assert rc == -7 and detail == 4


# ------------------------------------------------------------------ proxy compensation

def _proxy_inputs(p: common.Prepared):
    kc = oracle.cube_means(p.kt, p.vbs)
    vc = oracle.cube_sums(p.vt, p.vbs)
    return kc, vc


def _check_proxy(vsa, p: common.Prepared, items, tag, flags=0, plan=False, rule=True):
    """vsa_fwd_proxy against the oracle's proxy forward, every listed row: the card's
    rule against bf16_rne(oracle) (1/32-ulp midpoint reading), lse within the
    forward's bound."""
    kc, vc = _proxy_inputs(p)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    pl = vsa.plan(idx) if plan else None
    out, lse = vsa.fwd_proxy(q, k, v, idx, vbs, common.dev(kc), common.dev(vc), p.cfg.sm_scale, want_lse=True,
                             flags=flags, plan=pl)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    o64, l64 = oracle.fwd_proxy_items(p.qt, p.kt, p.vt, kc, vc, p.idx, p.vbs, p.cfg.sm_scale, items)
    rows = common.gather_items(out, items)
    res = common.compare(rows, o64, items[:, 1] + 1000 * items[:, 0])
    print(f"\n[{tag}] gate {res['gate']}\n[{tag}] vs fp64 {res['fp64']}")
    if rule:
        assert res["gate"]["ok"], res
    assert res["fp64"]["finite"] and res["fp64"]["min_head_cos"] >= 0.9999, res["fp64"]
    got_lse = common.gather_lse(lse, items)
    fin = np.isfinite(l64)
    assert np.array_equal(fin, np.isfinite(got_lse))
    bound = common.lse_bound(p.qt, p.kt, items, p.cfg.sm_scale, default_mode=flags == 0)
    assert np.all(np.abs(got_lse[fin] - l64[fin]) <= bound[fin]), float(np.max(np.abs(got_lse[fin] - l64[fin])))
    return out


@pytest.mark.parametrize("flags", [0, 1])
@pytest.mark.parametrize("plan", [False, True])
def test_fwd_proxy_mid_all_rows(vsa, flags, plan):
    """Ragged cubes, several tiles, one partial proxy step (27 cubes): every row."""
    p = common.prepare("wan480", H=3, grid=(9, 10, 11), topk=7, B=2)
    _check_proxy(vsa, p, oracle.all_items(p.cfg.B, p.cfg.H, p.nq), f"proxy-mid/{flags}/{int(plan)}", flags, plan)


@pytest.mark.parametrize("plan", [False, True])
def test_fwd_proxy_wan480_whole_heads(vsa, plan):
    """The Wan 832x480 cube count: five proxy steps per tile (the last one partial,
    48 cubes in its second half), every row of two heads."""
    p = common.prepare("wan480", H=2)
    _check_proxy(vsa, p, oracle.all_items(p.cfg.B, p.cfg.H, p.nq), f"proxy-wan480/{int(plan)}", 0, plan)


@pytest.mark.parametrize("seed,topk,dup", [(30, 1, False), (31, 3, True)])
def test_fwd_proxy_edge_lists(vsa, seed, topk, dup):
    """Empty cubes (no proxy, no tokens), a partial cube, duplicated selections, topk 1."""
    p = _small(seed, nq=9, H=2, topk=topk, dup=dup, vbs=[64, 0, 17, 33, 1, 64, 0, 48, 5])
    items = oracle.all_items(1, 2, 9)
    _check_proxy(vsa, p, items, f"proxy-edge{seed}/precise", flags=1)
    _check_proxy(vsa, p, items, f"proxy-edge{seed}/default", flags=0, rule=False)


def test_fwd_proxy_with_every_cube_selected_is_the_plain_forward(vsa):
    """topk = Nq: no cube is omitted, so no proxy key is used and the output equals vsa_fwd's."""
    p = _small(32, nq=6, H=2, topk=6)
    p.idx = np.broadcast_to(np.arange(6, dtype=np.int32), p.idx.shape).copy()
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda()
    kc, vc = _proxy_inputs(p)
    a, la = vsa.fwd_proxy(q, k, v, idx, vbs, common.dev(kc), common.dev(vc), p.cfg.sm_scale, want_lse=True)
    b, lb = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    assert torch.equal(a.float(), b.float()) and torch.equal(la, lb)


# ------------------------------------------------------------------ route formats (BSR, bitmaps)

def _i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _mask_dev(mask: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(mask).view(np.int32)).cuda()


def _check_bsr(p: common.Prepared, indptr, indices, out, lse, items, tag, flags=0, kc=None, vc=None, rule=True):
    """A forward over BSR rows (or bitmaps written out as BSR rows) against the oracle's,
    every listed row: the card's rule (rule=True), else for the plain forward the
    default mode's bound (with proxies the cosine and lse checks alone, as for
    vsa_fwd_proxy)."""
    bound_mode = not rule and kc is None
    got = oracle.fwd_bsr_items(p.qt, p.kt, p.vt, indptr, indices, p.vbs, p.cfg.sm_scale, items, kc=kc, vc=vc,
                               want_wabs=bound_mode)
    o64, l64, wabs = got if bound_mode else (*got, None)
    rows = common.gather_items(out, items)
    res = common.compare(rows, o64, items[:, 1] + 1000 * items[:, 0])
    print(f"\n[{tag}] gate {res['gate']}\n[{tag}] vs fp64 {res['fp64']}")
    if rule:
        assert res["gate"]["ok"], res
    elif bound_mode:
        bnd = common.within_default_bound(rows, o64, wabs)
        print(f"[{tag}] default-mode bound {bnd}")
        assert bnd["ok"], bnd
    assert res["fp64"]["finite"] and res["fp64"]["min_head_cos"] >= 0.9999, res["fp64"]
    got_lse = common.gather_lse(lse, items)
    fin = np.isfinite(l64)
    assert np.array_equal(fin, np.isfinite(got_lse))
    assert np.all(rows[~fin] == 0.0)
    bound = common.lse_bound(p.qt, p.kt, items, p.cfg.sm_scale, default_mode=flags == 0)
    assert np.all(np.abs(got_lse[fin] - l64[fin]) <= bound[fin]), float(np.max(np.abs(got_lse[fin] - l64[fin])))


@pytest.mark.parametrize("proxy", [False, True])
@pytest.mark.parametrize("plan", [False, True])
def test_fwd_route_formats_are_bit_identical(vsa, proxy, plan):
    """Distinct lists in ascending order as topk_idx rows, as BSR rows and as bitmaps:
    the same step lists, so bit-identical out and lse; every row against the oracle."""
    p = common.prepare("wan480", H=3, grid=(9, 10, 11), topk=7, B=2)
    p.idx = np.sort(p.idx, axis=-1).astype(np.int32)
    B, H, nq = p.cfg.B, p.cfg.H, p.nq
    indptr, indices = oracle.lists_to_bsr(p.idx)
    mask = oracle.bsr_to_bitmask(indptr, indices, B, H, nq)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    idx, vbs = _i32(p.idx), _i32(p.vbs)
    kc, vc = _proxy_inputs(p) if proxy else (None, None)
    kcd, vcd = (common.dev(kc), common.dev(vc)) if proxy else (None, None)
    pl = vsa.plan(idx) if plan else None
    if proxy:
        a, la = vsa.fwd_proxy(q, k, v, idx, vbs, kcd, vcd, p.cfg.sm_scale, want_lse=True, plan=pl)
    else:
        a, la = vsa.fwd(q, k, v, idx, vbs, p.cfg.sm_scale, want_lse=True, plan=pl)
    b, lb = vsa.fwd_bsr(q, k, v, _i32(indptr), _i32(indices), vbs, p.cfg.sm_scale, kc=kcd, vc=vcd, want_lse=True,
                        plan=pl)
    c, lc = vsa.fwd_bitmask(q, k, v, _mask_dev(mask), vbs, p.cfg.sm_scale, kc=kcd, vc=vcd, want_lse=True, plan=pl)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    for x, lx in ((b, lb), (c, lc)):
        assert torch.equal(a.view(torch.int16), x.view(torch.int16))
        assert torch.equal(la.view(torch.int32), lx.view(torch.int32))
    _check_bsr(p, indptr, indices, c, lc, oracle.all_items(B, H, nq), f"formats/{int(proxy)}/{int(plan)}", 0,
               kc=kc, vc=vc)


@pytest.mark.parametrize("flags", [0, 1])
@pytest.mark.parametrize("proxy", [False, True])
def test_fwd_bsr_variable_rows(vsa, flags, proxy):
    """BSR rows of 0 to 12 cubes in any order, repeats included, empty cubes: every row."""
    p = _small(40, nq=14, H=3, topk=1, vbs=[64, 0, 17, 33, 1, 64, 0, 48, 5, 64, 64, 9, 64, 22])
    g = np.random.default_rng(41)
    B, H, nq = 1, 3, 14
    indptr, indices = [0], []
    for r in range(B * H * nq):
        n = int(g.integers(0, 13)) if r % 7 else 0
        indices.extend(g.choice(nq, size=n, replace=bool(r % 3 == 0)).tolist())
        indptr.append(len(indices))
    indptr, indices = np.asarray(indptr, np.int32), np.asarray(indices, np.int32)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    kc, vc = _proxy_inputs(p) if proxy else (None, None)
    out, lse = vsa.fwd_bsr(q, k, v, _i32(indptr), _i32(indices), _i32(p.vbs), p.cfg.sm_scale,
                           kc=common.dev(kc) if proxy else None, vc=common.dev(vc) if proxy else None,
                           want_lse=True, flags=flags)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    _check_bsr(p, indptr, indices, out, lse, oracle.all_items(B, H, nq), f"bsr-var/{flags}/{int(proxy)}", flags,
               kc=kc, vc=vc, rule=flags == 1)


def test_fwd_bitmask_padding_bits_are_ignored(vsa):
    """Random bitmaps of a 37-cube grid: setting the 27 padding bits of every row's last
    word changes nothing (bit for bit, no error); every row against the oracle."""
    p = _small(42, nq=37, H=2, topk=1)
    g = np.random.default_rng(43)
    B, H, nq = 1, 2, 37
    mask = (g.random((B, H, nq, 2, 32)) < 0.2)
    mask[..., 1, 5:] = False
    words = (mask.astype(np.uint64) << np.arange(32, dtype=np.uint64)).sum(axis=-1).astype(np.uint32)
    dirty = words.copy()
    dirty[..., 1] |= np.uint32(0xFFFFFFE0)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    vbs = _i32(p.vbs)
    a, la = vsa.fwd_bitmask(q, k, v, _mask_dev(words), vbs, p.cfg.sm_scale, want_lse=True)
    b, lb = vsa.fwd_bitmask(q, k, v, _mask_dev(dirty), vbs, p.cfg.sm_scale, want_lse=True)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la.view(torch.int32),
                                                                                  lb.view(torch.int32))
    indptr, indices = oracle.bitmask_to_bsr(dirty, nq)
    _check_bsr(p, indptr, indices, b, lb, oracle.all_items(B, H, nq), "bitmask-pad", 0, rule=False)


def test_fwd_bsr_bad_rows_latch_error_and_are_empty(vsa):
    """A row reaching past nnz and a row with end < start latch error 5 and are taken as
    empty (out 0, lse -inf); an index out of range latches 1 and is dropped; the other
    rows are unaffected."""
    p = _small(44, nq=5, H=1, topk=1, vbs=[64, 64, 30, 64, 64])
    indptr = np.array([0, 2, 4, 3, 5, 9], np.int32)  # row 2: end < start; row 4: past nnz = 8
    indices = np.array([0, 1, 2, 3, 4, 0, 1, 2], np.int32)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    out, lse = vsa.fwd_bsr(q, k, v, _i32(indptr), _i32(indices), _i32(p.vbs), p.cfg.sm_scale, want_lse=True)
    rc, detail = vsa.device_status()
    assert rc == -7 and detail == 5
    clean_ptr = np.array([0, 2, 4, 4, 6, 6], np.int32)  # the same rows, the bad ones empty
    clean_idx = np.array([0, 1, 2, 3, 3, 4], np.int32)
    _check_bsr(p, clean_ptr, clean_idx, out, lse, oracle.all_items(1, 1, 5), "bsr-bad", 0, rule=False)
    bad = clean_idx.copy()
    bad[1] = 9
    out2 = vsa.fwd_bsr(q, k, v, _i32(clean_ptr), _i32(bad), _i32(p.vbs), p.cfg.sm_scale)
    rc, detail = vsa.device_status()
    assert rc == -7 and detail == 1
    assert torch.isfinite(out2.float()).all()


def test_fwd_bitmask_row_over_1024_cubes_keeps_its_first_1024(vsa):
    """1100 cubes, one row selecting all of them: error 5, and the row attends to its
    lowest 1024 cubes (the oracle over those); the other rows are unaffected."""
    nq = 1100
    p = _small(45, nq=nq, H=1, topk=1, vbs=np.full(nq, 64, np.int32))
    g = np.random.default_rng(46)
    W = (nq + 31) // 32
    words = np.zeros((1, 1, nq, W), np.uint32)
    sel = [g.choice(nq, size=5, replace=False) for _ in range(nq)]
    for i in range(nq):
        for c in sel[i]:
            words[0, 0, i, c // 32] |= np.uint32(1 << (c % 32))
    words[0, 0, 7] = np.uint32(0xFFFFFFFF)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    out, lse = vsa.fwd_bitmask(q, k, v, _mask_dev(words), _i32(p.vbs), p.cfg.sm_scale, want_lse=True)
    rc, detail = vsa.device_status()
    assert rc == -7 and detail == 5
    kept = words.copy()
    kept[0, 0, 7] = 0
    kept[0, 0, 7, :32] = np.uint32(0xFFFFFFFF)  # cubes 0..1023
    indptr, indices = oracle.bitmask_to_bsr(kept, nq)
    items = np.array([[0, 0, 7], [0, 0, 0], [0, 0, nq - 1]], np.int32)
    _check_bsr(p, indptr, indices, out, lse, items, "bitmask-1024", 0, rule=False)


def test_fwd_routes_live_under_cuda_graph_replay(vsa):
    """A captured forward reads its routes from the same buffers at every replay: new
    bitmaps (and new topk lists) written in place between replays give the results an
    eager call gives for them."""
    p = common.prepare("wan480", H=2, grid=(9, 10, 11), topk=6, B=1)
    B, H, nq = 1, 2, p.nq
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    vbs = _i32(p.vbs)
    g = np.random.default_rng(47)
    lists = [np.sort(synth.random_topk(int(s), B, H, nq, 6), axis=-1).astype(np.int32) for s in g.integers(0, 1000, 3)]
    masks = [oracle.bsr_to_bitmask(*oracle.lists_to_bsr(x), B, H, nq) for x in lists]
    mask_buf, idx_buf = _mask_dev(masks[0]), _i32(lists[0])
    out_m, out_l = torch.empty_like(q), torch.empty_like(q)
    lse_m = torch.empty(B, H, q.shape[1], dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside capture
        vsa.fwd_bitmask(q, k, v, mask_buf, vbs, p.cfg.sm_scale, out=out_m, lse=lse_m)
        vsa.fwd(q, k, v, idx_buf, vbs, p.cfg.sm_scale, out=out_l)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        vsa.fwd_bitmask(q, k, v, mask_buf, vbs, p.cfg.sm_scale, out=out_m, lse=lse_m)
        vsa.fwd(q, k, v, idx_buf, vbs, p.cfg.sm_scale, out=out_l)
    for x, m in zip(lists[1:], masks[1:]):
        mask_buf.copy_(_mask_dev(m))
        idx_buf.copy_(_i32(x))
        graph.replay()
        torch.cuda.synchronize()
        want_m, want_lse = vsa.fwd_bitmask(q, k, v, _mask_dev(m), vbs, p.cfg.sm_scale, want_lse=True)
        want_l = vsa.fwd(q, k, v, _i32(x), vbs, p.cfg.sm_scale)
        torch.cuda.synchronize()
        _no_device_error(vsa)
        assert torch.equal(out_m.view(torch.int16), want_m.view(torch.int16))
        assert torch.equal(lse_m.view(torch.int32), want_lse.view(torch.int32))
        assert torch.equal(out_l.view(torch.int16), want_l.view(torch.int16))
        assert torch.equal(out_m.view(torch.int16), out_l.view(torch.int16))
    del graph


# ------------------------------------------------------------------ short-KV cross-attention

def _cross_inputs(seed, B, nblk, S_kv, H, scale=1.0):
    g = np.random.default_rng(seed)
    q = synth.f32_to_bf16_bits((g.standard_normal((B, 64 * nblk, H, 128)) * scale).astype(np.float32))
    k = synth.f32_to_bf16_bits((g.standard_normal((B, S_kv, H, 128)) * scale).astype(np.float32))
    v = synth.f32_to_bf16_bits(g.standard_normal((B, S_kv, H, 128)).astype(np.float32))
    return q, k, v


def _check_cross(q, k, v, out, lse, items, sm_scale, tag, precise):
    """Each mode against its stated bound: the weights' rounding (2^-7 default, 2^-15
    precise, times sum w |v|) plus the fp32 accumulation of S_kv products (S_kv 2^-24
    sum w |v|), half an ulp for the output's rounding.  Rows over hundreds of random keys
    are means of many terms of both signs: the accumulation error, relative to the small
    result, moves more outputs across a bf16 midpoint than in the fine stage.  And the
    card's cosine against FP64."""
    o64, l64, wabs = oracle.cross_items(q, k, v, sm_scale, items, want_wabs=True)
    rows = common.gather_items(out, items)
    res = common.compare(rows, o64, items[:, 1] + 1000 * items[:, 0])
    print(f"\n[{tag}] gate {res['gate']}\n[{tag}] vs fp64 {res['fp64']}")
    weights = common.PRECISE_WEIGHT_BOUND if precise else common.DEFAULT_WEIGHT_BOUND
    bnd = common.within_default_bound(rows, o64, wabs, coeff=weights + k.shape[1] * 2.0 ** -24)
    print(f"[{tag}] bound {bnd}")
    assert bnd["ok"], bnd
    assert res["fp64"]["finite"] and res["fp64"]["min_head_cos"] >= 0.9999, res["fp64"]
    got_lse = common.gather_lse(lse, items)
    bound = common.lse_bound(q, k, items, sm_scale, default_mode=not precise)
    assert np.all(np.abs(got_lse - l64) <= bound), float(np.max(np.abs(got_lse - l64)))


@pytest.mark.parametrize("flags", [0, 1])
@pytest.mark.parametrize("S_kv", [512, 77, 1, 1000])
def test_cross_attn_every_row(vsa, S_kv, flags):
    """Every query row over every key of a short sequence: Wan's 512 text tokens, a
    ragged length (last cube partial), a single key, and 16 cubes (8 steps a tile)."""
    B, nblk, H = 2, 9, 3
    q, k, v = _cross_inputs(60 + S_kv, B, nblk, S_kv, H)
    sm = 128 ** -0.5
    out, lse = vsa.cross_attn(common.dev(q), common.dev(k), common.dev(v), sm, want_lse=True, flags=flags)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    _check_cross(q, k, v, out, lse, oracle.all_items(B, H, nblk), sm, f"cross/{S_kv}/{flags}", flags == 1)


def test_cross_attn_over_its_own_sequence_is_the_dense_forward(vsa):
    """K/V = the query sequence and every cube listed in order: the fine-stage forward's
    step lists exactly, so bit-identical results."""
    p = _small(61, nq=6, H=2, topk=6, vbs=[64] * 6)
    p.idx = np.broadcast_to(np.arange(6, dtype=np.int32), p.idx.shape).copy()
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    a, la = vsa.cross_attn(q, k, v, p.cfg.sm_scale, want_lse=True)
    b, lb = vsa.fwd(q, k, v, torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda(), p.cfg.sm_scale,
                    want_lse=True)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la.view(torch.int32),
                                                                                  lb.view(torch.int32))


def test_cross_attn_wan_shape_sampled(vsa):
    """Wan 832x480 queries (39936 tokens, 40 heads) over a 512-token text KV: sampled
    query blocks of every head against the oracle."""
    B, nblk, H, S_kv = 1, 624, 40, 512
    q, k, v = _cross_inputs(62, B, nblk, S_kv, H)
    sm = 128 ** -0.5
    out, lse = vsa.cross_attn(common.dev(q), common.dev(k), common.dev(v), sm, want_lse=True)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    items = common.sample_items(B, H, nblk, 120, seed=63)
    _check_cross(q, k, v, out, lse, items, sm, "cross/wan", False)


@pytest.mark.parametrize("nq,topk", [(8, 8), (6, 5)])
def test_fwd_four_step_tiles_many_per_cta(vsa, nq, topk):
    """Tiles of exactly four steps (one more than the S buffers) and more tiles than SMs:
    the epilogue hands the next tile's first step to its product only after taking that
    step's offsets, so the softmax cannot lap the correction warps on the three-buffer
    ring (which stalled this case until a bounded wait gave up).  Every row."""
    p = _small(64, nq=nq, H=40, topk=topk, vbs=[64] * nq)
    p.idx = np.sort(np.stack([np.stack([np.random.default_rng(65 + h).permutation(nq)[:topk] for _ in range(nq)])
                              for h in range(40)])[None], axis=-1).astype(np.int32)
    q, k, v = common.dev(p.qt), common.dev(p.kt), common.dev(p.vt)
    out, lse = vsa.fwd(q, k, v, torch.from_numpy(p.idx).cuda(), torch.from_numpy(p.vbs).cuda(), p.cfg.sm_scale,
                       want_lse=True)
    torch.cuda.synchronize()
    _no_device_error(vsa)
    _check_items(p, out, lse, oracle.all_items(1, 40, nq), f"four-step/{nq}", rule=False)
