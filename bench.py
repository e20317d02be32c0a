"""Benchmark of the VSA fine stage on B200: one step = the whole hot path on
one batch of synthetic Wan2.2 832x480/81f activations:

    tile q, k, v (raster -> cube-major, one launch that also forms the cube
    means of q and k)  ->  route (scores and top-k from those means)
    ->  plan (pair query cubes by selection overlap)
    ->  fine block-sparse attention forward  ->  untile the output

Metric: effective TFLOP/s of the step, FLOPs = 4 * B * S * topk * 64 * D * H
(the attention contractions; the other steps count no FLOPs).  Inputs are
resident in HBM when the timed region starts; they are larger than L2
(3 x 335 MB raster q, k, v per step), so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun every rank runs its own independent problem (weak scaling, no
data-path collective); rank 0 prints one JSON line.

Besides the headline, the line carries (rank 0, N=1): the forward with the
consecutive pairing and on random selection lists of the same shape (how the
paired kernel's speed depends on list overlap, with the steps per tile of
each), and the forward alone at the other configurations (Wan 1280x720 CFG
pair, the top-k sweep and the dense case); skip those with --no-extras.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "wan480"
METRIC = "VSA fine fwd ms/call & TFLOP/s at Wan2.2 832x480/81f; % B200 BF16 peak"


def flops(cfg, S):
    return 4.0 * cfg.B * S * cfg.topk * 64 * 128 * cfg.H


def config_block(cfg, S):
    return {
        "workload": "Wan2.2 T2V-A14B 832x480/81f VSA fine stage (tile q,k,v + cube means -> route -> plan -> fwd "
                    "-> untile)",
        "B": cfg.B, "latent_grid": list(cfg.grid), "S_padded": S, "H": cfg.H, "D": 128, "topk": cfg.topk,
        "sm_scale": cfg.sm_scale, "global_batch": cfg.B, "seq_len": S, "parallelism": "replicas (independent problem per GPU)",
        "l2": "inputs larger than L2 (1.0 GB raster q,k,v read per step); no flush",
        "inputs": "seeded synthetic: q,k ~ N(0,1)*U[1,8] per head with 4 shared outlier channels x20, v ~ N(0,1)",
    }


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d.get("bf16_tflops_sustained"), d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        # the raw samples (the JSON line carries their summary); VSA_CLOCK_DIR picks the folder
        folder = os.environ.get("VSA_CLOCK_DIR") or tempfile.gettempdir()
        self.path = os.path.join(folder, f"vsa_clocks_rank{index}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- ranks

def problem_config(rank: int, heads: int = 0):
    """The workload of one rank: an independent seeded problem per rank (weak scaling);
    `heads` overrides the head count (a reduced case for profiler captures only)."""
    import dataclasses

    cfg = dataclasses.replace(synth.CONFIGS[WORKLOAD], seed=rank)
    if heads:
        cfg = dataclasses.replace(cfg, H=heads)
    return cfg


def max_over_ranks(values, device) -> list[float]:
    """Every rank's timings -> their maximum over ranks, on every rank (one all-reduce
    when a process group of more than one rank is up; the values unchanged otherwise)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist = torch.distributed
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# --------------------------------------------------------------------------- GPU arm

def run_gpu(args, rank, world, local_rank):
    import video_block_sparse_b200 as vsa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = problem_config(rank, args.heads)
    T, Hh, W = cfg.grid
    vbs_h = vsa.cube_counts(T, Hh, W)
    nq = len(vbs_h)
    S = 64 * nq
    q_h, k_h, v_h = (synth.bits_to_torch(x) for x in synth.grid_qkv(cfg))
    q_g, k_g, v_g = (x.to(dev) for x in (q_h, k_h, v_h))
    vbs = vbs_h.to(dev)
    B, L, H, D = q_g.shape
    qt, kt, vt = (torch.empty(B, S, H, D, dtype=torch.bfloat16, device=dev) for _ in range(3))
    qc, kc = (torch.empty(B, H, nq, D, dtype=torch.bfloat16, device=dev) for _ in range(2))
    idx = torch.empty(B, H, nq, cfg.topk, dtype=torch.int32, device=dev)
    plan = torch.empty(B * H, (nq + 1) // 2, 2, dtype=torch.int32, device=dev)
    plan_ws = torch.empty(vsa.plan_workspace_size(B, H, nq, cfg.topk), dtype=torch.uint8, device=dev)
    out_t = torch.empty_like(qt)
    out_g = torch.empty_like(q_g)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev_f0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_f1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def step(i=None, src=(q_g, k_g, v_g), dst=None):
        vsa.tile_qkv(*src, cfg.grid, vbs, out=[qt, kt, vt, qc, kc])
        vsa.route_means(qc, kc, cfg.topk, out=idx)
        vsa.plan(idx, out=plan, workspace=plan_ws)
        if i is not None:
            ev_f0[i].record(stream)
        vsa.fwd(qt, kt, vt, idx, vbs, cfg.sm_scale, out=out_t, lse=lse, plan=plan)
        if i is not None:
            ev_f1[i].record(stream)
        vsa.untile(out_t, cfg.grid, out=out_g if dst is None else dst)

    launches_per_step = 1 + 1 + 3 + 1 + 1  # tile_qkv, route_means, plan (3 kernels), fwd, untile
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc, detail = vsa.device_status()
    if rc != 0:
        raise RuntimeError(f"device error {rc}/{detail} in warm-up")

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_total = t0.elapsed_time(t1)
    fwd_ms = [a.elapsed_time(b) for a, b in zip(ev_f0, ev_f1)]

    # end to end through the public API: pinned host raster q,k,v in, raster out back,
    # every step.  Two forms: serial (copy in, compute, copy out, one stream), and
    # pipelined (two device buffer sets; step i's inputs are copied in on one copy
    # stream and step i-1's result copied out on another while step i-1 computes),
    # as a stream of independent problems would run.  The line reports the pipelined
    # one and keeps the serial one beside it.
    q_p, k_p, v_p = (x.pin_memory() for x in (q_h, k_h, v_h))
    out_ps = [torch.empty(out_g.shape, dtype=out_g.dtype).pin_memory() for _ in range(2)]
    e2e_steps = max(1, min(args.steps, 10))

    def e2e_step():
        q_g.copy_(q_p, non_blocking=True)
        k_g.copy_(k_p, non_blocking=True)
        v_g.copy_(v_p, non_blocking=True)
        step()
        out_ps[0].copy_(out_g, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_serial_ms = e0.elapsed_time(e1) / e2e_steps

    sets = [(q_g, k_g, v_g, out_g), tuple(torch.empty_like(x) for x in (q_g, k_g, v_g, out_g))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run_pipelined(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        s_in.wait_event(p0)
        for i in range(n):
            qb, kb, vb, ob = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[i - 2])  # buffer set free: its last step's kernels are done
                qb.copy_(q_p, non_blocking=True)
                kb.copy_(k_p, non_blocking=True)
                vb.copy_(v_p, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])  # out buffer read back
            step(src=(qb, kb, vb), dst=ob)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                out_ps[i % 2].copy_(ob, non_blocking=True)
                ev_out[i].record(s_out)
        stream.wait_event(ev_out[n - 1])
        stream.wait_event(ev_in[n - 1])
        p1.record(stream)
        torch.cuda.synchronize()
        return p0.elapsed_time(p1) / n

    run_pipelined(2)
    e2e_ms = run_pipelined(e2e_steps)
    rc, detail = vsa.device_status()
    if rc != 0:
        raise RuntimeError(f"device error {rc}/{detail}")
    got = out_ps[(e2e_steps - 1) % 2].view(torch.int16)
    if not torch.equal(got, out_g.cpu().view(torch.int16)):
        raise RuntimeError("pipelined end-to-end result differs from the device-timed step's result")

    ms_step = ms_total / args.steps
    ms_step, e2e_ms, fwd_avg, e2e_serial_ms = max_over_ranks(
        [ms_step, e2e_ms, statistics.mean(fwd_ms), e2e_serial_ms], dev)
    extras = None
    if world == 1 and args.extras:
        extras = run_extras(vsa, dev, cfg, qt, kt, vt, qc, kc, idx, vbs, read_peaks()[0])
    return dict(cfg=cfg, S=S, ms_step=ms_step, e2e_ms=e2e_ms, e2e_serial_ms=e2e_serial_ms, fwd_ms=fwd_avg,
                fwd_list=fwd_ms,
                clocks=clk.summary(), launches=launches_per_step * args.steps, extras=extras,
                h2d=3 * q_h.numel() * 2, d2h=out_g.numel() * 2)


# --------------------------------------------------------------------------- extras

def lists_to_bitmask(idx: torch.Tensor) -> torch.Tensor:
    """[B, H, Nq, topk] lists of distinct cubes -> [B, H, Nq, ceil(Nq/32)] packed bitmaps
    (bit c % 32 of word c / 32 selects cube c), as int32 words."""
    B, H, nq, _ = idx.shape
    bits = torch.zeros(B, H, nq, (nq + 31) // 32, dtype=torch.int64, device=idx.device)
    bits.scatter_add_(3, (idx // 32).long(), torch.ones_like(idx, dtype=torch.int64) << (idx % 32).long())
    return torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits).to(torch.int32).contiguous()


def steps_per_tile(idx: np.ndarray, plan: np.ndarray | None, vbs: np.ndarray) -> np.ndarray:
    """Steps each tile of the paired forward walks: the distinct cubes with a valid
    token that either list names (every entry when a list repeats a cube), two per step.
    plan None: the consecutive pairing (2p, 2p + 1)."""
    B, H, nq, topk = idx.shape
    valid = vbs > 0
    out = []
    for bh in range(B * H):
        lists = idx[bh // H, bh % H]
        pairs = plan[bh] if plan is not None else [(2 * p, 2 * p + 1 if 2 * p + 1 < nq else -1)
                                                   for p in range((nq + 1) // 2)]
        for a, c in pairs:
            la = lists[a][valid[lists[a]]]
            if c < 0:
                n = len(la)
            else:
                lc = lists[c][valid[lists[c]]]
                dup = len(set(la.tolist())) < len(la) or len(set(lc.tolist())) < len(lc)
                n = len(la) + len(lc) if dup else len(set(la.tolist()) | set(lc.tolist()))
            out.append((n + 1) // 2)
    return np.array(out)


def time_fwd(vsa, args, n=10, warm=3, fn=None):
    """Average forward time (ms) over n calls, CUDA events on the current stream
    (fn: the call, vsa.fwd by default)."""
    fn = fn or vsa.fwd
    for _ in range(warm):
        fn(*args[0], **args[1])
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in ev:
        a.record()
        fn(*args[0], **args[1])
        b.record()
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def run_extras(vsa, dev, cfg, qt, kt, vt, qc, kc, idx, vbs, peak):
    """The forward alone: the headline workload with the consecutive pairing and on
    random selection lists, the proxy-compensated forward, then the other
    configurations."""
    out = torch.empty_like(qt)
    vbs_h = vbs.cpu().numpy()
    res = {}

    def fwd_case(q, k, v, ix, vb, c, plan):
        ms = time_fwd(vsa, ((q, k, v, ix, vb, c.sm_scale), {"out": out if out.shape == q.shape else None,
                                                              "plan": plan}))
        return ms

    # pairing and overlap
    ix_h = idx.cpu().numpy()
    plan = vsa.plan(idx)
    fl = flops(cfg, qt.shape[1])
    cases = {}
    for name, ix_dev, ix_np in (("routed", idx, ix_h),
                                ("random_lists", None, synth.random_topk(11, cfg.B, cfg.H, len(vbs_h), cfg.topk))):
        if ix_dev is None:
            ix_dev = torch.from_numpy(ix_np).to(dev)
        pl = vsa.plan(ix_dev)
        row = {}
        for tag, p in (("planned", pl), ("consecutive", None)):
            ms = fwd_case(qt, kt, vt, ix_dev, vbs, cfg, p)
            spt = steps_per_tile(ix_np, p.cpu().numpy() if p is not None else None, vbs_h)
            row[tag] = {"fwd_ms": ms, "tflops": fl / (ms * 1e-3) / 1e12, "frac": fl / (ms * 1e-3) / 1e12 / peak,
                        "steps_per_tile_mean": float(spt.mean()), "steps_total": int(spt.sum())}
        cases[name] = row
    res["pairing"] = cases

    # proxy compensation: the same call with every omitted cube's mean key and summed
    # value (vc formed by the fused tiling from the raster inputs)
    T, Hh, W = cfg.grid
    g = [synth.bits_to_torch(x).to(dev) for x in synth.grid_qkv(cfg)]
    tiled = [torch.empty_like(qt) for _ in range(3)]
    vc = torch.empty_like(kc)
    vsa.tile_qkv(*g, cfg.grid, vbs, means=False, sums=True, out=tiled + [None, None, vc])
    del g, tiled
    ms_plain = fwd_case(qt, kt, vt, idx, vbs, cfg, plan)
    ms_proxy = time_fwd(vsa, ((qt, kt, vt, idx, vbs, kc, vc, cfg.sm_scale), {"out": out, "plan": plan}),
                        fn=vsa.fwd_proxy)
    res["proxy"] = {"fwd_ms": ms_plain, "fwd_proxy_ms": ms_proxy, "overhead": ms_proxy / ms_plain - 1.0,
                    "proxy_steps_per_tile": (len(vbs_h) + 127) // 128}

    # route formats: the routed lists in ascending order as topk rows, BSR rows and
    # packed bitmaps (the same step lists), and the bitmaps with proxies
    ix_sorted = torch.sort(idx, dim=-1).values.contiguous()
    B, H, nq, topk = ix_sorted.shape
    indptr = (torch.arange(B * H * nq + 1, device=dev, dtype=torch.int32) * topk).contiguous()
    indices = ix_sorted.reshape(-1).contiguous()
    mask = lists_to_bitmask(ix_sorted)
    pl_s = vsa.plan(ix_sorted)
    fmt = {"fwd_lists_ms": fwd_case(qt, kt, vt, ix_sorted, vbs, cfg, pl_s)}
    fmt["fwd_bsr_ms"] = time_fwd(vsa, ((qt, kt, vt, indptr, indices, vbs, cfg.sm_scale), {"out": out, "plan": pl_s}),
                                 fn=vsa.fwd_bsr)
    fmt["fwd_bitmask_ms"] = time_fwd(vsa, ((qt, kt, vt, mask, vbs, cfg.sm_scale), {"out": out, "plan": pl_s}),
                                     fn=vsa.fwd_bitmask)
    fmt["fwd_bitmask_proxy_ms"] = time_fwd(
        vsa, ((qt, kt, vt, mask, vbs, cfg.sm_scale), {"out": out, "plan": pl_s, "kc": kc, "vc": vc}),
        fn=vsa.fwd_bitmask)
    res["route_formats"] = fmt
    del vc, mask, indices

    # short-KV cross-attention: the step's queries over a 512-token text key/value
    # sequence (seeded draws), every key attended
    S_kv = 512
    g = torch.Generator(device="cpu").manual_seed(512)
    kt_txt = torch.randn(cfg.B, S_kv, cfg.H, 128, generator=g).to(torch.bfloat16).to(dev)
    vt_txt = torch.randn(cfg.B, S_kv, cfg.H, 128, generator=g).to(torch.bfloat16).to(dev)
    ms_x = time_fwd(vsa, ((qt, kt_txt, vt_txt, cfg.sm_scale), {"out": out}), fn=vsa.cross_attn)
    fl_x = 4.0 * cfg.B * qt.shape[1] * S_kv * 128 * cfg.H
    res["cross_attn"] = {"S_q": qt.shape[1], "S_kv": S_kv, "tflop_per_call": fl_x / 1e12, "ms": ms_x,
                         "tflops": fl_x / (ms_x * 1e-3) / 1e12, "frac": fl_x / (ms_x * 1e-3) / 1e12 / peak}
    del kt_txt, vt_txt

    # other configurations: forward alone (inputs tiled and routed by the library first)
    cfgs = {}
    for name in ("sweep32", "sweep156", "sweep312", "dense624", "wan720"):
        c = synth.CONFIGS[name]
        if c.grid == cfg.grid and c.B == cfg.B and c.H == cfg.H:
            q_, k_, v_, qc_, kc_, vb_ = qt, kt, vt, qc, kc, vbs
        else:
            T, Hh, W = c.grid
            g = [synth.bits_to_torch(x).to(dev) for x in synth.grid_qkv(c)]
            vb_ = vsa.cube_counts(T, Hh, W).to(dev)
            q_, k_, v_, qc_, kc_ = vsa.tile_qkv(*g, c.grid, vb_)
            del g
        ix = vsa.route_means(qc_, kc_, c.topk)
        pl = vsa.plan(ix)
        o_ = torch.empty_like(q_)
        ms = time_fwd(vsa, ((q_, k_, v_, ix, vb_, c.sm_scale), {"out": o_, "plan": pl}), n=5, warm=2)
        f = flops(c, q_.shape[1])
        spt = steps_per_tile(ix.cpu().numpy(), pl.cpu().numpy(), vb_.cpu().numpy())
        cfgs[name] = {"B": c.B, "H": c.H, "latent_grid": list(c.grid), "S_padded": q_.shape[1], "topk": c.topk,
                      "tflop_per_call": f / 1e12, "fwd_ms": ms, "tflops": f / (ms * 1e-3) / 1e12,
                      "frac": f / (ms * 1e-3) / 1e12 / peak, "steps_per_tile_mean": float(spt.mean())}
        del q_, k_, v_, o_
    res["configs"] = cfgs
    rc, detail = vsa.device_status()
    if rc != 0:
        raise RuntimeError(f"device error {rc}/{detail} in the extra cases")
    return res


# --------------------------------------------------------------------------- oracle timing

class OracleWorkload:
    """The FP64 oracle on the bench workload, for a CPU baseline: inputs for
    two heads of the Wan shape are drawn, tiled and routed once; a 'step' then
    runs the oracle forward on a bounded chunk of query-cube work items."""

    def __init__(self, cfg, seed=0):
        import dataclasses

        import oracle

        self.oracle = oracle
        self.cfg = cfg
        T, Hh, W = cfg.grid
        sub = dataclasses.replace(cfg, H=2)
        q, k, v = synth.grid_qkv(sub)
        self.qt, self.kt, self.vt = (oracle.tile(x, T, Hh, W) for x in (q, k, v))
        self.vbs = oracle.cube_counts(T, Hh, W)
        self.idx = oracle.route(self.qt, self.kt, self.vbs, cfg.topk)
        items = oracle.all_items(1, 2, len(self.vbs))
        self.items = items[np.random.default_rng(seed).permutation(len(items))]
        self.pos = 0
        self.threads = oracle.num_threads()

    def step(self, n):
        chunk = self.items[self.pos: self.pos + n]
        if len(chunk) < n:
            self.pos = 0
            chunk = self.items[:n]
        self.pos += n
        t0 = time.perf_counter()
        self.oracle.fwd_items(self.qt, self.kt, self.vt, self.idx, self.vbs, self.cfg.sm_scale, chunk)
        return time.perf_counter() - t0, len(chunk) * 4.0 * 64 * self.cfg.topk * 64 * 128


def oracle_sample(cfg, seconds=15.0):
    """Time the oracle for about `seconds`: (TFLOP/s, items, seconds, threads)."""
    w = OracleWorkload(cfg)
    n = 2 * w.threads
    t_used, fl, items = 0.0, 0.0, 0
    while t_used < seconds and items < len(w.items):
        dt, f = w.step(n)
        t_used += dt
        fl += f
        items += n
    return fl / t_used / 1e12, items, t_used, w.threads


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=150)  # ~1 s timed: several clock samples
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--oracle-seconds", type=float, default=15.0,
                    help="CPU time for the oracle baseline sample (0 skips it)")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the extra forward cases (pairing, random lists, other configurations)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (a smaller case for ncu captures; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = synth.CONFIGS[WORKLOAD]
    S = 64 * int(np.prod([-(-x // 4) for x in cfg.grid]))

    if args.impl == "reference":
        if rank != 0:
            return
        w = OracleWorkload(cfg)
        n = 2 * w.threads
        for _ in range(args.warmup):
            w.step(n)
        t_used, fl = 0.0, 0.0
        for _ in range(args.steps):
            dt, f = w.step(n)
            t_used += dt
            fl += f
        tf, items, secs, threads = fl / t_used / 1e12, n * args.steps, t_used, w.threads
        value = tf
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": flops(cfg, S) / (value * 1e12) * 1e3,
            "ms_per_step_source": "extrapolated: the workload's FLOPs over the rate of the timed sample",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_block(cfg, S),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{items} query-cube work items of the workload (2 heads drawn), {secs:.1f} s"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    res = run_gpu(args, rank, world, local_rank)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    peak_burst, peak_sus, hbm, peak_kind = read_peaks()
    fl = flops(res["cfg"], res["S"])
    value = world * fl / (res["ms_step"] * 1e-3) / 1e12
    fwd_achieved = fl / (res["fwd_ms"] * 1e-3) / 1e12
    cpu = None
    if world == 1 and args.oracle_seconds > 0:
        tf, items, secs, threads = oracle_sample(res["cfg"], seconds=args.oracle_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{items} query-cube work items of the workload (2 heads drawn), {secs:.1f} s"}
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "fwd_traffic.json")
    if os.path.exists(tpath):
        # the counters are only valid for the kernel source they were taken on
        import hashlib

        t = json.load(open(tpath))
        # the sources of the kernel the default forward runs, as they were when the
        # counters were taken (the traffic of another kernel does not apply)
        srcs = t.get("kernel_sources", {})
        timed = {"video_block_sparse_b200/csrc/fwd_pair.cu", "video_block_sparse_b200/csrc/fwd_pair_common.cuh"}
        if set(srcs) == timed and all(
                os.path.exists(os.path.join(ROOT, f))
                and hashlib.sha256(open(os.path.join(ROOT, f), "rb").read()).hexdigest() == h
                for f, h in srcs.items()):
            traffic = t.get("bytes_per_launch")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_block(res["cfg"], res["S"]),
        "fwd_ms": res["fwd_ms"], "fwd_tflops": fwd_achieved,
        "roofline": {"bound": "tensor", "achieved": fwd_achieved, "peak": peak_burst, "unit": "TFLOP/s",
                     "frac": fwd_achieved / peak_burst, "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 burst (sustained {peak_sus})"},
        "cpu_baseline": cpu,
        "e2e": {"value": world * fl / (res["e2e_ms"] * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                "ms_per_step": res["e2e_ms"],
                "form": "pipelined: step i's inputs in and step i-1's result out on two copy streams "
                        "while the kernels of the step between run; two device buffer sets",
                "serial_value": world * fl / (res["e2e_serial_ms"] * 1e-3) / 1e12,
                "serial_ms_per_step": res["e2e_serial_ms"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    if res["extras"] is not None:
        line["fwd_extra"] = res["extras"]
    print(json.dumps(line))


if __name__ == "__main__":
    main()
