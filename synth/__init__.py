"""Seeded synthetic inputs for the VSA fine stage.

This module serves both the CUDA path (tests, bench) and the FP64 oracle.  It
holds none of the method's arithmetic: no tiling, no cube counts, no means,
no routing, no softmax.  It only draws random numbers and converts them to
bf16 bit patterns (``numpy.uint16``) with torch's round-to-nearest-even cast.

The captured Wan2.2 tensors that the dataset card "wan2.2_production_values"
scores on are not available, so these draws stand in for them with the
captures' shapes and dtypes (dataset card, sections "Shapes" and "Load"):

* ``tiny``     -- B=1, H=2, D=128, latent grid 5x6x7, topk=2;
                  q, k, v ~ N(0,1) * U[0.5, 4] per (tensor, head).
* ``wan480``   -- Wan2.2 T2V-A14B 832x480/81f: B=1, grid 21x30x52, H=40, D=128,
                  topk=78; q, k ~ N(0,1) * U[1, 8] per (tensor, head) with 4
                  outlier channels per head, shared by q and k, multiplied by 20;
                  v ~ N(0,1).
* ``adversarial`` -- the wan480 shape and draws, plus 3 heads whose q, k are
                  Student-t(nu=2) clipped to +-1e3, plus one head whose
                  selection is forced to include 20 cubes whose valid counts
                  are overridden to values in 1..8 (at least one equals 1).
* ``wan720``   -- Wan2.2 1280x720/81f CFG pair: B=2, grid 21x45x80, topk=180,
                  draws as wan480 (each batch entry independent).
* ``sweep``    -- the wan480 grid with topk in {32, 78, 156, 312}; topk=624 uses
                  the unpadded 24x32x52 grid (every cube full), i.e. dense.

Every (tensor, batch, head) slice has its own stream,
``PCG64(SeedSequence([seed, tensor_id, b, h]))``, so slices can be drawn in
parallel and any slice can be regenerated alone.  Values are drawn as
float32 standard normals, scaled in float32, then cast to bf16.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np
import torch

D_HEAD = 128

# tensor ids of the per-slice streams
_Q, _K, _V, _PARAMS, _OVERRIDE = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    grid: tuple  # (T, Hh, W) latent grid
    topk: int
    kind: str  # "tiny" | "wan"
    adversarial: bool = False
    seed: int = 0

    @property
    def tokens(self) -> int:
        T, Hh, W = self.grid
        return T * Hh * W

    @property
    def sm_scale(self) -> float:
        return 1.0 / float(np.sqrt(D_HEAD))


CONFIGS = {
    "tiny": Config("tiny", B=1, H=2, grid=(5, 6, 7), topk=2, kind="tiny"),
    "wan480": Config("wan480", B=1, H=40, grid=(21, 30, 52), topk=78, kind="wan"),
    "adversarial": Config("adversarial", B=1, H=40, grid=(21, 30, 52), topk=78, kind="wan", adversarial=True),
    "wan720": Config("wan720", B=2, H=40, grid=(21, 45, 80), topk=180, kind="wan"),
    "sweep32": Config("sweep32", B=1, H=40, grid=(21, 30, 52), topk=32, kind="wan"),
    "sweep156": Config("sweep156", B=1, H=40, grid=(21, 30, 52), topk=156, kind="wan"),
    "sweep312": Config("sweep312", B=1, H=40, grid=(21, 30, 52), topk=312, kind="wan"),
    "dense624": Config("dense624", B=1, H=40, grid=(24, 32, 52), topk=624, kind="wan"),
}

ADV_T_HEADS = (5, 17, 29)  # heads with Student-t q, k in the adversarial config
ADV_FORCED_HEAD = 33  # head whose selection includes the overridden cubes
ADV_N_FORCED = 20


def _rng(seed: int, tensor: int, b: int = 0, h: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, b, h])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), torch's nearest-even cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_torch(x: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 CPU tensor (no copy)."""
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)


def torch_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass
class HeadParams:
    scale: np.ndarray  # [3, B, H] float32 per (tensor, batch, head)
    outlier_ch: np.ndarray  # [B, H, 4] int, shared by q and k of a head (wan kinds)
    t_heads: tuple  # heads drawn from Student-t


def head_params(cfg: Config) -> HeadParams:
    """Per-(tensor, head) scales and the shared outlier channels."""
    scale = np.ones((3, cfg.B, cfg.H), dtype=np.float32)
    ch = np.zeros((cfg.B, cfg.H, 4), dtype=np.int64)
    for b in range(cfg.B):
        g = _rng(cfg.seed, _PARAMS, b)
        if cfg.kind == "tiny":
            scale[:, b, :] = g.uniform(0.5, 4.0, size=(3, cfg.H)).astype(np.float32)
        else:
            scale[:2, b, :] = g.uniform(1.0, 8.0, size=(2, cfg.H)).astype(np.float32)
            for h in range(cfg.H):
                ch[b, h] = g.choice(D_HEAD, size=4, replace=False)
    return HeadParams(scale, ch, ADV_T_HEADS if cfg.adversarial else ())


def _draw_slice(cfg: Config, hp: HeadParams, tensor: int, b: int, h: int, L: int) -> np.ndarray:
    g = _rng(cfg.seed, tensor, b, h)
    if tensor in (_Q, _K) and h in hp.t_heads:
        x = np.clip(g.standard_t(2.0, size=(L, D_HEAD)), -1e3, 1e3).astype(np.float32)
    else:
        x = g.standard_normal((L, D_HEAD), dtype=np.float32)
        x *= hp.scale[tensor, b, h]
        if cfg.kind == "wan" and tensor in (_Q, _K):
            x[:, hp.outlier_ch[b, h]] *= np.float32(20.0)
    return f32_to_bf16_bits(x)


def grid_qkv(cfg: Config, threads: int | None = None):
    """q, k, v in raster (grid) layout, [B, T*Hh*W, H, D] bf16 bit patterns."""
    hp = head_params(cfg)
    L = cfg.tokens
    out = [np.empty((cfg.B, L, cfg.H, D_HEAD), dtype=np.uint16) for _ in range(3)]
    jobs = [(t, b, h) for t in (_Q, _K, _V) for b in range(cfg.B) for h in range(cfg.H)]

    def run(job):
        t, b, h = job
        out[t][b, :, h, :] = _draw_slice(cfg, hp, t, b, h, L)

    with ThreadPoolExecutor(max_workers=threads or min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(run, jobs))
    return out[0], out[1], out[2]


def tiled_random(cfg: Config, S: int, tensor: int, fill_pads: bool = True) -> np.ndarray:
    """A [B, S, H, D] tensor drawn directly in tiled layout (every slot random).

    Used where pads must hold finite garbage that a kernel has to ignore."""
    hp = head_params(cfg)
    x = np.empty((cfg.B, S, cfg.H, D_HEAD), dtype=np.uint16)
    for b in range(cfg.B):
        for h in range(cfg.H):
            x[b, :, h, :] = _draw_slice(cfg, hp, tensor, b, h, S)
    return x


@dataclasses.dataclass
class Override:
    head: int
    cubes: np.ndarray  # [20] distinct cube ids
    counts: np.ndarray  # [20] valid counts in 1..8, counts[0] == 1


def adversarial_override(cfg: Config, nq: int) -> Override:
    """The forced cubes and their overridden valid counts (random draws only)."""
    g = _rng(cfg.seed, _OVERRIDE)
    cubes = g.choice(nq, size=ADV_N_FORCED, replace=False).astype(np.int32)
    counts = g.integers(1, 9, size=ADV_N_FORCED).astype(np.int32)
    counts[0] = 1
    return Override(ADV_FORCED_HEAD, cubes, counts)


def random_topk(seed: int, B: int, H: int, nq: int, topk: int, distinct: bool = True) -> np.ndarray:
    """A random selection list [B, H, nq, topk] int32 (for edge-case tests)."""
    g = _rng(seed, 7)
    if distinct:
        keys = g.random((B, H, nq, nq))
        return np.argsort(keys, axis=-1)[..., :topk].astype(np.int32)
    return g.integers(0, nq, size=(B, H, nq, topk)).astype(np.int32)
