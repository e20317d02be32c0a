"""FP64 CPU oracle for the VSA fine stage -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library in
``video_block_sparse_b200`` never loads it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, double precision); this module
only builds it with gcc and marshals numpy arrays through ctypes.  Every
function here cites the passage of the pages it follows in ``oracle.c``.

Tensors of bf16 values travel as ``numpy.uint16`` arrays holding the bf16 bit
patterns; index tensors are ``numpy.int32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (baseline x86-64 ISA, -O2, OpenMP).

    No -ffast-math: the summation order written in the C source is the one
    that runs."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
             "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.oracle_f64_to_bf16.argtypes = [P, P, I64]
        lib.oracle_bf16_to_f64.argtypes = [P, P, I64]
        lib.oracle_cube_counts.argtypes = [I, I, I, P, P]
        lib.oracle_tile.argtypes = [P, P, I, I, I, I, I, I]
        lib.oracle_untile.argtypes = [P, P, I, I, I, I, I, I]
        lib.oracle_cube_means.argtypes = [P, P, P, I, I, I, I, I]
        lib.oracle_route.argtypes = [P, P, P, P, I, I, I, I, I, I, P]
        lib.oracle_fwd_items.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, P, I64, P, P]
        lib.oracle_fwd_items_ex.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, P, I64, P, P, P]
        lib.oracle_num_threads.argtypes = []
        lib.oracle_plan.argtypes = [P, I, I, I, I, P]
        lib.oracle_cube_sums.argtypes = [P, P, P, I, I, I, I, I]
        lib.oracle_fwd_proxy_items.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, P, I64, P, P]
        lib.oracle_fwd_bsr_items.argtypes = [P, P, P, P, P, P, P, I64, P, I, I, I, I, I, ctypes.c_double, P, I64, P, P,
                                             P]
        lib.oracle_cross_items.argtypes = [P, P, P, I, I, I, I, I, ctypes.c_double, P, I64, P, P, P]
        for name in ("oracle_f64_to_bf16", "oracle_bf16_to_f64", "oracle_cube_counts", "oracle_tile",
                     "oracle_untile", "oracle_cube_means", "oracle_route", "oracle_fwd_items", "oracle_fwd_items_ex",
                     "oracle_num_threads", "oracle_plan", "oracle_cube_sums", "oracle_fwd_proxy_items",
                     "oracle_fwd_bsr_items", "oracle_cross_items"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with status {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round doubles to bf16 (nearest, ties to even) in one step; returns bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(x.shape, dtype=np.uint16)
    _check(_load().oracle_f64_to_bf16(_ptr(x), _ptr(y), x.size), "f64_to_bf16")
    return y


def bf16_to_f64(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    y = np.empty(x.shape, dtype=np.float64)
    _check(_load().oracle_bf16_to_f64(_ptr(x), _ptr(y), x.size), "bf16_to_f64")
    return y


def cube_counts(T: int, Hh: int, W: int) -> np.ndarray:
    """vbs[c]: real tokens in 4x4x4 cube c of a T x Hh x W latent grid."""
    nq = ctypes.c_int(0)
    _check(_load().oracle_cube_counts(T, Hh, W, None, ctypes.byref(nq)), "cube_counts")
    vbs = np.empty(nq.value, dtype=np.int32)
    _check(_load().oracle_cube_counts(T, Hh, W, _ptr(vbs), ctypes.byref(nq)), "cube_counts")
    return vbs


def tile(x_grid: np.ndarray, T: int, Hh: int, W: int) -> np.ndarray:
    """[B, T*Hh*W, H, D] raster -> [B, 64*Nq, H, D] cube-major (pads zero)."""
    B, L, H, D = x_grid.shape
    assert L == T * Hh * W
    nq = len(cube_counts(T, Hh, W))
    x_grid = np.ascontiguousarray(x_grid, dtype=np.uint16)
    out = np.empty((B, 64 * nq, H, D), dtype=np.uint16)
    _check(_load().oracle_tile(_ptr(x_grid), _ptr(out), B, T, Hh, W, H, D), "tile")
    return out


def untile(x_tiled: np.ndarray, T: int, Hh: int, W: int) -> np.ndarray:
    B, S, H, D = x_tiled.shape
    x_tiled = np.ascontiguousarray(x_tiled, dtype=np.uint16)
    out = np.empty((B, T * Hh * W, H, D), dtype=np.uint16)
    _check(_load().oracle_untile(_ptr(x_tiled), _ptr(out), B, T, Hh, W, H, D), "untile")
    return out


def cube_means(x: np.ndarray, vbs: np.ndarray) -> np.ndarray:
    """[B, S, H, D] bf16 -> [B, H, Nq, D] bf16 means over the valid tokens."""
    B, S, H, D = x.shape
    nq = S // 64
    x = np.ascontiguousarray(x, dtype=np.uint16)
    vbs = np.ascontiguousarray(vbs, dtype=np.int32)
    out = np.empty((B, H, nq, D), dtype=np.uint16)
    _check(_load().oracle_cube_means(_ptr(x), _ptr(vbs), _ptr(out), B, S, H, D, nq), "cube_means")
    return out


def cube_sums(x: np.ndarray, vbs: np.ndarray) -> np.ndarray:
    """[B, S, H, D] bf16 -> [B, H, Nq, D] bf16 sums over the valid tokens (the
    summed-V summaries of proxy compensation)."""
    B, S, H, D = x.shape
    nq = S // 64
    x = np.ascontiguousarray(x, dtype=np.uint16)
    vbs = np.ascontiguousarray(vbs, dtype=np.int32)
    out = np.empty((B, H, nq, D), dtype=np.uint16)
    _check(_load().oracle_cube_sums(_ptr(x), _ptr(vbs), _ptr(out), B, S, H, D, nq), "cube_sums")
    return out


def fwd_proxy_items(q, k, v, kc, vc, topk_idx, vbs, sm_scale: float, items: np.ndarray):
    """Proxy-compensated fine forward for the listed (b, h, query cube) items:
    selected cubes exact, every omitted cube with valid tokens through its mean
    key kc and summed value vc, the denominator weighted by the valid counts.
    Returns out [n, 64, D] and lse [n, 64] (natural log), float64."""
    B, S, H, D = q.shape
    nq = S // 64
    topk = topk_idx.shape[-1]
    assert topk_idx.shape == (B, H, nq, topk) and kc.shape == (B, H, nq, D) and vc.shape == kc.shape
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q, k, v, kc, vc)]
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    vbs = np.ascontiguousarray(vbs, dtype=np.int32)
    items = np.ascontiguousarray(items, dtype=np.int32).reshape(-1, 3)
    n = items.shape[0]
    out = np.empty((n, 64, D), dtype=np.float64)
    lse = np.empty((n, 64), dtype=np.float64)
    sigma = float(np.float32(sm_scale))
    _check(_load().oracle_fwd_proxy_items(*(_ptr(a) for a in arrs), _ptr(topk_idx), _ptr(vbs), B, S, H, D, nq, topk,
                                          sigma, _ptr(items), n, _ptr(out), _ptr(lse)), "fwd_proxy_items")
    return out, lse


def route(q: np.ndarray, k: np.ndarray, vbs: np.ndarray, topk: int, want_scores: bool = False):
    """topk_idx [B, H, Nq, topk] int32 from cube-mean q.k scores (and the scores if asked)."""
    B, S, H, D = q.shape
    nq = S // 64
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    vbs = np.ascontiguousarray(vbs, dtype=np.int32)
    idx = np.empty((B, H, nq, topk), dtype=np.int32)
    scores = np.empty((B, H, nq, nq), dtype=np.float64) if want_scores else None
    _check(_load().oracle_route(_ptr(q), _ptr(k), _ptr(vbs), _ptr(idx), B, S, H, D, nq, topk,
                                _ptr(scores) if want_scores else None), "route")
    return (idx, scores) if want_scores else idx


# ---- route formats (TensorRT-LLM PR #7, the embedded FlashInfer PR, "Bitmask format"):
# canonical BSR rows and packed UInt32 exact-block bitmaps, one row per (batch, head,
# query cube); in a bitmap, bit c % 32 of word c / 32 selects cube c (the bit order is a
# reading: least significant first), and bits at c >= Nq in the last word are ignored.

def lists_to_bsr(topk_idx: np.ndarray):
    """[B, H, Nq, topk] lists -> (indptr [B*H*Nq + 1], indices) int32, rows in order."""
    B, H, nq, topk = topk_idx.shape
    indptr = (np.arange(B * H * nq + 1, dtype=np.int64) * topk).astype(np.int32)
    return indptr, np.ascontiguousarray(topk_idx.reshape(-1), dtype=np.int32)


def bitmask_to_bsr(mask: np.ndarray, nq: int):
    """[B, H, Nq, W] 32-bit words -> (indptr, indices): each row's selected cubes in
    ascending order, padding bits ignored."""
    B, H, rows_nq, W = mask.shape
    assert rows_nq == nq and W == (nq + 31) // 32
    words = np.ascontiguousarray(mask).view(np.uint32).reshape(-1, W)
    indptr = [0]
    indices = []
    for row in words:
        sel = [32 * w + bit for w in range(W) for bit in range(32) if (int(row[w]) >> bit) & 1 and 32 * w + bit < nq]
        indices.extend(sel)
        indptr.append(len(indices))
    return np.asarray(indptr, np.int32), np.asarray(indices, np.int32)


def bsr_to_bitmask(indptr: np.ndarray, indices: np.ndarray, B: int, H: int, nq: int) -> np.ndarray:
    """BSR rows -> [B, H, Nq, ceil(Nq/32)] uint32 bitmaps (a cube named twice sets its
    bit once)."""
    W = (nq + 31) // 32
    out = np.zeros((B * H * nq, W), np.uint32)
    for r in range(B * H * nq):
        for c in indices[indptr[r]:indptr[r + 1]]:
            out[r, c // 32] |= np.uint32(1 << (c % 32))
    return out.reshape(B, H, nq, W)


def fwd_bsr_items(q, k, v, indptr, indices, vbs, sm_scale: float, items: np.ndarray, kc=None, vc=None,
                  want_wabs: bool = False):
    """The fine forward with the selections as BSR rows, plain or (kc, vc given)
    proxy-compensated, for the listed (b, h, query cube) items. Returns out [n, 64, D],
    lse [n, 64] (and, plain only, the weighted mean of |v| [n, 64, D]), float64.
    sm_scale is used as the binary32 value a GPU kernel receives."""
    B, S, H, D = q.shape
    nq = S // 64
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q, k, v)]
    kcv = [None, None] if kc is None else [np.ascontiguousarray(a, dtype=np.uint16) for a in (kc, vc)]
    indptr = np.ascontiguousarray(indptr, dtype=np.int32)
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    assert indptr.shape == (B * H * nq + 1,)
    vbs = np.ascontiguousarray(vbs, dtype=np.int32)
    items = np.ascontiguousarray(items, dtype=np.int32).reshape(-1, 3)
    n = items.shape[0]
    out = np.empty((n, 64, D), dtype=np.float64)
    lse = np.empty((n, 64), dtype=np.float64)
    wabs = np.empty((n, 64, D), dtype=np.float64) if want_wabs else None
    idx_buf = indices if indices.size else np.zeros(1, np.int32)
    opt = lambda a: None if a is None else _ptr(a)  # noqa: E731
    _check(_load().oracle_fwd_bsr_items(*(_ptr(a) for a in arrs), opt(kcv[0]), opt(kcv[1]), _ptr(indptr),
                                        _ptr(idx_buf), int(indices.size), _ptr(vbs), B, S, H, D, nq,
                                        float(np.float32(sm_scale)), _ptr(items), n, _ptr(out), _ptr(lse),
                                        opt(wabs)),
           "fwd_bsr_items")
    return (out, lse, wabs) if want_wabs else (out, lse)


def cross_items(q, k, v, sm_scale: float, items: np.ndarray, want_wabs: bool = False):
    """Short-KV cross-attention (every query row over every key of k, v [B, S_kv, H, D],
    one exact softmax) for the listed (b, h, query block of 64 rows) items of q [B, S, H, D].
    Returns out [n, 64, D] and lse [n, 64] (and the weighted mean of |v| [n, 64, D]),
    float64; sm_scale is used as the binary32 value a GPU kernel receives."""
    B, S, H, D = q.shape
    S_kv = k.shape[1]
    assert k.shape == (B, S_kv, H, D) and v.shape == k.shape and S % 64 == 0
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q, k, v)]
    items = np.ascontiguousarray(items, dtype=np.int32).reshape(-1, 3)
    n = items.shape[0]
    out = np.empty((n, 64, D), dtype=np.float64)
    lse = np.empty((n, 64), dtype=np.float64)
    wabs = np.empty((n, 64, D), dtype=np.float64) if want_wabs else None
    _check(_load().oracle_cross_items(*(_ptr(a) for a in arrs), B, S, S_kv, H, D, float(np.float32(sm_scale)),
                                      _ptr(items), n, _ptr(out), _ptr(lse), None if wabs is None else _ptr(wabs)),
           "cross_items")
    return (out, lse, wabs) if want_wabs else (out, lse)


def fwd_items(q, k, v, topk_idx, vbs, sm_scale: float, items: np.ndarray, want_wabs: bool = False):
    """Fine forward for the listed (b, h, query cube) items.

    Returns out [n, 64, D] float64 and lse [n, 64] float64 (natural log), and
    with want_wabs also wabs [n, 64, D] = sum_u softmax(x)_u |v_u[d]|.
    sm_scale is used as the binary32 value a GPU kernel receives."""
    B, S, H, D = q.shape
    nq = S // 64
    topk = topk_idx.shape[-1]
    assert topk_idx.shape == (B, H, nq, topk)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    vbs = np.ascontiguousarray(vbs, dtype=np.int32)
    items = np.ascontiguousarray(items, dtype=np.int32).reshape(-1, 3)
    n = items.shape[0]
    out = np.empty((n, 64, D), dtype=np.float64)
    lse = np.empty((n, 64), dtype=np.float64)
    sigma = float(np.float32(sm_scale))
    wabs = np.empty((n, 64, D), dtype=np.float64) if want_wabs else None
    _check(_load().oracle_fwd_items_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(topk_idx), _ptr(vbs),
                                       B, S, H, D, nq, topk, sigma, _ptr(items), n, _ptr(out), _ptr(lse),
                                       _ptr(wabs) if want_wabs else None),
           "fwd_items")
    return (out, lse, wabs) if want_wabs else (out, lse)


def all_items(B: int, H: int, nq: int) -> np.ndarray:
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(nq), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int32)


def fwd(q, k, v, topk_idx, vbs, sm_scale: float):
    """Full fine forward: out [B, S, H, D] float64, lse [B, H, S] float64."""
    B, S, H, D = q.shape
    nq = S // 64
    items = all_items(B, H, nq)
    o, l = fwd_items(q, k, v, topk_idx, vbs, sm_scale, items)
    out = o.reshape(B, H, nq, 64, D).transpose(0, 2, 3, 1, 4).reshape(B, S, H, D)
    lse = l.reshape(B, H, nq * 64)
    return np.ascontiguousarray(out), np.ascontiguousarray(lse)


def plan(topk_idx: np.ndarray) -> np.ndarray:
    """Pairing of the query cubes of every (b, h) by selection overlap:
    int32 [B*H, ceil(Nq/2), 2] (see oracle.c, "tile plan")."""
    B, H, nq, topk = topk_idx.shape
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    out = np.empty((B * H, (nq + 1) // 2, 2), dtype=np.int32)
    _check(_load().oracle_plan(_ptr(topk_idx), B, H, nq, topk, _ptr(out)), "plan")
    return out
