"""Python binding of libvsa, the B200 (sm_100a) library for the fine stage of
Video Sparse Attention.

Argument marshalling only: every step runs in the CUDA kernels behind the C
ABI declared in ``include/vsa.h``.  Tensors are torch CUDA tensors (torch is
used for device memory and streams); each call passes raw pointers, sizes
and the current stream to the library and raises ``VSAError`` on a non-zero
status.  There is no CPU or fallback path: if ``libvsa.so`` is missing or
cannot be loaded, the first call raises ImportError.

Names follow the C ABI: ``fwd`` (vsa_fwd / vsa_fwd_ex / vsa_fwd_planned),
``route``, ``route_means``, ``route_noalloc``, ``plan``, ``tile``,
``tile_qkv``, ``untile``, ``cube_counts``, ``device_status``,
``stall_check``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")

FWD_DEFAULT = 0
FWD_PRECISE_P = 1

_STATUS = {0: "VSA_OK", -1: "VSA_ERR_ARG", -2: "VSA_ERR_NULL", -3: "VSA_ERR_ALIGN", -4: "VSA_ERR_WORKSPACE",
           -5: "VSA_ERR_ARCH", -6: "VSA_ERR_LAUNCH", -7: "VSA_ERR_DEVICE"}

# every symbol include/vsa.h declares
EXPORTS = ("vsa_status_string", "vsa_can_implement", "vsa_fwd", "vsa_fwd_ex", "vsa_fwd_planned", "vsa_fwd_proxy",
           "vsa_fwd_bsr", "vsa_fwd_bitmask", "vsa_cross_attn",
           "vsa_plan_workspace_size", "vsa_plan", "vsa_route_workspace_size", "vsa_route", "vsa_route_means",
           "vsa_route_noalloc", "vsa_cube_counts", "vsa_tile", "vsa_tile_qkv", "vsa_untile", "vsa_stall_check",
           "vsa_device_status")


class VSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libvsa.so not built at {LIB_PATH}; run `python -m video_block_sparse_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.vsa_status_string.argtypes = [I]
    lib.vsa_status_string.restype = ctypes.c_char_p
    lib.vsa_can_implement.argtypes = [I, I]
    lib.vsa_fwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.vsa_fwd_ex.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.vsa_fwd_planned.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.vsa_plan_workspace_size.argtypes = [I, I, I, I]
    lib.vsa_plan_workspace_size.restype = Z
    lib.vsa_plan.argtypes = [P, P, I, I, I, I, P, Z, P]
    lib.vsa_route_workspace_size.argtypes = [I, I, I, I]
    lib.vsa_route_workspace_size.restype = Z
    lib.vsa_route.argtypes = [P, P, P, P, I, I, I, I, I, I, P, Z, P]
    lib.vsa_route_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, I, P]
    lib.vsa_cube_counts.argtypes = [I, I, I, P, P]
    lib.vsa_tile.argtypes = [P, P, I, I, I, I, I, I, P]
    lib.vsa_untile.argtypes = [P, P, I, I, I, I, I, I, P]
    lib.vsa_tile_qkv.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P]
    lib.vsa_fwd_proxy.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.vsa_fwd_bsr.argtypes = [P, P, P, P, P, I, P, P, P, P, P, P, I, I, I, I, I, F, I, P]
    lib.vsa_fwd_bitmask.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, P]
    lib.vsa_cross_attn.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, P]
    lib.vsa_route_means.argtypes = [P, P, P, I, I, I, I, I, P]
    lib.vsa_device_status.argtypes = [P, P]
    lib.vsa_stall_check.argtypes = [P, P]
    for name in ("vsa_can_implement", "vsa_fwd", "vsa_fwd_ex", "vsa_fwd_planned", "vsa_fwd_proxy", "vsa_fwd_bsr",
                 "vsa_fwd_bitmask", "vsa_cross_attn", "vsa_plan", "vsa_route",
                 "vsa_route_means", "vsa_route_noalloc", "vsa_cube_counts", "vsa_tile", "vsa_tile_qkv", "vsa_untile",
                 "vsa_device_status", "vsa_stall_check"):
        getattr(lib, name).restype = I
    return lib


_LIB = None


def get_lib():
    """The loaded libvsa (ctypes); raises ImportError if it is not built."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libvsa takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libvsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise VSAError(rc, what)


def _bf16(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16")


def status_string(status: int) -> str:
    return get_lib().vsa_status_string(status).decode()


def can_implement(D: int, sm_version: int) -> bool:
    return bool(get_lib().vsa_can_implement(D, sm_version))


def cube_counts(T: int, Hh: int, W: int) -> torch.Tensor:
    """Host int32 [Nq] valid-token counts of the 4x4x4 cubes of a T x Hh x W grid."""
    nq = ctypes.c_int(0)
    _check(get_lib().vsa_cube_counts(T, Hh, W, None, ctypes.byref(nq)), "vsa_cube_counts")
    vbs = torch.empty(nq.value, dtype=torch.int32)
    _check(get_lib().vsa_cube_counts(T, Hh, W, ctypes.c_void_p(vbs.data_ptr()), ctypes.byref(nq)), "vsa_cube_counts")
    return vbs


def tile(x_grid: torch.Tensor, grid, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """[B, T*Hh*W, H, D] raster -> [B, 64*Nq, H, D] cube-major (pads zero)."""
    T, Hh, W = grid
    B, L, H, D = x_grid.shape
    _bf16(x_grid, "x_grid")
    nq = ctypes.c_int(0)
    _check(get_lib().vsa_cube_counts(T, Hh, W, None, ctypes.byref(nq)), "vsa_cube_counts")
    if out is None:
        out = torch.empty(B, 64 * nq.value, H, D, dtype=x_grid.dtype, device=x_grid.device)
    if L != T * Hh * W or out.shape != (B, 64 * nq.value, H, D):
        raise ValueError("tile: shape mismatch")
    _check(get_lib().vsa_tile(_ptr(x_grid), _ptr(out), B, T, Hh, W, H, D, _stream(stream)), "vsa_tile")
    return out


def untile(x_tiled: torch.Tensor, grid, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """[B, 64*Nq, H, D] cube-major -> [B, T*Hh*W, H, D] raster."""
    T, Hh, W = grid
    B, S, H, D = x_tiled.shape
    _bf16(x_tiled, "x_tiled")
    if out is None:
        out = torch.empty(B, T * Hh * W, H, D, dtype=x_tiled.dtype, device=x_tiled.device)
    if out.shape != (B, T * Hh * W, H, D):
        raise ValueError("untile: shape mismatch")
    _check(get_lib().vsa_untile(_ptr(x_tiled), _ptr(out), B, T, Hh, W, H, D, _stream(stream)), "vsa_untile")
    return out


def tile_qkv(q_grid: torch.Tensor, k_grid: torch.Tensor, v_grid: torch.Tensor, grid, vbs: torch.Tensor | None = None,
             means: bool = True, out=None, sums: bool = False, stream=None):
    """vsa_tile_qkv: tile q, k, v ([B, T*Hh*W, H, D] raster) in one launch and,
    if `means`, form the cube means of q and k ([B, H, Nq, D]) in the same pass,
    and if `sums` the cube sums of v (the summed values of vsa_fwd_proxy).
    Returns (q_tiled, k_tiled, v_tiled, qc, kc), plus vc with `sums` (None
    for what was not asked).  `out` may hold preallocated tensors in that order."""
    T, Hh, W = grid
    B, L, H, D = q_grid.shape
    for t, n in ((q_grid, "q_grid"), (k_grid, "k_grid"), (v_grid, "v_grid")):
        _bf16(t, n)
        if t.shape != q_grid.shape:
            raise ValueError("tile_qkv: q, k, v shapes differ")
    nq = ctypes.c_int(0)
    _check(get_lib().vsa_cube_counts(T, Hh, W, None, ctypes.byref(nq)), "vsa_cube_counts")
    nq = nq.value
    if out is None:
        dev = q_grid.device
        out = [torch.empty(B, 64 * nq, H, D, dtype=q_grid.dtype, device=dev) for _ in range(3)]
        out += [torch.empty(B, H, nq, D, dtype=q_grid.dtype, device=dev) for _ in range(2)] if means else [None, None]
        out += [torch.empty(B, H, nq, D, dtype=q_grid.dtype, device=dev) if sums else None]
    out = list(out) + [None] * (6 - len(out))
    qt, kt, vt, qc, kc, vc = out
    if sums and (vc is None or vc.shape != (B, H, nq, D) or vbs is None):
        raise ValueError("tile_qkv: sums need vbs and a [B, H, Nq, D] output")
    if L != T * Hh * W or any(x.shape != (B, 64 * nq, H, D) for x in (qt, kt, vt)):
        raise ValueError("tile_qkv: shape mismatch")
    if means and (vbs is None or qc is None or kc is None or qc.shape != (B, H, nq, D) or kc.shape != qc.shape):
        raise ValueError("tile_qkv: means need vbs and [B, H, Nq, D] outputs")
    _check(get_lib().vsa_tile_qkv(_ptr(q_grid), _ptr(k_grid), _ptr(v_grid), _ptr(qt), _ptr(kt), _ptr(vt),
                                  _ptr(vbs) if (means or sums) else None, _ptr(qc) if means else None,
                                  _ptr(kc) if means else None, _ptr(vc) if sums else None, B, T, Hh, W, H, D,
                                  _stream(stream)), "vsa_tile_qkv")
    res = (qt, kt, vt, qc if means else None, kc if means else None)
    return res + (vc,) if sums else res


def route_means(qc: torch.Tensor, kc: torch.Tensor, topk: int, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """vsa_route_means: topk_idx [B, H, Nq, topk] int32 from cube means qc, kc [B, H, Nq, D]."""
    B, H, nq, D = qc.shape
    _bf16(qc, "qc")
    _bf16(kc, "kc")
    if kc.shape != qc.shape:
        raise ValueError("route_means: qc and kc shapes differ")
    if out is None:
        out = torch.empty(B, H, nq, topk, dtype=torch.int32, device=qc.device)
    _check(get_lib().vsa_route_means(_ptr(qc), _ptr(kc), _ptr(out), B, H, D, nq, topk, _stream(stream)),
           "vsa_route_means")
    return out


def route_workspace_size(B: int, H: int, nq: int, D: int = 128) -> int:
    return int(get_lib().vsa_route_workspace_size(B, H, nq, D))


def route(q: torch.Tensor, k: torch.Tensor, vbs: torch.Tensor, topk: int, out: torch.Tensor | None = None,
          workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """topk_idx [B, H, Nq, topk] int32 from cube-mean q.k scores."""
    B, S, H, D = q.shape
    nq = S // 64
    _bf16(q, "q")
    _bf16(k, "k")
    if out is None:
        out = torch.empty(B, H, nq, topk, dtype=torch.int32, device=q.device)
    need = route_workspace_size(B, H, nq, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(get_lib().vsa_route(_ptr(q), _ptr(k), _ptr(vbs), _ptr(out), B, S, H, D, nq, topk, _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream)), "vsa_route")
    return out


def plan_workspace_size(B: int, H: int, nq: int, topk: int) -> int:
    return int(get_lib().vsa_plan_workspace_size(B, H, nq, topk))


def plan(topk_idx: torch.Tensor, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    """Tile plan [B*H, ceil(Nq/2), 2] int32 pairing query cubes by selection overlap (vsa_plan)."""
    B, H, nq, topk = topk_idx.shape
    if topk_idx.dtype != torch.int32:
        raise ValueError("topk_idx must be int32")
    if out is None:
        out = torch.empty(B * H, (nq + 1) // 2, 2, dtype=torch.int32, device=topk_idx.device)
    need = plan_workspace_size(B, H, nq, topk)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=topk_idx.device)
    _check(get_lib().vsa_plan(_ptr(topk_idx), _ptr(out), B, H, nq, topk, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)), "vsa_plan")
    return out


def route_noalloc(q: torch.Tensor, k: torch.Tensor, vbs: torch.Tensor, topk: int, out: torch.Tensor,
                  stream=None) -> torch.Tensor:
    """vsa_route_noalloc: routing with the library's built-in scratch (no
    allocation by the library; `out` must be provided by the caller)."""
    B, S, H, D = q.shape
    _bf16(q, "q")
    _bf16(k, "k")
    _check(get_lib().vsa_route_noalloc(_ptr(q), _ptr(k), _ptr(vbs), _ptr(out), B, S, H, D, S // 64, topk,
                                       _stream(stream)), "vsa_route_noalloc")
    return out


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, topk_idx: torch.Tensor, vbs: torch.Tensor,
        sm_scale: float | None = None, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
        want_lse: bool = False, flags: int = FWD_DEFAULT, plan: torch.Tensor | None = None, stream=None):
    """Fine block-sparse attention forward; returns out (and lse if asked).
    plan: optional int32 [B*H, ceil(Nq/2), 2] tile plan (vsa_fwd_planned)."""
    B, S, H, D = q.shape
    nq = S // 64
    topk = topk_idx.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n)
    if topk_idx.dtype != torch.int32 or vbs.dtype != torch.int32:
        raise ValueError("topk_idx and vbs must be int32")
    if sm_scale is None:
        sm_scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    if plan is None:
        _check(get_lib().vsa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(topk_idx), _ptr(vbs), _ptr(out), _ptr(lse), B, S,
                                    H, D, nq, topk, float(sm_scale), int(flags), _stream(stream)), "vsa_fwd")
    else:
        if plan.dtype != torch.int32 or plan.numel() != B * H * ((nq + 1) // 2) * 2:
            raise ValueError("plan must be int32 [B*H, ceil(Nq/2), 2]")
        _check(get_lib().vsa_fwd_planned(_ptr(q), _ptr(k), _ptr(v), _ptr(topk_idx), _ptr(vbs), _ptr(plan), _ptr(out),
                                         _ptr(lse), B, S, H, D, nq, topk, float(sm_scale), int(flags),
                                         _stream(stream)), "vsa_fwd_planned")
    return (out, lse) if (want_lse or lse is not None) else out


def fwd_proxy(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, topk_idx: torch.Tensor, vbs: torch.Tensor,
              kc: torch.Tensor, vc: torch.Tensor, sm_scale: float | None = None, out: torch.Tensor | None = None,
              lse: torch.Tensor | None = None, want_lse: bool = False, flags: int = FWD_DEFAULT,
              plan: torch.Tensor | None = None, stream=None):
    """vsa_fwd_proxy: the fine forward with every omitted cube represented by its
    mean key kc and summed value vc ([B, H, Nq, D] bf16); returns out (and lse)."""
    B, S, H, D = q.shape
    nq = S // 64
    topk = topk_idx.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (kc, "kc"), (vc, "vc")):
        _bf16(t, n)
    if kc.shape != (B, H, nq, D) or vc.shape != kc.shape:
        raise ValueError("kc and vc must be [B, H, Nq, D]")
    if topk_idx.dtype != torch.int32 or vbs.dtype != torch.int32:
        raise ValueError("topk_idx and vbs must be int32")
    if plan is not None and (plan.dtype != torch.int32 or plan.numel() != B * H * ((nq + 1) // 2) * 2):
        raise ValueError("plan must be int32 [B*H, ceil(Nq/2), 2]")
    if sm_scale is None:
        sm_scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    _check(get_lib().vsa_fwd_proxy(_ptr(q), _ptr(k), _ptr(v), _ptr(topk_idx), _ptr(vbs), _ptr(kc), _ptr(vc),
                                   _ptr(plan), _ptr(out), _ptr(lse), B, S, H, D, nq, topk, float(sm_scale),
                                   int(flags), _stream(stream)), "vsa_fwd_proxy")
    return (out, lse) if (want_lse or lse is not None) else out


def _fwd_common(q, k, v, vbs, kc, vc, plan, sm_scale, out, lse, want_lse):
    B, S, H, D = q.shape
    nq = S // 64
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n)
    if (kc is None) != (vc is None):
        raise ValueError("kc and vc go together")
    if kc is not None:
        for t, n in ((kc, "kc"), (vc, "vc")):
            _bf16(t, n)
        if kc.shape != (B, H, nq, D) or vc.shape != kc.shape:
            raise ValueError("kc and vc must be [B, H, Nq, D]")
    if vbs.dtype != torch.int32:
        raise ValueError("vbs must be int32")
    if plan is not None and (plan.dtype != torch.int32 or plan.numel() != B * H * ((nq + 1) // 2) * 2):
        raise ValueError("plan must be int32 [B*H, ceil(Nq/2), 2]")
    if sm_scale is None:
        sm_scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    return B, S, H, D, nq, float(sm_scale), out, lse


def fwd_bsr(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_indptr: torch.Tensor,
            block_indices: torch.Tensor, vbs: torch.Tensor, sm_scale: float | None = None, kc=None, vc=None,
            out: torch.Tensor | None = None, lse: torch.Tensor | None = None, want_lse: bool = False,
            flags: int = FWD_DEFAULT, plan: torch.Tensor | None = None, stream=None):
    """vsa_fwd_bsr: the fine forward with the selections as BSR rows (block_indptr
    [B*H*Nq + 1], block_indices [nnz], int32); kc, vc: optional proxies. Returns out
    (and lse)."""
    B, S, H, D, nq, sc, out, lse = _fwd_common(q, k, v, vbs, kc, vc, plan, sm_scale, out, lse, want_lse)
    if block_indptr.dtype != torch.int32 or block_indices.dtype != torch.int32:
        raise ValueError("block_indptr and block_indices must be int32")
    if block_indptr.numel() != B * H * nq + 1:
        raise ValueError("block_indptr must hold B*H*Nq + 1 entries")
    nnz = block_indices.numel()
    _check(get_lib().vsa_fwd_bsr(_ptr(q), _ptr(k), _ptr(v), _ptr(block_indptr), _ptr(block_indices) if nnz else None,
                                 nnz, _ptr(vbs), _ptr(kc), _ptr(vc), _ptr(plan), _ptr(out), _ptr(lse), B, S, H, D,
                                 nq, sc, int(flags), _stream(stream)), "vsa_fwd_bsr")
    return (out, lse) if (want_lse or lse is not None) else out


def fwd_bitmask(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: torch.Tensor, vbs: torch.Tensor,
                sm_scale: float | None = None, kc=None, vc=None, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, want_lse: bool = False, flags: int = FWD_DEFAULT,
                plan: torch.Tensor | None = None, stream=None):
    """vsa_fwd_bitmask: the fine forward with the selections as packed bitmaps
    (mask [B, H, Nq, ceil(Nq/32)], 32-bit words, bit c % 32 of word c / 32 selects
    cube c; int32 or uint32 storage); kc, vc: optional proxies. Returns out (and lse)."""
    B, S, H, D, nq, sc, out, lse = _fwd_common(q, k, v, vbs, kc, vc, plan, sm_scale, out, lse, want_lse)
    if mask.dtype not in (torch.int32, torch.uint32) or tuple(mask.shape) != (B, H, nq, (nq + 31) // 32):
        raise ValueError("mask must be 32-bit [B, H, Nq, ceil(Nq/32)]")
    _check(get_lib().vsa_fwd_bitmask(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), _ptr(vbs), _ptr(kc), _ptr(vc),
                                     _ptr(plan), _ptr(out), _ptr(lse), B, S, H, D, nq, sc, int(flags),
                                     _stream(stream)), "vsa_fwd_bitmask")
    return (out, lse) if (want_lse or lse is not None) else out


def cross_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, sm_scale: float | None = None,
               out: torch.Tensor | None = None, lse: torch.Tensor | None = None, want_lse: bool = False,
               flags: int = FWD_DEFAULT, stream=None):
    """vsa_cross_attn: every query row of q [B, S, H, D] (S a multiple of 64) over every
    key of the short k, v [B, S_kv, H, D]; returns out (and lse [B, H, S])."""
    B, S, H, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n)
    S_kv = k.shape[1]
    if k.shape != (B, S_kv, H, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, S_kv, H, D]")
    if sm_scale is None:
        sm_scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    _check(get_lib().vsa_cross_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, S_kv, H, D,
                                    float(sm_scale), int(flags), _stream(stream)), "vsa_cross_attn")
    return (out, lse) if (want_lse or lse is not None) else out


def stall_check(stream=None) -> int:
    """Run the bounded-wait diagnostic (a wait that nothing completes must run out,
    latch error 3 and return); returns its result bits (bit 0: the wait succeeded,
    bit 1: the abort flag was raised) after the stream has finished."""
    s = stream if stream is not None else torch.cuda.current_stream()
    result = torch.zeros(1, dtype=torch.int32, device="cuda")
    if stream is not None:
        s.wait_stream(torch.cuda.current_stream())  # the zeroed result is ready on s
    rc = get_lib().vsa_stall_check(_ptr(result), _stream(s))
    if rc != 0:
        raise RuntimeError(f"vsa_stall_check: {status_string(rc)}")
    s.synchronize()
    return int(result.item())


def device_status(stream=None) -> tuple[int, int]:
    """Synchronise the stream and read (and clear) the device error word."""
    detail = ctypes.c_int(0)
    rc = get_lib().vsa_device_status(_stream(stream), ctypes.byref(detail))
    return rc, detail.value
