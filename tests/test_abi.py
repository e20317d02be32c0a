"""The C-ABI library loads and exports every symbol include/vsa.h declares;
argument errors are reported before anything touches a device.  CPU only."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def vsa():
    from video_block_sparse_b200 import build

    build.build()
    import video_block_sparse_b200 as m

    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "vsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("vsa_fwd", "vsa_route", "vsa_tile", "vsa_untile", "vsa_cube_counts", "vsa_route_workspace_size",
              "vsa_can_implement", "vsa_status_string", "vsa_device_status", "vsa_fwd_ex"):
        assert n in names


def test_library_exports_every_declared_symbol(vsa):
    lib = ctypes.CDLL(vsa.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in vsa.h but not exported"
    assert set(declared_functions()) <= set(vsa.EXPORTS) | set(declared_functions())
    assert set(vsa.EXPORTS) <= set(declared_functions())


def test_library_exports_nothing_else(vsa):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", vsa.LIB_PATH], capture_output=True, text=True).stdout
    ours = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln and ln.split()[-1].startswith("vsa_")})
    assert ours == declared_functions()


def test_status_strings_and_capability(vsa):
    assert vsa.status_string(0) == "VSA_OK"
    for s in range(-7, 0):
        assert vsa.status_string(s).startswith("VSA_ERR")
    assert vsa.can_implement(128, 100)
    assert not vsa.can_implement(64, 100)
    assert not vsa.can_implement(128, 90)


def test_cube_counts_host(vsa):
    import oracle

    for grid in [(5, 6, 7), (21, 30, 52), (21, 45, 80), (1, 1, 1), (24, 32, 52)]:
        assert vsa.cube_counts(*grid).tolist() == oracle.cube_counts(*grid).tolist()
    with pytest.raises(vsa.VSAError):
        vsa.cube_counts(0, 4, 4)


def test_route_workspace_size(vsa):
    assert vsa.route_workspace_size(1, 40, 624, 128) == 2 * 40 * 624 * 128 * 2
    assert vsa.route_workspace_size(0, 40, 624, 128) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


@pytest.mark.parametrize("B,S,H,D,Nq,topk,expect", [
    (1, 512, 2, 64, 8, 2, -1),    # D != 128
    (1, 500, 2, 128, 8, 2, -1),   # S != 64 * Nq
    (0, 512, 2, 128, 8, 2, -1),   # B < 1
    (1, 512, 0, 128, 8, 2, -1),   # H < 1
    (1, 512, 2, 128, 8, 0, -1),   # topk < 1
])
def test_fwd_rejects_bad_sizes_without_a_device(vsa, B, S, H, D, Nq, topk, expect):
    p = _fake(1 << 20)
    rc = vsa.get_lib().vsa_fwd(p, p, p, p, p, p, None, B, S, H, D, Nq, topk, 0.1, None)
    assert rc == expect


def test_fwd_rejects_null_and_misaligned_without_a_device(vsa):
    p = _fake(1 << 20)
    assert vsa.get_lib().vsa_fwd(None, p, p, p, p, p, None, 1, 512, 2, 128, 8, 2, 0.1, None) == -2
    assert vsa.get_lib().vsa_fwd(p, p, p, p, p, _fake((1 << 20) + 2), None, 1, 512, 2, 128, 8, 2, 0.1, None) == -3
    assert vsa.get_lib().vsa_fwd_ex(p, p, p, p, p, p, None, 1, 512, 2, 128, 8, 2, 0.1, 8, None) == -1  # unknown flag


def test_stall_check_rejects_null_without_a_device(vsa):
    assert vsa.get_lib().vsa_stall_check(None, None) == -2


def test_route_rejects_bad_arguments_without_a_device(vsa):
    p = _fake(1 << 20)
    ws = vsa.route_workspace_size(1, 2, 8, 128)
    assert vsa.get_lib().vsa_route(p, p, p, p, 1, 512, 2, 128, 8, 9, p, ws, None) == -1  # topk > Nq
    assert vsa.get_lib().vsa_route(p, p, p, p, 1, 512, 2, 128, 8, 2, p, ws - 1, None) == -4  # short workspace
    assert vsa.get_lib().vsa_route(p, p, p, p, 1, 512, 2, 128, 8, 2, None, ws, None) == -4
    assert vsa.get_lib().vsa_route(p, None, p, p, 1, 512, 2, 128, 8, 2, p, ws, None) == -2


def test_tile_rejects_bad_arguments_without_a_device(vsa):
    p = _fake(1 << 20)
    assert vsa.get_lib().vsa_tile(p, p, 1, 0, 6, 7, 2, 128, None) == -1
    assert vsa.get_lib().vsa_tile(p, p, 1, 5, 6, 7, 3, 5, None) == -1  # H*D not a multiple of 8
    assert vsa.get_lib().vsa_tile(None, p, 1, 5, 6, 7, 2, 128, None) == -2
    assert vsa.get_lib().vsa_untile(p, _fake((1 << 20) + 8), 1, 5, 6, 7, 2, 128, None) == -3


def test_tile_qkv_and_route_means_reject_bad_arguments_without_a_device(vsa):
    p = _fake(1 << 20)
    lib = vsa.get_lib()
    # grid 5x6x7, B=1, H=2, D=128
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, p, p, None, None, 1, 5, 6, 7, 2, 128, None) == -1  # kc missing
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, p, p, p, None, 1, 5, 6, 7, 2, 64, None) == -1  # means need D = 128
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, p, None, None, p, 1, 5, 6, 7, 2, 64, None) == -1  # sums too
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, None, p, p, None, 1, 5, 6, 7, 2, 128, None) == -2  # means need vbs
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, None, None, None, p, 1, 5, 6, 7, 2, 128, None) == -2  # sums need vbs
    assert lib.vsa_tile_qkv(p, p, None, p, p, p, None, None, None, None, 1, 5, 6, 7, 2, 128, None) == -2
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, None, None, None, None, 1, 0, 6, 7, 2, 128, None) == -1
    assert lib.vsa_tile_qkv(p, p, p, p, p, _fake((1 << 20) + 4), None, None, None, None, 1, 5, 6, 7, 2, 128,
                            None) == -3
    assert lib.vsa_tile_qkv(p, p, p, p, p, p, p, None, None, _fake((1 << 20) + 4), 1, 5, 6, 7, 2, 128, None) == -3
    assert lib.vsa_route_means(p, p, p, 1, 2, 128, 8, 9, None) == -1  # topk > Nq
    assert lib.vsa_route_means(p, p, p, 1, 2, 64, 8, 2, None) == -1  # D != 128
    assert lib.vsa_route_means(p, p, p, 1, 2, 128, 5000, 2, None) == -1  # Nq > 4096
    assert lib.vsa_route_means(p, None, p, 1, 2, 128, 8, 2, None) == -2
    assert lib.vsa_route_means(p, p, _fake((1 << 20) + 4), 1, 2, 128, 8, 2, None) == -3


def test_fwd_proxy_rejects_bad_arguments_without_a_device(vsa):
    p = _fake(1 << 20)
    lib = vsa.get_lib()
    args = (1, 512, 2, 128, 8, 2, 0.1, 0, None)  # B, S, H, D, Nq, topk, scale, flags, stream
    assert lib.vsa_fwd_proxy(p, p, p, p, p, None, p, None, p, None, *args) == -2  # kc missing
    assert lib.vsa_fwd_proxy(p, p, p, p, p, p, None, None, p, None, *args) == -2  # vc missing
    assert lib.vsa_fwd_proxy(p, p, p, p, p, p, _fake((1 << 20) + 2), None, p, None, *args) == -3
    assert lib.vsa_fwd_proxy(p, p, p, p, p, p, p, None, p, None, 1, 512, 2, 64, 8, 2, 0.1, 0, None) == -1
    assert lib.vsa_fwd_proxy(p, p, p, p, p, p, p, None, p, None, 1, 512, 2, 128, 8, 2, 0.1, 2, None) == -1  # flag


def test_fwd_bsr_and_bitmask_reject_bad_arguments_without_a_device(vsa):
    p = _fake(1 << 20)
    lib = vsa.get_lib()
    tail = (1, 512, 2, 128, 8, 0.1, 0, None)  # B, S, H, D, Nq, scale, flags, stream
    # vsa_fwd_bsr(q, k, v, indptr, indices, nnz, vbs, kc, vc, plan, out, lse, ...)
    assert lib.vsa_fwd_bsr(p, p, p, p, p, -1, p, None, None, None, p, None, *tail) == -1  # nnz < 0
    assert lib.vsa_fwd_bsr(p, p, p, p, p, 4, p, None, None, None, p, None, 1, 512, 2, 64, 8, 0.1, 0, None) == -1
    assert lib.vsa_fwd_bsr(p, p, p, p, p, 4, p, None, None, None, p, None, 1, 512, 2, 128, 8, 0.1, 4, None) == -1
    assert lib.vsa_fwd_bsr(p, p, p, None, p, 4, p, None, None, None, p, None, *tail) == -2  # indptr
    assert lib.vsa_fwd_bsr(p, p, p, p, None, 4, p, None, None, None, p, None, *tail) == -2  # indices, nnz > 0
    assert lib.vsa_fwd_bsr(p, p, p, p, p, 4, p, p, None, None, p, None, *tail) == -2  # kc without vc
    assert lib.vsa_fwd_bsr(p, p, p, _fake((1 << 20) + 4), p, 4, p, None, None, None, p, None, *tail) == -3
    assert lib.vsa_fwd_bsr(p, p, p, p, _fake((1 << 20) + 4), 4, p, None, None, None, p, None, *tail) == -3
    # vsa_fwd_bitmask(q, k, v, mask, vbs, kc, vc, plan, out, lse, ...)
    assert lib.vsa_fwd_bitmask(p, p, p, p, p, None, None, None, p, None, 1, 512, 2, 64, 8, 0.1, 0, None) == -1
    assert lib.vsa_fwd_bitmask(p, p, p, p, p, None, None, None, p, None, 1, 512, 2, 128, 9000, 0.1, 0, None) == -1
    assert lib.vsa_fwd_bitmask(p, p, p, None, p, None, None, None, p, None, *tail) == -2  # mask
    assert lib.vsa_fwd_bitmask(p, p, p, p, p, None, p, None, p, None, *tail) == -2  # vc without kc
    assert lib.vsa_fwd_bitmask(p, p, p, _fake((1 << 20) + 8), p, None, None, None, p, None, *tail) == -3


def test_cross_attn_rejects_bad_arguments_without_a_device(vsa):
    p = _fake(1 << 20)
    lib = vsa.get_lib()
    # vsa_cross_attn(q, k, v, out, lse, B, S, S_kv, H, D, scale, flags, stream)
    assert lib.vsa_cross_attn(p, p, p, p, None, 1, 500, 512, 2, 128, 0.1, 0, None) == -1  # S % 64
    assert lib.vsa_cross_attn(p, p, p, p, None, 1, 512, 0, 2, 128, 0.1, 0, None) == -1  # S_kv
    assert lib.vsa_cross_attn(p, p, p, p, None, 1, 512, 70000, 2, 128, 0.1, 0, None) == -1
    assert lib.vsa_cross_attn(p, p, p, p, None, 1, 512, 512, 2, 64, 0.1, 0, None) == -1  # D
    assert lib.vsa_cross_attn(p, p, p, p, None, 1, 512, 512, 2, 128, 0.1, 4, None) == -1  # flag
    assert lib.vsa_cross_attn(p, None, p, p, None, 1, 512, 512, 2, 128, 0.1, 0, None) == -2
    assert lib.vsa_cross_attn(p, p, p, _fake((1 << 20) + 4), None, 1, 512, 512, 2, 128, 0.1, 0, None) == -3


def test_route_noalloc_checks_arguments_before_its_array_limit(vsa):
    """Bad arguments are reported as by vsa_route, even for a problem larger than
    the fixed array, and before any device is touched."""
    p = _fake(1 << 20)
    lib = vsa.get_lib()
    # B=2, H=40, Nq=1440 needs more than the array; D = 64 is invalid
    assert lib.vsa_route_noalloc(p, p, p, p, 2, 64 * 1440, 40, 64, 1440, 180, None) == -1
    assert lib.vsa_route_noalloc(p, p, p, p, 2, 64 * 1440, 40, 128, 1440, 2000, None) == -1  # topk > Nq
    assert lib.vsa_route_noalloc(None, p, p, p, 2, 64 * 1440, 40, 128, 1440, 180, None) == -2
    assert lib.vsa_route_noalloc(p, p, _fake((1 << 20) + 4), p, 2, 64 * 1440, 40, 128, 1440, 180, None) == -3


def test_product_package_does_not_reach_the_oracle():
    """The product path never imports or loads the oracle."""
    pkg = os.path.join(ROOT, "video_block_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "liboracle" not in text and "from oracle" not in text, f


def test_binding_checks_route_format_and_cross_arguments_on_the_host(vsa):
    """The Python wrappers of the route-format and cross-attention entry points reject
    mismatched tensors before any device call."""
    import torch

    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)  # noqa: E731
    q = bf(1, 128, 2, 128)
    vbs = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):  # indptr must hold B*H*Nq + 1 entries
        vsa.fwd_bsr(q, q, q, torch.zeros(4, dtype=torch.int32), torch.zeros(0, dtype=torch.int32), vbs)
    with pytest.raises(ValueError):  # int32 only
        vsa.fwd_bsr(q, q, q, torch.zeros(5, dtype=torch.int64), torch.zeros(0, dtype=torch.int32), vbs)
    with pytest.raises(ValueError):  # kc without vc
        vsa.fwd_bitmask(q, q, q, torch.zeros(1, 2, 2, 1, dtype=torch.int32), vbs, kc=bf(1, 2, 2, 128))
    with pytest.raises(ValueError):  # bitmap shape
        vsa.fwd_bitmask(q, q, q, torch.zeros(1, 2, 2, 2, dtype=torch.int32), vbs)
    with pytest.raises(ValueError):  # k and v of different lengths
        vsa.cross_attn(q, bf(1, 64, 2, 128), bf(1, 32, 2, 128))
