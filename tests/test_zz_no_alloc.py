"""vsa_route_noalloc: routing for callers that cannot allocate device memory
(graph-capture regions that forbid allocation, plugins handed only their
input/output buffers, deployments with every allocation fixed at start-up).
The library supplies the scratch from a fixed array in its own device code.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.  It passes both after the other
tests and run alone in a fresh process (`pytest -m gpu tests/test_zz_no_alloc.py`),
where its first call is the first use of the library on the device and does
the one-time lookup of the array's address."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_block_sparse_b200 import build

    build.build()
    import video_block_sparse_b200 as m

    return m


def _inputs(seed, H):
    """Random cube-major q, k on the Wan 832x480 cube count, with partial cubes."""
    g = np.random.default_rng(seed)
    nq = 624
    q = synth.f32_to_bf16_bits((g.standard_normal((1, 64 * nq, H, 128)) * 3).astype(np.float32))
    k = synth.f32_to_bf16_bits((g.standard_normal((1, 64 * nq, H, 128)) * 3).astype(np.float32))
    vbs = np.full(nq, 64, np.int32)
    vbs[g.choice(nq, 100, replace=False)] = g.integers(0, 64, 100)
    dev = lambda a: synth.bits_to_torch(a).cuda()
    return dev(q), dev(k), torch.from_numpy(vbs).cuda(), nq


def _call_noalloc(vsa, q, k, vbs, out, topk):
    B, S, H, D = q.shape
    lib = vsa.get_lib()
    return lib.vsa_route_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                 ctypes.c_void_p(vbs.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, S, H, D,
                                 S // 64, topk, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_route_matches_workspace_route_twice(vsa):
    topk = 78
    for seed, H in ((21, 8), (22, 40)):  # two calls in a row, different problems
        q, k, vbs, nq = _inputs(seed, H)
        out = torch.full((1, H, nq, topk), -1, dtype=torch.int32, device="cuda")
        assert _call_noalloc(vsa, q, k, vbs, out, topk) == 0
        want = vsa.route(q, k, vbs, topk)
        torch.cuda.synchronize()
        assert vsa.device_status() == (0, 0)
        assert torch.equal(out, want), f"noalloc routing differs from vsa_route (H={H})"


def test_noalloc_route_rejects_problems_beyond_its_array(vsa):
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(q.data_ptr())
    o = ctypes.c_void_p(out.data_ptr())
    # B=2, H=40, Nq=1440 (the Wan 1280x720 CFG shape) needs 59 MB of means > 16 MiB
    rc = vsa.get_lib().vsa_route_noalloc(p, p, o, o, 2, 64 * 1440, 40, 128, 1440, 180, None)
    assert rc == -4  # VSA_ERR_WORKSPACE, nothing launched
