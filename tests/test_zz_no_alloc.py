"""vsa_coarse_select_noalloc: the coarse stage for callers that cannot
allocate device memory (for example a plugin inside an application that owns
every device allocation, or code that must not call cudaMalloc while work is
in flight).  It must give the same result as vsa_coarse_select, which takes a
caller-allocated workspace, and reject problems larger than its fixed scratch.

Called through the C ABI directly (ctypes on libvsa.so), twice in a row, and
compared with the workspace entry point: the selection must be identical and
the coarse output and logits equal within the coarse-stage tolerances of the
parity tests.  This file sorts last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from video_dit_block_vsa_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from video_dit_block_vsa_b200 import build
    build.build()
    from video_dit_block_vsa_b200 import vsa as mod
    assert mod.vsa_get_status() == 0
    return mod


def _tiled_inputs(vsa, w):
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    bufs = vsa.VsaBuffers(shape, w.topk, want_coarse=True)
    to_dev = lambda b: torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
    vsa.vsa_tile_permute(shape, to_dev(x["q"]), bufs.q_t, bufs.counts)
    vsa.vsa_tile_permute(shape, to_dev(x["k"]), bufs.k_t)
    vsa.vsa_tile_permute(shape, to_dev(x["v"]), bufs.v_t)
    return shape, bufs


def _noalloc_call(vsa, shape, bufs, topk, sel, o_c, logits):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return vsa._lib.vsa_coarse_select_noalloc(
        ctypes.byref(shape), p(bufs.q_t), p(bufs.k_t), p(bufs.v_t), p(bufs.counts), topk,
        p(o_c), p(sel), p(logits), stream)


@pytest.mark.parametrize("name", ["wan1.3b_480p_21x30x52", "tiny_k2"])
def test_noalloc_matches_workspace_entry_point_twice(vsa, name):
    w = wl.WORKLOADS[name]
    shape, bufs = _tiled_inputs(vsa, w)
    C = vsa.vsa_num_cubes(shape)
    B, H, d, k = w.batch, w.heads, w.head_dim, w.topk
    ref_logits = torch.empty(B, H, C, C, dtype=torch.float32, device="cuda")
    vsa.vsa_coarse_select(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, k, bufs.sel,
                          bufs.workspace, o_coarse=bufs.o_c, coarse_logits=ref_logits)
    torch.cuda.synchronize()
    for call in range(2):
        sel = torch.full_like(bufs.sel, -1)
        o_c = torch.full_like(bufs.o_c, float("nan"))
        logits = torch.full_like(ref_logits, float("nan"))
        rc = _noalloc_call(vsa, shape, bufs, k, sel, o_c, logits)
        assert rc == vsa.VSA_OK, vsa.vsa_strerror(rc)
        torch.cuda.synchronize()
        assert vsa.vsa_get_status() == 0
        assert torch.equal(sel, bufs.sel), f"call {call}: selection differs"
        assert torch.allclose(o_c, bufs.o_c, rtol=0, atol=1e-4), f"call {call}: coarse output"
        assert torch.allclose(logits, ref_logits, rtol=0, atol=2e-5), f"call {call}: logits"


def test_noalloc_rejects_problems_beyond_its_scratch(vsa):
    w = wl.WORKLOADS["wan14b_720p_21x45x80_k180"]  # 40 heads: 88 MB of pooled vectors
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    assert 3 * w.batch * w.heads * w.cubes * w.head_dim * 4 > 32 << 20
    dummy = ctypes.c_void_p(0x10000)
    rc = vsa._lib.vsa_coarse_select_noalloc(ctypes.byref(shape), dummy, dummy, dummy, dummy,
                                            w.topk, None, dummy, None, None)
    assert rc == vsa.VSA_ERR_TOO_LARGE
    assert "scratch" in vsa.vsa_strerror(rc)
    assert vsa.vsa_get_status() == 0
